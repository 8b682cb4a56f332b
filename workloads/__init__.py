"""Seeded synthetic inputs for the NVFP4 W4A4 path.

This module holds only input generation: counter-based random numbers,
distribution shaping and BF16 rounding of the inputs, plus the MoE routing
that decides group sizes.  It contains none of the quantization or GEMM
arithmetic, so the CPU oracle and the CUDA path can both be fed from it
without sharing any of the method.

Random numbers: SplitMix64 (Steele, Lea, Flood, "Fast splittable
pseudorandom number generators", OOPSLA 2014) evaluated at counters
1, 2, 3, ... of a per-stream seed, written here from its published
definition.  Uniforms take the top 53 bits, normals use Box-Muller, Laplace
uses the inverse CDF.  All values are rounded FP32 -> BF16 to nearest even.

Workloads (sizes from the LLM shapes the pages discuss):
  tiny     A [16,256] N(0,1) with 1% of entries x20; W [64,256] N(0,0.02)
  quant    activations [8192,4096] Laplace(0,1) with 0.1% of entries
           replaced by +-U[50,200]; weights [14336,4096] N(0,0.02)
  prefill  A [4096,4096] N(0,1); W [14336,4096] N(0,0.02)
  decode   M in {1,8,32,64}, K=5120, N=25600; A N(0,1) 1% x20; W N(0,0.02)
  moe      4096 tokens, hidden 2048, 128 experts of [1536,2048] N(0,0.02);
           router logits N(0,1) -> softmax -> top-8 -> rows grouped by expert
"""
from __future__ import annotations

import os

import numpy as np

_GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_seed(seed: int, stream: int) -> np.uint64:
    """Derive an independent stream seed from (seed, stream)."""
    with np.errstate(over="ignore"):
        z = np.array([np.uint64(seed) * _GAMMA + np.uint64(stream) + np.uint64(1)], np.uint64)
        return _mix(z)[0]


def splitmix64(seed: int, stream: int, n: int, start: int = 0) -> np.ndarray:
    """n 64-bit outputs of SplitMix64 at counters start+1 .. start+n."""
    s = stream_seed(seed, stream)
    with np.errstate(over="ignore"):
        ctr = np.arange(start + 1, start + n + 1, dtype=np.uint64)
        return _mix(s + ctr * _GAMMA)


_CHUNK = 1 << 20
_POOL = None


def _pool():
    global _POOL
    if _POOL is None:
        from concurrent.futures import ThreadPoolExecutor
        _POOL = ThreadPoolExecutor(max_workers=min(32, os.cpu_count() or 1))
    return _POOL


def _chunked(n: int, fill) -> np.ndarray:
    """out[i] for i in [0, n), computed chunk by chunk (counter-based, so the
    result does not depend on the chunking) on a thread pool."""
    out = np.empty(n, np.float64)
    starts = range(0, n, _CHUNK)
    list(_pool().map(lambda s0: fill(out, s0, min(n, s0 + _CHUNK)), starts))
    return out


def _uniform_at(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    z = splitmix64(seed, stream, count, start=start)
    return ((z >> np.uint64(11)).astype(np.float64) + 0.5) * (1.0 / 9007199254740992.0)


def uniform(seed: int, stream: int, n: int) -> np.ndarray:
    """Uniform doubles in the open interval (0, 1): u_i from counter i + 1."""
    def fill(out, a, b):
        out[a:b] = _uniform_at(seed, stream, a, b - a)
    return _chunked(n, fill)


def normal(seed: int, stream: int, n: int, std: float = 1.0) -> np.ndarray:
    """Box-Muller on consecutive uniform pairs (u_2p, u_2p+1): outputs 2p and
    2p+1 are R cos(theta) and R sin(theta)."""
    def fill(out, a, b):                     # a is even (chunk boundaries are)
        cnt = b - a
        pairs = (cnt + 1) // 2
        u = _uniform_at(seed, stream, a, 2 * pairs)
        r = std * np.sqrt(-2.0 * np.log(u[0::2]))
        t = 2.0 * np.pi * u[1::2]
        v = np.empty(2 * pairs, np.float64)
        v[0::2] = r * np.cos(t)
        v[1::2] = r * np.sin(t)
        out[a:b] = v[:cnt]
    return _chunked(n, fill)


def laplace(seed: int, stream: int, n: int, b: float = 1.0) -> np.ndarray:
    def fill(out, a, e):
        u = _uniform_at(seed, stream, a, e - a) - 0.5
        out[a:e] = -b * np.sign(u) * np.log1p(-2.0 * np.abs(u))
    return _chunked(n, fill)


def distinct_positions(seed: int, stream: int, n: int, count: int) -> np.ndarray:
    """`count` distinct positions in [0, n), in draw order."""
    if count <= 0:
        return np.zeros(0, np.int64)
    out = np.zeros(0, np.int64)
    start = 0
    while out.size < count:
        draw = 2 * (count - out.size) + 16
        z = splitmix64(seed, stream, draw, start=start)
        start += draw
        cand = (z % np.uint64(n)).astype(np.int64)
        merged = np.concatenate([out, cand])
        _, first = np.unique(merged, return_index=True)
        out = merged[np.sort(first)]
    return out[:count]


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round to BF16 (nearest even) and return the uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).reshape(-1).view(np.uint32)
    out = np.empty(u.size, np.uint16)

    def conv(a):
        b = min(u.size, a + _CHUNK)
        v = u[a:b]
        lsb = (v >> np.uint32(16)) & np.uint32(1)
        out[a:b] = ((v + np.uint32(0x7FFF) + lsb) >> np.uint32(16)).astype(np.uint16)
    list(_pool().map(conv, range(0, u.size, _CHUNK)))
    return out.reshape(np.shape(x))


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


# ---- tensors of the workloads ---------------------------------------------------

def gaussian_bf16(shape, seed: int, stream: int, std: float = 1.0,
                  outlier_frac: float = 0.0, outlier_mult: float = 20.0) -> np.ndarray:
    """N(0, std^2); floor(outlier_frac * n) distinct entries multiplied by
    outlier_mult.  Returns BF16 bits of the given shape."""
    n = int(np.prod(shape))
    x = normal(seed, stream, n, std).astype(np.float32)
    cnt = int(np.floor(outlier_frac * n))
    if cnt:
        pos = distinct_positions(seed, stream + 1000, n, cnt)
        x[pos] *= np.float32(outlier_mult)
    return to_bf16_bits(x).reshape(shape)


def laplace_outliers_bf16(shape, seed: int, stream: int, outlier_frac: float = 0.001,
                          lo: float = 50.0, hi: float = 200.0) -> np.ndarray:
    """Laplace(0,1) with floor(outlier_frac * n) distinct entries replaced by
    +-U[lo, hi] (random sign)."""
    n = int(np.prod(shape))
    x = laplace(seed, stream, n).astype(np.float32)
    cnt = int(np.floor(outlier_frac * n))
    if cnt:
        pos = distinct_positions(seed, stream + 1000, n, cnt)
        u = uniform(seed, stream + 2000, 2 * cnt)
        mag = lo + (hi - lo) * u[:cnt]
        sgn = np.where(u[cnt:] < 0.5, -1.0, 1.0)
        x[pos] = (sgn * mag).astype(np.float32)
    return to_bf16_bits(x).reshape(shape)


def tiny(seed: int = 0):
    a = gaussian_bf16((16, 256), seed, 1, 1.0, outlier_frac=0.01)
    w = gaussian_bf16((64, 256), seed, 2, 0.02)
    return a, w


def quant_act(seed: int = 0, rows: int = 8192, k: int = 4096):
    return laplace_outliers_bf16((rows, k), seed, 3)


def quant_weight(seed: int = 0, n: int = 14336, k: int = 4096):
    return gaussian_bf16((n, k), seed, 4, 0.02)


def prefill(seed: int = 0, m: int = 4096, n: int = 14336, k: int = 4096):
    a = gaussian_bf16((m, k), seed, 5, 1.0)
    w = gaussian_bf16((n, k), seed, 6, 0.02)
    return a, w


def decode_activations(m: int, seed: int = 0, k: int = 5120):
    return gaussian_bf16((m, k), seed, 7 + m, 1.0, outlier_frac=0.01)


def decode_weights(seed: int = 0, n: int = 25600, k: int = 5120):
    return gaussian_bf16((n, k), seed, 6000, 0.02)


def decode(m: int, seed: int = 0, n: int = 25600, k: int = 5120):
    return decode_activations(m, seed, k), decode_weights(seed, n, k)


def moe_routing(seed: int = 0, tokens: int = 4096, experts: int = 128, top_k: int = 8):
    """Seeded router: logits N(0,1) [tokens, experts] -> softmax -> top-k
    (ties to the lower expert index).  Returns (offsets [E+1] int32,
    token_of_row [tokens*top_k] int64) with rows grouped by expert and, inside
    an expert, in ascending token order.  Router weights are not applied."""
    logits = normal(seed, 8, tokens * experts).reshape(tokens, experts)
    p = np.exp(logits - logits.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    # stable sort on -p keeps the lower index first among equal probabilities
    order = np.argsort(-p, axis=1, kind="stable")[:, :top_k]
    tok = np.repeat(np.arange(tokens, dtype=np.int64), top_k)
    exp = order.reshape(-1)
    idx = np.lexsort((tok, exp))          # primary: expert, secondary: token
    counts = np.bincount(exp, minlength=experts)
    offsets = np.zeros(experts + 1, np.int32)
    offsets[1:] = np.cumsum(counts)
    return offsets, tok[idx]


def moe(seed: int = 0, tokens: int = 4096, hidden: int = 2048, experts: int = 128,
        inter: int = 1536, top_k: int = 8, with_weights: bool = True):
    """Returns (a_grouped [tokens*top_k, hidden] bf16 bits, offsets [E+1],
    w [E, inter, hidden] bf16 bits or None)."""
    offsets, token_of_row = moe_routing(seed, tokens, experts, top_k)
    x = gaussian_bf16((tokens, hidden), seed, 9, 1.0)
    a = np.ascontiguousarray(x[token_of_row])
    w = None
    if with_weights:
        w = gaussian_bf16((experts, inter, hidden), seed, 10, 0.02)
    return a, offsets, w


WORKLOADS = {
    "tiny": "A [16,256] N(0,1) 1% x20; W [64,256] N(0,0.02)",
    "quant": "activations [8192,4096] Laplace(0,1) + 0.1% +-U[50,200]; weights [14336,4096] N(0,0.02)",
    "prefill": "A [4096,4096] N(0,1) quantized per call x W nvfp4 [14336,4096] -> C bf16 [4096,14336]",
    "decode": "M in {1,8,32,64}, K=5120, N=25600; A N(0,1) 1% x20; W N(0,0.02)",
    "moe": "4096 tokens top-8 of 128 experts [1536,2048] -> C bf16 [32768,1536]",
}
