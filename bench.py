#!/usr/bin/env python
"""Benchmark of the NVFP4 W4A4 hot path on B200.

One step = one pass of the whole path over one batch: dynamic NVFP4
quantization of the BF16 activations (tensor amax, block scales, E2M1 codes)
followed by the block-scaled FP4 x FP4 GEMM against pre-quantized NVFP4
weights, BF16 output.  Default workload (the prefill-shaped GEMM):
A bf16 [4096, 4096] quantized per call, W nvfp4 [14336, 4096] (2D-quantized
once, outside the timed region), C bf16 [4096, 14336].

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload prefill|quant|decode|moe] [--decode-m M]

Prints one JSON line.  `value` is whole-job throughput (TFLOP/s of 2*M*N*K
per step, summed over ranks, divided by the slowest rank's time).  The steps
rotate over enough independent buffer sets that no step finds its inputs in
L2.  Timing: the K steps run as CUDA-graph replays on one stream between one
pair of CUDA events; per-kernel durations come from a copy of the same graph
with an event between consecutive kernels.  N > 1 runs N independent
replicas (the path needs no exchange between GPUs), one process per GPU.

With the default workload on one GPU the line also carries every other
configuration of the path, each with its own roofline, clocks and CPU
baseline: `quant_c2` (the activation quantizer on [8192,4096] Laplace with
outliers, plus its pre-scaled and MXFP4 forms), `weight_quant` (16x16 blocks
on [14336,4096]), `decode` (m in {1, 8, 32, 64}: step, quantizer, GEMM with
the weight-stream roofline, and the same GEMM as W4A16) and `moe` (grouped
quantizer and grouped GEMM, FP4 and HBM fractions, MMA padding).  Per-kernel
loops run at least 200 launches whatever --steps is.  `warmup` echoes the
requested count; `warmup_calls_run` counts the untimed calls actually made
(eager first calls and graph replays).

--impl reference times the CPU oracle (plain C, binary64 GEMM) on a bounded
sample of the same workload: rank 0 only.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FP4_PER_BF16 = 4.0            # dense FP4 / dense BF16 nominal ratio (9 / 2.25 PFLOP/s)
METRIC = "W4A4 NVFP4 GEMM TFLOPS (% dense FP4 peak); quantize GB/s (% HBM peak)"


def quant_bytes(rows: int, k: int, groups: int = 1) -> int:
    """Algorithmic bytes of one quantizer call: read BF16 once, write packed
    codes and one E4M3 scale per 16 values, and the FP32 global scale(s)."""
    n = rows * k
    return 2 * n + n // 2 + n // 16 + 4 * groups


def mx_quant_bytes(rows: int, k: int) -> int:
    """Algorithmic bytes of one MXFP4 quantizer call: read BF16 once, write
    packed codes and one E8M0 scale per 32 values."""
    n = rows * k
    return 2 * n + n // 2 + n // 32


_T_START = time.perf_counter()


def progress(what: str) -> None:
    """One line on stderr per section, with the seconds since start."""
    print(f"[bench +{time.perf_counter() - _T_START:6.1f} s] {what}", file=sys.stderr, flush=True)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except (OSError, KeyError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_TFLOPS,
                "bf16_tflops_sustained": FALLBACK_BF16_TFLOPS, "source": "fallback"}


# ---- clocks sampled during the timed region (NVML, read only) -------------------------

_REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
            0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
            0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, torch_device_index: int):
        self.samples = []
        self._stop = threading.Event()
        self._thr = None
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            uuid = str(torch.cuda.get_device_properties(torch_device_index).uuid)
            h = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                hi = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(hi)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    h = hi
            if h is None:
                h = pynvml.nvmlDeviceGetHandleByIndex(torch_device_index)
            self.h = h
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # noqa: BLE001 - clocks are reported as unavailable
            self.err = str(e)

    def _run(self):
        nv = self.nv
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                except AttributeError:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)
                self.samples.append((time.perf_counter(), mhz, rs))
            except Exception:  # noqa: BLE001
                pass
            time.sleep(0.002)

    def start(self):
        if self.ok:
            self._stop.clear()
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
            time.sleep(0.02)

    def stop(self):
        if self._thr:
            self._stop.set()
            self._thr.join()

    def summary(self, t0: float, t1: float):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": f"NVML unavailable: {self.err}"}
        inside = [s for s in self.samples if t0 <= s[0] <= t1]
        if not inside:   # very short timed region: nearest samples after it
            inside = [s for s in self.samples if s[0] >= t0][:5] or self.samples[-5:]
        mask = 0
        for s in inside:
            mask |= int(s[2])
        reasons = [name for bit, name in _REASONS.items() if mask & bit and bit != 0x1]
        return {"sm_mhz": statistics.median(s[1] for s in inside), "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(inside)}


# ---- distributed plumbing (replicas; the only collective is the timing reduction) -----

def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def reduce_max(value: float, world: int, device) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ---- workloads ----------------------------------------------------------------------------
#
# Each workload holds R independent buffer sets (activations, their NVFP4
# form, weights, output) and step i works on set i % R.  R is chosen so that
# between two uses of one set the other sets move at least twice the L2 size:
# every step finds its inputs in HBM, none left in L2 by an earlier step.

L2_BYTES = 128 << 20          # upper bound of the 126 MB L2


MAX_SETS = 16
# Idle time before each timed loop, so that every loop starts from the same
# power state: under a dense FP4 GEMM the board reaches its power cap after
# about 0.1 s and the SM clock steps down from 1965 MHz to about 1800 MHz.
REST_S = 0.5


def rotation_count(*set_bytes: int) -> int:
    """Sets needed so that, for each of the given per-set footprints (a whole
    step, or one kernel timed alone), the other sets move twice the L2 size;
    at most MAX_SETS (only a tiny decode activation would want more)."""
    return min(MAX_SETS, max(max(2, 1 + -(-2 * L2_BYTES // max(1, b))) for b in set_bytes))


def nbytes(*ts) -> int:
    return sum(t.numel() * t.element_size() for t in ts)


def to_device(torch, bits, dev):
    return torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)


def clone_q(nv, t):
    return nv.NVFP4Tensor(t.codes.clone(), t.scales.clone(), t.global_scale.clone(), t.rows, t.k, t.offsets)


class Prefill:
    name = "prefill"

    def __init__(self, nv, torch, dev, m=4096, n=14336, k=4096):
        import workloads as W
        self.m, self.n, self.k = m, n, k
        self._build(nv, torch, dev, *W.prefill(0, m, n, k))

    def _build(self, nv, torch, dev, a, w):
        m, n, k = self.m, self.n, self.k
        self.nv = nv
        self.a_host = a
        a0 = to_device(torch, a, dev)
        wdev = to_device(torch, w, dev)
        w0 = nv.quantize_weight_2d(wdev)              # offline: pre-quantized weights
        del wdev
        q0 = nv.quantize_act(a0)
        c0 = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        self.set_bytes = nbytes(a0, q0.codes, q0.scales, w0.codes, w0.scales, c0)
        self.kernel_bytes = (nbytes(a0, q0.codes, q0.scales), nbytes(q0.codes, q0.scales, w0.codes, w0.scales, c0))
        self.R = R = rotation_count(self.set_bytes, *self.kernel_bytes)
        self.a = [a0] + [a0.clone() for _ in range(R - 1)]
        self.qa = [q0] + [clone_q(nv, q0) for _ in range(R - 1)]
        self.w = [w0] + [clone_q(nv, w0) for _ in range(R - 1)]
        self.c = [c0] + [torch.empty_like(c0) for _ in range(R - 1)]
        self.flops = 2.0 * m * n * k
        self.qbytes = quant_bytes(m, k)
        self.wbytes = nbytes(w0.codes, w0.scales)
        self.launches_per_step = 2                    # one-launch quantizer, GEMM

    def quantize(self, i):
        j = i % self.R
        self.nv.quantize_act(self.a[j], out=self.qa[j])

    def gemm(self, i):
        j = i % self.R
        self.nv.gemm(self.qa[j], self.w[j], out=self.c[j])

    kernels = (quantize, gemm)

    def step(self, i):
        self.quantize(i)
        self.gemm(i)

    def result(self, i):
        return self.c[i % self.R]

    def next_layer_steps(self, nv, torch):
        """The next layer's dynamic quantization of this GEMM's output C, two
        ways, over the same rotating sets: the GEMM then the one-launch
        quantizer (amax and quantize passes over C), or the GEMM emitting C's
        global scale then the quantize pass alone."""
        qc = [nv.quantize_act(c) for c in self.c]
        gs = [torch.empty(1, dtype=torch.float32, device=c.device) for c in self.c]

        def one_phase(i):
            j = i % self.R
            self.nv.gemm(self.qa[j], self.w[j], out=self.c[j])
            self.nv.quantize_act(self.c[j], out=qc[j])

        def two_phase(i):
            j = i % self.R
            self.nv.gemm_emit_scale(self.qa[j], self.w[j], out=self.c[j], out_scale=gs[j])
            self.nv.quantize_act_scaled(self.c[j], gs[j], out=qc[j])
        return one_phase, two_phase

    def mx_steps(self, nv, torch, w_host):
        """The same workload in MXFP4: the activations quantized per call, the
        weights quantized once (R rotating copies of each)."""
        dev = self.a[0].device
        wdev = to_device(torch, w_host, dev)
        w0 = nv.quantize_mx(wdev)
        del wdev
        mw = [w0] + [nv.MXFP4Tensor(w0.codes.clone(), w0.scales.clone(), w0.rows, w0.k) for _ in range(self.R - 1)]
        ma = [nv.quantize_mx(a) for a in self.a]

        def quantize(i):
            j = i % self.R
            self.nv.quantize_mx(self.a[j], out=ma[j])

        def gemm(i):
            j = i % self.R
            self.nv.gemm_mx(ma[j], mw[j], out=self.c[j])

        def step(i):
            quantize(i)
            gemm(i)
        return quantize, gemm, step

    def gemm_label(self):
        if self.m <= 64:
            return "gemm_kernel (tcgen05 mxf4nvf4; 64 token rows x 192 weight rows per tile)"
        if self.m > 128:
            return "gemm_pair_kernel (tcgen05 mxf4nvf4, cta_group::2; 256 x 256 tiles)"
        return "gemm_kernel (tcgen05 mxf4nvf4; 128 x 192 tiles)"

    def config(self):
        return {"workload": f"prefill W4A4: A bf16 [{self.m},{self.k}] dynamically quantized (1D blocks) x "
                            f"W nvfp4 [{self.n},{self.k}] (2D blocks, pre-quantized) -> C bf16 [{self.m},{self.n}]",
                "m": self.m, "n": self.n, "k": self.k}


class Decode(Prefill):
    name = "decode"

    def __init__(self, nv, torch, dev, m=64, w_host=None):
        import workloads as W
        self.m, self.n, self.k = m, 25600, 5120
        w = w_host if w_host is not None else W.decode_weights()
        self._build(nv, torch, dev, W.decode_activations(m), w)
        self.abytes = quant_bytes(m, self.k) - 2 * m * self.k   # A codes, scales and g, read by the GEMM
        self.cbytes = 2 * m * self.n
        self.launches_per_step = 3                    # nvfp4_quantize_gemm: amax, quantize, GEMM

    def step(self, i):
        """One decode step through the one-call entry point: the two-kernel
        quantizer, then the GEMM as its programmatic dependent, streaming its
        first weight stages while the activations are quantized."""
        j = i % self.R
        self.nv.quantize_gemm(self.a[j], self.w[j], out=self.c[j], qa=self.qa[j])

    def separate_step(self, i):
        self.quantize(i)
        self.gemm(i)

    def prepare_two_phase(self):
        """Each buffer set's global scale, as the GEMM that produced the
        activations would have emitted it (nvfp4_gemm_emit_scale); taken
        before timing."""
        self.g_given = [self.nv.quantize_act(a).global_scale.clone() for a in self.a]

    def two_phase_step(self, i):
        """The step when the producing layer has already emitted x's global
        scale: the given-scale quantize pass, then the GEMM; no amax pass.
        The codes and scales equal the dynamic step's."""
        j = i % self.R
        self.nv.quantize_act_scaled(self.a[j], self.g_given[j], out=self.qa[j])
        self.gemm(i)

    def step_bytes(self):
        """Algorithmic HBM bytes of one step: x, the weights (codes, scales),
        A's codes and scales written and read once, C."""
        return 2 * self.m * self.k + self.wbytes + 2 * self.abytes + self.cbytes

    def config(self):
        return {"workload": f"decode W4A4: A bf16 [{self.m},{self.k}] quantized per call x W nvfp4 "
                            f"[{self.n},{self.k}] -> C bf16 [{self.m},{self.n}]", "m": self.m, "n": self.n, "k": self.k}


class Quant:
    name = "quant"

    def __init__(self, nv, torch, dev):
        import workloads as W
        self.nv = nv
        self.rows, self.k = 8192, 4096
        x = W.quant_act(0)
        self.a_host = x
        a0 = to_device(torch, x, dev)
        q0 = nv.quantize_act(a0)
        self.set_bytes = nbytes(a0, q0.codes, q0.scales)
        self.kernel_bytes = (self.set_bytes,)
        self.R = R = rotation_count(self.set_bytes)
        self.a = [a0] + [a0.clone() for _ in range(R - 1)]
        self.qa = [q0] + [clone_q(nv, q0) for _ in range(R - 1)]
        self.qbytes = quant_bytes(self.rows, self.k)
        self.flops = 0.0
        self.launches_per_step = 1                    # one cooperative launch
        # the weight variant (16 x 16 blocks), reported beside the step
        self.wn = 14336
        w0 = to_device(torch, W.quant_weight(0, self.wn, self.k), dev)
        qw0 = nv.quantize_weight_2d(w0)
        self.RW = RW = rotation_count(nbytes(w0, qw0.codes, qw0.scales))
        self.w = [w0] + [w0.clone() for _ in range(RW - 1)]
        self.qw = [qw0] + [clone_q(nv, qw0) for _ in range(RW - 1)]
        self.wqbytes = quant_bytes(self.wn, self.k)

    def quantize(self, i):
        j = i % self.R
        self.nv.quantize_act(self.a[j], out=self.qa[j])

    kernels = (quantize,)
    step = quantize

    def quantize_weight(self, i):
        j = i % self.RW
        self.nv.quantize_weight_2d(self.w[j], out=self.qw[j])

    def quantize_smooth(self, i):
        """The same activations with per-channel pre-scaling folded in."""
        j = i % self.R
        if not hasattr(self, "smooth"):
            import torch
            g = np.random.default_rng(1)
            self.smooth = torch.from_numpy(np.exp2(g.uniform(-3.0, 3.0, self.k)).astype(np.float32)).to(self.a[0].device)
        self.nv.quantize_act_smooth(self.a[j], self.smooth, out=self.qa[j])

    def quantize_mx(self, i):
        """The same activations quantized to MXFP4 (one pass, E8M0 per 32)."""
        j = i % self.R
        if not hasattr(self, "mx"):
            self.mx = [self.nv.quantize_mx(a) for a in self.a]
        self.nv.quantize_mx(self.a[j], out=self.mx[j])

    def result(self, i):
        return self.qa[i % self.R].codes

    def config(self):
        return {"workload": "activation quantizer: bf16 [8192,4096] Laplace(0,1) + 0.1% +-U[50,200] -> nvfp4 "
                            "(1D 16-element blocks)", "rows": self.rows, "k": self.k}


class Moe:
    name = "moe"

    def __init__(self, nv, torch, dev):
        import workloads as W
        self.nv = nv
        a, off, w = W.moe(0)
        E, N, K = w.shape
        self.E, self.n, self.k, self.rows = E, N, K, a.shape[0]
        self.a_host, self.off_host, self.w_host = a, off, w
        a0 = to_device(torch, a, dev)
        self.off = torch.from_numpy(off).to(dev)
        wdev = to_device(torch, w.reshape(E * N, K), dev)
        tw = [nv.quantize_weight_2d(wdev[e * N:(e + 1) * N]) for e in range(E)]
        del wdev
        b0 = (torch.stack([t.codes for t in tw]), torch.cat([t.scales for t in tw]),
              torch.cat([t.global_scale for t in tw]))
        del tw
        q0 = nv.quantize_act(a0, self.off)
        c0 = torch.empty((self.rows, N), dtype=torch.bfloat16, device=dev)
        self.set_bytes = nbytes(a0, q0.codes, q0.scales, b0[0], b0[1], c0)
        self.kernel_bytes = (nbytes(a0, q0.codes, q0.scales), nbytes(q0.codes, q0.scales, b0[0], b0[1], c0))
        self.R = R = rotation_count(self.set_bytes, *self.kernel_bytes)
        self.a = [a0] + [a0.clone() for _ in range(R - 1)]
        self.qa = [q0] + [clone_q(nv, q0) for _ in range(R - 1)]
        self.b = [b0] + [tuple(t.clone() for t in b0) for _ in range(R - 1)]
        self.c = [c0] + [torch.empty_like(c0) for _ in range(R - 1)]
        self.flops = 2.0 * self.rows * N * K
        self.qbytes = quant_bytes(self.rows, K, E)
        # the grouped GEMM reads every expert's weights and A's codes and scales once, writes C
        self.gemm_bytes = nbytes(b0[0], b0[1]) + quant_bytes(self.rows, K, E) - 2 * self.rows * K + nbytes(c0)
        self.launches_per_step = 2                    # one-launch grouped quantizer, grouped GEMM

    def quantize(self, i):
        j = i % self.R
        self.nv.quantize_act(self.a[j], self.off, out=self.qa[j])

    def gemm(self, i):
        j = i % self.R
        self.nv.grouped_gemm(self.qa[j], *self.b[j], self.n, out=self.c[j])

    kernels = (quantize, gemm)

    def step(self, i):
        self.quantize(i)
        self.gemm(i)

    def result(self, i):
        return self.c[i % self.R]

    def gemm_label(self):
        if self.n % 256 == 0:
            return ("moe_swap_kernel (tcgen05 mxf4nvf4, cta_group::2; 256 weight rows x up to 256 tokens "
                    "per tile)")
        return "gemm_pair_kernel<grouped> (tcgen05 mxf4nvf4, cta_group::2; 256 x 256 tiles per expert)"

    def padding(self):
        """Token columns of tensor-core work per expert, as the grouped GEMM
        tiles them, against the rows that hold tokens.  With n a multiple of
        256 the swapped kernel runs: tokens on the MMA's N side in tiles of
        256, the last part rounded up to a multiple of 32 (riding on the tile
        before it when it holds at most 64 tokens)."""
        sizes = np.diff(self.off.cpu().numpy().astype(np.int64))
        if self.n % 256 == 0:
            full = sizes // 256
            last = sizes - 256 * full
            padded = int(np.sum(256 * full + (-(-last // 32)) * 32))
            tiling = "tokens on N: 256-token tiles, the last part rounded up to 32"
        else:
            tile = 256 if sizes.sum() >= 192 * len(sizes) else 128
            padded = int(np.sum(-(-sizes // tile) * tile))
            tiling = f"tokens on the MMA's M side in {tile}-row tiles"
        return {"token_rows": int(sizes.sum()), "mma_rows": padded, "tiling": tiling,
                "padding_frac": 1.0 - sizes.sum() / padded if padded else 0.0}

    def config(self):
        return {"workload": f"MoE grouped W4A4: {self.rows // 8} tokens top-8 of {self.E} experts, A bf16 "
                            f"[{self.rows},{self.k}] quantized per expert group x W nvfp4 {self.E}x[{self.n},{self.k}] "
                            f"-> C bf16 [{self.rows},{self.n}]", "rows": self.rows, "n": self.n, "k": self.k,
                "experts": self.E}


# ---- timing helpers -------------------------------------------------------------------------
#
# The timed work runs as CUDA graphs captured on one side stream: a graph of
# R consecutive steps (one per buffer set) replayed, plus a graph of the
# remaining K mod R steps, so exactly K steps run between one pair of events.

def capture(torch, stream, calls):
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for f in calls:
            f()
    return g


class StepGraphs:
    """Exactly `n` calls fn(0), fn(1), ... (fn(i) works on buffer set i % R)
    as replays of captured graphs on `stream`."""

    def __init__(self, torch, stream, fn, R, n):
        self.torch, self.stream, self.n = torch, stream, n
        with torch.cuda.stream(stream):
            for i in range(R):                        # first calls on this stream: workspaces, attributes
                fn(i)
        stream.synchronize()
        self.full = capture(torch, stream, [lambda i=i: fn(i) for i in range(R)])
        self.reps, rem = divmod(n, R)
        self.part = capture(torch, stream, [lambda i=i: fn(i) for i in range(rem)]) if rem else None
        self.R, self.rem = R, rem
        self.setup_calls = R

    def warm(self, at_least: int) -> int:
        """Untimed replays (at least `at_least` calls, every graph once);
        returns the calls run, the first eager ones included."""
        done = self.setup_calls
        with self.torch.cuda.stream(self.stream):
            while True:
                self.full.replay()
                done += self.R
                if done >= at_least:
                    break
            if self.part is not None:
                self.part.replay()
                done += self.rem
        self.stream.synchronize()
        return done

    def run(self):
        """The n calls between two events; returns (start, end) events."""
        torch = self.torch
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.stream):
            e0.record()
            for _ in range(self.reps):
                self.full.replay()
            if self.part is not None:
                self.part.replay()
            e1.record()
        return e0, e1


def graph_seconds(torch, stream, fn, R, n):
    """Average seconds per call of fn over n graph-replayed calls (after one
    untimed pass over every graph)."""
    g = StepGraphs(torch, stream, fn, R, n)
    g.warm(0)
    e0, e1 = g.run()
    stream.synchronize()
    return e0.elapsed_time(e1) * 1e-3 / n


def timed_loop(torch, stream, fn, R, n, sampler):
    """(average seconds per call, clocks during the loop) of n graph-replayed
    calls of fn, after an untimed pass over every graph and a rest."""
    g = StepGraphs(torch, stream, fn, R, n)
    g.warm(0)
    time.sleep(REST_S)
    t0 = time.perf_counter()
    e0, e1 = g.run()
    stream.synchronize()
    t1 = time.perf_counter()
    return e0.elapsed_time(e1) * 1e-3 / n, sampler.summary(t0, t1)


# Launches per per-kernel timing loop, whatever --steps is.
KERNEL_ITERS = 200
NOMINAL_FP4_TFLOPS = 9000.0   # B200 dense FP4, datasheet (context beside the measured-derived peak)


def cpu_baseline_prefill(wl, max_seconds=12.0):
    """The oracle as it stands on the host cores: dynamic quantization of the
    whole A plus the binary64 GEMM of a sample of rows (W reconstructed once,
    outside the timing)."""
    import oracle as O
    import workloads as W
    a_host = wl.a_host
    w_bits = W.prefill(0, wl.m, wl.n, wl.k)[1] if wl.name == "prefill" else W.decode(wl.m)[1]
    wc, wsf, gw = O.quantize_2d(w_bits)
    wh = O.dequantize(wc, wsf, gw)
    t = time.perf_counter()
    ac, asf, ga = O.quantize_1d(a_host)
    ah = O.dequantize(ac, asf, ga)
    tq = time.perf_counter() - t
    t = time.perf_counter()
    O.gemm_f64_rows(ah, wh, np.arange(min(4, wl.m)))
    t_row = (time.perf_counter() - t) / min(4, wl.m)
    rows = int(max(1, min(wl.m, (max_seconds - tq) / max(t_row, 1e-6))))
    sel = np.linspace(0, wl.m - 1, rows).astype(np.int64)
    t = time.perf_counter()
    ac, asf, ga = O.quantize_1d(a_host)
    ah = O.dequantize(ac, asf, ga)
    O.gemm_f64_rows(ah, wh, sel)
    dt = time.perf_counter() - t
    flops = 2.0 * rows * wl.n * wl.k
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": O.num_threads(), "kind": "oracle",
            "sample": f"dynamic quantization of the whole A [{wl.m},{wl.k}] + binary64 GEMM of {rows} of "
                      f"{wl.m} rows against W [{wl.n},{wl.k}] ({dt:.1f} s)"}


def cpu_baseline_weight_quant(w_bits):
    import oracle as O
    t = time.perf_counter()
    O.quantize_2d(w_bits)
    dt = time.perf_counter() - t
    rows, k = w_bits.shape
    return {"value": quant_bytes(rows, k) / dt / 1e9, "unit": "GB/s", "cores": O.num_threads(), "kind": "oracle",
            "sample": f"one full 16x16-block quantization of [{rows},{k}] ({dt:.2f} s)"}


def cpu_baseline_decode(a_bits, wh, n, k, max_rows=8):
    """The oracle on one decode step: dynamic quantization of A, then the
    binary64 GEMM of up to max_rows of its rows against the reconstructed W
    (W reconstructed once, outside the timing)."""
    import oracle as O
    m = a_bits.shape[0]
    rows = min(m, max_rows)
    sel = np.linspace(0, m - 1, rows).astype(np.int64)
    t = time.perf_counter()
    ac, asf, ga = O.quantize_1d(a_bits)
    O.gemm_f64_rows(O.dequantize(ac, asf, ga), wh, sel)
    dt = time.perf_counter() - t
    return {"value": 2.0 * rows * n * k / dt / 1e12, "unit": "TFLOP/s", "cores": O.num_threads(), "kind": "oracle",
            "sample": f"dynamic quantization of A [{m},{k}] + binary64 GEMM of {rows} of {m} rows against "
                      f"W [{n},{k}] ({dt:.2f} s)"}


def cpu_baseline_moe(a_bits, off, w_bits, experts=4, rows_per_expert=2):
    """The oracle on the MoE step, sampled: grouped dynamic quantization of all
    of A, then for a few experts their weights' 2D quantization and the
    binary64 GEMM of a few of their rows."""
    import oracle as O
    E, N, K = w_bits.shape
    t = time.perf_counter()
    ac, asf, ga = O.quantize_1d_grouped(a_bits, off)
    flops = 0.0
    row0 = 0
    picked = np.linspace(0, E - 1, experts).astype(int)
    for e in range(E):
        r0, r1 = int(off[e]), int(off[e + 1])
        if e in picked and r1 > r0:
            wc, wsf, gw = O.quantize_2d(np.ascontiguousarray(w_bits[e]))
            sel = np.linspace(0, r1 - r0 - 1, min(rows_per_expert, r1 - r0)).astype(np.int64)
            ah = O.dequantize(ac[r0:r1], asf, float(ga[e]), sf_row0=row0, k=K)
            O.gemm_f64_rows(ah, O.dequantize(wc, wsf, gw), sel)
            flops += 2.0 * sel.size * N * K
        row0 += O.scale_rows(r1 - r0)
    dt = time.perf_counter() - t
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": O.num_threads(), "kind": "oracle",
            "sample": f"grouped dynamic quantization of A [{a_bits.shape[0]},{K}] ({E} groups) + for {experts} "
                      f"experts their 2D weight quantization and the binary64 GEMM of {rows_per_expert} rows "
                      f"({dt:.2f} s)"}


def cpu_baseline_quant(wl, max_seconds=12.0):
    import oracle as O
    t = time.perf_counter()
    O.quantize_1d(wl.a_host)
    dt = time.perf_counter() - t
    return {"value": wl.qbytes / dt / 1e9, "unit": "GB/s", "cores": O.num_threads(), "kind": "oracle",
            "sample": f"one full quantization of [{wl.rows},{wl.k}] ({dt:.2f} s)"}


# ---- the other configurations, measured beside the headline -------------------------------------

def _roofline(bound, kernel, achieved, peak, unit, traffic, avg_s, clocks, **extra):
    r = {"bound": bound, "kernel": kernel, "achieved": achieved, "peak": peak, "unit": unit,
         "frac": achieved / peak, "traffic": traffic, "avg_launch_ms": avg_s * 1e3,
         "launches_timed": KERNEL_ITERS, "clocks": clocks}
    r.update(extra)
    return r


def measure_quant_c2(nv, torch, dev, cs, sampler, peaks, with_cpu):
    """The activation quantizer on [8192, 4096] Laplace with outliers, and the
    16 x 16-block weight quantizer on [14336, 4096]."""
    import workloads as W
    hbm = peaks["hbm_gbs"]
    wl = Quant(nv, torch, dev)
    n = 1000
    step_s, clk = timed_loop(torch, cs, wl.step, wl.R, n, sampler)
    gbs = wl.qbytes / step_s / 1e9
    q = {"workload": wl.config()["workload"], "avg_ms": step_s * 1e3, "launches_timed": n, "gbs": gbs,
         "frac_hbm": gbs / hbm, "algorithmic_bytes": wl.qbytes,
         "roofline": _roofline("hbm", "quant1d_fused_kernel (one cooperative launch)", gbs, hbm, "GB/s",
                               load_traffic("quant_quant"), step_s, clk),
         "clocks": clk,
         "l2": f"{wl.R} rotating buffer sets of {wl.set_bytes / 1e6:.1f} MB (inputs larger than L2 between uses)"}
    wl.quantize_smooth(0)
    s_s, s_clk = timed_loop(torch, cs, wl.quantize_smooth, wl.R, KERNEL_ITERS, sampler)
    s_bytes = wl.qbytes + 4 * wl.k
    q["smooth"] = {"what": "x * s[column], s log-uniform in [1/8, 8], folded into the one-launch quantizer",
                   "avg_ms": s_s * 1e3, "gbs": s_bytes / s_s / 1e9, "frac_hbm": s_bytes / s_s / 1e9 / hbm,
                   "clocks": s_clk}
    wl.quantize_mx(0)
    x_s, x_clk = timed_loop(torch, cs, wl.quantize_mx, wl.R, KERNEL_ITERS, sampler)
    x_bytes = mx_quant_bytes(wl.rows, wl.k)
    q["mxfp4"] = {"what": "the same activations -> mxfp4 (E8M0 per 32 values, no tensor scale), one pass",
                  "avg_ms": x_s * 1e3, "gbs": x_bytes / x_s / 1e9, "frac_hbm": x_bytes / x_s / 1e9 / hbm,
                  "clocks": x_clk}
    w_s, w_clk = timed_loop(torch, cs, wl.quantize_weight, wl.RW, KERNEL_ITERS, sampler)
    w_gbs = wl.wqbytes / w_s / 1e9
    wq = {"workload": f"weight quantizer: bf16 [{wl.wn},{wl.k}] N(0,0.02) -> nvfp4, 16x16 blocks",
          "avg_ms": w_s * 1e3, "gbs": w_gbs, "frac_hbm": w_gbs / hbm, "algorithmic_bytes": wl.wqbytes,
          "roofline": _roofline("hbm", "amax_kernel + quant2d_kernel", w_gbs, hbm, "GB/s", None, w_s, w_clk),
          "clocks": w_clk}
    if with_cpu:
        q["cpu_baseline"] = cpu_baseline_quant(wl)
        wq["cpu_baseline"] = cpu_baseline_weight_quant(W.quant_weight(0, wl.wn, wl.k))
    del wl
    torch.cuda.empty_cache()
    return q, wq


def measure_decode(nv, torch, dev, cs, sampler, peaks, with_cpu, ms=(1, 8, 32, 64)):
    """The decode sweep: per m, the step (quantize + GEMM), each kernel alone,
    and the same GEMM as W4A16; the GEMM's roofline is the HBM stream of the
    weights and scales (plus A's codes and C)."""
    import workloads as W
    hbm = peaks["hbm_gbs"]
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    w_host = W.decode_weights()
    wh = None
    if with_cpu:
        import oracle as O
        wh = O.dequantize(*O.quantize_2d(w_host))
    out = {"workload": "decode W4A4: A bf16 [m,5120] quantized per call x W nvfp4 [25600,5120] (2D blocks) "
                       "-> C bf16 [m,25600]", "per_m": {}}
    for m in ms:
        progress(f"decode m = {m}")
        wl = Decode(nv, torch, dev, m=m, w_host=w_host)
        n = 1000
        step_s, clk = timed_loop(torch, cs, wl.step, wl.R, n, sampler)
        sep_s, sep_clk = timed_loop(torch, cs, wl.separate_step, wl.R, n, sampler)
        q_s, q_clk = timed_loop(torch, cs, lambda i: wl.quantize(i), wl.R, KERNEL_ITERS, sampler)
        g_s, g_clk = timed_loop(torch, cs, lambda i: wl.gemm(i), wl.R, KERNEL_ITERS, sampler)

        def w16(i):
            j = i % wl.R
            nv.gemm_w4a16(wl.a[j], wl.w[j], out=wl.c[j])
        t16, clk16 = timed_loop(torch, cs, w16, wl.R, KERNEL_ITERS, sampler)
        wl.prepare_two_phase()
        tp_s, tp_clk = timed_loop(torch, cs, wl.two_phase_step, wl.R, n, sampler)
        gbytes = wl.wbytes + wl.abytes + wl.cbytes
        g_gbs = gbytes / g_s / 1e9
        s_gbs = wl.step_bytes() / step_s / 1e9
        r = {"step_ms": step_s * 1e3, "steps_timed": n,
             "step_path": "nvfp4_quantize_gemm: amax_kernel, quant1d_kernel, then gemm_kernel as their "
                          "programmatic dependent with its first weight stages issued before its wait",
             "step_roofline": _roofline("hbm", "the step's three kernels", s_gbs, hbm, "GB/s", None, step_s, clk,
                                        algorithmic_bytes=wl.step_bytes(), launches_timed=n),
             "separate_step_ms": sep_s * 1e3, "separate_step_clocks": sep_clk,
             "two_phase_step_ms": tp_s * 1e3, "two_phase_step_clocks": tp_clk,
             "two_phase_step_path": "global scale emitted by the producing GEMM: nvfp4_quantize_act_scaled "
                                    "(quantize pass only), then nvfp4_gemm",
             "quantize_ms": q_s * 1e3, "gemm_ms": g_s * 1e3,
             "gemm_tflops": wl.flops / g_s / 1e12, "gemm_frac_fp4": wl.flops / g_s / 1e12 / fp4_peak,
             "weight_stream_gbs": wl.wbytes / g_s / 1e9, "weight_stream_frac_hbm": wl.wbytes / g_s / 1e9 / hbm,
             "step_weight_stream_gbs": wl.wbytes / step_s / 1e9,
             "roofline": _roofline("hbm", wl.gemm_label(), g_gbs, hbm, "GB/s",
                                   load_traffic("gemm_decode") if m == 64 else None, g_s, g_clk,
                                   algorithmic_bytes=gbytes),
             "w4a16": {"gemm_ms": t16 * 1e3, "weight_stream_gbs": (wl.wbytes + 2 * m * wl.k) / t16 / 1e9,
                       "frac_hbm": (wl.wbytes + 2 * m * wl.k) / t16 / 1e9 / hbm, "clocks": clk16},
             "clocks": clk, "quantize_clocks": q_clk}
        if with_cpu:
            r["cpu_baseline"] = cpu_baseline_decode(wl.a_host, wh, wl.n, wl.k)
        out["per_m"][str(m)] = r
        del wl, w16
        torch.cuda.empty_cache()
    return out


def measure_moe(nv, torch, dev, cs, sampler, peaks, with_cpu):
    """The MoE layer: grouped quantization of the routed activations and the
    grouped GEMM over 128 experts.  Below the FP4 ridge (about 565 flop per
    byte against ~1000), so the GEMM's roofline is the HBM traffic of the
    expert weights, A's codes and C; the FP4 fraction is reported beside it."""
    hbm = peaks["hbm_gbs"]
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    wl = Moe(nv, torch, dev)
    n = 200
    step_s, clk = timed_loop(torch, cs, wl.step, wl.R, n, sampler)
    q_s, q_clk = timed_loop(torch, cs, lambda i: wl.quantize(i), wl.R, KERNEL_ITERS, sampler)
    g_s, g_clk = timed_loop(torch, cs, lambda i: wl.gemm(i), wl.R, KERNEL_ITERS, sampler)
    tfl = wl.flops / g_s / 1e12
    g_gbs = wl.gemm_bytes / g_s / 1e9
    t_tensor, t_hbm = wl.flops / (fp4_peak * 1e12), wl.gemm_bytes / (hbm * 1e9)
    out = {"workload": wl.config()["workload"], "step_ms": step_s * 1e3, "steps_timed": n,
           "step_tflops": wl.flops / step_s / 1e12, "quantize_ms": q_s * 1e3,
           "quantize_gbs": wl.qbytes / q_s / 1e9, "quantize_frac_hbm": wl.qbytes / q_s / 1e9 / hbm,
           "gemm_ms": g_s * 1e3, "gemm_tflops": tfl, "gemm_frac_fp4": tfl / fp4_peak,
           "gemm_frac_nominal_fp4": tfl / NOMINAL_FP4_TFLOPS, "gemm_gbs": g_gbs, "gemm_frac_hbm": g_gbs / hbm,
           "roofline": (_roofline("hbm", wl.gemm_label(), g_gbs, hbm, "GB/s", load_traffic("gemm_moe"), g_s, g_clk,
                                  algorithmic_bytes=wl.gemm_bytes, tensor_bound_ms=t_tensor * 1e3)
                        if t_hbm >= t_tensor else
                        _roofline("tensor", wl.gemm_label(), tfl, fp4_peak, "TFLOP/s", load_traffic("gemm_moe"),
                                  g_s, g_clk, hbm_bound_ms=t_hbm * 1e3)),
           "mma_padding": wl.padding(), "clocks": clk, "quantize_clocks": q_clk}
    if with_cpu:
        out["cpu_baseline"] = cpu_baseline_moe(wl.a_host, wl.off_host, wl.w_host)
    del wl
    torch.cuda.empty_cache()
    return out


# ---- the two arms ------------------------------------------------------------------------------

def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    import oracle as O
    import workloads as W
    if args.workload == "quant":
        x = W.quant_act(0)
        unit = "GB/s"
        work = quant_bytes(8192, 4096)
        cfg = Quant.config(type("Q", (), {"rows": 8192, "k": 4096})())

        def step():
            O.quantize_1d(x)
        sample = "one full quantization of [8192,4096] per step"
    else:
        m, n, k = (4096, 14336, 4096) if args.workload == "prefill" else (args.decode_m, 25600, 5120)
        a, w = W.prefill(0, m, n, k) if args.workload == "prefill" else W.decode(m)
        wc, wsf, gw = O.quantize_2d(w)
        wh = O.dequantize(wc, wsf, gw)
        rows = min(m, args.ref_rows)
        sel = np.linspace(0, m - 1, rows).astype(np.int64)
        unit = "TFLOP/s"
        work = 2.0 * rows * n * k
        cfg = {"workload": f"{args.workload} W4A4 m={m} n={n} k={k}", "m": m, "n": n, "k": k}

        def step():
            ac, asf, ga = O.quantize_1d(a)
            O.gemm_f64_rows(O.dequantize(ac, asf, ga), wh, sel)
        sample = (f"per step: dynamic quantization of the whole A [{m},{k}] + binary64 GEMM of {rows} of {m} "
                  f"rows against W [{n},{k}]")
    for _ in range(args.warmup):
        step()
    t = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t
    value = work * args.steps / dt / (1e12 if unit == "TFLOP/s" else 1e9)
    line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": 0, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": dt / args.steps * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
            "impl": "reference",
            "cpu_baseline": {"value": value, "unit": unit, "kind": "oracle", "cores": O.num_threads(),
                             "sample": sample},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def load_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            t = json.load(f)
        from nvfp4_w4a4_quantized_05_b200 import build as B
        entry = t.get(kernel)
        if entry and entry.get("src_hash") == B._src_hash():
            return entry.get("bytes_per_launch")
    except (OSError, ValueError, ImportError):
        pass
    return None


def run_ours(args):
    import torch
    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        print(json.dumps({"metric": METRIC, "error": "no CUDA device"}))
        return 1
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    import nvfp4_w4a4_quantized_05_b200 as nv
    nv.lib()
    peaks = load_peaks()
    progress(f"building the {args.workload} workload")
    wl = {"prefill": Prefill, "decode": Decode, "quant": Quant, "moe": Moe}[args.workload]
    wl = wl(nv, torch, dev, m=args.decode_m) if args.workload == "decode" else wl(nv, torch, dev)
    cs = torch.cuda.Stream(dev)
    sampler = ClockSampler(local)
    sampler.start()

    progress("timed steps")
    # capture, then warm-up (eager first calls + one replay of every graph)
    steps = StepGraphs(torch, cs, wl.step, wl.R, args.steps)
    warm = steps.warm(max(3, args.warmup))
    nv.check_device_error()

    # ---- timed region: exactly K steps ----
    time.sleep(REST_S)
    barrier(world)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    e0, e1 = steps.run()
    torch.cuda.synchronize()
    barrier(world)
    t1 = time.perf_counter()
    nv.check_device_error()
    total = reduce_max(e0.elapsed_time(e1) * 1e-3, world, dev)
    clocks = sampler.summary(t0, t1)
    del steps

    # ---- per-kernel times: each kernel alone, back to back over the same buffer sets ----
    kiters = max(KERNEL_ITERS, min(args.steps, 2000))
    ktimes, kclocks = [], []
    for f in wl.kernels:
        time.sleep(REST_S)
        ta = time.perf_counter()
        ktimes.append(graph_seconds(torch, cs, lambda i, f=f: f(wl, i), wl.R, kiters))
        kclocks.append(sampler.summary(ta, time.perf_counter()))
    q_avg = ktimes[0]
    g_avg = ktimes[1] if len(ktimes) > 1 else None
    nv.check_device_error()

    # ---- end to end through the public API from pinned host memory ----
    e2e = None
    if not args.no_e2e:
        a_pinned = torch.from_numpy(wl.a_host.view(np.int16)).pin_memory()
        out0 = wl.result(0)
        out_pinned = torch.empty(out0.shape, dtype=out0.dtype).pin_memory()

        def e2e_step(i):
            wl.a[i % wl.R].view(torch.int16).copy_(a_pinned, non_blocking=True)
            wl.step(i)
            out_pinned.copy_(wl.result(i), non_blocking=True)
        n_e2e = max(5, min(args.steps, 50))
        with torch.cuda.stream(cs):
            for i in range(2):
                e2e_step(i)
            cs.synchronize()
            ea, eb = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            ea.record()
            for i in range(n_e2e):
                e2e_step(i)
            eb.record()
        cs.synchronize()
        e_avg = reduce_max(ea.elapsed_time(eb) * 1e-3 / n_e2e, world, dev)
        h2d = a_pinned.numel() * a_pinned.element_size()
        d2h = out_pinned.numel() * out_pinned.element_size()
        if wl.flops:
            ev, eu = world * wl.flops / e_avg / 1e12, "TFLOP/s"
        else:
            ev, eu = world * wl.qbytes / e_avg / 1e9, "GB/s"
        e2e = {"value": ev, "unit": eu, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "path": "eager calls of the Python binding on one stream; pinned host buffers"}

    ms = total / args.steps * 1e3
    fp4_peak = peaks["bf16_tflops"] * FP4_PER_BF16
    q_gbs = wl.qbytes / q_avg / 1e9
    line = {"metric": METRIC}
    if wl.flops:
        value = world * wl.flops * args.steps / total / 1e12
        line.update({"value": value, "unit": "TFLOP/s"})
    else:
        value = world * wl.qbytes * args.steps / total / 1e9
        line.update({"value": value, "unit": "GB/s"})
    line.update({"n_gpus": world, "steps": args.steps, "warmup": args.warmup, "warmup_calls_run": warm,
                 "ms_per_step": ms,
                 "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                 "dtype": "fp4 (e2m1 x e2m1, e4m3 block scales, f32 accumulate)",
                 "data": "synthetic (seeded; see workloads/)"})
    cfg = wl.config()
    l2 = (f"inputs larger than L2: steps rotate over {wl.R} buffer sets of {wl.set_bytes / 1e6:.1f} MB; "
          f"between two uses of a set the others move {(wl.R - 1) * wl.set_bytes / 1e6:.0f} MB (L2 126 MB)")
    small = min(wl.kernel_bytes)
    if (wl.R - 1) * small < 2 * L2_BYTES:
        l2 += (f"; the quantizer timed alone cycles through only {(wl.R - 1) * small / 1e6:.0f} MB, so its "
               f"{small / 1e6:.2f} MB of activations may sit in L2, as a previous layer's output would")
    cfg.update({"l2": l2,
                "launch": f"CUDA graphs of {wl.R} steps replayed on one stream; per-kernel times from graphs "
                          "of that kernel alone over the same buffer sets",
                "parallelism": f"replicas x{world}" if world > 1 else "single GPU"})
    line["config"] = cfg
    if g_avg is not None:
        g_tflops = wl.flops / g_avg / 1e12
        line["roofline"] = {"bound": "tensor", "kernel": wl.gemm_label(),
                            "achieved": g_tflops, "peak": fp4_peak, "unit": "TFLOP/s",
                            "frac": g_tflops / fp4_peak, "traffic": load_traffic(f"gemm_{wl.name}"),
                            "peak_note": f"{peaks['source']} bf16 burst {peaks['bf16_tflops']} x {FP4_PER_BF16} "
                                         "(dense FP4 / BF16 nominal ratio)",
                            "frac_of_nominal_fp4": g_tflops / NOMINAL_FP4_TFLOPS,
                            "nominal_fp4_tflops": NOMINAL_FP4_TFLOPS,
                            "avg_launch_ms": g_avg * 1e3, "launches_timed": kiters, "clocks": kclocks[1]}
    else:
        line["roofline"] = {"bound": "hbm", "kernel": "quant1d_fused_kernel (one cooperative launch)",
                            "achieved": q_gbs,
                            "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": q_gbs / peaks["hbm_gbs"],
                            "traffic": load_traffic(f"quant_{wl.name}"),
                            "peak_note": f"{peaks['source']} HBM copy bandwidth", "avg_launch_ms": q_avg * 1e3,
                            "launches_timed": kiters, "clocks": kclocks[0]}
    line["quantize"] = {"gbs": q_gbs, "frac_hbm": q_gbs / peaks["hbm_gbs"], "avg_ms": q_avg * 1e3,
                        "algorithmic_bytes": wl.qbytes}
    if hasattr(wl, "quantize_weight"):
        time.sleep(REST_S)
        w_avg = graph_seconds(torch, cs, wl.quantize_weight, wl.RW, kiters)
        w_gbs = wl.wqbytes / w_avg / 1e9
        line["weight_quantize"] = {"workload": f"bf16 [{wl.wn},{wl.k}] N(0,0.02) -> nvfp4, 16x16 blocks",
                                   "gbs": w_gbs, "frac_hbm": w_gbs / peaks["hbm_gbs"], "avg_ms": w_avg * 1e3,
                                   "algorithmic_bytes": wl.wqbytes, "kernels": "amax_kernel + quant2d_kernel"}
        wl.quantize_smooth(0)
        time.sleep(REST_S)
        s_avg = graph_seconds(torch, cs, wl.quantize_smooth, wl.R, kiters)
        s_bytes = wl.qbytes + 4 * wl.k
        line["smooth_quantize"] = {"workload": f"the same activations x * s[column], s log-uniform in [1/8, 8]",
                                   "gbs": s_bytes / s_avg / 1e9, "frac_hbm": s_bytes / s_avg / 1e9 / peaks["hbm_gbs"],
                                   "avg_ms": s_avg * 1e3, "algorithmic_bytes": s_bytes,
                                   "kernels": "quant1d_fused_kernel (pre-scaled form)"}
    if hasattr(wl, "quantize_mx"):
        wl.quantize_mx(0)
        time.sleep(REST_S)
        x_avg = graph_seconds(torch, cs, wl.quantize_mx, wl.R, kiters)
        x_bytes = mx_quant_bytes(wl.rows, wl.k)
        line["mx_quantize"] = {"workload": "the same activations -> mxfp4 (E8M0 scale per 32 values, no tensor scale)",
                               "gbs": x_bytes / x_avg / 1e9, "frac_hbm": x_bytes / x_avg / 1e9 / peaks["hbm_gbs"],
                               "avg_ms": x_avg * 1e3, "algorithmic_bytes": x_bytes,
                               "kernels": "quant1d_kernel (MXFP4 form, one pass)"}
    if isinstance(wl, Prefill):
        import workloads as W
        w_host = W.prefill(0, wl.m, wl.n, wl.k)[1] if type(wl) is Prefill else W.decode(wl.m)[1]
        mq, mg, ms = wl.mx_steps(nv, torch, w_host)
        del w_host
        time.sleep(REST_S)
        xq = graph_seconds(torch, cs, mq, wl.R, kiters)
        time.sleep(REST_S)
        xg = graph_seconds(torch, cs, mg, wl.R, kiters)
        time.sleep(REST_S)
        xs = graph_seconds(torch, cs, ms, wl.R, kiters)
        xq_bytes = mx_quant_bytes(wl.m, wl.k)
        line["mxfp4"] = {
            "what": "the same shapes in MXFP4: activations quantized per call (E8M0 per 32), weights pre-quantized",
            "quantize_ms": xq * 1e3, "quantize_gbs": xq_bytes / xq / 1e9,
            "gemm_ms": xg * 1e3, "gemm_tflops": wl.flops / xg / 1e12,
            "gemm_frac_fp4_peak": wl.flops / xg / 1e12 / fp4_peak, "step_ms": xs * 1e3,
            "kernels": "quant1d_kernel (MXFP4 form) + " + wl.gemm_label().replace("mxf4nvf4", "mxf4nvf4 block32")}
    if type(wl) is Prefill:
        one_phase, two_phase = wl.next_layer_steps(nv, torch)
        time.sleep(REST_S)
        t1 = graph_seconds(torch, cs, one_phase, wl.R, kiters)
        time.sleep(REST_S)
        t2 = graph_seconds(torch, cs, two_phase, wl.R, kiters)
        line["next_layer_quant"] = {
            "what": "GEMM + dynamic quantization of its BF16 output C [m, n] for the next layer",
            "one_phase_ms": t1 * 1e3, "two_phase_ms": t2 * 1e3, "gemm_alone_ms": g_avg * 1e3,
            "note": "one phase: GEMM, then the one-launch quantizer (amax pass + quantize pass over C); two phase: "
                    "GEMM emitting C's global scale from its epilogue, then the quantize pass alone"}
    if isinstance(wl, Decode):
        def w16(i):
            j = i % wl.R
            nv.gemm_w4a16(wl.a[j], wl.w[j], out=wl.c[j])
        time.sleep(REST_S)
        t16 = graph_seconds(torch, cs, w16, wl.R, kiters)
        line["w4a16"] = {
            "what": "the same decode GEMM as W4A16: activations kept in BF16, the same NVFP4 weights dequantized "
                    "to BF16 in the kernel, BF16 tensor-core MMAs (no activation quantization)",
            "gemm_ms": t16 * 1e3, "weight_stream_gbs": wl.wbytes / t16 / 1e9,
            "frac_hbm": wl.wbytes / t16 / 1e9 / peaks["hbm_gbs"],
            "w4a4_gemm_ms": g_avg * 1e3, "w4a4_step_ms": line["ms_per_step"],
            "traffic": load_traffic("w4a16_decode"),
            "kernels": "w4a16_kernel (tcgen05 kind::f16, 64 token rows x 192 weight rows per tile)"}
        line["weight_stream"] = {"gbs": wl.wbytes / g_avg / 1e9, "frac_hbm": wl.wbytes / g_avg / 1e9 / peaks["hbm_gbs"],
                                 "bytes": wl.wbytes}
    line["e2e"] = e2e
    line["gpu_launches"] = wl.launches_per_step * args.steps
    line["clocks"] = clocks
    sampler.stop()
    with_cpu = rank == 0 and world == 1 and not args.no_cpu_baseline
    progress("cpu baseline")
    if with_cpu:
        line["cpu_baseline"] = (cpu_baseline_quant(wl) if wl.name == "quant" else
                                cpu_baseline_prefill(wl) if wl.name in ("prefill", "decode") else
                                cpu_baseline_moe(wl.a_host, wl.off_host, wl.w_host))
    if args.workload == "prefill" and not args.no_extra and world == 1:
        # every other configuration of the path, each measured here with its
        # own roofline, clocks and CPU baseline (one GPU: per-GPU figures)
        del wl
        import gc
        gc.collect()
        torch.cuda.empty_cache()
        sampler.start()
        progress("activation and weight quantizers")
        line["quant_c2"], line["weight_quant"] = measure_quant_c2(nv, torch, dev, cs, sampler, peaks, with_cpu)
        progress("decode sweep")
        line["decode"] = measure_decode(nv, torch, dev, cs, sampler, peaks, with_cpu)
        progress("moe")
        line["moe"] = measure_moe(nv, torch, dev, cs, sampler, peaks, with_cpu)
        progress("done")
        sampler.stop()
        nv.check_device_error()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: enough for a >= 50 ms timed region on this workload)")
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=["prefill", "quant", "decode", "moe"], default="prefill")
    ap.add_argument("--decode-m", type=int, default=64)
    ap.add_argument("--ref-rows", type=int, default=4)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="prefill: skip the other configurations (activation and weight quantizers, decode sweep, MoE)")
    args = ap.parse_args(argv)
    if args.steps is None:
        args.steps = (20 if args.impl == "reference" else
                      {"prefill": 500, "quant": 2000, "decode": 2000, "moe": 300}[args.workload])
    if args.steps < 1:
        ap.error("--steps must be at least 1")
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
