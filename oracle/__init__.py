"""CPU oracle for NVFP4 W4A4 quantization and the block-scaled FP4 GEMM.

TEST INFRASTRUCTURE.  Only tests/, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package.  The product path
(``nvfp4_w4a4_quantized_05_b200``) never imports it and shares no code with it.

The arithmetic lives in plain C (``nvfp4_oracle.c``); this module only moves
numpy arrays across ctypes.  Inputs are BF16 bit patterns (``uint16``).

Parity pins (tests/test_oracle_*.py): E2M1 magnitudes from the pages; encoders
against brute-force nearest search; exactly representable round trips with
the global scale of Figure 1 of "Accelerating large language models with NVFP4
quantization"; the 4.5 bits/value storage rule; the outlier-error claim; the
GEMM against an exact integer sum and a library matmul; the given-scale and
pre-scaled quantizers against the plain one on exactly scaled inputs; the
block quantizer at tiny global scales, where 1 / d overflows binary32
(exact constructions whose codes are known: the round trip at g = 2^-123 and
blocks of v * 2^-130 at a rounded subnormal g); the single-scale baseline on
worked examples (its scale amax / 6 and its ties to the even code); the
MXFP4 scale choice as a property over every BF16 magnitude, its round trip,
nearest codes and 4.25 bits/value, and NVFP4's lower error on outliers; the
W4A16 product against one-hot rows, the W4A4 product and a library matmul
(tests/test_oracle_mx.py, tests/test_oracle_w4a16.py).  The scale-tile
layout is not on the pages: on the CPU only its bijection onto the padded
buffer is checked; on the GPU a library block-scaled NVFP4 GEMM (cuBLASLt
through torch's scaled_mm) reads scale bytes equal to the oracle's and must
give the oracle's product (tests/test_gpu_gemm.py).
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

_u8p = np.ctypeslib.ndpointer(np.uint8, flags="C_CONTIGUOUS")
_u16p = np.ctypeslib.ndpointer(np.uint16, flags="C_CONTIGUOUS")
_i32p = np.ctypeslib.ndpointer(np.int32, flags="C_CONTIGUOUS")
_i64p = np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS")
_f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
_f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
_i64 = ctypes.c_int64


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        sig = {
            "orc_e2m1_encode": (ctypes.c_uint8, [ctypes.c_float]),
            "orc_e2m1_decode": (ctypes.c_double, [ctypes.c_uint8]),
            "orc_e4m3_encode": (ctypes.c_uint8, [ctypes.c_float]),
            "orc_e4m3_decode": (ctypes.c_double, [ctypes.c_uint8]),
            "orc_e2m1_encode_array": (None, [_f32p, _u8p, _i64]),
            "orc_e4m3_encode_array": (None, [_f32p, _u8p, _i64]),
            "orc_scale_rows": (_i64, [_i64]),
            "orc_scale_cols": (_i64, [_i64]),
            "orc_sf_offset": (_i64, [_i64, _i64, _i64]),
            "orc_global_scale": (ctypes.c_float, [ctypes.c_float]),
            "orc_quantize_1d": (ctypes.c_int, [_u16p, _i64, _i64, _i64, _u8p, _u8p, _f32p]),
            "orc_quantize_1d_given_g": (ctypes.c_int, [_u16p, _i64, _i64, _i64, ctypes.c_float, _u8p, _u8p]),
            "orc_quantize_1d_smooth": (ctypes.c_int, [_u16p, _i64, _i64, _i64, _f32p, _u8p, _u8p, _f32p]),
            "orc_grouped_scale_rows": (_i64, [_i32p, ctypes.c_int]),
            "orc_quantize_1d_grouped": (ctypes.c_int, [_u16p, _i32p, ctypes.c_int, _i64, _i64,
                                                       _u8p, _u8p, _f32p]),
            "orc_quantize_2d": (ctypes.c_int, [_u16p, _i64, _i64, _i64, _u8p, _u8p,
                                               ctypes.c_void_p, _f32p]),
            "orc_dequantize": (None, [_u8p, _u8p, ctypes.c_float, _i64, _i64, _i64, _i64, _f64p]),
            "orc_gemm_f64": (None, [_f64p, _f64p, _i64, _i64, _i64, _f64p]),
            "orc_gemm_f64_rows": (None, [_f64p, _f64p, _i64p, _i64, _i64, _i64, _f64p]),
            "orc_gemm_exact_i64": (None, [_u8p, _u8p, _u8p, _u8p, _i64, _i64, _i64, _i64p]),
            "orc_single_scale_fp4": (None, [_u16p, _i64, _f64p]),
            "orc_mx_scale_cols": (_i64, [_i64]),
            "orc_e8m0_block_scale": (ctypes.c_uint8, [ctypes.c_double]),
            "orc_e8m0_decode": (ctypes.c_double, [ctypes.c_uint8]),
            "orc_quantize_1d_mx": (ctypes.c_int, [_u16p, _i64, _i64, _i64, _u8p, _u8p]),
            "orc_dequantize_mx": (None, [_u8p, _u8p, _i64, _i64, _f64p]),
            "orc_num_threads": (ctypes.c_int, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def num_threads() -> int:
    return lib().orc_num_threads()


# ---- scalar formats ---------------------------------------------------------

def e2m1_encode(v: float) -> int:
    return int(lib().orc_e2m1_encode(float(v)))


def e2m1_decode(code: int) -> float:
    return float(lib().orc_e2m1_decode(int(code)))


def e4m3_encode(a: float) -> int:
    return int(lib().orc_e4m3_encode(float(a)))


def e4m3_decode(code: int) -> float:
    return float(lib().orc_e4m3_decode(int(code)))


def e2m1_encode_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32).ravel()
    out = np.empty(v.size, np.uint8)
    lib().orc_e2m1_encode_array(v, out, v.size)
    return out


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32).ravel()
    out = np.empty(v.size, np.uint8)
    lib().orc_e4m3_encode_array(v, out, v.size)
    return out


# ---- layout ---------------------------------------------------------------------

def scale_rows(rows: int) -> int:
    return int(lib().orc_scale_rows(rows))


def scale_cols(k: int) -> int:
    return int(lib().orc_scale_cols(k))


def sf_offset(r: int, c: int, k: int) -> int:
    return int(lib().orc_sf_offset(r, c, scale_cols(k)))


def global_scale(amax: float) -> float:
    return float(lib().orc_global_scale(float(amax)))


# ---- quantizers -----------------------------------------------------------------

def _bf16(x):
    x = np.ascontiguousarray(x)
    if x.dtype != np.uint16:
        raise TypeError("oracle inputs are BF16 bit patterns (uint16)")
    return x


def quantize_1d(x_bf16: np.ndarray):
    """1D 16-element blocks.  Returns (codes [R, K/2] u8, scales (flat, tile
    layout) u8, g float)."""
    x = _bf16(x_bf16)
    rows, k = x.shape
    codes = np.zeros((rows, k // 2), np.uint8)
    sf = np.zeros(scale_rows(rows) * scale_cols(k), np.uint8)
    g = np.zeros(1, np.float32)
    rc = lib().orc_quantize_1d(x, rows, k, k, codes, sf, g)
    if rc != 0:
        raise ValueError(f"orc_quantize_1d failed ({rc})")
    return codes, sf, float(g[0])


def quantize_1d_given_g(x_bf16: np.ndarray, g: float):
    """1D quantization with the global scale g given (the two-phase form's
    second pass): steps 3-8 of the block quantizer with g from the caller."""
    x = _bf16(x_bf16)
    rows, k = x.shape
    codes = np.zeros((rows, k // 2), np.uint8)
    sf = np.zeros(scale_rows(rows) * scale_cols(k), np.uint8)
    rc = lib().orc_quantize_1d_given_g(x, rows, k, k, float(np.float32(g)), codes, sf)
    if rc != 0:
        raise ValueError(f"orc_quantize_1d_given_g failed ({rc})")
    return codes, sf


def quantize_1d_smooth(x_bf16: np.ndarray, s: np.ndarray):
    """1D quantization of x' = fp32(x) * s[column] (SmoothQuant-style
    per-channel pre-scaling folded into the quantizer).  Returns (codes,
    scales, g)."""
    x = _bf16(x_bf16)
    rows, k = x.shape
    sv = np.ascontiguousarray(s, dtype=np.float32)
    if sv.shape != (k,):
        raise ValueError("s must have one factor per column")
    codes = np.zeros((rows, k // 2), np.uint8)
    sf = np.zeros(scale_rows(rows) * scale_cols(k), np.uint8)
    g = np.zeros(1, np.float32)
    rc = lib().orc_quantize_1d_smooth(x, rows, k, k, sv, codes, sf, g)
    if rc != 0:
        raise ValueError(f"orc_quantize_1d_smooth failed ({rc})")
    return codes, sf, float(g[0])


def grouped_scale_rows(offsets: np.ndarray) -> int:
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    return int(lib().orc_grouped_scale_rows(off, off.size - 1))


def quantize_1d_grouped(x_bf16: np.ndarray, offsets: np.ndarray):
    """Per-group 1D quantization: rows [off[e], off[e+1]) form group e with its
    own global scale; group e's scale rows start at a multiple of 128."""
    x = _bf16(x_bf16)
    off = np.ascontiguousarray(offsets, dtype=np.int32)
    rows, k = x.shape
    E = off.size - 1
    codes = np.zeros((rows, k // 2), np.uint8)
    sf = np.zeros(grouped_scale_rows(off) * scale_cols(k), np.uint8)
    g = np.zeros(E, np.float32)
    rc = lib().orc_quantize_1d_grouped(x, off, E, k, k, codes, sf, g)
    if rc != 0:
        raise ValueError(f"orc_quantize_1d_grouped failed ({rc})")
    return codes, sf, g


def quantize_2d(w_bf16: np.ndarray, compact: bool = False):
    """16x16 blocks.  Returns (codes, scales in tile layout, g[, compact [R/16, K/16]])."""
    w = _bf16(w_bf16)
    rows, k = w.shape
    codes = np.zeros((rows, k // 2), np.uint8)
    sf = np.zeros(scale_rows(rows) * scale_cols(k), np.uint8)
    sfc = np.zeros((rows // 16, k // 16), np.uint8) if compact else None
    g = np.zeros(1, np.float32)
    rc = lib().orc_quantize_2d(w, rows, k, k, codes, sf,
                               sfc.ctypes.data if compact else None, g)
    if rc != 0:
        raise ValueError(f"orc_quantize_2d failed ({rc})")
    if compact:
        return codes, sf, float(g[0]), sfc
    return codes, sf, float(g[0])


def dequantize(codes: np.ndarray, sf: np.ndarray, g: float, sf_row0: int = 0,
               k: int | None = None) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    rows = codes.shape[0]
    k = codes.shape[1] * 2 if k is None else k
    out = np.empty((rows, k), np.float64)
    lib().orc_dequantize(codes, np.ascontiguousarray(sf, dtype=np.uint8), float(g),
                         rows, k, sf_row0, scale_cols(k), out)
    return out


def dequantize_grouped(codes, sf, g, offsets) -> np.ndarray:
    off = np.asarray(offsets, dtype=np.int64)
    k = codes.shape[1] * 2
    out = np.zeros((codes.shape[0], k), np.float64)
    row0 = 0
    for e in range(off.size - 1):
        a, b = int(off[e]), int(off[e + 1])
        if b > a:
            out[a:b] = dequantize(codes[a:b], sf, float(g[e]), sf_row0=row0, k=k)
        row0 += scale_rows(b - a)
    return out


# ---- MXFP4 ----------------------------------------------------------------------

def mx_scale_cols(k: int) -> int:
    return int(lib().orc_mx_scale_cols(k))


def e8m0_block_scale(bamax: float) -> int:
    """E8M0 byte of a 32-value block with maximum magnitude bamax."""
    return int(lib().orc_e8m0_block_scale(float(bamax)))


def e8m0_decode(b: int) -> float:
    return float(lib().orc_e8m0_decode(b))


def quantize_1d_mx(x_bf16: np.ndarray):
    """MXFP4: 32-value blocks with E8M0 scales, no tensor scale.  Returns
    (codes [R, K/2] u8, scales (flat, tile layout, k/32 columns rounded to 4) u8)."""
    x = _bf16(x_bf16)
    rows, k = x.shape
    codes = np.zeros((rows, k // 2), np.uint8)
    sf = np.zeros(scale_rows(rows) * mx_scale_cols(k), np.uint8)
    rc = lib().orc_quantize_1d_mx(x, rows, k, k, codes, sf)
    if rc != 0:
        raise ValueError(f"orc_quantize_1d_mx failed ({rc})")
    return codes, sf


def dequantize_mx(codes: np.ndarray, sf: np.ndarray, k: int | None = None) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    rows = codes.shape[0]
    k = codes.shape[1] * 2 if k is None else k
    out = np.empty((rows, k), np.float64)
    lib().orc_dequantize_mx(codes, np.ascontiguousarray(sf, dtype=np.uint8), rows, k, out)
    return out


# ---- GEMM -----------------------------------------------------------------------

def gemm_f64(a_hat: np.ndarray, w_hat: np.ndarray) -> np.ndarray:
    a = np.ascontiguousarray(a_hat, dtype=np.float64)
    w = np.ascontiguousarray(w_hat, dtype=np.float64)
    m, k = a.shape
    n = w.shape[0]
    c = np.empty((m, n), np.float64)
    lib().orc_gemm_f64(a, w, m, n, k, c)
    return c


def gemm_f64_rows(a_hat: np.ndarray, w_hat: np.ndarray, rows) -> np.ndarray:
    a = np.ascontiguousarray(a_hat, dtype=np.float64)
    w = np.ascontiguousarray(w_hat, dtype=np.float64)
    sel = np.ascontiguousarray(rows, dtype=np.int64)
    k = a.shape[1]
    n = w.shape[0]
    c = np.empty((sel.size, n), np.float64)
    lib().orc_gemm_f64_rows(a, w, sel, sel.size, n, k, c)
    return c


def gemm_w4a16_f64(a_bf16: np.ndarray, w_codes, w_sf, w_g: float) -> np.ndarray:
    """W4A16: BF16 activations (exact in binary64) times the reconstructed NVFP4
    weights, C = A * W_hat^T in binary64 ("W4A8 vs NVFP4 quantization on GPUs",
    weight-only quantization: only the weights are four-bit)."""
    return gemm_f64(bf16_to_f64(a_bf16), dequantize(w_codes, w_sf, w_g))


def gemm_exact_i64(a_codes, a_sf, w_codes, w_sf, k: int) -> np.ndarray:
    """sum_k (qa*sfa)(qw*sfw) * 2^20 as exact int64 (global scales excluded)."""
    a_codes = np.ascontiguousarray(a_codes, dtype=np.uint8)
    w_codes = np.ascontiguousarray(w_codes, dtype=np.uint8)
    m, n = a_codes.shape[0], w_codes.shape[0]
    c = np.empty((m, n), np.int64)
    lib().orc_gemm_exact_i64(a_codes, np.ascontiguousarray(a_sf, dtype=np.uint8), w_codes,
                             np.ascontiguousarray(w_sf, dtype=np.uint8), m, n, k, c)
    return c


def single_scale_fp4(x_bf16: np.ndarray) -> np.ndarray:
    x = _bf16(x_bf16)
    out = np.empty(x.size, np.float64)
    lib().orc_single_scale_fp4(x.ravel(), x.size, out)
    return out.reshape(x.shape)


def bf16_to_f64(x_bf16: np.ndarray) -> np.ndarray:
    """Exact widening of BF16 bit patterns (plain bit shift)."""
    x = _bf16(x_bf16)
    return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


__all__ = [n for n in dir() if not n.startswith("_")]

if os.environ.get("NVFP4_ORACLE_EAGER_BUILD"):
    lib()
