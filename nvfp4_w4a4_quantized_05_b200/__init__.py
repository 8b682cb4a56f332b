"""NVFP4 W4A4 inference hot path for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``libnvfp4.so`` (``include/nvfp4.h``):
argument marshalling only.  Every step of the path runs in the library's CUDA
kernels; PyTorch is used for device memory and streams.  There is no CPU
fallback: if the library cannot be loaded, every call raises.

Raw entry points keep the C names (``nvfp4_quantize_act``, ``nvfp4_gemm``, ...)
and take integer device addresses.  The tensor-level helpers
(``quantize_act``, ``quantize_weight_2d``, ``gemm``, ``grouped_gemm``)
allocate outputs with torch on the input's device and run on torch's current
stream.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass
from typing import Optional

__all__ = [
    "lib", "Nvfp4Error", "NVFP4Tensor",
    "nvfp4_codes_bytes", "nvfp4_scale_bytes", "nvfp4_grouped_scale_bytes", "nvfp4_workspace_bytes",
    "nvfp4_workspace_init", "nvfp4_quantize_act", "nvfp4_quantize_act_static", "nvfp4_quantize_weight_2d",
    "nvfp4_gemm", "nvfp4_gemm_emit_scale", "nvfp4_quantize_act_scaled", "nvfp4_quantize_act_smooth",
    "nvfp4_grouped_gemm", "nvfp4_get_last_device_error", "nvfp4_set_wait_limit_ns", "nvfp4_probe_cvt",
    "nvfp4_probe_bounded_wait", "nvfp4_status_string", "nvfp4_version",
    "quantize_act", "quantize_weight_2d", "gemm", "grouped_gemm", "check_device_error",
    "gemm_emit_scale", "quantize_act_scaled", "quantize_act_smooth",
    "mxfp4_scale_bytes", "mxfp4_quantize_act", "mxfp4_gemm", "MXFP4Tensor", "quantize_mx", "gemm_mx",
    "w4a16_gemm", "gemm_w4a16", "nvfp4_quantize_gemm", "quantize_gemm", "OP_QUANTIZE_GEMM",
    "OP_QUANTIZE_ACT", "OP_QUANTIZE_WEIGHT_2D", "OP_GEMM", "OP_GROUPED_GEMM", "OP_GEMM_EMIT_SCALE",
]

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libnvfp4.so")

OP_QUANTIZE_ACT, OP_QUANTIZE_WEIGHT_2D, OP_GEMM, OP_GROUPED_GEMM, OP_GEMM_EMIT_SCALE, OP_QUANTIZE_GEMM = 0, 1, 2, 3, 4, 5
STATUS = {0: "OK", 1: "INVALID_ARGUMENT", 2: "UNSUPPORTED_SHAPE", 3: "MISALIGNED", 4: "CUDA",
          5: "TIMEOUT", 6: "NO_DEVICE"}


class Nvfp4Error(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS.get(status, status)} ({_status_string(status)})")


_lib = None
_lock = threading.Lock()
_vp, _i64, _u64, _i32, _sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_int, ctypes.c_size_t

_SIGNATURES = {
    "nvfp4_status_string": (ctypes.c_char_p, [_i32]),
    "nvfp4_version": (ctypes.c_char_p, []),
    "nvfp4_codes_bytes": (_sz, [_i64, _i64]),
    "nvfp4_scale_bytes": (_sz, [_i64, _i64]),
    "nvfp4_grouped_scale_bytes": (_sz, [_i64, _i32, _i64]),
    "nvfp4_workspace_bytes": (_sz, [_i32, _i64, _i64, _i64, _i32]),
    "nvfp4_workspace_init": (_i32, [_vp, _sz, _vp]),
    "nvfp4_quantize_act": (_i32, [_vp, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _vp, _vp, _vp]),
    "nvfp4_quantize_act_static": (_i32, [_vp, _i64, _i64, _i64, _vp, _i32, _vp, _vp, _vp, _vp]),
    "nvfp4_quantize_weight_2d": (_i32, [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "nvfp4_gemm": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _vp, _vp]),
    "nvfp4_gemm_emit_scale": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _vp, _vp, _vp]),
    "nvfp4_quantize_act_scaled": (_i32, [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp]),
    "nvfp4_quantize_act_smooth": (_i32, [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "nvfp4_grouped_gemm": (_i32, [_vp, _vp, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _vp, _vp]),
    "nvfp4_quantize_gemm": (_i32, [_vp, _i64, _i64, _i64, _vp, _vp, _vp, _i64, _vp, _i64, _vp, _vp, _vp, _vp, _vp]),
    "mxfp4_scale_bytes": (_sz, [_i64, _i64]),
    "mxfp4_quantize_act": (_i32, [_vp, _i64, _i64, _i64, _vp, _vp, _vp]),
    "mxfp4_gemm": (_i32, [_vp, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _vp, _vp]),
    "w4a16_gemm": (_i32, [_vp, _i64, _vp, _vp, _vp, _vp, _i64, _i64, _i64, _i64, _vp]),
    "nvfp4_get_last_device_error": (_i32, [_vp]),
    "nvfp4_set_wait_limit_ns": (_u64, [_u64]),
    "nvfp4_probe_cvt": (_i32, [_vp, _vp, _vp, _i64, _vp]),
    "nvfp4_probe_bounded_wait": (_i32, [_vp, _u64, _vp]),
}


def lib() -> ctypes.CDLL:
    """Load libnvfp4.so (building it first if the sources are newer)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if os.environ.get("NVFP4_NO_AUTOBUILD") != "1":
                from . import build as _build
                if _build.needs_build():
                    _build.build()
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"libnvfp4.so not found at {LIB_PATH}; run "
                                  "`python -m nvfp4_w4a4_quantized_05_b200.build`")
            L = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in _SIGNATURES.items():
                f = getattr(L, name)
                f.restype = res
                f.argtypes = args
            _lib = L
    return _lib


def _status_string(status: int) -> str:
    try:
        return lib().nvfp4_status_string(int(status)).decode()
    except Exception:  # noqa: BLE001 - only used to format an error message
        return "?"


def _check(status: int, what: str) -> None:
    if status != 0:
        raise Nvfp4Error(status, what)


# ---- raw C ABI (integer addresses) ----------------------------------------------

def nvfp4_status_string(status: int) -> str:
    return lib().nvfp4_status_string(int(status)).decode()


def nvfp4_version() -> str:
    return lib().nvfp4_version().decode()


def nvfp4_codes_bytes(rows: int, k: int) -> int:
    return int(lib().nvfp4_codes_bytes(rows, k))


def nvfp4_scale_bytes(rows: int, k: int) -> int:
    return int(lib().nvfp4_scale_bytes(rows, k))


def nvfp4_grouped_scale_bytes(total_rows: int, num_groups: int, k: int) -> int:
    return int(lib().nvfp4_grouped_scale_bytes(total_rows, num_groups, k))


def nvfp4_workspace_bytes(op: int, rows: int = 0, n: int = 0, k: int = 0, num_groups: int = 0) -> int:
    return int(lib().nvfp4_workspace_bytes(op, rows, n, k, num_groups))


def nvfp4_workspace_init(workspace: int, nbytes: int, stream: int = 0) -> int:
    return lib().nvfp4_workspace_init(workspace, nbytes, stream)


def nvfp4_quantize_act(x, rows, k, ld, group_offsets, num_groups, codes, scales, global_scale, workspace,
                       stream=0) -> int:
    return lib().nvfp4_quantize_act(x, rows, k, ld, group_offsets, num_groups, codes, scales, global_scale,
                                    workspace, stream)


def nvfp4_quantize_act_static(x, rows, k, ld, group_offsets, num_groups, codes, scales, global_scale,
                              stream=0) -> int:
    """nvfp4_quantize_act with the library's fixed device scratch instead of a
    caller workspace (for callers that cannot allocate device memory)."""
    return lib().nvfp4_quantize_act_static(x, rows, k, ld, group_offsets, num_groups, codes, scales,
                                           global_scale, stream)


def nvfp4_quantize_weight_2d(w, n, k, ld, codes, scales, scales_compact, global_scale, workspace, stream=0) -> int:
    return lib().nvfp4_quantize_weight_2d(w, n, k, ld, codes, scales, scales_compact, global_scale, workspace,
                                          stream)


def nvfp4_gemm(a_codes, a_scales, a_global, b_codes, b_scales, b_global, c, ldc, m, n, k, workspace=None,
               stream=0) -> int:
    return lib().nvfp4_gemm(a_codes, a_scales, a_global, b_codes, b_scales, b_global, c, ldc, m, n, k,
                            workspace, stream)


def nvfp4_gemm_emit_scale(a_codes, a_scales, a_global, b_codes, b_scales, b_global, c, ldc, m, n, k,
                          c_global_scale, workspace, stream=0) -> int:
    return lib().nvfp4_gemm_emit_scale(a_codes, a_scales, a_global, b_codes, b_scales, b_global, c, ldc, m, n, k,
                                       c_global_scale, workspace, stream)


def nvfp4_quantize_act_smooth(x, rows, k, ld, smooth, codes, scales, global_scale, workspace, stream=0) -> int:
    return lib().nvfp4_quantize_act_smooth(x, rows, k, ld, smooth, codes, scales, global_scale, workspace, stream)


def nvfp4_quantize_act_scaled(x, rows, k, ld, global_scale, codes, scales, stream=0) -> int:
    return lib().nvfp4_quantize_act_scaled(x, rows, k, ld, global_scale, codes, scales, stream)


def nvfp4_grouped_gemm(a_codes, a_scales, a_global, offsets, num_experts, b_codes, b_scales, b_global, c, n, k,
                       total_rows, workspace=None, stream=0) -> int:
    return lib().nvfp4_grouped_gemm(a_codes, a_scales, a_global, offsets, num_experts, b_codes, b_scales,
                                    b_global, c, n, k, total_rows, workspace, stream)


def nvfp4_quantize_gemm(x, m, k, ldx, b_codes, b_scales, b_global, n, c, ldc, a_codes, a_scales, a_global,
                        workspace, stream=0) -> int:
    return lib().nvfp4_quantize_gemm(x, m, k, ldx, b_codes, b_scales, b_global, n, c, ldc, a_codes, a_scales,
                                     a_global, workspace, stream)


def mxfp4_scale_bytes(rows: int, k: int) -> int:
    return int(lib().mxfp4_scale_bytes(rows, k))


def mxfp4_quantize_act(x, rows, k, ld, codes, scales, stream=0) -> int:
    return lib().mxfp4_quantize_act(x, rows, k, ld, codes, scales, stream)


def mxfp4_gemm(a_codes, a_scales, b_codes, b_scales, c, ldc, m, n, k, workspace=None, stream=0) -> int:
    return lib().mxfp4_gemm(a_codes, a_scales, b_codes, b_scales, c, ldc, m, n, k, workspace, stream)


def w4a16_gemm(a, lda, b_codes, b_scales, b_global, c, ldc, m, n, k, stream=0) -> int:
    return lib().w4a16_gemm(a, lda, b_codes, b_scales, b_global, c, ldc, m, n, k, stream)


def nvfp4_get_last_device_error(stream=0) -> int:
    return lib().nvfp4_get_last_device_error(stream)


def nvfp4_set_wait_limit_ns(limit_ns: int) -> int:
    return int(lib().nvfp4_set_wait_limit_ns(limit_ns))


def nvfp4_probe_cvt(inp, out_e2m1, out_e4m3, n, stream=0) -> int:
    return lib().nvfp4_probe_cvt(inp, out_e2m1, out_e4m3, n, stream)


def nvfp4_probe_bounded_wait(flag, limit_ns, stream=0) -> int:
    return lib().nvfp4_probe_bounded_wait(flag, limit_ns, stream)


# ---- tensor-level helpers (torch for memory and streams) -----------------------------

@dataclass
class NVFP4Tensor:
    """An NVFP4-quantized [rows, k] tensor living on the device."""
    codes: "object"            # uint8 [rows, k/2]
    scales: "object"           # uint8, tiled scale layout
    global_scale: "object"     # float32 [groups]
    rows: int
    k: int
    offsets: Optional["object"] = None   # int32 [groups+1] for grouped tensors


_ws_cache: dict = {}


def _stream_ptr(torch, device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _workspace(torch, device, op: int, groups: int = 0):
    nbytes = nvfp4_workspace_bytes(op, 0, 0, 0, groups)
    if nbytes == 0:
        return None
    key = (device.index, op, groups, torch.cuda.current_stream(device).cuda_stream)
    ws = _ws_cache.get(key)
    if ws is None:
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def _gemm_workspace(torch, device, m: int, n: int, k: int):
    """Scratch for the GEMM's stream-K tail (None when the shape needs none):
    one zeroed buffer per device and stream, grown on demand; every call
    leaves it zeroed for the next."""
    nbytes = nvfp4_workspace_bytes(OP_GEMM, m, n, k, 0)
    if nbytes == 0:
        return None
    key = (device.index, OP_GEMM, 0, torch.cuda.current_stream(device).cuda_stream)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def quantize_act(x, offsets=None, out: Optional[NVFP4Tensor] = None) -> NVFP4Tensor:
    """Dynamic 1D NVFP4 quantization of a BF16 [rows, k] CUDA tensor (one
    global scale, or one per row group when int32 ``offsets`` [G+1] is given).
    ``out`` reuses the buffers of an earlier result of the same shape."""
    import torch
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise TypeError("x must be a 2-D bfloat16 CUDA tensor")
    if x.stride(1) != 1:
        raise ValueError("x must have unit stride along k")
    rows, k = x.shape
    dev = x.device
    groups = 0 if offsets is None else offsets.numel() - 1
    sbytes = nvfp4_scale_bytes(rows, k) if offsets is None else nvfp4_grouped_scale_bytes(rows, groups, k)
    if out is not None:
        if out.rows != rows or out.k != k or out.scales.numel() < sbytes or out.global_scale.numel() < max(1, groups):
            raise ValueError("out does not match the input shape")
        codes, scales, g = out.codes, out.scales, out.global_scale
    else:
        codes = torch.empty((rows, k // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty(sbytes, dtype=torch.uint8, device=dev)
        g = torch.empty(max(1, groups), dtype=torch.float32, device=dev)
    ws = _workspace(torch, dev, OP_QUANTIZE_ACT, groups)
    st = nvfp4_quantize_act(_ptr(x), rows, k, x.stride(0), _ptr(offsets), groups, _ptr(codes), _ptr(scales),
                            _ptr(g), _ptr(ws), _stream_ptr(torch, dev))
    _check(st, "nvfp4_quantize_act")
    if out is not None:
        out.offsets = offsets
        return out
    return NVFP4Tensor(codes, scales, g, rows, k, offsets)


def quantize_weight_2d(w, compact: bool = False, out: Optional[NVFP4Tensor] = None):
    """16x16-block NVFP4 quantization of a BF16 [n, k] CUDA tensor.  Returns
    the NVFP4Tensor (and the [n/16, k/16] compact scales when asked); `out`
    reuses the buffers of an earlier result of the same shape."""
    import torch
    if w.dtype != torch.bfloat16 or w.dim() != 2 or not w.is_cuda:
        raise TypeError("w must be a 2-D bfloat16 CUDA tensor")
    n, k = w.shape
    dev = w.device
    if out is not None:
        if out.rows != n or out.k != k or out.scales.numel() < nvfp4_scale_bytes(n, k) or out.offsets is not None:
            raise ValueError("out does not match the input shape")
        codes, scales, g = out.codes, out.scales, out.global_scale
    else:
        codes = torch.empty((n, k // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty(nvfp4_scale_bytes(n, k), dtype=torch.uint8, device=dev)
        g = torch.empty(1, dtype=torch.float32, device=dev)
    sfc = torch.empty((n // 16, k // 16), dtype=torch.uint8, device=dev) if compact else None
    ws = _workspace(torch, dev, OP_QUANTIZE_WEIGHT_2D)
    st = nvfp4_quantize_weight_2d(_ptr(w), n, k, w.stride(0), _ptr(codes), _ptr(scales), _ptr(sfc), _ptr(g),
                                  _ptr(ws), _stream_ptr(torch, dev))
    _check(st, "nvfp4_quantize_weight_2d")
    t = out if out is not None else NVFP4Tensor(codes, scales, g, n, k)
    return (t, sfc) if compact else t


def gemm(a: NVFP4Tensor, b: NVFP4Tensor, out=None):
    """C[m, n] = A * B^T of two NVFP4 tensors, BF16 output."""
    import torch
    if a.k != b.k:
        raise ValueError("k mismatch")
    dev = a.codes.device
    c = out if out is not None else torch.empty((a.rows, b.rows), dtype=torch.bfloat16, device=dev)
    ws = _gemm_workspace(torch, dev, a.rows, b.rows, a.k)
    st = nvfp4_gemm(_ptr(a.codes), _ptr(a.scales), _ptr(a.global_scale), _ptr(b.codes), _ptr(b.scales),
                    _ptr(b.global_scale), _ptr(c), c.stride(0), a.rows, b.rows, a.k, _ptr(ws), _stream_ptr(torch, dev))
    _check(st, "nvfp4_gemm")
    return c


def gemm_emit_scale(a: NVFP4Tensor, b: NVFP4Tensor, out=None, out_scale=None):
    """gemm() that also returns the global scale of its BF16 output for the
    next dynamic quantizer: (C, g) with g = max|C| / 2688 (1 for an all-zero
    C), a device FP32 [1] tensor."""
    import torch
    if a.k != b.k:
        raise ValueError("k mismatch")
    dev = a.codes.device
    c = out if out is not None else torch.empty((a.rows, b.rows), dtype=torch.bfloat16, device=dev)
    g = out_scale if out_scale is not None else torch.empty(1, dtype=torch.float32, device=dev)
    nbytes = nvfp4_workspace_bytes(OP_GEMM_EMIT_SCALE, a.rows, b.rows, a.k, 0)
    key = (dev.index, OP_GEMM_EMIT_SCALE, 0, torch.cuda.current_stream(dev).cuda_stream)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        _ws_cache[key] = ws
    st = nvfp4_gemm_emit_scale(_ptr(a.codes), _ptr(a.scales), _ptr(a.global_scale), _ptr(b.codes), _ptr(b.scales),
                               _ptr(b.global_scale), _ptr(c), c.stride(0), a.rows, b.rows, a.k, _ptr(g), _ptr(ws),
                               _stream_ptr(torch, dev))
    _check(st, "nvfp4_gemm_emit_scale")
    return c, g


def quantize_act_smooth(x, smooth, out: Optional[NVFP4Tensor] = None) -> NVFP4Tensor:
    """Dynamic 1D quantization of x' = x * smooth[column] (per-channel
    pre-scaling, SmoothQuant style) for a BF16 [rows, k] CUDA tensor and a
    device FP32 [k] factor vector."""
    import torch
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise TypeError("x must be a 2-D bfloat16 CUDA tensor")
    if x.stride(1) != 1:
        raise ValueError("x must have unit stride along k")
    rows, k = x.shape
    if smooth.dtype != torch.float32 or smooth.numel() != k or not smooth.is_cuda:
        raise TypeError("smooth must be a float32 CUDA tensor of k factors")
    dev = x.device
    if out is not None:
        if out.rows != rows or out.k != k or out.scales.numel() < nvfp4_scale_bytes(rows, k) or out.offsets is not None:
            raise ValueError("out does not match the input shape")
        codes, scales, g = out.codes, out.scales, out.global_scale
    else:
        codes = torch.empty((rows, k // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty(nvfp4_scale_bytes(rows, k), dtype=torch.uint8, device=dev)
        g = torch.empty(1, dtype=torch.float32, device=dev)
    ws = _workspace(torch, dev, OP_QUANTIZE_ACT)
    st = nvfp4_quantize_act_smooth(_ptr(x), rows, k, x.stride(0), _ptr(smooth), _ptr(codes), _ptr(scales), _ptr(g),
                                   _ptr(ws), _stream_ptr(torch, dev))
    _check(st, "nvfp4_quantize_act_smooth")
    return out if out is not None else NVFP4Tensor(codes, scales, g, rows, k)


def quantize_act_scaled(x, global_scale, out: Optional[NVFP4Tensor] = None) -> NVFP4Tensor:
    """The quantize pass alone, with a given device FP32 [1] global scale (from
    gemm_emit_scale on the GEMM that produced x)."""
    import torch
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise TypeError("x must be a 2-D bfloat16 CUDA tensor")
    if x.stride(1) != 1:
        raise ValueError("x must have unit stride along k")
    rows, k = x.shape
    dev = x.device
    if out is not None:
        if out.rows != rows or out.k != k or out.scales.numel() < nvfp4_scale_bytes(rows, k) or out.offsets is not None:
            raise ValueError("out does not match the input shape")
        codes, scales = out.codes, out.scales
    else:
        codes = torch.empty((rows, k // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty(nvfp4_scale_bytes(rows, k), dtype=torch.uint8, device=dev)
    st = nvfp4_quantize_act_scaled(_ptr(x), rows, k, x.stride(0), _ptr(global_scale), _ptr(codes), _ptr(scales),
                                   _stream_ptr(torch, dev))
    _check(st, "nvfp4_quantize_act_scaled")
    if out is not None:
        out.global_scale = global_scale
        return out
    return NVFP4Tensor(codes, scales, global_scale, rows, k)


@dataclass
class MXFP4Tensor:
    """An MXFP4-quantized [rows, k] tensor on the device (no global scale)."""
    codes: "object"            # uint8 [rows, k/2]
    scales: "object"           # uint8 E8M0, tiled scale layout, one column per 32 values
    rows: int
    k: int


def quantize_mx(x, out: Optional[MXFP4Tensor] = None) -> MXFP4Tensor:
    """MXFP4 quantization (E8M0 scale per 32 values along k) of a BF16
    [rows, k] CUDA tensor; activations and weights alike."""
    import torch
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise TypeError("x must be a 2-D bfloat16 CUDA tensor")
    if x.stride(1) != 1:
        raise ValueError("x must have unit stride along k")
    rows, k = x.shape
    dev = x.device
    sbytes = mxfp4_scale_bytes(rows, k)
    if out is not None:
        if out.rows != rows or out.k != k or out.scales.numel() < sbytes:
            raise ValueError("out does not match the input shape")
        codes, scales = out.codes, out.scales
    else:
        codes = torch.empty((rows, k // 2), dtype=torch.uint8, device=dev)
        scales = torch.empty(sbytes, dtype=torch.uint8, device=dev)
    st = mxfp4_quantize_act(_ptr(x), rows, k, x.stride(0), _ptr(codes), _ptr(scales), _stream_ptr(torch, dev))
    _check(st, "mxfp4_quantize_act")
    return out if out is not None else MXFP4Tensor(codes, scales, rows, k)


def gemm_mx(a: MXFP4Tensor, b: MXFP4Tensor, out=None):
    """C[m, n] = A * B^T of two MXFP4 tensors, BF16 output."""
    import torch
    if a.k != b.k:
        raise ValueError("k mismatch")
    dev = a.codes.device
    c = out if out is not None else torch.empty((a.rows, b.rows), dtype=torch.bfloat16, device=dev)
    ws = _gemm_workspace(torch, dev, a.rows, b.rows, a.k)
    st = mxfp4_gemm(_ptr(a.codes), _ptr(a.scales), _ptr(b.codes), _ptr(b.scales), _ptr(c), c.stride(0), a.rows,
                    b.rows, a.k, _ptr(ws), _stream_ptr(torch, dev))
    _check(st, "mxfp4_gemm")
    return c


def gemm_w4a16(a, b: NVFP4Tensor, out=None):
    """C[m, n] = A * dequant(B)^T with A a BF16 [m, k] CUDA tensor (m <= 64)
    and B NVFP4 weights; BF16 output."""
    import torch
    if a.dtype != torch.bfloat16 or a.dim() != 2 or not a.is_cuda:
        raise TypeError("a must be a 2-D bfloat16 CUDA tensor")
    if a.stride(1) != 1:
        raise ValueError("a must have unit stride along k")
    m, k = a.shape
    if k != b.k:
        raise ValueError("k mismatch")
    dev = a.device
    c = out if out is not None else torch.empty((m, b.rows), dtype=torch.bfloat16, device=dev)
    st = w4a16_gemm(_ptr(a), a.stride(0), _ptr(b.codes), _ptr(b.scales), _ptr(b.global_scale), _ptr(c), c.stride(0),
                    m, b.rows, k, _stream_ptr(torch, dev))
    _check(st, "w4a16_gemm")
    return c


def grouped_gemm(a: NVFP4Tensor, b_codes, b_scales, b_global, n: int, out=None):
    """Per-expert GEMM: rows of ``a`` grouped by ``a.offsets`` times expert
    weights ``b_codes`` [E, n, k/2] (scales: E blocks of nvfp4_scale_bytes(n, k))."""
    import torch
    if a.offsets is None:
        raise ValueError("a must be a grouped NVFP4 tensor")
    dev = a.codes.device
    E = a.offsets.numel() - 1
    c = out if out is not None else torch.empty((a.rows, n), dtype=torch.bfloat16, device=dev)
    st = nvfp4_grouped_gemm(_ptr(a.codes), _ptr(a.scales), _ptr(a.global_scale), _ptr(a.offsets), E,
                            _ptr(b_codes), _ptr(b_scales), _ptr(b_global), _ptr(c), n, a.k, a.rows, None,
                            _stream_ptr(torch, dev))
    _check(st, "nvfp4_grouped_gemm")
    return c


def _reset_workspaces(device_index: int) -> None:
    """Re-initialise every workspace this module keeps for one device.  A
    bounded wait that ran out leaves a workspace out of step (a grid barrier
    that gave up leaves some CTAs' generation words behind the others', a
    stream-K hand-off may leave a flag set), and every later call on it would
    wait in vain again.  All work on the device is finished first, so no
    kernel still uses one; each is then zeroed, as nvfp4_workspace_init
    would."""
    import torch
    mine = [ws for key, ws in _ws_cache.items() if key[0] == device_index]
    if not mine:
        return
    with torch.cuda.device(device_index):
        torch.cuda.synchronize()
        for ws in mine:
            ws.zero_()
        torch.cuda.synchronize()


def quantize_gemm(x, b: NVFP4Tensor, out=None, qa: Optional[NVFP4Tensor] = None):
    """One W4A4 step: quantize the BF16 [m, k] activations x dynamically and
    multiply by the NVFP4 weights b; returns (C, the quantized activations).
    For m <= 64 the weights start streaming while x is being quantized."""
    import torch
    if x.dtype != torch.bfloat16 or x.dim() != 2 or not x.is_cuda:
        raise TypeError("x must be a 2-D bfloat16 CUDA tensor")
    if x.stride(1) != 1:
        raise ValueError("x must have unit stride along k")
    m, k = x.shape
    if k != b.k:
        raise ValueError("k mismatch")
    dev = x.device
    c = out if out is not None else torch.empty((m, b.rows), dtype=torch.bfloat16, device=dev)
    if qa is None:
        qa = NVFP4Tensor(torch.empty((m, k // 2), dtype=torch.uint8, device=dev),
                         torch.empty(nvfp4_scale_bytes(m, k), dtype=torch.uint8, device=dev),
                         torch.empty(1, dtype=torch.float32, device=dev), m, k)
    nbytes = nvfp4_workspace_bytes(OP_QUANTIZE_GEMM, m, b.rows, k, 0)
    key = (dev.index, OP_QUANTIZE_GEMM, 0, torch.cuda.current_stream(dev).cuda_stream)
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=dev)
        _ws_cache[key] = ws
    st = nvfp4_quantize_gemm(_ptr(x), m, k, x.stride(0), _ptr(b.codes), _ptr(b.scales), _ptr(b.global_scale),
                             b.rows, _ptr(c), c.stride(0), _ptr(qa.codes), _ptr(qa.scales), _ptr(qa.global_scale),
                             _ptr(ws), _stream_ptr(torch, dev))
    _check(st, "nvfp4_quantize_gemm")
    return c, qa


def check_device_error(stream: int = 0) -> None:
    """Raise if a kernel of the library reported a bounded wait that ran out
    on the current device.  Before raising, the workspaces this module cached
    for that device are re-initialised, so the next call starts clean."""
    st = nvfp4_get_last_device_error(stream)
    if st == 5:
        import torch
        _reset_workspaces(torch.cuda.current_device())
    _check(st, "device")
