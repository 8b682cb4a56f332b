"""Helpers shared by the GPU tests: moving BF16 bit patterns and NVFP4
buffers between numpy and the device, and the GEMM tolerance check."""
import numpy as np
import pytest

# GEMM output tolerance (BF16 output of an FP32-accumulated FP4 GEMM against the
# binary64 oracle): relative Frobenius error and max error relative to the row
# maximum of the reference.
REL_FRO_TOL = 2e-3
ROW_MAX_TOL = 1e-2


def device():
    import torch
    if not torch.cuda.is_available():
        pytest.fail("GPU test needs a CUDA device")
    return torch.device("cuda:0")


def bf16_to_device(bits: np.ndarray):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.to(device()).view(torch.bfloat16)


def u8_to_device(a: np.ndarray):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).to(device())


def nvfp4_from_host(codes, sf, g, offsets=None):
    """Upload oracle-produced codes / scales / global scales as an NVFP4Tensor."""
    import torch
    import nvfp4_w4a4_quantized_05_b200 as nv
    rows = codes.shape[0]
    k = codes.shape[1] * 2
    gt = torch.tensor(np.atleast_1d(np.asarray(g, np.float32)), device=device())
    off = None if offsets is None else torch.from_numpy(np.asarray(offsets, np.int32)).to(device())
    return nv.NVFP4Tensor(u8_to_device(codes), u8_to_device(sf), gt, rows, k, off)


def to_host_f64(c):
    return c.float().cpu().numpy().astype(np.float64)


def assert_gemm_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    diff = got - ref
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(diff) / nref if nref > 0 else np.linalg.norm(diff)
    rowmax = np.abs(ref).max(axis=1, keepdims=True)
    worst = np.max(np.abs(diff) - ROW_MAX_TOL * rowmax)
    assert rel <= REL_FRO_TOL, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO_TOL}"
    assert worst <= 0, f"{what}: elementwise error exceeds {ROW_MAX_TOL} x row max by {worst:.3e}"
    return rel
