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


def gemm_refs(a_hat: np.ndarray, w_hat: np.ndarray):
    """The oracle's binary64 product of the reconstructed operands and the
    same product of their magnitudes (the bound of the summation error)."""
    import oracle as O
    return O.gemm_f64(a_hat, w_hat), O.gemm_f64(np.abs(a_hat), np.abs(w_hat))


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of BF16 numbers at |v| (8 significant bits): the binary32
    spacing times 2^16."""
    return np.spacing(np.abs(v).astype(np.float32)).astype(np.float64) * 65536.0


def assert_gemm_close(got: np.ndarray, ref: np.ndarray, absref: np.ndarray, k: int, what: str = ""):
    """The stated tolerance (relative Frobenius error and the error relative
    to each row's maximum), and element by element:
        |got - ref| <= ulp_bf16(max(|got|, |ref|)) + (k + 2) 2^-23 sum|a||w|.
    The products of reconstructed NVFP4 / MXFP4 / BF16 x NVFP4 operands are
    exact in binary32, so the FP32 accumulation of k of them in any order,
    with round-to-nearest or truncating additions (unit 2^-23), errs by at
    most (k - 1) 2^-23 sum|a||w|; the product of the global scales and the
    epilogue multiply add two more units; the BF16 output rounding adds at
    most half an ulp (a whole one is allowed: the rounding of the FP32 value
    can land on either side of ref)."""
    diff = got - ref
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(diff) / nref if nref > 0 else np.linalg.norm(diff)
    rowmax = np.abs(ref).max(axis=1, keepdims=True)
    worst = np.max(np.abs(diff) - ROW_MAX_TOL * rowmax)
    assert rel <= REL_FRO_TOL, f"{what}: relative Frobenius error {rel:.3e} > {REL_FRO_TOL}"
    assert worst <= 0, f"{what}: elementwise error exceeds {ROW_MAX_TOL} x row max by {worst:.3e}"
    bound = bf16_ulp(np.maximum(np.abs(got), np.abs(ref))) + (k + 2) * 2.0 ** -23 * absref
    excess = np.abs(diff) - bound
    bad = np.argwhere(excess > 0)
    assert bad.size == 0, (f"{what}: {len(bad)} outputs beyond one BF16 ulp plus the FP32 summation bound, "
                           f"first at {tuple(bad[0])}: got {got[tuple(bad[0])]!r}, ref {ref[tuple(bad[0])]!r}, "
                           f"bound {bound[tuple(bad[0])]:.3e}")
    return rel
