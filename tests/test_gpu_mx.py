"""MXFP4 on the GPU (E2M1 codes, one E8M0 power-of-two scale per 32 values,
no tensor scale): the quantizer's codes and scale bytes equal the oracle's
bit for bit, and the GEMM of oracle-made MXFP4 operands matches the oracle's
binary64 GEMM of the reconstructed operands within the GEMM tolerance, on
single-SM, decode, 2-SM pair and stream-K shapes, with k-tiles that use one
or both of their scale chunks."""
import numpy as np
import pytest

import oracle as O
import workloads as W
import nvfp4_w4a4_quantized_05_b200 as nv
from gpu_util import assert_gemm_close, bf16_to_device, gemm_refs, to_host_f64, u8_to_device

pytestmark = pytest.mark.gpu


def _sync():
    import torch
    torch.cuda.synchronize()
    nv.check_device_error()


def _mx_from_host(codes, sf):
    return nv.MXFP4Tensor(u8_to_device(codes), u8_to_device(sf), codes.shape[0], codes.shape[1] * 2)


def _check_quant(xb):
    q = nv.quantize_mx(bf16_to_device(xb))
    _sync()
    oc, osf = O.quantize_1d_mx(xb)
    assert np.array_equal(q.codes.cpu().numpy(), oc)
    assert np.array_equal(q.scales.cpu().numpy(), osf)


@pytest.mark.parametrize("shape", [(1, 32), (3, 96), (130, 4096), (300, 2080), (129, 960), (64, 5120),
                                   (1000, 1088), (257, 160), (2, 544)])
def test_mx_quantizer_matches_oracle(shape):
    _check_quant(W.laplace_outliers_bf16(shape, 0, 800 + shape[0], outlier_frac=0.01))


def test_mx_quantizer_full_activation_and_weight_workloads():
    _check_quant(W.quant_act(0))          # [8192, 4096] Laplace + outliers
    _check_quant(W.quant_weight(0))       # [14336, 4096] N(0, 0.02)


def test_mx_quantizer_extreme_magnitudes():
    """Blocks whose maxima span the whole BF16 range: subnormal and zero
    maxima (scale byte 0), maxima right at and just above 6 * 2^e, and values
    near the BF16 maximum (scale byte 253)."""
    rng = np.random.default_rng(5)
    rows, k = 256, 512
    e = rng.integers(-133, 128, (rows, k // 32))                 # block exponent
    mant = rng.integers(0, 128, (rows, k)).astype(np.uint32)
    expo = np.clip(np.repeat(e, 32, axis=1) + 127 - rng.integers(0, 12, (rows, k)), 0, 254).astype(np.uint32)
    sign = rng.integers(0, 2, (rows, k)).astype(np.uint32)
    xb = ((sign << 15) | (expo << 7) | mant).astype(np.uint16)   # finite BF16 patterns (exponent field <= 254)
    xb[:8] = 0                                                    # zero blocks
    xb[8, :32] = 0x3FC0                                           # 1.5: maximum exactly 6 * 2^-2
    xb[9, :32] = 0x40C0                                           # 6.0: exactly 6 * 2^0
    xb[10, :32] = 0x40C1                                          # just above 6
    xb[11, :32] = 0x7F7F                                          # BF16 maximum
    xb[12, :32] = 0x0001                                          # smallest subnormal
    _check_quant(xb)


def test_mx_quantizer_limits():
    import torch
    x = bf16_to_device(W.gaussian_bf16((8, 48), 0, 810, 1.0))
    with pytest.raises(nv.Nvfp4Error):                            # k % 32 != 0
        nv.quantize_mx(x)
    stream = torch.cuda.current_stream().cuda_stream
    assert nv.mxfp4_quantize_act(None, 0, 64, 64, None, None, stream) == 0      # empty: nothing touched
    buf = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    xx = bf16_to_device(W.gaussian_bf16((4, 64), 0, 811, 1.0))
    assert nv.mxfp4_quantize_act(xx.data_ptr(), 4, 64, 64, buf.data_ptr() + 8, buf.data_ptr() + 1024,
                                 stream) == 3                     # misaligned codes
    assert nv.mxfp4_scale_bytes(130, 96) == 256 * 4


@pytest.mark.parametrize("m,n,k", [
    (128, 256, 256),     # one full tile
    (200, 320, 320),     # ragged m and n, last k-tile one k-step (half a scale chunk)
    (65, 200, 64),       # smallest k
    (64, 200, 128),      # decode tiles
    (33, 304, 192),      # decode tiles, three k-steps (second scale chunk half used)
    (1, 64, 320),        # single token
    (129, 264, 128),     # 2-SM pair tile with one valid row in its second half
    (520, 776, 512),     # pair tiles, ragged edges
    (1000, 2072, 576),   # many pair tiles, partial last k-tile
    (2304, 2336, 512),   # every tile shared out stream-K
    (2350, 4104, 768),   # stream-K tiles at both ragged edges
])
def test_mx_gemm_matches_oracle(m, n, k):
    a = W.gaussian_bf16((m, k), 0, 900 + m, 1.0, outlier_frac=0.01)
    w = W.gaussian_bf16((n, k), 0, 901 + n, 0.02)
    ac, asf = O.quantize_1d_mx(a)
    wc, wsf = O.quantize_1d_mx(w)
    c = nv.gemm_mx(_mx_from_host(ac, asf), _mx_from_host(wc, wsf))
    _sync()
    ref, absref = gemm_refs(O.dequantize_mx(ac, asf), O.dequantize_mx(wc, wsf))
    assert_gemm_close(to_host_f64(c), ref, absref, k, f"mx {m}x{n}x{k}")


def test_mx_gemm_stream_k_workspace_and_none():
    import torch
    m, n, k = 2304, 2336, 512
    a = W.gaussian_bf16((m, k), 0, 930, 1.0, outlier_frac=0.01)
    w = W.gaussian_bf16((n, k), 0, 931, 0.02)
    ac, asf = O.quantize_1d_mx(a)
    wc, wsf = O.quantize_1d_mx(w)
    ta, tw = _mx_from_host(ac, asf), _mx_from_host(wc, wsf)
    ref, absref = gemm_refs(O.dequantize_mx(ac, asf), O.dequantize_mx(wc, wsf))
    ws = torch.zeros(nv.nvfp4_workspace_bytes(nv.OP_GEMM, m, n, k, 0), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for ws_ptr in (ws.data_ptr(), None, ws.data_ptr()):
        c = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device="cuda")
        st = nv.mxfp4_gemm(ta.codes.data_ptr(), ta.scales.data_ptr(), tw.codes.data_ptr(), tw.scales.data_ptr(),
                           c.data_ptr(), n, m, n, k, ws_ptr, stream)
        assert st == 0
        _sync()
        assert int(ws[:32768].to(torch.int64).sum()) == 0
        assert_gemm_close(to_host_f64(c), ref, absref, k, f"mx stream-K, workspace {ws_ptr is not None}")


def test_mx_prefill_workload_end_to_end():
    """Prefill shape: A [4096, 4096] and W [14336, 4096] quantized to MXFP4 on
    the GPU (bit-exact against the oracle), then the GEMM on sampled rows."""
    a, w = W.prefill(0)
    ta = nv.quantize_mx(bf16_to_device(a))
    tw = nv.quantize_mx(bf16_to_device(w))
    c = nv.gemm_mx(ta, tw)
    _sync()
    ac, asf = O.quantize_1d_mx(a)
    wc, wsf = O.quantize_1d_mx(w)
    assert np.array_equal(ta.codes.cpu().numpy(), ac) and np.array_equal(ta.scales.cpu().numpy(), asf)
    assert np.array_equal(tw.codes.cpu().numpy(), wc) and np.array_equal(tw.scales.cpu().numpy(), wsf)
    rows = np.unique(np.concatenate([np.arange(0, 4096, 128), np.arange(127, 4096, 128)[::4], [1, 2049, 4095]]))
    ref, absref = gemm_refs(O.dequantize_mx(ac, asf)[rows], O.dequantize_mx(wc, wsf))
    assert_gemm_close(to_host_f64(c[rows.tolist()]), ref, absref, 4096, "mx prefill")


def test_mx_decode_workload():
    """Decode shape m = 8: K = 5120, N = 25600."""
    a, w = W.decode(8)
    ac, asf = O.quantize_1d_mx(a)
    wc, wsf = O.quantize_1d_mx(w)
    c = nv.gemm_mx(nv.quantize_mx(bf16_to_device(a)), nv.quantize_mx(bf16_to_device(w)))
    _sync()
    ref, absref = gemm_refs(O.dequantize_mx(ac, asf), O.dequantize_mx(wc, wsf))
    assert_gemm_close(to_host_f64(c), ref, absref, 5120, "mx decode")


def test_mx_strided_input_zero_tensor_and_empty_gemm():
    import torch
    # a [300, 1088] view of a wider buffer (row stride 1152 elements)
    xb = W.laplace_outliers_bf16((300, 1152), 0, 820, outlier_frac=0.01)
    x = bf16_to_device(xb)[:, :1088]
    q = nv.quantize_mx(x)
    _sync()
    oc, osf = O.quantize_1d_mx(np.ascontiguousarray(xb[:, :1088]))
    assert np.array_equal(q.codes.cpu().numpy(), oc) and np.array_equal(q.scales.cpu().numpy(), osf)
    # all-zero tensor: zero codes, zero scale bytes
    z = nv.quantize_mx(torch.zeros((130, 256), dtype=torch.bfloat16, device="cuda"))
    _sync()
    assert not z.codes.any() and not z.scales.any()
    # empty GEMM and a GEMM into a strided output
    w = W.gaussian_bf16((96, 256), 0, 821, 0.02)
    wc, wsf = O.quantize_1d_mx(w)
    tw = _mx_from_host(wc, wsf)
    ta0 = nv.MXFP4Tensor(torch.empty((0, 128), dtype=torch.uint8, device="cuda"),
                         torch.empty(0, dtype=torch.uint8, device="cuda"), 0, 256)
    c0 = nv.gemm_mx(ta0, tw)
    a = W.gaussian_bf16((40, 256), 0, 822, 1.0)
    ac, asf = O.quantize_1d_mx(a)
    out = torch.full((40, 104), 7.0, dtype=torch.bfloat16, device="cuda")
    nv.gemm_mx(_mx_from_host(ac, asf), tw, out=out[:, :96])
    _sync()
    assert c0.shape == (0, 96)
    ref, absref = gemm_refs(O.dequantize_mx(ac, asf), O.dequantize_mx(wc, wsf))
    assert_gemm_close(to_host_f64(out[:, :96]), ref, absref, 256, "mx strided")
    assert torch.all(out[:, 96:] == 7.0)
