"""W4A16 on the GPU (BF16 activations x NVFP4 weights dequantized in the
kernel): the output matches the oracle's binary64 product of the BF16
activations and the reconstructed weights within the GEMM tolerance, for
1D- and 2D-quantized weights, ragged weight tiles, partial raw k-tiles, and
the decode workload end to end."""
import numpy as np
import pytest

import oracle as O
import workloads as W
import nvfp4_w4a4_quantized_05_b200 as nv
from gpu_util import assert_gemm_close, bf16_to_device, gemm_refs, nvfp4_from_host, to_host_f64


def _refs(a_bits, wc, wsf, gw):
    """The oracle's W4A16 product and the product of the operands' magnitudes."""
    ref = O.gemm_w4a16_f64(a_bits, wc, wsf, gw)
    _, absref = gemm_refs(O.bf16_to_f64(a_bits), O.dequantize(wc, wsf, gw))
    return ref, absref

pytestmark = pytest.mark.gpu


def _sync():
    import torch
    torch.cuda.synchronize()
    nv.check_device_error()


@pytest.mark.parametrize("m,n,k,two_d", [
    (1, 64, 64, True),        # one raw tile with one 64-wide slice, one ragged weight tile
    (8, 208, 320, True),      # two weight tiles (second starts mid scale block), partial raw k-tile
    (33, 384, 256, False),    # 1D-quantized weights, two full weight tiles
    (64, 144, 576, True),     # 64 tokens, ragged tile, nine slices
    (17, 1000, 1088, False),  # many tiles, partial last raw k-tile
    (64, 4096, 512, True),    # more tiles than SMs
])
def test_w4a16_matches_oracle(m, n, k, two_d):
    a = W.gaussian_bf16((m, k), 0, 960 + m, 1.0, outlier_frac=0.01)
    w = W.gaussian_bf16((n, k), 0, 961 + n, 0.02)
    wc, wsf, gw = O.quantize_2d(w) if two_d else O.quantize_1d(w)
    c = nv.gemm_w4a16(bf16_to_device(a), nvfp4_from_host(wc, wsf, gw))
    _sync()
    ref, absref = _refs(a, wc, wsf, gw)
    assert_gemm_close(to_host_f64(c), ref, absref, k, f"w4a16 {m}x{n}x{k}")


def test_w4a16_output_stride_and_limits():
    import torch
    m, n, k = 5, 96, 128
    a = W.gaussian_bf16((m, k), 0, 970, 1.0)
    wc, wsf, gw = O.quantize_2d(W.gaussian_bf16((n, k), 0, 971, 0.02))
    tw = nvfp4_from_host(wc, wsf, gw)
    out = torch.full((m, 136), 7.0, dtype=torch.bfloat16, device="cuda")
    nv.gemm_w4a16(bf16_to_device(a), tw, out=out[:, :96])
    _sync()
    assert_gemm_close(to_host_f64(out[:, :96]), *_refs(a, wc, wsf, gw), k, "w4a16 strided")
    assert torch.all(out[:, 96:] == 7.0)
    with pytest.raises(nv.Nvfp4Error):                     # m above the decode tile
        nv.gemm_w4a16(bf16_to_device(W.gaussian_bf16((65, k), 0, 972, 1.0)), tw)
    stream = torch.cuda.current_stream().cuda_stream
    assert nv.w4a16_gemm(None, k, None, None, None, None, n, 0, n, k, stream) == 0     # empty


@pytest.mark.parametrize("m", [1, 8, 32, 64])
def test_w4a16_decode_workload(m):
    a, w = W.decode(m)
    wc, wsf, gw = O.quantize_2d(w)
    tw = nv.quantize_weight_2d(bf16_to_device(w))
    c = nv.gemm_w4a16(bf16_to_device(a), tw)
    _sync()
    assert np.array_equal(tw.codes.cpu().numpy(), wc)
    assert_gemm_close(to_host_f64(c), *_refs(a, wc, wsf, gw), 5120, f"w4a16 decode m={m}")


def test_w4a16_strided_activations():
    """Activations as a [48, 512] view of a [48, 640] buffer (row stride 640)."""
    m, n, k = 48, 400, 512
    a_full = W.gaussian_bf16((m, 640), 0, 980, 1.0, outlier_frac=0.01)
    wc, wsf, gw = O.quantize_1d(W.gaussian_bf16((n, k), 0, 981, 0.02))
    c = nv.gemm_w4a16(bf16_to_device(a_full)[:, :k], nvfp4_from_host(wc, wsf, gw))
    _sync()
    ref, absref = _refs(np.ascontiguousarray(a_full[:, :k]), wc, wsf, gw)
    assert_gemm_close(to_host_f64(c), ref, absref, k, "w4a16 strided activations")
