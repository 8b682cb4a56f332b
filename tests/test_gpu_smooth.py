"""Per-channel pre-scaling folded into the activation quantizer (SmoothQuant
style): the GPU quantizes x' = x * s[column] bit-exactly like the oracle, and
the GEMM of the pre-scaled activations with inverse-scaled weights matches
the oracle's binary64 GEMM of the same reconstructed operands."""
import numpy as np
import pytest

import oracle as O
import workloads as W
import nvfp4_w4a4_quantized_05_b200 as nv
from gpu_util import assert_gemm_close, bf16_to_device, gemm_refs, to_host_f64

pytestmark = pytest.mark.gpu


def _factors(k, seed):
    rng = np.random.default_rng(seed)
    return np.exp2(rng.uniform(-3.0, 3.0, k)).astype(np.float32)     # log-uniform in [1/8, 8]


def _check(xb, s):
    import torch
    q = nv.quantize_act_smooth(bf16_to_device(xb), torch.from_numpy(s).cuda())
    torch.cuda.synchronize()
    nv.check_device_error()
    oc, osf, og = O.quantize_1d_smooth(xb, s)
    assert q.global_scale.cpu().numpy().view(np.uint32)[0] == np.array([og], np.float32).view(np.uint32)[0]
    assert np.array_equal(q.codes.cpu().numpy(), oc)
    assert np.array_equal(q.scales.cpu().numpy(), osf)


@pytest.mark.parametrize("shape", [(300, 2048), (129, 960), (64, 5120), (1, 6144), (200, 4160), (1000, 1088)])
def test_smooth_quantizer_matches_oracle(shape):
    xb = W.gaussian_bf16(shape, 0, 700 + shape[0], 1.0, outlier_frac=0.01)
    _check(xb, _factors(shape[1], shape[0]))


def test_smooth_quantizer_full_activation_workload():
    xb = W.quant_act(0)                                    # [8192, 4096] Laplace + outliers
    _check(xb, _factors(4096, 1))


def test_smooth_unit_factors_equal_plain_quantizer_and_limits():
    import torch
    xb = W.gaussian_bf16((256, 1024), 0, 711, 1.0)
    x = bf16_to_device(xb)
    q1 = nv.quantize_act_smooth(x, torch.ones(1024, device="cuda"))
    q0 = nv.quantize_act(x)
    torch.cuda.synchronize()
    assert torch.equal(q1.codes, q0.codes) and torch.equal(q1.scales, q0.scales)
    assert torch.equal(q1.global_scale, q0.global_scale)
    with pytest.raises(nv.Nvfp4Error):                     # k above the factor buffer
        nv.quantize_act_smooth(bf16_to_device(W.gaussian_bf16((4, 6208), 0, 712, 1.0)),
                               torch.ones(6208, device="cuda"))


def test_smooth_gemm_end_to_end():
    """X' = X s quantized on the fly, W' = bf16(W / s) quantized offline (2D):
    the GEMM matches the oracle's binary64 GEMM of the same reconstructed
    operands.  (With random factors the product is a poor approximation of
    X W^T; SmoothQuant picks the factors from the data.)"""
    import torch
    m, n, k = 256, 512, 1024
    xb = W.gaussian_bf16((m, k), 0, 720, 1.0, outlier_frac=0.01)
    wb = W.gaussian_bf16((n, k), 0, 721, 0.02)
    s = _factors(k, 5)
    w_scaled = O.bf16_to_f64(wb) / s[None, :].astype(np.float64)
    wsb = (w_scaled.astype(np.float32).view(np.uint32) + 0x7FFF + ((w_scaled.astype(np.float32).view(np.uint32) >> 16) & 1)) >> 16
    wsb = wsb.astype(np.uint16)                            # W / s rounded to BF16 (nearest even)
    ta = nv.quantize_act_smooth(bf16_to_device(xb), torch.from_numpy(s).cuda())
    tw = nv.quantize_weight_2d(bf16_to_device(wsb))
    c = nv.gemm(ta, tw)
    torch.cuda.synchronize()
    nv.check_device_error()
    ac, asf, ga = O.quantize_1d_smooth(xb, s)
    wc, wsf, gw = O.quantize_2d(wsb)
    ref, absref = gemm_refs(O.dequantize(ac, asf, ga), O.dequantize(wc, wsf, gw))
    assert_gemm_close(to_host_f64(c), ref, absref, k, "smooth")
