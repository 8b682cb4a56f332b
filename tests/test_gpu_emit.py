"""The two-phase form of dynamic quantization on a GEMM's output: the GEMM
takes max |C| in its epilogue (nvfp4_gemm_emit_scale) and the quantizer then
runs its quantize pass alone with that global scale
(nvfp4_quantize_act_scaled).  Checked against the one-phase quantizer on the
same output and against the oracle's given-scale quantizer."""
import numpy as np
import pytest

import oracle as O
import workloads as W
import nvfp4_w4a4_quantized_05_b200 as nv
from gpu_util import assert_gemm_close, gemm_refs, nvfp4_from_host, to_host_f64

pytestmark = pytest.mark.gpu


def _sync():
    import torch
    torch.cuda.synchronize()
    nv.check_device_error()


def _operands(m, n, k, seed, scale=1.0, with_ref=False):
    a = W.gaussian_bf16((m, k), seed, 600 + m, scale, outlier_frac=0.01)
    w = W.gaussian_bf16((n, k), seed, 601 + n, 0.02)
    qa = O.quantize_1d(a)
    qw = O.quantize_2d(w) if n % 16 == 0 else O.quantize_1d(w)
    ops = (nvfp4_from_host(*qa), nvfp4_from_host(*qw))
    if with_ref:
        return ops + (gemm_refs(O.dequantize(*qa), O.dequantize(*qw)),)
    return ops


def _expected_g(c):
    import torch
    bits = c.view(torch.int16).cpu().numpy().view(np.uint16)
    amax = float(np.max(np.abs(O.bf16_to_f64(bits)))) if bits.size else 0.0
    return np.float32(O.global_scale(amax)), bits


@pytest.mark.parametrize("m,n,k", [
    (2304, 2336, 512),   # pair tiles with a stream-K tail
    (520, 784, 512),     # pair tiles, ragged m and n (n % 16 == 0: C is quantizable)
    (100, 528, 320),     # 128 x 192 single-SM tiles, ragged rows in the tile
    (64, 608, 256),      # decode tiles (rows 64-127 of the MMA are not output)
    (1, 208, 128),       # one token
])
def test_emit_scale_and_two_phase_quantization(m, n, k):
    import torch
    ta, tw, (ref, absref) = _operands(m, n, k, 7, with_ref=True)
    c_ref = nv.gemm(ta, tw)
    c, g = nv.gemm_emit_scale(ta, tw)
    _sync()
    assert torch.equal(c, c_ref)                      # the same output bits
    assert_gemm_close(to_host_f64(c), ref, absref, k, f"emit {m}x{n}x{k}")
    g_exp, bits = _expected_g(c)
    assert g.cpu().numpy().view(np.uint32)[0] == np.array([g_exp]).view(np.uint32)[0]
    q2 = nv.quantize_act_scaled(c, g)                 # one read of C
    q1 = nv.quantize_act(c)                           # amax pass + quantize pass
    _sync()
    assert torch.equal(q1.global_scale, g)
    assert torch.equal(q1.codes, q2.codes) and torch.equal(q1.scales, q2.scales)
    oc, osf = O.quantize_1d_given_g(bits, float(g_exp))
    assert np.array_equal(q2.codes.cpu().numpy(), oc) and np.array_equal(q2.scales.cpu().numpy(), osf)


def test_emit_scale_repeated_calls_and_zero_output():
    """The running maximum and CTA count return to zero after every call, so
    a smaller output after a larger one gets its own scale; an all-zero C
    gets 1; an empty one too."""
    import torch
    m, n, k = 300, 528, 256
    for it, scale in enumerate([4.0, 0.25, 1.0]):
        ta, tw = _operands(m, n, k, 10 + it, scale)
        c, g = nv.gemm_emit_scale(ta, tw)
        _sync()
        g_exp, _ = _expected_g(c)
        assert g.item() == float(g_exp)
    ta, tw = _operands(m, n, k, 20)
    ta.codes.zero_()
    c, g = nv.gemm_emit_scale(ta, tw)
    _sync()
    assert int(c.view(torch.int16).abs().sum()) == 0 and g.item() == 1.0
    ta0 = nv.NVFP4Tensor(ta.codes[:0], ta.scales, ta.global_scale, 0, k)
    c0, g0 = nv.gemm_emit_scale(ta0, tw, out_scale=torch.full((1,), 7.0, device="cuda"))
    _sync()
    assert c0.numel() == 0 and g0.item() == 1.0


def test_emit_scale_prefill_workload():
    """Full prefill shape: the emitted scale is that of the output."""
    import torch
    a, w = W.prefill(0)
    ta = nv.quantize_act(torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16))
    tw = nv.quantize_weight_2d(torch.from_numpy(w.view(np.int16)).cuda().view(torch.bfloat16))
    c, g = nv.gemm_emit_scale(ta, tw)
    _sync()
    amax = c.float().abs().max().item()
    assert g.item() == float(np.float32(O.global_scale(amax)))
    q1 = nv.quantize_act(c)
    q2 = nv.quantize_act_scaled(c, g)
    _sync()
    assert torch.equal(q1.codes, q2.codes) and torch.equal(q1.scales, q2.scales)
