"""GPU GEMM parity: the tcgen05 block-scaled GEMM against the binary64 oracle
GEMM over the reconstructed operands, within the stated tolerance
(relative Frobenius <= 2e-3, max |error| <= 1e-2 x row max |ref|) and,
element by element, within one BF16 ulp plus the FP32 summation bound
(gpu_util.assert_gemm_close).  Small cases compare every output; the
full-size prefill / decode / MoE workloads compare sampled rows the oracle
computes one by one.  Every operand of a reference is the oracle's."""
import numpy as np
import pytest

import oracle as O
import workloads as W
import nvfp4_w4a4_quantized_05_b200 as nv
from gpu_util import assert_gemm_close, bf16_to_device, gemm_refs, nvfp4_from_host, to_host_f64

pytestmark = pytest.mark.gpu


def _sync():
    import torch
    torch.cuda.synchronize()
    nv.check_device_error()


def _oracle_operands(m, n, k, seed):
    a = W.gaussian_bf16((m, k), seed, 300 + m, 1.0, outlier_frac=0.01)
    w = W.gaussian_bf16((n, k), seed, 301 + n, 0.02)
    qa = O.quantize_1d(a)
    qw = O.quantize_2d(w) if n % 16 == 0 else O.quantize_1d(w)
    return qa, qw


def test_tiny_workload_end_to_end():
    a, w = W.tiny(0)
    ta = nv.quantize_act(bf16_to_device(a))
    tw = nv.quantize_weight_2d(bf16_to_device(w))
    c = nv.gemm(ta, tw)
    _sync()
    ac, asf, ga = O.quantize_1d(a)
    wc, wsf, gw = O.quantize_2d(w)
    assert np.array_equal(ta.codes.cpu().numpy(), ac) and np.array_equal(tw.codes.cpu().numpy(), wc)
    ref, absref = gemm_refs(O.dequantize(ac, asf, ga), O.dequantize(wc, wsf, gw))
    got = to_host_f64(c)
    assert_gemm_close(got, ref, absref, 256, "tiny")
    # the exact integer sum, scaled, rounds to within one BF16 step of the output
    exact = O.gemm_exact_i64(ac, asf, wc, wsf, 256).astype(np.float64) * 2.0 ** -20 * float(np.float32(ga) * np.float32(gw))
    assert np.all(np.abs(got - exact) <= 2.0 ** -7 * np.abs(exact) + 1e-30)


@pytest.mark.parametrize("m,n,k", [
    (128, 256, 256),     # one full tile
    (200, 320, 320),     # ragged m, ragged n tile, partial last k-tile
    (256, 512, 1024),    # several tiles
    (65, 200, 64),       # smallest k; just above the decode-tile threshold (m <= 64)
    (64, 200, 128),      # decode tiles: 64 token rows, ragged second weight tile
    (33, 304, 192),      # decode tiles with 33 tokens
    (17, 136, 64),       # decode tiles, one weight tile of 136 rows
    (16, 64, 256),       # decode tiles, 16 tokens x 64 weight rows
    (1, 64, 320),        # single token
    (300, 16, 448),      # narrow n
    (129, 264, 128),     # 2-SM pair tile with one valid row in its second half
    (520, 776, 512),     # pair tiles: ragged m (3 row tiles) and n (4th column tile 8 wide)
    (1000, 2072, 576),   # many pair tiles, both edges ragged, partial last k-tile
    (2304, 2336, 256),   # more pair tiles than resident pairs, one k-tile: a partial second wave
    (2560, 4000, 128),   # ditto, with the last wave at the ragged n edge
    (2304, 2336, 512),   # 90 pair tiles, two k-tiles: every tile shared out stream-K
    (4608, 4352, 1088),  # 306 tiles: 222 whole, the k-tiles of 84 shared out; partial last k-tile
    (2350, 4104, 768),   # 170 tiles: stream-K tiles at both ragged edges (last column tile 8 wide)
])
def test_gemm_matches_oracle(m, n, k):
    (ac, asf, ga), (wc, wsf, gw) = _oracle_operands(m, n, k, 0)
    c = nv.gemm(nvfp4_from_host(ac, asf, ga), nvfp4_from_host(wc, wsf, gw))
    _sync()
    ref, absref = gemm_refs(O.dequantize(ac, asf, ga), O.dequantize(wc, wsf, gw))
    assert_gemm_close(to_host_f64(c), ref, absref, k, f"{m}x{n}x{k}")


def test_gemm_output_row_stride():
    import torch
    (ac, asf, ga), (wc, wsf, gw) = _oracle_operands(150, 96, 128, 1)
    out = torch.full((150, 136), 7.0, dtype=torch.bfloat16, device="cuda")
    nv.gemm(nvfp4_from_host(ac, asf, ga), nvfp4_from_host(wc, wsf, gw), out=out[:, :96])
    _sync()
    ref, absref = gemm_refs(O.dequantize(ac, asf, ga), O.dequantize(wc, wsf, gw))
    assert_gemm_close(to_host_f64(out[:, :96]), ref, absref, 128, "strided")
    assert torch.all(out[:, 96:] == 7.0)                  # nothing written past n


def test_stream_k_workspace_reuse_and_without_workspace():
    """A shape that splits tiles between pairs: repeated calls on one
    workspace, and a call with no workspace (every tile whole), all match the
    oracle; the workspace counters return to zero after each call."""
    import torch
    m, n, k = 2304, 2336, 512
    need = nv.nvfp4_workspace_bytes(nv.OP_GEMM, m, n, k, 0)
    assert need > 0
    assert nv.nvfp4_workspace_bytes(nv.OP_GEMM, 64, n, k, 0) == 0          # decode tiles: none
    (ac, asf, ga), (wc, wsf, gw) = _oracle_operands(m, n, k, 3)
    ta, tw = nvfp4_from_host(ac, asf, ga), nvfp4_from_host(wc, wsf, gw)
    ref, absref = gemm_refs(O.dequantize(ac, asf, ga), O.dequantize(wc, wsf, gw))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    for it in range(3):
        c = torch.full((m, n), float("nan"), dtype=torch.bfloat16, device="cuda")
        for ws_ptr in (ws.data_ptr(), None):
            st = nv.nvfp4_gemm(ta.codes.data_ptr(), ta.scales.data_ptr(), ta.global_scale.data_ptr(),
                               tw.codes.data_ptr(), tw.scales.data_ptr(), tw.global_scale.data_ptr(), c.data_ptr(),
                               n, m, n, k, ws_ptr, stream)
            assert st == 0
            _sync()
            assert int(ws[:32768].to(torch.int64).sum()) == 0
            assert_gemm_close(to_host_f64(c), ref, absref, k, f"stream-K call {it}, workspace {ws_ptr is not None}")
    # a misaligned workspace is refused before anything runs
    assert nv.nvfp4_gemm(ta.codes.data_ptr(), ta.scales.data_ptr(), ta.global_scale.data_ptr(),
                         tw.codes.data_ptr(), tw.scales.data_ptr(), tw.global_scale.data_ptr(), c.data_ptr(),
                         n, m, n, k, ws.data_ptr() + 4, stream) == 3     # NVFP4_ERR_MISALIGNED


@pytest.fixture(scope="module")
def prefill_case():
    a, w = W.prefill(0)
    return a, w, O.quantize_1d(a), O.quantize_2d(w)


def test_prefill_workload_sampled_rows(prefill_case):
    """Quantize on the GPU, check both operands against the oracle's bit for
    bit, then the GEMM on sampled rows against the oracle's operands."""
    a, w, (ac, asf, ga), (wc, wsf, gw) = prefill_case
    ta = nv.quantize_act(bf16_to_device(a))
    tw = nv.quantize_weight_2d(bf16_to_device(w))
    c = nv.gemm(ta, tw)
    _sync()
    assert np.array_equal(ta.codes.cpu().numpy(), ac) and np.array_equal(ta.scales.cpu().numpy(), asf)
    assert np.array_equal(tw.codes.cpu().numpy(), wc) and np.array_equal(tw.scales.cpu().numpy(), wsf)
    assert ta.global_scale.item() == float(np.float32(ga)) and tw.global_scale.item() == float(np.float32(gw))
    rows = np.unique(np.concatenate([np.arange(0, 4096, 128), np.arange(127, 4096, 128)[::4], [1, 2049, 4095]]))
    ref, absref = gemm_refs(O.dequantize(ac, asf, ga)[rows], O.dequantize(wc, wsf, gw))
    got = to_host_f64(c[rows.tolist()])
    assert_gemm_close(got, ref, absref, 4096, "prefill")


@pytest.fixture(scope="module")
def decode_weights():
    _, w = W.decode(1)
    wc, wsf, gw = O.quantize_2d(w)
    return w, (wc, wsf, gw), O.dequantize(wc, wsf, gw)


@pytest.mark.parametrize("m", [1, 8, 32, 64])
def test_decode_workload_full(m, decode_weights):
    w, (wc, wsf, gw), wh = decode_weights
    a, _ = W.decode(m)
    ac, asf, ga = O.quantize_1d(a)
    ta = nv.quantize_act(bf16_to_device(a))
    c = nv.gemm(ta, nvfp4_from_host(wc, wsf, gw))
    _sync()
    assert np.array_equal(ta.codes.cpu().numpy(), ac)
    ref, absref = gemm_refs(O.dequantize(ac, asf, ga), wh)
    assert_gemm_close(to_host_f64(c), ref, absref, 5120, f"decode m={m}")


@pytest.mark.parametrize("sizes,k,n", [
    ([0, 5, 128, 130, 0, 1, 257, 64], 320, 200),               # small experts: 128 x 192 single-SM tiles
    # experts of >= 192 rows on average: 256 x 256 pair tiles; an expert of 129
    # rows (one valid row in the second half), of exactly 256, of 1, of 0, and
    # ragged n (last column tile 8 wide) with a partial last k-tile
    ([300, 0, 129, 256, 511, 1, 385, 200], 576, 520),
    # n % 256 == 0: the swapped kernel (weights on the 256-row side, tokens
    # on N in tiles of 256; a last part of <= 64 tokens rides on the tile
    # before it as a second MMA, a larger one is a tile of its own, each
    # rounded up to 32 tokens): experts of 0, 1, 16, 31, 32, 33 ... 700 rows
    # (one, two and three token tiles; parts of every box height; riding
    # parts of 1 and 44 tokens; partial last 32-token chunks), a partial last
    # k-tile (k = 320) and two weight tiles
    ([256] * 3 + [255, 257], 1024, 256),
    ([0, 1, 16, 31, 32, 33, 100, 128, 129, 255, 256, 257, 300, 511, 512, 513, 700, 0], 320, 512),
    ([40, 97, 64], 2048, 1536),
])
def test_grouped_gemm_ragged_experts(sizes, k, n):
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    a = W.gaussian_bf16((int(off[-1]), k), 0, 44, 1.0, outlier_frac=0.01)
    ac, asf, ga = O.quantize_1d_grouped(a, off)
    E = len(sizes)
    wq = [O.quantize_1d(W.gaussian_bf16((n, k), 0, 500 + e, 0.02)) for e in range(E)]
    wc = np.stack([q[0] for q in wq])
    wsf = np.concatenate([q[1] for q in wq])
    gw = np.array([q[2] for q in wq], np.float32)
    ta = nvfp4_from_host(ac, np.concatenate([asf, np.zeros(nv.nvfp4_grouped_scale_bytes(int(off[-1]), E, k) - asf.size, np.uint8)]), ga, off)
    from gpu_util import u8_to_device
    import torch
    c = nv.grouped_gemm(ta, u8_to_device(wc), u8_to_device(wsf), torch.tensor(gw, device="cuda"), n)
    _sync()
    ah = O.dequantize_grouped(ac, asf, ga, off)
    got = to_host_f64(c)
    for e in range(E):
        r0, r1 = off[e], off[e + 1]
        if r1 > r0:
            ref, absref = gemm_refs(ah[r0:r1], O.dequantize(wq[e][0], wq[e][1], wq[e][2]))
            assert_gemm_close(got[r0:r1], ref, absref, k, f"expert {e}")


def test_moe_workload_sampled_rows():
    """The MoE workload end to end on the GPU: grouped activation
    quantization and each expert's 2D weight quantization are checked against
    the oracle's bit for bit, then the grouped GEMM on sampled rows of every
    expert against the binary64 product of the oracle's operands."""
    import torch
    a, off, w = W.moe(0)
    E, N, K = w.shape
    ta = nv.quantize_act(bf16_to_device(a), torch.from_numpy(off).cuda())
    wdev = bf16_to_device(w.reshape(E * N, K))
    tw = [nv.quantize_weight_2d(wdev[e * N:(e + 1) * N]) for e in range(E)]
    b_codes = torch.stack([t.codes for t in tw])
    b_scales = torch.cat([t.scales for t in tw])
    b_global = torch.cat([t.global_scale for t in tw])
    c = nv.grouped_gemm(ta, b_codes, b_scales, b_global, N)
    _sync()
    ac, asf, ga = O.quantize_1d_grouped(a, off)
    assert np.array_equal(ta.codes.cpu().numpy(), ac)
    assert np.array_equal(ta.scales.cpu().numpy()[:asf.size], asf)
    assert np.array_equal(ta.global_scale.cpu().numpy().view(np.uint32), np.asarray(ga, np.float32).view(np.uint32))
    wq = [O.quantize_2d(np.ascontiguousarray(w[e])) for e in range(E)]
    sbytes = nv.nvfp4_scale_bytes(N, K)
    dev_codes, dev_scales, dev_g = b_codes.cpu().numpy(), b_scales.cpu().numpy(), b_global.cpu().numpy()
    for e in range(E):
        assert np.array_equal(dev_codes[e], wq[e][0]), f"expert {e} weight codes"
        assert np.array_equal(dev_scales[e * sbytes:(e + 1) * sbytes], wq[e][1]), f"expert {e} weight scales"
        assert dev_g[e] == np.float32(wq[e][2]), f"expert {e} weight global scale"
    row0 = 0
    got = to_host_f64(c)
    for e in range(E):
        r0, r1 = int(off[e]), int(off[e + 1])
        n_e = r1 - r0
        if n_e:
            sel = np.unique([r0, r0 + n_e // 2, r1 - 1, min(r1 - 1, r0 + 127), min(r1 - 1, r0 + 128)])
            a_hat = O.dequantize(ac[r0:r1], asf, float(ga[e]), sf_row0=row0, k=K)[sel - r0]
            w_hat = O.dequantize(*wq[e])
            ref, absref = gemm_refs(a_hat, w_hat)
            assert_gemm_close(got[sel], ref, absref, K, f"moe expert {e}")
        row0 += O.scale_rows(n_e)


@pytest.mark.parametrize("m,n,k", [(384, 256, 1024), (200, 272, 320)])
def test_scale_layout_read_by_library_block_scaled_gemm(m, n, k):
    """The scale bytes the quantizers write, unmodified, read by another
    block-scaled NVFP4 GEMM on this GPU (torch's scaled_mm: E2M1 operands,
    E4M3 scales per 16 values, 32 x 4 x 4 swizzled scale layout): its output
    must be the oracle's product of the block-scaled operands (no global
    scales) to the GEMM tolerance.  A layout this library only agreed with
    itself on would fail here.  Several 128 x 4 scale tiles along both rows
    and columns; the second shape has padded rows and columns."""
    import torch
    import torch.nn.functional as F
    a = W.gaussian_bf16((m, k), 0, 1300 + m, 1.0, outlier_frac=0.01)
    w = W.gaussian_bf16((n, k), 0, 1301 + n, 0.02)
    ta = nv.quantize_act(bf16_to_device(a))
    tw = nv.quantize_weight_2d(bf16_to_device(w))
    _sync()
    ac, asf, _ = O.quantize_1d(a)
    wc, wsf, _ = O.quantize_2d(w)
    assert np.array_equal(ta.codes.cpu().numpy(), ac) and np.array_equal(ta.scales.cpu().numpy(), asf)
    assert np.array_equal(tw.codes.cpu().numpy(), wc) and np.array_equal(tw.scales.cpu().numpy(), wsf)
    c = F.scaled_mm(ta.codes.view(torch.float4_e2m1fn_x2), tw.codes.view(torch.float4_e2m1fn_x2).t(),
                    ta.scales.view(torch.float8_e4m3fn), F.ScalingType.BlockWise1x16,
                    tw.scales.view(torch.float8_e4m3fn), F.ScalingType.BlockWise1x16,
                    swizzle_a=F.SwizzleType.SWIZZLE_32_4_4, swizzle_b=F.SwizzleType.SWIZZLE_32_4_4,
                    output_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    ref, absref = gemm_refs(O.dequantize(ac, asf, 1.0), O.dequantize(wc, wsf, 1.0))
    assert_gemm_close(to_host_f64(c), ref, absref, k, f"library GEMM on our scale bytes {m}x{n}x{k}")


@pytest.mark.parametrize("m,n,k", [(1, 25600, 5120), (8, 208, 320), (33, 416, 1024), (64, 25600, 5120), (64, 200, 64),
                                   (4, 28608, 128), (200, 528, 576)])
def test_quantize_gemm_equals_separate_calls(m, n, k):
    """nvfp4_quantize_gemm (dynamic quantization, then the GEMM, the weights
    streaming early for m <= 64) gives the same quantized activations and the
    same output bits as nvfp4_quantize_act followed by nvfp4_gemm, twice in a
    row on one workspace, and the oracle's product within the bound."""
    import torch
    a = W.gaussian_bf16((m, k), 0, 1400 + m, 1.0, outlier_frac=0.01)
    w = W.gaussian_bf16((n, k), 0, 1401 + n, 0.02)
    wq = O.quantize_2d(w) if n % 16 == 0 else O.quantize_1d(w)
    tw = nvfp4_from_host(*wq)
    x = bf16_to_device(a)
    for _ in range(2):
        c1, qa1 = nv.quantize_gemm(x, tw)
        qa2 = nv.quantize_act(x)
        c2 = nv.gemm(qa2, tw)
        _sync()
        assert torch.equal(qa1.codes, qa2.codes) and torch.equal(qa1.scales, qa2.scales)
        assert torch.equal(qa1.global_scale, qa2.global_scale)
        assert torch.equal(c1, c2)
    ac, asf, ga = O.quantize_1d(a)
    assert np.array_equal(qa1.codes.cpu().numpy(), ac)
    ref, absref = gemm_refs(O.dequantize(ac, asf, ga), O.dequantize(*wq))
    assert_gemm_close(to_host_f64(c1), ref, absref, k, f"quantize_gemm {m}x{n}x{k}")


def _check_qa_against_oracle(a_host, qa):
    oc, osf, og = O.quantize_1d(a_host)
    assert np.array_equal(qa.codes.cpu().numpy(), oc)
    assert np.array_equal(qa.scales.cpu().numpy(), osf)
    assert qa.global_scale.cpu().numpy().view(np.uint32)[0] == np.array([np.float32(og)]).view(np.uint32)[0]
    return oc, osf, og


@pytest.mark.parametrize("m,n,k", [(64, 208, 8192), (5, 400, 4096), (64, 416, 64), (40, 27008, 1024)])
def test_quantize_gemm_decode_shapes(m, n, k):
    """Decode-sized nvfp4_quantize_gemm (two-kernel quantizer, then the GEMM
    streaming its first weight stages early) on long k (8192: 32 k-tiles,
    more stages than the early weight stream covers), one partial k-tile
    (k = 64), a two-tile n and a 141-tile n.  Codes, scale bytes (pad rows
    zero) and g are the oracle's bit for bit; C is within the bound."""
    a = W.gaussian_bf16((m, k), 2, 1500 + m, 1.0, outlier_frac=0.01)
    w = W.gaussian_bf16((n, k), 2, 1501 + n, 0.02)
    wq = O.quantize_2d(w)
    tw = nvfp4_from_host(*wq)
    c, qa = nv.quantize_gemm(bf16_to_device(a), tw)
    _sync()
    ac, asf, ga = _check_qa_against_oracle(a, qa)
    ref, absref = gemm_refs(O.dequantize(ac, asf, ga), O.dequantize(*wq))
    assert_gemm_close(to_host_f64(c), ref, absref, k, f"quantize_gemm {m}x{n}x{k}")


def test_quantize_gemm_decode_call_sequence_on_one_workspace():
    """One workspace through calls whose GEMM grids differ (n = 208: 2 CTAs,
    n = 25600: 134), whose m changes, and whose amax goes up, down, to a tiny
    global scale (g < 2^-64, the scaled reciprocal) and to zero (g = 1): the
    quantizer's amax words come back to zero after every call, so each
    call's quantization is the oracle's for its own x, and C equals
    nvfp4_gemm on those codes."""
    import torch
    k = 1024
    weights = {n: nvfp4_from_host(*O.quantize_2d(W.gaussian_bf16((n, k), 3, 1600 + n, 0.02))) for n in (208, 25600)}
    seq = [(64, 25600, 1.0), (1, 208, 4.0), (17, 25600, 0.25), (64, 208, 1e-20), (8, 25600, 0.0), (64, 25600, 2.0)]
    for i, (m, n, scale) in enumerate(seq):
        if scale == 0.0:
            a = np.zeros((m, k), np.uint16)
        else:
            a = W.gaussian_bf16((m, k), 3, 1700 + i, scale, outlier_frac=0.01)
        c, qa = nv.quantize_gemm(bf16_to_device(a), weights[n])
        c2 = nv.gemm(qa, weights[n])
        _sync()
        _check_qa_against_oracle(a, qa)
        assert torch.equal(c, c2), f"call {i}"


def test_quantize_gemm_decode_strided_activations():
    """x as a view with a row stride above k (ldx = k + 64)."""
    import torch
    m, n, k = 48, 1040, 2048
    a = W.gaussian_bf16((m, k + 64), 4, 1800, 1.0, outlier_frac=0.01)
    xw = bf16_to_device(a)
    x = xw[:, :k]
    assert x.stride(0) == k + 64
    tw = nvfp4_from_host(*O.quantize_2d(W.gaussian_bf16((n, k), 4, 1801, 0.02)))
    c, qa = nv.quantize_gemm(x, tw)
    _sync()
    _check_qa_against_oracle(np.ascontiguousarray(a[:, :k]), qa)
    assert torch.equal(c, nv.gemm(qa, tw))
