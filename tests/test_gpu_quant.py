"""GPU quantizer parity: codes, scale bytes (whole buffer, pads included) and
global scales must equal the CPU oracle bit for bit on the same seeded
inputs; the hardware conversions must equal the oracle's encoders over wide
binary32 sweeps.  Calls go through the C ABI (via the thin binding)."""
import numpy as np
import pytest

import oracle as O
import workloads as W
import nvfp4_w4a4_quantized_05_b200 as nv
from gpu_util import bf16_to_device, device

pytestmark = pytest.mark.gpu


def _gpu_q1d(xb, offsets=None):
    import torch
    x = bf16_to_device(xb)
    off = None if offsets is None else torch.from_numpy(np.asarray(offsets, np.int32)).to(device())
    q = nv.quantize_act(x, off)
    torch.cuda.synchronize()
    nv.check_device_error()
    return q.codes.cpu().numpy(), q.scales.cpu().numpy(), q.global_scale.cpu().numpy()


def _assert_same_1d(xb):
    c, s, g = _gpu_q1d(xb)
    oc, osf, og = O.quantize_1d(xb)
    assert np.float32(og).view(np.uint32) == g[0].view(np.uint32), (og, g[0])
    assert s.size == osf.size
    bad = np.nonzero(c != oc)
    assert bad[0].size == 0, f"{bad[0].size} code bytes differ, first at {bad[0][0]},{bad[1][0]}"
    badsf = np.nonzero(s != osf)[0]
    assert badsf.size == 0, f"{badsf.size} scale bytes differ, first at {badsf[:4]}"


# ---- hardware conversions vs the oracle's encoders ----------------------------------

def _sweep_compare(lo_pattern, hi_pattern, step, which):
    import torch
    chunk = 1 << 26
    for start in range(lo_pattern, hi_pattern, chunk * step):
        stop = min(hi_pattern, start + chunk * step)
        pats = np.arange(start, stop, step, dtype=np.uint64).astype(np.uint32)
        vals = pats.view(np.float32)
        x = torch.from_numpy(pats.view(np.int32)).to(device()).view(torch.float32)
        out = torch.empty(vals.size, dtype=torch.uint8, device=device())
        if which == "e2m1":
            st = nv.nvfp4_probe_cvt(x.data_ptr(), out.data_ptr(), None, vals.size)
            want = O.e2m1_encode_array(vals)
        else:
            st = nv.nvfp4_probe_cvt(x.data_ptr(), None, out.data_ptr(), vals.size)
            want = O.e4m3_encode_array(np.abs(vals))
        assert st == 0
        got = out.cpu().numpy()
        bad = np.nonzero(got != want)[0]
        assert bad.size == 0, (f"{which}: {bad.size} mismatches in [{start:#x},{stop:#x}); first value "
                               f"{vals[bad[0]]!r} hw {got[bad[0]]:#x} oracle {want[bad[0]]:#x}")


def test_cvt_e2m1_every_pattern_below_8():
    _sweep_compare(0, 0x41000001, 1, "e2m1")                    # every +0 .. 8.0
    _sweep_compare(0x80000000, 0xC1000001, 1, "e2m1")          # every -0 .. -8.0


def test_cvt_e2m1_large_and_sign_sample():
    _sweep_compare(0x41000000, 0x7F800000, 257, "e2m1")        # 8 .. FLT_MAX, sampled
    _sweep_compare(0xC1000000, 0xFF800000, 263, "e2m1")


def test_cvt_e4m3_every_pattern_below_1024():
    _sweep_compare(0, 0x44800001, 1, "e4m3")
    _sweep_compare(0x44800000, 0x7F800000, 251, "e4m3")        # saturating range, sampled


# ---- 1D activations ------------------------------------------------------------------

@pytest.mark.parametrize("shape", [(16, 256), (1, 16), (3, 48), (130, 320), (257, 4112), (64, 5120), (1, 5120),
                                   (300, 3072), (1000, 2080), (200, 1040), (5000, 3104), (5000, 3136), (700, 1088),
                                   (129, 960)])
def test_quantize_act_matches_oracle(shape):
    xb = W.gaussian_bf16(shape, 0, 100 + shape[0], 1.0, outlier_frac=0.01)
    _assert_same_1d(xb)


def test_quantize_act_full_activation_workload():
    _assert_same_1d(W.quant_act(0))          # [8192, 4096] Laplace + 0.1% +-U[50,200]


def test_quantize_act_prefill_activations():
    a, _ = W.prefill(0, n=16)
    _assert_same_1d(a)                       # [4096, 4096] N(0,1)


@pytest.mark.parametrize("case", ["zeros", "signed_zeros", "constant", "subnormal", "huge", "tiny_and_huge"])
def test_quantize_act_edge_values(case):
    rng = np.random.default_rng(7)
    shape = (40, 96)
    n = shape[0] * shape[1]
    if case == "zeros":
        xb = np.zeros(shape, np.uint16)
    elif case == "signed_zeros":
        xb = (rng.integers(0, 2, size=shape) * 0x8000).astype(np.uint16)
    elif case == "constant":
        xb = np.full(shape, 0x3FC0, np.uint16)          # 1.5
    elif case == "subnormal":
        xb = (rng.integers(1, 0x80, size=n) | (rng.integers(0, 2, size=n) << 15)).astype(np.uint16).reshape(shape)
    elif case == "huge":
        xb = (rng.integers(0x7F00, 0x7F80, size=n) | (rng.integers(0, 2, size=n) << 15)).astype(np.uint16).reshape(shape)
    else:
        lo = rng.integers(1, 0x0100, size=n)
        hi = rng.integers(0x7E00, 0x7F80, size=n)
        pick = rng.random(n) < 0.02
        xb = np.where(pick, hi, lo).astype(np.uint16).reshape(shape)
    _assert_same_1d(xb)



# ---- tiny global scales (1 / d beyond binary32) -----------------------------------------

def _tiny_bf16(shape, stream, scale_pow):
    """N(0,1) values times 2^scale_pow, rounded to BF16 (subnormal BF16 values
    included for the smallest scales)."""
    x = W.bf16_bits_to_f32(W.gaussian_bf16(shape, 0, stream, 1.0, outlier_frac=0.01))
    return W.to_bf16_bits((x * np.float32(2.0 ** scale_pow)).astype(np.float32))


@pytest.mark.parametrize("scale_pow", [-60, -110, -118, -124, -128])
@pytest.mark.parametrize("shape", [(160, 96), (160, 1088), (70, 2048)])
def test_quantize_act_tiny_global_scale(shape, scale_pow):
    """Tensors whose amax puts g below 2^-64 (the kernels' tiny form of r)
    and, from 2^-118 down, d = decode(sf) g below 2^-128, where 1 / d
    overflows binary32: codes and scales equal the oracle's bit for bit.
    k = 96 takes the two-kernel path, 1088 and 2048 the one-launch path."""
    xb = _tiny_bf16(shape, 500 + shape[1], scale_pow)
    _assert_same_1d(xb)


@pytest.mark.parametrize("k", [1024, 1040])
def test_grouped_quantize_tiny_and_normal_groups(k):
    """Groups of very different magnitude in one call: each group takes the
    tiny form of r or not by its own global scale (one-launch form for
    k = 1024, two-kernel form for 1040)."""
    sizes = [130, 64, 0, 200, 17]
    pows = [0, -120, 0, -126, -100]
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    parts = [_tiny_bf16((n, k), 600 + e, p) for e, (n, p) in enumerate(zip(sizes, pows))]
    _assert_same_grouped(np.concatenate(parts, axis=0), off)


def test_quantize_weight_2d_tiny_global_scale():
    import torch
    wb = _tiny_bf16((96, 160), 700, -122)
    t = nv.quantize_weight_2d(bf16_to_device(wb))
    torch.cuda.synchronize()
    oc, osf, og = O.quantize_2d(wb)
    assert t.global_scale.cpu().numpy()[0].view(np.uint32) == np.float32(og).view(np.uint32)
    assert np.array_equal(t.codes.cpu().numpy(), oc)
    assert np.array_equal(t.scales.cpu().numpy(), osf)


@pytest.mark.parametrize("g_bits", [0x04000000, 0x00800000, 0x00001234])   # 2^-119, 2^-126, subnormal
@pytest.mark.parametrize("scale_pow", [0, -118])
def test_quantize_act_scaled_tiny_given_scale(g_bits, scale_pow):
    """The given-scale pass with g below 2^-64: on a tensor of matching size,
    and on one far too large for g, whose codes saturate at 6."""
    import torch
    xb = _tiny_bf16((150, 320), 710, scale_pow)
    g = np.array([g_bits], np.uint32).view(np.float32)
    q = nv.quantize_act_scaled(bf16_to_device(xb), torch.from_numpy(g.copy()).to(device()))
    torch.cuda.synchronize()
    oc, osf = O.quantize_1d_given_g(xb, g[0])
    assert np.array_equal(q.codes.cpu().numpy(), oc)
    assert np.array_equal(q.scales.cpu().numpy(), osf)


def test_quantize_act_smooth_tiny_global_scale():
    import torch
    xb = _tiny_bf16((130, 2048), 720, -121)
    s = (0.5 + W.uniform(0, 721, 2048)).astype(np.float32)
    q = nv.quantize_act_smooth(bf16_to_device(xb), torch.from_numpy(s).to(device()))
    torch.cuda.synchronize()
    oc, osf, og = O.quantize_1d_smooth(xb, s)
    assert q.global_scale.cpu().numpy()[0].view(np.uint32) == np.float32(og).view(np.uint32)
    assert np.array_equal(q.codes.cpu().numpy(), oc)
    assert np.array_equal(q.scales.cpu().numpy(), osf)

@pytest.mark.parametrize("amax_bits", [0x3F80, 0x4340, 0x3B4D, 0x0B00, 0x0080, 0x0001, 0x7F7F])
def test_block_scale_every_bf16_block_amax(amax_bits):
    """One block per positive BF16 value up to the tensor amax: each block's
    amax is that value (at a random position, random sign), so the block
    scale rounding meets every E4M3 rounding boundary the quotient can hit,
    exact midpoints included.  Amax 0x0080 / 0x0001 make 6 g subnormal."""
    rng = np.random.default_rng(amax_bits)
    pats = np.arange(1, amax_bits + 1, dtype=np.uint32)
    nb = pats.size
    bpr = 64                                            # blocks per row: k = 1024
    rows = -(-nb // bpr)
    blocks = np.zeros((rows * bpr, 16), np.uint16)
    peak = (pats << 16).view(np.float32)
    frac = rng.random((nb, 16), dtype=np.float32)
    others = ((peak[:, None] * frac).view(np.uint32) >> 16).astype(np.uint16)   # truncation: |v| <= peak
    others |= (rng.integers(0, 2, size=(nb, 16)) << 15).astype(np.uint16)
    pos = rng.integers(0, 16, size=nb)
    others[np.arange(nb), pos] = pats.astype(np.uint16) | (rng.integers(0, 2, size=nb) << 15).astype(np.uint16)
    blocks[:nb] = others
    xb = blocks.reshape(rows, bpr * 16)
    _assert_same_1d(xb)


def test_quantize_act_strided_rows():
    import torch
    wide = W.gaussian_bf16((70, 384), 0, 41, 1.0, outlier_frac=0.01)
    x = bf16_to_device(wide)[:, :320]                   # ld = 384 > k = 320
    q = nv.quantize_act(x)
    torch.cuda.synchronize()
    oc, osf, og = O.quantize_1d(np.ascontiguousarray(wide[:, :320]))
    assert np.array_equal(q.codes.cpu().numpy(), oc)
    assert np.array_equal(q.scales.cpu().numpy(), osf)
    assert q.global_scale.cpu().numpy()[0] == np.float32(og)


def test_quantize_act_strided_rows_large():
    """Row stride > k on a tensor large enough that part of it is re-read from L2."""
    import torch
    wide = W.gaussian_bf16((10000, 2176), 0, 43, 1.0, outlier_frac=0.001)
    x = bf16_to_device(wide)[:, :2048]
    q = nv.quantize_act(x)
    torch.cuda.synchronize()
    nv.check_device_error()
    oc, osf, og = O.quantize_1d(np.ascontiguousarray(wide[:, :2048]))
    assert np.array_equal(q.codes.cpu().numpy(), oc)
    assert np.array_equal(q.scales.cpu().numpy(), osf)
    assert q.global_scale.cpu().numpy()[0] == np.float32(og)


def test_workspace_reusable_across_calls():
    """The workspace carries state between calls (grid-barrier generations):
    repeated calls on one workspace, and a re-initialized one, give the
    oracle's results; the counter words stay zero."""
    import torch
    xb = W.gaussian_bf16((300, 512), 0, 42, 1.0)
    x = bf16_to_device(xb)
    dev = device()
    ws = torch.zeros(nv.nvfp4_workspace_bytes(nv.OP_QUANTIZE_ACT), dtype=torch.uint8, device=dev)
    codes = torch.empty((300, 256), dtype=torch.uint8, device=dev)
    scales = torch.empty(nv.nvfp4_scale_bytes(300, 512), dtype=torch.uint8, device=dev)
    g = torch.empty(1, dtype=torch.float32, device=dev)
    oc, osf, og = O.quantize_1d(xb)
    stream = torch.cuda.current_stream().cuda_stream
    for it in range(5):
        if it == 3:
            assert nv.nvfp4_workspace_init(ws.data_ptr(), ws.numel(), stream) == 0
        codes.fill_(0xAA)
        st = nv.nvfp4_quantize_act(x.data_ptr(), 300, 512, 512, None, 0, codes.data_ptr(), scales.data_ptr(),
                                   g.data_ptr(), ws.data_ptr(), stream)
        assert st == 0
        torch.cuda.synchronize()
        nv.check_device_error()
        assert int(ws[32896:32912].abs().sum()) == 0      # the two-kernel path's counters
        assert np.array_equal(codes.cpu().numpy(), oc) and np.array_equal(scales.cpu().numpy(), osf)
        assert g.cpu().numpy()[0] == np.float32(og)


# ---- grouped (MoE) ---------------------------------------------------------------------

def _assert_same_grouped(xb, off):
    c, s, g = _gpu_q1d(xb, off)
    oc, osf, og = O.quantize_1d_grouped(xb, off)
    assert np.array_equal(g.view(np.uint32), og.view(np.uint32))
    assert np.array_equal(c, oc)
    assert s.size >= osf.size
    bad = np.nonzero(s[:osf.size] != osf)[0]
    assert bad.size == 0, f"{bad.size} scale bytes differ, first at {bad[:4]}"


@pytest.mark.parametrize("k", [2048, 960, 4160, 2064])
def test_grouped_quantize_ragged_groups(k):
    # k % 64 == 0: the one-launch grouped form (k < 1024: narrow tasks; 4160:
    # a partial last task); 2064: the two-kernel form
    sizes = [0, 5, 128, 130, 0, 1, 257, 64]
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    xb = W.gaussian_bf16((int(off[-1]), k), 0, 43, 1.0, outlier_frac=0.01)
    _assert_same_grouped(xb, off)


@pytest.mark.parametrize("groups", [1024, 1100])
def test_grouped_quantize_many_groups(groups):
    """Up to 1024 groups take the one-launch form, more the two-kernel form;
    group sizes 0..40 with runs of empty groups, and one all-zero group."""
    rng = np.random.default_rng(groups)
    sizes = rng.integers(0, 41, groups)
    sizes[10:20] = 0
    sizes[-3:] = 0
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    xb = W.gaussian_bf16((int(off[-1]), 128), 0, 45, 1.0, outlier_frac=0.01)
    z = int(np.argmax(sizes > 5))
    xb[off[z]:off[z + 1]] = 0
    _assert_same_grouped(xb, off)


def test_grouped_and_single_calls_share_a_workspace():
    """Grouped and one-tensor calls alternate on one workspace (sized for the
    groups): every result is the oracle's."""
    import torch
    dev = device()
    sizes = [300, 0, 129, 256]
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    rows, k = int(off[-1]), 1024
    ws = torch.zeros(nv.nvfp4_workspace_bytes(nv.OP_QUANTIZE_ACT, rows, 0, k, len(sizes)), dtype=torch.uint8,
                     device=dev)
    stream = torch.cuda.current_stream().cuda_stream
    offd = torch.from_numpy(off).to(dev)
    for it in range(4):
        xb = W.gaussian_bf16((rows, k), it, 46, 1.0 + it, outlier_frac=0.01)
        x = bf16_to_device(xb)
        codes = torch.empty((rows, k // 2), dtype=torch.uint8, device=dev)
        if it % 2 == 0:
            scales = torch.zeros(nv.nvfp4_grouped_scale_bytes(rows, len(sizes), k), dtype=torch.uint8, device=dev)
            g = torch.empty(len(sizes), dtype=torch.float32, device=dev)
            st = nv.nvfp4_quantize_act(x.data_ptr(), rows, k, k, offd.data_ptr(), len(sizes), codes.data_ptr(),
                                       scales.data_ptr(), g.data_ptr(), ws.data_ptr(), stream)
            oc, osf, og = O.quantize_1d_grouped(xb, off)
        else:
            scales = torch.zeros(nv.nvfp4_scale_bytes(rows, k), dtype=torch.uint8, device=dev)
            g = torch.empty(1, dtype=torch.float32, device=dev)
            st = nv.nvfp4_quantize_act(x.data_ptr(), rows, k, k, None, 0, codes.data_ptr(), scales.data_ptr(),
                                       g.data_ptr(), ws.data_ptr(), stream)
            oc, osf, og = O.quantize_1d(xb)
        assert st == 0
        torch.cuda.synchronize()
        nv.check_device_error()
        assert np.array_equal(codes.cpu().numpy(), oc)
        assert np.array_equal(scales.cpu().numpy()[:np.asarray(osf).size], np.asarray(osf).reshape(-1))
        assert np.array_equal(g.cpu().numpy().view(np.uint32), np.atleast_1d(np.float32(og)).view(np.uint32))


def test_grouped_quantize_moe_workload():
    a, off, _ = W.moe(0, with_weights=False)        # [32768, 2048], 128 experts, top-8 routing
    _assert_same_grouped(a, off)


# ---- 2D weights --------------------------------------------------------------------------

@pytest.mark.parametrize("shape", [(64, 256), (16, 16), (48, 80), (272, 4112)])
def test_quantize_weight_2d_matches_oracle(shape):
    import torch
    wb = W.gaussian_bf16(shape, 0, 200 + shape[0], 0.02)
    t, sfc = nv.quantize_weight_2d(bf16_to_device(wb), compact=True)
    torch.cuda.synchronize()
    oc, osf, og, osfc = O.quantize_2d(wb, compact=True)
    assert t.global_scale.cpu().numpy()[0] == np.float32(og)
    assert np.array_equal(t.codes.cpu().numpy(), oc)
    assert np.array_equal(t.scales.cpu().numpy(), osf)
    assert np.array_equal(sfc.cpu().numpy(), osfc)


def test_quantize_weight_2d_full_weight_workload():
    import torch
    wb = W.quant_weight(0)                          # [14336, 4096] N(0, 0.02)
    t = nv.quantize_weight_2d(bf16_to_device(wb))
    torch.cuda.synchronize()
    oc, osf, og = O.quantize_2d(wb)
    assert t.global_scale.cpu().numpy()[0] == np.float32(og)
    assert np.array_equal(t.codes.cpu().numpy(), oc)
    assert np.array_equal(t.scales.cpu().numpy(), osf)


def test_out_buffers_reused_across_inputs():
    """`out=` writes a second input's result over the first one's buffers
    (activations and 2D weights): the result is the oracle's for the second
    input, with nothing left from the first."""
    import torch
    x1 = W.gaussian_bf16((200, 1024), 0, 301, 1.0)
    x2 = W.laplace_outliers_bf16((200, 1024), 0, 302)
    qa = nv.quantize_act(bf16_to_device(x1))
    nv.quantize_act(bf16_to_device(x2), out=qa)
    torch.cuda.synchronize()
    oc, osf, og = O.quantize_1d(x2)
    assert np.array_equal(qa.codes.cpu().numpy(), oc) and np.array_equal(qa.scales.cpu().numpy(), osf)
    assert qa.global_scale.cpu().numpy()[0] == np.float32(og)
    w1 = W.gaussian_bf16((96, 512), 0, 303, 0.02)
    w2 = W.gaussian_bf16((96, 512), 0, 304, 3.0)
    qw = nv.quantize_weight_2d(bf16_to_device(w1))
    nv.quantize_weight_2d(bf16_to_device(w2), out=qw)
    torch.cuda.synchronize()
    oc, osf, og = O.quantize_2d(w2)
    assert np.array_equal(qw.codes.cpu().numpy(), oc) and np.array_equal(qw.scales.cpu().numpy(), osf)
    assert qw.global_scale.cpu().numpy()[0] == np.float32(og)
    with pytest.raises(ValueError):
        nv.quantize_weight_2d(bf16_to_device(W.gaussian_bf16((80, 512), 0, 305, 0.02)), out=qw)
