"""Canary bytes around every output buffer.

Each call writes into views of larger device buffers whose bytes were all
set to a canary value; after the call every byte outside the output (before
it, after it, and between the rows of a C with a row stride above n) must
still hold that value.  The outputs themselves must equal, bit for bit,
those of the same call on freshly allocated buffers: the canaries change
only where the results live, never what they are.  The shapes cover every
kernel that writes: the one-launch and two-kernel quantizers (one tensor,
row groups, the no-allocation entry point, pre-scaled and given-scale
forms), the 16x16 weight quantizer with its compact scales, the MXFP4
quantizer, the decode, single-SM, pair and stream-K GEMM tiles, the
output-maximum GEMM, both grouped GEMMs, the one-call decode and prefill
steps, the MXFP4 GEMM and the W4A16 GEMM."""
import numpy as np
import pytest

import workloads as W
import nvfp4_w4a4_quantized_05_b200 as nv
from gpu_util import bf16_to_device

pytestmark = pytest.mark.gpu

PAD = 4096          # canary bytes on each side (keeps every view 512-byte aligned)
FILL = 0xA5


class Canaried:
    """A device byte buffer: PAD canary bytes, the output region, PAD more."""

    def __init__(self, nbytes: int):
        import torch
        self.nbytes = int(nbytes)
        self.buf = torch.full((PAD + self.nbytes + PAD,), FILL, dtype=torch.uint8, device="cuda")

    def u8(self, *shape):
        v = self.buf[PAD:PAD + self.nbytes]
        return v.view(*shape) if shape else v

    def f32(self, n: int):
        import torch
        return self.buf[PAD:PAD + 4 * n].view(torch.float32)

    def bf16(self, rows: int, ld: int, cols: int):
        import torch
        return self.buf[PAD:PAD + 2 * rows * ld].view(torch.bfloat16).view(rows, ld)[:, :cols]

    def check(self, what: str, row_gaps=None):
        """Every byte outside the region (and, for a strided C, in the row
        gaps: (rows, ld, cols) in BF16 elements) still holds the canary."""
        h = self.buf.cpu().numpy()
        assert np.all(h[:PAD] == FILL), f"{what}: bytes written before the output"
        assert np.all(h[PAD + self.nbytes:] == FILL), f"{what}: bytes written past the output"
        if row_gaps is not None:
            rows, ld, cols = row_gaps
            body = h[PAD:PAD + self.nbytes].reshape(rows, 2 * ld)
            assert np.all(body[:, 2 * cols:] == FILL), f"{what}: bytes written between output rows"


def _sync():
    import torch
    torch.cuda.synchronize()
    nv.check_device_error()


def _bytes(t) -> np.ndarray:
    import torch
    return t.contiguous().view(torch.uint8).cpu().numpy()


def _same(got, want, what):
    assert np.array_equal(_bytes(got), _bytes(want)), f"{what}: differs from the plain call"


def _weights(n, k, seed):
    """NVFP4 weights [n, k]: 16x16 blocks where n % 16 == 0, else 1D blocks."""
    w = bf16_to_device(W.gaussian_bf16((n, k), seed, n, 0.02))
    return nv.quantize_weight_2d(w) if n % 16 == 0 else nv.quantize_act(w)


def _nvfp4_out(rows, k, sbytes, groups=1):
    cc, cs, cg = Canaried(rows * k // 2), Canaried(sbytes), Canaried(4 * groups)
    t = nv.NVFP4Tensor(cc.u8(rows, k // 2), cs.u8(), cg.f32(groups), rows, k)
    return t, (cc, cs, cg)


def _check_nvfp4(t, ref, cans, what, scale_used=None):
    """Codes, scales and global scales equal the plain call's; nothing written
    outside them.  scale_used: the scale bytes the call defines (a grouped
    call fills a prefix of its upper-bound buffer and leaves the rest)."""
    _same(t.codes, ref.codes, f"{what} codes")
    if scale_used is None:
        _same(t.scales, ref.scales, f"{what} scales")
    else:
        _same(t.scales[:scale_used], ref.scales[:scale_used], f"{what} scales")
        assert np.all(_bytes(t.scales[scale_used:]) == FILL), f"{what}: scale bytes written past the groups' tiles"
    _same(t.global_scale, ref.global_scale, f"{what} global scale")
    for c, part in zip(cans, ("codes", "scales", "global scale")):
        c.check(f"{what} {part}")


@pytest.mark.parametrize("rows,k", [
    (300, 4160),    # one-launch quantizer, ragged 128-row scale tile, k/64 odd
    (77, 80),       # k % 64 != 0: amax kernel + quantize kernel
    (1, 64),        # one row, one scale column
    (129, 2048),    # one row into the second scale tile
])
def test_quantize_act_writes_only_its_outputs(rows, k):
    x = bf16_to_device(W.gaussian_bf16((rows, k), 5, rows + k, 1.0, outlier_frac=0.01))
    ref = nv.quantize_act(x)
    t, cans = _nvfp4_out(rows, k, nv.nvfp4_scale_bytes(rows, k))
    nv.quantize_act(x, out=t)
    _sync()
    _check_nvfp4(t, ref, cans, f"quantize_act {rows}x{k}")


@pytest.mark.parametrize("k", [320, 80])
def test_grouped_quantize_writes_only_its_outputs(k):
    import torch
    off_h = np.array([0, 5, 5, 133, 300], np.int32)
    rows, groups = int(off_h[-1]), len(off_h) - 1
    x = bf16_to_device(W.gaussian_bf16((rows, k), 6, k, 1.0, outlier_frac=0.01))
    off = torch.from_numpy(off_h).cuda()
    ref = nv.quantize_act(x, off)
    t, cans = _nvfp4_out(rows, k, nv.nvfp4_grouped_scale_bytes(rows, groups, k), groups)
    nv.quantize_act(x, off, out=t)
    _sync()
    # each group's rows start a 128-row scale block; a block row of the
    # layout is 512 bytes per 64 values of k
    used = sum((int(n) + 127) // 128 for n in np.diff(off_h)) * ((k + 63) // 64) * 512
    _check_nvfp4(t, ref, cans, f"grouped quantize k={k}", scale_used=used)


@pytest.mark.parametrize("rows,k", [(300, 4160), (77, 80)])
def test_static_quantizer_writes_only_its_outputs(rows, k):
    import torch
    x = bf16_to_device(W.gaussian_bf16((rows, k), 7, rows, 1.0, outlier_frac=0.01))
    ref = nv.quantize_act(x)
    t, cans = _nvfp4_out(rows, k, nv.nvfp4_scale_bytes(rows, k))
    st = nv.nvfp4_quantize_act_static(x.data_ptr(), rows, k, k, None, 0, t.codes.data_ptr(), t.scales.data_ptr(),
                                      t.global_scale.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0
    _sync()
    _check_nvfp4(t, ref, cans, f"static quantizer {rows}x{k}")


def test_prescaled_and_given_scale_quantizers_write_only_their_outputs():
    import torch
    rows, k = 129, 256
    x = bf16_to_device(W.gaussian_bf16((rows, k), 8, 1, 1.0, outlier_frac=0.01))
    smooth = torch.from_numpy(np.exp2(np.arange(k) % 5 - 2).astype(np.float32)).cuda()
    ref = nv.quantize_act_smooth(x, smooth)
    t, cans = _nvfp4_out(rows, k, nv.nvfp4_scale_bytes(rows, k))
    nv.quantize_act_smooth(x, smooth, out=t)
    _sync()
    _check_nvfp4(t, ref, cans, "pre-scaled quantizer")

    g = torch.tensor([0.01], dtype=torch.float32, device="cuda")
    ref = nv.quantize_act_scaled(x, g)
    cc, cs = Canaried(rows * k // 2), Canaried(nv.nvfp4_scale_bytes(rows, k))
    t = nv.NVFP4Tensor(cc.u8(rows, k // 2), cs.u8(), g, rows, k)
    nv.quantize_act_scaled(x, g, out=t)
    _sync()
    _same(t.codes, ref.codes, "given-scale codes")
    _same(t.scales, ref.scales, "given-scale scales")
    cc.check("given-scale codes")
    cs.check("given-scale scales")


@pytest.mark.parametrize("n,k", [(208, 512), (4096, 128)])
def test_weight_quantizer_writes_only_its_outputs(n, k):
    import torch
    w = bf16_to_device(W.gaussian_bf16((n, k), 9, n, 0.02))
    ref, ref_c = nv.quantize_weight_2d(w, compact=True)
    t, cans = _nvfp4_out(n, k, nv.nvfp4_scale_bytes(n, k))
    csf = Canaried((n // 16) * (k // 16))
    ws = nv._workspace(torch, w.device, nv.OP_QUANTIZE_WEIGHT_2D)
    st = nv.nvfp4_quantize_weight_2d(w.data_ptr(), n, k, k, t.codes.data_ptr(), t.scales.data_ptr(),
                                     csf.buf.data_ptr() + PAD, t.global_scale.data_ptr(),
                                     0 if ws is None else ws.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert st == 0
    _sync()
    _check_nvfp4(t, ref, cans, f"weight quantizer {n}x{k}")
    _same(csf.u8(n // 16, k // 16), ref_c, "compact scales")
    csf.check("compact scales")


@pytest.mark.parametrize("m,n,k", [
    (33, 200, 192),      # decode tiles, ragged weight tile
    (100, 264, 128),     # single-SM tiles with two accumulators
    (520, 776, 512),     # pair tiles, ragged m and n
    (2304, 2336, 512),   # pair tiles shared out stream-K
])
def test_gemm_writes_only_c(m, n, k):
    a = nv.quantize_act(bf16_to_device(W.gaussian_bf16((m, k), 10, m, 1.0, outlier_frac=0.01)))
    b = _weights(n, k, 10)
    ref = nv.gemm(a, b)
    ld = n + 24                                  # a row stride above n: the gaps must stay untouched
    cc = Canaried(2 * m * ld)
    c = nv.gemm(a, b, out=cc.bf16(m, ld, n))
    _sync()
    _same(c, ref, f"gemm {m}x{n}x{k}")
    cc.check(f"gemm {m}x{n}x{k}", row_gaps=(m, ld, n))

    # the output-maximum form: C and the emitted global scale
    ref_c, ref_g = nv.gemm_emit_scale(a, b)
    cc, cg = Canaried(2 * m * ld), Canaried(4)
    c, g = nv.gemm_emit_scale(a, b, out=cc.bf16(m, ld, n), out_scale=cg.f32(1))
    _sync()
    _same(c, ref_c, f"gemm_emit_scale {m}x{n}x{k}")
    _same(g, ref_g, f"gemm_emit_scale {m}x{n}x{k} scale")
    cc.check(f"gemm_emit_scale {m}x{n}x{k}", row_gaps=(m, ld, n))
    cg.check(f"gemm_emit_scale {m}x{n}x{k} scale")


@pytest.mark.parametrize("sizes,n,k", [
    ([0, 1, 33, 255, 256, 300, 64], 256, 256),   # weights on the 256-row side (n % 256 == 0)
    ([300, 0, 257, 250], 320, 256),              # pair tiles per expert (>= 192 rows on average)
    ([40, 97, 64], 192, 128),                    # single-SM tiles per expert
])
def test_grouped_gemm_writes_only_c(sizes, n, k):
    import torch
    off_h = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    rows, E = int(off_h[-1]), len(sizes)
    a = nv.quantize_act(bf16_to_device(W.gaussian_bf16((rows, k), 11, rows, 1.0, outlier_frac=0.01)),
                        torch.from_numpy(off_h).cuda())
    wd = bf16_to_device(W.gaussian_bf16((E * n, k), 11, n, 0.02))
    tw = [nv.quantize_weight_2d(wd[e * n:(e + 1) * n]) for e in range(E)]
    b_codes = torch.stack([t.codes for t in tw])
    b_scales = torch.cat([t.scales for t in tw])
    b_global = torch.cat([t.global_scale for t in tw])
    ref = nv.grouped_gemm(a, b_codes, b_scales, b_global, n)
    cc = Canaried(2 * rows * n)
    c = nv.grouped_gemm(a, b_codes, b_scales, b_global, n, out=cc.bf16(rows, n, n))
    _sync()
    _same(c, ref, f"grouped gemm n={n}")
    cc.check(f"grouped gemm n={n}")


@pytest.mark.parametrize("m,n,k", [(64, 400, 4096), (5, 208, 320), (300, 256, 512)])
def test_quantize_gemm_writes_only_its_outputs(m, n, k):
    x = bf16_to_device(W.gaussian_bf16((m, k), 12, m, 1.0, outlier_frac=0.01))
    b = _weights(n, k, 12)
    ref_c, ref_qa = nv.quantize_gemm(x, b)
    ld = n + 8
    cc = Canaried(2 * m * ld)
    qa, cans = _nvfp4_out(m, k, nv.nvfp4_scale_bytes(m, k))
    c, qa = nv.quantize_gemm(x, b, out=cc.bf16(m, ld, n), qa=qa)
    _sync()
    _same(c, ref_c, f"quantize_gemm {m}x{n}x{k}")
    cc.check(f"quantize_gemm {m}x{n}x{k}", row_gaps=(m, ld, n))
    _check_nvfp4(qa, ref_qa, cans, f"quantize_gemm {m}x{n}x{k} activations")


def test_mxfp4_writes_only_its_outputs():
    m, n, k = 300, 776, 512
    x = bf16_to_device(W.gaussian_bf16((m, k), 13, m, 1.0, outlier_frac=0.01))
    w = bf16_to_device(W.gaussian_bf16((n, k), 13, n, 0.02))
    ref = nv.quantize_mx(x)
    cc, cs = Canaried(m * k // 2), Canaried(nv.mxfp4_scale_bytes(m, k))
    a = nv.quantize_mx(x, out=nv.MXFP4Tensor(cc.u8(m, k // 2), cs.u8(), m, k))
    _sync()
    _same(a.codes, ref.codes, "MXFP4 codes")
    _same(a.scales, ref.scales, "MXFP4 scales")
    cc.check("MXFP4 codes")
    cs.check("MXFP4 scales")
    b = nv.quantize_mx(w)
    ref_c = nv.gemm_mx(a, b)
    ld = n + 16
    cc = Canaried(2 * m * ld)
    c = nv.gemm_mx(a, b, out=cc.bf16(m, ld, n))
    _sync()
    _same(c, ref_c, "MXFP4 GEMM")
    cc.check("MXFP4 GEMM", row_gaps=(m, ld, n))


def test_w4a16_writes_only_c():
    m, n, k = 33, 200, 192
    a = bf16_to_device(W.gaussian_bf16((m, k), 14, m, 1.0))
    b = _weights(n, k, 14)
    ref = nv.gemm_w4a16(a, b)
    ld = n + 8
    cc = Canaried(2 * m * ld)
    c = nv.gemm_w4a16(a, b, out=cc.bf16(m, ld, n))
    _sync()
    _same(c, ref, "W4A16 GEMM")
    cc.check("W4A16 GEMM", row_gaps=(m, ld, n))
