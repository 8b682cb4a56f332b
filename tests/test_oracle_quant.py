"""Pins of the oracle's quantizers (no GPU).

* Exact round trip: a tensor built as fp4 x block_scale x global_scale with
  global scale 0.00390625 (the value in Figure 1 of "Accelerating large
  language models with NVFP4 quantization") and block scales on the E4M3
  grid must come back with those very codes, scales and global scale, and
  reconstruct exactly ("NVFP4 Explained", "How NVFP4 Represents a Value").
  A wrong 6 * 448 constant, a wrong block-scale formula or a wrong
  reconstruction fails it.
* Storage: 4 bits per value plus one 8-bit scale per 16 values plus one FP32
  per tensor = 4.5 bits/value ("W4A8 vs NVFP4 quantization on GPUs", "Scale
  layout changes the real storage cost"); 16/4.5 and 8/4.5 match the ~3.5x and
  ~1.8x of "NVFP4 Explained", "Memory and Accuracy".
* Outliers: per-16 block scales give lower error than one scale per tensor
  on outlier-laden data ("NVFP4 Explained", "Why Blocks of 16 Improve
  Accuracy").
* Element rounding: each code is the E2M1 value nearest to x * r.
* 2D blocks ("What is NVFP4?", "Why does scaling matter so much?") reduce to
  1D blocks when a tile's 16 rows are equal; grouped quantization equals
  independent quantization of each group.
"""
import json
import os

import numpy as np
import pytest

import oracle as O
import workloads as W

GRID = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)


def _facts(golden_dir):
    with open(os.path.join(golden_dir, "format_facts.json")) as f:
        return {k: v["value"] for k, v in json.load(f).items() if not k.startswith("_")}


def _build_exact(rng, rows, k, g, block_rows=1):
    """x = v * s * g with v on the E2M1 grid (every block holds a +-6) and s an
    E4M3 value; one block uses s = 448 so amax = 6 * 448 * g."""
    nb_r, nb_c = rows // block_rows, k // 16
    s_codes = rng.integers(1, 0x7E, size=(nb_r, nb_c)).astype(np.uint8)
    s_codes[rng.integers(nb_r), rng.integers(nb_c)] = 0x7E
    mag_idx = rng.integers(1, 8, size=(rows, k))          # no zeros: avoids the +-0 ambiguity
    sign = rng.integers(0, 2, size=(rows, k))
    for br in range(nb_r):
        for bc in range(nb_c):
            r = br * block_rows + rng.integers(block_rows)
            mag_idx[r, bc * 16 + rng.integers(16)] = 7   # a +-6 in every block
    v = GRID[mag_idx] * np.where(sign == 1, -1.0, 1.0)
    s = np.array([O.e4m3_decode(c) for c in range(256)])[s_codes]
    s_el = np.repeat(np.repeat(s, block_rows, axis=0), 16, axis=1)
    x = v * s_el * g
    xb = W.to_bf16_bits(x.astype(np.float32))
    assert np.array_equal(W.bf16_bits_to_f32(xb).astype(np.float64), x), "construction must be exact in BF16"
    codes = (mag_idx | (sign << 3)).astype(np.uint8)
    return xb, x, codes, s_codes


def _unpack(codes):
    lo, hi = codes & 0xF, codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)


def test_exact_round_trip_1d_fig1_global_scale(golden_dir):
    g_fig1 = _facts(golden_dir)["example_global_scale"]
    rng = np.random.default_rng(1)
    rows, k = 160, 96                                   # 2 scale row tiles, ragged columns
    xb, x, want_codes, want_s = _build_exact(rng, rows, k, g_fig1)
    codes, sf, g = O.quantize_1d(xb)
    assert g == g_fig1
    assert np.array_equal(_unpack(codes), want_codes)
    # element 2i in the low nibble of byte i
    assert np.array_equal(codes, (want_codes[:, 0::2] | (want_codes[:, 1::2] << 4)).astype(np.uint8))
    for r in range(rows):
        for b in range(k // 16):
            assert sf[O.sf_offset(r, b, k)] == want_s[r, b]
    assert np.array_equal(O.dequantize(codes, sf, g), x)


def test_exact_round_trip_2d_fig1_global_scale(golden_dir):
    g_fig1 = _facts(golden_dir)["example_global_scale"]
    rng = np.random.default_rng(2)
    rows, k = 48, 64
    xb, x, want_codes, want_s = _build_exact(rng, rows, k, g_fig1, block_rows=16)
    codes, sf, g, sfc = O.quantize_2d(xb, compact=True)
    assert g == g_fig1
    assert np.array_equal(_unpack(codes), want_codes)
    assert np.array_equal(sfc, want_s)
    for r in range(rows):
        for b in range(k // 16):
            assert sf[O.sf_offset(r, b, k)] == want_s[r // 16, b]
    assert np.array_equal(O.dequantize(codes, sf, g), x)


def test_storage_is_4p5_bits_per_value(golden_dir):
    f = _facts(golden_dir)
    for rows, k in [(128, 64), (256, 4096), (8192, 4096)]:
        n = rows * k
        code_bytes = rows * k // 2
        scale_bytes = O.scale_rows(rows) * O.scale_cols(k)
        total_bits = 8 * (code_bytes + scale_bytes) + f["tensor_scale_bits"]
        assert scale_bytes * 8 == n // f["block_size_1d"] * f["scale_bits_per_block"]
        assert (total_bits - f["tensor_scale_bits"]) / n == f["bits_per_value"]
    ratio16, ratio8 = 16 / f["bits_per_value"], 8 / f["bits_per_value"]
    # 16/4.5 = 3.56 reads as "~3.5x"; 8/4.5 = 1.78 reads as "~1.8x"
    assert f["memory_ratio_vs_fp16"] <= ratio16 < f["memory_ratio_vs_fp16"] + 0.1
    assert abs(ratio8 - f["memory_ratio_vs_fp8"]) < 0.05


@pytest.mark.parametrize("which", ["tiny", "laplace"])
def test_block_scaling_beats_single_scale_on_outliers(which):
    if which == "tiny":
        xb, _ = W.tiny(0)
    else:
        xb = W.laplace_outliers_bf16((512, 1024), 0, 3)
    x = O.bf16_to_f64(xb)
    codes, sf, g = O.quantize_1d(xb)
    xh = O.dequantize(codes, sf, g)
    xs = O.single_scale_fp4(xb)
    e_blk = (x - xh) ** 2
    e_one = (x - xs) ** 2
    assert e_blk.mean() <= e_one.mean()
    per_blk = e_blk.reshape(-1, 16).sum(1)
    per_one = e_one.reshape(-1, 16).sum(1)
    assert np.mean(per_blk <= per_one) >= 0.95


def test_codes_are_nearest_e2m1_of_scaled_input():
    xb = W.laplace_outliers_bf16((256, 512), 0, 3, outlier_frac=0.01)
    codes, sf, g = O.quantize_1d(xb)
    rows, k = xb.shape
    x = W.bf16_bits_to_f32(xb)
    sfb = np.array([[sf[O.sf_offset(r, b, k)] for b in range(k // 16)] for r in range(rows)])
    dec_s = np.array([O.e4m3_decode(c) for c in range(256)], np.float32)[sfb]
    d = (dec_s * np.float32(g)).astype(np.float32)
    with np.errstate(divide="ignore"):
        r = np.where(d == 0, np.float32(0), np.float32(1) / d).astype(np.float32)
    y = (x * np.repeat(r, 16, axis=1)).astype(np.float32)
    dec = np.array([O.e2m1_decode(c) for c in range(16)])[_unpack(codes)]
    # nearest grid magnitude, ties to the even code, saturating at 6
    ay = np.abs(y.astype(np.float64))
    dist = np.abs(ay[..., None] - GRID)
    best = dist.min(-1)
    assert np.all(np.abs(np.abs(dec) - ay) == best)
    # a block whose scale is a normal E4M3 value reaches the top code 6
    normal_blocks = sfb >= 0x08
    top = np.abs(dec).reshape(rows, k // 16, 16).max(-1)
    assert np.all(top[normal_blocks] == 6.0)


def test_2d_reduces_to_1d_when_tile_rows_are_equal():
    base = W.gaussian_bf16((4, 128), 0, 11, 0.02)
    xb = np.repeat(base, 16, axis=0)                   # every 16-row tile has equal rows
    c1, s1, g1 = O.quantize_1d(xb)
    c2, s2, g2 = O.quantize_2d(xb)
    assert g1 == g2 and np.array_equal(c1, c2) and np.array_equal(s1, s2)


def test_2d_scale_replicated_over_tile_rows():
    xb = W.gaussian_bf16((64, 256), 0, 12, 0.02)
    codes, sf, g, sfc = O.quantize_2d(xb, compact=True)
    for r in range(64):
        for b in range(16):
            assert sf[O.sf_offset(r, b, 256)] == sfc[r // 16, b]


def test_grouped_equals_independent_groups():
    rng = np.random.default_rng(3)
    sizes = [0, 5, 128, 130, 0, 1, 257]
    off = np.concatenate([[0], np.cumsum(sizes)]).astype(np.int32)
    xb = W.gaussian_bf16((int(off[-1]), 64), 0, 13, 1.0, outlier_frac=0.01)
    codes, sf, g = O.quantize_1d_grouped(xb, off)
    C = O.scale_cols(64)
    row0 = 0
    for e, n in enumerate(sizes):
        a, b = off[e], off[e + 1]
        if n:
            c1, s1, g1 = O.quantize_1d(xb[a:b])
            assert g[e] == g1
            assert np.array_equal(codes[a:b], c1)
            assert np.array_equal(sf[row0 * C:(row0 + O.scale_rows(n)) * C], s1)
        else:
            assert g[e] == 1.0
        row0 += O.scale_rows(n)
    assert sf.size == row0 * C


def test_zero_tensor_and_signed_zero():
    xb = np.zeros((3, 32), np.uint16)
    xb[1, 3] = 0x8000                                  # BF16 -0.0
    codes, sf, g = O.quantize_1d(xb)
    assert g == 1.0 and not sf.any()
    u = _unpack(codes)
    assert u[1, 3] == 0x8 and (u.sum() == 0x8)


def test_nonfinite_input_rejected():
    xb = np.zeros((1, 16), np.uint16)
    xb[0, 5] = 0x7F80                                  # +inf
    with pytest.raises(ValueError):
        O.quantize_1d(xb)


def test_scale_layout_is_a_bijection():
    for rows, k in [(128, 64), (200, 80), (1, 16)]:
        R, C = O.scale_rows(rows), O.scale_cols(k)
        offs = {O.sf_offset(r, c, k) for r in range(R) for c in range(C)}
        assert offs == set(range(R * C))


def test_given_scale_matches_dynamic_and_moves_the_scale_exponent():
    """The given-scale quantizer (second pass of the two-phase form) equals
    the dynamic one when given the tensor's own global scale.  With g doubled
    every block scale drops by exactly one E4M3 exponent step (all blocks here
    stay in the normal range) and, d = dec(sf) g being unchanged, every code
    stays the same."""
    x = W.gaussian_bf16((64, 256), 0, 71, 1.0)
    c0, s0, g0 = O.quantize_1d(x)
    c1, s1 = O.quantize_1d_given_g(x, g0)
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1)
    c2, s2 = O.quantize_1d_given_g(x, np.float32(2.0) * np.float32(g0))
    assert np.array_equal(c0, c2)
    used = s0 != 0                                   # padding bytes stay 0
    d0 = np.array([O.e4m3_decode(int(b)) for b in s0[used]])
    d2 = np.array([O.e4m3_decode(int(b)) for b in s2[used]])
    assert d0.min() >= 2.0 ** -5                     # halving keeps every scale normal
    assert np.array_equal(d2, d0 / 2)
    with pytest.raises(ValueError):
        O.quantize_1d_given_g(x, 0.0)


def test_smooth_quantizer_pins():
    """Per-channel pre-scaling folded into the quantizer.  s = 1 is the plain
    quantizer.  With powers of two per channel every product is exact, so the
    result is the plain quantizer of the BF16 tensor x * 2^j[c] (in range).
    A uniform factor 2^j moves only g: codes and scale bytes stay."""
    x = W.laplace_outliers_bf16((48, 512), 0, 72)
    c0, s0, g0 = O.quantize_1d(x)
    c1, s1, g1 = O.quantize_1d_smooth(x, np.ones(512, np.float32))
    assert np.array_equal(c0, c1) and np.array_equal(s0, s1) and g0 == g1
    rng = np.random.default_rng(3)
    j = rng.integers(-6, 7, 512)
    xs = O.bf16_to_f64(x) * np.exp2(j)[None, :]          # exact in float32 and in BF16 (8-bit mantissas kept)
    xb = (xs.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(O.bf16_to_f64(xb), xs)
    c2, s2, g2 = O.quantize_1d_smooth(x, np.exp2(j).astype(np.float32))
    c3, s3, g3 = O.quantize_1d(xb)
    assert np.array_equal(c2, c3) and np.array_equal(s2, s3) and g2 == g3
    c4, s4, g4 = O.quantize_1d_smooth(x, np.full(512, 8.0, np.float32))
    assert np.array_equal(c4, c0) and np.array_equal(s4, s0) and g4 == g0 * 8
    with pytest.raises(ValueError):
        O.quantize_1d_smooth(x, np.zeros(512, np.float32))


def _overflow_blocks(sf, g, rows, k):
    """Blocks whose 1 / (decode(sf) g) overflows binary32."""
    sfb = np.array([[sf[O.sf_offset(r, b, k)] for b in range(k // 16)] for r in range(rows)])
    d = (np.array([O.e4m3_decode(c) for c in range(256)], np.float32)[sfb] * np.float32(g)).astype(np.float32)
    with np.errstate(divide="ignore", over="ignore"):
        return np.isinf(np.float32(1) / d[d != 0]).sum()


@pytest.mark.parametrize("block_rows", [1, 16])
def test_exact_round_trip_at_a_tiny_global_scale(block_rows):
    """The exact construction at g = 2^-123 (Figure 1's 2^-8 moved down by
    2^-115; every value stays exact in BF16, down to its smallest subnormal
    2^-133).  Blocks with a block scale at or below 2^-5 have d <= 2^-128,
    where 1 / d overflows binary32; their codes must still be the ones the
    tensor was built from, because x / d is exactly a grid value ("NVFP4
    Explained", "How NVFP4 Represents a Value").  Capping 1 / d at FLT_MAX
    instead would shrink those codes by up to 2^4."""
    g_tiny = 2.0 ** -123
    rng = np.random.default_rng(5 + block_rows)
    rows, k = (160, 96) if block_rows == 1 else (48, 96)
    xb, x, want_codes, want_s = _build_exact(rng, rows, k, g_tiny, block_rows=block_rows)
    if block_rows == 1:
        codes, sf, g = O.quantize_1d(xb)
    else:
        codes, sf, g = O.quantize_2d(xb)
    assert g == g_tiny
    assert _overflow_blocks(sf, g, rows, k) > 0, "the construction must reach the overflow branch"
    assert np.array_equal(_unpack(codes), want_codes)
    for r in range(rows):
        for b in range(k // 16):
            assert sf[O.sf_offset(r, b, k)] == want_s[r // block_rows, b]
    assert np.array_equal(O.dequantize(codes, sf, g), x)
    if block_rows == 1:
        c2, s2 = O.quantize_1d_given_g(xb, g_tiny)
        assert np.array_equal(c2, codes) and np.array_equal(s2, sf)


def test_codes_known_by_construction_at_a_rounded_subnormal_global_scale():
    """x = v D with D = 2^-130 and v on the E2M1 grid; blocks peak at 6 D, 3 D
    or 1.5 D.  Worked by hand: g = RN(6 D / 2688) = 1170 * 2^-149 (a rounded
    subnormal), 6 g = 7020 * 2^-149 exactly, so the block-scale quotients are
    448.1 (saturates to 448, byte 0x7E), 224.05 (-> 224, byte 0x76) and
    112.03 (-> 112, byte 0x6E); d = 524160, 262080 and 131040 times 2^-149,
    all below 2^-128.  x / d is then v, 2 v and 4 v times (1 + 2.4e-4), whose
    nearest codes are v, 2 v and 4 v."""
    D = 2.0 ** -130
    rng = np.random.default_rng(9)
    rows, k = 24, 96
    peaks = {6.0: (1, 0x7E), 3.0: (2, 0x76), 1.5: (4, 0x6E)}
    mag = np.zeros((rows, k))
    want_mag = np.zeros((rows, k))
    want_s = np.zeros((rows, k // 16), np.uint8)
    for r in range(rows):
        for b in range(k // 16):
            peak = [6.0, 3.0, 1.5][(r + b) % 3]
            mult, byte = peaks[peak]
            allowed = GRID[GRID <= peak]
            vals = rng.choice(allowed, 16)
            vals[rng.integers(16)] = peak
            mag[r, b * 16:(b + 1) * 16] = vals
            want_mag[r, b * 16:(b + 1) * 16] = vals * mult
            want_s[r, b] = byte
    mag[0, :16] = 6.0                                      # the tensor amax is 6 D
    want_mag[0, :16] = 6.0
    want_s[0, 0] = 0x7E
    sign = rng.integers(0, 2, size=(rows, k))
    x = mag * D * np.where(sign == 1, -1.0, 1.0)
    xb = W.to_bf16_bits(x.astype(np.float32))
    assert np.array_equal(W.bf16_bits_to_f32(xb).astype(np.float64), x)
    codes, sf, g = O.quantize_1d(xb)
    assert np.float32(g).view(np.uint32) == 1170             # 1170 * 2^-149
    assert _overflow_blocks(sf, g, rows, k) == rows * k // 16
    want_codes = np.searchsorted(GRID, want_mag) | (sign << 3)
    want_codes = np.where(mag == 0, sign << 3, want_codes)   # a signed zero keeps its sign bit
    assert np.array_equal(_unpack(codes), want_codes)
    for r in range(rows):
        for b in range(k // 16):
            assert sf[O.sf_offset(r, b, k)] == want_s[r, b]


def test_single_scale_baseline_worked_examples():
    """One scale amax / 6 for the whole tensor, codes rounded to the nearest
    E2M1 value with ties to the even code ("NVFP4 Explained", "Why Blocks of 16
    Improve Accuracy": one scale over many values lets the outlier set it).
    [0.5, 1, 60]: scale 10, quotients 0.05, 0.1, 6 -> 0, 0, 6 -> [0, 0, 60].
    amax 6 (scale 1) with every tie of the grid: 0.25 -> 0, 0.75 -> 1,
    1.25 -> 1, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4; the sign is kept."""
    x = np.array([0.5, 1.0, 60.0], np.float32)
    assert np.array_equal(O.single_scale_fp4(W.to_bf16_bits(x)), [0.0, 0.0, 60.0])
    t = np.array([6, 0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, -5, -1.75, 0.5], np.float32)
    want = [6, 0, 1, 1, 2, 2, 4, 4, -4, -2, 0.5]
    assert np.array_equal(O.single_scale_fp4(W.to_bf16_bits(t)), want)
    # amax 12 (scale 2): every value is halved before rounding, then doubled back
    assert np.array_equal(O.single_scale_fp4(W.to_bf16_bits(np.array([12, 1.5, -2.5, 7], np.float32))),
                          [12, 2, -2, 8])
    assert not O.single_scale_fp4(np.zeros(4, np.uint16)).any()
