"""Pins of the oracle's W4A16 product (no GPU): BF16 activations times the
reconstructed NVFP4 weights ("W4A8 vs NVFP4 quantization on GPUs",
weight-only quantization).

* One-hot activation rows scaled by powers of two pick weight columns
  exactly: C[i][n] = 2^p_i * W_hat[n][j_i].
* When the activations are themselves exactly an NVFP4 tensor's
  reconstruction, the W4A16 product equals the W4A4 oracle's product of the
  two reconstructions, bit for bit (same values, same summation order).
* A library matmul of the same binary64 operands agrees to rounding.
"""
import numpy as np

import oracle as O
import workloads as W


def test_one_hot_rows_pick_weight_columns():
    k, n = 256, 48
    wb = W.gaussian_bf16((n, k), 0, 950, 0.02)
    wc, wsf, gw = O.quantize_2d(wb)
    wh = O.dequantize(wc, wsf, gw)
    rng = np.random.default_rng(2)
    cols = rng.integers(0, k, 10)
    pw = rng.integers(-8, 9, 10)
    a = np.zeros((10, k), np.float64)
    a[np.arange(10), cols] = np.exp2(pw)
    ab = W.to_bf16_bits(a.astype(np.float32))
    c = O.gemm_w4a16_f64(ab, wc, wsf, gw)
    assert np.array_equal(c, np.exp2(pw)[:, None] * wh[:, cols].T)


def test_reduces_to_w4a4_on_exactly_quantized_activations():
    m, k, n = 24, 320, 48
    ab = W.gaussian_bf16((m, k), 0, 951, 1.0, outlier_frac=0.01)
    ac, asf, ga = O.quantize_1d(ab)
    ah = O.dequantize(ac, asf, ga)
    ahb = W.to_bf16_bits(ah.astype(np.float32))
    if not np.array_equal(O.bf16_to_f64(ahb), ah):       # reconstruction exact in BF16 for this g
        ga2 = 2.0 ** np.round(np.log2(ga))
        ah = O.dequantize(ac, asf, ga2)
        ahb = W.to_bf16_bits(ah.astype(np.float32))
    assert np.array_equal(O.bf16_to_f64(ahb), ah)
    wb = W.gaussian_bf16((n, k), 0, 952, 0.02)
    wc, wsf, gw = O.quantize_2d(wb)
    assert np.array_equal(O.gemm_w4a16_f64(ahb, wc, wsf, gw), O.gemm_f64(ah, O.dequantize(wc, wsf, gw)))


def test_matches_library_matmul():
    m, k, n = 16, 512, 64
    ab = W.gaussian_bf16((m, k), 0, 953, 1.0)
    wc, wsf, gw = O.quantize_2d(W.gaussian_bf16((n, k), 0, 954, 0.02))
    ref = O.bf16_to_f64(ab) @ O.dequantize(wc, wsf, gw).T
    got = O.gemm_w4a16_f64(ab, wc, wsf, gw)
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-14)
