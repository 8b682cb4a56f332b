"""Pins of the oracle's W4A4 GEMM (no GPU).

* Exact: every product (qa*sfa)*(qw*sfw) is a multiple of 2^-20 below 2^23, so
  on the tiny workload the sum is computed exactly in int64 (an independent
  integer decoding) and the binary64 GEMM over reconstructed values must
  agree with it times gA*gW to binary64 rounding.
* Library: the same binary64 GEMM equals numpy's matmul of the reconstructed
  operands.
* Orientation: C = A * W^T; a one-hot W picks columns of A, which fails on a
  transposed operand or a swapped index.
"""
import numpy as np

import oracle as O
import workloads as W


def test_gemm_f64_matches_exact_integer_sum_tiny():
    a, w = W.tiny(0)
    ac, asf, ga = O.quantize_1d(a)
    wc, wsf, gw = O.quantize_2d(w)
    ah, wh = O.dequantize(ac, asf, ga), O.dequantize(wc, wsf, gw)
    c = O.gemm_f64(ah, wh)
    exact = O.gemm_exact_i64(ac, asf, wc, wsf, 256)
    ref = exact.astype(np.float64) * 2.0 ** -20 * (float(np.float32(ga)) * float(np.float32(gw)))
    err = np.abs(c - ref)
    assert np.all(err <= 1e-12 * np.maximum(np.abs(ref), np.abs(ref).max()))
    assert np.abs(exact).max() > 0


def test_gemm_f64_matches_numpy_matmul():
    a = W.gaussian_bf16((40, 320), 0, 21, 1.0, outlier_frac=0.01)
    w = W.gaussian_bf16((48, 320), 0, 22, 0.02)
    ac, asf, ga = O.quantize_1d(a)
    wc, wsf, gw = O.quantize_2d(w)
    ah, wh = O.dequantize(ac, asf, ga), O.dequantize(wc, wsf, gw)
    c = O.gemm_f64(ah, wh)
    ref = ah @ wh.T
    assert np.allclose(c, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    rows = np.array([39, 0, 17])
    assert np.array_equal(O.gemm_f64_rows(ah, wh, rows), c[rows])


def test_gemm_orientation_one_hot():
    rng = np.random.default_rng(5)
    m, n, k = 7, 11, 32
    a = rng.standard_normal((m, k))
    cols = rng.integers(0, k, size=n)
    w = np.zeros((n, k))
    w[np.arange(n), cols] = 1.0
    c = O.gemm_f64(a, w)
    assert np.array_equal(c, a[:, cols])
