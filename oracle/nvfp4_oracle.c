/*
 * nvfp4_oracle.c -- plain, slow CPU oracle for the NVFP4 W4A4 path.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by tests/, the smoke check and the CPU
 * baseline leg of the benchmark, never by the product path.  Shares no code
 * with the CUDA kernels.  See nvfp4_oracle.h for the passages it follows and
 * the readings taken where the pages are silent.
 *
 * Build: gcc -O2 -std=c11 -fopenmp -ffp-contract=off -fPIC -shared (no
 * fast-math), so each float expression below is one IEEE binary32 operation
 * rounded to nearest even.
 */
#include "nvfp4_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------ */
/* E2M1 ("What is NVFP4?", "What does NVFP4 mean?"): 1 sign bit, 2 exponent
 * bits (bias 1), 1 mantissa bit.  Exponent field 0 holds 0 and 0.5; the
 * normal values are (1 + m/2) * 2^(e-1): 1, 1.5, 2, 3, 4, 6.               */

uint8_t orc_e2m1_encode(float v) {
    uint8_t sign = signbit(v) ? 0x8 : 0x0;
    float a = fabsf(v);
    uint8_t mag;
    if (!(a < 6.0f)) {
        mag = 0x7;                            /* saturate at the largest finite value, 6 */
    } else if (a < 1.0f) {
        /* below the smallest normal (1.0) the spacing is 0.5 */
        float m = rintf(a * 2.0f);            /* exact scaling, then ties-to-even */
        mag = (uint8_t)m;                     /* 0, 1 or 2 (2 is the code of 1.0) */
    } else {
        int e2;
        frexpf(a, &e2);                       /* a = f * 2^e2 with f in [0.5, 1) */
        int e = e2 - 1;                       /* unbiased exponent: 0, 1 or 2 */
        float m = rintf(ldexpf(a, 1 - e));    /* significand in half-units: [2, 4) -> 2, 3, 4 */
        if (m == 4.0f) { e += 1; m = 2.0f; }  /* rounded up to the next binade */
        mag = (e > 2) ? 0x7 : (uint8_t)(((e + 1) << 1) | ((int)m - 2));
    }
    return (uint8_t)(sign | mag);
}

double orc_e2m1_decode(uint8_t code) {
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

/* ------------------------------------------------------------------------ */
/* E4M3 block scale ("NVFP4 Explained", "Why the Block Scale Uses FP8 E4M3"):
 * 4 exponent bits (bias 7), 3 mantissa bits; exponent field 0 is subnormal
 * with spacing 2^-9; largest finite value 1.75 * 2^8 = 448 (code 0x7E; 0x7F
 * is NaN and is never produced).  Encoding rounds to nearest, ties to even,
 * and saturates at 448.                                                     */

uint8_t orc_e4m3_encode(float x) {
    float a = fabsf(x);
    if (!(a < 448.0f)) return 0x7E;
    if (a < 0.015625f) {                      /* below 2^-6, the smallest normal */
        float m = rintf(ldexpf(a, 9));        /* multiples of 2^-9: 0..8 (8 is 2^-6, code 0x08) */
        return (uint8_t)m;
    }
    int e2;
    frexpf(a, &e2);
    int e = e2 - 1;                           /* unbiased exponent -6..8 */
    float m = rintf(ldexpf(a, 3 - e));        /* significand in eighths: [8, 16) */
    if (m == 16.0f) { e += 1; m = 8.0f; }
    int code = ((e + 7) << 3) | ((int)m - 8);
    if (code > 0x7E) code = 0x7E;
    return (uint8_t)code;
}

double orc_e4m3_decode(uint8_t code) {
    int e = (code >> 3) & 0xF, m = code & 7;
    double mag = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return (code & 0x80) ? -mag : mag;
}

float orc_bf16_to_f32(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return f;
}

void orc_e2m1_encode_array(const float* v, uint8_t* out, int64_t n) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e2m1_encode(v[i]);
}

void orc_e4m3_encode_array(const float* v, uint8_t* out, int64_t n) {
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = orc_e4m3_encode(v[i]);
}

/* ------------------------------------------------------------------------ */
/* Scale layout: 128-row x 4-column tiles of 512 bytes, tiles ordered with
 * the scale-column tile fastest.  Inside a tile, row r and column c sit at
 * (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4).  This is the block-scale
 * layout of the Blackwell block-scaled MMA (checked on the GPU by a library
 * NVFP4 GEMM reading these bytes); the pages do not describe it.            */

int64_t orc_scale_rows(int64_t rows) { return (rows + 127) / 128 * 128; }
int64_t orc_scale_cols(int64_t k) { return (k / 16 + 3) / 4 * 4; }

int64_t orc_sf_offset(int64_t r, int64_t c, int64_t scale_cols) {
    int64_t tile = (r / 128) * (scale_cols / 4) + c / 4;
    return tile * 512 + (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4);
}

/* ------------------------------------------------------------------------ */
/* Global scale: the FP32 tensor scale maps the largest block onto the top of
 * the E4M3 range, so that block_scale = block_amax / (6 * g) <= 448.  It is
 * kept as a decode multiplier (reconstructed = fp4 x block_scale x g).      */

float orc_global_scale(float amax) {
    return (amax == 0.0f) ? 1.0f : amax / 2688.0f;   /* 2688 = 6 * 448 */
}

/* One scale block: values xv[0..n), sharing block amax bamax.  Writes n codes
 * (unpacked, one per byte) and returns the E4M3 scale byte.
 *
 * Each code is the E2M1 value nearest x / d, d = decode(sf) * g, the divisor
 * that the reconstruction fp4 x block_scale x global_scale implies ("NVFP4
 * Explained", "How NVFP4 Represents a Value").  The quotient is formed as
 * x * r with r = 1 / d, each rounded to binary32's 24-bit significand.  When
 * 1 / d is too large for binary32 (d at or below 2^-128, so g below about
 * 2^-119), the same two roundings are done one exponent range lower: d and x
 * are first multiplied by 2^64, which leaves the quotient unchanged and is
 * exact for d (d * 2^64 is a normal number).  x * 2^64 or the product can
 * overflow only where x / d is far above 6, which saturates to 6 either way;
 * with g from the tensor's own amax, x is below 2^-100 there and nothing
 * overflows. */
static uint8_t quantize_block(const float* xv, int n, float bamax, float g, uint8_t* code_out) {
    const float two64 = 18446744073709551616.0f;   /* 2^64 */
    float k6 = 6.0f * g;
    uint8_t sf = orc_e4m3_encode(bamax / k6);
    float d = (float)orc_e4m3_decode(sf) * g;      /* decoded block scale times g */
    if (d == 0.0f) {                                /* zero block scale: every magnitude is 0 */
        for (int i = 0; i < n; ++i) code_out[i] = orc_e2m1_encode(xv[i] * 0.0f);
        return sf;
    }
    float r = 1.0f / d;
    if (isinf(r)) {
        float r64 = 1.0f / (d * two64);            /* r / 2^64 */
        for (int i = 0; i < n; ++i) code_out[i] = orc_e2m1_encode((xv[i] * two64) * r64);
    } else {
        for (int i = 0; i < n; ++i) code_out[i] = orc_e2m1_encode(xv[i] * r);
    }
    return sf;
}

static int check_finite_rows(const uint16_t* x, int64_t r0, int64_t r1, int64_t k, int64_t ld) {
    int bad = 0;
    #pragma omp parallel for reduction(|:bad) schedule(static)
    for (int64_t r = r0; r < r1; ++r)
        for (int64_t j = 0; j < k; ++j)
            if (!isfinite(orc_bf16_to_f32(x[r * ld + j]))) bad = 1;
    return bad;
}

static float amax_rows(const uint16_t* x, int64_t r0, int64_t r1, int64_t k, int64_t ld) {
    float amax = 0.0f;
    #pragma omp parallel for reduction(max:amax) schedule(static)
    for (int64_t r = r0; r < r1; ++r)
        for (int64_t j = 0; j < k; ++j) {
            float a = fabsf(orc_bf16_to_f32(x[r * ld + j]));
            if (a > amax) amax = a;
        }
    return amax;
}

/* 1D quantization of rows [r0, r1) with global scale g; their scale rows
 * start at sf_row0 (scale row of row r is sf_row0 + r - r0).                */
static void quantize_rows_1d(const uint16_t* x, int64_t r0, int64_t r1, int64_t k, int64_t ld,
                             float g, uint8_t* codes, uint8_t* sf, int64_t sf_row0) {
    int64_t scale_cols = orc_scale_cols(k);
    #pragma omp parallel for schedule(static)
    for (int64_t r = r0; r < r1; ++r) {
        for (int64_t b = 0; b < k / 16; ++b) {
            float xv[16];
            uint8_t c[16];
            float bamax = 0.0f;
            for (int i = 0; i < 16; ++i) {
                xv[i] = orc_bf16_to_f32(x[r * ld + b * 16 + i]);
                if (fabsf(xv[i]) > bamax) bamax = fabsf(xv[i]);
            }
            uint8_t s = quantize_block(xv, 16, bamax, g, c);
            sf[orc_sf_offset(sf_row0 + (r - r0), b, scale_cols)] = s;
            for (int i = 0; i < 8; ++i)
                codes[r * (k / 2) + b * 8 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
        }
    }
}

int orc_quantize_1d(const uint16_t* x, int64_t rows, int64_t k, int64_t ld,
                    uint8_t* codes, uint8_t* sf, float* g_out) {
    if (rows < 0 || k <= 0 || k % 16 != 0 || ld < k) return 1;
    if (check_finite_rows(x, 0, rows, k, ld)) return 2;
    memset(sf, 0, (size_t)(orc_scale_rows(rows) * orc_scale_cols(k)));
    float g = orc_global_scale(amax_rows(x, 0, rows, k, ld));
    quantize_rows_1d(x, 0, rows, k, ld, g, codes, sf, 0);
    *g_out = g;
    return 0;
}

/* SmoothQuant-style per-channel pre-scaling folded into the 1D quantizer:
 * the values quantized are x'[r][c] = fp32(x[r][c]) * s[c] (one IEEE
 * product), and every step of orc_quantize_1d then runs on x' (amax, global
 * scale, block amax, block scale, codes).  s: k positive finite factors;
 * every product must be finite. */
int orc_quantize_1d_smooth(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, const float* s,
                           uint8_t* codes, uint8_t* sf, float* g_out) {
    if (rows < 0 || k <= 0 || k % 16 != 0 || ld < k) return 1;
    for (int64_t j = 0; j < k; ++j)
        if (!(s[j] > 0.0f) || !isfinite(s[j])) return 1;
    if (check_finite_rows(x, 0, rows, k, ld)) return 2;
    float amax = 0.0f;
    int bad = 0;
    #pragma omp parallel for reduction(max:amax) reduction(|:bad) schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < k; ++j) {
            float v = orc_bf16_to_f32(x[r * ld + j]) * s[j];
            if (!isfinite(v)) bad = 1;
            if (fabsf(v) > amax) amax = fabsf(v);
        }
    if (bad) return 2;
    float g = orc_global_scale(amax);
    int64_t scale_cols = orc_scale_cols(k);
    memset(sf, 0, (size_t)(orc_scale_rows(rows) * scale_cols));
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < k / 16; ++b) {
            float xv[16];
            uint8_t c[16];
            float bamax = 0.0f;
            for (int i = 0; i < 16; ++i) {
                xv[i] = orc_bf16_to_f32(x[r * ld + b * 16 + i]) * s[b * 16 + i];
                if (fabsf(xv[i]) > bamax) bamax = fabsf(xv[i]);
            }
            sf[orc_sf_offset(r, b, scale_cols)] = quantize_block(xv, 16, bamax, g, c);
            for (int i = 0; i < 8; ++i)
                codes[r * (k / 2) + b * 8 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
        }
    }
    *g_out = g;
    return 0;
}

int64_t orc_grouped_scale_rows(const int32_t* off, int num_groups) {
    int64_t t = 0;
    for (int e = 0; e < num_groups; ++e) t += orc_scale_rows((int64_t)off[e + 1] - off[e]);
    return t;
}

/* The same block quantizer with the global scale g given by the caller: the
   second pass of a two-phase form whose amax was taken elsewhere (by the GEMM
   that produced x).  g must be positive and finite. */
int orc_quantize_1d_given_g(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, float g,
                            uint8_t* codes, uint8_t* sf) {
    if (rows < 0 || k <= 0 || k % 16 != 0 || ld < k || !(g > 0.0f) || !isfinite(g)) return 1;
    if (check_finite_rows(x, 0, rows, k, ld)) return 2;
    memset(sf, 0, (size_t)(orc_scale_rows(rows) * orc_scale_cols(k)));
    quantize_rows_1d(x, 0, rows, k, ld, g, codes, sf, 0);
    return 0;
}

int orc_quantize_1d_grouped(const uint16_t* x, const int32_t* off, int num_groups,
                            int64_t k, int64_t ld, uint8_t* codes, uint8_t* sf,
                            float* g_out) {
    if (num_groups <= 0 || k <= 0 || k % 16 != 0 || ld < k || off[0] < 0) return 1;
    for (int e = 0; e < num_groups; ++e)
        if (off[e + 1] < off[e]) return 1;
    if (check_finite_rows(x, off[0], off[num_groups], k, ld)) return 2;
    memset(sf, 0, (size_t)(orc_grouped_scale_rows(off, num_groups) * orc_scale_cols(k)));
    int64_t sf_row0 = 0;
    for (int e = 0; e < num_groups; ++e) {
        float g = orc_global_scale(amax_rows(x, off[e], off[e + 1], k, ld));
        quantize_rows_1d(x, off[e], off[e + 1], k, ld, g, codes, sf, sf_row0);
        g_out[e] = g;
        sf_row0 += orc_scale_rows((int64_t)off[e + 1] - off[e]);
    }
    return 0;
}

/* 2D quantization ("What is NVFP4?", "Why does scaling matter so much?":
 * 16 x 16 weight blocks share one scale).  The tile's scale is stored for
 * each of its 16 rows in the tensor-core layout.                            */
int orc_quantize_2d(const uint16_t* x, int64_t rows, int64_t k, int64_t ld,
                    uint8_t* codes, uint8_t* sf, uint8_t* sf_compact, float* g_out) {
    if (rows < 0 || rows % 16 != 0 || k <= 0 || k % 16 != 0 || ld < k) return 1;
    if (check_finite_rows(x, 0, rows, k, ld)) return 2;
    int64_t scale_cols = orc_scale_cols(k);
    memset(sf, 0, (size_t)(orc_scale_rows(rows) * scale_cols));
    float g = orc_global_scale(amax_rows(x, 0, rows, k, ld));
    #pragma omp parallel for schedule(static)
    for (int64_t tr = 0; tr < rows / 16; ++tr) {
        for (int64_t b = 0; b < k / 16; ++b) {
            float xv[256];
            uint8_t c[256];
            float bamax = 0.0f;
            for (int i = 0; i < 16; ++i)
                for (int j = 0; j < 16; ++j) {
                    float v = orc_bf16_to_f32(x[(tr * 16 + i) * ld + b * 16 + j]);
                    xv[i * 16 + j] = v;
                    if (fabsf(v) > bamax) bamax = fabsf(v);
                }
            uint8_t s = quantize_block(xv, 256, bamax, g, c);
            if (sf_compact) sf_compact[tr * (k / 16) + b] = s;
            for (int i = 0; i < 16; ++i) {
                int64_t r = tr * 16 + i;
                sf[orc_sf_offset(r, b, scale_cols)] = s;
                for (int j = 0; j < 8; ++j)
                    codes[r * (k / 2) + b * 8 + j] =
                        (uint8_t)(c[i * 16 + 2 * j] | (c[i * 16 + 2 * j + 1] << 4));
            }
        }
    }
    *g_out = g;
    return 0;
}

/* ------------------------------------------------------------------------ */
/* Reconstruction ("NVFP4 Explained", "How NVFP4 Represents a Value"):
 * reconstructed = fp4_value x block_scale x global_scale.  The product has at
 * most 2 + 4 + 24 significant bits, so it is exact in binary64.             */
void orc_dequantize(const uint8_t* codes, const uint8_t* sf, float g,
                    int64_t rows, int64_t k, int64_t sf_row0, int64_t scale_cols,
                    double* out) {
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < k; ++j) {
            uint8_t byte = codes[r * (k / 2) + j / 2];
            uint8_t code = (j % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            double s = orc_e4m3_decode(sf[orc_sf_offset(sf_row0 + r, j / 16, scale_cols)]);
            out[r * k + j] = orc_e2m1_decode(code) * s * (double)g;
        }
}

/* ------------------------------------------------------------------------ */
/* W4A4 GEMM over the reconstructed operands, C = A_hat * W_hat^T, binary64
 * accumulation in k order.                                                   */
void orc_gemm_f64(const double* a_hat, const double* w_hat,
                  int64_t m, int64_t n, int64_t k, double* c) {
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < m; ++i)
        for (int64_t j = 0; j < n; ++j) {
            double acc = 0.0;
            for (int64_t t = 0; t < k; ++t) acc += a_hat[i * k + t] * w_hat[j * k + t];
            c[i * n + j] = acc;
        }
}

void orc_gemm_f64_rows(const double* a_hat, const double* w_hat, const int64_t* rows_sel,
                       int64_t n_rows_sel, int64_t n, int64_t k, double* c) {
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < n_rows_sel; ++i)
        for (int64_t j = 0; j < n; ++j) {
            double acc = 0.0;
            const double* a = a_hat + rows_sel[i] * k;
            for (int64_t t = 0; t < k; ++t) acc += a[t] * w_hat[j * k + t];
            c[i * n + j] = acc;
        }
}

/* Integer forms: 2 * e2m1 value and 2^9 * e4m3 value are integers.          */
static int64_t e2m1_times2(uint8_t code) {
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    int64_t v = (e == 0) ? m : (int64_t)(2 + m) << (e - 1);
    return s ? -v : v;
}
static int64_t e4m3_times512(uint8_t code) {
    int e = (code >> 3) & 0xF, m = code & 7;
    return (e == 0) ? m : (int64_t)(8 + m) << (e - 1);
}

void orc_gemm_exact_i64(const uint8_t* a_codes, const uint8_t* a_sf,
                        const uint8_t* w_codes, const uint8_t* w_sf,
                        int64_t m, int64_t n, int64_t k, int64_t* c) {
    int64_t sc_a = orc_scale_cols(k), sc_w = sc_a;
    #pragma omp parallel for collapse(2) schedule(static)
    for (int64_t i = 0; i < m; ++i)
        for (int64_t j = 0; j < n; ++j) {
            int64_t acc = 0;
            for (int64_t t = 0; t < k; ++t) {
                uint8_t ba = a_codes[i * (k / 2) + t / 2], bw = w_codes[j * (k / 2) + t / 2];
                uint8_t ca = (t % 2 == 0) ? (ba & 0xF) : (ba >> 4);
                uint8_t cw = (t % 2 == 0) ? (bw & 0xF) : (bw >> 4);
                int64_t va = e2m1_times2(ca) * e4m3_times512(a_sf[orc_sf_offset(i, t / 16, sc_a)]);
                int64_t vw = e2m1_times2(cw) * e4m3_times512(w_sf[orc_sf_offset(j, t / 16, sc_w)]);
                acc += va * vw;
            }
            c[i * n + j] = acc;
        }
}

/* ------------------------------------------------------------------------ */
/* Single-scale FP4 baseline ("NVFP4 Explained", "Why Blocks of 16 Improve
 * Accuracy": one scale over many values lets an outlier stretch the range).
 * One FP32 scale amax/6 for the whole tensor, no block scales.              */
void orc_single_scale_fp4(const uint16_t* x, int64_t n, double* x_hat) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(orc_bf16_to_f32(x[i]));
        if (a > amax) amax = a;
    }
    float s = amax / 6.0f;
    for (int64_t i = 0; i < n; ++i) {
        if (s == 0.0f) { x_hat[i] = 0.0; continue; }
        uint8_t code = orc_e2m1_encode(orc_bf16_to_f32(x[i]) / s);
        x_hat[i] = orc_e2m1_decode(code) * (double)s;
    }
}

/* ------------------------------------------------------------------------ */
/* MXFP4, the other four-bit format of the same tensor cores.  "NVFP4
 * Explained: NVIDIA's 4-Bit Format for Faster AI Inference", "Why Blocks of
 * 16 Improve Accuracy" and "Why the Block Scale Uses FP8 E4M3"; "What is
 * NVFP4?", "NVFP4 versus MXFP4": the same E2M1 elements, one E8M0 scale --
 * a bare power of two, 2^(byte - 127) -- shared by 32 values, and no
 * tensor-wide scale.  How the power is chosen is not on the pages.  Reading
 * used here: the smallest 2^e with 6 * 2^e >= block amax, so that the block
 * maximum fits the E2M1 range without saturating (NVFP4's block scale puts
 * it exactly on 6), with e clamped to [-127, 127]; a block of zeros takes
 * byte 0.  code = E2M1_RNE(x / 2^e), sign kept.  Scale bytes use the same
 * 128 x 4 tiles, one scale column per 32 values.                            */

int64_t orc_mx_scale_cols(int64_t k) { return (k / 32 + 3) / 4 * 4; }

uint8_t orc_e8m0_block_scale(double bamax) {
    int e = -127;
    while (e < 127 && 6.0 * ldexp(1.0, e) < bamax) ++e;   /* smallest e that holds the block */
    return (uint8_t)(e + 127);
}

double orc_e8m0_decode(uint8_t b) { return ldexp(1.0, (int)b - 127); }   /* 0xFF (NaN) never produced */

int orc_quantize_1d_mx(const uint16_t* x, int64_t rows, int64_t k, int64_t ld,
                       uint8_t* codes, uint8_t* sf) {
    if (rows < 0 || k <= 0 || k % 32 != 0 || ld < k) return 1;
    if (check_finite_rows(x, 0, rows, k, ld)) return 2;
    int64_t scale_cols = orc_mx_scale_cols(k);
    memset(sf, 0, (size_t)(orc_scale_rows(rows) * scale_cols));
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
        for (int64_t b = 0; b < k / 32; ++b) {
            double xv[32];
            double bamax = 0.0;
            for (int i = 0; i < 32; ++i) {
                xv[i] = (double)orc_bf16_to_f32(x[r * ld + b * 32 + i]);
                if (fabs(xv[i]) > bamax) bamax = fabs(xv[i]);
            }
            uint8_t s = orc_e8m0_block_scale(bamax);
            double scale = orc_e8m0_decode(s);
            sf[orc_sf_offset(r, b, scale_cols)] = s;
            uint8_t c[32];
            /* x / 2^e is exact in binary64; its binary32 rounding only touches
             * magnitudes far below 0.25, which encode to (signed) zero anyway */
            for (int i = 0; i < 32; ++i) c[i] = orc_e2m1_encode((float)(xv[i] / scale));
            for (int i = 0; i < 16; ++i)
                codes[r * (k / 2) + b * 16 + i] = (uint8_t)(c[2 * i] | (c[2 * i + 1] << 4));
        }
    }
    return 0;
}

void orc_dequantize_mx(const uint8_t* codes, const uint8_t* sf, int64_t rows, int64_t k, double* out) {
    int64_t scale_cols = orc_mx_scale_cols(k);
    #pragma omp parallel for schedule(static)
    for (int64_t r = 0; r < rows; ++r)
        for (int64_t j = 0; j < k; ++j) {
            uint8_t byte = codes[r * (k / 2) + j / 2];
            uint8_t code = (j % 2 == 0) ? (byte & 0xF) : (byte >> 4);
            out[r * k + j] = orc_e2m1_decode(code) * orc_e8m0_decode(sf[orc_sf_offset(r, j / 32, scale_cols)]);
        }
}
