/*
 * nvfp4_oracle.h -- plain, slow CPU oracle for NVFP4 W4A4 quantization and
 * the block-scaled FP4 x FP4 GEMM.
 *
 * TEST INFRASTRUCTURE ONLY.  Only tests/, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant with the CUDA path, and the CUDA path never
 * calls it.
 *
 * What it follows (page title, section):
 *   - "What is NVFP4? 4-bit AI inference on NVIDIA Blackwell explained",
 *     "What does NVFP4 mean?": E2M1 = 1 sign, 2 exponent, 1 mantissa bit,
 *     magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6}; value = E2M1 x local FP8
 *     (E4M3) scale x global FP32 scale.
 *   - same page, "Why does scaling matter so much?": one scale per
 *     16-element block for activations (1D); 16 x 16 blocks for weights (2D).
 *   - "NVFP4 Explained: NVIDIA's 4-Bit Format for Faster AI Inference",
 *     "How NVFP4 Represents a Value": reconstructed = fp4 x block_scale x
 *     global_scale; "Why the Block Scale Uses FP8 E4M3": the FP32 tensor
 *     scale restores the range E4M3 lacks.
 *   - "Accelerating large language models with NVFP4 quantization",
 *     Figure 1: group size 16, FP8 group scale, FP32 tensor-level scale.
 *   - "W4A8 vs NVFP4 quantization on GPUs", "Scale layout changes the real
 *     storage cost": 8/16 = 0.5 bit of scale per value, 4.5 bits per value
 *     plus one FP32 per tensor.
 *
 * Readings where the pages are silent (each listed in the design notes):
 *   g  = amax / (6 * 448) as a decode multiplier (1.0 when amax == 0);
 *   sf = E4M3_RNE_satfinite(block_amax / (6 * g));
 *   d  = decode(sf) * g;  r = 1 / d (0 when d == 0);
 *   code = E2M1_RNE_satfinite(x * r), sign bit kept (also for zero); r and
 *   x * r are rounded to binary32's 24-bit significand without binary32's
 *   exponent ceiling: where 1 / d overflows, d and x are scaled by 2^64
 *   first, so the code stays the one nearest x / d;
 *   element 2i in bits 3:0 of byte i, element 2i+1 in bits 7:4;
 *   scales stored in 128-row x 4-column tiles of 512 bytes (tensor-core
 *   block-scale layout), pad bytes zero.
 *
 * Also: the quantize steps with g given (two-phase form); the quantizer of
 * x * s[column] (per-column pre-scaling, one binary32 product); MXFP4 --
 * "What is NVFP4?", "NVFP4 versus MXFP4": E2M1 codes, one E8M0 power-of-two
 * scale per 32 values, no tensor scale, the power read as the smallest 2^e
 * with 6 * 2^e >= block amax.
 *
 * Every float operation is a single IEEE-754 binary32 operation rounded to
 * nearest even (built with -ffp-contract=off, no fast-math); the MXFP4
 * scaling x / 2^e is done in binary64, where it is exact.
 */
#ifndef NVFP4_ORACLE_H
#define NVFP4_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- element formats ---------------------------------------------------- */
uint8_t orc_e2m1_encode(float v);            /* 4-bit code, RNE, saturate at 6 */
double  orc_e2m1_decode(uint8_t code);       /* low 4 bits used */
uint8_t orc_e4m3_encode(float a);            /* a >= 0 (sign ignored), RNE, saturate at 448 */
double  orc_e4m3_decode(uint8_t code);       /* 0x7F (NaN) never produced */
float   orc_bf16_to_f32(uint16_t bits);

void orc_e2m1_encode_array(const float* v, uint8_t* out, int64_t n);
void orc_e4m3_encode_array(const float* v, uint8_t* out, int64_t n);

/* ---- scale layout --------------------------------------------------------- */
int64_t orc_scale_rows(int64_t rows);        /* rows rounded up to 128 */
int64_t orc_scale_cols(int64_t k);           /* k/16 rounded up to 4 */
int64_t orc_sf_offset(int64_t r, int64_t c, int64_t scale_cols);

/* ---- quantizers ------------------------------------------------------------
 * x: BF16 bit patterns, row-major with leading dimension ld (elements).
 * codes: [rows, k/2] bytes.  sf: orc_scale_rows(rows) * orc_scale_cols(k)
 * bytes (whole buffer written, pads zero).  Return 0 on success, nonzero on
 * an invalid argument or a non-finite input.                               */
float orc_global_scale(float amax);
int orc_quantize_1d(const uint16_t* x, int64_t rows, int64_t k, int64_t ld,
                    uint8_t* codes, uint8_t* sf, float* g_out);
/* Groups of rows [off[e], off[e+1]); group e has its own g and its scale rows
 * start at sum_{j<e} orc_scale_rows(off[j+1]-off[j]).  sf must hold
 * orc_grouped_scale_rows(...) * orc_scale_cols(k) bytes.                    */
int64_t orc_grouped_scale_rows(const int32_t* off, int num_groups);
/* 1D quantization with a caller-given global scale g (> 0, finite). */
int orc_quantize_1d_given_g(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, float g,
                            uint8_t* codes, uint8_t* sf);
/* 1D quantization of x'[r][c] = fp32(x[r][c]) * s[c] (per-channel pre-scaling, SmoothQuant style). */
int orc_quantize_1d_smooth(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, const float* s,
                           uint8_t* codes, uint8_t* sf, float* g_out);
int orc_quantize_1d_grouped(const uint16_t* x, const int32_t* off, int num_groups,
                            int64_t k, int64_t ld, uint8_t* codes, uint8_t* sf,
                            float* g_out);
/* 16x16 blocks; rows % 16 == 0.  sf_compact (optional) is [rows/16, k/16]. */
int orc_quantize_2d(const uint16_t* x, int64_t rows, int64_t k, int64_t ld,
                    uint8_t* codes, uint8_t* sf, uint8_t* sf_compact, float* g_out);

/* ---- reconstruction: x_hat = e2m1 x e4m3 x g (exact in binary64) --------- */
void orc_dequantize(const uint8_t* codes, const uint8_t* sf, float g,
                    int64_t rows, int64_t k, int64_t sf_row0, int64_t scale_cols,
                    double* out);

/* ---- GEMM: C[m,n] = sum_k a_hat[m,k] * w_hat[n,k], binary64 --------------- */
void orc_gemm_f64(const double* a_hat, const double* w_hat,
                  int64_t m, int64_t n, int64_t k, double* c);
/* Selected rows only: C[i, n] for m = rows_sel[i]. */
void orc_gemm_f64_rows(const double* a_hat, const double* w_hat, const int64_t* rows_sel,
                       int64_t n_rows_sel, int64_t n, int64_t k, double* c);
/* Exact integer form: sum_k (qa*sfa)*(qw*sfw) * 2^20 as int64 (no global
 * scales).  Every product is a multiple of 2^-20 below 2^23 in magnitude.   */
void orc_gemm_exact_i64(const uint8_t* a_codes, const uint8_t* a_sf,
                        const uint8_t* w_codes, const uint8_t* w_sf,
                        int64_t m, int64_t n, int64_t k, int64_t* c);

/* ---- single-scale FP4 baseline: one scale amax/6, no block scales -------- */
void orc_single_scale_fp4(const uint16_t* x, int64_t n, double* x_hat);

/* ---- MXFP4: E2M1 elements, one E8M0 power-of-two scale per 32 values, no
 * tensor scale; scale = smallest 2^e with 6 * 2^e >= block amax (reading),
 * e in [-127, 127].  k % 32 == 0.  Scales in the 128 x 4 tile layout with
 * orc_mx_scale_cols(k) = k/32 rounded up to 4 columns.                      */
int64_t orc_mx_scale_cols(int64_t k);
uint8_t orc_e8m0_block_scale(double bamax);
double  orc_e8m0_decode(uint8_t b);
int orc_quantize_1d_mx(const uint16_t* x, int64_t rows, int64_t k, int64_t ld,
                       uint8_t* codes, uint8_t* sf);
void orc_dequantize_mx(const uint8_t* codes, const uint8_t* sf, int64_t rows, int64_t k, double* out);

int orc_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
