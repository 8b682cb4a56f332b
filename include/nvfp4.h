/*
 * nvfp4.h -- C ABI of libnvfp4.so: NVFP4 W4A4 inference on NVIDIA B200
 * (sm_100a).  Two stages: dynamic NVFP4 quantization of BF16 tensors, and a
 * block-scaled FP4 x FP4 GEMM on the tcgen05 tensor cores.
 *
 * Format (all entry points):
 *   Element: E2M1, 1 sign / 2 exponent / 1 mantissa bit, magnitudes
 *     {0, 0.5, 1, 1.5, 2, 3, 4, 6} ("What is NVFP4? 4-bit AI inference on
 *     NVIDIA Blackwell explained", "What does NVFP4 mean?").
 *   Block scale: FP8 E4M3, one per 16 consecutive values along K (1D), or one
 *     per 16 x 16 tile for weights (2D) (same page, "Why does scaling matter
 *     so much?"; "NVFP4 Explained: NVIDIA's 4-Bit Format for Faster AI
 *     Inference", "Why the Block Scale Uses FP8 E4M3").
 *   Tensor scale: one FP32 per tensor (or per group), kept as a decode
 *     multiplier:  reconstructed = fp4 x block_scale x global_scale
 *     ("NVFP4 Explained", "How NVFP4 Represents a Value").
 *   Readings where the pages are silent:
 *     global_scale g = amax / (6 * 448), or 1 when amax == 0;
 *     block scale   = E4M3_rne_satfinite(block_amax / (6 * g));
 *     code          = E2M1_rne_satfinite(x * r), r = 1 / (block_scale * g),
 *                     r = 0 when block_scale * g == 0; the sign bit of x is
 *                     kept, also for zero codes.  r and x * r are rounded
 *                     to binary32's 24-bit significand without binary32's
 *                     exponent ceiling, so the code is the one nearest
 *                     x / (block_scale * g) even where 1 / (block_scale * g)
 *                     overflows binary32 (a global scale below ~2^-119).
 *   Storage: codes [rows, k/2] bytes, row-major, element 2i in bits 3:0 and
 *     element 2i+1 in bits 7:4 of byte i -- 4 bits per value; scales 1 byte
 *     per 16 values; 4.5 bits per value plus 4 bytes per tensor ("W4A8 vs
 *     NVFP4 quantization on GPUs", "Scale layout changes the real storage
 *     cost").
 *   Scale layout (not on the pages; the block-scale layout of the sm_100
 *   block-scaled MMA, which the tests also check by having a library NVFP4
 *   GEMM, cuBLASLt through torch's scaled_mm, read these bytes):
 *     rows padded to a multiple of 128, scale columns (k/16) padded to a
 *     multiple of 4, stored as 512-byte tiles of 128 rows x 4 columns, tiles
 *     ordered row-tile major, column-tile minor; inside a tile row r and
 *     column c sit at byte (r % 32) * 16 + ((r % 128) / 32) * 4 + (c % 4).
 *     Pad bytes are written as zero.
 *
 * Conventions:
 *   - Every buffer is owned by the caller.  Pointers marked "device" must be
 *     device memory of the current device; all device pointers must be
 *     16-byte aligned.  No entry point allocates device memory.
 *   - stream is a cudaStream_t (NULL = legacy default stream).  All compute
 *     entry points are asynchronous on it; argument errors are returned
 *     before anything is launched.  Device-side failures (a bounded wait
 *     that ran out) are reported by nvfp4_get_last_device_error.
 *   - Global scales and group offsets stay on the device: no call waits on
 *     the host for them.
 *   - workspace: device scratch of nvfp4_workspace_bytes(...) bytes, for one
 *     device.  It must be zero before its first use (nvfp4_workspace_init);
 *     after that, leave it untouched between calls: every call that returns
 *     NVFP4_OK leaves it ready for the next (the one-tensor quantizer keeps a
 *     per-CTA generation count in it; the GEMM returns its hand-off counters
 *     to zero).  Calls sharing one workspace must be ordered on one stream.
 *     After NVFP4_ERR_TIMEOUT, zero it again.
 */
#ifndef NVFP4_H
#define NVFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARGUMENT = 1,  /* null pointer, negative size, bad group offsets count */
    NVFP4_ERR_UNSUPPORTED_SHAPE = 2, /* k % 16 (quantize) or k % 64 (GEMM) != 0, n % 16 != 0 (2D), too large */
    NVFP4_ERR_MISALIGNED = 3,        /* a device pointer or leading dimension breaks 16-byte alignment */
    NVFP4_ERR_CUDA = 4,              /* a CUDA runtime call failed (launch, driver entry point) */
    NVFP4_ERR_TIMEOUT = 5,           /* a kernel's bounded wait ran out; results are invalid */
    NVFP4_ERR_NO_DEVICE = 6          /* no sm_100 device current */
} nvfp4_status_t;

/* Status code -> static string.  Never NULL. */
const char* nvfp4_status_string(nvfp4_status_t status);

/* Library version, "major.minor.patch". */
const char* nvfp4_version(void);

/* ---- sizes --------------------------------------------------------------- */

/* Bytes of packed E2M1 codes for a [rows, k] tensor: rows * k / 2. */
size_t nvfp4_codes_bytes(int64_t rows, int64_t k);

/* Bytes of the tiled E4M3 scale buffer for a [rows, k] tensor:
 * ceil(rows / 128) * 128 * ceil(k / 64) * 4. */
size_t nvfp4_scale_bytes(int64_t rows, int64_t k);

/* Upper bound of the scale buffer for grouped quantization of total_rows rows
 * in num_groups groups: each group's scale rows start at a multiple of 128,
 * so at most ((total_rows + 127 * num_groups) / 128) * 128 rows of scales. */
size_t nvfp4_grouped_scale_bytes(int64_t total_rows, int num_groups, int64_t k);

/* Workspace bytes an operation needs (operations below); 0 if none. */
enum { NVFP4_OP_QUANTIZE_ACT = 0, NVFP4_OP_QUANTIZE_WEIGHT_2D = 1, NVFP4_OP_GEMM = 2,
       NVFP4_OP_GROUPED_GEMM = 3, NVFP4_OP_GEMM_EMIT_SCALE = 4, NVFP4_OP_QUANTIZE_GEMM = 5 };
size_t nvfp4_workspace_bytes(int op, int64_t rows, int64_t n, int64_t k, int num_groups);

/* Zero a workspace before its first use (cudaMemsetAsync on stream). */
nvfp4_status_t nvfp4_workspace_init(void* workspace, size_t bytes, void* stream);

/* ---- stage 1: dynamic quantization ----------------------------------------
 *
 * nvfp4_quantize_act -- 1D 16-element blocks, global scale from the tensor
 * amax computed in the same call (dynamic activation quantization: "NVFP4
 * Dynamic Quantization in Practice", "The Meaning and Advantages of W4A4";
 * "NVFP4 Explained", FAQ "Can NVFP4 quantize both weights and activations?").
 *
 *   x            device, BF16 [rows, k] with row stride ld elements (ld >= k,
 *                ld % 8 == 0).  Finite values only (NaN/Inf: undefined codes).
 *   rows, k      rows >= 0, k > 0, k % 16 == 0.
 *   group_offsets NULL: one tensor.  Otherwise device int32 [num_groups + 1],
 *                non-decreasing, offsets[0] >= 0, offsets[num_groups] <= rows:
 *                rows [offsets[e], offsets[e+1]) form group e with its own
 *                global scale; group e's scale rows start at
 *                sum_{j<e} ceil128(offsets[j+1] - offsets[j]).  Rows outside
 *                [offsets[0], offsets[num_groups]) are not touched.
 *                The offsets are not validated on the device.
 *   codes        device, nvfp4_codes_bytes(rows, k) bytes.
 *   scales       device, nvfp4_scale_bytes(rows, k) bytes (one tensor) or
 *                nvfp4_grouped_scale_bytes(rows, num_groups, k) (grouped);
 *                every byte of each group's padded scale block is written.
 *   global_scale device, FP32 [max(1, num_groups)].
 *   workspace    nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE_ACT, rows, 0, k, num_groups).
 * When k % 64 == 0 (and, with groups, num_groups <= 1024): one cooperative
 * launch, one CTA per SM -- an amax pass (per group, folded into the
 * workspace), a grid barrier through the workspace, a quantize pass; the
 * launch waits until every SM can take its CTA.  Otherwise two kernels: a
 * per-group (or whole-tensor) amax reduction, then the quantizer (launched
 * with programmatic dependent launch so its start overlaps the reduction's
 * end).
 * After nvfp4_get_last_device_error reports NVFP4_ERR_TIMEOUT, initialize the
 * workspace again before reusing it.
 */
nvfp4_status_t nvfp4_quantize_act(const void* x, int64_t rows, int64_t k, int64_t ld,
                                  const int32_t* group_offsets, int num_groups,
                                  uint8_t* codes, uint8_t* scales, float* global_scale,
                                  void* workspace, void* stream);

/* nvfp4_quantize_act_smooth -- nvfp4_quantize_act of one tensor with a
 * per-channel pre-scaling folded in (SmoothQuant style: per-channel factors
 * move activation outliers into the weights; the pages discuss such
 * outlier handling next to NVFP4's block scales): the tensor quantized is
 * x'[r][c] = fp32(x[r][c]) * smooth[c] (one IEEE product), and every step --
 * amax, global scale, block scales, codes -- runs on x'.  The weights take
 * the inverse factors before their (offline) quantization.
 *   smooth: device FP32 [k], positive and finite; every product finite.
 *   k % 64 == 0 and k <= 6144 (the factors sit in shared memory); else
 *   NVFP4_ERR_UNSUPPORTED_SHAPE.  Other arguments as nvfp4_quantize_act with
 *   group_offsets NULL (same workspace).  One cooperative launch. */
nvfp4_status_t nvfp4_quantize_act_smooth(const void* x, int64_t rows, int64_t k, int64_t ld,
                                         const float* smooth, uint8_t* codes, uint8_t* scales,
                                         float* global_scale, void* workspace, void* stream);

/* nvfp4_quantize_act_scaled -- the quantize pass of nvfp4_quantize_act with
 * the global scale given (one tensor): codes and scales exactly as
 * nvfp4_quantize_act would write them if the tensor's amax were
 * global_scale[0] * 2688.  With the scale from nvfp4_gemm_emit_scale on the
 * GEMM's own output, the result equals nvfp4_quantize_act of that output,
 * for one read of it instead of two.
 *   x, rows, k, ld, codes, scales: as nvfp4_quantize_act (one tensor).
 *   global_scale: device FP32 [1], > 0 and finite; read, not written.
 * One launch; no workspace.  The launch waits for the previous work on
 * stream (it may be the kernel that wrote x). */
nvfp4_status_t nvfp4_quantize_act_scaled(const void* x, int64_t rows, int64_t k, int64_t ld,
                                         const float* global_scale, uint8_t* codes, uint8_t* scales,
                                         void* stream);

/* nvfp4_quantize_act_static -- nvfp4_quantize_act without the workspace
 * argument: this entry point allocates nothing and takes no scratch from the
 * caller.  The pages have no counterpart; it exists for callers that cannot
 * allocate device memory where they quantize -- a plugin whose host engine
 * owns every byte of device memory and hands out no allocator, or a
 * latency-critical path that may not call cudaMalloc (it can synchronize the
 * whole device).
 *   Scratch: a fixed 49408-byte array in the library's device image (each GPU
 *   that loads the library holds it until the process exits), enough for at
 *   most 1024 row groups; num_groups > 1024 returns
 *   NVFP4_ERR_UNSUPPORTED_SHAPE.
 *   The first call on a device looks up the array's device address with that
 *   device current; make that first call before any stream capture.  The
 *   address is kept for the life of the device's primary context (it does not
 *   survive cudaDeviceReset).
 *   Each call first clears the array with an asynchronous memset on stream;
 *   otherwise it behaves exactly like nvfp4_quantize_act (same arguments,
 *   results, errors).
 *   All calls on a device share the one array and it keeps the last call's
 *   contents: calls that overlap on the GPU (e.g. on two streams without an
 *   ordering between them) race and produce wrong results.
 *   It calls no cudaMalloc, cudaFree or other allocating routine. */
nvfp4_status_t nvfp4_quantize_act_static(const void* x, int64_t rows, int64_t k, int64_t ld,
                                         const int32_t* group_offsets, int num_groups,
                                         uint8_t* codes, uint8_t* scales, float* global_scale,
                                         void* stream);

/* nvfp4_quantize_weight_2d -- 16 x 16 blocks share one E4M3 scale ("What is
 * NVFP4?", "Why does scaling matter so much?").  The tile's scale is written
 * to the tiled scale layout for each of its 16 rows (so the GEMM reads it like
 * 1D scales); scales_compact, if not NULL, receives it once per tile as a
 * row-major [n/16, k/16] byte array.
 *   w: device BF16 [n, k], row stride ld (ld >= k, ld % 8 == 0); n % 16 == 0,
 *   k % 16 == 0.  Other arguments as nvfp4_quantize_act (one tensor). */
nvfp4_status_t nvfp4_quantize_weight_2d(const void* w, int64_t n, int64_t k, int64_t ld,
                                        uint8_t* codes, uint8_t* scales,
                                        uint8_t* scales_compact, float* global_scale,
                                        void* workspace, void* stream);

/* ---- stage 2: block-scaled FP4 x FP4 GEMM ----------------------------------
 *
 * nvfp4_gemm -- C[m, n] = bf16_rn( (sum_k qa[m,k] sa[m,k/16] qb[n,k] sb[n,k/16])
 *                                  * (a_global[0] * b_global[0]) )
 * i.e. the product of the two reconstructed NVFP4 operands ("NVFP4 Explained",
 * "How NVFP4 Represents a Value"), with FP32 accumulation on the tcgen05
 * block-scaled tensor cores (native FP4 x FP4: "NVFP4 Dynamic Quantization in
 * Practice", "Impact on the Open-Source Community and LLM Deployment
 * Industry").  A is [m, k] activations, B is [n, k] weights, both K-major as
 * written by the quantizers above ("TN").
 *   a_codes, a_scales, a_global: device; output of nvfp4_quantize_act on [m, k].
 *   b_codes, b_scales, b_global: device; output of either quantizer on [n, k].
 *   c: device BF16 [m, n], row stride ldc elements (ldc >= n, ldc % 8 == 0).
 *   m >= 0, n > 0, k > 0, k % 64 == 0.  m == 0 reads and writes nothing (the
 *   operand pointers may then be NULL).
 *   workspace: nvfp4_workspace_bytes(NVFP4_OP_GEMM, m, n, k, 0) bytes, 16-byte
 *   aligned, zeroed before first use (see above); NULL is allowed.  For m > 128
 *   the kernel runs on pairs of SMs with 256 x 256 output tiles; when the tiles
 *   do not fill whole waves of pairs, the k-range of the last tiles is shared
 *   out between pairs (stream-K), and a pair hands its FP32 partial sums to the
 *   pair that owns the tile through this workspace (about 19 MB on a B200).
 *   With NULL, or when the size is 0, every tile is computed whole; the result
 *   differs only in the FP32 summation order of those last tiles.
 * For m <= 64 the 128-row MMA side loads only 64 token rows per stage and the
 * weights take the 192-wide side, so that the whole weight matrix streams in
 * one wave: decode is bound by reading the weights ("W4A8 vs NVFP4
 * quantization on GPUs", "Batch size can change the winner"). */
nvfp4_status_t nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global,
                          const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global,
                          void* c, int64_t ldc, int64_t m, int64_t n, int64_t k,
                          void* workspace, void* stream);

/* nvfp4_quantize_gemm -- one W4A4 layer step: dynamic quantization of the
 * BF16 activations x (exactly as nvfp4_quantize_act, one tensor), then
 * C = A_q * B^T as nvfp4_gemm ("NVFP4 Dynamic Quantization in Practice",
 * W4A4: activations quantized on the fly against pre-quantized weights).
 * Results are bit-identical to calling the two entry points in turn.
 * For decode-sized activations (m <= 64) the weights' stream starts while the
 * activations are still being quantized: decode is bound by reading the
 * weights ("W4A8 vs NVFP4 quantization on GPUs", "Batch size can change the
 * winner"), and this call knows that none of its own kernels writes them.
 * So b_codes and b_scales must not be written by the kernel that runs just
 * before this call on the stream (as for any kernel input, the caller orders
 * their producer before the call).
 *   x: device BF16 [m, k], row stride ldx (ldx >= k, ldx % 8 == 0); k % 64 == 0.
 *   b_codes, b_scales, b_global, n, c, ldc: as nvfp4_gemm.
 *   a_codes, a_scales, a_global: receive the quantized activations, as the
 *   outputs of nvfp4_quantize_act (codes [m, k/2], nvfp4_scale_bytes(m, k)
 *   scale bytes, one FP32 global scale).
 *   workspace: nvfp4_workspace_bytes(NVFP4_OP_QUANTIZE_GEMM, m, n, k, 0)
 *   bytes, 16-byte aligned, zeroed before first use; the quantizer's part
 *   first, then the GEMM's.  Calls on one workspace must not overlap.
 *   m == 0 returns NVFP4_OK without launching anything. */
nvfp4_status_t nvfp4_quantize_gemm(const void* x, int64_t m, int64_t k, int64_t ldx, const uint8_t* b_codes,
                                   const uint8_t* b_scales, const float* b_global, int64_t n, void* c, int64_t ldc,
                                   uint8_t* a_codes, uint8_t* a_scales, float* a_global, void* workspace,
                                   void* stream);

/* nvfp4_gemm_emit_scale -- nvfp4_gemm that also takes the amax of its BF16
 * output in the epilogue and writes the global scale the next layer's
 * dynamic quantizer needs: c_global_scale[0] = max|C| / (6 * 448), or 1 when
 * C is all zeros (C as stored, after BF16 rounding).  With
 * nvfp4_quantize_act_scaled it splits dynamic activation quantization into
 * its two passes so that the amax pass costs no read of C: the output-side
 * fusion of the pages' W4A4 pipeline ("NVFP4 Dynamic Quantization in
 * Practice"; the dequantization / extra-pass overhead of "W4A8 vs NVFP4
 * quantization on GPUs").
 *   Arguments as nvfp4_gemm, plus c_global_scale: device FP32 [1].
 *   workspace: nvfp4_workspace_bytes(NVFP4_OP_GEMM_EMIT_SCALE, m, n, k, 0)
 *   bytes, 16-byte aligned, zeroed before first use; required (not NULL).
 *   The first 256 bytes hold a running maximum and a CTA count that every
 *   call returns to zero; the rest serves as nvfp4_gemm's workspace. */
nvfp4_status_t nvfp4_gemm_emit_scale(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global,
                                     const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global,
                                     void* c, int64_t ldc, int64_t m, int64_t n, int64_t k,
                                     float* c_global_scale, void* workspace, void* stream);

/* nvfp4_grouped_gemm -- one GEMM per expert over row groups (mixture of
 * experts: "NVFP4 Dynamic Quantization in Practice", "The Practical
 * Significance of Full Gemma-4 Quantization Coverage").  For expert e, rows
 * [offsets[e], offsets[e+1]) of A (quantized per group by nvfp4_quantize_act
 * with the same offsets) multiply expert e's weights:
 *   C[r, :] = bf16_rn( (A_e[r, :] . B_e^T) * a_global[e] * b_global[e] ).
 *   a_codes [total_rows, k/2]; a_scales grouped layout (see nvfp4_quantize_act);
 *   a_global [num_experts]; offsets device int32 [num_experts + 1] with
 *   offsets[0] == 0 and offsets[num_experts] == total_rows;
 *   b_codes [num_experts, n, k/2]; b_scales num_experts consecutive blocks of
 *   nvfp4_scale_bytes(n, k) bytes; b_global [num_experts];
 *   c BF16 [total_rows, n] (row stride n), rows in grouped order.
 *   Limits, checked before any launch:
 *     k % 64 == 0, 1 <= num_experts <= 256, total_rows < 2^31 and
 *     n * num_experts < 2^31, else NVFP4_ERR_UNSUPPORTED_SHAPE (the per-expert
 *     tile table lives in the kernel's shared memory, 256 entries);
 *     n % 8 == 0 and 16-byte aligned code, scale and output pointers, else
 *     NVFP4_ERR_MISALIGNED (each output row must start on a 16-byte boundary
 *     for the tensor-memory-accelerator store).
 *   The grouped quantizer takes up to 65535 groups, so a layer of more than
 *   256 experts quantizes its activations in one call and splits its GEMM
 *   into calls of at most 256 experts (offsets rebased to the first row of
 *   each call, the A pointers advanced to it).
 *   workspace: unused (NULL accepted). */
nvfp4_status_t nvfp4_grouped_gemm(const uint8_t* a_codes, const uint8_t* a_scales,
                                  const float* a_global, const int32_t* offsets, int num_experts,
                                  const uint8_t* b_codes, const uint8_t* b_scales,
                                  const float* b_global, void* c, int64_t n, int64_t k,
                                  int64_t total_rows, void* workspace, void* stream);

/* ---- MXFP4: the other four-bit format of the same tensor cores --------------
 * "What is NVFP4? 4-bit AI inference on NVIDIA Blackwell explained", "NVFP4
 * versus MXFP4"; "NVFP4 Explained", "Why Blocks of 16 Improve Accuracy" and
 * "Why the Block Scale Uses FP8 E4M3": the same E2M1 elements and nibble
 * packing, one E8M0 scale (a power of two, 2^(byte - 127)) per 32 values
 * along k, and no tensor-wide scale.  Scale bytes use the 128 x 4 tile layout
 * of the NVFP4 scales with one column per 32 values; pad bytes are 0. */

/* Bytes of the tiled E8M0 scale buffer of a [rows, k] MXFP4 tensor:
 * ceil(rows / 128) * 128 * ceil(k / 128) * 4. */
size_t mxfp4_scale_bytes(int64_t rows, int64_t k);

/* mxfp4_quantize_act -- quantize a BF16 [rows, k] tensor (row stride ld
 * elements) to MXFP4.  The pages do not say how the power of two is chosen;
 * here it is the smallest 2^e with 6 * 2^e >= the block's largest magnitude
 * (the block maximum never saturates), e clamped to [-127, 127]; a block of
 * zeros takes byte 0.  code = E2M1 round-to-nearest-even of x / 2^e, sign kept.
 * Activations and weights use the same call (blocks run along k).
 *   codes  device, nvfp4_codes_bytes(rows, k) bytes.
 *   scales device, mxfp4_scale_bytes(rows, k) bytes; every byte written.
 * k % 32 == 0 (else NVFP4_ERR_UNSUPPORTED_SHAPE); x, codes, scales 16-byte
 * aligned and ld % 8 == 0 (else NVFP4_ERR_MISALIGNED).  rows == 0 returns
 * NVFP4_OK at once (pointers may be NULL).  One pass, one launch; no
 * workspace.  The launch waits for the previous work on stream.  NaN/Inf
 * inputs are outside the contract. */
nvfp4_status_t mxfp4_quantize_act(const void* x, int64_t rows, int64_t k, int64_t ld,
                                  uint8_t* codes, uint8_t* scales, void* stream);

/* mxfp4_gemm -- C[m, n] = bf16_rn(sum_k (qa * 2^ea)(qw * 2^ew)) for MXFP4
 * operands from mxfp4_quantize_act: A [m, k], B [n, k] (both K-major), C BF16
 * with row stride ldc.  The same tensor-core kernels and tiling as nvfp4_gemm
 * (the block-scaled MMA with UE8M0 scales, 32-element blocks), FP32
 * accumulation.  Arguments, limits, errors and workspace as nvfp4_gemm
 * (nvfp4_workspace_bytes(NVFP4_OP_GEMM, m, n, k, 0); NULL computes every tile
 * whole), without the global scales. */
nvfp4_status_t mxfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes,
                          const uint8_t* b_scales, void* c, int64_t ldc, int64_t m, int64_t n, int64_t k,
                          void* workspace, void* stream);

/* ---- W4A16: BF16 activations x NVFP4 weights, for decode-sized m --------------
 * The weight-only alternative that "W4A8 vs NVFP4 quantization on GPUs"
 * ("Batch size can change the winner", "Dequantization can erase a four-bit
 * win") weighs against W4A4 at small batch: the same NVFP4 weight stream, the
 * activations kept in BF16, the weights dequantized to BF16 inside the kernel
 * (E2M1 x E4M3, exact) and multiplied on the BF16 tensor cores.
 *
 * w4a16_gemm -- C[m, n] = bf16_rn(b_global * sum_k a[m][k] * (qw[n][k] * sfw)),
 * FP32 accumulation.
 *   a        device BF16 [m, k], row stride lda elements (lda >= k, lda % 8 == 0).
 *   b_codes, b_scales, b_global: NVFP4 weights [n, k] as for nvfp4_gemm (1D or
 *            2D scales), global scale device FP32 [1].
 *   c        device BF16 [m, n], row stride ldc (ldc >= n, ldc % 8 == 0).
 * 0 <= m <= 64 and k % 64 == 0 (else NVFP4_ERR_UNSUPPORTED_SHAPE); a, b_codes,
 * b_scales, c 16-byte aligned (else NVFP4_ERR_MISALIGNED).  m == 0 returns
 * NVFP4_OK at once (pointers may be NULL).  One launch, no workspace; bounded
 * waits as nvfp4_gemm. */
nvfp4_status_t w4a16_gemm(const void* a, int64_t lda, const uint8_t* b_codes, const uint8_t* b_scales,
                          const float* b_global, void* c, int64_t ldc, int64_t m, int64_t n, int64_t k,
                          void* stream);

/* ---- diagnostics ------------------------------------------------------------ */

/* Synchronizes stream, then returns NVFP4_ERR_TIMEOUT if any kernel of this
 * library set its device error word since the last query (and clears it),
 * NVFP4_ERR_CUDA if the stream holds a CUDA error, else NVFP4_OK. */
nvfp4_status_t nvfp4_get_last_device_error(void* stream);

/* Limit, in nanoseconds, of every bounded wait inside the GEMM kernels
 * (mbarrier waits).  Default 2e9 (2 s).  Returns the previous limit.  Used by
 * tests to make a wait run out quickly; not thread-safe. */
uint64_t nvfp4_set_wait_limit_ns(uint64_t limit_ns);

/* Hardware format probes: convert n FP32 values with the same conversion
 * instructions the quantizer uses.  out_e2m1[i] = E2M1 code of in[i] (low
 * nibble); out_e4m3[i] = E4M3 byte of |in[i]|.  Device pointers.  Used to pin
 * the kernels' rounding against the CPU definition over wide sweeps. */
nvfp4_status_t nvfp4_probe_cvt(const float* in, uint8_t* out_e2m1, uint8_t* out_e4m3,
                               int64_t n, void* stream);

/* Waits on a device flag that nothing sets, bounded by limit_ns, and reports
 * the outcome like the GEMM kernels do (sets the device error word).  Lets a
 * test check that a wait which runs out returns NVFP4_ERR_TIMEOUT through
 * nvfp4_get_last_device_error instead of hanging. */
nvfp4_status_t nvfp4_probe_bounded_wait(const uint32_t* flag, uint64_t limit_ns, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* NVFP4_H */
