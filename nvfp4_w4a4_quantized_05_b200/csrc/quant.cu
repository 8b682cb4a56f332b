// quant.cu -- stage 1 of the W4A4 path: dynamic NVFP4 quantization on sm_100a.
//
// Per tensor (or per row group) the path computes ("NVFP4 Explained: NVIDIA's
// 4-Bit Format for Faster AI Inference", "How NVFP4 Represents a Value" and
// "Why the Block Scale Uses FP8 E4M3"; "What is NVFP4? 4-bit AI inference on
// NVIDIA Blackwell explained", "Why does scaling matter so much?"):
//   amax = max |x|                      (tensor amax, kernel 1)
//   g    = amax / (6 * 448)  (1 if amax == 0)   FP32 global decode scale
//   per 16-element block (1D) or 16x16 tile (2D), kernel 2:
//     sf   = e4m3_rn_satfinite(block_amax / (6 g))
//     d    = float(sf) * g ;  r = d == 0 ? 0 : 1 / d
//     code = e2m1_rn_satfinite(x * r)
// r and x * r are rounded to binary32's 24-bit significand without binary32's
// exponent ceiling, so each code is the one nearest x / d (the divisor that
// the reconstruction fp4 x block_scale x global_scale implies) even where
// 1 / d overflows: for a global scale below 2^-64 the kernels keep r / 2^32
// and multiply each product back by 2^32, both steps exact (see block_recip).
// Every step rounds as one IEEE binary32 operation to nearest even would
// (compiled with -fmad=false), and the roundings to E4M3 / E2M1 are the
// hardware cvt.rn.satfinite instructions, so the codes and scale bytes are
// bit-identical to the CPU definition.  Two steps take an exact shortcut:
// the block-scale quotient is bracketed between two products with the
// reciprocal (the division runs only when the bracket straddles an E4M3
// rounding boundary), and r comes from a 128-entry table per global scale.
//
// One tensor (the activation path): one cooperative launch, one CTA per SM.
// Pass 1 streams the tensor from HBM through per-warp shared-memory slots for
// the amax and keeps ~45% of it on chip; a grid barrier in the workspace
// (one generation-tagged word per CTA) hands every CTA the same g; pass 2
// quantizes the on-chip part, then the rest re-read from L2 by TMA.  A warp
// task is 1024 values of one row; lane l owns blocks 2 l and 2 l + 1, so its
// 16 code bytes leave in one store and two lanes make one 4-byte word of the
// 512-byte scale tile.
//
// Row groups (MoE activations) and shapes outside the one-launch layout
// (k % 64 != 0, very large tensors): kernel 1 reduces per-group amaxes with
// 16-byte loads, 8 in flight per thread, and a "last CTA" step publishes the
// global scales and group scale offsets; kernel 2 (programmatic dependent
// launch) issues its first loads before waiting for kernel 1, then quantizes
// with one 16-value block per lane.  Weights: 16 x 16 blocks, one scale per
// tile written to each of its 16 rows.
#include <cuda_runtime.h>
#include <cfloat>
#include <cstdint>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4 {
namespace {

constexpr int kThreads = 256;
constexpr int kWarps = kThreads / 32;
constexpr unsigned kFull = 0xFFFFFFFFu;
constexpr float kGlobalDen = 2688.0f;   // 6 (largest E2M1) * 448 (largest E4M3)

struct Groups {
    const int32_t* offsets;  // nullptr: one group [0, rows)
    int rows;
    __device__ __forceinline__ void range(int e, int& r0, int& r1) const {
        if (offsets) {
            r0 = offsets[e];
            r1 = offsets[e + 1];
            if (r1 < r0) r1 = r0;
        } else {
            r0 = 0;
            r1 = rows;
        }
    }
};

__device__ __forceinline__ int round128(int v) { return (v + 127) & ~127; }

// max(|a|, |b|) lane-wise on packed BF16 pairs (exact; the sign bit of the
// result is the xor of the input signs and is cleared by absmax_bits).
__device__ __forceinline__ uint32_t bmax_abs(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}
__device__ __forceinline__ uint32_t absmax8_packed(const uint4& v) {
    return bmax_abs(bmax_abs(v.x, v.y), bmax_abs(v.z, v.w));
}
// Packed BF16 magnitudes -> the larger one as a 16-bit pattern (for
// non-negative BF16 the bit patterns order like the values).
__device__ __forceinline__ uint32_t absmax_bits(uint32_t packed) {
    const uint32_t m = packed & 0x7FFF7FFFu;
    return max(m & 0xFFFFu, m >> 16);
}

__device__ __forceinline__ uint64_t pack_rr(float r) {
    uint64_t rr;
    asm("mov.b64 %0, {%1, %1};" : "=l"(rr) : "f"(r));
    return rr;
}

// Global scales below this take the tiny form of r (block_recip).
constexpr float kTinyG = 0x1p-64f;

// r for a block with d = float(sf) g: RN(1 / d), 0 when d == 0.  With a tiny
// global scale (g < 2^-64) it returns RN(1 / (d 2^32)) = RN(1 / d) / 2^32
// instead, and the caller multiplies each product x * r by 2^32:
//   - g >= 2^-64: d >= 2^-9 g >= 2^-73 (or 0), so 1 / d <= 2^73 never
//     overflows and plain binary32 is the reading;
//   - g < 2^-64: d < 448 * 2^-64, so d 2^32 is exact and normal (d >= 2^-149)
//     and 1 / (d 2^32) lies in [2^23, 2^117], where binary32 rounds it as an
//     unbounded exponent range would; RN(x * r / 2^32) * 2^32 equals that
//     range's RN(x * r) whenever x * r >= 2^-94, and below that both give a
//     signed zero code; a product that overflows is far above 6 and saturates
//     to 6, as x / d would.
__device__ __forceinline__ float block_recip(float d, bool tiny) {
    if (d == 0.0f) return 0.0f;
    return __frcp_rn(tiny ? __fmul_rn(d, 0x1p32f) : d);
}

// (lo, hi) BF16 pair times (r, r): two IEEE round-to-nearest products (TINY:
// r holds r / 2^32 and both products are then multiplied by 2^32, exactly).
template <bool TINY = false>
__device__ __forceinline__ void mul_bf16x2(uint32_t w, uint64_t rr, float& lo, float& hi) {
    uint64_t x, y;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "r"(w << 16), "r"(w & 0xFFFF0000u));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(y) : "l"(x), "l"(rr));
    if constexpr (TINY) asm("mul.rn.f32x2 %0, %0, %1;" : "+l"(y) : "l"(pack_rr(0x1p32f)));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(y));
}

// Eight BF16 values times r -> eight packed E2M1 codes.
template <bool TINY = false>
__device__ __forceinline__ uint32_t quant8(const uint4& v, uint64_t rr) {
    float x[8];
    mul_bf16x2<TINY>(v.x, rr, x[0], x[1]);
    mul_bf16x2<TINY>(v.y, rr, x[2], x[3]);
    mul_bf16x2<TINY>(v.z, rr, x[4], x[5]);
    mul_bf16x2<TINY>(v.w, rr, x[6], x[7]);
    return cvt_e2m1x8(x[0], x[1], x[2], x[3], x[4], x[5], x[6], x[7]);
}

// Block scale byte and element multiplier from the block amax (exact IEEE steps;
// used by the 16 x 16 weight quantizer, where it runs once per 256 values).
__device__ __forceinline__ uint32_t block_scale(float bamax, float g, float k6, bool tiny, float& r) {
    const uint32_t sf = cvt_e4m3(__fdiv_rn(bamax, k6));
    r = block_recip(__fmul_rn(e4m3_to_f32(sf), g), tiny);
    return sf;
}

// Per-CTA constants of the 1D block quantizer for one global scale g.
struct BlockQ {
    float k6;           // 6 g
    uint64_t inv_lo2;   // (il, il): il = RN(RN(1 / (6 g)) * (1 - 2^-20)); 0 when 6 g is subnormal
    uint64_t inv_hi2;   // (ih, ih): ih = RN(RN(1 / (6 g)) * (1 + 2^-20)); +inf when 6 g is subnormal
};
__device__ __forceinline__ BlockQ make_blockq(float g) {
    BlockQ c;
    c.k6 = __fmul_rn(6.0f, g);
    float il = 0.0f, ih = __int_as_float(0x7F800000);
    if (c.k6 >= FLT_MIN) {   // else RN(1 / (6 g)) may overflow: every block takes the division
        const float inv = __frcp_rn(c.k6);
        il = __fmul_rn(inv, 1.0f - 0x1p-20f);
        ih = __fmul_rn(inv, 1.0f + 0x1p-20f);
    }
    c.inv_lo2 = pack_rr(il);
    c.inv_hi2 = pack_rr(ih);
    return c;
}

// sf = e4m3_rn_satfinite(RN(bamax / (6 g))), bit-exact, mostly without a
// division.  lo = RN(bamax * il) and hi = RN(bamax * ih) bracket the correctly
// rounded quotient strictly (il and ih are within 2^-21 relative of 1 / (6 g)
// on either side, far more than the 2^-24 error of each rounding), and
// rounding to E4M3 is monotone: when lo and hi round to the same byte, so does
// the quotient.  Otherwise (an E4M3 rounding boundary within ~2^-20 relative,
// or 6 g subnormal) the exact IEEE quotient is rounded.
__device__ __forceinline__ uint32_t block_sf(float bamax, const BlockQ& c) {
    const uint32_t lo = cvt_e4m3(__fmul_rn(bamax, __uint_as_float((uint32_t)c.inv_lo2)));
    const uint32_t hi = cvt_e4m3(__fmul_rn(bamax, __uint_as_float((uint32_t)c.inv_hi2)));
    return lo == hi ? lo : cvt_e4m3(__fdiv_rn(bamax, c.k6));
}
// The scale bytes of two blocks, sf0 | sf1 << 8: both brackets with two paired
// multiplies and two paired conversions, one branch for both.
__device__ __forceinline__ uint32_t block_sf2(float b0, float b1, const BlockQ& c) {
    uint64_t bb, lo, hi;
    asm("mov.b64 %0, {%1, %2};" : "=l"(bb) : "f"(b0), "f"(b1));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(lo) : "l"(bb), "l"(c.inv_lo2));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(hi) : "l"(bb), "l"(c.inv_hi2));
    float lo0, lo1, hi0, hi1;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo0), "=f"(lo1) : "l"(lo));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(hi0), "=f"(hi1) : "l"(hi));
    const uint32_t plo = cvt_e4m3x2(lo1, lo0);
    if (plo == cvt_e4m3x2(hi1, hi0)) return plo;
    return cvt_e4m3x2(__fdiv_rn(b1, c.k6), __fdiv_rn(b0, c.k6));
}

// rtab[sf] = (r, r) for a block with scale byte sf: r = block_recip(float(sf) * g)
// (r / 2^32 for a tiny g), stored as the FP32 pair that the paired multiplies
// take.  128 entries (bytes 0..127; 127 is never produced by the saturating
// conversion).  Threads 0..127 fill it.
__device__ __forceinline__ void fill_rtab(uint64_t* rtab, float g, int tid) {
    if (tid < 128) rtab[tid] = pack_rr(block_recip(__fmul_rn(e4m3_to_f32((uint32_t)tid), g), g < kTinyG));
}

// Exact block scales without a division, for a BF16 block amax and a normal
// 6 g (g >= 2^-64).  Write b = m_b 2^(e_b - 127) with m_b = 1 + i / 128 and
// 6 g = m_k 2^(e_k - 127).  Scaling by a power of two does not round, so
// RN(b / (6 g)) = RN(m_b / m_k) 2^(e_b - e_k) whenever the quotient is a
// normal binary32 number.  qtab[i] holds the bits of RN((1 + i / 128) / m_k)
// minus e_k << 23, so the quotient's bits are qtab[i] + (e_b << 23).  A
// quotient below 2^-126 (E4M3 byte 0 either way) comes out as a binary32
// subnormal or, below that, as a negative integer, clamped to +0; so does a
// zero or BF16-subnormal b (its exponent sum is at most 128 - e_k, e_k >= 66).
// No quotient overflows: with g from the tensor's own amax it is at most
// 448 (1 + 2^-23).  The threads with tid in [0, 128) fill the table.
__device__ __forceinline__ void fill_qtab(int32_t* qtab, float k6, int tid) {
    if ((unsigned)tid < 128u) {
        const uint32_t kb = __float_as_uint(k6);
        const float mk = __uint_as_float((kb & 0x807FFFFFu) | (127u << 23));
        const float q = __fdiv_rn(__uint_as_float((127u << 23) | ((uint32_t)tid << 16)), mk);
        qtab[tid] = (int32_t)__float_as_uint(q) - (int32_t)(kb & 0x7F800000u);
    }
}
// Scale bytes sf0 | sf1 << 8 of blocks 2 lane and 2 lane + 1, whose BF16
// amaxes are the low and high halves of m (sign bits ignored).
__device__ __forceinline__ uint32_t block_sf2_tab(uint32_t m, const int32_t* qtab) {
    const int32_t q0 = max(qtab[m & 0x7Fu] + (int32_t)((m << 16) & 0x7F800000u), 0);
    const int32_t q1 = max(qtab[(m >> 16) & 0x7Fu] + (int32_t)(m & 0x7F800000u), 0);
    return cvt_e4m3x2(__int_as_float(q1), __int_as_float(q0));
}

__device__ __forceinline__ int64_t sf_tile_offset(int srow, int scol, int scale_cols) {
    return ((int64_t)(srow >> 7) * (scale_cols >> 2) + (scol >> 2)) * 512 + (srow & 31) * 16 +
           ((srow >> 5) & 3) * 4 + (scol & 3);
}

// One warp task: 512 consecutive values of one row, segment seg.  Lane l holds
// block l (values v0, v1) and quantizes it; its 8 code bytes leave in one store
// (the warp writes 256 contiguous bytes) and lanes 4i store the scale word of
// blocks 4i..4i+3.  Rows past the tensor (row_ok false) and columns past k hold
// zeros, so they produce zero scale bytes for the padded scale tile.  valid
// false (warp-uniform) stores nothing: callers run a fixed number of tasks
// side by side without branches between them.
__device__ __forceinline__ void quantize_task(const uint4& v0, const uint4& v1, bool row_ok, int seg, int lane,
                                              int k, int scale_cols, uint8_t* code_row, uint8_t* scales, int srow,
                                              const BlockQ& c, const uint64_t* rtab, bool tiny, bool valid = true) {
    const uint32_t am = absmax_bits(bmax_abs(absmax8_packed(v0), absmax8_packed(v1)));
    const uint32_t sf = block_sf(__uint_as_float(am << 16), c);
    const int col = seg * 512 + lane * 16;
    if (valid && row_ok && col < k) {
        const uint64_t rr = rtab[sf];
        uint2 q;
        if (tiny) {   // uniform across the grid row: one global scale
            q.x = quant8<true>(v0, rr);
            q.y = quant8<true>(v1, rr);
        } else {
            q.x = quant8(v0, rr);
            q.y = quant8(v1, rr);
        }
        *reinterpret_cast<uint2*>(code_row + col / 2) = q;
    }
    const uint32_t p = sf | (__shfl_down_sync(kFull, sf, 1) << 8);
    const uint32_t word = p | (__shfl_down_sync(kFull, p, 2) << 16);
    const int scol = seg * 32 + lane;
    if (valid && (lane & 3) == 0 && scol < scale_cols)
        *reinterpret_cast<uint32_t*>(scales + sf_tile_offset(srow, scol, scale_cols)) = word;
}

// MXFP4 form of the task: lanes 2i and 2i+1 hold the 32-value block i of
// the 512 values (16 each).  Its E8M0 byte is e + 127 for the smallest e with
// 6 * 2^e >= the block maximum, read off the maximum's FP32 bits: for
// m * 2^E (1 <= m < 2), e = E - 2 when m <= 1.5, else E - 1; e is clamped to
// -127 (byte 0), which also covers zero and subnormal maxima.  The codes are
// E2M1(x * 2^-e): 2^-e is a normal FP32 power of two, so each product is x / 2^e
// rounded only where it falls far below the smallest E2M1 step.  Lanes 8j
// store the scale word of blocks 4j..4j+3 (scale columns seg * 16 + 4j + i).
__device__ __forceinline__ void quantize_task_mx(const uint4& v0, const uint4& v1, bool row_ok, int seg, int lane,
                                                 int k, int scale_cols, uint8_t* code_row, uint8_t* scales, int srow) {
    const uint32_t h = absmax_bits(bmax_abs(absmax8_packed(v0), absmax8_packed(v1)));
    const uint32_t fb = max(h, __shfl_xor_sync(kFull, h, 1)) << 16;   // block maximum, FP32 bits
    const int eb = max(0, (int)(fb >> 23) - 2 + ((fb & 0x7FFFFFu) > 0x400000u ? 1 : 0));
    const int col = seg * 512 + lane * 16;
    if (row_ok && col < k) {
        const uint64_t rr = pack_rr(__uint_as_float((uint32_t)(254 - eb) << 23));   // 2^-e
        uint2 q;
        q.x = quant8(v0, rr);
        q.y = quant8(v1, rr);
        *reinterpret_cast<uint2*>(code_row + col / 2) = q;
    }
    const uint32_t p = (uint32_t)eb | (__shfl_down_sync(kFull, (uint32_t)eb, 2) << 8);
    const uint32_t word = p | (__shfl_down_sync(kFull, p, 4) << 16);
    const int scol = seg * 16 + (lane >> 1);
    if ((lane & 7) == 0 && scol < scale_cols)
        *reinterpret_cast<uint32_t*>(scales + sf_tile_offset(srow, scol, scale_cols)) = word;
}

// Exclusive prefix over groups of round128(group rows), by one CTA.
__device__ void write_pad_rows(const Groups& gr, int num_groups, int32_t* pad_rows) {
    __shared__ int part[kThreads];
    const int per = (num_groups + kThreads - 1) / kThreads;
    const int g0 = threadIdx.x * per;
    int s = 0;
    for (int i = 0; i < per; ++i) {
        const int e = g0 + i;
        if (e < num_groups) {
            int r0, r1;
            gr.range(e, r0, r1);
            s += round128(r1 - r0);
        }
    }
    part[threadIdx.x] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        int acc = 0;
        for (int t = 0; t < kThreads; ++t) {
            const int v = part[t];
            part[t] = acc;
            acc += v;
        }
        pad_rows[num_groups] = acc;
    }
    __syncthreads();
    int acc = part[threadIdx.x];
    for (int i = 0; i < per; ++i) {
        const int e = g0 + i;
        if (e < num_groups) {
            int r0, r1;
            gr.range(e, r0, r1);
            pad_rows[e] = acc;
            acc += round128(r1 - r0);
        }
    }
}

// ---- kernel 1: tensor / group amax -> global scale --------------------------------
struct AmaxArgs {
    const uint16_t* x;
    int64_t ld;
    int k;
    Groups groups;
    int num_groups;
    uint32_t* ws;        // [0]: CTA counter, [4 + e]: amax bits of group e
    int32_t* pad_rows;   // nullptr for one tensor
    float* gscale;
};

constexpr int kAmaxUnroll = 8;

// The kernels below let the next kernel in the stream launch as soon as all
// their CTAs run (griddepcontrol.launch_dependents): a dependent kernel's
// griddepcontrol.wait still waits for this grid's completion and writes, so
// it may only do independent work earlier (prefetch its own inputs that this
// kernel does not write).  The amax kernel is itself launched as a
// dependent (it may start while the kernel before it, perhaps the producer
// of x, is finishing), so it waits before anything else and only then lets
// its own dependent start: that one may read x before its wait.
__global__ void __launch_bounds__(kThreads, 4) amax_kernel(AmaxArgs a) {
    pdl_wait();
    pdl_launch_dependents();
    const int e = blockIdx.y;
    int r0, r1;
    a.groups.range(e, r0, r1);
    const int kc = a.k / 8;                            // 16-byte chunks per row
    const int64_t items = (int64_t)(r1 - r0) * kc;
    const int64_t stride = (int64_t)gridDim.x * kThreads;
    const bool dense = (a.ld == (int64_t)a.k);
    const uint16_t* base = a.x + (int64_t)r0 * a.ld;
    uint32_t acc = 0;   // packed BF16 running max of |x|
    for (int64_t i0 = (int64_t)blockIdx.x * kThreads + threadIdx.x; i0 < items; i0 += stride * kAmaxUnroll) {
        uint4 v[kAmaxUnroll];
#pragma unroll
        for (int u = 0; u < kAmaxUnroll; ++u) {
            const int64_t i = i0 + u * stride;
            v[u] = make_uint4(0, 0, 0, 0);
            if (i < items) {
                const uint16_t* p;
                if (dense) {
                    p = base + i * 8;
                } else {
                    const int64_t r = i / kc;
                    p = base + r * a.ld + (i - r * kc) * 8;
                }
                v[u] = ld_nc_v4(p);
            }
        }
#pragma unroll
        for (int u = 0; u < kAmaxUnroll; ++u) acc = bmax_abs(acc, absmax8_packed(v[u]));
    }
    uint32_t m = absmax_bits(acc);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(kFull, m, o));
    __shared__ uint32_t red[kWarps];
    __shared__ bool last;
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t b = red[0];
        for (int w = 1; w < kWarps; ++w) b = max(b, red[w]);
        atomicMax(&a.ws[4 + e], b << 16);   // FP32 bit pattern of the BF16 amax
        __threadfence();
        const unsigned total = gridDim.x * gridDim.y;
        last = (atomicAdd(&a.ws[0], 1u) == total - 1);
    }
    __syncthreads();
    if (last) {
        __threadfence();
        for (int gi = threadIdx.x; gi < a.num_groups; gi += kThreads) {
            const float amax = __uint_as_float(atomicExch(&a.ws[4 + gi], 0u));
            a.gscale[gi] = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, kGlobalDen);
        }
        if (a.pad_rows) write_pad_rows(a.groups, a.num_groups, a.pad_rows);
        if (threadIdx.x == 0) a.ws[0] = 0;
    }
}

// ---- kernel 2: 1D 16-element blocks (one tensor or row groups) ---------------------
struct Quant1dArgs {
    const uint16_t* x;
    int64_t ld;
    int k;
    int nseg;         // ceil(k / 512): 512-element warp tasks per row
    int scale_cols;   // ceil(k / 64) * 4
    Groups groups;
    const int32_t* pad_rows;   // nullptr: one tensor, scale rows from 0
    const float* gscale;
    uint8_t* codes;
    uint8_t* scales;
};

constexpr int kQuantUnroll = 2;

// Position (row, segment) of a warp task, advanced without divisions.
struct TaskPos {
    int row, seg;
    __device__ __forceinline__ void advance(int drow, int dseg, int nseg) {
        row += drow;
        seg += dseg;
        if (seg >= nseg) {
            seg -= nseg;
            ++row;
        }
    }
};

__device__ __forceinline__ void load_block16(const Quant1dArgs& a, int r0, int nrows, const TaskPos& t, int lane,
                                             uint64_t pol, uint4& v0, uint4& v1) {
    const int col = t.seg * 512 + lane * 16;
    v0 = make_uint4(0, 0, 0, 0);
    v1 = make_uint4(0, 0, 0, 0);
    if (t.row < nrows && col < a.k) {
        const uint16_t* p = a.x + (int64_t)(r0 + t.row) * a.ld + col;
        v0 = ld_nc_v4_hint(p, pol);
        v1 = ld_nc_v4_hint(p + 8, pol);
    }
}

// MX: the MXFP4 task (one tensor, no global scale; gscale unused).
template <bool MX = false>
__global__ void __launch_bounds__(kThreads, 4) quant1d_kernel(Quant1dArgs a) {
    pdl_launch_dependents();
    const int e = blockIdx.y;
    int r0, r1;
    a.groups.range(e, r0, r1);
    const int nrows = r1 - r0;
    const int lane = threadIdx.x & 31;
    const int prows = round128(nrows);
    const int w0 = blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int wstride = gridDim.x * kWarps;
    const int nseg = a.nseg;
    // task t -> (t / nseg, t % nseg); step kQuantUnroll * wstride tasks per iteration
    TaskPos t0{w0 / nseg, w0 % nseg};
    const int step = kQuantUnroll * wstride;
    const int drow = step / nseg, dseg = step - (step / nseg) * nseg;
    const int d1row = wstride / nseg, d1seg = wstride - d1row * nseg;
    const uint64_t pol = l2_policy_evict_first();
    const int64_t kbytes = a.k / 2;

    // The input does not depend on kernel 1: start the first loads before waiting.
    uint4 v[kQuantUnroll][2];
    TaskPos tp[kQuantUnroll];
    tp[0] = t0;
#pragma unroll
    for (int u = 1; u < kQuantUnroll; ++u) {
        tp[u] = tp[u - 1];
        tp[u].advance(d1row, d1seg, nseg);
    }
#pragma unroll
    for (int u = 0; u < kQuantUnroll; ++u) load_block16(a, r0, nrows, tp[u], lane, pol, v[u][0], v[u][1]);

    pdl_wait();   // g (and the group scale offsets) come from amax_kernel
    const int srow0 = a.pad_rows ? a.pad_rows[e] : 0;
    __shared__ uint64_t rtab[128];
    BlockQ c{};
    bool tiny = false;
    if constexpr (!MX) {
        const float g = a.gscale[e];
        fill_rtab(rtab, g, threadIdx.x);
        c = make_blockq(g);
        tiny = g < kTinyG;
        __syncthreads();
    }

    while (tp[0].row < prows) {
#pragma unroll
        for (int u = 0; u < kQuantUnroll; ++u) {
            const TaskPos t = tp[u];
            if (t.row >= prows) break;   // uniform across the warp
            if constexpr (MX)
                quantize_task_mx(v[u][0], v[u][1], t.row < nrows, t.seg, lane, a.k, a.scale_cols,
                                 a.codes + (int64_t)(r0 + t.row) * kbytes, a.scales, srow0 + t.row);
            else
                quantize_task(v[u][0], v[u][1], t.row < nrows, t.seg, lane, a.k, a.scale_cols,
                              a.codes + (int64_t)(r0 + t.row) * kbytes, a.scales, srow0 + t.row, c, rtab, tiny);
        }
#pragma unroll
        for (int u = 0; u < kQuantUnroll; ++u) {
            tp[u].advance(drow, dseg, nseg);
            load_block16(a, r0, nrows, tp[u], lane, pol, v[u][0], v[u][1]);
        }
    }
}

// ---- one launch for one tensor: amax, grid barrier, quantize ---------------------
//
// One CTA of 1024 threads per SM (the grid is launched cooperatively, so all CTAs
// are resident together).  A warp task is 1024 consecutive values of one row;
// lane l owns values 32 l .. 32 l + 31 of it, i.e. blocks 2 l and 2 l + 1, so its
// 16 code bytes leave in one store and two lanes make one scale word.  CTA c
// owns a contiguous range of tasks and warp w of it a contiguous run of those.
// Each warp owns kStage task slots of shared memory (2 KB each; 192 KB per SM)
// and streams its tasks through them, kStage tasks in flight.  Pass 1 copies
// with cp.async (each lane moves 16-byte units lane, 32 + lane, ...; zero fill
// past the tensor) and reduces each landed task to the amax; the warp's last
// kStage tasks stay in their slots (~28 MB of the tensor on chip across the
// GPU).  A grid barrier in the
// workspace publishes the per-CTA amaxes; every CTA reduces them in the same
// order, so all hold the same g.  Pass 2 quantizes the tasks still on chip
// first, refilling each freed slot with one of the warp's other tasks by TMA
// (one 3-D box per task, 128-byte swizzle, zero fill past the tensor; L2 hits:
// the tensor was just read), then works through those as they land.
constexpr int kFThreads = 1024;
constexpr int kFWarps = kFThreads / 32;
constexpr int kTaskVals = 1024;                  // values per warp task
constexpr int kTaskBytes = kTaskVals * 2;
constexpr int kStage = 3;                        // task slots per warp

constexpr int kTmTasks = 4;                      // tasks a warp can park in tensor memory (64 columns)
constexpr int kMaxFusedGroups = 1024;            // row groups the one-launch form takes
constexpr int kMaxSmoothK = 6144;                // k of the pre-scaled form (its factors sit in shared memory)

struct FusedArgs {
    const uint16_t* x;
    int64_t ld;
    int rows, k, nseg, scale_cols;
    int tasks;        // padded rows * nseg: one tensor round128(rows); grouped an upper bound,
                      // the exact count follows from the offsets on the device
    int full_segs;    // segments that need no guards: k / 1024
    uint32_t sc4x512; // (scale_cols / 4) * 512: bytes of one 128-row band of scale tiles
    float* gscale;    // [groups]
    uint8_t* codes;
    uint8_t* scales;
    uint64_t* part;   // per-CTA generation << 32 words, kPartStrideWords apart
    uint32_t* bar;    // grid barrier: arrival counter, amax words of even and odd generations
    uint64_t* gword;  // grouped: per-group generation << 32 | amax words
    int tm_tasks;     // tasks per warp parked in tensor memory (0: none allocated)
    const int32_t* offsets;   // grouped: [groups + 1]; nullptr for one tensor
    int groups;
    const float* smooth;      // pre-scaled form: per-column factors [k]; nullptr otherwise
    uint64_t limit;
    unsigned* err;
};

// A task sits in its slot as 16 rows of 128 bytes (64 values each) in the TMA
// 128-byte swizzle: 16-byte unit u (values 8 u .. 8 u + 7) at unit
// (u & ~7) | ((u & 7) ^ ((u >> 3) & 7)).  Lane l reads units 4 l .. 4 l + 3 and
// copies units 32 i + l; either way every 8-lane phase touches 8 distinct
// 16-byte bank groups.
__device__ __forceinline__ int slot_unit(int u) { return (u & ~7) | ((u & 7) ^ ((u >> 3) & 7)); }

// Per-lane constants of the one-launch path.
struct LaneC {
    int lane;
    uint32_t ld_off[4];   // byte offsets of units 4 lane + i in a slot
    uint32_t st_off[4];   // byte offsets of units 32 i + lane in a slot
    uint32_t s_off;       // (lane / 2) * 512: the lane pair's scale tile within the segment
};
__device__ __forceinline__ LaneC make_lanec(int lane) {
    LaneC lc;
    lc.lane = lane;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        lc.ld_off[i] = (uint32_t)slot_unit(4 * lane + i) * 16u;
        lc.st_off[i] = (uint32_t)slot_unit(32 * i + lane) * 16u;
    }
    lc.s_off = (uint32_t)(lane >> 1) * 512u;
    return lc;
}

// Tasks run over padded rows: the scale layout gives each group of rows
// (one group for one tensor) a whole number of 128-row scale blocks.  Group
// e owns padded rows [128 blk[e], 128 blk[e + 1]); padded row pr of it is
// tensor row off[e] + pr - 128 blk[e] while that is below off[e + 1], and
// padding (zero values: zero scale bytes, no codes) after.
struct GroupTab {       // offsets and block prefixes, in shared memory
    const int* off;     // [G + 1]
    const int* blk;     // [G + 1]
    int G;
};
struct RowMap {
    int e;        // group of the current padded row
    int pbeg;     // its first padded row
    int pend;     // its first padded row past the group
    int base;     // tensor row = padded row + base
    int rlast;    // the group's rows end at this tensor row
    __device__ __forceinline__ void one(int rows) {
        e = 0;
        pbeg = 0;
        pend = 0x7FFFFFFF;
        base = 0;
        rlast = rows;
    }
    __device__ __forceinline__ void set(const GroupTab& gt, int g) {
        e = g;
        pbeg = 128 * gt.blk[g];
        pend = 128 * gt.blk[g + 1];
        base = gt.off[g] - 128 * gt.blk[g];
        rlast = gt.off[g + 1];
    }
    // the last group whose first padded row is at or before pr (it holds pr:
    // empty groups start where the next one does)
    __device__ __forceinline__ void seek(const GroupTab& gt, int pr) {
        int lo = 0, hi = gt.G;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (128 * gt.blk[mid] <= pr) lo = mid; else hi = mid;
        }
        set(gt, lo);
    }
    __device__ __forceinline__ void step(const GroupTab& gt, int pr) {
        while (pr >= pend && e + 1 < gt.G) set(gt, e + 1);
    }
    __device__ __forceinline__ void step_back(const GroupTab& gt, int pr) {
        while (pr < pbeg && e > 0) set(gt, e - 1);
    }
};

// Task positions walk one task at a time, row-major over (padded row, segment).
template <bool GROUPED>
struct SrcCursor {   // which values a task holds
    int row, seg;
    RowMap m;
    __device__ __forceinline__ void init(const FusedArgs& a, const GroupTab& gt, int t) {
        row = t / a.nseg;
        seg = t - row * a.nseg;
        if constexpr (GROUPED) m.seek(gt, row); else m.one(a.rows);
    }
    __device__ __forceinline__ void next(const FusedArgs& a, const GroupTab& gt) {
        if (++seg == a.nseg) {
            seg = 0;
            ++row;
            if constexpr (GROUPED) m.step(gt, row);
        }
    }
    __device__ __forceinline__ void prev(const FusedArgs& a, const GroupTab& gt) {
        if (seg-- == 0) {
            seg = a.nseg - 1;
            --row;
            if constexpr (GROUPED) m.step_back(gt, row);
        }
    }
    __device__ __forceinline__ bool valid() const { return row + m.base < m.rlast; }
    __device__ __forceinline__ int real() const { return row + m.base; }
};
template <bool GROUPED>
struct DstCursor {   // where a task's codes and scale words go (32-bit byte offsets)
    int row, seg;
    RowMap m;
    uint32_t co;     // tensor row * k / 2 + seg * 512 (used for rows that hold values)
    uint32_t so;     // scale word of the segment's first four blocks (padded row)
    __device__ __forceinline__ void set_row(const FusedArgs& a) {
        const uint32_t r = (uint32_t)row;
        co = (uint32_t)(row + m.base) * (uint32_t)(a.k >> 1) + ((uint32_t)seg << 9);
        so = (r >> 7) * a.sc4x512 + (r & 31u) * 16u + ((r >> 5) & 3u) * 4u + ((uint32_t)seg << 13);
    }
    __device__ __forceinline__ void init(const FusedArgs& a, const GroupTab& gt, int t) {
        row = t / a.nseg;
        seg = t - row * a.nseg;
        if constexpr (GROUPED) m.seek(gt, row); else m.one(a.rows);
        set_row(a);
    }
    __device__ __forceinline__ void next(const FusedArgs& a, const GroupTab& gt) {
        if (++seg == a.nseg) {
            seg = 0;
            ++row;
            if constexpr (GROUPED) m.step(gt, row);
            set_row(a);
        } else {
            co += kTaskVals / 2;
            so += 8192u;   // 16 scale tiles of 512 bytes per segment
        }
    }
    __device__ __forceinline__ void prev(const FusedArgs& a, const GroupTab& gt) {
        if (seg-- == 0) {
            seg = a.nseg - 1;
            --row;
            if constexpr (GROUPED) m.step_back(gt, row);
            set_row(a);
        } else {
            co -= kTaskVals / 2;
            so -= 8192u;
        }
    }
    __device__ __forceinline__ bool valid() const { return row + m.base < m.rlast; }
};

// Factors of the pre-scaled form in shared memory: per 1024-column segment,
// 16-byte unit u (columns 4 u .. 4 u + 3) at unit (u & ~7) | ((u & 7) ^ ((u >> 3) & 7)),
// so that lane l's eight units 8 l .. 8 l + 7 (its 32 columns) fall in eight
// different bank groups for every 8-lane phase of a 16-byte load.
__device__ __forceinline__ float4 smooth_unit(const float* seg_base, int lane, int i) {
    return reinterpret_cast<const float4*>(seg_base)[8 * lane + (i ^ (lane & 7))];
}

// Eight BF16 values, each times its column factor (x' = x s, one IEEE product),
// then times r -> eight packed E2M1 codes (TINY: r / 2^32, then times 2^32).
template <bool TINY>
__device__ __forceinline__ uint32_t quant8_smooth(const uint4& v, const float4& s0, const float4& s1, uint64_t rr) {
    const float r = __uint_as_float((uint32_t)rr);
    const float up = TINY ? 0x1p32f : 1.0f;
    float x[8];
    x[0] = __fmul_rn(__fmul_rn(__uint_as_float(v.x << 16), s0.x), r);
    x[1] = __fmul_rn(__fmul_rn(__uint_as_float(v.x & 0xFFFF0000u), s0.y), r);
    x[2] = __fmul_rn(__fmul_rn(__uint_as_float(v.y << 16), s0.z), r);
    x[3] = __fmul_rn(__fmul_rn(__uint_as_float(v.y & 0xFFFF0000u), s0.w), r);
    x[4] = __fmul_rn(__fmul_rn(__uint_as_float(v.z << 16), s1.x), r);
    x[5] = __fmul_rn(__fmul_rn(__uint_as_float(v.z & 0xFFFF0000u), s1.y), r);
    x[6] = __fmul_rn(__fmul_rn(__uint_as_float(v.w << 16), s1.z), r);
    x[7] = __fmul_rn(__fmul_rn(__uint_as_float(v.w & 0xFFFF0000u), s1.w), r);
    if constexpr (TINY) {
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = __fmul_rn(x[i], up);
    }
    return cvt_e2m1x8(x[0], x[1], x[2], x[3], x[4], x[5], x[6], x[7]);
}
// max |x s| over the eight values of a unit.
__device__ __forceinline__ float absmax8_smooth(const uint4& v, const float4& s0, const float4& s1) {
    float m = fabsf(__fmul_rn(__uint_as_float(v.x << 16), s0.x));
    m = fmaxf(m, fabsf(__fmul_rn(__uint_as_float(v.x & 0xFFFF0000u), s0.y)));
    m = fmaxf(m, fabsf(__fmul_rn(__uint_as_float(v.y << 16), s0.z)));
    m = fmaxf(m, fabsf(__fmul_rn(__uint_as_float(v.y & 0xFFFF0000u), s0.w)));
    m = fmaxf(m, fabsf(__fmul_rn(__uint_as_float(v.z << 16), s1.x)));
    m = fmaxf(m, fabsf(__fmul_rn(__uint_as_float(v.z & 0xFFFF0000u), s1.y)));
    m = fmaxf(m, fabsf(__fmul_rn(__uint_as_float(v.w << 16), s1.z)));
    return fmaxf(m, fabsf(__fmul_rn(__uint_as_float(v.w & 0xFFFF0000u), s1.w)));
}

// Per-group quantizer constants: the global scale g, the bracket constants and
// whether g takes the tiny form of r.
struct GroupQ {
    float g;
    bool tiny;
    BlockQ c;
};
__device__ __forceinline__ GroupQ make_groupq(uint32_t amax_fbits) {   // FP32 bits of the amax
    GroupQ q;
    const float amax = __uint_as_float(amax_fbits);
    q.g = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, kGlobalDen);
    q.tiny = q.g < kTinyG;
    q.c = make_blockq(q.g);
    return q;
}
// (r, r) for scale byte sf: the same value the table of the one-tensor form holds.
__device__ __forceinline__ uint64_t block_rr(uint32_t sf, const GroupQ& q) {
    return pack_rr(block_recip(__fmul_rn(e4m3_to_f32(sf), q.g), q.tiny));
}

// A lane's 16 code bytes and, from even lanes, the scale word of its lane pair.
template <bool FULL, bool GROUPED>
__device__ __forceinline__ void store_task(const FusedArgs& a, const uint4& q, uint32_t pair, const DstCursor<GROUPED>& t,
                                           const LaneC& lc) {
    const uint32_t word = __byte_perm(pair, __shfl_down_sync(kFull, pair, 1), 0x5410);
    const bool even = (lc.lane & 1) == 0;
    uint8_t* dst = a.codes + t.co + 16 * lc.lane;
    uint32_t* sw = reinterpret_cast<uint32_t*>(a.scales + t.so + lc.s_off);
    if (FULL) {
        *reinterpret_cast<uint4*>(dst) = q;
        if (even) *sw = word;
    } else {
        // Padding rows and values past k arrived as zeros: their scale bytes
        // are 0, as the padded scale tile wants; no codes are stored there.
        if (t.valid() && t.seg * kTaskVals + 32 * lc.lane < a.k) *reinterpret_cast<uint4*>(dst) = q;
        if (even && t.seg * (kTaskVals / 16) + 2 * lc.lane < a.scale_cols) *sw = word;
    }
}

// One tensor with g >= 2^-64: the block amaxes m come from pass 1 (packed
// BF16, block 2 lane low), the scale bytes from the quotient table.
template <bool FULL>
__device__ __forceinline__ void quantize_plain(const FusedArgs& a, const uint4 (&u)[4], uint32_t m,
                                               const DstCursor<false>& t, const LaneC& lc, const uint64_t* rtab,
                                               const int32_t* qtab) {
    const uint32_t pair = block_sf2_tab(m, qtab);
    const uint64_t rr0 = rtab[pair & 0xFFu];
    const uint64_t rr1 = rtab[pair >> 8];
    uint4 q;
    q.x = quant8(u[0], rr0);
    q.y = quant8(u[1], rr0);
    q.z = quant8(u[2], rr1);
    q.w = quant8(u[3], rr1);
    store_task<FULL, false>(a, q, pair, t, lc);
}

// Quantize one task whose values the lane holds in u (its 32 values, units
// 4 lane .. 4 lane + 3 of the task).  FULL: the whole task is inside the
// tensor.  One tensor: r from the per-CTA table; grouped: r computed per
// block.  TINY: the group's g takes the tiny form of r (block_recip).
template <bool FULL, bool GROUPED, bool SMOOTH, bool TINY>
__device__ __forceinline__ void quantize_vals(const FusedArgs& a, const uint4 (&u)[4], const DstCursor<GROUPED>& t,
                                              const LaneC& lc, const GroupQ& gq, const uint64_t* rtab,
                                              const float* ssm) {
    float b0, b1;
    float4 sv[8];   // pre-scaled form: the factors of this lane's 32 columns
    if constexpr (SMOOTH) {
#pragma unroll
        for (int i = 0; i < 8; ++i) sv[i] = smooth_unit(ssm + t.seg * kTaskVals, lc.lane, i);
        b0 = fmaxf(absmax8_smooth(u[0], sv[0], sv[1]), absmax8_smooth(u[1], sv[2], sv[3]));
        b1 = fmaxf(absmax8_smooth(u[2], sv[4], sv[5]), absmax8_smooth(u[3], sv[6], sv[7]));
    } else {
        // Packed maxima of |x| per block, then both blocks' halves against each other:
        // m = (amax of block 2 lane + 1 in the high half, of block 2 lane in the low).
        const uint32_t m0 = bmax_abs(absmax8_packed(u[0]), absmax8_packed(u[1]));
        const uint32_t m1 = bmax_abs(absmax8_packed(u[2]), absmax8_packed(u[3]));
        const uint32_t m = bmax_abs(__byte_perm(m0, m1, 0x5410), __byte_perm(m0, m1, 0x7632));
        b0 = __uint_as_float((m << 16) & 0x7FFF0000u);
        b1 = __uint_as_float(m & 0x7FFF0000u);
    }
    const uint32_t pair = block_sf2(b0, b1, gq.c);   // scale bytes of blocks 2 lane, 2 lane + 1
    uint64_t rr0, rr1;
    if constexpr (GROUPED) {
        rr0 = block_rr(pair & 0xFFu, gq);
        rr1 = block_rr(pair >> 8, gq);
    } else {
        rr0 = rtab[pair & 0xFFu];
        rr1 = rtab[pair >> 8];
    }
    uint4 q;
    if constexpr (SMOOTH) {
        q.x = quant8_smooth<TINY>(u[0], sv[0], sv[1], rr0);
        q.y = quant8_smooth<TINY>(u[1], sv[2], sv[3], rr0);
        q.z = quant8_smooth<TINY>(u[2], sv[4], sv[5], rr1);
        q.w = quant8_smooth<TINY>(u[3], sv[6], sv[7], rr1);
    } else {
        q.x = quant8<TINY>(u[0], rr0);
        q.y = quant8<TINY>(u[1], rr0);
        q.z = quant8<TINY>(u[2], rr1);
        q.w = quant8<TINY>(u[3], rr1);
    }
    store_task<FULL, GROUPED>(a, q, pair, t, lc);
}
template <bool GROUPED, bool SMOOTH>
__device__ __forceinline__ void quantize_any(const FusedArgs& a, const uint4 (&u)[4], const DstCursor<GROUPED>& t,
                                             const LaneC& lc, const GroupQ& gq, const uint64_t* rtab,
                                             const float* ssm) {
    const bool full = t.valid() && t.seg < a.full_segs;
    if (gq.tiny) {   // warp-uniform (one g per group): a global scale below 2^-64
        if (full) quantize_vals<true, GROUPED, SMOOTH, true>(a, u, t, lc, gq, rtab, ssm);
        else quantize_vals<false, GROUPED, SMOOTH, true>(a, u, t, lc, gq, rtab, ssm);
    } else if (full) {
        quantize_vals<true, GROUPED, SMOOTH, false>(a, u, t, lc, gq, rtab, ssm);
    } else {
        quantize_vals<false, GROUPED, SMOOTH, false>(a, u, t, lc, gq, rtab, ssm);
    }
}
// The lane's 32 values of the task in shared-memory slot sb.
__device__ __forceinline__ void load_slot(const char* sb, const LaneC& lc, uint4 (&u)[4]) {
#pragma unroll
    for (int i = 0; i < 4; ++i) u[i] = *reinterpret_cast<const uint4*>(sb + lc.ld_off[i]);
}
// ... and of the task parked in tensor memory at address ta (16 columns of
// the warp's lane quarter, lane i holding lane i's values).
__device__ __forceinline__ void load_tmem(uint32_t ta, uint4 (&u)[4]) {
    uint32_t r[16];
    tmem_ld_32x32b_x16(ta, r);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 4; ++i) u[i] = make_uint4(r[4 * i], r[4 * i + 1], r[4 * i + 2], r[4 * i + 3]);
}

// Grid barrier and, for one tensor, the amax reduction.  Every CTA knows the
// call's generation gen from its own word (one more than its last call's;
// every CTA of a call holds the same).  Arrival: fold the CTA's amax into
// amax word gen & 1, then add one to the arrival counter with release
// semantics; CTA 0 also zeroes the other amax word for the next call (no CTA
// of this call uses it, and the previous call is over).  All CTAs of call
// gen have arrived when the counter reads gen * G (mod 2^32: it never resets
// and each call adds exactly G).  Lane 0 of warp 0 polls it with acquire
// loads; false if that wait ran out (error word set).
__device__ __forceinline__ void grid_arrive(uint32_t* bar, uint32_t gen, uint32_t amax_bits, bool first_cta) {
    if (amax_bits) atomicMax(bar + 1 + (gen & 1u), amax_bits);
    if (first_cta) st_relaxed_gpu_u32(bar + 1 + ((gen + 1u) & 1u), 0u);
    red_release_gpu_add_u32(bar, 1u);
}
__device__ __forceinline__ bool grid_wait(const uint32_t* bar, uint32_t gen, int G, uint64_t limit, unsigned* err,
                                          uint32_t& amax_bits) {
    const uint32_t target = gen * (uint32_t)G;
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu_u32(bar) != target) {
        if (globaltimer_ns() - t0 > limit) {
            atomicOr(err, 1u);
            return false;
        }
    }
    amax_bits = ld_relaxed_gpu_u32(bar + 1 + (gen & 1u));
    return true;
}

// Grouped form: fold a warp's amax bits m of group e into the group's word.
// The first fold of this call (word of an older generation) replaces the
// stale value; later ones take the max.
__device__ __forceinline__ void fold_group_amax(uint64_t* w, uint32_t gen, uint32_t m) {
    uint64_t old = ld_relaxed_gpu_u64(w);
    while (true) {
        const uint32_t cur = (uint32_t)(old >> 32) == gen ? (uint32_t)old : 0u;
        const uint64_t nw = ((uint64_t)gen << 32) | max(cur, m);
        if (nw == old) return;
        const uint64_t prev = atom_cas_gpu_u64(w, old, nw);
        if (prev == old) return;
        old = prev;
    }
}
// Grouped form: the amax bits of group e after the barrier (0 for a group no
// row of which was seen this call, i.e. an empty group).
__device__ __forceinline__ uint32_t group_amax(const uint64_t* w, uint32_t gen) {
    const uint64_t v = ld_relaxed_gpu_u64(w);
    return (uint32_t)(v >> 32) == gen ? (uint32_t)v : 0u;
}

// A warp's slot ring: slot s is kTaskBytes at base + (warp + 32 s) * kTaskBytes,
// filled by one TMA box and completed on bar[s].
struct Ring {
    char* base;
    uint64_t* bar;     // this warp's kStage barriers
    int warp;
    uint32_t phase;    // bit s: parity of the next completion of slot s
    uint32_t box_bytes;
    __device__ __forceinline__ char* slot(int s) const { return base + (warp + 32 * s) * kTaskBytes; }
};
// Lane 0 starts the copy of task t into slot s; the warp's reads of the slot's
// previous task are done (the caller's __syncwarp).  Padding rows read past
// the tensor, where the copy fills zeros.
template <bool GROUPED>
__device__ __forceinline__ void stage(const CUtensorMap* tmap, const FusedArgs& a, Ring& r, int s,
                                      const SrcCursor<GROUPED>& t, uint64_t pol, int lane) {
    if (lane == 0) {
        fence_proxy_async_smem();
        mbar_arrive_expect_tx(&r.bar[s], r.box_bytes);
        tma_load_3d(r.slot(s), tmap, &r.bar[s], 0, t.seg * (kTaskVals / 64), t.valid() ? t.real() : a.rows, pol);
    }
}
// Wait (bounded) until the copy into slot s has landed.
__device__ __forceinline__ void land(Ring& r, int s, const FusedArgs& a) {
    if (!mbar_wait(&r.bar[s], (r.phase >> s) & 1u, a.limit)) atomicOr(a.err, 1u);
    r.phase ^= 1u << s;
}

// Pass 1 copy: the warp starts the cp.async copy of task t into slot s.
template <bool GROUPED>
__device__ __forceinline__ void stage_cp(const FusedArgs& a, const Ring& r, int s, const SrcCursor<GROUPED>& t,
                                         const LaneC& lc, uint64_t pol) {
    const bool row_in = t.valid();
    const uint16_t* p = a.x + (int64_t)(row_in ? t.real() : 0) * a.ld + t.seg * kTaskVals + 8 * lc.lane;
    const uint32_t d = smem_u32(r.slot(s));
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const bool in = row_in && t.seg * kTaskVals + 256 * i + 8 * lc.lane < a.k;
        cp_async16(d + lc.st_off[i], in ? p + 256 * i : a.x, in ? 16u : 0u, pol);
    }
}

// Per-warp state of pass 2: the constants of the group being quantized.
template <bool GROUPED>
struct Pass2Q {
    GroupQ q;
    int e = -1;
    __device__ __forceinline__ const GroupQ& at(const FusedArgs& a, const DstCursor<GROUPED>& t, uint32_t gen) {
        if constexpr (GROUPED) {
            if (t.m.e != e) {   // warp-uniform
                e = t.m.e;
                q = make_groupq(group_amax(a.gword + e, gen));
            }
        }
        return q;
    }
};

// Pass 2 of one warp with tasks tw .. tw + n - 1.  Pass 1 left the last
// nres = min(kStage, n) of them in the warp's shared-memory slots (task
// n - nres + k in slot (n - nres + k) % kStage) and the first nt (at most
// kTmTasks) in the warp's tensor-memory columns (task j at column tcol + 16 j);
// the nl = n - nres - nt in between come back from L2, newest first -- task
// nt + nl - 1, nt + nl - 2, ..., nt -- because pass 1 read them in increasing
// order, so the later ones are the likeliest to be still in L2.  Order: the
// slot tasks (each one's slot then takes the next refill), the
// tensor-memory tasks (while the refills are in flight), the refills.
// One tensor (not pre-scaled): the block amaxes of the tasks kept on chip,
// computed in pass 1, and the per-CTA quotient table.  bm points at this
// lane's word of on-chip task 0; task j's is kFWarps * 32 words further.
struct OnChip {
    const uint32_t* bm;
    const int32_t* qtab;
};
template <bool GROUPED, bool SMOOTH>
__device__ __forceinline__ void quantize_onchip(const FusedArgs& a, const uint4 (&u)[4], int j, const OnChip& oc,
                                                const DstCursor<GROUPED>& t, const LaneC& lc, const GroupQ& gq,
                                                const uint64_t* rtab, const float* ssm) {
    if constexpr (!GROUPED && !SMOOTH) {
        if (!gq.tiny) {   // warp-uniform
            const uint32_t m = oc.bm[j * kFWarps * 32];
            if (t.valid() && t.seg < a.full_segs)
                quantize_plain<true>(a, u, m, t, lc, rtab, oc.qtab);
            else
                quantize_plain<false>(a, u, m, t, lc, rtab, oc.qtab);
            return;
        }
    }
    quantize_any<GROUPED, SMOOTH>(a, u, t, lc, gq, rtab, ssm);
}

// Pass 2 of the one-tensor form (g >= 2^-64) when every task of the warp is
// on chip: tasks 0 .. nt - 1 in tensor memory, tasks nt .. n - 1 in slot
// i % kStage, where pass 1 left them.  One loop in task order with little
// live state: the values, the block amaxes from pass 1, the scale bytes from
// the quotient table, and a destination cursor advanced in place.
__device__ __forceinline__ void plain_pass2(const FusedArgs& a, const Ring& r, const LaneC& lc, int tw, int n, int nt,
                                            uint32_t tcol, const uint32_t* bm, const uint64_t* rtab,
                                            const int32_t* qtab) {
    int row = tw / a.nseg, seg = tw - row * a.nseg;
    const uint32_t kb2 = (uint32_t)(a.k >> 1);
    auto scale_off = [&](int rw, int sg) {
        const uint32_t rr = (uint32_t)rw;
        return (rr >> 7) * a.sc4x512 + (rr & 31u) * 16u + ((rr >> 5) & 3u) * 4u + ((uint32_t)sg << 13);
    };
    uint32_t co = (uint32_t)row * kb2 + ((uint32_t)seg << 9);
    uint32_t so = scale_off(row, seg);
    uint8_t* const cbase = a.codes + 16 * lc.lane;
    uint8_t* const sbase = a.scales + lc.s_off;
    const bool even = (lc.lane & 1) == 0;
    int s = nt % kStage;
    for (int i = 0; i < n; ++i) {
        uint4 u[4];
        uint32_t m;
        if (i < nt) {   // warp-uniform
            load_tmem(tcol + 16u * (uint32_t)i, u);
            m = bm[i * kFWarps * 32];
        } else {
            load_slot(r.slot(s), lc, u);
            m = bm[(kTmTasks + i - nt) * kFWarps * 32];
            s = (s + 1 == kStage) ? 0 : s + 1;
        }
        const uint32_t pair = block_sf2_tab(m, qtab);
        const uint64_t rr0 = rtab[pair & 0xFFu];
        const uint64_t rr1 = rtab[pair >> 8];
        uint4 q;
        q.x = quant8(u[0], rr0);
        q.y = quant8(u[1], rr0);
        q.z = quant8(u[2], rr1);
        q.w = quant8(u[3], rr1);
        const uint32_t word = __byte_perm(pair, __shfl_down_sync(kFull, pair, 1), 0x5410);
        if (row < a.rows && seg < a.full_segs) {
            *reinterpret_cast<uint4*>(cbase + co) = q;
            if (even) *reinterpret_cast<uint32_t*>(sbase + so) = word;
        } else {
            // padding rows and values past k: no codes; zero scale bytes in the padded tile
            if (row < a.rows && seg * kTaskVals + 32 * lc.lane < a.k) *reinterpret_cast<uint4*>(cbase + co) = q;
            if (even && seg * (kTaskVals / 16) + 2 * lc.lane < a.scale_cols)
                *reinterpret_cast<uint32_t*>(sbase + so) = word;
        }
        if (++seg == a.nseg) {
            seg = 0;
            ++row;
            co = (uint32_t)row * kb2;
            so = scale_off(row, 0);
        } else {
            co += kTaskVals / 2;
            so += 8192u;   // 16 scale tiles of 512 bytes per segment
        }
    }
}

template <bool GROUPED, bool SMOOTH>
__device__ __forceinline__ void fused_pass2(const CUtensorMap* tmap, const FusedArgs& a, const GroupTab& gt, Ring& r,
                                            const uint64_t* rtab, Pass2Q<GROUPED>& pq, uint32_t gen, int tw, int n,
                                            int nt, uint32_t tcol, const LaneC& lc, const float* ssm,
                                            const OnChip& oc) {
    const uint64_t pol = l2_policy_evict_first();   // last use
    const int nres = n < kStage ? n : kStage;
    const int nl = n - nres - nt;
    DstCursor<GROUPED> rp, lq;
    SrcCursor<GROUPED> lp;
    rp.init(a, gt, tw + n - nres);
    if (nl > 0) {
        lq.init(a, gt, tw + nt + nl - 1);
        lp.init(a, gt, tw + nt + nl - 1);
    }
    uint4 u[4];
    int s = (n - nres) % kStage;
    for (int k = 0; k < nres; ++k) {
        load_slot(r.slot(s), lc, u);
        __syncwarp();   // every lane is done reading the slot
        if (k < nl) {
            stage<GROUPED>(tmap, a, r, s, lp, pol, lc.lane);
            lp.prev(a, gt);
        }
        quantize_onchip<GROUPED, SMOOTH>(a, u, kTmTasks + k, oc, rp, lc, pq.at(a, rp, gen), rtab, ssm);
        rp.next(a, gt);
        s = (s + 1 == kStage) ? 0 : s + 1;
    }
    if (nt > 0) {
        DstCursor<GROUPED> tp;
        tp.init(a, gt, tw);
        for (int j = 0; j < nt; ++j) {
            load_tmem(tcol + 16u * (uint32_t)j, u);
            quantize_onchip<GROUPED, SMOOTH>(a, u, j, oc, tp, lc, pq.at(a, tp, gen), rtab, ssm);
            tp.next(a, gt);
        }
    }
    // s is back at the slot of the first slot task, where the first refill lands.
    for (int q = 0; q < nl; ++q) {
        land(r, s, a);
        load_slot(r.slot(s), lc, u);
        __syncwarp();
        if (q + kStage < nl) {
            stage<GROUPED>(tmap, a, r, s, lp, pol, lc.lane);
            lp.prev(a, gt);
        }
        quantize_any<GROUPED, SMOOTH>(a, u, lq, lc, pq.at(a, lq, gen), rtab, ssm);
        lq.prev(a, gt);
        s = (s + 1 == kStage) ? 0 : s + 1;
    }
}

// SMOOTH: the pre-scaled form (one tensor): x' = x s[column] is quantized.
template <bool GROUPED, bool SMOOTH = false>
__global__ void __launch_bounds__(kFThreads, 1)
    quant1d_fused_kernel(const __grid_constant__ CUtensorMap tmap, FusedArgs a, uint32_t box_bytes) {
    extern __shared__ __align__(1024) uint8_t dsm[];   // kStage task slots per warp (+ alignment pad)
    __shared__ __align__(8) uint64_t sbar[kStage * kFWarps];
    __shared__ uint64_t rtab[128];
    __shared__ uint32_t red[kFWarps];
    __shared__ int s_off[GROUPED ? kMaxFusedGroups + 1 : 1];
    __shared__ int s_blk[GROUPED ? kMaxFusedGroups + 1 : 1];
    __shared__ __align__(16) float s_smooth[SMOOTH ? kMaxSmoothK : 4];
    __shared__ uint32_t s_amax, s_gen, s_tmem;
    __shared__ int s_ok;
    constexpr bool kPlain = !GROUPED && !SMOOTH;
    // one tensor: packed block amaxes of the tasks kept on chip, [task][warp][lane]
    // (tensor-memory tasks 0 .. kTmTasks - 1, then the slot tasks)
    __shared__ uint32_t s_bm[kPlain ? (kTmTasks + kStage) * kFWarps * 32 : 1];
    __shared__ int32_t s_qtab[kPlain ? 128 : 1];
    // Launched as a programmatic dependent: everything below may read what
    // the previous kernel wrote (x, this workspace).
    pdl_wait();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int G = gridDim.x;
    const int t0 = (int)((int64_t)a.tasks * blockIdx.x / G);
    const int cnt = (int)((int64_t)a.tasks * (blockIdx.x + 1) / G) - t0;
    // Warp w takes a contiguous run of the CTA's tasks.
    const int tw = t0 + cnt * warp / kFWarps;
    int n = t0 + cnt * (warp + 1) / kFWarps - tw;
    // this CTA's word: the generation of its last call (read early, used late)
    const uint64_t gen_word = tid == 0 ? ld_relaxed_gpu_u64(a.part + kPartStrideWords * blockIdx.x) : 0ull;
    GroupTab gt;
    gt.off = s_off;
    gt.blk = s_blk;
    gt.G = a.groups;
    Ring r;
    r.base = reinterpret_cast<char*>(dsm) + ((1024u - (smem_u32(dsm) & 1023u)) & 1023u);   // 128-byte swizzle: 1 KB aligned
    r.bar = &sbar[warp * kStage];
    r.warp = warp;
    r.phase = 0;
    r.box_bytes = box_bytes;
    const LaneC lc = make_lanec(lane);
    const uint64_t pol_keep = l2_policy_evict_normal();   // read again in pass 2
    const uint64_t pol_last = l2_policy_evict_first();    // stays on chip: not read again
    SrcCursor<GROUPED> sp, lp;                            // pass 1: next task to copy; next task to land
    int nt = 0;   // this warp's first nt tasks stay in tensor memory
    // The first kStage copies of pass 1 (one commit group each, empty past n).
    // One tensor: issued before the set-up below, which they overlap.
    auto first_copies = [&]() {
        nt = max(0, min(a.tm_tasks, n - kStage));
        sp.init(a, gt, tw);
        lp.init(a, gt, tw);
#pragma unroll
        for (int i = 0; i < kStage; ++i) {
            if (i < n) {
                stage_cp<GROUPED>(a, r, i, sp, lc, (i < nt || i >= n - kStage) ? pol_last : pol_keep);
                sp.next(a, gt);
            }
            cp_async_commit();
        }
    };
    if constexpr (!GROUPED) first_copies();
    if (tid < kStage * kFWarps) mbar_init(&sbar[tid], 1);
    // Tensor memory (all 512 columns: 64 per warp, in the warp's own lane
    // quarter) when some warp has more tasks than shared-memory slots.
    if (a.tm_tasks > 0 && warp == 0) {
        tmem_alloc(&s_tmem, 512);
        tmem_relinquish();
    }
    if constexpr (GROUPED) {
        // offsets and the exclusive prefix of the groups' 128-row block counts
        // (a.groups <= kMaxFusedGroups = kFThreads)
        const int e = tid;
        int nb = 0;
        if (e < a.groups) {
            const int o0 = a.offsets[e], o1 = a.offsets[e + 1];
            s_off[e] = o0;
            if (e == a.groups - 1) s_off[a.groups] = o1;
            nb = (o1 - o0 + 127) / 128;
        }
        int inc = nb;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(kFull, inc, o);
            if (lane >= o) inc += v;
        }
        if (lane == 31) red[warp] = (uint32_t)inc;
        __syncthreads();
        int wbase = 0;
        for (int w = 0; w < warp; ++w) wbase += (int)red[w];
        if (e < a.groups) s_blk[e] = wbase + inc - nb;
        if (e == a.groups - 1) s_blk[a.groups] = wbase + inc;
    }
    if constexpr (SMOOTH) {
        // the factors, zero past k up to the last task's end (k <= kMaxSmoothK)
        const int kt = a.nseg * kTaskVals;
        for (int i = tid; i < kt; i += kFThreads) {
            const int seg = i / kTaskVals, u = (i % kTaskVals) >> 2;
            const int pu = (u & ~7) | ((u & 7) ^ ((u >> 3) & 7));
            s_smooth[seg * kTaskVals + pu * 4 + (i & 3)] = i < a.k ? a.smooth[i] : 0.0f;
        }
    }
    if (GROUPED && tid == 0) s_gen = (uint32_t)(gen_word >> 32) + 1u;   // grouped: every warp folds with it
    fence_mbar_init();
    __syncthreads();
    // one more than this CTA's last call's generation (the same in every CTA);
    // one tensor: only thread 0 uses it
    const uint32_t gen = GROUPED ? s_gen : (uint32_t)(gen_word >> 32) + 1u;
    if constexpr (GROUPED) {
        // the exact task count: tasks past it belong to no group
        const int real = 128 * s_blk[a.groups] * a.nseg;
        n = max(0, min(tw + n, real) - tw);
        first_copies();
    }
    if (lane == 0) prefetch_tmap(&tmap);
    // the first nt tasks stay in tensor memory, at columns tcol + 16 j
    uint32_t tcol = 0;
    if (a.tm_tasks > 0) {
        tc_fence_after();
        tcol = s_tmem + ((uint32_t)((warp & 3) * 32) << 16) + (uint32_t)((warp >> 2) * 16 * kTmTasks);
    }

    // ---- pass 1: amax through the slot ring; the first nt tasks are parked in
    // tensor memory, the last kStage stay in their slots
    uint32_t acc = 0;      // packed BF16 running max |x|
    float accf = 0.0f;     // pre-scaled form: running max |x s|
    {
        int cur = lp.m.e;                                     // grouped: the group acc belongs to
        // One commit group per step (empty once nothing is left): with at most
        // kStage - 1 groups pending, the oldest copy has landed.
        int s = 0;
        for (int i = 0; i < n; ++i) {
            cp_async_wait<kStage - 1>();
            __syncwarp();   // every lane's copies into the slot have landed
            int seg_now = 0;
            if constexpr (GROUPED || SMOOTH) {
                if constexpr (GROUPED) {
                    if (lp.m.e != cur) {   // warp-uniform: a new group starts with this task
                        uint32_t m = absmax_bits(acc) << 16;   // FP32 bits
#pragma unroll
                        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(kFull, m, o));
                        if (lane == 0) fold_group_amax(a.gword + cur, gen, m);
                        cur = lp.m.e;
                        acc = 0;
                    }
                }
                seg_now = lp.seg;
                lp.next(a, gt);
            }
            uint4 u[4];
            load_slot(r.slot(s), lc, u);
            if constexpr (SMOOTH) {
                const float* sb2 = s_smooth + seg_now * kTaskVals;
#pragma unroll
                for (int q = 0; q < 4; ++q)
                    accf = fmaxf(accf, absmax8_smooth(u[q], smooth_unit(sb2, lane, 2 * q),
                                                      smooth_unit(sb2, lane, 2 * q + 1)));
            } else if constexpr (GROUPED) {
#pragma unroll
                for (int q = 0; q < 4; ++q) acc = bmax_abs(acc, absmax8_packed(u[q]));
            } else {
                // block maxima (blocks 2 lane, 2 lane + 1), kept for the tasks
                // that stay on chip, then folded into the running maximum
                const uint32_t m0 = bmax_abs(absmax8_packed(u[0]), absmax8_packed(u[1]));
                const uint32_t m1 = bmax_abs(absmax8_packed(u[2]), absmax8_packed(u[3]));
                acc = bmax_abs(acc, bmax_abs(m0, m1));
                const int res0 = n - min(n, kStage);   // first slot task
                if (i < nt || i >= res0) {
                    const int j = i < nt ? i : kTmTasks + (i - res0);
                    s_bm[(j * kFWarps + warp) * 32 + lane] =
                        bmax_abs(__byte_perm(m0, m1, 0x5410), __byte_perm(m0, m1, 0x7632));
                }
            }
            if (i < nt) {
                const uint32_t w[16] = {u[0].x, u[0].y, u[0].z, u[0].w, u[1].x, u[1].y, u[1].z, u[1].w,
                                        u[2].x, u[2].y, u[2].z, u[2].w, u[3].x, u[3].y, u[3].z, u[3].w};
                tmem_st_32x32b_x16(tcol + 16u * (uint32_t)i, w);
            }
            if (i + kStage < n) {
                __syncwarp();   // every lane is done reading the slot
                stage_cp<GROUPED>(a, r, s, sp, lc,
                                  (i + kStage < nt || i + kStage >= n - kStage) ? pol_last : pol_keep);
                sp.next(a, gt);
            }
            cp_async_commit();
            s = (s + 1 == kStage) ? 0 : s + 1;
        }
        cp_async_wait<0>();
        if (nt > 0) tmem_st_wait();
        __syncwarp();
        if constexpr (GROUPED) {
            if (n > 0) {
                uint32_t m = absmax_bits(acc) << 16;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(kFull, m, o));
                if (lane == 0) fold_group_amax(a.gword + cur, gen, m);
            }
        }
    }
    if constexpr (!GROUPED) {
        uint32_t m = SMOOTH ? __float_as_uint(accf) : absmax_bits(acc) << 16;   // FP32 bits
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(kFull, m, o));
        if (lane == 0) red[warp] = m;
    }
    __syncthreads();

    // ---- grid barrier: arrive with this CTA's amax, wait for everyone's
    if (tid == 0) {
        uint32_t b = 0;
        if constexpr (!GROUPED)
            for (int w = 0; w < kFWarps; ++w) b = max(b, red[w]);
        st_relaxed_gpu_u64(a.part + kPartStrideWords * blockIdx.x, (uint64_t)gen << 32);   // next call: gen + 1
        // grouped: every warp's folds (ordered before this by the CTA barrier)
        // are released with the arrival
        if constexpr (GROUPED) fence_acq_rel_gpu();
        grid_arrive(a.bar, gen, b, blockIdx.x == 0);
        uint32_t amax_bits = 0;
        const bool got = grid_wait(a.bar, gen, G, a.limit, a.err, amax_bits);
        if constexpr (GROUPED) fence_acq_rel_gpu();   // the group words after every CTA's arrival
        s_ok = got ? 1 : 0;
        s_amax = amax_bits;
    }
    __syncthreads();
    const bool ok = s_ok != 0;
    // The next kernel in the stream may launch now: its CTAs cannot share an
    // SM with these (shared memory), so they start as each SM frees, and its
    // wait still covers this grid's completion and writes.
    pdl_launch_dependents();
    if (ok) {
        Pass2Q<GROUPED> pq;
        if constexpr (GROUPED) {
            for (int e = blockIdx.x * kFThreads + tid; e < a.groups; e += G * kFThreads)
                a.gscale[e] = make_groupq(group_amax(a.gword + e, gen)).g;
        } else {
            pq.q = make_groupq(s_amax);
            if (blockIdx.x == 0 && tid == 0) a.gscale[0] = pq.q.g;
            fill_rtab(rtab, pq.q.g, tid);
            if (kPlain && !pq.q.tiny) fill_qtab(s_qtab, pq.q.c.k6, tid - 128);
            __syncthreads();
        }
        const OnChip oc{s_bm + warp * 32 + lane, s_qtab};
        bool done = false;
        if constexpr (kPlain) {
            if (!pq.q.tiny && n - min(n, kStage) - nt == 0) {   // warp-uniform: every task on chip
                plain_pass2(a, r, lc, tw, n, nt, tcol, oc.bm, rtab, s_qtab);
                done = true;
            }
        }
        if (!done) fused_pass2<GROUPED, SMOOTH>(&tmap, a, gt, r, rtab, pq, gen, tw, n, nt, tcol, lc, s_smooth, oc);
    }
    if (a.tm_tasks > 0) {   // every warp's tensor-memory reads are done (tcgen05.wait::ld after each)
        tc_fence_before();
        __syncthreads();
        if (warp == 0) tmem_dealloc(s_tmem, 512);
    }
}

// ---- kernel 2 (weights): 16 x 16 blocks -------------------------------------------
struct Quant2dArgs {
    const uint16_t* x;
    int64_t ld;
    int n, k, nseg, scale_cols;
    const float* gscale;
    uint8_t* codes;
    uint8_t* scales;
    uint8_t* compact;   // optional [n/16, k/16]
};

__global__ void __launch_bounds__(kThreads) quant2d_kernel(Quant2dArgs a) {
    pdl_launch_dependents();
    pdl_wait();
    const float g = a.gscale[0];
    const float k6 = __fmul_rn(6.0f, g);
    const bool tiny = g < kTinyG;
    const int ntasks = (round128(a.n) / 16) * a.nseg;
    const int lane = threadIdx.x & 31;
    const int wstride = gridDim.x * kWarps;
    const int64_t kbytes = a.k / 2;
    for (int t = blockIdx.x * kWarps + (threadIdx.x >> 5); t < ntasks; t += wstride) {
        const int tr = t / a.nseg;
        const int seg = t - tr * a.nseg;
        const int col = seg * 256 + lane * 8;
        const bool valid = (tr * 16 < a.n) && (col < a.k);
        uint4 v[16];
#pragma unroll
        for (int i = 0; i < 16; ++i)
            v[i] = valid ? ld_nc_v4(a.x + (int64_t)(tr * 16 + i) * a.ld + col) : make_uint4(0, 0, 0, 0);
        uint32_t pm = 0;
#pragma unroll
        for (int i = 0; i < 16; ++i) pm = bmax_abs(pm, absmax8_packed(v[i]));
        uint32_t am = absmax_bits(pm);
        am = max(am, __shfl_xor_sync(kFull, am, 1));
        float r;
        const uint32_t sf = block_scale(__uint_as_float(am << 16), g, k6, tiny, r);
        const uint64_t rr = pack_rr(r);
        if (valid) {
            uint8_t* dst = a.codes + (int64_t)(tr * 16) * kbytes + col / 2;
            if (tiny) {   // uniform: one global scale
#pragma unroll
                for (int i = 0; i < 16; ++i) *reinterpret_cast<uint32_t*>(dst + i * kbytes) = quant8<true>(v[i], rr);
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) *reinterpret_cast<uint32_t*>(dst + i * kbytes) = quant8(v[i], rr);
            }
            if (a.compact && (lane & 1) == 0) a.compact[(int64_t)tr * (a.k / 16) + col / 16] = (uint8_t)sf;
        }
        const uint32_t s1 = __shfl_down_sync(kFull, sf, 2);
        const uint32_t s2 = __shfl_down_sync(kFull, sf, 4);
        const uint32_t s3 = __shfl_down_sync(kFull, sf, 6);
        const int scol = seg * 16 + (lane >> 1);
        if ((lane & 7) == 0 && scol < a.scale_cols) {
            const uint32_t word = (tr * 16 < a.n) ? (sf | (s1 << 8) | (s2 << 16) | (s3 << 24)) : 0u;
#pragma unroll
            for (int i = 0; i < 16; ++i)
                *reinterpret_cast<uint32_t*>(a.scales + sf_tile_offset(tr * 16 + i, scol, a.scale_cols)) = word;
        }
    }
}

// ---- format probe -------------------------------------------------------------------
__global__ void probe_cvt_kernel(const float* in, uint8_t* e2m1, uint8_t* e4m3, int64_t n) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
        const float x = in[i];
        if (e2m1) e2m1[i] = (uint8_t)cvt_e2m1(x);
        if (e4m3) e4m3[i] = (uint8_t)cvt_e4m3(fabsf(x));
    }
}

int clamp_grid(int64_t want, int64_t hi) {
    if (want < 1) want = 1;
    if (want > hi) want = hi;
    if (want < 1) want = 1;
    return (int)want;
}

cudaError_t launch_pdl(const void* func, dim3 grid, dim3 block, void** args, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = 0;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelExC(&cfg, func, args);
}

// One-launch quantization of one tensor, or of row groups (offsets != nullptr,
// at most kMaxFusedGroups).  Returns NVFP4_ERR_UNSUPPORTED_SHAPE (nothing
// launched) when the tensor does not fit its layout -- k % 64 != 0, or codes /
// scales too large for 32-bit offsets -- or the device cannot hold one such
// CTA per SM; the caller then takes the two-kernel path.
nvfp4_status_t run_fused(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, const int32_t* offsets, int groups,
                         uint8_t* codes, uint8_t* scales, float* gscale, void* workspace, cudaStream_t s,
                         const float* smooth = nullptr) {
    constexpr int kSmemMax = kStage * kFWarps * kTaskBytes + 1024;
    const bool grouped = offsets != nullptr;
    if (grouped && groups > kMaxFusedGroups) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (smooth && (grouped || round_up(k, kTaskVals) > kMaxSmoothK)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const int64_t prow = round_up(rows + (grouped ? 127 * (int64_t)groups : 0), 128);   // padded rows, at most
    if (k % 64 != 0 || prow * k >= ((int64_t)1 << 31)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    static std::mutex mu;
    static int ready[64] = {};   // per device: 0 unknown, 1 usable, -1 not usable
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NVFP4_ERR_CUDA;
    {
        std::lock_guard<std::mutex> lk(mu);
        if (ready[dev] == 0) {
            int occ0 = 0, occ1 = 0, occ2 = 0;
            const bool ok =
                tensor_map_encoder() != nullptr &&
                cudaFuncSetAttribute(quant1d_fused_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kSmemMax) == cudaSuccess &&
                cudaFuncSetAttribute(quant1d_fused_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kSmemMax) == cudaSuccess &&
                cudaFuncSetAttribute(quant1d_fused_kernel<false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kSmemMax) == cudaSuccess &&
                cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ0, quant1d_fused_kernel<false>, kFThreads,
                                                              kSmemMax) == cudaSuccess &&
                cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ1, quant1d_fused_kernel<true>, kFThreads,
                                                              kSmemMax) == cudaSuccess &&
                cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ2, quant1d_fused_kernel<false, true>, kFThreads,
                                                              kSmemMax) == cudaSuccess &&
                occ0 >= 1 && occ1 >= 1 && occ2 >= 1;
            ready[dev] = ok ? 1 : -1;
        }
        if (ready[dev] < 0) {
            cudaGetLastError();
            return NVFP4_ERR_UNSUPPORTED_SHAPE;
        }
    }
    // x as a 3-D tensor [rows][k / 64][64]: one box = one task (16 x 64 values of a
    // row; narrower when k < 1024), 128-byte swizzle, zero fill past the tensor.
    const cuuint32_t box1 = (cuuint32_t)(k / 64 < kTaskVals / 64 ? k / 64 : kTaskVals / 64);
    CUtensorMap tmap;
    {
        const cuuint64_t dims[3] = {64, (cuuint64_t)(k / 64), (cuuint64_t)(rows > 0 ? rows : 1)};
        const cuuint64_t strides[2] = {128, (cuuint64_t)ld * 2};
        const cuuint32_t box[3] = {64, box1, 1};
        const cuuint32_t estr[3] = {1, 1, 1};
        if (tensor_map_encoder()(&tmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<uint16_t*>(x), dims, strides,
                                 box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                 CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return NVFP4_ERR_UNSUPPORTED_SHAPE;
    }
    uint32_t box_bytes = box1 * 128u;
    FusedArgs a;
    a.x = x;
    a.ld = ld;
    a.rows = (int)rows;
    a.k = (int)k;
    a.nseg = (int)((k + kTaskVals - 1) / kTaskVals);
    a.scale_cols = (int)(k / 16);
    a.tasks = (int)(prow * a.nseg);
    a.full_segs = (int)(k / kTaskVals);
    a.sc4x512 = (uint32_t)(a.scale_cols / 4) * 512u;
    // One CTA per SM, for every tensor: the grid-barrier generations live in
    // the CTAs' own words, so the grid must not change from call to call.
    const int G = num_sms() < kMaxFusedCtas ? num_sms() : kMaxFusedCtas;
    const int64_t per = (a.tasks + G - 1) / G;
    const int64_t per_warp = (per + kFWarps - 1) / kFWarps;
    const int depth = (int)(per_warp < kStage ? per_warp : kStage);
    a.gscale = gscale;
    a.codes = codes;
    a.scales = scales;
    a.part = reinterpret_cast<uint64_t*>(workspace);
    a.bar = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(workspace) + quant_ws_bar_off());
    a.gword = reinterpret_cast<uint64_t*>(reinterpret_cast<uint8_t*>(workspace) + quant_ws_gword_off(groups));
    // Warps with more tasks than slots park up to kTmTasks of them in tensor
    // memory, so that pass 2 re-reads none (or fewer) from L2.
    a.tm_tasks = per_warp > kStage ? kTmTasks : 0;
    a.offsets = offsets;
    a.groups = grouped ? groups : 1;
    a.smooth = smooth;
    a.limit = wait_limit_ns();
    a.err = device_error_word();
    if (!a.err) return NVFP4_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)G);
    cfg.blockDim = dim3(kFThreads);
    cfg.dynamicSmemBytes = (size_t)(depth > 0 ? depth : 1) * kFWarps * kTaskBytes + 1024;
    cfg.stream = s;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeCooperative;   // all CTAs resident at once (grid barrier)
    attr[0].val.cooperative = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;   // may launch early; waits first
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    void* args[] = {&tmap, &a, &box_bytes};
    const void* kern = grouped  ? reinterpret_cast<const void*>(&quant1d_fused_kernel<true>)
                       : smooth ? reinterpret_cast<const void*>(&quant1d_fused_kernel<false, true>)
                                : reinterpret_cast<const void*>(&quant1d_fused_kernel<false>);
    return cuda_status(cudaLaunchKernelExC(&cfg, kern, args));
}

nvfp4_status_t run_amax(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, const int32_t* offsets, int groups,
                        void* workspace, float* gscale, cudaStream_t s) {
    AmaxArgs a;
    a.x = x;
    a.ld = ld;
    a.k = (int)k;
    a.groups.offsets = offsets;
    a.groups.rows = (int)rows;
    a.num_groups = groups;
    a.ws = reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(workspace) + quant_ws_two_off());
    a.pad_rows = offsets ? reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(workspace) + quant_ws_pad_off(groups))
                         : nullptr;
    a.gscale = gscale;
    const int64_t chunks = rows * (k / 8);
    const int64_t per_group = (chunks + groups - 1) / groups;
    const int gx = clamp_grid((per_group + kThreads * kAmaxUnroll - 1) / (kThreads * kAmaxUnroll),
                              (int64_t)num_sms() * 4 / groups);
    void* args[] = {&a};
    return cuda_status(launch_pdl(reinterpret_cast<const void*>(&amax_kernel), dim3(gx, groups), dim3(kThreads), args, s));
}

}  // namespace

// The two-kernel form: the amax kernel, then the quantize kernel launched as
// its programmatic dependent (its first loads of x precede its wait).  Small
// CTAs (256 threads): a dependent GEMM's CTAs fit beside them on every SM.
nvfp4_status_t run_two_kernel(const uint16_t* xb, int64_t rows, int64_t k, int64_t ld, const int32_t* group_offsets,
                              int groups, uint8_t* codes, uint8_t* scales, float* global_scale, void* workspace,
                              cudaStream_t s) {
    nvfp4_status_t st = run_amax(xb, rows, k, ld, group_offsets, groups, workspace, global_scale, s);
    if (st != NVFP4_OK) return st;

    Quant1dArgs q;
    q.x = xb;
    q.ld = ld;
    q.k = (int)k;
    q.nseg = (int)((k + 511) / 512);
    q.scale_cols = (int)(round_up(k / 16, 4));
    q.groups.offsets = group_offsets;
    q.groups.rows = (int)rows;
    q.pad_rows = group_offsets ? reinterpret_cast<const int32_t*>(reinterpret_cast<uint8_t*>(workspace) +
                                                                 quant_ws_pad_off(groups))
                               : nullptr;
    q.gscale = global_scale;
    q.codes = codes;
    q.scales = scales;
    const int64_t tasks = (round_up(rows, 128) + (group_offsets ? 127 * (int64_t)groups : 0)) * q.nseg;
    const int64_t per_group = (tasks + groups - 1) / groups;
    const int qx = clamp_grid((per_group + kWarps * kQuantUnroll - 1) / (kWarps * kQuantUnroll),
                              (int64_t)num_sms() * 4 / groups);
    void* args[] = {&q};
    return cuda_status(launch_pdl(reinterpret_cast<const void*>(&quant1d_kernel<false>), dim3(qx, groups), dim3(kThreads),
                                  args, s));
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status_t nvfp4_quantize_act(const void* x, int64_t rows, int64_t k, int64_t ld,
                                             const int32_t* group_offsets, int num_groups, uint8_t* codes,
                                             uint8_t* scales, float* global_scale, void* workspace,
                                             void* stream) {
    if (rows < 0 || k <= 0 || ld < k) return NVFP4_ERR_INVALID_ARGUMENT;
    if (!x || !codes || !scales || !global_scale || !workspace) return NVFP4_ERR_INVALID_ARGUMENT;
    if (group_offsets && num_groups < 1) return NVFP4_ERR_INVALID_ARGUMENT;
    if (!group_offsets && num_groups > 1) return NVFP4_ERR_INVALID_ARGUMENT;
    if (k % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const int groups = group_offsets ? num_groups : 1;
    if (groups > 65535) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const int64_t nseg = (k + 255) / 256;
    if (rows * (k / 8) >= (int64_t)1 << 40 || round_up(rows + 127 * (int64_t)groups, 128) * nseg >= ((int64_t)1 << 31) ||
        rows >= ((int64_t)1 << 31) || k >= ((int64_t)1 << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(workspace) ||
        (reinterpret_cast<uintptr_t>(global_scale) & 3u) || (group_offsets && (reinterpret_cast<uintptr_t>(group_offsets) & 3u)) ||
        ld % 8 != 0)
        return NVFP4_ERR_MISALIGNED;
    if (num_sms() <= 0) return NVFP4_ERR_NO_DEVICE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const uint16_t* xb = reinterpret_cast<const uint16_t*>(x);
    {
        const nvfp4_status_t fs =
            run_fused(xb, rows, k, ld, group_offsets, groups, codes, scales, global_scale, workspace, s);
        if (fs != NVFP4_ERR_UNSUPPORTED_SHAPE) return fs;
    }
    return run_two_kernel(xb, rows, k, ld, group_offsets, groups, codes, scales, global_scale, workspace, s);
}

extern "C" nvfp4_status_t nvfp4_quantize_weight_2d(const void* w, int64_t n, int64_t k, int64_t ld, uint8_t* codes,
                                                   uint8_t* scales, uint8_t* scales_compact, float* global_scale,
                                                   void* workspace, void* stream) {
    if (n < 0 || k <= 0 || ld < k) return NVFP4_ERR_INVALID_ARGUMENT;
    if (!w || !codes || !scales || !global_scale || !workspace) return NVFP4_ERR_INVALID_ARGUMENT;
    if (k % 16 != 0 || n % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const int64_t nseg = (k + 255) / 256;
    if (n >= ((int64_t)1 << 31) || k >= ((int64_t)1 << 31) || (round_up(n, 128) / 16) * nseg >= ((int64_t)1 << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(w) || !aligned16(codes) || !aligned16(scales) || !aligned16(workspace) ||
        (reinterpret_cast<uintptr_t>(global_scale) & 3u) || ld % 8 != 0)
        return NVFP4_ERR_MISALIGNED;
    if (num_sms() <= 0) return NVFP4_ERR_NO_DEVICE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const uint16_t* wb = reinterpret_cast<const uint16_t*>(w);
    nvfp4_status_t st = run_amax(wb, n, k, ld, nullptr, 1, workspace, global_scale, s);
    if (st != NVFP4_OK) return st;
    Quant2dArgs q;
    q.x = wb;
    q.ld = ld;
    q.n = (int)n;
    q.k = (int)k;
    q.nseg = (int)nseg;
    q.scale_cols = (int)round_up(k / 16, 4);
    q.gscale = global_scale;
    q.codes = codes;
    q.scales = scales;
    q.compact = scales_compact;
    const int64_t tasks = (round_up(n, 128) / 16) * nseg;
    const int qx = clamp_grid((tasks + kWarps - 1) / kWarps, (int64_t)num_sms() * 8);
    void* args[] = {&q};
    return cuda_status(launch_pdl(reinterpret_cast<const void*>(&quant2d_kernel), dim3(qx), dim3(kThreads), args, s));
}

extern "C" nvfp4_status_t nvfp4_probe_cvt(const float* in, uint8_t* out_e2m1, uint8_t* out_e4m3, int64_t n,
                                          void* stream) {
    if (n < 0 || !in || (!out_e2m1 && !out_e4m3)) return NVFP4_ERR_INVALID_ARGUMENT;
    if (n == 0) return NVFP4_OK;
    if (num_sms() <= 0) return NVFP4_ERR_NO_DEVICE;
    const int grid = clamp_grid((n + 255) / 256, (int64_t)num_sms() * 16);
    probe_cvt_kernel<<<grid, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(in, out_e2m1, out_e4m3, n);
    return cuda_status(cudaGetLastError());
}

extern "C" nvfp4_status_t nvfp4_quantize_act_smooth(const void* x, int64_t rows, int64_t k, int64_t ld,
                                                    const float* smooth, uint8_t* codes, uint8_t* scales,
                                                    float* global_scale, void* workspace, void* stream) {
    if (rows < 0 || k <= 0 || ld < k) return NVFP4_ERR_INVALID_ARGUMENT;
    if (!x || !smooth || !codes || !scales || !global_scale || !workspace) return NVFP4_ERR_INVALID_ARGUMENT;
    if (k % 64 != 0 || round_up(k, kTaskVals) > kMaxSmoothK || rows >= ((int64_t)1 << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || !aligned16(workspace) ||
        (reinterpret_cast<uintptr_t>(smooth) & 3u) || (reinterpret_cast<uintptr_t>(global_scale) & 3u) || ld % 8 != 0)
        return NVFP4_ERR_MISALIGNED;
    if (num_sms() <= 0) return NVFP4_ERR_NO_DEVICE;
    return run_fused(reinterpret_cast<const uint16_t*>(x), rows, k, ld, nullptr, 1, codes, scales, global_scale,
                     workspace, reinterpret_cast<cudaStream_t>(stream), smooth);
}

extern "C" nvfp4_status_t nvfp4_quantize_act_scaled(const void* x, int64_t rows, int64_t k, int64_t ld,
                                                    const float* global_scale, uint8_t* codes, uint8_t* scales,
                                                    void* stream) {
    if (rows < 0 || k <= 0 || ld < k) return NVFP4_ERR_INVALID_ARGUMENT;
    if (!x || !codes || !scales || !global_scale) return NVFP4_ERR_INVALID_ARGUMENT;
    if (k % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const int64_t nseg = (k + 511) / 512;
    if (rows * (k / 8) >= (int64_t)1 << 40 || round_up(rows, 128) * nseg >= ((int64_t)1 << 31) ||
        rows >= ((int64_t)1 << 31) || k >= ((int64_t)1 << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) ||
        (reinterpret_cast<uintptr_t>(global_scale) & 3u) || ld % 8 != 0)
        return NVFP4_ERR_MISALIGNED;
    if (num_sms() <= 0) return NVFP4_ERR_NO_DEVICE;
    if (rows == 0) return NVFP4_OK;
    Quant1dArgs q;
    q.x = reinterpret_cast<const uint16_t*>(x);
    q.ld = ld;
    q.k = (int)k;
    q.nseg = (int)nseg;
    q.scale_cols = (int)(round_up(k / 16, 4));
    q.groups.offsets = nullptr;
    q.groups.rows = (int)rows;
    q.pad_rows = nullptr;
    q.gscale = global_scale;
    q.codes = codes;
    q.scales = scales;
    const int64_t tasks = round_up(rows, 128) * q.nseg;
    const int qx = clamp_grid((tasks + kWarps * kQuantUnroll - 1) / (kWarps * kQuantUnroll), (int64_t)num_sms() * 4);
    // A plain launch: x may come from the previous kernel on the stream, whose
    // end this kernel must not overlap (its first loads precede its
    // griddepcontrol.wait, which returns at once without the launch attribute).
    quant1d_kernel<false><<<dim3(qx, 1), kThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(q);
    return cuda_status(cudaGetLastError());
}

extern "C" nvfp4_status_t mxfp4_quantize_act(const void* x, int64_t rows, int64_t k, int64_t ld, uint8_t* codes,
                                             uint8_t* scales, void* stream) {
    if (rows < 0 || k <= 0 || ld < k) return NVFP4_ERR_INVALID_ARGUMENT;
    if (rows == 0) return NVFP4_OK;   // nothing to read or write (the pointers may be NULL)
    if (!x || !codes || !scales) return NVFP4_ERR_INVALID_ARGUMENT;
    if (k % 32 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    const int64_t nseg = (k + 511) / 512;
    if (rows * (k / 8) >= (int64_t)1 << 40 || round_up(rows, 128) * nseg >= ((int64_t)1 << 31) ||
        rows >= ((int64_t)1 << 31) || k >= ((int64_t)1 << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || ld % 8 != 0) return NVFP4_ERR_MISALIGNED;
    if (num_sms() <= 0) return NVFP4_ERR_NO_DEVICE;
    Quant1dArgs q;
    q.x = reinterpret_cast<const uint16_t*>(x);
    q.ld = ld;
    q.k = (int)k;
    q.nseg = (int)nseg;
    q.scale_cols = (int)(round_up(k / 32, 4));
    q.groups.offsets = nullptr;
    q.groups.rows = (int)rows;
    q.pad_rows = nullptr;
    q.gscale = nullptr;
    q.codes = codes;
    q.scales = scales;
    const int64_t tasks = round_up(rows, 128) * q.nseg;
    const int qx = clamp_grid((tasks + kWarps * kQuantUnroll - 1) / (kWarps * kQuantUnroll), (int64_t)num_sms() * 4);
    quant1d_kernel<true><<<dim3(qx, 1), kThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(q);
    return cuda_status(cudaGetLastError());
}

// ---- quantization without a caller-provided workspace --------------------------------
//
// Some callers cannot allocate device memory at the point where they quantize:
// a plugin whose host engine owns every byte of device memory and hands out no
// allocator, or a latency-critical path where cudaMalloc (which may
// synchronize the device) is not allowed.  For them the scratch lives in a
// fixed array in this library's device image, sized for up to
// kStaticMaxGroups row groups; every GPU that loads the library holds it
// until the process exits.
namespace nvfp4 {
namespace {
constexpr int kStaticMaxGroups = 1024;
constexpr int64_t kStaticScratchBytes = quant_ws_bytes(kStaticMaxGroups);   // 49408 bytes
std::mutex g_static_mu;
void* g_static_ptr[64] = {};
}  // namespace
}  // namespace nvfp4

static __device__ __align__(256) uint8_t g_static_quant_scratch[nvfp4::kStaticScratchBytes];

namespace nvfp4 {
namespace {
// Device address of g_static_quant_scratch on the current device.  Host code
// must not pass the symbol itself to a kernel: on the host it names a
// host-side stand-in, not device memory.  Looked up once per device, with
// that device current, and kept for the life of the device's primary context
// (the address does not survive a cudaDeviceReset, after which this library
// cannot be used on that device).  A failed lookup is also cleared from the
// runtime's last-error slot, so that no later, unrelated call reports it.
void* static_scratch() {
    int d = -1;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(g_static_mu);
    if (!g_static_ptr[d]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_quant_scratch) != cudaSuccess || !p) {
            cudaGetLastError();
            return nullptr;
        }
        g_static_ptr[d] = p;
    }
    return g_static_ptr[d];
}
}  // namespace
}  // namespace nvfp4

extern "C" nvfp4_status_t nvfp4_quantize_act_static(const void* x, int64_t rows, int64_t k, int64_t ld,
                                                    const int32_t* group_offsets, int num_groups, uint8_t* codes,
                                                    uint8_t* scales, float* global_scale, void* stream) {
    if (rows < 0 || k <= 0 || ld < k || !x || !codes || !scales || !global_scale) return NVFP4_ERR_INVALID_ARGUMENT;
    if (group_offsets && num_groups < 1) return NVFP4_ERR_INVALID_ARGUMENT;
    if (!group_offsets && num_groups > 1) return NVFP4_ERR_INVALID_ARGUMENT;
    if (k % 16 != 0) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (group_offsets && num_groups > kStaticMaxGroups) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (num_sms() <= 0) return NVFP4_ERR_NO_DEVICE;
    void* ws = static_scratch();
    if (!ws) return NVFP4_ERR_CUDA;
    const int groups = group_offsets ? num_groups : 1;
    // The workspace must be as a fresh one (zeros); the array keeps whatever
    // the previous call on this device left in it.
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, (size_t)quant_ws_bytes(groups), s) != cudaSuccess) return NVFP4_ERR_CUDA;
    return nvfp4_quantize_act(x, rows, k, ld, group_offsets, num_groups, codes, scales, global_scale, ws, stream);
}
