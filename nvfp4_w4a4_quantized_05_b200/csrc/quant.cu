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
//     d    = float(sf) * g ;  r = d == 0 ? 0 : min(1 / d, FLT_MAX)
//     code = e2m1_rn_satfinite(x * r)
// Every step is one IEEE binary32 operation rounded to nearest even
// (__fdiv_rn / __fmul_rn / __frcp_rn, compiled with -fmad=false), and the
// roundings to E4M3 / E2M1 are the hardware cvt.rn.satfinite instructions, so
// the codes and scale bytes are bit-identical to the CPU definition.
//
// Memory-bound design.  Kernel 1 (amax) runs as one wave of CTAs that stream
// the tensor with 16-byte loads, 8 in flight per thread, keeping a packed
// BF16 running max (max.xorsign.abs.bf16x2: one instruction per 2 x 2 values);
// the tensor normally stays in the 126 MB L2 for the second pass.  It ends with a
// "last CTA" step that publishes g, writes the group scale offsets and
// re-zeroes the workspace.  Kernel 2 (quantize) is launched with programmatic
// dependent launch: its CTAs issue their first loads (tagged evict_first)
// before waiting for kernel 1, since only g depends on it.  A warp task is
// 512 consecutive elements of one row; lane l owns 16-element block l (two
// 16-byte loads), so the block amax, the E4M3 scale and the reciprocal are
// computed once per block; the 16 codes leave as one 8-byte store (the warp
// writes 256 contiguous bytes) and 4 scale bytes are gathered by shuffles
// into one word of the 512-byte scale tile.  Task stepping is division-free.
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
__device__ __forceinline__ uint32_t absmax8_bits(const uint4& v) { return absmax_bits(absmax8_packed(v)); }

// (lo, hi) BF16 pair times (r, r): two IEEE round-to-nearest products.
__device__ __forceinline__ void mul_bf16x2(uint32_t w, uint64_t rr, float& lo, float& hi) {
    uint64_t x, y;
    asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "r"(w << 16), "r"(w & 0xFFFF0000u));
    asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(y) : "l"(x), "l"(rr));
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(y));
}
__device__ __forceinline__ uint64_t pack_rr(float r) {
    uint64_t rr;
    asm("mov.b64 %0, {%1, %1};" : "=l"(rr) : "f"(r));
    return rr;
}

// Eight BF16 values times r -> eight packed E2M1 codes.
__device__ __forceinline__ uint32_t quant8(const uint4& v, uint64_t rr) {
    float x[8];
    mul_bf16x2(v.x, rr, x[0], x[1]);
    mul_bf16x2(v.y, rr, x[2], x[3]);
    mul_bf16x2(v.z, rr, x[4], x[5]);
    mul_bf16x2(v.w, rr, x[6], x[7]);
    return cvt_e2m1x8(x[0], x[1], x[2], x[3], x[4], x[5], x[6], x[7]);
}

// Block scale byte and element multiplier from the block amax.
__device__ __forceinline__ uint32_t block_scale(float bamax, float g, float k6, float& r) {
    const uint32_t sf = cvt_e4m3(__fdiv_rn(bamax, k6));
    const float d = __fmul_rn(e4m3_to_f32(sf), g);
    r = (d == 0.0f) ? 0.0f : fminf(__frcp_rn(d), FLT_MAX);
    return sf;
}

__device__ __forceinline__ int64_t sf_tile_offset(int srow, int scol, int scale_cols) {
    return ((int64_t)(srow >> 7) * (scale_cols >> 2) + (scol >> 2)) * 512 + (srow & 31) * 16 +
           ((srow >> 5) & 3) * 4 + (scol & 3);
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

__global__ void __launch_bounds__(kThreads, 4) amax_kernel(AmaxArgs a) {
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
    pdl_launch_dependents();
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

__global__ void __launch_bounds__(kThreads, 4) quant1d_kernel(Quant1dArgs a) {
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
    const float g = a.gscale[e];
    const float k6 = __fmul_rn(6.0f, g);

    while (tp[0].row < prows) {
#pragma unroll
        for (int u = 0; u < kQuantUnroll; ++u) {
            const TaskPos t = tp[u];
            if (t.row >= prows) break;   // uniform across the warp
            const int col = t.seg * 512 + lane * 16;
            const uint32_t am = absmax_bits(bmax_abs(absmax8_packed(v[u][0]), absmax8_packed(v[u][1])));
            float r;
            const uint32_t sf = block_scale(__uint_as_float(am << 16), g, k6, r);
            if (t.row < nrows && col < a.k) {
                const uint64_t rr = pack_rr(r);
                uint2 q;
                q.x = quant8(v[u][0], rr);
                q.y = quant8(v[u][1], rr);
                *reinterpret_cast<uint2*>(a.codes + (int64_t)(r0 + t.row) * kbytes + col / 2) = q;
            }
            const uint32_t s1 = __shfl_down_sync(kFull, sf, 1);
            const uint32_t s2 = __shfl_down_sync(kFull, sf, 2);
            const uint32_t s3 = __shfl_down_sync(kFull, sf, 3);
            const int scol = t.seg * 32 + lane;
            if ((lane & 3) == 0 && scol < a.scale_cols) {
                const uint32_t word = (t.row < nrows) ? (sf | (s1 << 8) | (s2 << 16) | (s3 << 24)) : 0u;
                *reinterpret_cast<uint32_t*>(a.scales + sf_tile_offset(srow0 + t.row, scol, a.scale_cols)) = word;
            }
        }
#pragma unroll
        for (int u = 0; u < kQuantUnroll; ++u) {
            tp[u].advance(drow, dseg, nseg);
            load_block16(a, r0, nrows, tp[u], lane, pol, v[u][0], v[u][1]);
        }
    }
    pdl_launch_dependents();
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
    pdl_wait();
    const float g = a.gscale[0];
    const float k6 = __fmul_rn(6.0f, g);
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
        const uint32_t sf = block_scale(__uint_as_float(am << 16), g, k6, r);
        const uint64_t rr = pack_rr(r);
        if (valid) {
#pragma unroll
            for (int i = 0; i < 16; ++i)
                *reinterpret_cast<uint32_t*>(a.codes + (int64_t)(tr * 16 + i) * kbytes + col / 2) =
                    quant8(v[i], rr);
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
    pdl_launch_dependents();
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

nvfp4_status_t run_amax(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, const int32_t* offsets, int groups,
                        void* workspace, float* gscale, cudaStream_t s) {
    AmaxArgs a;
    a.x = x;
    a.ld = ld;
    a.k = (int)k;
    a.groups.offsets = offsets;
    a.groups.rows = (int)rows;
    a.num_groups = groups;
    a.ws = reinterpret_cast<uint32_t*>(workspace);
    a.pad_rows = offsets ? reinterpret_cast<int32_t*>(reinterpret_cast<uint8_t*>(workspace) + quant_ws_pad_off(groups))
                         : nullptr;
    a.gscale = gscale;
    const int64_t chunks = rows * (k / 8);
    const int64_t per_group = (chunks + groups - 1) / groups;
    const int gx = clamp_grid((per_group + kThreads * kAmaxUnroll - 1) / (kThreads * kAmaxUnroll),
                              (int64_t)num_sms() * 4 / groups);
    amax_kernel<<<dim3(gx, groups), kThreads, 0, s>>>(a);
    return cuda_status(cudaGetLastError());
}

}  // namespace
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
    return cuda_status(launch_pdl(reinterpret_cast<const void*>(&quant1d_kernel), dim3(qx, groups), dim3(kThreads),
                                  args, s));
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
constexpr int64_t kStaticScratchBytes = quant_ws_bytes(kStaticMaxGroups);   // 8448 bytes
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
// that device current.
void* static_scratch() {
    int d = -1;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 64) return nullptr;
    std::lock_guard<std::mutex> lk(g_static_mu);
    if (!g_static_ptr[d]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_quant_scratch) != cudaSuccess || !p) return nullptr;
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
    // The CTA counter and the amax slots must start at zero; the array keeps
    // whatever the previous call on this device left in it.
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaMemsetAsync(ws, 0, (size_t)quant_ws_pad_off(groups), s) != cudaSuccess) return NVFP4_ERR_CUDA;
    return nvfp4_quantize_act(x, rows, k, ld, group_offsets, num_groups, codes, scales, global_scale, ws, stream);
}
