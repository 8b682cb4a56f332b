// w4a16.cu -- BF16 activations x NVFP4 weights (W4A16) for decode-sized m.
//
// The weight-only form that "W4A8 vs NVFP4 quantization on GPUs" ("Batch size
// can change the winner", "Dequantization can erase a four-bit win") sets
// against W4A4: the same NVFP4 weight stream, dequantized to BF16 inside the
// kernel and fed to BF16 tensor-core MMAs, with the activations left in BF16.
//
// One CTA per SM (persistent), 14 warps:
//   warps 0..11  dequantize: one 64-wide k-slice of the tile's 192 weight rows
//                per step, E2M1 x E4M3 -> BF16 (exact: at most 6 significant
//                bits, magnitudes 2^-10 .. 2688), written in the MMA's
//                128-byte-swizzled K-major layout.  Warps 0 and 1 also drain
//                the accumulator.
//   warp 12      TMA producer: activation slices [64 tokens x 64] (BF16) and
//                raw weight tiles [192 rows x 256 values] (FP4 codes, 128-byte
//                swizzle) with their scale chunks (bulk copies).
//   warp 13      MMA issuer (tcgen05.mma kind::f16, BF16 x BF16 -> FP32, M = 64
//                token rows, N = 192 weight rows, K = 16) and tensor-memory
//                owner.  With M = 64 the accumulator rows 16 q .. 16 q + 15 sit
//                in tensor-memory lanes 32 q .. 32 q + 15, so dequantizing warps
//                0..3 (one per lane quarter) drain it.
// Every wait is bounded; on expiry the kernel sets the library's error word
// and every role leaves its loop.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4 {
namespace {

constexpr int kW16Tokens = 64;               // token rows: the MMA's M
constexpr int kW16BN = 192;                  // weight rows per tile
constexpr int kW16DqWarps = 12;
constexpr int kW16Threads = 32 * (kW16DqWarps + 2);
constexpr int kW16AStages = 6;               // activation slices in flight
constexpr int kW16RStages = 3;               // raw weight tiles in flight
constexpr int kW16DStages = 3;               // dequantized slices in flight
constexpr uint32_t kW16ABytes = kW16Tokens * 128;        // 64 rows x 64 BF16
constexpr uint32_t kW16DBytes = kW16BN * 128;            // 192 rows x 64 BF16
constexpr uint32_t kW16RBytes = kW16BN * 128;            // 192 rows x 256 FP4
constexpr uint32_t kW16SfBytes = 2 * 2048;               // <= 2 row blocks x 4 chunks
constexpr uint32_t kW16TmemCols = 256;
constexpr uint32_t kW16IDesc =                           // kind::f16: F32 D, BF16 A and B, K-major
    (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(kW16BN >> 3) << 17) | ((uint32_t)(kW16Tokens >> 4) << 24);
static_assert(kW16DqWarps * 32 == 2 * kW16BN, "one 32-value item per dequantizing thread per slice");

struct W16Tail {
    uint64_t a_full[kW16AStages], a_empty[kW16AStages];
    uint64_t r_full[kW16RStages], r_empty[kW16RStages];
    uint64_t d_full[kW16DStages], d_empty[kW16DStages];
    uint64_t acc_full, acc_empty;
    uint32_t tmem_base;
    int abort_flag;
};

constexpr size_t kW16Smem = 1024 + (size_t)kW16AStages * kW16ABytes + (size_t)kW16DStages * kW16DBytes +
                            (size_t)kW16RStages * (kW16RBytes + kW16SfBytes) + sizeof(W16Tail);
static_assert(kW16Smem <= 232448, "shared memory");

struct W16Args {
    const uint8_t* sfb;      // weight scales, tiled layout
    int64_t sf_rb_stride;    // bytes per 128-row scale block
    int sf_blocks;           // 128-row scale blocks of the weights
    const float* gb;         // weight global scale
    __nv_bfloat16* c;
    int64_t ldc;
    int m, n, num_ks, tiles;
    uint64_t wait_limit_ns;
    unsigned int* err;
};

__device__ __forceinline__ void w16_abort(W16Tail* t, unsigned int* err) {
    t->abort_flag = 1;
    if (err) atomicOr(err, 1u);
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}
__device__ __forceinline__ uint32_t or_byte_signs(uint32_t v, uint32_t s) {   // v | (s & 0x80808080)
    uint32_t d;
    asm("lop3.b32 %0, %1, %2, 0x80808080, 0xF8;" : "=r"(d) : "r"(v), "r"(s));
    return d;
}
__device__ __forceinline__ uint32_t mul_bf16x2(uint32_t a, uint32_t b) {
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Eight E2M1 codes (value e in bits 4e..4e+3) -> eight BF16 values times the
// BF16 pair s2, as four packed pairs.  The magnitudes come from two byte tables
// by prmt: BF16 high bytes 00 3F 3F 3F 40 40 40 40 and low bytes 00 00 80 C0
// 00 40 80 C0 for 0, 0.5, 1, 1.5, 2, 3, 4, 6.  The sign bits go into the high
// bytes before they are interleaved with the low bytes: the sign of value 2i
// is the top bit of byte i of w << 4, that of value 2i + 1 the top bit of byte
// i of w, so one prmt gathers four of them onto the top bits of a word whose
// bytes line up with a high-byte table result.  Every product is exact.
__device__ __forceinline__ void dequant8(uint32_t w, uint32_t s2, uint32_t* out) {
    constexpr uint32_t kHi0 = 0x3F3F3F00u, kHi1 = 0x40404040u, kLo0 = 0xC0800000u, kLo1 = 0xC0804000u;
    const uint32_t mag = w & 0x77777777u;
    const uint32_t mag_hi = mag >> 16;
    const uint32_t w4 = w << 4;
    const uint32_t lo_a = prmt(kLo0, kLo1, mag), lo_b = prmt(kLo0, kLo1, mag_hi);
    const uint32_t hi_a = or_byte_signs(prmt(kHi0, kHi1, mag), prmt(w4, w, 0x5140));      // values 0..3
    const uint32_t hi_b = or_byte_signs(prmt(kHi0, kHi1, mag_hi), prmt(w4, w, 0x7362));   // values 4..7
    out[0] = mul_bf16x2(prmt(lo_a, hi_a, 0x5140), s2);
    out[1] = mul_bf16x2(prmt(lo_a, hi_a, 0x7362), s2);
    out[2] = mul_bf16x2(prmt(lo_b, hi_b, 0x5140), s2);
    out[3] = mul_bf16x2(prmt(lo_b, hi_b, 0x7362), s2);
}

// Two E4M3 scale bytes (low byte first) -> FP32 values (exact).
__device__ __forceinline__ void e4m3x2_to_f32(uint32_t two, float& s0, float& s1) {
    uint32_t h2;
    const uint16_t in = (uint16_t)(two & 0xFFFFu);
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\tcvt.f32.f16 %0, lo;\n\tcvt.f32.f16 %1, hi;\n\t}"
        : "=f"(s0), "=f"(s1)
        : "r"(h2));
}
__device__ __forceinline__ uint32_t bf16x2_splat(float s) {
    uint32_t d;
    asm("cvt.rn.bf16x2.f32 %0, %1, %1;" : "=r"(d) : "f"(s));
    return d;
}

__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

__global__ void __launch_bounds__(kW16Threads, 1)
    w4a16_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmW, const W16Args p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    // layout: activation slices, dequantized slices, raw tiles, scales
    uint8_t* sA = smem;
    uint8_t* sD = sA + kW16AStages * kW16ABytes;
    uint8_t* sR = sD + kW16DStages * kW16DBytes;
    uint8_t* sSF = sR + kW16RStages * kW16RBytes;
    W16Tail* tail = reinterpret_cast<W16Tail*>(sSF + kW16RStages * kW16SfBytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t limit = p.wait_limit_ns;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kW16AStages; ++s) {
            mbar_init(&tail->a_full[s], 1);
            mbar_init(&tail->a_empty[s], 1);
        }
        for (int s = 0; s < kW16RStages; ++s) {
            mbar_init(&tail->r_full[s], 1);
            mbar_init(&tail->r_empty[s], kW16DqWarps);
        }
        for (int s = 0; s < kW16DStages; ++s) {
            mbar_init(&tail->d_full[s], kW16DqWarps);
            mbar_init(&tail->d_empty[s], 1);
        }
        mbar_init(&tail->acc_full, 1);
        mbar_init(&tail->acc_empty, 4);
        tail->abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmW);
    }
    if (warp == kW16DqWarps + 1) {
        tmem_alloc(&tail->tmem_base, kW16TmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tail->tmem_base;
    const int num_ks = p.num_ks;

    if (warp == kW16DqWarps) {
        // ---------------- TMA producer ----------------
        if (lane == 0) {
            uint32_t as = 0, aph = 0, rs = 0, rph = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < p.tiles && ok; t += gridDim.x) {
                const int n0 = t * kW16BN;
                const int blk0 = n0 / 128;
                const int nblk = min(2, p.sf_blocks - blk0);
                for (int ks = 0; ks < num_ks; ++ks) {
                    if ((ks & 3) == 0) {
                        if (!mbar_wait(&tail->r_empty[rs], rph ^ 1u, limit) || tail->abort_flag) {
                            ok = false;
                            break;
                        }
                        const int kt = ks >> 2;
                        const uint32_t nat = (uint32_t)min(4, num_ks - ks);
                        uint64_t* bar = &tail->r_full[rs];
                        mbar_arrive_expect_tx(bar, kW16RBytes + (uint32_t)nblk * nat * 512u);
                        tma_load_2d(sR + rs * kW16RBytes, &tmW, bar, kt * 128, n0);
                        for (int b = 0; b < nblk; ++b)
                            bulk_load(sSF + rs * kW16SfBytes + b * 2048,
                                      p.sfb + (int64_t)(blk0 + b) * p.sf_rb_stride + (int64_t)kt * 2048, nat * 512u,
                                      bar);
                        if (++rs == kW16RStages) {
                            rs = 0;
                            rph ^= 1u;
                        }
                    }
                    if (!mbar_wait(&tail->a_empty[as], aph ^ 1u, limit) || tail->abort_flag) {
                        ok = false;
                        break;
                    }
                    mbar_arrive_expect_tx(&tail->a_full[as], kW16ABytes);
                    tma_load_2d(sA + as * kW16ABytes, &tmA, &tail->a_full[as], ks * 64, 0);
                    if (++as == kW16AStages) {
                        as = 0;
                        aph ^= 1u;
                    }
                }
            }
            if (!ok) w16_abort(tail, p.err);
        }
    } else if (warp == kW16DqWarps + 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            uint32_t as = 0, aph = 0, ds = 0, dph = 0;
            bool ok = true;
            int it = 0;
            for (int t = blockIdx.x; t < p.tiles && ok; t += gridDim.x, ++it) {
                if (!mbar_wait(&tail->acc_empty, ((uint32_t)it & 1u) ^ 1u, limit) || tail->abort_flag) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int ks = 0; ks < num_ks; ++ks) {
                    if (!mbar_wait(&tail->a_full[as], aph, limit) || !mbar_wait(&tail->d_full[ds], dph, limit) ||
                        tail->abort_flag) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(sA + as * kW16ABytes), b0 = smem_u32(sD + ds * kW16DBytes);
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        mma_bf16(tmem, sdesc_kmajor_sw128(a0 + j * 32), sdesc_kmajor_sw128(b0 + j * 32), kW16IDesc,
                                 (ks > 0 || j > 0) ? 1u : 0u);
                    tc_commit(&tail->a_empty[as]);
                    tc_commit(&tail->d_empty[ds]);
                    if (++as == kW16AStages) {
                        as = 0;
                        aph ^= 1u;
                    }
                    if (++ds == kW16DStages) {
                        ds = 0;
                        dph ^= 1u;
                    }
                }
                if (ok) tc_commit(&tail->acc_full);
            }
            if (!ok) w16_abort(tail, p.err);
        }
    } else {
        // ---------------- dequantization (and, warps 0..3, the epilogue) ----------------
        // Item of thread i per slice: weight row r = i % 192 of the tile, values
        // 32 h .. 32 h + 31 of the 64-wide slice (h = i / 192): one 16-byte
        // chunk of the raw tile, four 16-byte units of the dequantized slice.
        const int i = threadIdx.x;
        const int h = i / kW16BN, r = i % kW16BN;
        uint32_t rs = 0, rph = 0, ds = 0, dph = 0;
        bool ok = true;
        int it = 0;
        for (int t = blockIdx.x; t < p.tiles && ok; t += gridDim.x, ++it) {
            const int n0 = t * kW16BN;
            const int g = n0 % 128 + r;                       // row inside the tile's first scale block
            const bool row_ok = n0 + r < p.n;
            const uint32_t sf_off = (uint32_t)((g >> 7) * 2048 + (g & 31) * 16 + ((g >> 5) & 3) * 4);
            for (int ks = 0; ks < num_ks; ++ks) {
                const int j = ks & 3;
                if (j == 0 && (!mbar_wait(&tail->r_full[rs], rph, limit) || tail->abort_flag)) {
                    ok = false;
                    break;
                }
                if (!mbar_wait(&tail->d_empty[ds], dph ^ 1u, limit) || tail->abort_flag) {
                    ok = false;
                    break;
                }
                const uint32_t raw = smem_u32(sR + rs * kW16RBytes);
                const int chunk = 2 * j + h;                  // 16-byte chunk of the raw row (128-byte swizzle)
                const uint4 q = ld_shared_v4(raw + (uint32_t)(r * 128 + ((chunk ^ (r & 7)) << 4)));
                uint32_t sw;
                asm volatile("ld.shared.b32 %0, [%1];"
                             : "=r"(sw)
                             : "r"(smem_u32(sSF + rs * kW16SfBytes) + sf_off + (uint32_t)j * 512u));
                float s0, s1;
                e4m3x2_to_f32(row_ok ? (sw >> (16 * h)) : 0u, s0, s1);
                const uint32_t s0x2 = bf16x2_splat(s0), s1x2 = bf16x2_splat(s1);
                uint32_t o[16];
                dequant8(q.x, s0x2, o);
                dequant8(q.y, s0x2, o + 4);
                dequant8(q.z, s1x2, o + 8);
                dequant8(q.w, s1x2, o + 12);
                const uint32_t dst = smem_u32(sD + ds * kW16DBytes) + (uint32_t)((r >> 3) * 1024 + (r & 7) * 128);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int unit = 4 * h + u;               // 16-byte unit of the BF16 row (128-byte swizzle)
                    st_shared_v4(dst + (uint32_t)((unit ^ (r & 7)) << 4),
                                 make_uint4(o[4 * u], o[4 * u + 1], o[4 * u + 2], o[4 * u + 3]));
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&tail->d_full[ds]);
                    if (j == 3 || ks == num_ks - 1) mbar_arrive(&tail->r_empty[rs]);
                }
                if (j == 3 || ks == num_ks - 1) {
                    if (++rs == kW16RStages) {
                        rs = 0;
                        rph ^= 1u;
                    }
                }
                if (++ds == kW16DStages) {
                    ds = 0;
                    dph ^= 1u;
                }
            }
            if (warp < 4 && ok) {
                // epilogue: lanes 32 warp .. 32 warp + 15 hold token rows 16 warp ..
                if (!mbar_wait(&tail->acc_full, (uint32_t)it & 1u, limit) || tail->abort_flag) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const int tok = lane < 16 ? warp * 16 + lane : p.m;   // lanes 16..31: no row
                const float gw = p.gb[0];
                const int ncols = min(kW16BN, p.n - n0);
                const uint32_t tq = tmem + ((uint32_t)(warp * 32) << 16);
#pragma unroll 1
                for (int ch = 0; ch < kW16BN / 32; ++ch) {
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tq + ch * 32, v);
                    tmem_ld_wait();
                    if (tok >= p.m || ch * 32 >= ncols) continue;
                    __nv_bfloat16* crow = p.c + (int64_t)tok * p.ldc + n0 + ch * 32;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int c0 = ch * 32 + 8 * u;
                        uint32_t w[4];
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(v[8 * u + 2 * e]) * gw,
                                                                      __uint_as_float(v[8 * u + 2 * e + 1]) * gw);
                            w[e] = *reinterpret_cast<uint32_t*>(&b2);
                        }
                        if (c0 + 8 <= ncols) {
                            st_global_v4(crow + 8 * u, w[0], w[1], w[2], w[3]);
                        } else {
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                if (c0 + e < ncols)
                                    crow[8 * u + e] = __float2bfloat16_rn(__uint_as_float(v[8 * u + e]) * gw);
                        }
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tail->acc_empty);
            }
        }
        if (!ok && lane == 0) w16_abort(tail, p.err);
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kW16DqWarps + 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kW16TmemCols);
    }
}

bool make_map_2d(CUtensorMap* map, CUtensorMapDataType dtype, const void* base, int64_t inner, int64_t rows,
                 int64_t row_bytes, uint32_t box_inner, uint32_t box_rows) {
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {box_inner, box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    return fn(map, dtype, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace
}  // namespace nvfp4

using namespace nvfp4;

extern "C" nvfp4_status_t w4a16_gemm(const void* a, int64_t lda, const uint8_t* b_codes, const uint8_t* b_scales,
                                     const float* b_global, void* c, int64_t ldc, int64_t m, int64_t n, int64_t k,
                                     void* stream) {
    if (m < 0 || n <= 0 || k <= 0 || lda < k || ldc < n) return NVFP4_ERR_INVALID_ARGUMENT;
    if (m > kW16Tokens || k % 64 != 0 || n >= ((int64_t)1 << 31) || k >= ((int64_t)1 << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (m == 0) return NVFP4_OK;   // nothing to read or write (the pointers may be NULL)
    if (!a || !b_codes || !b_scales || !b_global || !c) return NVFP4_ERR_INVALID_ARGUMENT;
    if (!aligned16(a) || !aligned16(b_codes) || !aligned16(b_scales) || !aligned16(c) || lda % 8 != 0 ||
        ldc % 8 != 0 || (reinterpret_cast<uintptr_t>(b_global) & 3u))
        return NVFP4_ERR_MISALIGNED;
    const int sms = num_sms();
    if (sms <= 0) return NVFP4_ERR_NO_DEVICE;
    CUtensorMap ta, tw;
    if (!make_map_2d(&ta, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a, k, m, lda * 2, 64u, (uint32_t)kW16Tokens) ||
        !make_map_2d(&tw, CU_TENSOR_MAP_DATA_TYPE_UINT8, b_codes, k / 2, n, k / 2, 128u, (uint32_t)kW16BN))
        return NVFP4_ERR_CUDA;
    W16Args p;
    p.sfb = b_scales;
    p.sf_rb_stride = 128 * (k / 16);
    p.sf_blocks = (int)((n + 127) / 128);
    p.gb = b_global;
    p.c = reinterpret_cast<__nv_bfloat16*>(c);
    p.ldc = ldc;
    p.m = (int)m;
    p.n = (int)n;
    p.num_ks = (int)(k / 64);
    p.tiles = (int)((n + kW16BN - 1) / kW16BN);
    p.wait_limit_ns = wait_limit_ns();
    p.err = device_error_word();
    if (!p.err) return NVFP4_ERR_CUDA;
    static std::atomic<unsigned long long> attr_done{0};
    if (!smem_attr_on_device(reinterpret_cast<const void*>(&w4a16_kernel), (int)kW16Smem, attr_done))
        return NVFP4_ERR_CUDA;
    const int grid = std::min(p.tiles, sms);
    w4a16_kernel<<<grid, kW16Threads, kW16Smem, reinterpret_cast<cudaStream_t>(stream)>>>(ta, tw, p);
    return cuda_status(cudaGetLastError());
}
