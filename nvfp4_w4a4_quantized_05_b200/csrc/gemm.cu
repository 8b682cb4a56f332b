// gemm.cu -- stage 2 of the W4A4 path: block-scaled FP4 x FP4 GEMM on the
// sm_100a tcgen05 tensor cores.
//
//   C[m, n] = bf16_rn( (sum_k qa[m,k] sa[m,k/16] qb[n,k] sb[n,k/16]) * ga * gb )
//
// i.e. the product of the two reconstructed NVFP4 operands ("NVFP4 Explained:
// NVIDIA's 4-Bit Format for Faster AI Inference", "How NVFP4 Represents a
// Value"): the E2M1 codes and their E4M3 block scales go to the tensor core
// unchanged (tcgen05.mma .kind::mxf4nvf4, 16-element scale blocks), FP32
// accumulation stays in tensor memory, and the two FP32 tensor scales are
// applied once in the epilogue.  No dequantization pass: on Blackwell FP4 x FP4
// is a native tensor-core mode ("NVFP4 Dynamic Quantization in Practice",
// "Impact on the Open-Source Community and LLM Deployment Industry"; "W4A8 vs
// NVFP4 quantization on GPUs", "Dequantization can erase a four-bit win").
//
// Kernel structure (one CTA per SM, persistent over output tiles, 10 warps):
//   warp 0     TMA producer: codes tiles by tensor-map copies (128-byte
//              swizzle), scale tiles by bulk copies, into a STAGES-deep ring
//              guarded by mbarriers.  No cluster multicast.
//   warp 1     allocates tensor memory; one thread issues the MMAs (128 x BN
//              x 64 each) and commits to the stage's "empty" barrier, the
//              scale buffer's "free" barrier and, per tile, the accumulator
//              buffer's "full" barrier.
//   warps 2-5  epilogue: tcgen05.ld of the FP32 accumulator, x (ga * gb),
//              round to BF16, store.  Two accumulator buffers in tensor
//              memory, so the epilogue of one tile overlaps the next tile's
//              mainloop (when 2 x BN columns and the scale buffers fit).
//   warps 6-9  scale staging: each warp owns one 32-lane quarter of tensor
//              memory and writes the stage's scale tiles there with
//              tcgen05.st, in the replicated layout the block-scaled MMA
//              reads (lane i, column c of a 128-row block's k-step holds the
//              four scales of row i + 32c).  Moving scales with tcgen05.cp
//              would put ~100 cycles per copy on the tensor pipe, in series
//              with the MMAs (12 copies per 128x256x256 k-tile); tcgen05.st
//              from the otherwise idle warps keeps the tensor pipe for MMAs.
// Every mbarrier wait is bounded (globaltimer); a wait that runs out sets the
// library's device error word and the CTA winds down instead of hanging.
//
// Operand roles: the "A side" (activations) fills the 128-row MMA dimension,
// the "B side" (weights) the BN-wide dimension.  For m > 128 the 2-SM pair
// kernel below takes over (256 x 256 tiles, persistent over tiles, with a
// stream-K share-out of the last waves' k-tiles so that all pairs finish
// together).  The grouped form walks (expert, m-tile, n-tile) triples built
// from the device offsets array.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>
#include <type_traits>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4 {
namespace {

constexpr int kThreads = 320;         // 10 warps, roles above
constexpr uint32_t kTmemCols = 512;
constexpr int kMaxStages = 8;
constexpr int kMaxScaleBufs = 8;
constexpr int kMaxGroups = 256;

struct GemmArgs {
    const uint8_t* sfa;        // A-side scales, tiled layout
    int64_t sfa_rb_stride;     // bytes per 128-row scale block
    const uint8_t* sfb;        // B-side scales
    int64_t sfb_rb_stride;
    int64_t sfb_group_stride;  // bytes between groups' B scales (grouped)
    int sfb_rb_per_group;      // 128-row scale blocks per B group
    const float* ga;           // global scales (index = group)
    const float* gb;
    __nv_bfloat16* c;
    int64_t ldc;
    int rows_a;                // A-side rows (plain) / total rows (grouped)
    int rows_b;                // B-side rows per group
    int num_ks;                // k / 64
    int num_kt;                // ceil(num_ks / 4): k-tiles of 256 elements
    int tiles_m;               // plain: ceil(rows_a / 128)
    int tiles_n;               // ceil(rows_b / BN)
    const int32_t* offsets;    // grouped: [num_groups + 1]
    int num_groups;
    uint64_t wait_limit_ns;
    unsigned int* err;
    // pair kernel, stream-K tail (see PairWork): tiles [0, dp_tiles) are whole;
    // the k-tiles of the rest are shared out evenly
    int dp_tiles;
    int64_t sk_units;
    float* partial;            // per CTA of each pair: FP32 [BN / 4][128] x 4 partial sums
    uint32_t* sk_flags;        // per CTA of each pair: a ready counter, kSkFlagStride words apart
    // optional: the amax of the BF16 output, as the next quantizer's global scale
    uint32_t* c_amax;          // [0] running max |C| (BF16 bits), [1] CTAs done; both 0 between calls
    float* c_gscale;           // receives amax(C) / 2688 (1 when amax is 0)
    // single-SM kernel, plain form: B (codes and scales) was not written by the
    // kernel this one depends on, so the producer may load the first stages'
    // B tiles before griddepcontrol.wait (the weight stream starts while the
    // activations are still being quantized)
    int b_early;
    // 1: let the next kernel on the stream launch at this grid's start (its
    // CTAs take SMs as these leave; it waits for this grid before reading
    // what this one writes).  Off for decode-size and grouped shapes, whose
    // steps measured slower with it.
    int pdl_trigger;
};

// The largest |value| of packed BF16 pairs, as a 16-bit pattern.
__device__ __forceinline__ uint32_t bf16x2_abs_bits(uint32_t packed) {
    const uint32_t m = packed & 0x7FFF7FFFu;
    return max(m & 0xFFFFu, m >> 16);
}
// An epilogue warp's running output maximum (packed), folded into the call's word.
__device__ __forceinline__ void fold_c_amax(const GemmArgs& p, uint32_t cam) {
    uint32_t m = bf16x2_abs_bits(cam);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0 && m != 0u) atomicMax(&p.c_amax[0], m);
}
// Thread 0 of every CTA, after all its epilogue warps have folded: the last
// CTA turns the maximum into the global scale and returns both words to zero.
__device__ __forceinline__ void finish_c_amax(const GemmArgs& p) {
    __threadfence();
    if (atomicAdd(&p.c_amax[1], 1u) == gridDim.x - 1) {
        __threadfence();
        const float amax = __uint_as_float(atomicExch(&p.c_amax[0], 0u) << 16);
        p.c_gscale[0] = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, 2688.0f);   // 6 x 448, as the quantizer
        atomicExch(&p.c_amax[1], 0u);
    }
}

struct alignas(8) SmemTail {
    uint64_t full[kMaxStages];
    uint64_t empty[kMaxStages];
    uint64_t acc_full[2];
    uint64_t acc_empty[2];
    uint64_t sf_full[kMaxScaleBufs];
    uint64_t sf_empty[kMaxScaleBufs];
    uint32_t tmem_base;
    volatile int abort_flag;
    int total_tiles;
    int pad_;
    int tile_prefix[kMaxGroups + 1];
    int blk_prefix[kMaxGroups + 1];
};

struct TileInfo {
    int a_row0;   // tensor-map row of the first A-side row
    int a_rows;   // valid A-side rows in this tile
    int sfa_rb;   // A-side 128-row scale block
    int b_row0;   // tensor-map row of the first B-side row
    int b_col0;   // index of the first B-side row inside its group
    int b_rows;   // valid B-side rows
    int group;
};

template <int BN, bool GROUPED>
__device__ __forceinline__ TileInfo tile_info(const GemmArgs& p, const SmemTail* tail, int t) {
    TileInfo ti;
    if constexpr (!GROUPED) {
        const int tm = t % p.tiles_m, tn = t / p.tiles_m;
        ti.a_row0 = tm * 128;
        ti.a_rows = min(128, p.rows_a - ti.a_row0);
        ti.sfa_rb = tm;
        ti.b_col0 = tn * BN;
        ti.b_row0 = ti.b_col0;
        ti.b_rows = min(BN, p.rows_b - ti.b_col0);
        ti.group = 0;
    } else {
        int lo = 0, hi = p.num_groups;   // largest e with tile_prefix[e] <= t
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (tail->tile_prefix[mid] <= t) lo = mid; else hi = mid;
        }
        const int e = lo;
        const int r0 = p.offsets[e], n_e = p.offsets[e + 1] - r0;
        const int mt = (n_e + 127) / 128;
        const int local = t - tail->tile_prefix[e];
        const int tm = local % mt, tn = local / mt;
        ti.a_row0 = r0 + tm * 128;
        ti.a_rows = min(128, n_e - tm * 128);
        ti.sfa_rb = tail->blk_prefix[e] + tm;
        ti.b_col0 = tn * BN;
        ti.b_row0 = e * p.rows_b + ti.b_col0;
        ti.b_rows = min(BN, p.rows_b - ti.b_col0);
        ti.group = e;
    }
    return ti;
}

__device__ __forceinline__ void raise_abort(SmemTail* tail, unsigned int* err) {
    tail->abort_flag = 1;
    if (err) atomicOr(err, 1u);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
}

// Compile-time shape of one kernel configuration.
template <int BN_, int STAGES_, int ACC_, int NSB_ = 2, int AROWS_ = 128>
struct Cfg {
    static constexpr int AROWS = AROWS_;                      // A rows loaded per stage (the MMA reads 128)
    static constexpr int BN = BN_;
    static constexpr int STAGES = STAGES_;
    static constexpr int ACC = ACC_;                          // accumulator buffers in tensor memory
    static constexpr int NSB = NSB_;                          // scale buffers in tensor memory
    // 128-row scale blocks a B tile can touch: tiles start at multiples of BN,
    // i.e. at a row offset 0 or 64 inside a block for BN = 192.
    static constexpr int NSFB = BN == 192 ? 2 : (BN + 127) / 128;
    static constexpr uint32_t A_BYTES = AROWS * 128;          // AROWS rows x 256 FP4
    static constexpr uint32_t B_BYTES = BN * 128;
    static constexpr uint32_t SFA_BYTES = 4 * 512;            // 4 k-steps x (128 rows x 4 scales)
    static constexpr uint32_t SFB_BYTES = NSFB * 4 * 512;
    static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr uint32_t SF_COLS = 16 + 16 * NSFB;       // tensor-memory columns per k-tile of scales
    static constexpr uint32_t SF_STRIDE = (SF_COLS + 31) / 32 * 32;   // buffers start 32-column aligned
    static constexpr uint32_t SF_BASE = ACC * BN;             // first scale column
    // epilogue staging: per epilogue warp two 32-row x 64-byte BF16 boxes
    static constexpr uint32_t EPI_BYTES = 4 * 2 * 2048;
    static constexpr size_t SMEM = 1024 + (size_t)STAGES * STAGE_BYTES + EPI_BYTES + sizeof(SmemTail);
    static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "BN");
    static_assert(STAGES <= kMaxStages, "stages");
    static_assert(ACC == 1 || ACC == 2, "accumulator buffers");
    static_assert(NSB >= 2 && NSB <= kMaxScaleBufs, "scale buffers");
    static_assert(SF_BASE + NSB * SF_STRIDE <= kTmemCols, "tensor memory budget");
    static_assert(SF_BASE % 32 == 0, "wide tensor-memory stores start at a multiple of their width");
    static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
    static_assert(SMEM <= 232448, "shared memory");
    static_assert(SF_COLS == 32 || SF_COLS == 48, "scale staging writes 32 (+16) columns per k-tile");
};

// EMIT (plain form only): also fold max |C| and write C's global scale.
// MX (plain form only): MXFP4 operands -- one UE8M0 scale per 32 elements, so a
// k-tile of 256 holds two 512-byte scale chunks per 128-row block instead of
// four, k-step j reads chunk j / 2 at byte pair 2 (j % 2), and there is no
// global scale (C = bf16(acc)).
template <class C, bool GROUPED, bool EMIT = false, bool MX = false>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmC, const GemmArgs p) {
    constexpr int BN = C::BN, STAGES = C::STAGES, ACC = C::ACC, NSFB = C::NSFB;
    constexpr int CW = BN >= 32 ? 32 : 16;                   // epilogue column chunk
    constexpr uint32_t IDESC = idesc_mxf4nvf4(128, BN);
    constexpr uint32_t IDESC_MX0 = idesc_mxf4_e8m0(128, BN, 0), IDESC_MX2 = idesc_mxf4_e8m0(128, BN, 2);
    constexpr int SF_KT = MX ? 1024 : 2048;      // scale bytes of one k-tile per 128-row block
    constexpr int NCH = MX ? 2 : 4;              // 512-byte scale chunks per k-tile
    static_assert(!(MX && (GROUPED || EMIT)), "MXFP4: plain form only");

    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* epi_smem = smem + STAGES * C::STAGE_BYTES;
    SmemTail* tail = reinterpret_cast<SmemTail*>(epi_smem + C::EPI_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint64_t limit = p.wait_limit_ns;
    if (p.pdl_trigger) pdl_launch_dependents();

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&tail->full[s], 1);
            mbar_init(&tail->empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&tail->acc_full[b], 1);
            mbar_init(&tail->acc_empty[b], 4);
        }
        for (int b = 0; b < C::NSB; ++b) {
            mbar_init(&tail->sf_full[b], 4);
            mbar_init(&tail->sf_empty[b], 1);
        }
        tail->abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmC);
    }
    // b_early: thread 0 (the producer) sends the B half -- codes and scales --
    // of its first tile's first `pre` stages (the ring is fresh: stage kt)
    // before any wait, so that the weights stream while the kernel this one
    // depends on is still running; the A half follows in the producer loop.
    const bool b_early = !GROUPED && p.b_early != 0;
    int pre = 0;
    auto b_half = [&](const TileInfo& ti, int kt, uint64_t* bar, uint8_t* sB, uint8_t* sSFB, uint32_t nch, int nsfb) {
        const uint8_t* sfb_src =
            p.sfb + (int64_t)ti.group * p.sfb_group_stride + (int64_t)(ti.b_col0 / 128) * p.sfb_rb_stride;
        tma_load_2d(sB, &tmB, bar, kt * 128, ti.b_row0);
        for (int rb = 0; rb < nsfb; ++rb)
            bulk_load(sSFB + rb * 2048, sfb_src + (int64_t)rb * p.sfb_rb_stride + (int64_t)kt * SF_KT, nch * 512u,
                      bar);
    };
    const bool first_tile = !GROUPED && threadIdx.x == 0 && (int)blockIdx.x < p.tiles_m * p.tiles_n;
    if (b_early && first_tile) {
        const TileInfo ti = tile_info<BN, GROUPED>(p, tail, blockIdx.x);
        const int nsfb = min(NSFB, p.sfb_rb_per_group - ti.b_col0 / 128);
        pre = min(STAGES, p.num_kt);
        for (int kt = 0; kt < pre; ++kt) {
            const int nat = min(4, p.num_ks - kt * 4);
            const uint32_t nch = MX ? (uint32_t)(nat + 1) / 2 : (uint32_t)nat;
            uint8_t* sA = smem + kt * C::STAGE_BYTES;
            uint8_t* sSFA = sA + C::A_BYTES + C::B_BYTES;
            uint64_t* bar = &tail->full[kt];
            mbar_arrive_expect_tx(bar, C::A_BYTES + C::B_BYTES + nch * 512u * (1u + (uint32_t)nsfb));
            b_half(ti, kt, bar, sA + C::A_BYTES, sSFA + C::SFA_BYTES, nch, nsfb);
        }
    }
    if (warp == 1) {
        tmem_alloc(&tail->tmem_base, kTmemCols);
        tmem_relinquish();
    }
    // Everything read below (codes, scales, global scales, offsets) may be
    // written by the previous kernel in the stream.
    pdl_wait();
    if constexpr (GROUPED) {
        if (warp == 2) {
            const int E = p.num_groups;
            const int per = (E + 31) / 32;
            int t_loc = 0, b_loc = 0;
            for (int i = 0; i < per; ++i) {
                const int e = lane * per + i;
                if (e < E) {
                    const int mt = (p.offsets[e + 1] - p.offsets[e] + 127) / 128;
                    t_loc += mt * p.tiles_n;
                    b_loc += mt;
                }
            }
            int t_inc = t_loc, b_inc = b_loc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int tv = __shfl_up_sync(0xFFFFFFFFu, t_inc, o);
                const int bv = __shfl_up_sync(0xFFFFFFFFu, b_inc, o);
                if (lane >= o) {
                    t_inc += tv;
                    b_inc += bv;
                }
            }
            int t_run = t_inc - t_loc, b_run = b_inc - b_loc;
            for (int i = 0; i < per; ++i) {
                const int e = lane * per + i;
                if (e < E) {
                    tail->tile_prefix[e] = t_run;
                    tail->blk_prefix[e] = b_run;
                    const int mt = (p.offsets[e + 1] - p.offsets[e] + 127) / 128;
                    t_run += mt * p.tiles_n;
                    b_run += mt;
                }
            }
            if (lane == 31) {
                tail->tile_prefix[E] = t_inc;
                tail->blk_prefix[E] = b_inc;
                tail->total_tiles = t_inc;
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tail->tmem_base;
    const int total_tiles = GROUPED ? tail->total_tiles : p.tiles_m * p.tiles_n;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
                const TileInfo ti = tile_info<BN, GROUPED>(p, tail, t);
                const uint8_t* sfa_src = p.sfa + (int64_t)ti.sfa_rb * p.sfa_rb_stride;
                const int nsfb = min(NSFB, p.sfb_rb_per_group - ti.b_col0 / 128);
                for (int kt = 0; kt < p.num_kt; ++kt) {
                    if (!mbar_wait(&tail->empty[stage], phase ^ 1u, limit) || tail->abort_flag) {
                        ok = false;
                        break;
                    }
                    const int nat = min(4, p.num_ks - kt * 4);
                    const uint32_t nch = MX ? (uint32_t)(nat + 1) / 2 : (uint32_t)nat;   // scale chunks used
                    uint8_t* sA = smem + stage * C::STAGE_BYTES;
                    uint8_t* sB = sA + C::A_BYTES;
                    uint8_t* sSFA = sB + C::B_BYTES;
                    uint8_t* sSFB = sSFA + C::SFA_BYTES;
                    uint64_t* bar = &tail->full[stage];
                    const bool b_done = t == (int)blockIdx.x && kt < pre;   // B half already issued
                    if (!b_done) {
                        mbar_arrive_expect_tx(bar, C::A_BYTES + C::B_BYTES + nch * 512u * (1u + (uint32_t)nsfb));
                        b_half(ti, kt, bar, sB, sSFB, nch, nsfb);
                    }
                    tma_load_2d(sA, &tmA, bar, kt * 128, ti.a_row0);
                    bulk_load(sSFA, sfa_src + (int64_t)kt * SF_KT, nch * 512u, bar);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) raise_abort(tail, p.err);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            uint32_t stage = 0, phase = 0, ktg = 0;
            int it = 0;
            bool ok = true;
            for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x, ++it) {
                const TileInfo ti = tile_info<BN, GROUPED>(p, tail, t);
                const uint32_t ab = ACC == 2 ? (uint32_t)(it & 1) : 0u;
                const uint32_t au = ACC == 2 ? (uint32_t)(it >> 1) : (uint32_t)it;
                if (!mbar_wait(&tail->acc_empty[ab], (au & 1u) ^ 1u, limit) || tail->abort_flag) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + ab * BN;
                const uint32_t sfb_off = 16 + (uint32_t)((ti.b_col0 % 128) / 32);
                for (int kt = 0; kt < p.num_kt; ++kt, ++ktg) {
                    const uint32_t sb = ktg % C::NSB, su = ktg / C::NSB;
                    if (!mbar_wait(&tail->full[stage], phase, limit) ||
                        !mbar_wait(&tail->sf_full[sb], su & 1u, limit) || tail->abort_flag) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nat = min(4, p.num_ks - kt * 4);
                    const uint32_t sA = smem_u32(smem + stage * C::STAGE_BYTES);
                    const uint32_t sB = sA + C::A_BYTES;
                    const uint32_t sf = tmem + C::SF_BASE + sb * C::SF_STRIDE;
                    for (int j = 0; j < nat; ++j) {
                        if constexpr (MX)
                            mma_mxf4nvf4<true>(d_tmem, sdesc_kmajor_sw128(sA + j * 32), sdesc_kmajor_sw128(sB + j * 32),
                                               (j & 1) ? IDESC_MX2 : IDESC_MX0, sf + (j >> 1) * 4, sf + sfb_off + (j >> 1) * 4 * NSFB,
                                               (kt > 0 || j > 0) ? 1u : 0u);
                        else
                            mma_mxf4nvf4(d_tmem, sdesc_kmajor_sw128(sA + j * 32), sdesc_kmajor_sw128(sB + j * 32),
                                         IDESC, sf + j * 4, sf + sfb_off + j * 4 * NSFB, (kt > 0 || j > 0) ? 1u : 0u);
                    }
                    tc_commit(&tail->empty[stage]);
                    tc_commit(&tail->sf_empty[sb]);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
                if (ok) tc_commit(&tail->acc_full[ab]);
            }
            if (!ok) raise_abort(tail, p.err);
        }
    } else if (warp >= 6) {
        // ---------------- scale staging (warps 6..9, one lane quarter each) ----------------
        const int q = warp & 3;
        const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16) + C::SF_BASE;
        uint32_t stage = 0, phase = 0, ktg = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < total_tiles && ok; t += gridDim.x) {
            for (int kt = 0; kt < p.num_kt; ++kt, ++ktg) {
                const uint32_t sb = ktg % C::NSB, su = ktg / C::NSB;
                // read the stage's scale words first, then wait for the buffer
                if (!mbar_wait(&tail->full[stage], phase, limit) || tail->abort_flag) {
                    ok = false;
                    break;
                }
                const uint32_t sSFA = smem_u32(smem + stage * C::STAGE_BYTES) + C::A_BYTES + C::B_BYTES;
                const uint32_t sSFB = sSFA + C::SFA_BYTES;
                // one k-tile of scales in tensor-memory column order: A k-step j at 4j,
                // B k-step j, 128-row block rb at 16 + 4 * NSFB * j + 4 * rb
                uint32_t w[C::SF_COLS];
                if constexpr (MX) {   // chunks 2 and 3 are unused
#pragma unroll
                    for (int i = 0; i < (int)C::SF_COLS; ++i) w[i] = 0u;
                }
#pragma unroll
                for (int j = 0; j < NCH; ++j) {
                    const uint4 v = ld_shared_v4(sSFA + j * 512 + lane * 16);
                    w[4 * j + 0] = v.x;
                    w[4 * j + 1] = v.y;
                    w[4 * j + 2] = v.z;
                    w[4 * j + 3] = v.w;
                }
#pragma unroll
                for (int j = 0; j < NCH; ++j)
#pragma unroll
                    for (int rb = 0; rb < NSFB; ++rb) {
                        const uint4 v = ld_shared_v4(sSFB + rb * 2048 + j * 512 + lane * 16);
                        w[16 + 4 * NSFB * j + 4 * rb + 0] = v.x;
                        w[16 + 4 * NSFB * j + 4 * rb + 1] = v.y;
                        w[16 + 4 * NSFB * j + 4 * rb + 2] = v.z;
                        w[16 + 4 * NSFB * j + 4 * rb + 3] = v.w;
                    }
                if (!mbar_wait(&tail->sf_empty[sb], (su & 1u) ^ 1u, limit) || tail->abort_flag) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t dst = tq + sb * C::SF_STRIDE;
                tmem_st_32x32b_x32(dst, w);
                if constexpr (C::SF_COLS == 48) tmem_st_32x32b_x16(dst + 32, w + 32);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tail->sf_full[sb]);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) raise_abort(tail, p.err);
    } else {
        // ---------------- epilogue (warps 2..5) ----------------
        // Each warp converts its 32 rows x 32 columns of FP32 accumulator to
        // BF16 in a swizzled 2 KB shared-memory box (two boxes per warp,
        // alternating) and writes it with a TMA tensor store; the tensor bounds
        // clip ragged tiles.  The last slab of an expert's rows in the grouped
        // form (rows past the group belong to the next expert) uses direct
        // stores.
        const int q = warp & 3;                       // tensor-memory lane quarter of this warp
        const int rloc = q * 32 + lane;               // A-side row inside the tile
        const uint32_t stg = smem_u32(epi_smem) + (uint32_t)(warp - 2) * 4096u;
        uint32_t cam = 0;                             // running max |C| of this lane's rows (packed)
        int it = 0;
        for (int t = blockIdx.x; t < total_tiles; t += gridDim.x, ++it) {
            const TileInfo ti = tile_info<BN, GROUPED>(p, tail, t);
            const uint32_t ab = ACC == 2 ? (uint32_t)(it & 1) : 0u;
            const uint32_t au = ACC == 2 ? (uint32_t)(it >> 1) : (uint32_t)it;
            if (!mbar_wait(&tail->acc_full[ab], au & 1u, limit) || tail->abort_flag) {
                if (lane == 0) raise_abort(tail, p.err);
                break;
            }
            tc_fence_after();
            const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16) + ab * BN;
            const float alpha = MX ? 1.0f : __fmul_rn(p.ga[ti.group], p.gb[ti.group]);
            const bool a_ok = rloc < ti.a_rows;
            const bool use_tma = !GROUPED || q * 32 + 32 <= ti.a_rows;
#pragma unroll 1
            for (int ch = 0; ch < BN / CW; ++ch) {
                uint32_t v[CW];
                if constexpr (CW == 32) {
                    tmem_ld_32x32b_x32(tq + ch * CW, v);
                } else {
                    tmem_ld_32x32b_x16(tq + ch * CW, v);
                }
                tmem_ld_wait();
                if (ch * CW >= ti.b_rows) continue;      // uniform: whole chunk past n
                if (use_tma) {
                    const uint32_t box = stg + (uint32_t)(ch & 1) * 2048u;
                    if (lane == 0) bulk_wait_group_read<1>();   // the box's previous store has read it
                    __syncwarp();
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(v[8 * j + 0]) * alpha, __uint_as_float(v[8 * j + 1]) * alpha);
                        w.y = pack_bf16x2(__uint_as_float(v[8 * j + 2]) * alpha, __uint_as_float(v[8 * j + 3]) * alpha);
                        w.z = pack_bf16x2(__uint_as_float(v[8 * j + 4]) * alpha, __uint_as_float(v[8 * j + 5]) * alpha);
                        w.w = pack_bf16x2(__uint_as_float(v[8 * j + 6]) * alpha, __uint_as_float(v[8 * j + 7]) * alpha);
                        if (EMIT && a_ok)
                            cam = max_abs_bf16x2(max_abs_bf16x2(cam, max_abs_bf16x2(w.x, w.y)), max_abs_bf16x2(w.z, w.w));
                        // 64-byte swizzle: 16-byte chunk j of row r sits at chunk j ^ ((r >> 1) & 3)
                        st_shared_v4(box + (uint32_t)lane * 64u + (uint32_t)((j ^ ((lane >> 1) & 3)) * 16), w);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&tmC, box, ti.b_col0 + ch * CW, ti.a_row0 + q * 32);
                        bulk_commit_group();
                    }
                } else if (a_ok) {
                    __nv_bfloat16* crow = p.c + (int64_t)(ti.a_row0 + rloc) * p.ldc + ti.b_col0 + ch * CW;
                    const int ncols = ti.b_rows - ch * CW;
#pragma unroll
                    for (int i = 0; i < CW; ++i)
                        if (i < ncols) crow[i] = __float2bfloat16_rn(__uint_as_float(v[i]) * alpha);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tail->acc_empty[ab]);
        }
        if (EMIT) fold_c_amax(p, cam);
        if (lane == 0) bulk_wait_group_all();   // stores done before the CTA's shared memory goes away
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (EMIT && threadIdx.x == 0) finish_c_amax(p);
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---- pair kernel: 2-SM tcgen05 MMA (M = 256 over a CTA pair) ------------------------
//
// A cluster of two CTAs on two SMs computes a 256 x BN output tile: CTA r loads
// A rows [128r, 128r + 128) and B rows [r * BN/2, (r + 1) * BN/2) of the tile
// (so per SM the operand traffic per MMA is lower than for a single-CTA
// 128 x BN tile), the leader (rank 0) issues tcgen05.mma.cta_group::2, and
// each CTA ends up with its 128 rows x BN columns of FP32 accumulator in its
// own tensor memory.  Both CTAs' operand loads complete on the leader's "full"
// barrier; the leader's MMA commits arrive on both CTAs' barriers.  Each CTA
// stages, at the same tensor-memory address as its peer, the scale factors of
// its own 128 A rows and of all BN columns of B (the B codes are split over
// the pair, but each SM's MMA datapath reads every column's B scales from its
// own tensor memory).  Warps: 0 producer, 1 MMA (leader), 2-9 epilogue (two
// per tensor-memory lane quarter), 10-13 scale staging.  Tensor memory per CTA
// (256 x 256 tiles): one 256-column accumulator and four packed scale buffers
// of 48 columns (16 for A, 8 per k-step for B).
template <int BN_, int STAGES_, int NSB_, int ACC_, int EPI_WARPS_ = 8>
struct PairCfg {
    static constexpr int BN = BN_;                    // pair tile width
    static constexpr int BH = BN / 2;                 // B rows loaded per CTA
    static constexpr int STAGES = STAGES_;
    static constexpr int NSB = NSB_;                  // scale buffers in tensor memory
    static constexpr int ACC = ACC_;                  // accumulator buffers in tensor memory
    static constexpr int NBC = BN / 32;               // B scale columns per k-step (all BN columns)
    static constexpr uint32_t A_BYTES = 128 * 128;
    static constexpr uint32_t B_BYTES = BH * 128;
    static constexpr uint32_t SFA_BYTES = 4 * 512;
    static constexpr uint32_t SFB_BYTES = 2 * 4 * 512;    // BN rows starting at 0 or 64 in a block: <= 2 blocks
    static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr uint32_t SF_COLS = 16 + 4 * NBC;
    static constexpr uint32_t SF_STRIDE = SF_COLS;     // packed buffers, written with 8-column stores
    static constexpr uint32_t SF_BASE = ACC * BN;      // accumulator buffers first
    static constexpr int EPI_WARPS = EPI_WARPS_;      // 8 or 16: two or four per tensor-memory lane quarter
    static constexpr int THREADS = 32 * (2 + EPI_WARPS + 4);   // producer, MMA, epilogue, scale staging
    static constexpr int EPI_COLS = BN * 4 / EPI_WARPS;         // accumulator columns one epilogue warp drains
    static constexpr int EPI_CP = EPI_COLS / 64;                // ... in 64-column reads
    static constexpr int EPI_BOXES = EPI_WARPS == 8 ? 2 : 1;     // 2 KB output staging boxes per epilogue warp
    static constexpr uint32_t EPI_BYTES = EPI_WARPS * EPI_BOXES * 2048;
    static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
    static_assert(SF_BASE + NSB * SF_STRIDE <= kTmemCols, "tensor memory budget");
    static_assert(EPI_WARPS == 8 || EPI_WARPS == 16, "epilogue warps");
    static_assert(EPI_COLS % 64 == 0, "each epilogue warp drains whole 64-column reads");
    static_assert(SF_BASE % 8 == 0 && SF_STRIDE % 8 == 0, "8-column stores start at a multiple of 8");
    static_assert(BN % 64 == 0 && (BN <= 192 || BN == 256),
                  "a B tile starts at row 0 or 64 of a scale block and spans <= 2 blocks");
    static_assert(ACC == 1 || ACC == 2, "accumulator buffers");
};
// 256 x 256 tiles with one accumulator: the kernel is bound by the operand
// bytes each SM pulls from L2, and a square tile needs 14% fewer of them per
// flop than 256 x 192 with two accumulators (measured: 149.5 vs 161.8 us on
// the 4096 x 14336 x 4096 prefill).  While the epilogue drains the
// accumulator the producer keeps filling the 5 stages.
using PairUse = PairCfg<256, 5, 4, 1>;

// ---- stream-K tail of the pair kernel ----------------------------------------------
//
// With T tiles on P resident pairs and T % P != 0, the last partial wave would
// leave most pairs idle (prefill 4096 x 14336: 896 tiles on 74 pairs, so 8
// pairs run a 13th tile while 66 wait).  Instead every pair first takes whole
// tiles pair, pair + P, ... below dp_tiles = (T / P - 1) * P, then an equal
// share of the k-tiles of the remaining T - dp_tiles tiles (between P and
// 2P - 1 of them) in tile order.  A share holds at least one tile's k-tiles,
// so a tile is split between at most two consecutive pairs: pair c computes
// its first k-tiles [0, ke) last in its share (the "head", owner of the
// output); pair c + 1 computes the rest [kb, num_kt) first in its own share
// (the "continuation").  The continuation's epilogue stores its FP32
// accumulator to a workspace slot and counts its epilogue warps in a
// per-CTA counter; once the head's MMAs are done, one thread of its epilogue
// waits (bounded) for the full count, copies the slot into the now idle stage
// buffers with bulk copies and returns the counter to zero for the next
// launch; the epilogue adds the copy to its own accumulator before scaling
// and storing as usual.
constexpr int kSkFlagStride = 16;      // uint32 words: one 64-byte line per CTA

// Calls f(std::integral_constant<int, i>) for i = 0 .. N-1 (compile-time indices).
template <int N, int I = 0, class F>
__device__ __forceinline__ void static_for(F&& f) {
    if constexpr (I < N) {
        f(std::integral_constant<int, I>{});
        static_for<N, I + 1>(f);
    }
}

struct PairWork {
    int t = -1, kb = 0, ke = 0;        // current item: tile t, k-tiles [kb, ke)
    int u = -1;                        // next stream-K unit (sk_units < 2^31, host), -1 in the whole-tile phase
    __device__ bool next(const GemmArgs& p, int cluster, int dp_tiles) {
        const int P = (int)(gridDim.x >> 1);
        if (u < 0) {
            t = t < 0 ? cluster : t + P;
            if (t < dp_tiles) {
                kb = 0;
                ke = p.num_kt;
                return true;
            }
            u = (int)(p.sk_units * cluster / P);
        }
        const int u1 = (int)(p.sk_units * (cluster + 1) / P);
        if (u >= u1) return false;
        const int j = u / p.num_kt;
        t = dp_tiles + j;
        kb = u - j * p.num_kt;
        ke = min(p.num_kt, kb + (u1 - u));
        u += ke - kb;
        return true;
    }
};

// Bounded wait until all `warps` epilogue warps of the continuation have counted in.
__device__ __forceinline__ bool sk_wait_ready(const uint32_t* ready, uint32_t warps, uint64_t limit_ns,
                                              volatile int* abort_flag) {
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu_u32(ready) < warps) {
        if (*abort_flag || globaltimer_ns() - t0 > limit_ns) return false;
        __nanosleep(128);
    }
    return true;
}

struct PairGroups {                  // grouped form: per-expert prefixes of pair tiles and scale blocks
    int total_tiles;
    int tile_prefix[kMaxGroups + 1];
    int blk_prefix[kMaxGroups + 1];
};
struct PairNoGroups {};

template <class P, bool GROUPED = false>
struct alignas(8) PairTail : std::conditional_t<GROUPED, PairGroups, PairNoGroups> {
    uint64_t full[P::STAGES];        // leader: both CTAs' A/B bytes
    uint64_t empty[P::STAGES];       // each CTA: released by the leader's MMA commit
    uint64_t sfl[P::STAGES];         // each CTA: its own scale bytes landed
    uint64_t acc_full[P::ACC];       // each CTA: accumulator buffer ready
    uint64_t acc_empty[P::ACC];      // leader: the epilogue warps of both CTAs released it
    uint64_t sf_ready[P::NSB];       // leader: 8 scale warps staged a buffer
    uint64_t sf_free[P::NSB];        // each CTA: MMAs reading a scale buffer done
    uint64_t sk_bar;                 // each CTA: the next pair's partial sums landed (stream-K head)
    uint32_t cmax[P::EPI_WARPS * 32];   // output-maximum variant: each epilogue lane's running max |C|
    uint32_t tmem_base;
    volatile int abort_flag;
};

// Where pair tile t lies, for the CTA of rank `rank`.  Plain: tiles run over
// (256-row m-tile fastest, n-tile).  Grouped: expert e owns tiles
// [tile_prefix[e], tile_prefix[e + 1]), ceil(n_e / 256) m-tiles per n-tile, m
// fastest; its rows start at offsets[e] and its 128-row scale blocks at
// blk_prefix[e]; the rows of a CTA past the expert's end belong to the next
// expert and are neither scaled from its blocks nor stored.
struct PairTile {
    int a_row;       // first A (and output) row of this CTA's half
    int a_rows;      // valid rows of the half (<= 0: none)
    int sfa_rb;      // 128-row A scale block of the half
    bool sfa_ok;     // that block holds this half's rows
    int n0;          // first output column
    int b_row0;      // first B tensor-map row of the pair tile
    int group;
};
template <int BN, bool GROUPED, class TAIL>
__device__ __forceinline__ PairTile pair_tile(const GemmArgs& p, const TAIL* tail, int t, uint32_t rank) {
    PairTile pt;
    int tm, tn, n_e, blocks;
    if constexpr (GROUPED) {
        int lo = 0, hi = p.num_groups;   // largest e with tile_prefix[e] <= t
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (tail->tile_prefix[mid] <= t) lo = mid; else hi = mid;
        }
        const int e = lo, r0 = p.offsets[e];
        n_e = p.offsets[e + 1] - r0;
        const int mt2 = (n_e + 255) / 256;
        const int local = t - tail->tile_prefix[e];
        tm = local % mt2;
        tn = local / mt2;
        pt.a_row = r0 + tm * 256 + 128 * (int)rank;
        pt.sfa_rb = tail->blk_prefix[e] + 2 * tm + (int)rank;
        blocks = (n_e + 127) / 128;
        pt.b_row0 = e * p.rows_b + tn * BN;
        pt.group = e;
    } else {
        const int tiles_m2 = (p.rows_a + 255) / 256;
        tm = t % tiles_m2;
        tn = t / tiles_m2;
        n_e = p.rows_a;
        pt.a_row = tm * 256 + 128 * (int)rank;
        pt.sfa_rb = 2 * tm + (int)rank;
        blocks = (p.rows_a + 127) / 128;
        pt.b_row0 = tn * BN;
        pt.group = 0;
    }
    pt.a_rows = n_e - (tm * 256 + 128 * (int)rank);
    pt.sfa_ok = 2 * tm + (int)rank < blocks;
    pt.n0 = tn * BN;
    return pt;
}

// MX: MXFP4 operands, as in gemm_kernel (plain form only).
template <class P, bool GROUPED, bool EMIT = false, bool MX = false>
__global__ void __launch_bounds__(P::THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const __grid_constant__ CUtensorMap tmC, const GemmArgs p) {
    constexpr int BN = P::BN, BH = P::BH, STAGES = P::STAGES, NBC = P::NBC;
    constexpr uint32_t IDESC = idesc_mxf4nvf4(256, BN);
    constexpr uint32_t IDESC_MX0 = idesc_mxf4_e8m0(256, BN, 0), IDESC_MX2 = idesc_mxf4_e8m0(256, BN, 2);
    constexpr int SF_KT = MX ? 1024 : 2048;      // scale bytes of one k-tile per 128-row block
    constexpr int NCH = MX ? 2 : 4;              // 512-byte scale chunks per k-tile
    static_assert(!(MX && (GROUPED || EMIT)), "MXFP4: plain form only");
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* epi_smem = smem + STAGES * P::STAGE_BYTES;
    PairTail<P, GROUPED>* tail = reinterpret_cast<PairTail<P, GROUPED>*>(epi_smem + P::EPI_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster = blockIdx.x >> 1;
    const uint64_t limit = p.wait_limit_ns;
    if (p.pdl_trigger) pdl_launch_dependents();   // as in gemm_kernel

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&tail->full[s], 1);
            mbar_init(&tail->empty[s], 1);
            mbar_init(&tail->sfl[s], 1);
        }
        for (int b = 0; b < P::ACC; ++b) {
            mbar_init(&tail->acc_full[b], 1);
            mbar_init(&tail->acc_empty[b], 2 * P::EPI_WARPS);
        }
        for (int b = 0; b < P::NSB; ++b) {
            mbar_init(&tail->sf_ready[b], 8);
            mbar_init(&tail->sf_free[b], 1);
        }
        mbar_init(&tail->sk_bar, 1);
        tail->abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmA);
        prefetch_tmap(&tmB);
        prefetch_tmap(&tmC);
    }
    if (warp == 1) {
        tmem_alloc_pair(&tail->tmem_base, kTmemCols);
        tmem_relinquish_pair();
    }
    pdl_wait();
    if constexpr (GROUPED) {
        // per-expert prefixes (the offsets may come from the previous kernel)
        if (warp == 2) {
            const int E = p.num_groups;
            const int per = (E + 31) / 32;
            int t_loc = 0, b_loc = 0;
            for (int i = 0; i < per; ++i) {
                const int e = lane * per + i;
                if (e < E) {
                    const int n_e = p.offsets[e + 1] - p.offsets[e];
                    t_loc += (n_e + 255) / 256 * p.tiles_n;
                    b_loc += (n_e + 127) / 128;
                }
            }
            int t_inc = t_loc, b_inc = b_loc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const int tv = __shfl_up_sync(0xFFFFFFFFu, t_inc, o);
                const int bv = __shfl_up_sync(0xFFFFFFFFu, b_inc, o);
                if (lane >= o) {
                    t_inc += tv;
                    b_inc += bv;
                }
            }
            int t_run = t_inc - t_loc, b_run = b_inc - b_loc;
            for (int i = 0; i < per; ++i) {
                const int e = lane * per + i;
                if (e < E) {
                    tail->tile_prefix[e] = t_run;
                    tail->blk_prefix[e] = b_run;
                    const int n_e = p.offsets[e + 1] - p.offsets[e];
                    t_run += (n_e + 255) / 256 * p.tiles_n;
                    b_run += (n_e + 127) / 128;
                }
            }
            if (lane == 31) {
                tail->tile_prefix[E] = t_inc;
                tail->blk_prefix[E] = b_inc;
                tail->total_tiles = t_inc;
            }
        }
    }
    tc_fence_before();
    cluster_sync();          // both CTAs' barriers initialized, tensor memory allocated (and prefixes written)
    tc_fence_after();
    const uint32_t tmem = tail->tmem_base;
    int dp_tiles = p.dp_tiles;               // grouped: every tile whole
    if constexpr (GROUPED) dp_tiles = tail->total_tiles;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs) ----------------
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            PairWork w;
            while (ok && w.next(p, cluster, dp_tiles)) {
                const PairTile pt = pair_tile<BN, GROUPED>(p, tail, w.t, rank);
                const int a_row = pt.a_row;
                const int g0 = pt.b_row0 + BH * (int)rank;        // first B row of this CTA's half
                const bool sfa_ok = pt.sfa_ok;
                const int a0 = pt.n0 / 128;                       // B scales: all BN rows of the tile
                const int nsfb = max(0, min((pt.n0 % 128 + BN + 127) / 128, p.sfb_rb_per_group - a0));
                const uint8_t* sfa_src = p.sfa + (int64_t)pt.sfa_rb * p.sfa_rb_stride;
                const uint8_t* sfb_src =
                    p.sfb + (int64_t)pt.group * p.sfb_group_stride + (int64_t)a0 * p.sfb_rb_stride;
                for (int kt = w.kb; kt < w.ke; ++kt) {
                    if (!mbar_wait(&tail->empty[stage], phase ^ 1u, limit) || tail->abort_flag) {
                        ok = false;
                        break;
                    }
                    const int nat = min(4, p.num_ks - kt * 4);
                    uint8_t* sA = smem + stage * P::STAGE_BYTES;
                    uint8_t* sB = sA + P::A_BYTES;
                    uint8_t* sSFA = sB + P::B_BYTES;
                    uint8_t* sSFB = sSFA + P::SFA_BYTES;
                    const uint32_t full0 = mapa_shared(smem_u32(&tail->full[stage]), 0);
                    if (leader) mbar_arrive_expect_tx(&tail->full[stage], 2u * (P::A_BYTES + P::B_BYTES));
                    tma_load_2d_pair(sA, &tmA, full0, kt * 128, a_row);
                    tma_load_2d_pair(sB, &tmB, full0, kt * 128, g0);
                    uint64_t* sbar = &tail->sfl[stage];
                    const uint32_t nch = MX ? (uint32_t)(nat + 1) / 2 : (uint32_t)nat;   // scale chunks used
                    const uint32_t sbytes = nch * 512u * ((sfa_ok ? 1u : 0u) + (uint32_t)nsfb);
                    mbar_arrive_expect_tx(sbar, sbytes);
                    if (sfa_ok) bulk_load(sSFA, sfa_src + (int64_t)kt * SF_KT, nch * 512u, sbar);
                    for (int rb = 0; rb < nsfb; ++rb)
                        bulk_load(sSFB + rb * 2048, sfb_src + (int64_t)rb * p.sfb_rb_stride + (int64_t)kt * SF_KT,
                                  nch * 512u, sbar);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                tail->abort_flag = 1;
                if (p.err) atomicOr(p.err, 1u);
            }
        }
    } else if (warp == 1) {
        if (leader && lane == 0) {
            // ---------------- MMA issuer (pair leader) ----------------
            uint32_t stage = 0, phase = 0, sb = 0, sph = 0;
            int it = 0;
            bool ok = true;
            PairWork w;
            for (; ok && w.next(p, cluster, dp_tiles); ++it) {
                const uint32_t ab = (uint32_t)(it % P::ACC), au = (uint32_t)(it / P::ACC);
                if (!mbar_wait(&tail->acc_empty[ab], (au & 1u) ^ 1u, limit) || tail->abort_flag) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d_tmem = tmem + ab * BN;
                for (int kt = w.kb; kt < w.ke; ++kt) {
                    if (!mbar_wait(&tail->full[stage], phase, limit) ||
                        !mbar_wait(&tail->sf_ready[sb], sph, limit) || tail->abort_flag) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nat = min(4, p.num_ks - kt * 4);
                    const uint32_t sA = smem_u32(smem + stage * P::STAGE_BYTES);
                    const uint32_t sB = sA + P::A_BYTES;
                    const uint32_t sf = tmem + P::SF_BASE + sb * P::SF_STRIDE;
                    for (int j = 0; j < nat; ++j) {
                        if constexpr (MX)
                            mma_mxf4nvf4_pair<true>(d_tmem, sdesc_kmajor_sw128(sA + j * 32),
                                                    sdesc_kmajor_sw128(sB + j * 32), (j & 1) ? IDESC_MX2 : IDESC_MX0,
                                                    sf + (j >> 1) * 4, sf + 16 + (j >> 1) * NBC,
                                                    (kt > w.kb || j > 0) ? 1u : 0u);
                        else
                            mma_mxf4nvf4_pair(d_tmem, sdesc_kmajor_sw128(sA + j * 32), sdesc_kmajor_sw128(sB + j * 32),
                                              IDESC, sf + j * 4, sf + 16 + j * NBC, (kt > w.kb || j > 0) ? 1u : 0u);
                    }
                    tc_commit_pair(&tail->empty[stage], 0x3);
                    tc_commit_pair(&tail->sf_free[sb], 0x3);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    if (++sb == (uint32_t)P::NSB) {
                        sb = 0;
                        sph ^= 1u;
                    }
                }
                if (ok) tc_commit_pair(&tail->acc_full[ab], 0x3);
            }
            if (!ok) {
                tail->abort_flag = 1;
                if (p.err) atomicOr(p.err, 1u);
            }
        }
    } else if (warp >= 2 + P::EPI_WARPS) {
        // ---------------- scale staging (both CTAs; warps 10..13, one lane quarter each) ----------------
        const int q = warp & 3;
        const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16) + P::SF_BASE;
        const uint32_t ready0 = mapa_shared(smem_u32(&tail->sf_ready[0]), 0);
        const uint32_t ready_step = (uint32_t)(smem_u32(&tail->sf_ready[1]) - smem_u32(&tail->sf_ready[0]));
        uint32_t stage = 0, phase = 0, sb = 0, sph = 0;
        bool ok = true;
        PairWork wk;
        while (ok && wk.next(p, cluster, dp_tiles)) {
            const int off = pair_tile<BN, GROUPED>(p, tail, wk.t, rank).n0 % 128;   // first tile row in its first scale block
            for (int kt = wk.kb; kt < wk.ke; ++kt) {
                // read this k-tile's scale words as soon as they land, then wait
                // for the tensor-memory buffer: only the stores stay on the
                // MMA's critical path
                if (!mbar_wait(&tail->sfl[stage], phase, limit) || tail->abort_flag) {
                    ok = false;
                    break;
                }
                const uint32_t sSFA = smem_u32(smem + stage * P::STAGE_BYTES) + P::A_BYTES + P::B_BYTES;
                const uint32_t sSFB = sSFA + P::SFA_BYTES;
                // one k-tile of scales, in tensor-memory column order: A k-step j at
                // 4j, B k-step j at 16 + NBC * j (column c = tile rows 32c..32c+31)
                uint32_t w[P::SF_COLS];
                if constexpr (MX) {   // chunks 2 and 3 are unused
#pragma unroll
                    for (int i = 0; i < (int)P::SF_COLS; ++i) w[i] = 0u;
                }
#pragma unroll
                for (int j = 0; j < NCH; ++j) {
                    const uint4 v = ld_shared_v4(sSFA + j * 512 + lane * 16);
                    w[4 * j + 0] = v.x;
                    w[4 * j + 1] = v.y;
                    w[4 * j + 2] = v.z;
                    w[4 * j + 3] = v.w;
                }
#pragma unroll
                for (int j = 0; j < NCH; ++j)
#pragma unroll
                    for (int c = 0; c < NBC; ++c) {
                        // tile row 32c + lane of B: its 4 scales of k-step j
                        const int rr = off + 32 * c + lane;           // row relative to the first loaded block
                        const uint32_t addr = sSFB + (uint32_t)((rr >> 7) * 2048 + j * 512 + (rr & 31) * 16 +
                                                                ((rr >> 5) & 3) * 4);
                        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(w[16 + NBC * j + c]) : "r"(addr));
                    }
                if (!mbar_wait(&tail->sf_free[sb], sph ^ 1u, limit) || tail->abort_flag) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // 8-column stores (the buffers are packed SF_COLS columns apart)
                const uint32_t dst = tq + sb * P::SF_STRIDE;
#pragma unroll
                for (int i = 0; i < (int)P::SF_COLS / 8; ++i) tmem_st_32x32b_x8(dst + 8 * i, w + 8 * i);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(ready0 + sb * ready_step);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
                if (++sb == (uint32_t)P::NSB) {
                    sb = 0;
                    sph ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) {
            tail->abort_flag = 1;
            if (p.err) atomicOr(p.err, 1u);
        }
    } else if (warp >= 2) {
        // ---------------- epilogue (both CTAs; warps 2..9) ----------------
        // Two warps per tensor-memory lane quarter, each draining half of the
        // tile's columns; a warp releases the accumulator right after its last
        // tensor-memory reads, before staging and storing, so the next tile's
        // MMAs wait only for the reads (measured on the prefill shape: 4 warps
        // 143 us, 8 warps 139 us, 8 warps reading 64 columns at a time 135 us,
        // converting all of them before the stores 133 us; 16 warps were slower).
        constexpr int NCP = P::EPI_CP;
        const int q = warp & 3;
        const int c0 = ((warp - 2) >> 2) * (2 * NCP);      // first 32-column chunk of this warp
        const uint32_t stg = smem_u32(epi_smem) + (uint32_t)(warp - 2) * (P::EPI_BOXES * 2048u);
        const uint32_t empty0 = mapa_shared(smem_u32(&tail->acc_empty[0]), 0);
        const uint32_t empty_step = (uint32_t)sizeof(uint64_t);
        // output-maximum variant: the lane's running max |C| lives in shared
        // memory, not in a register held across the whole loop
        uint32_t* cmax = &tail->cmax[(warp - 2) * 32 + lane];
        if (EMIT) *cmax = 0u;
        int it = 0;
        PairWork w;
        for (; w.next(p, cluster, dp_tiles); ++it) {
            const uint32_t ab = (uint32_t)(it % P::ACC), au = (uint32_t)(it / P::ACC);
            // stream-K roles of this item: a continuation hands its partial sums
            // to the previous pair; a head adds those of the next pair
            const bool give = w.kb > 0, take = w.ke < p.num_kt;
            const int slot_idx = (give ? cluster : cluster + 1) * 2 + (int)rank;
            bool wait_ok = mbar_wait(&tail->acc_full[ab], au & 1u, limit) && !tail->abort_flag;
            if (wait_ok && take) {
                // The head is this pair's last item: with its MMAs done the stage
                // buffers are free, so one bulk copy brings the next pair's partial
                // sums (128 x BN FP32) on chip while the accumulator is read.
                if (warp == 2 && lane == 0) {
                    wait_ok = sk_wait_ready(p.sk_flags + slot_idx * kSkFlagStride, (uint32_t)P::EPI_WARPS, limit,
                                            &tail->abort_flag);
                    if (wait_ok) {
                        fence_proxy_async_global();
                        constexpr uint32_t kPart = 128u * BN * 4u, kPiece = 16384u;
                        mbar_arrive_expect_tx(&tail->sk_bar, kPart);
                        const uint8_t* src = reinterpret_cast<const uint8_t*>(p.partial) + (size_t)slot_idx * kPart;
                        for (uint32_t o = 0; o < kPart; o += kPiece) bulk_load(smem + o, src + o, kPiece, &tail->sk_bar);
                    }
                }
                wait_ok = __shfl_sync(0xffffffffu, wait_ok ? 1 : 0, 0) != 0;
                if (wait_ok) wait_ok = mbar_wait(&tail->sk_bar, 0u, limit) && !tail->abort_flag;
                // the copy has read the slot: clear the counter for the next launch
                if (wait_ok && warp == 2 && lane == 0) st_relaxed_gpu_u32(p.sk_flags + slot_idx * kSkFlagStride, 0u);
            }
            if (!wait_ok) {
                if (lane == 0) {
                    tail->abort_flag = 1;
                    if (p.err) atomicOr(p.err, 1u);
                }
                break;
            }
            tc_fence_after();
            const PairTile pt = pair_tile<BN, GROUPED>(p, tail, w.t, rank);
            const int a_row0 = pt.a_row;
            const int n0 = pt.n0;
            const int a_rows = pt.a_rows;
            const int b_cols = min(BN, p.rows_b - n0);
            const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16) + ab * BN;
            const float alpha = MX ? 1.0f : __fmul_rn(p.ga[pt.group], p.gb[pt.group]);
            // One 32-column chunk (16 BF16 pairs per lane) through a staging box to C.
            auto store_chunk = [&](int ch, const uint32_t* w16) {
                if (ch * 32 >= b_cols || q * 32 >= a_rows) return;   // uniform per warp
                if (GROUPED && q * 32 + 32 > a_rows) {
                    // the expert's last rows: the next rows of C belong to the next
                    // expert, so no 32-row box; each lane stores its own row
                    if (q * 32 + lane < a_rows) {
                        __nv_bfloat16* crow = p.c + (int64_t)(a_row0 + q * 32 + lane) * p.ldc + n0 + ch * 32;
                        if (b_cols - ch * 32 >= 32) {
#pragma unroll
                            for (int j = 0; j < 4; ++j)
                                *reinterpret_cast<uint4*>(crow + 8 * j) =
                                    make_uint4(w16[4 * j], w16[4 * j + 1], w16[4 * j + 2], w16[4 * j + 3]);
                        } else {
                            const int ncols = b_cols - ch * 32;
#pragma unroll
                            for (int i = 0; i < 32; ++i)
                                if (i < ncols)
                                    crow[i] = __ushort_as_bfloat16((unsigned short)(w16[i >> 1] >> (16 * (i & 1))));
                        }
                    }
                    return;
                }
                const uint32_t box = stg + (P::EPI_BOXES == 2 ? (uint32_t)(ch & 1) * 2048u : 0u);
                if (lane == 0) {
                    if constexpr (P::EPI_BOXES == 2) bulk_wait_group_read<1>(); else bulk_wait_group_read<0>();
                }
                __syncwarp();
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 v = make_uint4(w16[4 * j], w16[4 * j + 1], w16[4 * j + 2], w16[4 * j + 3]);
                    st_shared_v4(box + (uint32_t)lane * 64u + (uint32_t)((j ^ ((lane >> 1) & 3)) * 16), v);
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tma_store_2d(&tmC, box, n0 + ch * 32, a_row0 + q * 32);
                    bulk_commit_group();
                }
            };
            if (give) {
                // Continuation: FP32 partial sums to the workspace slot, 4-column
                // group g of row r at slot[g * 128 + r] (lane-contiguous 16-byte
                // pieces), then one count per warp.
                float4* slot = reinterpret_cast<float4*>(p.partial + (size_t)slot_idx * (128 * BN)) + q * 32 + lane;
                // 32 columns at a time: this rare path keeps few values live
#pragma unroll 1
                for (int ch = 0; ch < 2 * NCP; ++ch) {
                    uint32_t va[32];
                    tmem_ld_32x32b_x32(tq + (c0 + ch) * 32, va);
                    tmem_ld_wait();
                    if (ch == 2 * NCP - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(empty0 + ab * empty_step);
                    }
                    float4* part = slot + (c0 + ch) * 8 * 128;   // one base, immediate offsets
                    static_for<8>([&](auto ic) {
                        constexpr int i = decltype(ic)::value;
                        st_global_v4_at<i * 2048>(part, va[4 * i], va[4 * i + 1], va[4 * i + 2], va[4 * i + 3]);
                    });
                }
                // the warp barrier orders every lane's stores before lane 0's
                // release, which carries them to the acquiring head (cumulativity)
                __syncwarp();
                if (lane == 0) red_release_gpu_add_u32(p.sk_flags + slot_idx * kSkFlagStride, 1u);
                continue;
            }
            if (take) {
                // Head: add the next pair's partial sums (now in the stage
                // buffers, same layout) before scaling.
                const uint32_t slot_s = smem_u32(smem) + (uint32_t)(q * 32 + lane) * 16u;
#pragma unroll
                for (int cp = 0; cp < NCP; ++cp) {
                    uint32_t va0[32], va1[32];
                    tmem_ld_32x32b_x32(tq + (c0 + cp * 2) * 32, va0);
                    tmem_ld_32x32b_x32(tq + (c0 + cp * 2) * 32 + 32, va1);
                    tmem_ld_wait();
                    if (cp == NCP - 1) {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(empty0 + ab * empty_step);
                    }
                    const uint32_t part_s = slot_s + (uint32_t)((c0 + cp * 2) * 8 * 128) * 16u;
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        uint4 x[4];
#pragma unroll
                        for (int i = 0; i < 4; ++i) x[i] = ld_shared_v4(part_s + (uint32_t)((4 * g + i) * 128) * 16u);
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            uint32_t* v = (g < 2 ? va0 : va1) + 16 * (g & 1) + 4 * i;
                            v[0] = __float_as_uint(__uint_as_float(v[0]) + __uint_as_float(x[i].x));
                            v[1] = __float_as_uint(__uint_as_float(v[1]) + __uint_as_float(x[i].y));
                            v[2] = __float_as_uint(__uint_as_float(v[2]) + __uint_as_float(x[i].z));
                            v[3] = __float_as_uint(__uint_as_float(v[3]) + __uint_as_float(x[i].w));
                        }
                    }
                    uint32_t bh[32];
#pragma unroll
                    for (int i = 0; i < 16; ++i) {
                        bh[i] = pack_bf16x2(__uint_as_float(va0[2 * i]) * alpha, __uint_as_float(va0[2 * i + 1]) * alpha);
                        bh[16 + i] =
                            pack_bf16x2(__uint_as_float(va1[2 * i]) * alpha, __uint_as_float(va1[2 * i + 1]) * alpha);
                    }
                    if (EMIT && q * 32 + lane < a_rows) {
                        uint32_t cm = *cmax;
#pragma unroll
                        for (int i = 0; i < 32; ++i) cm = max_abs_bf16x2(cm, bh[i]);
                        *cmax = cm;
                    }
                    store_chunk(c0 + cp * 2, bh);
                    store_chunk(c0 + cp * 2 + 1, bh + 16);
                }
                continue;
            }
            // Whole tile: read the warp's BN / 2 columns 64 at a time and
            // convert them to BF16 in registers; release the accumulator after
            // the last read, then stage and store.
            uint32_t bf[NCP * 32];
            uint32_t cm = 0;   // output-maximum variant: this tile's max |C| in the lane's row
#pragma unroll
            for (int cp = 0; cp < NCP; ++cp) {
                uint32_t va0[32], va1[32];
                tmem_ld_32x32b_x32(tq + (c0 + cp * 2) * 32, va0);
                tmem_ld_32x32b_x32(tq + (c0 + cp * 2) * 32 + 32, va1);
                tmem_ld_wait();
                if (cp == NCP - 1) {
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_cluster(empty0 + ab * empty_step);
                }
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    bf[cp * 32 + i] = pack_bf16x2(__uint_as_float(va0[2 * i]) * alpha,
                                                  __uint_as_float(va0[2 * i + 1]) * alpha);
                    bf[cp * 32 + 16 + i] = pack_bf16x2(__uint_as_float(va1[2 * i]) * alpha,
                                                       __uint_as_float(va1[2 * i + 1]) * alpha);
                    if (EMIT) cm = max_abs_bf16x2(cm, max_abs_bf16x2(bf[cp * 32 + i], bf[cp * 32 + 16 + i]));
                }
            }
            if (EMIT && q * 32 + lane < a_rows) *cmax = max_abs_bf16x2(*cmax, cm);
#pragma unroll
            for (int h = 0; h < 2 * NCP; ++h) store_chunk(c0 + h, bf + h * 16);
        }
        if (EMIT) fold_c_amax(p, *cmax);
        if (lane == 0) bulk_wait_group_all();
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (EMIT && threadIdx.x == 0) finish_c_amax(p);
    cluster_sync();          // no CTA leaves while its peer may still touch its shared memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

// ---- grouped GEMM with the operands swapped (MoE) ----------------------------------
//
// Per expert e (rows [r0, r0 + n_e) of A, weights W_e [n, k]) the pair kernel
// above puts the tokens on the MMA's 256-row side, so an expert of 257 rows
// takes two 256-row tiles.  Here the weights take the 256-row side (n % 256
// == 0: M = 256 over the CTA pair, 128 weight rows per CTA) and the expert's
// tokens the N side, in tiles of 256 tokens.  A last part of at most 64
// tokens rides on the tile before it as a second MMA into a second
// accumulator, against the same weight stages; any other last part is a tile
// of its own.  Each part's N is its token count rounded up to a multiple of
// 32 (cta_group::2 MMAs take N in steps of 16), so an expert pads fewer than
// 32 rows.  Each CTA loads N / 2 token rows of a part (tensor maps with
// boxes of 16, 32, 64 and 128 rows; the smallest that holds them) and stages
// the scales of all token columns; token tiles start at multiples of 256
// rows of the expert, i.e. at row 0 of a 128-row scale block.  Tiles of
// expert e run (weight tile, token tile) with the token tile fastest, so the
// CTAs working on one weight tile at the same time share it through L2.
//
// The accumulators hold weight rows in tensor-memory lanes and tokens in
// columns (the second part's from column 256), so the epilogue writes C
// transposed: each warp reads 32 token columns of its 32 lanes (one weight
// row per thread) and converts them to BF16; neighbouring lanes swap values
// so that each holds two adjacent output columns of one token, and one warp
// store writes 64 contiguous bytes of each of two token rows of C.  Stores
// stop at the expert's last token (the next rows of C belong to the next
// expert).
//
// Warps: 0 producer, 1 MMA (leader), 2-9 epilogue (two per tensor-memory lane
// quarter, alternate 32-column chunks), 10-13 scale staging.  Tensor memory
// per CTA: the 256 + 64 accumulator columns, three scale buffers of 56.
struct SwapCfg {
    static constexpr int STAGES = 5;
    static constexpr int NSB = 3;                          // scale buffers in tensor memory
    static constexpr int N2_MAX = 64;                      // tokens of a second part
    static constexpr uint32_t A_BYTES = 128 * 128;         // 128 weight rows x 256 FP4
    static constexpr uint32_t B_BYTES = 128 * 128;         // up to 128 token rows x 256 FP4
    static constexpr uint32_t B2_BYTES = (N2_MAX / 2) * 128;   // a second part's token rows
    static constexpr uint32_t SFA_BYTES = 4 * 512;         // the CTA's 128 weight rows
    static constexpr uint32_t SFB_BYTES = 3 * 4 * 512;     // <= 320 token rows from row 0 of a block: 3 blocks
    static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES + B2_BYTES + SFA_BYTES + SFB_BYTES;
    static constexpr int NBC = (256 + N2_MAX) / 32;        // token scale columns per k-step
    static constexpr uint32_t SF_COLS = 16 + 4 * NBC;
    static constexpr uint32_t SF_STRIDE = SF_COLS;
    static constexpr uint32_t SF_BASE = 256 + N2_MAX;      // after the accumulators
    static constexpr int EPI_WARPS = 8;
    static constexpr int THREADS = 32 * (2 + EPI_WARPS + 4);
    static constexpr int NUM_BOXES = 4;                    // token maps with boxes of 16, 32, 64, 128 rows
    static constexpr int MAX_CHUNKS = NBC;                 // 32-column accumulator chunks
    static_assert(STAGE_BYTES % 1024 == 0, "stage alignment");
    static_assert((A_BYTES + B_BYTES) % 1024 == 0, "second token box alignment (128-byte swizzle)");
    static_assert(SF_BASE + NSB * SF_STRIDE <= kTmemCols, "tensor memory budget");
    static_assert(SF_BASE % 8 == 0 && SF_STRIDE % 8 == 0, "8-column stores start at a multiple of 8");
};

struct alignas(8) SwapTail {
    uint64_t full[SwapCfg::STAGES];      // leader: both CTAs' weight and token bytes
    uint64_t empty[SwapCfg::STAGES];     // each CTA: released by the leader's MMA commit
    uint64_t sfl[SwapCfg::STAGES];       // each CTA: its own scale bytes landed
    uint64_t acc_full;                   // each CTA: accumulators ready
    uint64_t acc_empty;                  // leader: the epilogue warps of both CTAs read them
    uint64_t sf_ready[SwapCfg::NSB];     // leader: 8 scale warps staged a buffer
    uint64_t sf_free[SwapCfg::NSB];      // each CTA: MMAs reading a scale buffer done
    uint32_t tmem_base;
    volatile int abort_flag;
    int total_tiles;
    int tile_prefix[kMaxGroups + 1];     // first tile of expert e
    int blk_prefix[kMaxGroups + 1];      // first 128-row token scale block of expert e
};
constexpr size_t kSwapSmem = 1024 + (size_t)SwapCfg::STAGES * SwapCfg::STAGE_BYTES + sizeof(SwapTail);
static_assert(kSwapSmem <= 232448, "shared memory");

// Token maps: one per box height (16 << i rows).
struct SwapMaps {
    CUtensorMap x[SwapCfg::NUM_BOXES];
};

// Token tiles of an expert of n_e rows: 256 each; a last part of at most 64
// tokens joins the tile before it.
__device__ __forceinline__ int swap_token_tiles(int n_e) {
    const int full = n_e >> 8, rem = n_e & 255;
    return full + ((rem > 0 && (full == 0 || rem > SwapCfg::N2_MAX)) ? 1 : 0);
}
__device__ __forceinline__ int swap_box(int rows) { return rows <= 16 ? 0 : rows <= 32 ? 1 : rows <= 64 ? 2 : 3; }

// Where tile t lies.
struct SwapTile {
    int e;
    int w_row;      // first weight tensor-map row of this CTA's 128
    int tok0;       // first token row of the tile (A / C row)
    int ntok;       // valid tokens of the tile (<= 256 + 64)
    int N1, N2;     // MMA N of the two parts (tokens rounded up to 32; N2 = 0: one part)
    int x1_row;     // first token row of this CTA's half of part 1
    int x2_row;     // ... of part 2
    int box1, box2; // token map of each part: 16 << box >= N / 2
    int sfw_blk;    // weight scale block (128 rows) of this CTA, within the expert's weights
    int sfx_blk;    // first token scale block of the tile
    int nsfx;       // token scale blocks the tile touches (1 to 3)
    int wcol0;      // first output column of this CTA's 128 weight rows
};
__device__ __forceinline__ SwapTile swap_tile(const GemmArgs& p, const SwapTail* tail, int t, uint32_t rank) {
    int lo = 0, hi = p.num_groups;   // largest e with tile_prefix[e] <= t
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (tail->tile_prefix[mid] <= t) lo = mid; else hi = mid;
    }
    SwapTile s;
    const int e = lo;
    const int r0 = p.offsets[e], n_e = p.offsets[e + 1] - r0;
    const int T = swap_token_tiles(n_e);
    const int local = t - tail->tile_prefix[e];
    const int wt = local / T, j = local - wt * T;
    s.e = e;
    s.ntok = j < T - 1 ? 256 : n_e - 256 * j;
    s.N1 = (min(s.ntok, 256) + 31) & ~31;
    s.N2 = s.ntok > 256 ? (s.ntok - 256 + 31) & ~31 : 0;
    s.tok0 = r0 + 256 * j;
    s.x1_row = s.tok0 + (s.N1 >> 1) * (int)rank;
    s.x2_row = s.tok0 + 256 + (s.N2 >> 1) * (int)rank;
    s.box1 = swap_box(s.N1 >> 1);
    s.box2 = swap_box(s.N2 >> 1);
    s.wcol0 = wt * 256 + 128 * (int)rank;
    s.w_row = e * p.rows_b + s.wcol0;
    s.sfw_blk = 2 * wt + (int)rank;
    s.sfx_blk = tail->blk_prefix[e] + 2 * j;
    s.nsfx = (s.N1 + s.N2 + 127) / 128;
    return s;
}

__global__ void __launch_bounds__(SwapCfg::THREADS, 1)
    moe_swap_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ SwapMaps tmX,
                    const __grid_constant__ CUtensorMap tmC, const GemmArgs p) {
    using P = SwapCfg;
    constexpr int STAGES = P::STAGES, NBC = P::NBC;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    SwapTail* tail = reinterpret_cast<SwapTail*>(smem + STAGES * P::STAGE_BYTES);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const bool leader = rank == 0;
    const int cluster = blockIdx.x >> 1;
    const int P2 = (int)(gridDim.x >> 1);
    const uint64_t limit = p.wait_limit_ns;
    // No early launch of the next kernel here: on the MoE step the next one is
    // the grouped one-launch quantizer, and starting it while this grid's
    // pairs finish unevenly cost ≈ 4 us per step (measured).

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(&tail->full[s], 1);
            mbar_init(&tail->empty[s], 1);
            mbar_init(&tail->sfl[s], 1);
        }
        mbar_init(&tail->acc_full, 1);
        mbar_init(&tail->acc_empty, 2 * P::EPI_WARPS);
        for (int b = 0; b < P::NSB; ++b) {
            mbar_init(&tail->sf_ready[b], 8);
            mbar_init(&tail->sf_free[b], 1);
        }
        tail->abort_flag = 0;
        fence_mbar_init();
        prefetch_tmap(&tmW);
        for (int i = 0; i < P::NUM_BOXES; ++i) prefetch_tmap(&tmX.x[i]);
        prefetch_tmap(&tmC);
    }
    if (warp == 1) {
        tmem_alloc_pair(&tail->tmem_base, kTmemCols);
        tmem_relinquish_pair();
    }
    pdl_wait();
    if (warp == 2) {
        // per-expert prefixes of tiles and token scale blocks (the offsets may
        // come from the previous kernel)
        const int E = p.num_groups, W = p.rows_b / 256;
        const int per = (E + 31) / 32;
        int t_loc = 0, b_loc = 0;
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            if (e < E) {
                const int n_e = p.offsets[e + 1] - p.offsets[e];
                t_loc += swap_token_tiles(n_e) * W;
                b_loc += (n_e + 127) / 128;
            }
        }
        int t_inc = t_loc, b_inc = b_loc;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int tv = __shfl_up_sync(0xFFFFFFFFu, t_inc, o);
            const int bv = __shfl_up_sync(0xFFFFFFFFu, b_inc, o);
            if (lane >= o) {
                t_inc += tv;
                b_inc += bv;
            }
        }
        int t_run = t_inc - t_loc, b_run = b_inc - b_loc;
        for (int i = 0; i < per; ++i) {
            const int e = lane * per + i;
            if (e < E) {
                tail->tile_prefix[e] = t_run;
                tail->blk_prefix[e] = b_run;
                const int n_e = p.offsets[e + 1] - p.offsets[e];
                t_run += swap_token_tiles(n_e) * W;
                b_run += (n_e + 127) / 128;
            }
        }
        if (lane == 31) {
            tail->tile_prefix[E] = t_inc;
            tail->blk_prefix[E] = b_inc;
            tail->total_tiles = t_inc;
        }
    }
    tc_fence_before();
    cluster_sync();          // both CTAs' barriers initialized, tensor memory allocated, prefixes written
    tc_fence_after();
    const uint32_t tmem = tail->tmem_base;
    const int total_tiles = tail->total_tiles;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs) ----------------
            uint32_t stage = 0, phase = 0;
            bool ok = true;
            for (int t = cluster; t < total_tiles && ok; t += P2) {
                const SwapTile st = swap_tile(p, tail, t, rank);
                const uint32_t xbytes = (16u << st.box1) * 128u + (st.N2 ? (16u << st.box2) * 128u : 0u);
                const uint8_t* sfw_src =
                    p.sfb + (int64_t)st.e * p.sfb_group_stride + (int64_t)st.sfw_blk * p.sfb_rb_stride;
                const uint8_t* sfx_src = p.sfa + (int64_t)st.sfx_blk * p.sfa_rb_stride;
                for (int kt = 0; kt < p.num_kt; ++kt) {
                    if (!mbar_wait(&tail->empty[stage], phase ^ 1u, limit) || tail->abort_flag) {
                        ok = false;
                        break;
                    }
                    const int nat = min(4, p.num_ks - kt * 4);
                    uint8_t* sA = smem + stage * P::STAGE_BYTES;
                    uint8_t* sB = sA + P::A_BYTES;
                    uint8_t* sB2 = sB + P::B_BYTES;
                    uint8_t* sSFA = sB2 + P::B2_BYTES;
                    uint8_t* sSFB = sSFA + P::SFA_BYTES;
                    const uint32_t full0 = mapa_shared(smem_u32(&tail->full[stage]), 0);
                    if (leader) mbar_arrive_expect_tx(&tail->full[stage], 2u * (P::A_BYTES + xbytes));
                    tma_load_2d_pair(sA, &tmW, full0, kt * 128, st.w_row);
                    tma_load_2d_pair(sB, &tmX.x[st.box1], full0, kt * 128, st.x1_row);
                    if (st.N2) tma_load_2d_pair(sB2, &tmX.x[st.box2], full0, kt * 128, st.x2_row);
                    uint64_t* sbar = &tail->sfl[stage];
                    const uint32_t nch = (uint32_t)nat;
                    mbar_arrive_expect_tx(sbar, nch * 512u * (1u + (uint32_t)st.nsfx));
                    bulk_load(sSFA, sfw_src + (int64_t)kt * 2048, nch * 512u, sbar);
                    for (int rb = 0; rb < st.nsfx; ++rb)
                        bulk_load(sSFB + rb * 2048, sfx_src + (int64_t)rb * p.sfa_rb_stride + (int64_t)kt * 2048,
                                  nch * 512u, sbar);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                }
            }
            if (!ok) {
                tail->abort_flag = 1;
                if (p.err) atomicOr(p.err, 1u);
            }
        }
    } else if (warp == 1) {
        if (leader && lane == 0) {
            // ---------------- MMA issuer (pair leader) ----------------
            uint32_t stage = 0, phase = 0, sb = 0, sph = 0;
            int it = 0;
            bool ok = true;
            for (int t = cluster; t < total_tiles && ok; t += P2, ++it) {
                const SwapTile st = swap_tile(p, tail, t, rank);
                const uint32_t idesc1 = idesc_mxf4nvf4(256, st.N1);
                const uint32_t idesc2 = idesc_mxf4nvf4(256, st.N2 ? st.N2 : 32);
                if (!mbar_wait(&tail->acc_empty, ((uint32_t)it & 1u) ^ 1u, limit) || tail->abort_flag) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kt = 0; kt < p.num_kt; ++kt) {
                    if (!mbar_wait(&tail->full[stage], phase, limit) ||
                        !mbar_wait(&tail->sf_ready[sb], sph, limit) || tail->abort_flag) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const int nat = min(4, p.num_ks - kt * 4);
                    const uint32_t sA = smem_u32(smem + stage * P::STAGE_BYTES);
                    const uint32_t sB = sA + P::A_BYTES;
                    const uint32_t sB2 = sB + P::B_BYTES;
                    const uint32_t sf = tmem + P::SF_BASE + sb * P::SF_STRIDE;
                    for (int j = 0; j < nat; ++j) {
                        const uint64_t da = sdesc_kmajor_sw128(sA + j * 32);
                        const uint32_t acc = (kt > 0 || j > 0) ? 1u : 0u;
                        mma_mxf4nvf4_pair(tmem, da, sdesc_kmajor_sw128(sB + j * 32), idesc1, sf + j * 4,
                                          sf + 16 + j * NBC, acc);
                        if (st.N2)   // the second part: tokens 256.. (scale columns 8..)
                            mma_mxf4nvf4_pair(tmem + 256, da, sdesc_kmajor_sw128(sB2 + j * 32), idesc2, sf + j * 4,
                                              sf + 16 + j * NBC + 8, acc);
                    }
                    tc_commit_pair(&tail->empty[stage], 0x3);
                    tc_commit_pair(&tail->sf_free[sb], 0x3);
                    if (++stage == STAGES) {
                        stage = 0;
                        phase ^= 1u;
                    }
                    if (++sb == (uint32_t)P::NSB) {
                        sb = 0;
                        sph ^= 1u;
                    }
                }
                if (ok) tc_commit_pair(&tail->acc_full, 0x3);
            }
            if (!ok) {
                tail->abort_flag = 1;
                if (p.err) atomicOr(p.err, 1u);
            }
        }
    } else if (warp >= 2 + P::EPI_WARPS) {
        // ---------------- scale staging (both CTAs; warps 10..13, one lane quarter each) ----------------
        const int q = warp & 3;
        const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16) + P::SF_BASE;
        const uint32_t ready0 = mapa_shared(smem_u32(&tail->sf_ready[0]), 0);
        const uint32_t ready_step = (uint32_t)(smem_u32(&tail->sf_ready[1]) - smem_u32(&tail->sf_ready[0]));
        uint32_t stage = 0, phase = 0, sb = 0, sph = 0;
        bool ok = true;
        for (int t = cluster; t < total_tiles && ok; t += P2) {
            for (int kt = 0; kt < p.num_kt; ++kt) {
                if (!mbar_wait(&tail->sfl[stage], phase, limit) || tail->abort_flag) {
                    ok = false;
                    break;
                }
                const uint32_t sSFA =
                    smem_u32(smem + stage * P::STAGE_BYTES) + P::A_BYTES + P::B_BYTES + P::B2_BYTES;
                const uint32_t sSFB = sSFA + P::SFA_BYTES;
                // one k-tile of scales, in tensor-memory column order: weight
                // k-step j at 4j, token k-step j at 16 + NBC * j (column c =
                // tokens 32c..32c+31; columns past a part's N are not read)
                uint32_t w[P::SF_COLS];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint4 v = ld_shared_v4(sSFA + j * 512 + lane * 16);
                    w[4 * j + 0] = v.x;
                    w[4 * j + 1] = v.y;
                    w[4 * j + 2] = v.z;
                    w[4 * j + 3] = v.w;
                }
#pragma unroll
                for (int j = 0; j < 4; ++j)
#pragma unroll
                    for (int c = 0; c < NBC; ++c) {
                        const int rr = 32 * c + lane;   // token row of the tile
                        const uint32_t addr =
                            sSFB + (uint32_t)((rr >> 7) * 2048 + j * 512 + (rr & 31) * 16 + ((rr >> 5) & 3) * 4);
                        asm volatile("ld.shared.b32 %0, [%1];" : "=r"(w[16 + NBC * j + c]) : "r"(addr));
                    }
                if (!mbar_wait(&tail->sf_free[sb], sph ^ 1u, limit) || tail->abort_flag) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t dst = tq + sb * P::SF_STRIDE;
#pragma unroll
                for (int i = 0; i < (int)P::SF_COLS / 8; ++i) tmem_st_32x32b_x8(dst + 8 * i, w + 8 * i);
                tmem_st_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(ready0 + sb * ready_step);
                if (++stage == STAGES) {
                    stage = 0;
                    phase ^= 1u;
                }
                if (++sb == (uint32_t)P::NSB) {
                    sb = 0;
                    sph ^= 1u;
                }
            }
        }
        if (!ok && lane == 0) {
            tail->abort_flag = 1;
            if (p.err) atomicOr(p.err, 1u);
        }
    } else if (warp >= 2) {
        // ---------------- epilogue (both CTAs; warps 2..9) ----------------
        const int q = warp & 3;                       // tensor-memory lane quarter: weight rows 32q..32q+31
        const int hh = (warp - 2) >> 2;               // this warp's chunks: hh, hh + 2, ...
        const uint32_t empty0 = mapa_shared(smem_u32(&tail->acc_empty), 0);
        const bool odd = lane & 1;
        constexpr int WCH = (P::MAX_CHUNKS + 1) / 2;  // chunks per warp
        int it = 0;
        for (int t = cluster; t < total_tiles; t += P2, ++it) {
            if (!mbar_wait(&tail->acc_full, (uint32_t)it & 1u, limit) || tail->abort_flag) {
                if (lane == 0) {
                    tail->abort_flag = 1;
                    if (p.err) atomicOr(p.err, 1u);
                }
                break;
            }
            tc_fence_after();
            const SwapTile st = swap_tile(p, tail, t, rank);
            const float alpha = __fmul_rn(p.ga[st.e], p.gb[st.e]);
            const uint32_t tq = tmem + ((uint32_t)(q * 32) << 16);
            // chunk c: accumulator columns (tokens) 32c..32c+31; part 1 fills
            // chunks [0, N1 / 32), part 2 chunks [8, 8 + N2 / 32)
            auto live = [&](int c) { return c < (st.N1 >> 5) || (c >= 8 && c < 8 + (st.N2 >> 5)); };
            // all of this warp's chunks to registers as BF16 pairs of
            // neighbouring tokens, then release the accumulators
            uint32_t bf[WCH][16];
#pragma unroll
            for (int ci = 0; ci < WCH; ++ci) {
                const int c = hh + 2 * ci;
                if (live(c)) {   // uniform
                    uint32_t v[32];
                    tmem_ld_32x32b_x32(tq + (uint32_t)(c * 32), v);
                    tmem_ld_wait();
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        bf[ci][i] = pack_bf16x2(__uint_as_float(v[2 * i]) * alpha, __uint_as_float(v[2 * i + 1]) * alpha);
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(empty0);
            // C[tok0 + 32c + i][col + lane]: lanes 2a, 2a + 1 (columns 2a,
            // 2a + 1) swap halves, the even lane keeping even tokens and the
            // odd lane odd ones, each as a BF16 pair of the two columns
            __nv_bfloat16* cbase = p.c + (int64_t)st.tok0 * p.ldc + st.wcol0 + q * 32 + (lane & ~1);
#pragma unroll
            for (int ci = 0; ci < WCH; ++ci) {
                const int c = hh + 2 * ci;
                if (!live(c)) continue;                     // uniform
                const int nt = min(32, st.ntok - 32 * c);   // valid tokens of the chunk
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    const uint32_t own = bf[ci][k];
                    const uint32_t nb = __shfl_xor_sync(0xFFFFFFFFu, own, 1);
                    const uint32_t word = odd ? prmt_b32(nb, own, 0x7632) : prmt_b32(own, nb, 0x5410);
                    const int row = 2 * k + (odd ? 1 : 0);
                    if (row < nt)
                        *reinterpret_cast<uint32_t*>(cbase + (int64_t)(32 * c + row) * p.ldc) = word;
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    cluster_sync();          // no CTA leaves while its peer may still touch its shared memory
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem, kTmemCols);
    }
}

// ---- host side -----------------------------------------------------------------

// 2-D uint8 view [rows, row_bytes] of packed codes, 128-byte x box_rows boxes,
// 128-byte swizzle, zero fill outside the tensor.
bool make_codes_map(CUtensorMap* map, const void* base, int64_t rows, int64_t row_bytes, int box_rows) {
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)row_bytes, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)row_bytes};
    cuuint32_t box[2] = {128u, (cuuint32_t)box_rows};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

template <class C, bool GROUPED, bool EMIT = false, bool MX = false>
nvfp4_status_t launch(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, const GemmArgs& args,
                      int grid, cudaStream_t s) {
    auto kern = gemm_kernel<C, GROUPED, EMIT, MX>;
    static std::atomic<unsigned long long> attr_done{0};
    if (!smem_attr_on_device(reinterpret_cast<const void*>(kern), (int)C::SMEM, attr_done)) return NVFP4_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = C::SMEM;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, ta, tb, tc, args));
}

template <bool GROUPED>
constexpr size_t kPairSmem =
    1024 + (size_t)PairUse::STAGES * PairUse::STAGE_BYTES + PairUse::EPI_BYTES + sizeof(PairTail<PairUse, GROUPED>);
static_assert(kPairSmem<true> <= 232448, "shared memory");

template <bool GROUPED>
cudaLaunchConfig_t pair_config(int clusters, cudaStream_t s, cudaLaunchAttribute (&attr)[2]) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters);
    cfg.blockDim = dim3(PairUse::THREADS);
    cfg.dynamicSmemBytes = kPairSmem<GROUPED>;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cfg;
}

// Number of CTA pairs that can be resident at once (one CTA per SM), per device.
template <bool GROUPED = false>
int pair_clusters_resident() {
    static std::mutex mu;
    static int cached[64] = {};
    int d = -1;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 64) return 0;
    std::lock_guard<std::mutex> lk(mu);
    if (cached[d] == 0) {
        auto kern = gemm_pair_kernel<PairUse, GROUPED>;
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kPairSmem<GROUPED>) !=
            cudaSuccess)
            return 0;
        cudaLaunchAttribute attr[2];
        cudaLaunchConfig_t cfg = pair_config<GROUPED>(1, nullptr, attr);
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n <= 0) return 0;
        cached[d] = n;
    }
    return cached[d];
}

// How the pair kernel covers an m x n x k product: resident pairs, whole
// tiles, and the stream-K k-tiles of the rest (0 when the tiles fill whole
// waves, or a tile has a single k-tile and cannot be split).
struct PairPlan {
    int clusters = 0;
    int64_t tiles = 0;
    int dp_tiles = 0;
    int64_t sk_units = 0;
};

bool pair_plan(int64_t m, int64_t n, int64_t k, PairPlan& pl) {
    if (m <= 128) return false;
    const int clusters_max = pair_clusters_resident();
    const int sms = num_sms();
    if (clusters_max <= 0 || sms < 2) return false;
    const int64_t tiles = ((m + 255) / 256) * ((n + PairUse::BN - 1) / PairUse::BN);
    if (tiles >= ((int64_t)1 << 31)) return false;
    pl.tiles = tiles;
    pl.clusters = (int)std::min<int64_t>(tiles, std::min(clusters_max, sms / 2));
    const int64_t num_kt = (k / 64 + 3) / 4;
    const int64_t P = pl.clusters;
    if (tiles > P && tiles % P != 0 && num_kt > 1 && P <= 256 && (2 * P) * num_kt < ((int64_t)1 << 31)) {
        pl.dp_tiles = (int)((tiles / P - 1) * P);
        pl.sk_units = (tiles - pl.dp_tiles) * num_kt;
    } else {
        pl.dp_tiles = (int)tiles;
        pl.sk_units = 0;
    }
    return true;
}

// Workspace of the stream-K tail: the counters (one 64-byte line per CTA),
// then one FP32 128 x BN slot per CTA.
constexpr size_t kSkFlagsBytes = 256 * 2 * kSkFlagStride * sizeof(uint32_t);   // up to 256 pairs
size_t sk_workspace_bytes(int clusters) {
    return kSkFlagsBytes + (size_t)clusters * 2 * 128 * PairUse::BN * sizeof(float);
}

template <bool GROUPED = false, bool EMIT = false, bool MX = false>
nvfp4_status_t launch_pair(const CUtensorMap& ta, const CUtensorMap& tb, const CUtensorMap& tc, const GemmArgs& args,
                           int clusters, cudaStream_t s) {
    auto kern = gemm_pair_kernel<PairUse, GROUPED, EMIT, MX>;
    static std::atomic<unsigned long long> attr_done{0};
    if (!smem_attr_on_device(reinterpret_cast<const void*>(kern), (int)kPairSmem<GROUPED>, attr_done))
        return NVFP4_ERR_CUDA;
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = pair_config<GROUPED>(clusters, s, attr);
    return cuda_status(cudaLaunchKernelEx(&cfg, kern, ta, tb, tc, args));
}

// Kernel configurations: 64 < m <= 128 and the grouped form use 128 x 192
// tiles with two accumulator buffers (2 x 192 + 2 x 48 scale columns of
// tensor memory).
using CfgWide = Cfg<192, 4, 2>;
// Decode (m <= 64): the tokens stay on the 128-row MMA side (the MMA work is
// free in this weight-bound regime) but only 64 rows of them are loaded per
// stage -- the MMA's rows 64..127 read the stage's other bytes and those
// accumulator rows are never stored -- which leaves room for a fifth stage of
// weights in flight.  Weights take the 192-wide side: 134 tiles for n = 25600,
// one wave on 148 SMs (measured: 21-23 us for m = 1..64 against 29-36 us with
// the weights on the 128-row side in 200 tiles).
using CfgDecW = Cfg<192, 5, 2, 2, 64>;

// BF16 [rows, cols] output with row stride ldc elements, 32 x 32 boxes,
// 64-byte swizzle (matches the epilogue's staging layout).
bool make_out_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ldc) {
    auto fn = tensor_map_encoder();
    if (!fn) return false;
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)(ldc * 2)};
    cuuint32_t box[2] = {32u, 32u};
    cuuint32_t estr[2] = {1u, 1u};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

bool ptr_ok(const void* p) { return p && aligned16(p); }

}  // namespace

size_t gemm_workspace_bytes(int64_t m, int64_t n, int64_t k) {
    PairPlan pl;
    if (m <= 0 || n <= 0 || k <= 0 || !pair_plan(m, n, k, pl) || pl.sk_units == 0) return 0;
    return sk_workspace_bytes(pl.clusters);
}
}  // namespace nvfp4

using namespace nvfp4;

namespace nvfp4 {
namespace {
__global__ void set_one_kernel(float* g) { g[0] = 1.0f; }

// The dense GEMM.  c_amax / c_gscale (optional): also fold max |C| and write
// the global scale of C for the next quantizer (see nvfp4_gemm_emit_scale).
// mx: MXFP4 operands (E8M0 scales per 32 elements, no global scales; the
// global-scale pointers are ignored and c_amax must be NULL).
nvfp4_status_t gemm_impl(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global,
                         const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global, void* c, int64_t ldc,
                         int64_t m, int64_t n, int64_t k, void* workspace, uint32_t* c_amax, float* c_gscale,
                         void* stream, bool mx = false, bool b_early = false) {
    if (m < 0 || n <= 0 || k <= 0 || ldc < n) return NVFP4_ERR_INVALID_ARGUMENT;
    if (k % 64 != 0 || m >= ((int64_t)1 << 31) || n >= ((int64_t)1 << 31) || k >= ((int64_t)1 << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (m == 0) {   // nothing to read or write (the operand pointers may be NULL)
        if (c_gscale) {   // an empty C: amax 0, global scale 1
            set_one_kernel<<<1, 1, 0, s>>>(c_gscale);
            return cuda_status(cudaGetLastError());
        }
        return NVFP4_OK;
    }
    if (mx) {
        a_global = b_global = nullptr;
        if (c_amax) return NVFP4_ERR_INVALID_ARGUMENT;
    } else if (!a_global || !b_global) {
        return NVFP4_ERR_INVALID_ARGUMENT;
    }
    if (!a_codes || !a_scales || !b_codes || !b_scales || !c) return NVFP4_ERR_INVALID_ARGUMENT;
    if (!ptr_ok(a_codes) || !ptr_ok(a_scales) || !ptr_ok(b_codes) || !ptr_ok(b_scales) || !ptr_ok(c) ||
        (reinterpret_cast<uintptr_t>(a_global) & 3u) || (reinterpret_cast<uintptr_t>(b_global) & 3u) || ldc % 8 != 0)
        return NVFP4_ERR_MISALIGNED;
    if (reinterpret_cast<uintptr_t>(workspace) & 15u) return NVFP4_ERR_MISALIGNED;
    const int sms = num_sms();
    if (sms <= 0) return NVFP4_ERR_NO_DEVICE;
    // scale bytes per 128-row block: 128 rows x (k/16 or k/32 rounded up to 4) columns
    const int64_t sf_rb_stride = mx ? 128 * round_up(k / 32, 4) : 128 * (k / 16);
    GemmArgs p = {};
    p.c_amax = c_amax;
    p.c_gscale = c_gscale;
    p.num_ks = (int)(k / 64);
    p.num_kt = (p.num_ks + 3) / 4;
    p.c = reinterpret_cast<__nv_bfloat16*>(c);
    p.ldc = ldc;
    p.sfa_rb_stride = sf_rb_stride;
    p.sfb_rb_stride = sf_rb_stride;
    p.sfb_group_stride = 0;
    p.offsets = nullptr;
    p.num_groups = 1;
    p.wait_limit_ns = wait_limit_ns();
    p.err = device_error_word();
    if (!p.err) return NVFP4_ERR_CUDA;
    CUtensorMap ta, tb, tc;
    if (m <= 64) {
        if (!make_codes_map(&ta, a_codes, m, k / 2, CfgDecW::AROWS) ||
            !make_codes_map(&tb, b_codes, n, k / 2, CfgDecW::BN) || !make_out_map(&tc, c, m, n, ldc))
            return NVFP4_ERR_CUDA;
        p.sfa = a_scales;
        p.sfb = b_scales;
        p.sfb_rb_per_group = (int)((n + 127) / 128);
        p.ga = a_global;
        p.gb = b_global;
        p.rows_a = (int)m;
        p.rows_b = (int)n;
        p.tiles_m = 1;
        p.tiles_n = (int)((n + CfgDecW::BN - 1) / CfgDecW::BN);
        p.b_early = b_early ? 1 : 0;
        const int grid = (int)std::min<int64_t>((int64_t)p.tiles_n, sms);
        if (mx) return launch<CfgDecW, false, false, true>(ta, tb, tc, p, grid, s);
        return c_amax ? launch<CfgDecW, false, true>(ta, tb, tc, p, grid, s) : launch<CfgDecW, false>(ta, tb, tc, p, grid, s);
    }
    PairPlan pl;
    if (pair_plan(m, n, k, pl)) {
        // prefill-class: 2-SM pair tiles of 256 x 256, stream-K over the last waves
        if (!make_codes_map(&ta, a_codes, m, k / 2, 128) ||
            !make_codes_map(&tb, b_codes, n, k / 2, PairUse::BH) || !make_out_map(&tc, c, m, n, ldc))
            return NVFP4_ERR_CUDA;
        p.sfa = a_scales;
        p.sfb = b_scales;
        p.sfb_rb_per_group = (int)((n + 127) / 128);
        p.ga = a_global;
        p.gb = b_global;
        p.rows_a = (int)m;
        p.rows_b = (int)n;
        p.tiles_m = (int)((m + 255) / 256);
        p.tiles_n = (int)((n + PairUse::BN - 1) / PairUse::BN);
        // without a workspace every tile stays whole
        const bool sk = pl.sk_units > 0 && workspace != nullptr;
        p.dp_tiles = sk ? pl.dp_tiles : (int)pl.tiles;
        p.sk_units = sk ? pl.sk_units : 0;
        p.sk_flags = sk ? reinterpret_cast<uint32_t*>(workspace) : nullptr;
        p.pdl_trigger = 1;
        p.partial = sk ? reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(workspace) + kSkFlagsBytes) : nullptr;
        if (mx) return launch_pair<false, false, true>(ta, tb, tc, p, pl.clusters, s);
        return c_amax ? launch_pair<false, true>(ta, tb, tc, p, pl.clusters, s)
                      : launch_pair<false>(ta, tb, tc, p, pl.clusters, s);
    }
    constexpr int BN = CfgWide::BN;
    if (!make_codes_map(&ta, a_codes, m, k / 2, 128) || !make_codes_map(&tb, b_codes, n, k / 2, BN) ||
        !make_out_map(&tc, c, m, n, ldc))
        return NVFP4_ERR_CUDA;
    p.sfa = a_scales;
    p.sfb = b_scales;
    p.sfb_rb_per_group = (int)((n + 127) / 128);
    p.ga = a_global;
    p.gb = b_global;
    p.rows_a = (int)m;
    p.rows_b = (int)n;
    p.tiles_m = (int)((m + 127) / 128);
    p.tiles_n = (int)((n + BN - 1) / BN);
    const int64_t tiles = (int64_t)p.tiles_m * p.tiles_n;
    if (tiles >= ((int64_t)1 << 31)) return NVFP4_ERR_UNSUPPORTED_SHAPE;
    p.pdl_trigger = 1;
    const int grid = (int)std::min<int64_t>(tiles, sms);
    if (mx) return launch<CfgWide, false, false, true>(ta, tb, tc, p, grid, s);
    return c_amax ? launch<CfgWide, false, true>(ta, tb, tc, p, grid, s) : launch<CfgWide, false>(ta, tb, tc, p, grid, s);
}
}  // namespace
}  // namespace nvfp4

extern "C" nvfp4_status_t nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global,
                                     const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global, void* c,
                                     int64_t ldc, int64_t m, int64_t n, int64_t k, void* workspace, void* stream) {
    return gemm_impl(a_codes, a_scales, a_global, b_codes, b_scales, b_global, c, ldc, m, n, k, workspace, nullptr,
                     nullptr, stream);
}

extern "C" nvfp4_status_t mxfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const uint8_t* b_codes,
                                     const uint8_t* b_scales, void* c, int64_t ldc, int64_t m, int64_t n, int64_t k,
                                     void* workspace, void* stream) {
    return gemm_impl(a_codes, a_scales, nullptr, b_codes, b_scales, nullptr, c, ldc, m, n, k, workspace, nullptr,
                     nullptr, stream, true);
}

extern "C" nvfp4_status_t nvfp4_gemm_emit_scale(const uint8_t* a_codes, const uint8_t* a_scales,
                                                const float* a_global, const uint8_t* b_codes,
                                                const uint8_t* b_scales, const float* b_global, void* c, int64_t ldc,
                                                int64_t m, int64_t n, int64_t k, float* c_global_scale,
                                                void* workspace, void* stream) {
    if (!c_global_scale || !workspace) return NVFP4_ERR_INVALID_ARGUMENT;
    if ((reinterpret_cast<uintptr_t>(c_global_scale) & 3u) || (reinterpret_cast<uintptr_t>(workspace) & 15u))
        return NVFP4_ERR_MISALIGNED;
    uint8_t* ws = reinterpret_cast<uint8_t*>(workspace);
    return gemm_impl(a_codes, a_scales, a_global, b_codes, b_scales, b_global, c, ldc, m, n, k,
                     ws + kEmitScaleWsBytes, reinterpret_cast<uint32_t*>(ws), c_global_scale, stream);
}

namespace nvfp4 {
namespace {
cudaLaunchConfig_t swap_config(int clusters, cudaStream_t s, cudaLaunchAttribute (&attr)[2]) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * clusters);
    cfg.blockDim = dim3(SwapCfg::THREADS);
    cfg.dynamicSmemBytes = kSwapSmem;
    cfg.stream = s;
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cfg;
}
// Pairs of moe_swap_kernel that can be resident at once, per device (0: unavailable).
int swap_clusters_resident() {
    static std::mutex mu;
    static int cached[64] = {};
    int d = -1;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= 64) return 0;
    std::lock_guard<std::mutex> lk(mu);
    if (cached[d] == 0) {
        if (cudaFuncSetAttribute(moe_swap_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSwapSmem) !=
            cudaSuccess)
            return 0;
        cudaLaunchAttribute attr[2];
        cudaLaunchConfig_t cfg = swap_config(1, nullptr, attr);
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, moe_swap_kernel, &cfg) != cudaSuccess || n <= 0) return 0;
        cached[d] = n;
    }
    return cached[d];
}
nvfp4_status_t launch_swap(const CUtensorMap& tw, const SwapMaps& tx, const CUtensorMap& tc, const GemmArgs& args,
                           int clusters, cudaStream_t s) {
    static std::atomic<unsigned long long> attr_done{0};
    if (!smem_attr_on_device(reinterpret_cast<const void*>(moe_swap_kernel), (int)kSwapSmem, attr_done))
        return NVFP4_ERR_CUDA;
    cudaLaunchAttribute attr[2];
    cudaLaunchConfig_t cfg = swap_config(clusters, s, attr);
    return cuda_status(cudaLaunchKernelEx(&cfg, moe_swap_kernel, tw, tx, tc, args));
}
}  // namespace
}  // namespace nvfp4

extern "C" nvfp4_status_t nvfp4_grouped_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global,
                                             const int32_t* offsets, int num_experts, const uint8_t* b_codes,
                                             const uint8_t* b_scales, const float* b_global, void* c, int64_t n,
                                             int64_t k, int64_t total_rows, void* workspace, void* stream) {
    (void)workspace;
    if (num_experts < 1 || n <= 0 || k <= 0 || total_rows < 0) return NVFP4_ERR_INVALID_ARGUMENT;
    if (!a_codes || !a_scales || !a_global || !offsets || !b_codes || !b_scales || !b_global || !c)
        return NVFP4_ERR_INVALID_ARGUMENT;
    if (k % 64 != 0 || num_experts > kMaxGroups || total_rows >= ((int64_t)1 << 31) ||
        n * (int64_t)num_experts >= ((int64_t)1 << 31) || k >= ((int64_t)1 << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!ptr_ok(a_codes) || !ptr_ok(a_scales) || !ptr_ok(b_codes) || !ptr_ok(b_scales) || !ptr_ok(c) ||
        (reinterpret_cast<uintptr_t>(a_global) & 3u) || (reinterpret_cast<uintptr_t>(b_global) & 3u) ||
        (reinterpret_cast<uintptr_t>(offsets) & 3u) || n % 8 != 0)
        return NVFP4_ERR_MISALIGNED;
    if (total_rows == 0) return NVFP4_OK;
    const int sms = num_sms();
    if (sms <= 0) return NVFP4_ERR_NO_DEVICE;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    constexpr int BN = CfgWide::BN;
    const int64_t sf_rb_stride = 128 * (k / 16);
    GemmArgs p = {};
    p.num_ks = (int)(k / 64);
    p.num_kt = (p.num_ks + 3) / 4;
    p.c = reinterpret_cast<__nv_bfloat16*>(c);
    p.ldc = n;
    p.sfa = a_scales;
    p.sfa_rb_stride = sf_rb_stride;
    p.sfb = b_scales;
    p.sfb_rb_stride = sf_rb_stride;
    p.sfb_group_stride = (int64_t)nvfp4_scale_bytes(n, k);
    p.sfb_rb_per_group = (int)((n + 127) / 128);
    p.ga = a_global;
    p.gb = b_global;
    p.rows_a = (int)total_rows;
    p.rows_b = (int)n;
    p.tiles_m = 0;
    p.tiles_n = (int)((n + BN - 1) / BN);
    p.offsets = offsets;
    p.num_groups = num_experts;
    p.wait_limit_ns = wait_limit_ns();
    p.err = device_error_word();
    if (!p.err) return NVFP4_ERR_CUDA;
    CUtensorMap ta, tb, tc;
    // Weights in whole 256-row tiles: the swapped kernel (weights on the
    // 256-row MMA side, each expert's tokens on N, padded to 32 at most).
    const int swap_max = swap_clusters_resident();
    if (n % 256 == 0 && swap_max > 0 && sms >= 2) {
        SwapMaps tx;
        if (!make_codes_map(&tb, b_codes, n * num_experts, k / 2, 128) || !make_out_map(&tc, c, total_rows, n, n))
            return NVFP4_ERR_CUDA;
        for (int i = 0; i < SwapCfg::NUM_BOXES; ++i)
            if (!make_codes_map(&tx.x[i], a_codes, total_rows, k / 2, 16 << i)) return NVFP4_ERR_CUDA;
        // upper bound of the tile count: sum_e ceil(n_e / 256) <= total_rows / 256 + num_experts
        const int64_t max_tiles = (total_rows / 256 + num_experts) * (n / 256);
        const int clusters = (int)std::min<int64_t>(max_tiles, std::min(swap_max, sms / 2));
        return launch_swap(tb, tx, tc, p, clusters, s);
    }
    // Experts of 192 rows or more on average (prefill-sized MoE): 256 x 256
    // pair tiles, every tile whole; smaller groups would mostly pad a 256-row
    // tile, so they take the 128 x 192 single-SM tiles.
    const int clusters_max = pair_clusters_resident<true>();
    if (clusters_max > 0 && sms >= 2 && total_rows >= 192 * (int64_t)num_experts) {
        if (!make_codes_map(&ta, a_codes, total_rows, k / 2, 128) ||
            !make_codes_map(&tb, b_codes, n * num_experts, k / 2, PairUse::BH) ||
            !make_out_map(&tc, c, total_rows, n, n))
            return NVFP4_ERR_CUDA;
        p.tiles_n = (int)((n + PairUse::BN - 1) / PairUse::BN);
        p.dp_tiles = 0;
        p.sk_units = 0;
        // upper bound of the tile count: sum_e ceil(n_e / 256) <= total_rows / 256 + num_experts
        const int64_t max_tiles = (total_rows / 256 + num_experts) * (int64_t)p.tiles_n;
        const int clusters = (int)std::min<int64_t>(max_tiles, std::min(clusters_max, sms / 2));
        return launch_pair<true>(ta, tb, tc, p, clusters, s);
    }
    if (!make_codes_map(&ta, a_codes, total_rows, k / 2, 128) ||
        !make_codes_map(&tb, b_codes, n * num_experts, k / 2, BN) || !make_out_map(&tc, c, total_rows, n, n))
        return NVFP4_ERR_CUDA;
    // upper bound of the tile count: sum_e ceil(n_e / 128) <= total_rows / 128 + num_experts
    const int64_t max_tiles = (total_rows / 128 + num_experts) * (int64_t)p.tiles_n;
    const int grid = (int)std::min<int64_t>(max_tiles, sms);
    return launch<CfgWide, true>(ta, tb, tc, p, grid, s);
}

// Dynamic activation quantization followed by the GEMM, in one call.  For
// decode-sized activations (m <= 64) the quantizer runs as the two-kernel
// form, whose small CTAs leave room on every SM, and the GEMM is launched as
// its programmatic dependent with b_early: its CTAs start streaming the
// weights (which no kernel of this call writes) while the activations are
// still being quantized, and wait only before reading them.  Larger m: the
// one-launch quantizer, then the GEMM.
extern "C" nvfp4_status_t nvfp4_quantize_gemm(const void* x, int64_t m, int64_t k, int64_t ldx, const uint8_t* b_codes,
                                              const uint8_t* b_scales, const float* b_global, int64_t n, void* c,
                                              int64_t ldc, uint8_t* a_codes, uint8_t* a_scales, float* a_global,
                                              void* workspace, void* stream) {
    if (m < 0 || n <= 0 || k <= 0 || ldx < k || ldc < n) return NVFP4_ERR_INVALID_ARGUMENT;
    if (m == 0) return NVFP4_OK;
    if (!x || !b_codes || !b_scales || !b_global || !c || !a_codes || !a_scales || !a_global || !workspace)
        return NVFP4_ERR_INVALID_ARGUMENT;
    if (k % 64 != 0 || m >= ((int64_t)1 << 31) || n >= ((int64_t)1 << 31) || k >= ((int64_t)1 << 31))
        return NVFP4_ERR_UNSUPPORTED_SHAPE;
    if (!ptr_ok(x) || !ptr_ok(workspace) || ldx % 8 != 0) return NVFP4_ERR_MISALIGNED;
    uint8_t* gemm_ws = reinterpret_cast<uint8_t*>(workspace) + quant_ws_bytes(1);
    if (m > 64) {
        const nvfp4_status_t st =
            nvfp4_quantize_act(x, m, k, ldx, nullptr, 0, a_codes, a_scales, a_global, workspace, stream);
        if (st != NVFP4_OK) return st;
        return nvfp4_gemm(a_codes, a_scales, a_global, b_codes, b_scales, b_global, c, ldc, m, n, k,
                          gemm_workspace_bytes(m, n, k) ? gemm_ws : nullptr, stream);
    }
    // argument checks of both halves before anything is launched
    if (!ptr_ok(a_codes) || !ptr_ok(a_scales) || !ptr_ok(b_codes) || !ptr_ok(b_scales) || !ptr_ok(c) ||
        (reinterpret_cast<uintptr_t>(a_global) & 3u) || (reinterpret_cast<uintptr_t>(b_global) & 3u) || ldc % 8 != 0)
        return NVFP4_ERR_MISALIGNED;
    if (num_sms() <= 0) return NVFP4_ERR_NO_DEVICE;
    const nvfp4_status_t st = run_two_kernel(reinterpret_cast<const uint16_t*>(x), m, k, ldx, nullptr, 1, a_codes,
                                             a_scales, a_global, workspace, reinterpret_cast<cudaStream_t>(stream));
    if (st != NVFP4_OK) return st;
    return gemm_impl(a_codes, a_scales, a_global, b_codes, b_scales, b_global, c, ldc, m, n, k, nullptr, nullptr,
                     nullptr, stream, false, true);
}
