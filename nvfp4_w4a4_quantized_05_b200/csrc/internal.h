// internal.h -- host-side helpers shared by the translation units of libnvfp4.
#pragma once

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>
#include <atomic>
#include <cstdint>

#include "../../include/nvfp4.h"

namespace nvfp4 {

// Device address of this library's error word on the current device
// (nonzero after a bounded wait in a kernel ran out).  nullptr on failure.
unsigned int* device_error_word();

// Number of SMs of the current device (cached per device).
int num_sms();

// The driver's cuTensorMapEncodeTiled (looked up once), or nullptr.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder();
// Scratch bytes nvfp4_gemm wants for an m x n x k product on the current
// device (the stream-K tail of the pair kernel); 0 when it needs none.
size_t gemm_workspace_bytes(int64_t m, int64_t n, int64_t k);
// nvfp4_gemm_emit_scale's workspace: its output-amax words first, then the
// plain GEMM's workspace.
constexpr int64_t kEmitScaleWsBytes = 256;

// Raises a kernel's dynamic shared-memory limit to `bytes` on the current
// device, once per device (the attribute belongs to the device's context);
// `done` holds one bit per device.  False if the runtime refuses it.
inline bool smem_attr_on_device(const void* kernel, int bytes, std::atomic<unsigned long long>& done) {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
    const unsigned long long bit = 1ull << dev;
    if (done.load(std::memory_order_acquire) & bit) return true;
    if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) != cudaSuccess) return false;
    done.fetch_or(bit, std::memory_order_acq_rel);
    return true;
}

// Current limit of the bounded waits, in ns.
uint64_t wait_limit_ns();

// Dynamic 1D quantization of one tensor (offsets == nullptr, groups == 1) or of
// row groups by the two-kernel form: the amax kernel, then the quantize kernel
// as its programmatic dependent.  Arguments as nvfp4_quantize_act, already
// checked by the caller.
nvfp4_status_t run_two_kernel(const uint16_t* x, int64_t rows, int64_t k, int64_t ld, const int32_t* group_offsets,
                              int groups, uint8_t* codes, uint8_t* scales, float* global_scale, void* workspace,
                              cudaStream_t s);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

inline nvfp4_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

// Workspace layout of the quantizers (bytes); G = number of row groups:
//   [0, 128 * kMaxFusedCtas)  one-launch path: the word of CTA c at 128 c,
//                  generation << 32 (uint64, one per 128-byte line): the
//                  generation of the CTA's last call.  At a fixed place, so
//                  that every call on the workspace, with or without groups,
//                  steps the same generation count.
//   [B, B + 128)   one-launch path, grid barrier (B = quant_ws_bar_off()):
//                  word 0 counts CTA arrivals (uint32, one per CTA per call,
//                  never reset: all CTAs of call gen have arrived when it
//                  reads gen * grid size); words 1 and 2 hold the tensor
//                  amax of calls with even and odd generation (FP32 bits,
//                  folded with atomicMax; each call zeroes the other one for
//                  the next call).
//   [T, T + 4)     two-kernel path: CTA completion counter (uint32), T = quant_ws_two_off()
//   [T + 16, T + 16 + 4G)  two-kernel path: per-group amax as FP32 bit patterns (uint32)
//   [pad_off, +4(G+1))     per-group first scale row (int32), written each call
//   [gword_off, +8G)       one-launch grouped path: per-group generation << 32 | amax bits (uint64)
constexpr int kMaxFusedCtas = 256;
constexpr int kPartStrideWords = 16;   // uint64 words: 128 bytes
constexpr int64_t quant_ws_bar_off() { return 128 * (int64_t)kMaxFusedCtas; }
constexpr int64_t quant_ws_two_off() { return quant_ws_bar_off() + 128; }
constexpr int64_t quant_ws_pad_off(int groups) { return round_up(quant_ws_two_off() + 16 + 4 * (int64_t)groups, 16); }
constexpr int64_t quant_ws_gword_off(int groups) {
    return round_up(quant_ws_pad_off(groups) + 4 * ((int64_t)groups + 1), 128);
}
constexpr int64_t quant_ws_bytes(int groups) { return round_up(quant_ws_gword_off(groups) + 8 * (int64_t)groups, 256); }

}  // namespace nvfp4
