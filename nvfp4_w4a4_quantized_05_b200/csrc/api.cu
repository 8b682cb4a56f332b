// api.cu -- size helpers, status reporting and diagnostics of libnvfp4.
#include <cuda_runtime.h>
#include <atomic>
#include <cstdint>
#include <mutex>

#include "internal.h"
#include "ptx.cuh"

namespace nvfp4 {

// Set (atomicOr) by any kernel of this library whose bounded wait ran out.
__device__ unsigned int g_device_error;

namespace {
constexpr int kMaxDevices = 64;
std::mutex g_mu;
unsigned int* g_err_ptr[kMaxDevices] = {};
int g_sms[kMaxDevices] = {};
std::atomic<uint64_t> g_wait_limit_ns{2000000000ull};

int current_device() {
    int d = -1;
    if (cudaGetDevice(&d) != cudaSuccess || d < 0 || d >= kMaxDevices) return -1;
    return d;
}

__global__ void bounded_wait_probe_kernel(const volatile uint32_t* flag, uint64_t limit_ns, unsigned int* err) {
    const uint64_t t0 = globaltimer_ns();
    while (*flag == 0u) {
        if (globaltimer_ns() - t0 > limit_ns) {
            atomicOr(err, 1u);
            return;
        }
        __nanosleep(1000);
    }
}
}  // namespace

unsigned int* device_error_word() {
    const int d = current_device();
    if (d < 0) return nullptr;
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_err_ptr[d]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        g_err_ptr[d] = reinterpret_cast<unsigned int*>(p);
    }
    return g_err_ptr[d];
}

int num_sms() {
    const int d = current_device();
    if (d < 0) return 0;
    std::lock_guard<std::mutex> lk(g_mu);
    if (g_sms[d] == 0) {
        int major = 0, sms = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, d) != cudaSuccess || major != 10)
            return 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, d) != cudaSuccess) return 0;
        g_sms[d] = sms;
    }
    return g_sms[d];
}

uint64_t wait_limit_ns() { return g_wait_limit_ns.load(); }

PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    });
    return fn;
}

}  // namespace nvfp4

using namespace nvfp4;

extern "C" const char* nvfp4_status_string(nvfp4_status_t s) {
    switch (s) {
        case NVFP4_OK: return "ok";
        case NVFP4_ERR_INVALID_ARGUMENT: return "invalid argument";
        case NVFP4_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case NVFP4_ERR_MISALIGNED: return "misaligned pointer or leading dimension";
        case NVFP4_ERR_CUDA: return "CUDA runtime error";
        case NVFP4_ERR_TIMEOUT: return "device wait timed out";
        case NVFP4_ERR_NO_DEVICE: return "no sm_100 device";
    }
    return "unknown status";
}

extern "C" const char* nvfp4_version(void) { return "0.1.0"; }

extern "C" size_t nvfp4_codes_bytes(int64_t rows, int64_t k) {
    if (rows < 0 || k < 0) return 0;
    return (size_t)(rows * (k / 2));
}

extern "C" size_t nvfp4_scale_bytes(int64_t rows, int64_t k) {
    if (rows < 0 || k < 0) return 0;
    return (size_t)(round_up(rows, 128) * round_up(k / 16, 4));
}

extern "C" size_t mxfp4_scale_bytes(int64_t rows, int64_t k) {
    if (rows < 0 || k < 0) return 0;
    return (size_t)(round_up(rows, 128) * round_up(k / 32, 4));
}

extern "C" size_t nvfp4_grouped_scale_bytes(int64_t total_rows, int num_groups, int64_t k) {
    if (total_rows < 0 || num_groups < 1 || k < 0) return 0;
    return (size_t)(((total_rows + 127 * (int64_t)num_groups) / 128) * 128 * round_up(k / 16, 4));
}

extern "C" size_t nvfp4_workspace_bytes(int op, int64_t rows, int64_t n, int64_t k, int num_groups) {
    switch (op) {
        case NVFP4_OP_QUANTIZE_ACT: return (size_t)quant_ws_bytes(num_groups > 1 ? num_groups : 1);
        case NVFP4_OP_QUANTIZE_WEIGHT_2D: return (size_t)quant_ws_bytes(1);
        case NVFP4_OP_GEMM: return gemm_workspace_bytes(rows, n, k);
        case NVFP4_OP_GEMM_EMIT_SCALE: return (size_t)kEmitScaleWsBytes + gemm_workspace_bytes(rows, n, k);
        case NVFP4_OP_GROUPED_GEMM: return 0;
        case NVFP4_OP_QUANTIZE_GEMM: return (size_t)quant_ws_bytes(1) + gemm_workspace_bytes(rows, n, k);
    }
    return 0;
}

extern "C" nvfp4_status_t nvfp4_workspace_init(void* workspace, size_t bytes, void* stream) {
    if (!workspace && bytes) return NVFP4_ERR_INVALID_ARGUMENT;
    if (!bytes) return NVFP4_OK;
    return cuda_status(cudaMemsetAsync(workspace, 0, bytes, reinterpret_cast<cudaStream_t>(stream)));
}

extern "C" nvfp4_status_t nvfp4_get_last_device_error(void* stream) {
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    if (cudaStreamSynchronize(s) != cudaSuccess) return NVFP4_ERR_CUDA;
    unsigned int* w = device_error_word();
    if (!w) return NVFP4_ERR_CUDA;
    unsigned int v = 0;
    if (cudaMemcpy(&v, w, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (v) {
        const unsigned int zero = 0;
        if (cudaMemcpy(w, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return NVFP4_ERR_CUDA;
        return NVFP4_ERR_TIMEOUT;
    }
    return NVFP4_OK;
}

extern "C" uint64_t nvfp4_set_wait_limit_ns(uint64_t limit_ns) {
    if (limit_ns == 0) limit_ns = 1;
    return g_wait_limit_ns.exchange(limit_ns);
}

extern "C" nvfp4_status_t nvfp4_probe_bounded_wait(const uint32_t* flag, uint64_t limit_ns, void* stream) {
    if (!flag) return NVFP4_ERR_INVALID_ARGUMENT;
    if (!aligned16(flag)) return NVFP4_ERR_MISALIGNED;
    if (limit_ns > 10000000000ull) return NVFP4_ERR_INVALID_ARGUMENT;   // at most 10 s
    if (num_sms() <= 0) return NVFP4_ERR_NO_DEVICE;
    unsigned int* err = device_error_word();
    if (!err) return NVFP4_ERR_CUDA;
    bounded_wait_probe_kernel<<<1, 1, 0, reinterpret_cast<cudaStream_t>(stream)>>>(flag, limit_ns, err);
    return cuda_status(cudaGetLastError());
}
