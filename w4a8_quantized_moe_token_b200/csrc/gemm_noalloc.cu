// w4a8_gemm_noalloc: the dense W4A8 GEMM for callers that cannot allocate.
//
// w4a8_gemm needs a small device workspace from its caller (the INT8 rows copied
// into the tensor-core tile layout, plus a few words of metadata).  Some callers
// have no way to provide one: a plugin running inside a host framework that owns
// every device allocation and forbids new ones on its execution path, code that
// runs where a cudaMalloc would synchronise the device or is not permitted (for
// example between the steps of a latency-critical loop driven by another runtime),
// or a caller written in a language binding with no allocator at hand.  For them
// this file keeps the scratch in a fixed, file-scope device array and calls the
// regular entry point with it.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/w4a8.h"
#include "w4a8_common.cuh"

#define W4A8_EXPORT extern "C" __attribute__((visibility("default")))

namespace w4a8 {
namespace {

// 8 MiB, reserved on every GPU that loads the library, for as long as the process
// runs.  Enough for M x Kp up to about 8.3 million INT8 values (for example M = 1024
// tokens at K = 7168).
constexpr size_t kNoAllocScratchBytes = 8u << 20;
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

// Device address of the scratch array on the current device.  The name of a
// __device__ array in host code is only a host-side stand-in, so the address is
// looked up once per device (with that device current) and cached.
int scratch_address(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return W4A8_ECUDA;
    if (dev < 0 || dev >= kMaxDevices) return W4A8_EUNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_mu);
    if (g_scratch_ptr[dev] == nullptr) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return W4A8_ECUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return W4A8_OK;
}

}  // namespace
}  // namespace w4a8

W4A8_EXPORT int w4a8_gemm_noalloc(const int8_t* qa, const float* sa, int M, const void* packed, int N, int K,
                                  float* y, int32_t* partials_opt, void* stream) {
    const size_t need = w4a8_gemm_workspace_bytes(M, N, K);
    if (need == 0) return W4A8_EINVAL;
    if (need > w4a8::kNoAllocScratchBytes) return W4A8_ENOSPACE;
    void* scratch = nullptr;
    const int r = w4a8::scratch_address(&scratch);
    if (r != W4A8_OK) return r;
    return w4a8_gemm(qa, sa, M, packed, N, K, y, partials_opt, scratch, w4a8::kNoAllocScratchBytes, stream);
}

W4A8_EXPORT int w4a8_gemm_noalloc_last_error(void* stream) {
    void* scratch = nullptr;
    const int r = w4a8::scratch_address(&scratch);
    if (r != W4A8_OK) return r;
    // the dense GEMM keeps its device error word in the first bytes of its workspace
    return w4a8_last_device_error(scratch, stream);
}
