// fa_backward_noalloc: the backward pass with its scratch in a static device
// array, for callers that cannot allocate device memory (see include/fa.h).
// The kernels are those of fa_backward; only where the per-row statistic D
// lives differs.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "fa_internal.h"

namespace fa {
namespace {

// Scratch for D_i = rowsum(dO o O): one float per query row, FA_NOALLOC_MAX_ROWS rows.
static __device__ __align__(256) float g_bwd_noalloc_scratch[FA_NOALLOC_MAX_ROWS];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
float* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up once
// per device with that device current, and then passed to the kernels.
int scratch_for_current_device(float** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* ptr = nullptr;
        if (cudaGetSymbolAddress(&ptr, g_bwd_noalloc_scratch) != cudaSuccess || ptr == nullptr) return FA_ERR_CUDA;
        g_scratch_ptr[dev] = static_cast<float*>(ptr);
    }
    *out = g_scratch_ptr[dev];
    return FA_OK;
}

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" int fa_backward_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                   const float* lse, void* dq, void* dk, void* dv, int B, int H, int Lq, int Lk,
                                   int d, float scale, int causal, int o_dtype, void* stream) {
    // the same checks as fa_backward, then the one limit of the fixed scratch
    int rc = bwd_check_args(q, k, v, o, dO, lse, dq, dk, dv, B, H, Lq, Lk, d, scale, causal, o_dtype);
    if (rc != FA_OK) return rc;
    if (static_cast<long long>(B) * H * Lq > FA_NOALLOC_MAX_ROWS) return FA_ERR_TOO_LARGE;
    int* status = nullptr;
    if ((rc = prepare_device(&status)) != FA_OK) return rc;
    float* scratch = nullptr;
    if ((rc = scratch_for_current_device(&scratch)) != FA_OK) return rc;
    // the pre-kernel writes every D_i before the main kernels read it
    return bwd_launch_checked(q, k, v, o, dO, lse, dq, dk, dv, B, H, Lq, Lk, d, scale, causal, o_dtype, scratch,
                              static_cast<cudaStream_t>(stream));
}
