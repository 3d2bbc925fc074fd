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

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace fa

using namespace fa;

extern "C" int fa_backward_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                                   const float* lse, void* dq, void* dk, void* dv, int B, int H, int Lq, int Lk,
                                   int d, float scale, int causal, int o_dtype, void* stream) {
    if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128) return FA_ERR_UNSUPPORTED;
    if (o_dtype != FA_DT_BF16 && o_dtype != FA_DT_F32) return FA_ERR_UNSUPPORTED;
    if (!shape_ok(B, H, Lq, d) || !shape_ok(B, H, Lk, d)) return FA_ERR_INVALID_ARG;
    if (causal && Lq > Lk) return FA_ERR_INVALID_ARG;
    if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) || !aligned16(dO) || !aligned16(dq) ||
        !aligned16(dk) || !aligned16(dv) || (reinterpret_cast<uintptr_t>(lse) & 3u) != 0)
        return FA_ERR_INVALID_ARG;
    if (static_cast<long long>(B) * H * Lq > FA_NOALLOC_MAX_ROWS) return FA_ERR_TOO_LARGE;

    int* status = nullptr;
    int rc = prepare_device(&status);
    if (rc != FA_OK) return rc;
    float* scratch = nullptr;
    if ((rc = scratch_for_current_device(&scratch)) != FA_OK) return rc;

    BwdParams p{};
    const int BH = B * H;
    if ((rc = encode_tile_map(&p.tm_q, q, BH, Lq, d, 128)) != FA_OK) return rc;
    if ((rc = encode_tile_map(&p.tm_k, k, BH, Lk, d, 128)) != FA_OK) return rc;
    if ((rc = encode_tile_map(&p.tm_v, v, BH, Lk, d, 128)) != FA_OK) return rc;
    if ((rc = encode_tile_map(&p.tm_do, dO, BH, Lq, d, 128)) != FA_OK) return rc;
    p.o = o;
    p.dO = dO;
    p.lse = lse;
    p.dsum = scratch;  // the pre-kernel writes every D_i before the main kernels read it
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.status = status;
    p.B = B;
    p.H = H;
    p.Lq = Lq;
    p.Lk = Lk;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    p.o_dtype = o_dtype;
    const cudaError_t e = launch_bwd(p, d, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}
