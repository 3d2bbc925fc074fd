// C ABI of the library (declared in include/fa.h): argument checks, TMA
// descriptor encoding, launches, and the per-device status word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <mutex>
#include <unordered_map>

#include "fa_internal.h"

namespace fa {
namespace {

__device__ int g_status;  // one per device; kernels record device-side conditions here
// Forward unit schedulers: (ticket, finished-CTA count) pairs.  Each stream gets
// its own pair the first time it launches a forward (launches on one stream run
// one after another, so they never share a pair while running), and the last CTA
// of each launch returns its pair to zero.
constexpr unsigned kSchedSlots = 256;
__device__ unsigned int g_fwd_sched[2 * kSchedSlots];

constexpr int kMaxDevices = 64;

struct DeviceState {
    bool probed = false;
    bool supported = false;
    int num_sms = 0;
    int* status_ptr = nullptr;
    unsigned int* sched_ptr = nullptr;
    // stream (by its process-unique id) -> scheduler pair; pairs are never handed back
    std::unordered_map<unsigned long long, unsigned> stream_slot;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Resolves (once per device) whether the device is sm_100 and where its status word lives.
int device_state(DeviceState** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return FA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState& st = g_dev[dev];
    if (!st.probed) {
        int major = 0, minor = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
            return FA_ERR_CUDA;
        st.supported = (major == 10 && minor == 0);
        if (cudaDeviceGetAttribute(&st.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return FA_ERR_CUDA;
        if (st.supported) {
            void* ptr = nullptr;
            if (cudaGetSymbolAddress(&ptr, g_status) != cudaSuccess) return FA_ERR_CUDA;
            st.status_ptr = static_cast<int*>(ptr);
            if (cudaGetSymbolAddress(&ptr, g_fwd_sched) != cudaSuccess) return FA_ERR_CUDA;
            st.sched_ptr = static_cast<unsigned int*>(ptr);
        }
        st.probed = true;
    }
    if (!st.supported) return FA_ERR_DEVICE;
    if (!g_encode) {
        void* fn = nullptr;
        cudaDriverEntryPointQueryResult q{};
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess || fn == nullptr)
            return FA_ERR_CUDA;
        g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
    }
    *out = &st;
    return FA_OK;
}

// Scheduler counters for a forward launch on `stream`, or null for the static
// deal (each CTA takes a fixed, snake-ordered share of the units).  The static
// deal is used while the stream is being captured into a graph -- a graph may
// later be replayed on any stream, also on several at once -- and for streams
// beyond the first kSchedSlots that launched a forward on this device.  Streams
// are told apart by cudaStreamGetId, which never repeats within a process, so a
// stream created with the handle of a destroyed one gets a pair of its own.
int fwd_sched(DeviceState* st, cudaStream_t stream, unsigned int** out) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess) return FA_ERR_CUDA;
    *out = nullptr;
    if (cs != cudaStreamCaptureStatusNone) return FA_OK;
    unsigned long long id = 0;
    if (cudaStreamGetId(stream, &id) != cudaSuccess) return FA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_mu);
    auto it = st->stream_slot.find(id);
    if (it == st->stream_slot.end()) {
        if (st->stream_slot.size() >= kSchedSlots) return FA_OK;
        it = st->stream_slot.emplace(id, static_cast<unsigned>(st->stream_slot.size())).first;
    }
    *out = st->sched_ptr + 2 * it->second;
    return FA_OK;
}

// View a contiguous bf16 [BH, L, d] tensor as a 3-D TMA map with 128-row x
// 64-column boxes and 128-byte swizzle (64 bf16 = one 128-byte swizzle span).
// Rows past L read as zero; nothing outside the tensor is touched.
int encode_rows_map(CUtensorMap* map, const void* base, int BH, int L, int d, int box_rows) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * 2, static_cast<cuuint64_t>(L) * d * 2};
    cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
                          estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// A paged K or V pool [rows][d] bf16 (rows = num_pages * Hkv * page_size) as a
// 2-D map with boxes of 64 columns x box_rows rows and 128-byte swizzle.
int encode_pool_map(CUtensorMap* map, const void* base, long long rows, int d, int box_rows) {
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(rows)};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(d) * 2};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// O written by TMA stores: [BH, L, d] in fp32 or bf16, boxes of 32 rows x
// 128 bytes (32 fp32 or 64 bf16 columns), 128-byte swizzle.  Rows past L are
// clipped by the copy engine.
int encode_out_map_impl(CUtensorMap* map, void* base, int BH, int L, int d, int o_dtype) {
    const int esz = o_dtype == FA_DT_F32 ? 4 : 2;
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(L), static_cast<cuuint64_t>(BH)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * esz, static_cast<cuuint64_t>(L) * d * esz};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / esz), 32, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, o_dtype == FA_DT_F32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16,
                          3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

// A packed token-major tensor [total, H, d] (bf16 or fp32) as a 3-D TMA map
// {d, H, total} with boxes of 128 bytes x 1 head x box_rows tokens, so a box
// lands in shared memory exactly like a batched [rows][128 bytes] box.
// 128-byte swizzle.  Rows past total read as zero / are clipped on stores.
int encode_packed_map_impl(CUtensorMap* map, const void* base, int total, int H, int d, int box_rows,
                           int elem_bytes) {
    cuuint64_t dims[3] = {static_cast<cuuint64_t>(d), static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(total)};
    cuuint64_t strides[2] = {static_cast<cuuint64_t>(d) * elem_bytes, static_cast<cuuint64_t>(H) * d * elem_bytes};
    cuuint32_t box[3] = {static_cast<cuuint32_t>(128 / elem_bytes), 1, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[3] = {1, 1, 1};
    CUresult r = g_encode(map, elem_bytes == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                          const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? FA_OK : FA_ERR_CUDA;
}

bool dims_ok(int B, int H, int L, int d) {
    if (B <= 0 || H <= 0 || L <= 0) return false;
    const long long bh = static_cast<long long>(B) * H;
    if (bh > (1LL << 30)) return false;
    if (static_cast<long long>(L) * d * 2 >= (1LL << 40)) return false;
    return true;
}

}  // namespace

// Internal helpers shared with other translation units of this library.
int prepare_device(int** status_ptr) {
    DeviceState* st = nullptr;
    const int rc = device_state(&st);
    if (rc == FA_OK) *status_ptr = st->status_ptr;
    return rc;
}
int encode_tile_map(CUtensorMap* map, const void* base, int BH, int L, int d, int box_rows) {
    return encode_rows_map(map, base, BH, L, d, box_rows);
}
bool shape_ok(int B, int H, int L, int d) { return dims_ok(B, H, L, d); }
int encode_out_map(CUtensorMap* map, void* base, int BH, int L, int d, int o_dtype) {
    return encode_out_map_impl(map, base, BH, L, d, o_dtype);
}
int encode_packed_map(CUtensorMap* map, const void* base, int total, int H, int d, int box_rows, int elem_bytes,
                      bool) {
    return encode_packed_map_impl(map, base, total, H, d, box_rows, elem_bytes);
}

// Argument checks of the backward entry points (everything but the scratch).
int bwd_check_args(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                   const void* dq, const void* dk, const void* dv, int B, int H, int Lq, int Lk, int d, float scale,
                   int causal, int o_dtype) {
    if (!q || !k || !v || !o || !dO || !lse || !dq || !dk || !dv) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
    if (o_dtype != FA_DT_BF16 && o_dtype != FA_DT_F32) return FA_ERR_UNSUPPORTED;
    if (!dims_ok(B, H, Lq, d) || !dims_ok(B, H, Lk, d)) return FA_ERR_INVALID_ARG;
    if (causal && Lq > Lk) return FA_ERR_INVALID_ARG;
    if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(dO, 16) ||
        !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || !aligned(lse, 4))
        return FA_ERR_INVALID_ARG;
    const long long bh = static_cast<long long>(B) * H;
    if (bh * ((Lq + 127) / 128) > 0x7FFFFFFFLL || bh * ((Lk + 127) / 128) * 2 > 0x7FFFFFFFLL ||
        bh * Lq * (d / 8) / 256 > 0x7FFFFFFFLL)
        return FA_ERR_INVALID_ARG;
    return FA_OK;
}

// Encodes the maps and launches the backward kernels; dsum is the scratch for D.
int bwd_launch_checked(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                       void* dq, void* dk, void* dv, int B, int H, int Lq, int Lk, int d, float scale, int causal,
                       int o_dtype, float* dsum, cudaStream_t stream) {
    DeviceState* st = nullptr;
    int rc = device_state(&st);
    if (rc != FA_OK) return rc;
    BwdParams p{};
    const int BH = B * H;
    if ((rc = encode_rows_map(&p.tm_q, q, BH, Lq, d, 128)) != FA_OK) return rc;
    if ((rc = encode_rows_map(&p.tm_k, k, BH, Lk, d, 128)) != FA_OK) return rc;
    if ((rc = encode_rows_map(&p.tm_v, v, BH, Lk, d, 128)) != FA_OK) return rc;
    if ((rc = encode_rows_map(&p.tm_do, dO, BH, Lq, d, 128)) != FA_OK) return rc;
    if (d == 256) {
        if ((rc = encode_rows_map(&p.tm_q64, q, BH, Lq, d, 64)) != FA_OK) return rc;
        if ((rc = encode_rows_map(&p.tm_k64, k, BH, Lk, d, 64)) != FA_OK) return rc;
        if ((rc = encode_rows_map(&p.tm_v64, v, BH, Lk, d, 64)) != FA_OK) return rc;
        if ((rc = encode_rows_map(&p.tm_do64, dO, BH, Lq, d, 64)) != FA_OK) return rc;
    }
    p.o = o;
    p.dO = dO;
    p.lse = lse;
    p.dsum = dsum;
    p.dq = dq;
    p.dk = dk;
    p.dv = dv;
    p.status = st->status_ptr;
    p.B = B;
    p.H = H;
    p.Lq = Lq;
    p.Lk = Lk;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    p.o_dtype = o_dtype;
    p.hg_kv = heads_per_l2_group(2LL * Lq * d * 2, BH);
    p.hg_q = heads_per_l2_group(2LL * Lk * d * 2, BH);
    const cudaError_t e = launch_bwd(p, d, stream);
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

}  // namespace fa

using namespace fa;

extern "C" {

const char* fa_status_string(int status) {
    switch (status) {
        case FA_OK: return "FA_OK";
        case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG: invalid argument";
        case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED: unsupported head dimension or dtype";
        case FA_ERR_WORKSPACE: return "FA_ERR_WORKSPACE: workspace missing or too small";
        case FA_ERR_CUDA: return "FA_ERR_CUDA: CUDA runtime error";
        case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT: a bounded wait inside a kernel ran out";
        case FA_ERR_DEVICE: return "FA_ERR_DEVICE: current device is not compute capability 10.0 (sm_100a)";
        case FA_ERR_KV_LEN: return "FA_ERR_KV_LEN: a decode cache length was outside [0, cap]";
        case FA_ERR_TOO_LARGE:
            return "FA_ERR_TOO_LARGE: B*H*Lq exceeds FA_NOALLOC_MAX_ROWS, the fixed scratch of fa_backward_noalloc";
        case FA_ERR_PAGE:
            return "FA_ERR_PAGE: a block-table entry used by a valid key was outside [0, num_pages) (read as page 0)";
        case FA_ERR_SEQLEN:
            return "FA_ERR_SEQLEN: a packed sequence's offsets or lengths were invalid; its rows were skipped";
        default: return "unknown fa_status";
    }
}

int fa_forward(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Lq, int Lk,
               int d, float scale, int causal, int o_dtype, void* stream) {
    if (!q || !k || !v || !o || !lse) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
    if (o_dtype != FA_DT_BF16 && o_dtype != FA_DT_F32) return FA_ERR_UNSUPPORTED;
    if (!dims_ok(B, H, Lq, d) || !dims_ok(B, H, Lk, d)) return FA_ERR_INVALID_ARG;
    if (causal && Lq > Lk) return FA_ERR_INVALID_ARG;
    if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
        return FA_ERR_INVALID_ARG;
    // units: 256 query rows (d <= 128) or 128 (d = 256) of one (b, h)
    const long long n_ctas = static_cast<long long>(B) * H * ((Lq + 127) / 128);
    if (n_ctas > 0x7FFFFFFFLL) return FA_ERR_INVALID_ARG;

    DeviceState* st = nullptr;
    int rc = device_state(&st);
    if (rc != FA_OK) return rc;

    FwdParams p{};
    const int BH = B * H;
    const int kv_rows = d == 256 ? kFwd256BN : kFwdBN;  // keys per K/V tile
    if ((rc = encode_rows_map(&p.tm_q, q, BH, Lq, d, kFwdBM)) != FA_OK) return rc;
    if ((rc = encode_rows_map(&p.tm_k, k, BH, Lk, d, kv_rows)) != FA_OK) return rc;
    if ((rc = encode_rows_map(&p.tm_v, v, BH, Lk, d, kv_rows)) != FA_OK) return rc;
    if ((rc = encode_out_map_impl(&p.tm_o, o, BH, Lq, d, o_dtype)) != FA_OK) return rc;
    p.o = o;
    p.lse = lse;
    p.status = st->status_ptr;
    if ((rc = fwd_sched(st, static_cast<cudaStream_t>(stream), &p.sched)) != FA_OK) return rc;
    p.B = B;
    p.H = H;
    p.Lq = Lq;
    p.Lk = Lk;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    p.o_dtype = o_dtype;
    p.head_group = heads_per_l2_group(2LL * Lk * d * 2, BH);
    cudaError_t e = d == 256 ? launch_fwd256(p, st->num_sms, static_cast<cudaStream_t>(stream))
                             : launch_fwd(p, d, st->num_sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_forward_blocksparse_workspace_size(int B, int H, int Lq, int Lk) {
    if (B <= 0 || H <= 0 || Lq <= 0 || Lk <= 0) return 0;
    if ((static_cast<long long>(Lk) + kFwdBN - 1) / kFwdBN > kBsMaxKeyBlocks) return 0;
    return bs_workspace_bytes(B, H, Lq, Lk);
}

int fa_forward_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse,
                           const unsigned char* block_mask, long long mask_stride_b, long long mask_stride_h, int B,
                           int H, int Lq, int Lk, int d, float scale, int causal, int o_dtype, void* workspace,
                           size_t workspace_bytes, void* stream) {
    if (!q || !k || !v || !o || !lse || !block_mask) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
    if (o_dtype != FA_DT_BF16 && o_dtype != FA_DT_F32) return FA_ERR_UNSUPPORTED;
    if (!dims_ok(B, H, Lq, d) || !dims_ok(B, H, Lk, d)) return FA_ERR_INVALID_ARG;
    if (causal && Lq > Lk) return FA_ERR_INVALID_ARG;
    if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
    if (mask_stride_b < 0 || mask_stride_h < 0) return FA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4))
        return FA_ERR_INVALID_ARG;
    const long long n_pairs = (Lq + kFwdRowsPerCta - 1) / kFwdRowsPerCta;
    const long long tk = (static_cast<long long>(Lk) + kFwdBN - 1) / kFwdBN;
    if (static_cast<long long>(B) * H * n_pairs > 0x7FFFFFFFLL || tk > kBsMaxKeyBlocks) return FA_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < bs_workspace_bytes(B, H, Lq, Lk))
        return FA_ERR_WORKSPACE;

    DeviceState* st = nullptr;
    int rc = device_state(&st);
    if (rc != FA_OK) return rc;

    const size_t n_units = static_cast<size_t>(B) * H * n_pairs;
    BsPlanParams plan{};
    plan.mask = block_mask;
    plan.stride_b = mask_stride_b;
    plan.stride_h = mask_stride_h;
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    char* ws = static_cast<char*>(workspace);
    plan.meta = reinterpret_cast<int4*>(ws);
    plan.list = reinterpret_cast<uint16_t*>(ws + up(n_units * sizeof(int4)));
    plan.own = reinterpret_cast<uint16_t*>(ws + up(n_units * sizeof(int4)) +
                                           up(n_units * static_cast<size_t>(tk) * sizeof(uint16_t)));
    plan.B = B;
    plan.H = H;
    plan.Lq = Lq;
    plan.Lk = Lk;
    plan.n_pairs = static_cast<int>(n_pairs);
    plan.tk = static_cast<int>(tk);
    plan.causal = causal ? 1 : 0;

    FwdParams p{};
    const int BH = B * H;
    if ((rc = encode_rows_map(&p.tm_q, q, BH, Lq, d, kFwdBM)) != FA_OK) return rc;
    const int kv_rows = d == 256 ? kFwd256BN : kFwdBN;  // keys per K/V tile
    if ((rc = encode_rows_map(&p.tm_k, k, BH, Lk, d, kv_rows)) != FA_OK) return rc;
    if ((rc = encode_rows_map(&p.tm_v, v, BH, Lk, d, kv_rows)) != FA_OK) return rc;
    if ((rc = encode_out_map_impl(&p.tm_o, o, BH, Lq, d, o_dtype)) != FA_OK) return rc;
    p.o = o;
    p.lse = lse;
    p.status = st->status_ptr;
    if ((rc = fwd_sched(st, static_cast<cudaStream_t>(stream), &p.sched)) != FA_OK) return rc;
    p.bs_meta = plan.meta;
    p.bs_list = plan.list;
    p.bs_own = plan.own;
    p.bs_tk = plan.tk;
    p.B = B;
    p.H = H;
    p.Lq = Lq;
    p.Lk = Lk;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = plan.causal;
    p.o_dtype = o_dtype;
    p.head_group = heads_per_l2_group(2LL * Lk * d * 2, BH);
    cudaError_t e = launch_fwd_blocksparse(plan, p, d, st->num_sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_decode_workspace_size(int B, int H, int cap, int d) {
    if (B <= 0 || H <= 0 || cap <= 0 || (d != 64 && d != 128 && d != 256)) return 0;
    return decode_workspace_bytes(B, H, cap, d);
}

int fa_decode(const void* q, const void* kcache, const void* vcache, const int* kv_lens, void* o, float* lse,
              int B, int H, int cap, int d, float scale, int o_dtype, void* workspace, size_t workspace_bytes,
              void* stream) {
    if (!q || !kcache || !vcache || !kv_lens || !o || !lse) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
    if (o_dtype != FA_DT_BF16 && o_dtype != FA_DT_F32) return FA_ERR_UNSUPPORTED;
    if (!dims_ok(B, H, cap, d) || !scale_ok(scale)) return FA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(kcache, 16) || !aligned(vcache, 16) || !aligned(o, 16) ||
        !aligned(kv_lens, 4) || !aligned(lse, 4))
        return FA_ERR_INVALID_ARG;
    const long long items = static_cast<long long>(B) * H * ((cap + kDecodeSplit - 1) / kDecodeSplit);
    if (items > 0x7FFFFFFFLL || static_cast<long long>(B) * H > 0x7FFFFFFFLL) return FA_ERR_INVALID_ARG;
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < decode_workspace_bytes(B, H, cap, d))
        return FA_ERR_WORKSPACE;

    DeviceState* st = nullptr;
    int rc = device_state(&st);
    if (rc != FA_OK) return rc;

    DecodeParams p{};
    p.q = q;
    p.k = kcache;
    p.v = vcache;
    p.kv_lens = kv_lens;
    p.o = o;
    p.lse = lse;
    p.status = st->status_ptr;
    p.B = B;
    p.H = H;
    p.cap = cap;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.o_dtype = o_dtype;
    decode_carve_workspace(p, workspace, B, H, cap, d);
    cudaError_t e = launch_decode(p, d, st->num_sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_backward_workspace_size(int B, int H, int Lq, int Lk, int d) {
    if (B <= 0 || H <= 0 || Lq <= 0 || Lk <= 0 || (d != 64 && d != 128 && d != 256)) return 0;
    return bwd_workspace_bytes(B, H, Lq);
}

int fa_backward(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                void* dq, void* dk, void* dv, int B, int H, int Lq, int Lk, int d, float scale, int causal,
                int o_dtype, void* workspace, size_t workspace_bytes, void* stream) {
    int rc = bwd_check_args(q, k, v, o, dO, lse, dq, dk, dv, B, H, Lq, Lk, d, scale, causal, o_dtype);
    if (rc != FA_OK) return rc;
    if (!workspace || !aligned(workspace, 256) || workspace_bytes < bwd_workspace_bytes(B, H, Lq))
        return FA_ERR_WORKSPACE;
    return bwd_launch_checked(q, k, v, o, dO, lse, dq, dk, dv, B, H, Lq, Lk, d, scale, causal, o_dtype,
                              static_cast<float*>(workspace), static_cast<cudaStream_t>(stream));
}

int fa_forward_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens_q,
                      const int* cu_seqlens_k, int B, int H, int total_q, int total_k, int max_seqlen_q, int d,
                      float scale, int causal, int o_dtype, void* stream) {
    if (!q || !k || !v || !o || !lse || !cu_seqlens_q || !cu_seqlens_k) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
    if (o_dtype != FA_DT_BF16 && o_dtype != FA_DT_F32) return FA_ERR_UNSUPPORTED;
    if (B <= 0 || H <= 0 || total_q < 0 || total_k < 0 || max_seqlen_q < 0) return FA_ERR_INVALID_ARG;
    if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
        !aligned(cu_seqlens_q, 4) || !aligned(cu_seqlens_k, 4))
        return FA_ERR_INVALID_ARG;
    if (static_cast<long long>(total_q) * H > 0x7FFFFFFFLL || static_cast<long long>(total_k) * H > 0x7FFFFFFFLL)
        return FA_ERR_INVALID_ARG;
    // units of 256 query rows (two 128-row tiles); at d = 256 single 128-row tiles
    const int unit_rows = d == 256 ? kFwdBM : kFwdRowsPerCta;
    const long long max_pairs = (static_cast<long long>(max_seqlen_q) + unit_rows - 1) / unit_rows;
    if (static_cast<long long>(B) * H * max_pairs > 0x7FFFFFFFLL || max_pairs * unit_rows > 0x7FFFFFFFLL)
        return FA_ERR_INVALID_ARG;
    if (total_q == 0 || max_pairs == 0) return FA_OK;
    if (total_k == 0) return FA_ERR_INVALID_ARG;

    DeviceState* st = nullptr;
    int rc = device_state(&st);
    if (rc != FA_OK) return rc;
    FwdParams p{};
    if ((rc = encode_packed_map_impl(&p.tm_q, q, total_q, H, d, kFwdBM, 2)) != FA_OK) return rc;
    const int kv_rows = d == 256 ? kFwd256BN : kFwdBN;  // keys per K/V tile
    if ((rc = encode_packed_map_impl(&p.tm_k, k, total_k, H, d, kv_rows, 2)) != FA_OK) return rc;
    if ((rc = encode_packed_map_impl(&p.tm_v, v, total_k, H, d, kv_rows, 2)) != FA_OK) return rc;
    if ((rc = encode_packed_map_impl(&p.tm_o, o, total_q, H, d, 32, o_dtype == FA_DT_F32 ? 4 : 2)) != FA_OK)
        return rc;
    p.o = o;
    p.lse = lse;
    p.status = st->status_ptr;
    if ((rc = fwd_sched(st, static_cast<cudaStream_t>(stream), &p.sched)) != FA_OK) return rc;
    p.cu_q = cu_seqlens_q;
    p.cu_k = cu_seqlens_k;
    p.max_pairs = static_cast<int>(max_pairs);
    p.B = B;
    p.H = H;
    p.Lq = total_q;
    p.Lk = total_k;
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.causal = causal ? 1 : 0;
    p.o_dtype = o_dtype;
    cudaError_t e = d == 256 ? launch_fwd256_varlen(p, st->num_sms, static_cast<cudaStream_t>(stream))
                             : launch_fwd_varlen(p, d, st->num_sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

size_t fa_decode_paged_workspace_size(int B, int H, int max_blocks, int page_size, int d) {
    if (B <= 0 || H <= 0 || max_blocks <= 0 || page_size <= 0 || (d != 64 && d != 128 && d != 256)) return 0;
    const long long cap = static_cast<long long>(max_blocks) * page_size;
    if (cap > 0x7FFFFFFFLL) return 0;
    return decode_workspace_bytes(B, H, static_cast<int>(cap), d);
}

int fa_decode_paged(const void* q, const void* kpages, const void* vpages, const int* block_table,
                    const int* kv_lens, void* o, float* lse, int B, int H, int Hkv, int num_pages, int page_size,
                    int max_blocks, int d, float scale, int o_dtype, void* workspace, size_t workspace_bytes,
                    void* stream) {
    if (!q || !kpages || !vpages || !block_table || !kv_lens || !o || !lse) return FA_ERR_INVALID_ARG;
    if (d != 64 && d != 128 && d != 256) return FA_ERR_UNSUPPORTED;
    if (o_dtype != FA_DT_BF16 && o_dtype != FA_DT_F32) return FA_ERR_UNSUPPORTED;
    if (B <= 0 || H <= 0 || Hkv <= 0 || H % Hkv != 0 || num_pages <= 0 || max_blocks <= 0) return FA_ERR_INVALID_ARG;
    if (page_size <= 0 || page_size > 65536 || (page_size & (page_size - 1)) != 0) return FA_ERR_INVALID_ARG;
    const long long cap = static_cast<long long>(max_blocks) * page_size;
    if (cap > 0x7FFFFFFFLL || static_cast<long long>(B) * H > (1LL << 30) ||
        static_cast<long long>(B) * max_blocks > 0x7FFFFFFFLL)
        return FA_ERR_INVALID_ARG;
    if (!scale_ok(scale)) return FA_ERR_INVALID_ARG;
    if (!aligned(q, 16) || !aligned(kpages, 16) || !aligned(vpages, 16) || !aligned(o, 16) || !aligned(lse, 4) ||
        !aligned(block_table, 4) || !aligned(kv_lens, 4))
        return FA_ERR_INVALID_ARG;
    const size_t need = decode_workspace_bytes(B, H, static_cast<int>(cap), d);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256)) return FA_ERR_WORKSPACE;
    const long long max_splits = (cap + kDecodeSplit - 1) / kDecodeSplit;
    if (static_cast<long long>(B) * H * max_splits > 0x7FFFFFFFLL) return FA_ERR_INVALID_ARG;

    DeviceState* st = nullptr;
    int rc = device_state(&st);
    if (rc != FA_OK) return rc;
    DecodeParams p{};
    p.q = q;
    p.k = kpages;
    p.v = vpages;
    p.kv_lens = kv_lens;
    p.o = o;
    p.lse = lse;
    p.status = st->status_ptr;
    p.B = B;
    p.H = H;
    p.cap = static_cast<int>(cap);
    p.scale = scale;
    p.scale_log2 = scale * 1.4426950408889634f;
    p.o_dtype = o_dtype;
    p.block_table = block_table;
    p.Hkv = Hkv;
    p.num_pages = num_pages;
    int shift = 0;
    while ((1 << shift) < page_size) ++shift;
    p.page_shift = shift;
    p.max_blocks = max_blocks;
    // the tensor-core kernel needs boxes of at least 8 rows (one 1,024-byte swizzle atom)
    // and pool row indices that fit the map's int32 coordinates
    const long long pool_rows = static_cast<long long>(num_pages) * Hkv * page_size;
    p.pool_box_rows = 0;
    if ((d == 64 || d == 128) && page_size >= 8 && pool_rows <= 0x7FFFFFFFLL) {
        const int br = page_size < 64 ? page_size : 64;
        if ((rc = encode_pool_map(&p.tm_kpool, kpages, pool_rows, d, br)) != FA_OK) return rc;
        if ((rc = encode_pool_map(&p.tm_vpool, vpages, pool_rows, d, br)) != FA_OK) return rc;
        p.pool_box_rows = br;
    }
    decode_carve_workspace(p, workspace, B, H, static_cast<int>(cap), d);
    cudaError_t e = launch_decode_paged(p, d, st->num_sms, static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}

int fa_check_status(void* stream) {
    DeviceState* st = nullptr;
    int rc = device_state(&st);
    if (rc != FA_OK) return rc;
    (void)stream;  // the status word is per device: wait for every stream of it
    if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
    int h = 0;
    if (cudaMemcpy(&h, st->status_ptr, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return FA_ERR_CUDA;
    if (h != 0) {
        if (cudaMemset(st->status_ptr, 0, sizeof(int)) != cudaSuccess) return FA_ERR_CUDA;
        if (cudaDeviceSynchronize() != cudaSuccess) return FA_ERR_CUDA;
    }
    return h;
}

#ifdef FA_TEST_HOOKS
// Fault injection for the tests of the bounded waits; exported by the test build
// (libfa_sm100_testhooks.so) only.  where: 1 = forward K tile, 2 = dK/dV K/V
// tiles, 3 = paged-decode stage (d <= 128), 4 = paged-decode stage (d = 256).
// Arms a one-shot fault on the current device.
int fa_test_inject_fault(int where) {
    DeviceState* st = nullptr;
    const int rc = device_state(&st);
    if (rc != FA_OK) return rc;
    cudaError_t e = cudaErrorInvalidValue;
    if (where == 1) e = fwd_test_arm_skip_k();
    else if (where == 2) e = bwd_test_arm_skip_kv();
    else if (where == 3) e = paged_mma_test_arm_skip_stage();
    else if (where == 4) e = paged_test_arm_skip_stage();
    else return FA_ERR_INVALID_ARG;
    return e == cudaSuccess ? FA_OK : FA_ERR_CUDA;
}
#endif

}  // extern "C"
