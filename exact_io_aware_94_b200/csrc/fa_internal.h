// Internal declarations shared by the host API and the kernel translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "fa.h"

namespace fa {

// Every bounded wait in a kernel gives up after this long (nanoseconds of
// %globaltimer), records FA_ERR_TIMEOUT and lets the CTA exit.  The fault-
// injection build used by the tests (FA_TEST_HOOKS) waits 20 ms instead.
#ifdef FA_TEST_HOOKS
constexpr uint64_t kWaitTimeoutNs = 20000000ull;
#else
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;
#endif

#ifdef FA_TEST_HOOKS
// Fault injection (test build only): arm a one-shot fault in one kernel's
// producer.  Each returns a CUDA error code.
cudaError_t fwd_test_arm_skip_k();      // forward: the next K tile a producer would load is never loaded
cudaError_t bwd_test_arm_skip_kv();     // dK/dV kernel: the next CTA's K/V tiles are never loaded
cudaError_t paged_test_arm_skip_stage();  // paged decode, d = 256: the next stage's copies are never issued
cudaError_t paged_mma_test_arm_skip_stage();  // paged decode, d <= 128: the same
#endif

// Forward kernel tiling: two 128-row Q tiles per CTA (one per softmax
// warpgroup), 128-key K/V tiles.
constexpr int kFwdBM = 128;
constexpr int kFwdBN = 128;
constexpr int kFwdRowsPerCta = 2 * kFwdBM;
constexpr int kFwdThreads = 384;  // 2 softmax warpgroups + a warpgroup holding the TMA and MMA warps
constexpr int kBwdThreads = 320;  // 2 elementwise warpgroups + TMA warp + MMA warp
// Register split of the forward kernel (setmaxnreg): the two softmax warpgroups
// grow to kFwdRegsSoftmax, the TMA/MMA warpgroup shrinks to kFwdRegsOther.  The
// launch allocation must cover the split: kFwdThreads x (registers the kernel is
// compiled with) >= 2*128*kFwdRegsSoftmax + 128*kFwdRegsOther; launch_fwd checks.
constexpr int kFwdRegsSoftmax = 200;
constexpr int kFwdRegsOther = 104;

struct __align__(64) FwdParams {
    CUtensorMap tm_q;  // [B*H, Lq, d] bf16, box {64, 128, 1}, 128B swizzle
    CUtensorMap tm_k;  // [B*H, Lk, d]
    CUtensorMap tm_v;  // [B*H, Lk, d]
    CUtensorMap tm_o;  // O as [B*H, Lq, d] (fp32 or bf16), box {128 bytes, 32 rows, 1}, 128B swizzle
    void* o;
    float* lse;
    int* status;
    unsigned int* sched;  // [0]: next unit ticket, [1]: CTAs finished; both zero between launches.
                          // Null: static deal (no counters).
    // packed variable-length batch (fa_forward_varlen): sequence b owns rows [cu_q[b], cu_q[b+1])
    // of q, o [total_q, H, d] and [cu_k[b], cu_k[b+1]) of k, v [total_k, H, d]; Lq = total_q,
    // Lk = total_k, and max_pairs = ceil(max_seqlen_q / 256) (d = 256: ceil(max_seqlen_q / 128),
    // the kernel's units being single 128-row tiles).  Null for a batched call.
    const int* cu_q;
    const int* cu_k;
    int max_pairs;
    // block-sparse forward (fa_forward_blocksparse), per unit ui = (b*H + h) * n_pairs + pair:
    //   bs_meta[ui] = {entries of the union list, union index of the last entry of query block 0,
    //                  the same for query block 1 (-1 if it does not exist),
    //                  own-list lengths n0 | n1 << 16};
    //   union list at bs_list + ui * bs_tk: key-block index (bits 0-13), bit 14 / 15 set when
    //   query block 0 / 1 of the pair takes part in the entry;
    //   own list of query block w at bs_own + (2 * ui + w) * bs_tk: key-block index, bit 15
    //   set when the block takes part only to write its empty rows (every score masked).
    // Null otherwise.
    const int4* bs_meta;
    const uint16_t* bs_list;
    const uint16_t* bs_own;
    int bs_tk;
    int B, H, Lq, Lk;
    float scale;       // multiplies q.k
    float scale_log2;  // scale * log2(e)
    int causal;
    int o_dtype;
    int head_group;    // batched and block-sparse kernels: heads per group of the unit order (>= 1)
};

// Heads whose K and V (or, for the backward, whose re-read tensors) are kept in
// L2 together by the unit and block orders: bytes_per_head of the re-read data
// against a budget of about a quarter of the 126 MB L2.  When not even two heads
// fit, the heads are not grouped at all (one group of all of them): with many
// CTAs on each long head, interleaving the heads measured faster than taking
// them one at a time.
inline int heads_per_l2_group(long long bytes_per_head, int BH) {
    const long long budget = 32LL << 20;
    long long g = bytes_per_head > 0 ? budget / bytes_per_head : BH;
    if (g < 2 || g > BH) g = BH;
    return static_cast<int>(g);
}

struct __align__(64) BwdParams {
    CUtensorMap tm_q;   // [B*H, Lq, d] bf16, box {64, 128, 1}
    CUtensorMap tm_k;   // [B*H, Lk, d]
    CUtensorMap tm_v;   // [B*H, Lk, d]
    CUtensorMap tm_do;  // [B*H, Lq, d]
    // d = 256 only: the same tensors with 64-row boxes (64-query tiles of the dK/dV
    // kernel, 64-key tiles of the dQ kernel)
    CUtensorMap tm_q64, tm_k64, tm_v64, tm_do64;
    const void* o;      // forward output, o_dtype
    const void* dO;     // bf16 [B, H, Lq, d]
    const float* lse;   // [B, H, Lq]
    float* dsum;        // workspace: D_i = rowsum(dO o O), [B, H, Lq]
    void* dq;           // bf16 outputs
    void* dk;
    void* dv;
    int* status;
    int B, H, Lq, Lk;
    float scale, scale_log2;
    int causal;
    int o_dtype;
    // block orders: heads per group whose Q and dO (dK/dV kernels) or K and V (dQ
    // kernels) stay in L2 together (>= 1)
    int hg_kv, hg_q;
};

// Block b of a grid of BH * n tiles, in groups of G heads: within a group, tile
// index t = 0, 1, ... slowest, heads interleaved.  Returns (t, bh).
__device__ __forceinline__ void grouped_block(int b, int BH, int n, int G, int& t, int& bh) {
    const int grp = b / (G * n);
    const int r = b - grp * G * n;
    const int gsz = min(G, BH - grp * G);
    t = r / gsz;
    bh = grp * G + r % gsz;
}

size_t bwd_workspace_bytes(int B, int H, int Lq);

// Helpers implemented in api.cu for the other entry points.
int prepare_device(int** status_ptr);
int bwd_check_args(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                   const void* dq, const void* dk, const void* dv, int B, int H, int Lq, int Lk, int d, float scale,
                   int causal, int o_dtype);
int bwd_launch_checked(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                       void* dq, void* dk, void* dv, int B, int H, int Lq, int Lk, int d, float scale, int causal,
                       int o_dtype, float* dsum, cudaStream_t stream);
int encode_tile_map(CUtensorMap* map, const void* base, int BH, int L, int d, int box_rows);
bool shape_ok(int B, int H, int L, int d);
// Every kernel takes the running maximum over raw scores q.k and applies the
// scale inside the exponent, and masks scores to -inf before it: that is only
// right for a positive, finite scale (zero would turn -inf * 0 into NaN).
inline bool scale_ok(float scale) { return scale > 0.0f && scale <= 3.4028234663852886e38f; }
cudaError_t launch_bwd(const BwdParams& p, int d, cudaStream_t stream);
cudaError_t launch_bwd256_main(const BwdParams& p, cudaStream_t stream);

// Decode: keys of each sequence are cut into chunks of kDecodeSplit keys.
constexpr int kDecodeSplit = 1024;
constexpr int kDecodeThreads = 256;

struct __align__(64) DecodeParams {
    // paged cache on the tensor cores (d = 64, 128, page_size >= 8): the K and V page pools as
    // 2-D maps [num_pages * Hkv * page_size rows][d], boxes of 64 columns x pool_box_rows rows
    // (min(page_size, 64)), 128-byte swizzle.  pool_box_rows = 0: the CUDA-core kernel instead.
    CUtensorMap tm_kpool, tm_vpool;
    int pool_box_rows;
    const void* q;        // [B, H, d] bf16
    const void* k;        // [B, H, cap, d] bf16
    const void* v;        // [B, H, cap, d] bf16
    const int* kv_lens;   // [B]
    void* o;              // [B, H, d]
    float* lse;           // [B, H]
    int* status;
    // workspace
    float* part_o;        // [B*H, max_splits, d] normalised partial outputs
    float* part_lse;      // [B*H, max_splits]
    int* lens;            // [B] clamped lengths
    int* cum;             // [B+1] prefix sums of chunk counts
    int B, H, cap, max_splits;
    float scale, scale_log2;
    int o_dtype;
    // paged cache (fa_decode_paged); block_table is null for the contiguous cache
    const int* block_table;  // [B, max_blocks] page indices
    int Hkv, num_pages, page_shift, max_blocks;  // page_size = 1 << page_shift
};

size_t decode_workspace_bytes(int B, int H, int cap, int d);
void decode_carve_workspace(DecodeParams& p, void* ws, int B, int H, int cap, int d);
cudaError_t launch_decode(const DecodeParams& p, int d, int num_sms, cudaStream_t stream);
cudaError_t launch_decode_paged(const DecodeParams& p, int d, int num_sms, cudaStream_t stream);
// The split step of the paged decode at d = 64, 128 on the tensor cores (the
// combine is launched by launch_decode_paged).
cudaError_t launch_paged_mma_split(const DecodeParams& p, int d, int num_sms, cudaStream_t stream);

// Block-sparse planning: per 256-row unit, the key blocks (after the causal cut)
// that either of its two 128-row query blocks may see, in increasing order.
constexpr int kBsMaxKeyBlocks = 1 << 14;
constexpr int kBsEntryTile = (1 << 14) - 1;
constexpr int kBsOwnMasked = 1 << 15;
struct BsPlanParams {
    const uint8_t* mask;  // block mask of (b, h) at mask + b * stride_b + h * stride_h, [Tq][Tk]
    long long stride_b, stride_h;
    int4* meta;           // [B*H*n_pairs]
    uint16_t* list;       // [B*H*n_pairs][Tk]
    uint16_t* own;        // [B*H*n_pairs][2][Tk]
    int B, H, Lq, Lk, n_pairs, tk, causal;
};
size_t bs_workspace_bytes(int B, int H, int Lq, int Lk);

int fwd_smem_bytes(int d);
cudaError_t launch_fwd(const FwdParams& p, int d, int num_sms, cudaStream_t stream);
// Head dimension 256: one 128-row Q tile per unit, K/V tiles of kFwd256BN keys.
constexpr int kFwd256BN = 64;
cudaError_t launch_fwd256(const FwdParams& p, int num_sms, cudaStream_t stream);
// Packed batch at d = 256: p.max_pairs is the number of 128-row query tiles of the longest sequence.
cudaError_t launch_fwd256_varlen(const FwdParams& p, int num_sms, cudaStream_t stream);
// Block-sparse batch at d = 256 (after the plan): p.bs_* set.
cudaError_t launch_fwd256_blocksparse(const FwdParams& p, int num_sms, cudaStream_t stream);
cudaError_t launch_fwd_varlen(const FwdParams& p, int d, int num_sms, cudaStream_t stream);
cudaError_t launch_fwd_blocksparse(const BsPlanParams& plan, const FwdParams& p, int d, int num_sms,
                                   cudaStream_t stream);
int encode_packed_map(CUtensorMap* map, const void* base, int total, int H, int d, int box_rows, int elem_bytes,
                      bool swizzle_box64);
int encode_out_map(CUtensorMap* map, void* base, int BH, int L, int d, int o_dtype);

}  // namespace fa
