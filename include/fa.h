/*
 * fa.h -- C ABI of the exact IO-aware attention library for NVIDIA B200 (sm_100a).
 *
 * The library computes exact scaled-dot-product attention
 *     O = softmax(scale * Q K^T + mask) V
 * tile by tile with the online-softmax recurrence (running max m_i, running
 * sum l_i, unnormalised accumulator rescaled by exp(m_i - m_i_new), final
 * division O_i = O~_i / l_i), so the L x L score and probability matrices never
 * reach device memory.  Definitions follow the pages:
 *   - "Flash Attention" glossary entry, "How it works": blocks of Q, K, V are
 *     combined in on-chip memory with a running normalisation; the backward
 *     pass recomputes intermediates instead of storing them.
 *   - "What Is FlashAttention?", "What FlashAttention does instead": running
 *     maximum and running sum per row; the score tile never reaches HBM.
 *   - "How Flash Attention Improves Transformer Memory Efficiency ...",
 *     "The Three Running Statistics" (the update rules above) and "Backward
 *     Pass Efficiency" (per-row statistics D_i instead of stored matrices);
 *     "Basic Flash Attention Forward Pass": q, k, v of shape (B, H, L, D),
 *     scale = 1/sqrt(D), causal flag.
 *
 * Conventions shared by every call
 *   Layout      Q, O, dO, dQ: contiguous row-major [B, H, Lq, d]; K, V, dK, dV:
 *               [B, H, Lk, d]; LSE: fp32 [B, H, Lq]; decode caches [B, H, cap, d].
 *   Types       Q, K, V, dO, caches: bfloat16.  O: bfloat16 or fp32 (o_dtype).
 *               dQ, dK, dV: bfloat16.  Accumulation is fp32 throughout.
 *   Mask        causal != 0 permits key j for query row i iff j <= i + (Lk - Lq)
 *               (bottom-right alignment; identical to j <= i when Lq == Lk).
 *               Causal calls require Lq <= Lk.
 *   LSE         LSE_i = ln sum_j exp(scale * q_i . k_j) over permitted keys
 *               (natural log, scaled-score units).
 *   Scale       scale must be finite and > 0 (FA_ERR_INVALID_ARG otherwise): the
 *               kernels take the running maximum over the raw scores q.k and
 *               apply the scale inside the exponent.
 *   Pointers    All tensor pointers are DEVICE pointers on the current CUDA
 *               device, 16-byte aligned.  The caller owns every buffer; the
 *               library never allocates, frees or synchronises.  Calls are
 *               asynchronous on `stream` (a cudaStream_t; NULL = legacy default).
 *   Workspace   A workspace holds one call's scratch from its launch until its
 *               kernels finish: calls that may run at the same time (on different
 *               streams) need different workspaces.
 *   Forwards    fa_forward, fa_forward_varlen and fa_forward_blocksparse hand out
 *               their work units from a per-stream counter (each of the first 256
 *               streams that launch a forward on a device gets its own; calls on
 *               one stream run one after another, and each call's last block
 *               returns the counter to zero).  While `stream` is being captured
 *               into a CUDA graph, and on streams beyond the first 256, a call
 *               deals its units statically instead, so a captured graph may be
 *               replayed on any number of streams at once.
 *   Devices     Compute capability 10.0 (sm_100a) only; elsewhere calls return
 *               FA_ERR_DEVICE.  There is no fallback path.  The library looks up
 *               the device addresses of its static arrays (status word, forward
 *               counters, fa_backward_noalloc's scratch) once per device and keeps
 *               them, so resetting a device (cudaDeviceReset) while the library is
 *               loaded is not supported.
 *   Errors      Argument errors are returned synchronously and nothing is
 *               launched.  A failed launch returns FA_ERR_CUDA.  Conditions met
 *               on the device (a bounded wait that ran out, a cache length outside
 *               [0, cap]) are recorded in a per-device status word read by
 *               fa_check_status().  No kernel traps.
 */
#ifndef EXACT_IO_AWARE_FA_H
#define EXACT_IO_AWARE_FA_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    FA_OK = 0,
    FA_ERR_INVALID_ARG = 1, /* null pointer, non-positive size or scale, misalignment, causal with Lq > Lk */
    FA_ERR_UNSUPPORTED = 2, /* head dimension not supported by the call (see each call), dtype code unknown */
    FA_ERR_WORKSPACE = 3,   /* workspace pointer null or smaller than *_workspace_size() */
    FA_ERR_CUDA = 4,        /* a CUDA runtime call or launch failed */
    FA_ERR_TIMEOUT = 5,     /* device: a bounded wait inside a kernel ran out */
    FA_ERR_DEVICE = 6,      /* current device is not compute capability 10.0 */
    FA_ERR_KV_LEN = 7,      /* device: a decode cache length was outside [0, cap] (clamped) */
    FA_ERR_TOO_LARGE = 8,   /* problem larger than the fixed scratch of fa_backward_noalloc */
    FA_ERR_PAGE = 9,        /* device: a block-table entry used by a valid key was outside [0, num_pages) */
    FA_ERR_SEQLEN = 10      /* device: a packed sequence's offsets or lengths were invalid (sequence skipped) */
} fa_status;

enum { FA_DT_BF16 = 0, FA_DT_F32 = 1 };

/*
 * Forward pass ("How it works" of the glossary entry; "The Three Running
 * Statistics").  Reads q [B,H,Lq,d], k and v [B,H,Lk,d] (bf16); writes
 * o [B,H,Lq,d] (bf16 if o_dtype == FA_DT_BF16, fp32 if FA_DT_F32) and
 * lse [B,H,Lq] (fp32).  scale multiplies q.k before the softmax (typically
 * 1/sqrt(d)).  d must be 64, 128 or 256 ("Basic Flash Attention Forward Pass"
 * leaves D free; d = 256 runs a kernel with 128-row query tiles and 64-key K/V
 * tiles).  Rows never see keys beyond Lk; nothing past the end of any tensor is
 * read.
 */
int fa_forward(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Lq, int Lk,
               int d, float scale, int causal, int o_dtype, void* stream);

/*
 * Workspace bytes fa_backward needs for these sizes: the per-row statistic
 * D [B,H,Lq] (fp32), rounded up to 256 bytes.  (dQ is computed in its own
 * pass, so there is no fp32 dQ accumulator.)  Returns 0 for invalid sizes.
 */
size_t fa_backward_workspace_size(int B, int H, int Lq, int Lk, int d);

/*
 * Backward pass with recomputation ("Backward Pass Efficiency"; glossary "How
 * it works").  Inputs: q, k, v, the forward output o (o_dtype) and its
 * lse, and the output gradient dO [B,H,Lq,d] (bf16).  Outputs dq [B,H,Lq,d],
 * dk and dv [B,H,Lk,d] (bf16).  P is recomputed from lse; no L x L matrix is
 * stored.  workspace: device memory of at least fa_backward_workspace_size()
 * bytes, 256-byte aligned, owned by the caller; its contents on entry do not
 * matter and on return are unspecified.
 */
int fa_backward(const void* q, const void* k, const void* v, const void* o, const void* dO, const float* lse,
                void* dq, void* dk, void* dv, int B, int H, int Lq, int Lk, int d, float scale, int causal,
                int o_dtype, void* workspace, size_t workspace_bytes, void* stream);

/*
 * fa_backward without a workspace argument, for callers that cannot allocate
 * device memory at all: for example a plugin whose host framework owns every
 * device allocation and offers no workspace hook, or a latency-critical loop in
 * which cudaMalloc's implicit device synchronisation is not acceptable.  The
 * pages have no counterpart to this call; it is a packaging variant of
 * fa_backward.
 *
 * Same arguments, layout and results as fa_backward.  Its scratch (the per-row
 * statistic D, 4 bytes per query row) lives in a statically allocated device
 * array of FA_NOALLOC_MAX_ROWS floats (4 MiB) that every GPU loading this
 * library holds until the process exits.  No call allocates or frees memory.
 *   - B*H*Lq > FA_NOALLOC_MAX_ROWS returns FA_ERR_TOO_LARGE; nothing is launched.
 *   - The first call on a device (with that device current) looks up the
 *     array's device address once; make that first call before any stream
 *     capture.
 *   - Every call on a device shares the one array, and the array keeps the last
 *     call's contents.  Each call writes every D_i it reads before reading it,
 *     so nothing has to start at zero.  Calls whose kernels overlap on the GPU
 *     (for example on two streams at once) race on the array: serialise them.
 */
#define FA_NOALLOC_MAX_ROWS (1 << 20)
int fa_backward_noalloc(const void* q, const void* k, const void* v, const void* o, const void* dO,
                        const float* lse, void* dq, void* dk, void* dv, int B, int H, int Lq, int Lk, int d,
                        float scale, int causal, int o_dtype, void* stream);

/*
 * Workspace bytes fa_decode needs: split-KV partial results (fp32 output
 * vector and LSE per split) for B*H heads and up to ceil(cap / split) splits.
 */
size_t fa_decode_workspace_size(int B, int H, int cap, int d);

/*
 * Single-query decode over a KV cache (the decode phase of "What Is
 * FlashAttention?", "What it changes for you": the cache lives in HBM and is
 * read once).  q [B,H,d] (bf16); kcache, vcache [B,H,cap,d] (bf16); kv_lens
 * int32 [B] on the device, the number of valid cache rows of each sequence.
 * Writes o [B,H,d] (o_dtype) and lse [B,H] (fp32).  d is 64, 128 or 256.  Keys [0, kv_lens[b]) are
 * split into fixed-size chunks processed in parallel; their partial
 * (O, LSE) pairs are merged by a log-sum-exp combine.  A length outside
 * [0, cap] is clamped and flagged as FA_ERR_KV_LEN in the status word; a
 * length of 0 gives o = 0 and lse = -inf.  Slots at or past kv_lens[b] are
 * never read.
 */
int fa_decode(const void* q, const void* kcache, const void* vcache, const int* kv_lens, void* o, float* lse,
              int B, int H, int cap, int d, float scale, int o_dtype, void* workspace, size_t workspace_bytes,
              void* stream);

/*
 * Forward pass over a packed batch of sequences of different lengths (the
 * prefill of a batch of prompts; chunked prefill when a sequence's queries are
 * the last Lq of its Lk keys).  Each sequence is attended to on its own with
 * the same computation as fa_forward ("What FlashAttention does instead",
 * "The Three Running Statistics"); packing sequences end to end is not on the
 * pages.
 *   q [total_q, H, d], k, v [total_k, H, d] (bf16, token-major: row t holds all
 *   heads of token t); cu_seqlens_q, cu_seqlens_k int32 [B+1] on the device:
 *   sequence b owns query rows [cu_q[b], cu_q[b+1]) and key rows
 *   [cu_k[b], cu_k[b+1]), with cu[0] = 0 and cu[B] = total.
 *   max_seqlen_q >= every cu_q[b+1] - cu_q[b] (it sizes the work).
 *   o [total_q, H, d] (o_dtype), lse [H, total_q] fp32.
 * d is 64, 128 or 256.
 * Causal masking is bottom-right per sequence (query i of a sequence sits at
 * key position i + Lk_b - Lq_b) and needs Lq_b <= Lk_b.  q, k, v, o must be
 * 16-byte aligned.  total_q = 0 returns FA_OK without a launch.  On the
 * device, a sequence whose offsets are out of range or decreasing, that is
 * longer than max_seqlen_q rounded up to 256 (128 at d = 256), that has
 * queries but no keys, or
 * (causal) more queries than keys is skipped (its rows are not written) and
 * flagged FA_ERR_SEQLEN in the status word.  Asynchronous on `stream`.
 */
int fa_forward_varlen(const void* q, const void* k, const void* v, void* o, float* lse, const int* cu_seqlens_q,
                      const int* cu_seqlens_k, int B, int H, int total_q, int total_k, int max_seqlen_q, int d,
                      float scale, int causal, int o_dtype, void* stream);

/*
 * Workspace bytes fa_decode_paged needs: the same split-KV partials as
 * fa_decode for B*H query heads and a logical capacity of
 * max_blocks * page_size keys.
 */
size_t fa_decode_paged_workspace_size(int B, int H, int max_blocks, int page_size, int d);

/*
 * Single-query decode over a paged KV cache with grouped key/value heads.
 * Source: "What Is FlashAttention?", "What it changes for you" (the key/value
 * cache of a generation lives in HBM and grows with every token) and "The
 * general lesson" (paged attention named among the data-movement techniques);
 * the attention itself is the same as fa_decode.
 *   q           [B, H, d] bf16.
 *   kpages,
 *   vpages      [num_pages, Hkv, page_size, d] bf16: page p holds page_size
 *               consecutive token positions of one sequence, for every KV head.
 *   block_table int32 [B, max_blocks] on the device: logical key j of sequence
 *               b is row j % page_size of page block_table[b][j / page_size].
 *   kv_lens     int32 [B] on the device, valid keys per sequence.
 *   o, lse      [B, H, d] (o_dtype) and [B, H] fp32.
 * Query head h reads KV head h / (H / Hkv).  H must be a multiple of Hkv and
 * page_size a power of two (1 .. 65536); d is 64, 128 or 256.  q, kpages, vpages and
 * o must be 16-byte aligned, the workspace 256-byte aligned (any torch
 * allocation is).  Lengths outside [0, max_blocks *
 * page_size] are clamped and flagged FA_ERR_KV_LEN; a table entry that a valid
 * key uses and that lies outside [0, num_pages) is flagged FA_ERR_PAGE in the
 * status word and read as page 0, so no read leaves the page pool.  Table
 * entries past a sequence's last used block are never read.  A length of 0
 * gives o = 0 and lse = -inf.  No host synchronisation; asynchronous on `stream`.
 * (Not on the pages: the page layout, the table format and the head grouping
 * follow the common serving convention.)
 */
int fa_decode_paged(const void* q, const void* kpages, const void* vpages, const int* block_table,
                    const int* kv_lens, void* o, float* lse, int B, int H, int Hkv, int num_pages, int page_size,
                    int max_blocks, int d, float scale, int o_dtype, void* workspace, size_t workspace_bytes,
                    void* stream);

/*
 * Forward pass under a block-sparse mask.  The glossary entry's "Common
 * misconceptions" names a block-sparse extension that changes which query/key
 * pairs attend, as distinct from the dense exact calculation; the pages give no
 * mask format, so this is the plainest one: the score matrix of each (b, h) is
 * cut into blocks of FA_BLOCKSPARSE_BLOCK query rows by FA_BLOCKSPARSE_BLOCK
 * keys, and one byte per block permits its pairs (nonzero) or removes them
 * (zero) before the softmax.  A key is permitted for a query row when fa_forward
 * would permit it (length bound, causal mask) AND its block byte is nonzero;
 * the result is the exact softmax attention over the permitted keys.  A row
 * with no permitted key gets O = 0 and LSE = -inf.
 *   q, k, v, o, lse, scale, causal, o_dtype: as fa_forward (d is 64, 128 or 256).
 *   block_mask: DEVICE bytes; the mask of (b, h) is row-major [Tq][Tk] at
 *   block_mask + b * mask_stride_b + h * mask_stride_h, with
 *   Tq = ceil(Lq / 128), Tk = ceil(Lk / 128); strides are in bytes, >= 0
 *   (0 shares one mask across that dimension).  Only bytes inside these
 *   [Tq][Tk] masks are read.  Lk <= 128 * 16384.
 *   workspace: caller-owned device scratch of at least
 *   fa_forward_blocksparse_workspace_size() bytes, 256-byte aligned; it holds
 *   the per-unit lists of key blocks that a small planning kernel builds
 *   before the forward kernel (both launched on `stream`).
 * Blocks whose byte is zero cost no tensor-core work unless the other
 * 128-row query block that shares a 256-row work unit needs them (at d = 256
 * a work unit is a single query block).
 */
#define FA_BLOCKSPARSE_BLOCK 128
size_t fa_forward_blocksparse_workspace_size(int B, int H, int Lq, int Lk);
int fa_forward_blocksparse(const void* q, const void* k, const void* v, void* o, float* lse,
                           const unsigned char* block_mask, long long mask_stride_b, long long mask_stride_h, int B,
                           int H, int Lq, int Lk, int d, float scale, int causal, int o_dtype, void* workspace,
                           size_t workspace_bytes, void* stream);

/*
 * Synchronises the whole current device (every stream: the status word is shared
 * by all of them), then returns the device's status word (FA_OK if no kernel
 * recorded a condition since the last call) and clears it.  `stream` is not used.
 * Returns FA_ERR_CUDA if the synchronisation itself fails.  Must not be called
 * while a stream of the device is being captured.
 *
 * After FA_ERR_TIMEOUT has been recorded, every later kernel of this library on
 * the device sees it when it starts and exits at once without writing its
 * outputs (the calls still return FA_OK); calls compute again once
 * fa_check_status() has returned and cleared the condition.
 */
int fa_check_status(void* stream);

/* Static, human-readable name of a status code. */
const char* fa_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* EXACT_IO_AWARE_FA_H */
