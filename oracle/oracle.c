/*
 * Reference ("oracle") implementation of exact scaled-dot-product attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the plain, slow definition of what the
 * GPU library computes, in double precision, so that the GPU results can be
 * checked against it.  Only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark may load it.  The product path never calls it and has no
 * CPU fallback.  It shares no code, header or constant with the CUDA sources.
 *
 * Sources (web pages on FlashAttention; cited by page title and section):
 *   [G]  "Flash Attention" glossary entry -- "How it works" (queries, keys and
 *        values combined through normalised scores), "Worked example" (the
 *        4,096 x 4,096 score matrix), "Common misconceptions" (exact does not
 *        mean bit-identical).
 *   [W]  "What Is FlashAttention? Why Long Context Got Cheap" -- "The problem it
 *        solves" (the textbook method builds the n x n score matrix, applies
 *        softmax, multiplies by V), "What FlashAttention does instead"
 *        (running max and running sum per row), "What it changes for you"
 *        (the key/value cache kept in HBM during generation) and "The general
 *        lesson" (paged attention named among the data-movement techniques).
 *   [L]  "How Flash Attention Improves Transformer Memory Efficiency Compared
 *        to Standard Attention" -- "The Three Running Statistics" (the m, l and
 *        unnormalised-output update rules and the final division), "Backward
 *        Pass Efficiency" (statistics D_i, l_i, m_i), "Basic Flash Attention
 *        Forward Pass" (shapes (B, H, L, D) and scale = 1/sqrt(D)).
 *
 * Conventions (readings where the pages are silent):
 *   - Layout: every tensor is contiguous row-major [B, H, L, d].
 *   - Scores are t_ij = scale * (q_i . k_j); the mask removes keys before the
 *     softmax.  A key j is permitted for query row i when j < Lk and, under the
 *     causal mask, j <= i + (Lk - Lq) (query i sits at absolute position
 *     i + Lk - Lq, the reading that fits a cached prefix of keys).
 *   - LSE_i = ln sum_j exp(t_ij) over the permitted keys (natural log, in units
 *     of the scaled score).  A row with no permitted key has O_i = 0 and
 *     LSE_i = -inf.
 *   - Inputs may be given as doubles or as bfloat16 bit patterns (uint16); a
 *     bfloat16 value converts to double exactly.
 *
 * Pinned by tests/test_oracle_pins.py against closed forms, limits, a brute
 * force finite-difference gradient and the counts printed in [G] and [W].
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORACLE_F64 0
#define ORACLE_BF16 1

/* bfloat16 is the upper half of an IEEE binary32; widening is exact. */
static double bf16_bits_to_double(uint16_t h) {
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

static double elem(const void* p, int64_t i, int dtype) {
    if (dtype == ORACLE_BF16) return bf16_bits_to_double(((const uint16_t*)p)[i]);
    return ((const double*)p)[i];
}

/* Number of permitted keys for query row i: keys 0 .. n-1 (the causal mask and
 * the length bound both cut a prefix). */
int64_t oracle_permitted_keys(int64_t i, int64_t Lq, int64_t Lk, int causal) {
    int64_t n = Lk;
    if (causal) {
        int64_t last = i + (Lk - Lq);          /* highest permitted key index */
        if (last + 1 < n) n = last + 1;
    }
    return n < 0 ? 0 : n;
}

/* Worked example of [G] and "The problem it solves" of [W]: the number of
 * entries of the B x H x Lq x Lk score matrix the textbook method builds. */
int64_t oracle_score_elements(int64_t B, int64_t H, int64_t Lq, int64_t Lk) {
    return B * H * Lq * Lk;
}

/*
 * One query row, two passes over its permitted keys ([W] "The problem it
 * solves": scores, softmax over the whole row, weighted sum of V rows):
 *   t_j = scale * q . k_j           for j < n
 *   M   = max_j t_j
 *   Z   = sum_j exp(t_j - M)
 *   O   = sum_j (exp(t_j - M) / Z) v_j
 *   LSE = M + ln Z
 * t is caller scratch of length >= n (one score row, never an n x n matrix).
 */
static void attend_row(const void* q, int64_t q_off, const void* k, const void* v,
                       int64_t kv_off, int64_t n, int64_t d, double scale, int dtype,
                       double* t, double* o_row, double* lse_out) {
    for (int64_t c = 0; c < d; ++c) o_row[c] = 0.0;
    if (n <= 0) {
        *lse_out = -INFINITY;
        return;
    }
    double M = -INFINITY;
    for (int64_t j = 0; j < n; ++j) {
        double s = 0.0;
        for (int64_t c = 0; c < d; ++c)
            s += elem(q, q_off + c, dtype) * elem(k, kv_off + j * d + c, dtype);
        t[j] = scale * s;
        if (t[j] > M) M = t[j];
    }
    double Z = 0.0;
    for (int64_t j = 0; j < n; ++j) Z += exp(t[j] - M);
    for (int64_t j = 0; j < n; ++j) {
        double p = exp(t[j] - M) / Z;
        for (int64_t c = 0; c < d; ++c) o_row[c] += p * elem(v, kv_off + j * d + c, dtype);
    }
    *lse_out = M + log(Z);
}

/*
 * Forward pass, all rows: O [B,H,Lq,d] and LSE [B,H,Lq] in double.
 */
void oracle_forward(const void* q, const void* k, const void* v, int dtype,
                    double* o, double* lse, int64_t B, int64_t H, int64_t Lq,
                    int64_t Lk, int64_t d, double scale, int causal) {
    int64_t rows = B * H * Lq;
#pragma omp parallel
    {
        double* t = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < rows; ++r) {
            int64_t bh = r / Lq, i = r % Lq;
            int64_t n = oracle_permitted_keys(i, Lq, Lk, causal);
            attend_row(q, r * d, k, v, bh * Lk * d, n, d, scale, dtype, t, o + r * d,
                       lse + r);
        }
        free(t);
    }
}

/*
 * Forward pass over a packed batch of sequences of different lengths.  The
 * pages' problem statement is per sequence ([W] "The problem it solves"; [L]
 * "Basic Flash Attention Forward Pass" gives one (B, H, L, D) batch); packing
 * sequences of different lengths end to end is not on the pages.  Sequence b
 * owns query rows [cu_q[b], cu_q[b+1]) and key rows [cu_k[b], cu_k[b+1]) of the
 * packed tensors q [total_q, H, d] and k, v [total_k, H, d]; each sequence is
 * attended to on its own, exactly as oracle_forward with Lq = cu_q[b+1] - cu_q[b]
 * and Lk = cu_k[b+1] - cu_k[b] (bottom-right causal alignment).
 * Outputs o [total_q, H, d] and lse [H, total_q].
 */
void oracle_forward_varlen(const void* q, const void* k, const void* v, int dtype, double* o, double* lse,
                           const int32_t* cu_q, const int32_t* cu_k, int64_t B, int64_t H, int64_t total_q,
                           int64_t d, double scale, int causal) {
    int64_t max_k = 1;
    for (int64_t b = 0; b < B; ++b)
        if (cu_k[b + 1] - cu_k[b] > max_k) max_k = cu_k[b + 1] - cu_k[b];
    const int64_t rows = total_q * H;
#pragma omp parallel
    {
        double* t = (double*)malloc(sizeof(double) * (size_t)max_k);
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < rows; ++r) {
            const int64_t h = r % H, row = r / H;  // packed row, head
            int64_t b = 0;
            while (b + 1 < B && cu_q[b + 1] <= row) ++b;
            const int64_t Lq = cu_q[b + 1] - cu_q[b], Lk = cu_k[b + 1] - cu_k[b];
            const int64_t i = row - cu_q[b];
            const int64_t n = oracle_permitted_keys(i, Lq, Lk, causal);
            double* orow = o + (row * H + h) * d;
            for (int64_t c = 0; c < d; ++c) orow[c] = 0.0;
            if (n <= 0) {
                lse[h * total_q + row] = -INFINITY;
                continue;
            }
            double M = -INFINITY;
            for (int64_t j = 0; j < n; ++j) {
                const int64_t krow = ((cu_k[b] + j) * H + h) * d;
                double sdot = 0.0;
                for (int64_t c = 0; c < d; ++c) sdot += elem(q, (row * H + h) * d + c, dtype) * elem(k, krow + c, dtype);
                t[j] = scale * sdot;
                if (t[j] > M) M = t[j];
            }
            double Z = 0.0;
            for (int64_t j = 0; j < n; ++j) Z += exp(t[j] - M);
            for (int64_t j = 0; j < n; ++j) {
                const double pj = exp(t[j] - M) / Z;
                const int64_t vrow = ((cu_k[b] + j) * H + h) * d;
                for (int64_t c = 0; c < d; ++c) orow[c] += pj * elem(v, vrow + c, dtype);
            }
            lse[h * total_q + row] = M + log(Z);
        }
        free(t);
    }
}

/*
 * Forward pass under a block-sparse mask.  [G] "Common misconceptions" names a
 * block-sparse extension that changes which query/key pairs attend, as
 * distinct from the dense exact calculation; the pages give no mask format.
 * Reading: the score matrix of each (b, h) is cut into blocks of block_q query
 * rows by block_k key columns, and a byte per block says whether its pairs may
 * attend (nonzero) or not (zero).  A key j is permitted for query row i when
 * it is permitted by the dense rules (length bound and, with causal set, the
 * bottom-right causal mask) AND its block is nonzero; the result is then the
 * exact softmax attention over the permitted keys, two passes per row as in
 * attend_row.  The mask of (b, h) starts at mask[b * mask_stride_b + h *
 * mask_stride_h] and is row-major [ceil(Lq / block_q)][ceil(Lk / block_k)]
 * (a stride of 0 shares one mask across that dimension).  A row with no
 * permitted key has O = 0 and LSE = -inf.
 */
void oracle_forward_blocksparse(const void* q, const void* k, const void* v, int dtype, double* o,
                                double* lse, const uint8_t* mask, int64_t mask_stride_b,
                                int64_t mask_stride_h, int64_t block_q, int64_t block_k, int64_t B,
                                int64_t H, int64_t Lq, int64_t Lk, int64_t d, double scale, int causal) {
    const int64_t tk = (Lk + block_k - 1) / block_k;  /* key blocks per mask row */
    const int64_t rows = B * H * Lq;
#pragma omp parallel
    {
        double* t = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
        int64_t* keys = (int64_t*)malloc(sizeof(int64_t) * (size_t)(Lk > 0 ? Lk : 1));
#pragma omp for schedule(dynamic, 16)
        for (int64_t r = 0; r < rows; ++r) {
            const int64_t bh = r / Lq, i = r % Lq;
            const int64_t b = bh / H, h = bh % H;
            const uint8_t* mrow = mask + b * mask_stride_b + h * mask_stride_h + (i / block_q) * tk;
            /* the permitted keys of row i, in increasing order */
            const int64_t n_dense = oracle_permitted_keys(i, Lq, Lk, causal);
            int64_t n = 0;
            for (int64_t j = 0; j < n_dense; ++j)
                if (mrow[j / block_k]) keys[n++] = j;
            double* orow = o + r * d;
            for (int64_t c = 0; c < d; ++c) orow[c] = 0.0;
            if (n == 0) {
                lse[r] = -INFINITY;
                continue;
            }
            const int64_t kv_off = bh * Lk * d;
            double M = -INFINITY;
            for (int64_t x = 0; x < n; ++x) {
                double sdot = 0.0;
                for (int64_t c = 0; c < d; ++c)
                    sdot += elem(q, r * d + c, dtype) * elem(k, kv_off + keys[x] * d + c, dtype);
                t[x] = scale * sdot;
                if (t[x] > M) M = t[x];
            }
            double Z = 0.0;
            for (int64_t x = 0; x < n; ++x) Z += exp(t[x] - M);
            for (int64_t x = 0; x < n; ++x) {
                const double p = exp(t[x] - M) / Z;
                for (int64_t c = 0; c < d; ++c) orow[c] += p * elem(v, kv_off + keys[x] * d + c, dtype);
            }
            lse[r] = M + log(Z);
        }
        free(keys);
        free(t);
    }
}

/*
 * Forward pass on a chosen set of rows.  rows[s] is a flat row index
 * (b*H + h)*Lq + i; the result for it goes to o_out[s*d ...] and lse_out[s].
 * Row sampling is exact: each row of the output depends on that query row
 * and all keys/values of its head only.
 */
void oracle_forward_rows(const void* q, const void* k, const void* v, int dtype,
                         const int64_t* rows, int64_t n_rows, double* o_out,
                         double* lse_out, int64_t B, int64_t H, int64_t Lq, int64_t Lk,
                         int64_t d, double scale, int causal) {
    (void)B;
    (void)H;
#pragma omp parallel
    {
        double* t = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t s = 0; s < n_rows; ++s) {
            int64_t r = rows[s];
            int64_t bh = r / Lq, i = r % Lq;
            int64_t n = oracle_permitted_keys(i, Lq, Lk, causal);
            attend_row(q, r * d, k, v, bh * Lk * d, n, d, scale, dtype, t,
                       o_out + s * d, lse_out + s);
        }
        free(t);
    }
}

/*
 * The blockwise recurrence of [L] "The Three Running Statistics", taken
 * literally on one row at a time: start from m = -inf, l = 0, O~ = 0; for each
 * block of `block` keys,
 *   m_new = max(m, max_j t_j)
 *   l    <- exp(m - m_new) l + sum_j exp(t_j - m_new)
 *   O~   <- exp(m - m_new) O~ + sum_j exp(t_j - m_new) v_j
 *   m    <- m_new
 * and finally O = O~ / l.  The running max is carried in scaled-score units.
 * Used only to check that the recurrence reproduces the two-pass result.
 */
void oracle_forward_blockwise(const void* q, const void* k, const void* v, int dtype,
                              double* o, double* lse, int64_t B, int64_t H, int64_t Lq,
                              int64_t Lk, int64_t d, double scale, int causal,
                              int64_t block) {
    int64_t rows = B * H * Lq;
    double* acc = (double*)malloc(sizeof(double) * (size_t)d);
    for (int64_t r = 0; r < rows; ++r) {
        int64_t bh = r / Lq, i = r % Lq;
        int64_t n = oracle_permitted_keys(i, Lq, Lk, causal);
        const int64_t kv_off = bh * Lk * d;
        double m = -INFINITY, l = 0.0;
        for (int64_t c = 0; c < d; ++c) acc[c] = 0.0;
        for (int64_t j0 = 0; j0 < n; j0 += block) {
            int64_t j1 = j0 + block < n ? j0 + block : n;
            double m_new = m;
            for (int64_t j = j0; j < j1; ++j) {
                double s = 0.0;
                for (int64_t c = 0; c < d; ++c)
                    s += elem(q, r * d + c, dtype) * elem(k, kv_off + j * d + c, dtype);
                if (scale * s > m_new) m_new = scale * s;
            }
            double alpha = (m == -INFINITY) ? 0.0 : exp(m - m_new);
            l *= alpha;
            for (int64_t c = 0; c < d; ++c) acc[c] *= alpha;
            for (int64_t j = j0; j < j1; ++j) {
                double s = 0.0;
                for (int64_t c = 0; c < d; ++c)
                    s += elem(q, r * d + c, dtype) * elem(k, kv_off + j * d + c, dtype);
                double p = exp(scale * s - m_new);
                l += p;
                for (int64_t c = 0; c < d; ++c) acc[c] += p * elem(v, kv_off + j * d + c, dtype);
            }
            m = m_new;
        }
        for (int64_t c = 0; c < d; ++c) o[r * d + c] = (n > 0) ? acc[c] / l : 0.0;
        lse[r] = (n > 0) ? m + log(l) : -INFINITY;
    }
    free(acc);
}

/*
 * Backward pass by differentiating the definition row by row ([L] "Backward
 * Pass Efficiency" names the per-row statistic D_i; [G] "How it works" says the
 * probabilities are recomputed rather than stored).  For each row i with its
 * permitted keys j:
 *   P_ij  = exp(t_ij - LSE_i)            (recomputed from the definition)
 *   dP_ij = dO_i . v_j
 *   D_i   = sum_j P_ij dP_ij             (equals dO_i . O_i)
 *   dS_ij = P_ij (dP_ij - D_i)
 *   dQ_i  = scale * sum_j dS_ij k_j
 *   dK_j += scale * dS_ij q_i
 *   dV_j += P_ij dO_i
 * Also returns D [B,H,Lq] when d_out is not NULL.  Parallel over heads only,
 * since every row of a head adds into that head's dK and dV.
 */
void oracle_backward(const void* q, const void* k, const void* v, const void* dO,
                     int dtype, double* dq, double* dk, double* dv, double* d_out,
                     int64_t B, int64_t H, int64_t Lq, int64_t Lk, int64_t d,
                     double scale, int causal) {
    int64_t heads = B * H;
#pragma omp parallel
    {
        double* t = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
        double* p = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
        double* dp = (double*)malloc(sizeof(double) * (size_t)(Lk > 0 ? Lk : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t bh = 0; bh < heads; ++bh) {
            const int64_t kv_off = bh * Lk * d;
            double* dk_h = dk + kv_off;
            double* dv_h = dv + kv_off;
            for (int64_t x = 0; x < Lk * d; ++x) {
                dk_h[x] = 0.0;
                dv_h[x] = 0.0;
            }
            for (int64_t i = 0; i < Lq; ++i) {
                int64_t r = bh * Lq + i;
                int64_t n = oracle_permitted_keys(i, Lq, Lk, causal);
                double* dq_i = dq + r * d;
                for (int64_t c = 0; c < d; ++c) dq_i[c] = 0.0;
                if (n <= 0) {
                    if (d_out) d_out[r] = 0.0;
                    continue;
                }
                double M = -INFINITY;
                for (int64_t j = 0; j < n; ++j) {
                    double s = 0.0;
                    for (int64_t c = 0; c < d; ++c)
                        s += elem(q, r * d + c, dtype) * elem(k, kv_off + j * d + c, dtype);
                    t[j] = scale * s;
                    if (t[j] > M) M = t[j];
                }
                double Z = 0.0;
                for (int64_t j = 0; j < n; ++j) Z += exp(t[j] - M);
                double lse = M + log(Z);
                double D = 0.0;
                for (int64_t j = 0; j < n; ++j) {
                    p[j] = exp(t[j] - lse);
                    double s = 0.0;
                    for (int64_t c = 0; c < d; ++c)
                        s += elem(dO, r * d + c, dtype) * elem(v, kv_off + j * d + c, dtype);
                    dp[j] = s;
                    D += p[j] * dp[j];
                }
                if (d_out) d_out[r] = D;
                for (int64_t j = 0; j < n; ++j) {
                    double ds = p[j] * (dp[j] - D);
                    for (int64_t c = 0; c < d; ++c) {
                        dq_i[c] += scale * ds * elem(k, kv_off + j * d + c, dtype);
                        dk_h[j * d + c] += scale * ds * elem(q, r * d + c, dtype);
                        dv_h[j * d + c] += p[j] * elem(dO, r * d + c, dtype);
                    }
                }
            }
        }
        free(t);
        free(p);
        free(dp);
    }
}

/*
 * Single-query decode over a key/value cache: for each (b, h), the forward
 * pass with one query row and keys [0, kv_lens[b]) of a cache of capacity cap.
 * q [B,H,d], caches [B,H,cap,d], o [B,H,d], lse [B,H].  kv_lens outside
 * [0, cap] are clamped to that range.
 */
void oracle_decode(const void* q, const void* kcache, const void* vcache, int dtype,
                   const int32_t* kv_lens, double* o, double* lse, int64_t B, int64_t H,
                   int64_t cap, int64_t d, double scale) {
    int64_t heads = B * H;
#pragma omp parallel
    {
        double* t = (double*)malloc(sizeof(double) * (size_t)(cap > 0 ? cap : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t bh = 0; bh < heads; ++bh) {
            int64_t n = kv_lens[bh / H];
            if (n < 0) n = 0;
            if (n > cap) n = cap;
            attend_row(q, bh * d, kcache, vcache, bh * cap * d, n, d, scale, dtype, t,
                       o + bh * d, lse + bh);
        }
        free(t);
    }
}

/*
 * Single-query attention over a paged cache.  [W] "What it changes for you":
 * during generation the keys and values of every processed token are kept in
 * a cache in HBM that grows with each token; [W] "The general lesson" names
 * paged attention among the ways of moving less data.  Here a sequence's cache
 * is a list of fixed-size pages: logical key j of sequence b is row
 * j % page_size of page block_table[b * max_blocks + j / page_size].  Pages are
 * laid out [num_pages, Hkv, page_size, d].  Query heads share key/value heads
 * in equal groups: query head h reads KV head h / (H / Hkv).
 * The result is plain attention (as oracle_decode) over keys [0, kv_len_b),
 * kv_len clamped to [0, max_blocks * page_size].
 * Returns 0, or 1 if a page index that a valid key would use is outside
 * [0, num_pages) (nothing is read then), or 2 if H is not a multiple of Hkv.
 */
int oracle_decode_paged(const void* q, const void* kpages, const void* vpages, int dtype,
                        const int32_t* block_table, const int32_t* kv_lens, double* o,
                        double* lse, int64_t B, int64_t H, int64_t Hkv, int64_t num_pages,
                        int64_t page_size, int64_t max_blocks, int64_t d, double scale) {
    if (Hkv <= 0 || H % Hkv != 0 || page_size <= 0) return 2;
    const int64_t group = H / Hkv;
    const int64_t cap = max_blocks * page_size;
    for (int64_t b = 0; b < B; ++b) {
        int64_t n = kv_lens[b];
        if (n < 0) n = 0;
        if (n > cap) n = cap;
        for (int64_t blk = 0; blk * page_size < n; ++blk) {
            const int32_t pg = block_table[b * max_blocks + blk];
            if (pg < 0 || pg >= num_pages) return 1;
        }
    }
    const int64_t heads = B * H;
#pragma omp parallel
    {
        double* t = (double*)malloc(sizeof(double) * (size_t)(cap > 0 ? cap : 1));
#pragma omp for schedule(dynamic, 1)
        for (int64_t bh = 0; bh < heads; ++bh) {
            const int64_t b = bh / H, h = bh % H, g = h / group;
            int64_t n = kv_lens[b];
            if (n < 0) n = 0;
            if (n > cap) n = cap;
            double* orow = o + bh * d;
            for (int64_t c = 0; c < d; ++c) orow[c] = 0.0;
            if (n == 0) {
                lse[bh] = -INFINITY;
                continue;
            }
            double M = -INFINITY;
            for (int64_t j = 0; j < n; ++j) {
                const int64_t pg = block_table[b * max_blocks + j / page_size];
                const int64_t row = ((pg * Hkv + g) * page_size + j % page_size) * d;
                double sdot = 0.0;
                for (int64_t c = 0; c < d; ++c) sdot += elem(q, bh * d + c, dtype) * elem(kpages, row + c, dtype);
                t[j] = scale * sdot;
                if (t[j] > M) M = t[j];
            }
            double Z = 0.0;
            for (int64_t j = 0; j < n; ++j) Z += exp(t[j] - M);
            for (int64_t j = 0; j < n; ++j) {
                const int64_t pg = block_table[b * max_blocks + j / page_size];
                const int64_t row = ((pg * Hkv + g) * page_size + j % page_size) * d;
                const double pj = exp(t[j] - M) / Z;
                for (int64_t c = 0; c < d; ++c) orow[c] += pj * elem(vpages, row + c, dtype);
            }
            lse[bh] = M + log(Z);
        }
        free(t);
    }
    return 0;
}

/*
 * Merge of partial results over disjoint key sets.  Given, for one row, parts
 * s = 0..n-1 with normalised outputs O_s (d each) and LSE_s, the result over
 * the union of the key sets is
 *   LSE = ln sum_s exp(LSE_s)      O = sum_s exp(LSE_s - LSE) O_s .
 * This is the recurrence of [L] "The Three Running Statistics" applied to whole
 * blocks (m = LSE_s, l = 1, O~ = O_s for each part).  Parts with LSE_s = -inf
 * (empty key sets) contribute nothing.
 */
void oracle_merge(const double* o_parts, const double* lse_parts, int64_t n, int64_t d,
                  double* o, double* lse) {
    double M = -INFINITY;
    for (int64_t s = 0; s < n; ++s)
        if (lse_parts[s] > M) M = lse_parts[s];
    for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
    if (M == -INFINITY) {
        *lse = -INFINITY;
        return;
    }
    double Z = 0.0;
    for (int64_t s = 0; s < n; ++s) Z += exp(lse_parts[s] - M);
    double L = M + log(Z);
    for (int64_t s = 0; s < n; ++s) {
        double w = exp(lse_parts[s] - L);
        for (int64_t c = 0; c < d; ++c) o[c] += w * o_parts[s * d + c];
    }
    *lse = L;
}

int oracle_num_threads(void) {
    int n = 1;
#pragma omp parallel
    {
#pragma omp single
        {
#ifdef _OPENMP
            n = omp_get_num_threads();
#endif
        }
    }
    return n;
}

/* Threads of the following parallel regions (timing only; results do not depend on it). */
void oracle_set_num_threads(int n) {
#ifdef _OPENMP
    if (n > 0) omp_set_num_threads(n);
#else
    (void)n;
#endif
}
