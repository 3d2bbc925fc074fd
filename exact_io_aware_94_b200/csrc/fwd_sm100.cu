// Forward pass of exact attention for sm_100a.
//
// Follows the blockwise method of the pages (glossary "How it works"; "What
// FlashAttention does instead"; "The Three Running Statistics"): for each
// query tile, stream K/V tiles through on-chip memory, compute the score tile,
// update the running max m and running sum l per row, rescale the unnormalised
// output O~ when the max moves, accumulate P~ V, and divide by l at the end.
//
// B200 mapping.  A work unit is 256 query rows of one (b, h): two 128-row Q
// tiles, one per softmax warpgroup.  The kernel is persistent (one CTA per SM)
// and claims units one at a time from its stream's ticket counter, in a fixed
// heavy-first order, so the CTAs finish within a unit of one another (under
// graph capture, a static snake-ordered deal of the same order instead).  The
// producer warp claims each unit and hands it to the other roles through a
// small ring in shared memory.  Each warpgroup's Q tile of
// the next unit is loaded as soon as that warpgroup's last S MMA of the current
// unit is done with the buffer, and a K slot is refilled once its S MMAs are
// done (a V slot once its PV MMAs are), so loads, MMAs and the epilogue of
// consecutive units overlap.
//   warp 8      TMA producer: Q tiles per unit, K_j / V_j through a smem ring.
//   warp 9      MMA issuer: S_w = Q_w K_j^T into TMEM (SS MMA),
//               O_w += P_w V_j with P_w read from TMEM (TS MMA), for both
//               warpgroups in a fixed alternating order.
//   warps 9, 10 block-sparse kernel only: one MMA issuer per softmax
//               warpgroup (w = warp - 9), so a query block whose key-block
//               list is shorter or sparser never waits behind the other's
//               entries; the two meet only at the K/V ring.
//               In the producer and issuer warps the whole warp runs the
//               control flow and one lane chosen by elect.sync issues each
//               copy or MMA: the operands then stay warp-uniform, which keeps
//               the issue cost per MMA well under the MMA's own 64 cycles.
//   warps 10-11 otherwise idle (they complete the third warpgroup, whose
//               registers setmaxnreg hands to the softmax warpgroups).
//   warps 0-3   softmax warpgroup 0 (rows 0..127 of the unit), warps 4-7
//               warpgroup 1 (rows 128..255).  One thread owns one row: it loads
//               its score row from TMEM, applies the mask, updates m and l,
//               rescales its O~ row in TMEM when needed, writes bf16 P~ back
//               over its score row for the PV MMA, and finally stores O, LSE.
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+d) O1 [256+d,256+2d).
//
// Rescaling is deferred while the running max has grown by no more than
// 2^kRescaleLog2 in exp2 units: O = O~ / l holds for any common reference
// value, so the result is unchanged; only overflow headroom is spent.
// The LSE uses the running sum of the unrounded P~.  O is normalised by that
// sum plus, per tile, the bf16 rounding error of the tile's largest P~ (the
// term that dominates a peaky row), so numerator and denominator weigh the
// dominant key alike.  P~ is handed to the MMA in two halves of 64 keys.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fa_internal.h"
#include "ptx.cuh"

namespace fa {
namespace {

constexpr float kRescaleLog2 = 8.0f;
constexpr int kUnitRing = 4;  // units published ahead by the producer

#ifdef FA_TEST_HOOKS
// One-shot fault (test build only): the next K tile a producer would load is
// skipped -- neither its expected byte count nor its copy is issued -- so the
// MMA warp's wait for it runs out.
__device__ int g_test_skip_k;
#endif



template <int D>
struct FwdLayout {
    static constexpr int kBoxBytes = 128 * 64 * 2;     // one TMA box: 128 rows x 64 bf16
    static constexpr int kBoxes = D / 64;              // boxes per 128-row tile
    static constexpr int kTileBytes = kBoxBytes * kBoxes;
    static constexpr int kStages = (D == 128) ? 2 : 4;  // K/V ring depth
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kQOff + 2 * kTileBytes;
    static constexpr int kVOff = kKOff + kStages * kTileBytes;
    static constexpr int kBarOff = kVOff + kStages * kTileBytes;
    // barriers: q[2], q_free[2], k[S], v[S], k_free[S], v_free[S], s[2], p[2][2 halves], o[2], o_free[2],
    // drain[2]
    static constexpr int kNumBars = 4 + 4 * kStages + 10 + 2 + 2 * 4;  // + unit ring full/free
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    // unit ring: 4 unit indices, 4 int4 block-sparse metadata, 4 decoded units (32 bytes each)
    static constexpr int kRingOff = kMiscOff + 16;
    // epilogue staging for the O tile stores: 4 KB per softmax warp (32 rows x 128 bytes,
    // 128-byte swizzle, so 1024-byte aligned)
    static constexpr int kStageOff = (kRingOff + 16 + 64 + 128 + 1023) / 1024 * 1024;
    static constexpr int kBytes = kStageOff + 8 * 4096 + 1024;  // + alignment slack
};

// One work unit: which (b*H + h), which pair of 128-row tiles, how many KV tiles each needs,
// and where its sequence lives (packed first rows and lengths; 0, 0, Lq, Lk for a batched call).
struct Unit {
    int bh, i0, n_kv0, n_kv1;
    int q0, k0, lq, lk;
};

// Units in a fixed global order: the (b, h) pairs are taken in groups of
// p.head_group heads whose K and V fit in L2 together; within a group, longest
// causal rows first (pair index descending), heads interleaved.  At any time the
// CTAs then read the K/V of about one group, which stays in L2, and the last
// units of the launch are still the shortest.
__device__ __forceinline__ void unit_pair_head(const FwdParams& p, int u, int n_pairs, int& pair, int& bh) {
    const int BH = p.B * p.H;
    const int G = p.head_group;
    const int grp = u / (G * n_pairs);
    const int r = u - grp * G * n_pairs;
    const int gsz = min(G, BH - grp * G);  // heads in this group (the last one may be short)
    pair = n_pairs - 1 - r / gsz;
    bh = grp * G + r % gsz;
}

__device__ __forceinline__ Unit unit_of(const FwdParams& p, int u) {
    const int n_pairs = (p.Lq + kFwdRowsPerCta - 1) / kFwdRowsPerCta;
    Unit r;
    int pair;
    unit_pair_head(p, u, n_pairs, pair, r.bh);
    r.i0 = pair * kFwdRowsPerCta;
    const int n_kv_all = (p.Lk + kFwdBN - 1) / kFwdBN;
    const int off = p.Lk - p.Lq;  // causal: query i sits at key position i + off
    int n[2];
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        const int first = r.i0 + w * kFwdBM;
        if (first >= p.Lq) {
            n[w] = 0;
        } else if (p.causal) {
            const int last = min(first + kFwdBM - 1, p.Lq - 1);
            n[w] = min(n_kv_all, (last + off) / kFwdBN + 1);
        } else {
            n[w] = n_kv_all;
        }
    }
    r.n_kv0 = n[0];
    r.n_kv1 = n[1];
    r.q0 = 0;
    r.k0 = 0;
    r.lq = p.Lq;
    r.lk = p.Lk;
    return r;
}

// Packed variable-length batch: unit u is (pair, b*H + h) in a virtual space of
// max_pairs pairs per (b, h), longest causal rows first.  Units past a
// sequence's end are empty (no KV tiles).  A sequence whose offsets are out of
// range or decreasing, that is longer than max_pairs * 256 rows, that has
// queries but no keys, or (causal) more queries than keys is skipped and
// flagged FA_ERR_SEQLEN (once, from its pair-0 unit).
__device__ __forceinline__ Unit unit_of_varlen(const FwdParams& p, int u) {
    const int BH = p.B * p.H;
    Unit r;
    const int pair = p.max_pairs - 1 - u / BH;
    r.bh = u % BH;
    r.i0 = pair * kFwdRowsPerCta;
    r.n_kv0 = 0;
    r.n_kv1 = 0;
    const int b = r.bh / p.H;
    const int q0 = p.cu_q[b], q1 = p.cu_q[b + 1], k0 = p.cu_k[b], k1 = p.cu_k[b + 1];
    r.q0 = q0;
    r.k0 = k0;
    r.lq = q1 - q0;
    r.lk = k1 - k0;
    const bool bad = q0 < 0 || q1 < q0 || q1 > p.Lq || k0 < 0 || k1 < k0 || k1 > p.Lk ||
                     r.lq > p.max_pairs * kFwdRowsPerCta || (r.lq > 0 && r.lk == 0) || (p.causal && r.lq > r.lk);
    if (bad) {
        if (pair == 0) atomicCAS(p.status, 0, FA_ERR_SEQLEN);
        r.lq = 0;
        return r;
    }
    const int n_kv_all = (r.lk + kFwdBN - 1) / kFwdBN;
    const int off = r.lk - r.lq;
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        const int first = r.i0 + w * kFwdBM;
        int n = 0;
        if (first < r.lq)
            n = p.causal ? min(n_kv_all, (min(first + kFwdBM - 1, r.lq - 1) + off) / kFwdBN + 1) : n_kv_all;
        if (w == 0) r.n_kv0 = n; else r.n_kv1 = n;
    }
    return r;
}

// Block-sparse: the batched unit order.  The producer and the MMA issuer walk the unit's
// union list of key blocks (planned before the launch, at least one entry); each entry's
// bits say which query block takes part in it.
__device__ __forceinline__ size_t bsparse_index(const FwdParams& p, int bh, int i0) {
    const int n_pairs = (p.Lq + kFwdRowsPerCta - 1) / kFwdRowsPerCta;
    return static_cast<size_t>(bh) * n_pairs + i0 / kFwdRowsPerCta;
}

// meta: the unit's bs_meta entry (its first field is the union-list length).
__device__ __forceinline__ Unit unit_of_bsparse(const FwdParams& p, int u, const int4& meta) {
    const int n_pairs = (p.Lq + kFwdRowsPerCta - 1) / kFwdRowsPerCta;
    Unit r;
    int pair;
    unit_pair_head(p, u, n_pairs, pair, r.bh);
    r.i0 = pair * kFwdRowsPerCta;
    const int cnt = meta.x;
    r.n_kv0 = cnt;
    r.n_kv1 = (r.i0 + kFwdBM < p.Lq) ? cnt : 0;
    r.q0 = 0;
    r.k0 = 0;
    r.lq = p.Lq;
    r.lk = p.Lk;
    return r;
}

// The planned union list of a block-sparse unit.
__device__ __forceinline__ const uint16_t* bsparse_list(const FwdParams& p, const Unit& un) {
    return p.bs_list + bsparse_index(p, un.bh, un.i0) * p.bs_tk;
}

// Unit u, decoded by the producer (block-sparse units need their metadata, meta);
// the producer publishes it with the unit index.
template <bool VARLEN, bool BSPARSE>
__device__ __forceinline__ Unit get_unit(const FwdParams& p, int u, const int4& meta) {
    if constexpr (VARLEN) return unit_of_varlen(p, u);
    else if constexpr (BSPARSE) return unit_of_bsparse(p, u, meta);
    else return unit_of(p, u);
}

// A unit as published by the producer.  A batched unit's sequence fields are the
// launch's own (0, 0, Lq, Lk): taking them from the parameters keeps them out of
// the registers of the consumers' loops.
template <bool VARLEN>
__device__ __forceinline__ Unit read_unit(const FwdParams& p, const Unit* slot) {
    Unit r;
    r.bh = slot->bh;
    r.i0 = slot->i0;
    r.n_kv0 = slot->n_kv0;
    r.n_kv1 = slot->n_kv1;
    if constexpr (VARLEN) {
        r.q0 = slot->q0;
        r.k0 = slot->k0;
        r.lq = slot->lq;
        r.lk = slot->lk;
    } else {
        r.q0 = 0;
        r.k0 = 0;
        r.lq = p.Lq;
        r.lk = p.Lk;
    }
    return r;
}

// The block-sparse metadata of unit u (read by the producer only).
__device__ __forceinline__ int4 bsparse_meta_of(const FwdParams& p, int u) {
    const int n_pairs = (p.Lq + kFwdRowsPerCta - 1) / kFwdRowsPerCta;
    int pair, bh;
    unit_pair_head(p, u, n_pairs, pair, bh);
    return __ldg(p.bs_meta + bsparse_index(p, bh, pair * kFwdRowsPerCta));
}

// Entry j of a unit's key-block list, read 32 entries at a time by the whole
// warp (one coalesced load per 32 entries) and handed out by shuffle.  j must be
// warp-uniform and visited in increasing order; n is the list's length.
struct ListWindow {
    int base = -32;
    uint32_t ent = 0;
    __device__ __forceinline__ int get(const uint16_t* lst, int j, int n) {
        const int b = j & ~31;
        if (b != base) {
            base = b;
            const int lane = threadIdx.x & 31;
            ent = (b + lane < n) ? __ldg(lst + b + lane) : 0u;
        }
        return static_cast<int>(__shfl_sync(0xffffffffu, ent, j & 31));
    }
};

template <int D, bool VARLEN, bool BSPARSE>
__global__ void __launch_bounds__(kFwdThreads, 1) fa_fwd_kernel(const __grid_constant__ FwdParams p) {
    using Lay = FwdLayout<D>;
    constexpr int S = Lay::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + Lay::kQOff;
    uint8_t* sK = smem + Lay::kKOff;
    uint8_t* sV = smem + Lay::kVOff;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
    uint64_t* bar_q = bars;           // [w]: Q_w landed
    uint64_t* bar_q_free = bars + 2;  // [w]: the S MMAs of warpgroup w's unit are done with Q_w
    uint64_t* bar_k = bars + 4;
    uint64_t* bar_v = bars + 4 + S;
    // A K slot is free once the S MMAs that read it are done, a V slot once the
    // PV MMAs are: K runs a tile further ahead than V.
    uint64_t* bar_kfree = bars + 4 + 2 * S;
    uint64_t* bar_vfree = bars + 4 + 3 * S;
    uint64_t* bar_s = bars + 4 + 4 * S;
    uint64_t* bar_p = bar_s + 2;  // [2 * w + half]
    uint64_t* bar_o = bar_p + 4;
    uint64_t* bar_ofree = bar_o + 2;
    uint64_t* bar_drain = bar_ofree + 2;  // [i]: MMA issuer i's last MMAs are done
    // Unit ring: the producer claims units from the launch's ticket counter and
    // publishes them here; the MMA warp(s) and the 8 softmax warps read each entry.
    uint64_t* bar_ufull = bar_drain + 2;
    uint64_t* bar_ufree = bar_ufull + kUnitRing;
    volatile int* s_unit = reinterpret_cast<volatile int*>(smem + Lay::kRingOff);
    int4* s_meta = reinterpret_cast<int4*>(smem + Lay::kRingOff + 16);  // block-sparse unit metadata
    // The producer decodes each unit once and publishes it here.  The consumers' own
    // decodes (integer divisions; for a packed batch, sequence offsets read from global
    // memory) sat on the critical path at every unit boundary.
    Unit* s_units = reinterpret_cast<Unit*>(smem + Lay::kRingOff + 80);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_units = p.B * p.H * (VARLEN ? p.max_pairs : (p.Lq + kFwdRowsPerCta - 1) / kFwdRowsPerCta);

    // ---- setup
    if (threadIdx.x == 0) {
        for (int w = 0; w < 2; ++w) {
            mbar_init(&bar_q[w], 1);
            mbar_init(&bar_q_free[w], 1);
        }
        for (int s = 0; s < S; ++s) {
            mbar_init(&bar_k[s], 1);
            mbar_init(&bar_v[s], 1);
            // block-sparse: one arrival from each of the two MMA issuers
            mbar_init(&bar_kfree[s], BSPARSE ? 2 : 1);
            mbar_init(&bar_vfree[s], BSPARSE ? 2 : 1);
        }
        for (int w = 0; w < 2; ++w) {
            mbar_init(&bar_s[w], 1);
            mbar_init(&bar_p[2 * w], 4 * 32);
            mbar_init(&bar_p[2 * w + 1], 4 * 32);
            mbar_init(&bar_o[w], 1);
            mbar_init(&bar_ofree[w], 4 * 32);
        }
        mbar_init(&bar_drain[0], 1);
        mbar_init(&bar_drain[1], 1);
        for (int r = 0; r < kUnitRing; ++r) {
            mbar_init(&bar_ufull[r], 1);
            mbar_init(&bar_ufree[r], (BSPARSE ? 2 : 1) + 8);  // MMA warp(s) + 8 softmax warps
        }
        *abort_flag = (atomicAdd(p.status, 0) == FA_ERR_TIMEOUT) ? 1 : 0;
        fence_barrier_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if (warp == 8 && lane == 0) {
        tma_prefetch_desc(&p.tm_q);
        tma_prefetch_desc(&p.tm_k);
        tma_prefetch_desc(&p.tm_v);
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    // Registers move from the TMA/MMA warpgroup (warps 8-11) to the softmax
    // warpgroups (warps 0-7); each setmaxnreg sits in its own role's branch.
    if (warp >= 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kFwdRegsOther));
    }
    if (warp == 8) {
        // ================= TMA producer =================
        // The whole warp runs the loop; one elected lane issues each copy.
        auto wait = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.status));
        };
        if (!*abort_flag) {
            int kc = 0;                // K/V tiles started so far (ring position)
            int nk = 0, nv = 0;        // K and V tiles whose loads were issued
            int q_iter[2] = {0, 0};    // Q tiles requested per warpgroup
            unsigned claims = 0;       // units claimed by this CTA (static deal)
            int skipped_k = -1;        // test build: ring position of a K tile never loaded
            bool ok = true;
            for (int it = 0; ok; ++it) {
                // claim the next unit (heavy-first order) and publish it
                const int rs = it % kUnitRing;
                if (it >= kUnitRing && !(ok = wait(&bar_ufree[rs], ((it / kUnitRing) - 1) & 1))) break;
                int u;
                Unit un;
                int4 meta = make_int4(0, 0, 0, 0);
                for (;;) {  // a packed batch's virtual units past a sequence's end are skipped here
                    unsigned int ticket = 0;
                    if (p.sched) {
                        if (lane == 0) ticket = atomicAdd(p.sched, 1u);
                        ticket = __shfl_sync(0xffffffffu, ticket, 0);
                    } else {
                        // static deal: claim k of CTA c is unit k*G + c, snake-ordered
                        const unsigned G = gridDim.x, k = claims++;
                        ticket = k * G + ((k & 1u) ? G - 1u - blockIdx.x : blockIdx.x);
                    }
                    u = static_cast<int>(min(ticket, static_cast<unsigned>(n_units)));
                    if (u >= n_units) break;
                    if constexpr (BSPARSE) meta = bsparse_meta_of(p, u);
                    un = get_unit<VARLEN, BSPARSE>(p, u, meta);
                    if (!VARLEN || un.n_kv0 > 0 || un.n_kv1 > 0) break;
                }
                if (lane == 0) {
                    s_unit[rs] = u;
                    if constexpr (BSPARSE) s_meta[rs] = meta;
                    if (u < n_units) s_units[rs] = un;
                    mbar_arrive(&bar_ufull[rs]);
                }
                __syncwarp();
                if (u >= n_units) break;
                const int n_max = max(un.n_kv0, un.n_kv1);
                // Q_w as soon as warpgroup w's S MMAs of its previous unit are done with the
                // buffer (under a causal mask warpgroup 0 lets go of it a tile earlier).
                // Order Q_0, K_0, Q_1, V_0, K_1, ...
                auto load_q = [&](int w) -> bool {
                    if (q_iter[w] > 0 && !wait(&bar_q_free[w], (q_iter[w] - 1) & 1)) return false;
                    mbar_arrive_expect_tx_w(&bar_q[w], Lay::kTileBytes);
                    // batched maps are [B*H][L][d]; packed maps are [total][H][d]
                    const int cy = VARLEN ? un.bh % p.H : un.i0 + w * kFwdBM;
                    const int cz = VARLEN ? un.q0 + un.i0 + w * kFwdBM : un.bh;
                    for (int b = 0; b < Lay::kBoxes; ++b)
                        tma_load_3d_w(sQ + w * Lay::kTileBytes + b * Lay::kBoxBytes, &p.tm_q, &bar_q[w], b * 64, cy,
                                      cz);
                    ++q_iter[w];
                    return true;
                };
                if (!(ok = load_q(0))) break;
                const uint16_t* bs_list = nullptr;
                if constexpr (BSPARSE) bs_list = bsparse_list(p, un);
                ListWindow lw;
                for (int j = 0; j < n_max; ++j, ++kc) {
                    const int s = kc % S;
                    int kvt = j;  // key block loaded as the unit's j-th tile
                    if constexpr (BSPARSE) kvt = lw.get(bs_list, j, n_max) & kBsEntryTile;
                    if (kc >= S && !(ok = wait(&bar_kfree[s], ((kc / S) - 1) & 1))) break;
                    const int ky = VARLEN ? un.bh % p.H : kvt * kFwdBN;
                    const int kz = VARLEN ? un.k0 + j * kFwdBN : un.bh;
                    bool skip = false;
#ifdef FA_TEST_HOOKS
                    int armed = 0;
                    if (lane == 0) armed = atomicExch(&g_test_skip_k, 0);
                    skip = __shfl_sync(0xffffffffu, armed, 0) != 0;
                    if (skip) skipped_k = kc;
#endif
                    if (!skip) {
                        mbar_arrive_expect_tx_w(&bar_k[s], Lay::kTileBytes);
                        for (int b = 0; b < Lay::kBoxes; ++b)
                            tma_load_3d_w(sK + s * Lay::kTileBytes + b * Lay::kBoxBytes, &p.tm_k, &bar_k[s], b * 64,
                                          ky, kz);
                    }
                    ++nk;
                    if (j == 0 && un.n_kv1 > 0 && !(ok = load_q(1))) break;
                    if (kc >= S && !(ok = wait(&bar_vfree[s], ((kc / S) - 1) & 1))) break;
                    mbar_arrive_expect_tx_w(&bar_v[s], Lay::kTileBytes);
                    for (int b = 0; b < Lay::kBoxes; ++b)
                        tma_load_3d_w(sV + s * Lay::kTileBytes + b * Lay::kBoxBytes, &p.tm_v, &bar_v[s], b * 64, ky,
                                      kz);
                    ++nv;
                }
            }
            // Every copy this warp issued lands before the CTA's shared memory goes
            // away, also when a wait elsewhere in the CTA ran out after this loop
            // ended.  (Each barrier waited on here is at the phase of its last copy.)
            for (int w = 0; w < 2; ++w)
                if (q_iter[w] > 0) mbar_wait_drain(&bar_q[w], (q_iter[w] - 1) & 1, p.status);
            for (int t = max(0, nk - S); t < nk; ++t)
                if (t != skipped_k) mbar_wait_drain(&bar_k[t % S], (t / S) & 1, p.status);
            for (int t = max(0, nv - S); t < nv; ++t) mbar_wait_drain(&bar_v[t % S], (t / S) & 1, p.status);
        }
    } else if (!BSPARSE && warp == 9) {
        // ================= MMA issuer (dense and packed kernels) =================
        // One issuer for both warpgroups, in the fixed order PV0(j), S0(j+1), PV1(j),
        // S1(j+1): the two softmax warpgroups stay half a tile period apart, so their
        // exponential phases do not collide and the tensor pipe alternates between
        // them.  (Two free-running issuers measured 9-26% slower here.)
        // The whole warp runs the loop, so descriptors and TMEM addresses are
        // warp-uniform; one elected lane issues each MMA and commit.
        auto wait = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.status));
        };
        {
            constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 0, 1);
            const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
            auto issue_s = [&](int w, int s) {
                const uint32_t t_s = tmem_base + w * 128;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * Lay::kBoxBytes + (kk & 3) * 32;
                    const uint64_t a = smem_desc_sw128(sQa + w * Lay::kTileBytes + koff, 16, 1024);
                    const uint64_t b = smem_desc_sw128(sKa + s * Lay::kTileBytes + koff, 16, 1024);
                    umma_ss_w(t_s, a, b, kIdescQK, kk > 0 ? 1u : 0u);
                }
                umma_commit_w(&bar_s[w]);
            };
            // PV for one half of the tile's keys (h = 0: keys 0-63, h = 1: keys 64-127);
            // the warpgroup's first PV of a unit overwrites O_w.
            auto issue_pv_half = [&](int w, int s, bool first, int h) {
                const uint32_t t_p = tmem_base + w * 128;
                const uint32_t t_o = tmem_base + 256 + w * D;
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    const int kk = h * 4 + k4;
                    const uint64_t b =
                        smem_desc_sw128(sVa + s * Lay::kTileBytes + kk * 2048, Lay::kBoxBytes, 1024);
                    umma_ts_w(t_o, t_p + kk * 8, b, kIdescPV, (!first || kk > 0) ? 1u : 0u);
                }
            };
            int kc = 0;                // K/V ring position
            int q_iter[2] = {0, 0};    // Q tiles consumed per warpgroup
            int tp[2] = {0, 0};        // P tiles consumed per warpgroup
            int units_w[2] = {0, 0};   // units whose O_w was handed to the epilogue
            bool ok = true;
            for (int it = 0; ok; ++it) {
                const int rs = it % kUnitRing;
                if (!(ok = wait(&bar_ufull[rs], (it / kUnitRing) & 1))) break;
                const int u = s_unit[rs];
                const Unit un = read_unit<VARLEN>(p, &s_units[rs]);  // read before the slot is handed back
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_ufree[rs]);
                if (u >= n_units) break;
                const int n0 = un.n_kv0, n1 = un.n_kv1;
                const int n_max = max(n0, n1);
                if (!(ok = wait(&bar_k[kc % S], (kc / S) & 1))) break;
                tc_fence_after();
                if (!(ok = wait(&bar_q[0], q_iter[0] & 1))) break;
                ++q_iter[0];
                tc_fence_after();
                issue_s(0, kc % S);
                if (n0 == 1) umma_commit_w(&bar_q_free[0]);
                if (n1 > 0) {
                    if (!(ok = wait(&bar_q[1], q_iter[1] & 1))) break;
                    ++q_iter[1];
                    tc_fence_after();
                    issue_s(1, kc % S);
                    if (n1 == 1) umma_commit_w(&bar_q_free[1]);
                }
                umma_commit_w(&bar_kfree[kc % S]);
                for (int j = 0; ok && j < n_max; ++j) {
                    const int s = (kc + j) % S;
                    const int s1 = (kc + j + 1) % S;
                    if (!(ok = wait(&bar_v[s], ((kc + j) / S) & 1))) break;
                    bool k_ready = false;
#pragma unroll
                    for (int w = 0; w < 2; ++w) {
                        const int nw = (w == 0) ? n0 : n1;
                        if (j < nw) {
                            if (j == 0 && units_w[w] > 0) {
                                // O_w still holds the previous unit until its epilogue has read it
                                if (!(ok = wait(&bar_ofree[w], (units_w[w] - 1) & 1)))
                                    break;
                            }
                            if (!(ok = wait(&bar_p[2 * w], tp[w] & 1))) break;
                            tc_fence_after();
                            issue_pv_half(w, s, j == 0, 0);
                            if (!(ok = wait(&bar_p[2 * w + 1], tp[w] & 1))) break;
                            ++tp[w];
                            tc_fence_after();
                            issue_pv_half(w, s, j == 0, 1);
                            if (j == nw - 1) {
                                umma_commit_w(&bar_o[w]);
                                ++units_w[w];
                            }
                        }
                        if (j + 1 < nw) {
                            if (!k_ready) {
                                if (!(ok = wait(&bar_k[s1], ((kc + j + 1) / S) & 1)))
                                    break;
                                tc_fence_after();
                                k_ready = true;
                            }
                            issue_s(w, s1);
                            if (j + 2 == nw) umma_commit_w(&bar_q_free[w]);  // last S_w of this unit issued
                        }
                    }
                    if (!ok) break;
                    if (j + 1 < n_max) umma_commit_w(&bar_kfree[s1]);
                    umma_commit_w(&bar_vfree[s]);
                }
                kc += n_max;
            }
            // Drain: every MMA issued by this thread completes before TMEM is freed.
            umma_commit_w(&bar_drain[0]);
            mbar_wait_drain(&bar_drain[0], 0, p.status);
        }
    } else if (BSPARSE && (warp == 9 || warp == 10)) {
        // ================= MMA issuers (block-sparse kernel): warp 9 for warpgroup 0, warp 10 for 1 ======
        // Each issuer serves one softmax warpgroup, so neither waits on the other's
        // softmax or epilogue; they meet only at the K/V ring, whose free barriers
        // take one arrival from each.  The whole warp runs the loop, so descriptors
        // and TMEM addresses are warp-uniform; one elected lane issues each MMA,
        // commit and arrival (tcgen05.commit tracks the MMAs of the issuing thread).
        const int w = warp - 9;
        auto wait = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.status));
        };
        auto arrive1 = [&](uint64_t* bar) {
            if (lane == 0) mbar_arrive(bar);
            __syncwarp();
        };
        {
            constexpr uint32_t kIdescQK = idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t kIdescPV = idesc_bf16_f32(128, D, 0, 1);
            const uint32_t sQa = smem_u32(sQ) + w * Lay::kTileBytes, sKa = smem_u32(sK), sVa = smem_u32(sV);
            const uint32_t t_s = tmem_base + w * 128;       // S_w, and P_w over it
            const uint32_t t_o = tmem_base + 256 + w * D;   // O_w
            // S_w = Q_w K_s^T into TMEM
            auto issue_s = [&](int s) {
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * Lay::kBoxBytes + (kk & 3) * 32;
                    const uint64_t a = smem_desc_sw128(sQa + koff, 16, 1024);
                    const uint64_t b = smem_desc_sw128(sKa + s * Lay::kTileBytes + koff, 16, 1024);
                    umma_ss_w(t_s, a, b, kIdescQK, kk > 0 ? 1u : 0u);
                }
                umma_commit_w(&bar_s[w]);
            };
            // PV for one half of the tile's keys (h = 0: keys 0-63, h = 1: keys 64-127);
            // the first PV of a unit overwrites O_w.
            auto issue_pv_half = [&](int s, bool first, int h) {
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    const int kk = h * 4 + k4;
                    const uint64_t b =
                        smem_desc_sw128(sVa + s * Lay::kTileBytes + kk * 2048, Lay::kBoxBytes, 1024);
                    umma_ts_w(t_o, t_s + kk * 8, b, kIdescPV, (!first || kk > 0) ? 1u : 0u);
                }
            };
            int kc = 0;        // ring position of the unit's first K/V tile
            int q_iter = 0;    // Q_w tiles consumed
            int tp = 0;        // P_w tiles consumed
            int units_w = 0;   // units whose O_w was handed to the epilogue
            bool ok = true;
            for (int it = 0; ok; ++it) {
                const int rs = it % kUnitRing;
                if (!(ok = wait(&bar_ufull[rs], (it / kUnitRing) & 1))) break;
                const int u = s_unit[rs];
                const int4 meta = s_meta[rs];  // read before the slot is handed back
                const Unit un = read_unit<VARLEN>(p, &s_units[rs]);
                __syncwarp();
                if (lane == 0) mbar_arrive(&bar_ufree[rs]);
                if (u >= n_units) break;
                // The unit's K/V tiles occupy ring positions kc .. kc + n_pos - 1; this
                // warpgroup uses some of them (dense: the first n_w; block-sparse: the
                // union-list entries with its bit), the last one at position `last`.
                int n_pos, last;
                const uint16_t* lst = nullptr;
                ListWindow lw;
                if constexpr (BSPARSE) {
                    n_pos = meta.x;
                    last = w == 0 ? meta.y : meta.z;
                    lst = bsparse_list(p, un);
                } else {
                    n_pos = max(un.n_kv0, un.n_kv1);
                    last = (w == 0 ? un.n_kv0 : un.n_kv1) - 1;
                }
                auto uses = [&](int j) -> bool {
                    if constexpr (BSPARSE) return j <= last && ((lw.get(lst, j, n_pos) >> (14 + w)) & 1);
                    else return j <= last;
                };
                // A position this warpgroup does not use still needs its arrivals on the
                // free barriers; waiting for the tile's load first keeps each arrival in
                // that position's phase (the load follows the previous phase of the slot).
                auto skip = [&](int j) -> bool {
                    const int pos = kc + j, s = pos % S;
                    if (!wait(&bar_k[s], (pos / S) & 1)) return false;
                    arrive1(&bar_kfree[s]);
                    if (!wait(&bar_v[s], (pos / S) & 1)) return false;
                    arrive1(&bar_vfree[s]);
                    return true;
                };
                // S for used position j: Q_w comes with the unit's first S, and the last S
                // of the unit releases Q_w to the producer.
                bool q_seen = false;
                auto issue_s_at = [&](int j) -> bool {
                    const int pos = kc + j, s = pos % S;
                    if (!wait(&bar_k[s], (pos / S) & 1)) return false;
                    if (!q_seen) {
                        if (!wait(&bar_q[w], q_iter & 1)) return false;
                        ++q_iter;
                        q_seen = true;
                    }
                    tc_fence_after();
                    issue_s(s);
                    umma_commit_w(&bar_kfree[s]);
                    if (j == last) umma_commit_w(&bar_q_free[w]);
                    return true;
                };
                int cur = 0;
                while (ok && cur < n_pos && !uses(cur)) ok = skip(cur++);
                if (ok && cur < n_pos) ok = issue_s_at(cur);
                bool first_pv = true;
                while (ok && cur < n_pos) {
                    // PV for position cur (its S was issued), then the S of the next used
                    // position: S_w and P_w share TMEM columns, and MMAs run in issue order.
                    const int pos = kc + cur, s = pos % S;
                    if (!(ok = wait(&bar_v[s], (pos / S) & 1))) break;
                    if (first_pv && units_w > 0) {
                        // O_w still holds the previous unit until its epilogue has read it
                        if (!(ok = wait(&bar_ofree[w], (units_w - 1) & 1))) break;
                    }
                    if (!(ok = wait(&bar_p[2 * w], tp & 1))) break;
                    tc_fence_after();
                    issue_pv_half(s, first_pv, 0);
                    if (!(ok = wait(&bar_p[2 * w + 1], tp & 1))) break;
                    ++tp;
                    tc_fence_after();
                    issue_pv_half(s, first_pv, 1);
                    first_pv = false;
                    umma_commit_w(&bar_vfree[s]);
                    if (cur == last) {
                        umma_commit_w(&bar_o[w]);
                        ++units_w;
                    }
                    int nxt = cur + 1;
                    while (ok && nxt < n_pos && !uses(nxt)) ok = skip(nxt++);
                    if (ok && nxt < n_pos) ok = issue_s_at(nxt);
                    cur = nxt;
                }
                kc += n_pos;
            }
            // Drain: every MMA issued by this thread completes before TMEM is freed.
            umma_commit_w(&bar_drain[w]);
            mbar_wait_drain(&bar_drain[w], 0, p.status);
        }
    } else if (warp < 8) {
        // ================= softmax warpgroups =================
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kFwdRegsSoftmax));
        const int w = warp >> 2;
        const int wq = warp & 3;
        const int row_in_tile = wq * 32 + lane;
        const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t t_s = tmem_base + lane_bits + w * 128;
        const uint32_t t_o = tmem_base + lane_bits + 256 + w * D;
        const float sl2 = p.scale_log2;
        int ts = 0;      // S tiles consumed by this warpgroup
        int nunits = 0;  // units finished by this warpgroup
        bool ok = true;
        for (int it = 0; ok; ++it) {
            const int rs = it % kUnitRing;
            ok = __all_sync(0xffffffffu, mbar_wait(&bar_ufull[rs], (it / kUnitRing) & 1, abort_flag, p.status));
            if (!ok) break;
            const int u = s_unit[rs];
            int4 meta = make_int4(0, 0, 0, 0);
            if constexpr (BSPARSE) meta = s_meta[rs];
            const Unit un = read_unit<VARLEN>(p, &s_units[rs]);  // read before the slot is handed back
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_ufree[rs]);
            if (u >= n_units) break;
            int n = (w == 0) ? un.n_kv0 : un.n_kv1;
            const uint16_t* bs_own = nullptr;  // block-sparse: this query block's own list
            if constexpr (BSPARSE) {
                const size_t ui = bsparse_index(p, un.bh, un.i0);
                n = (meta.w >> (16 * w)) & 0xffff;
                bs_own = p.bs_own + (2 * ui + w) * p.bs_tk;
            }
            if (n == 0) continue;
            const int tile_first_row = un.i0 + w * kFwdBM;
            const int row = tile_first_row + row_in_tile;
            const int off = un.lk - un.lq;  // causal: query i sits at key position i + off
            const int limit = p.causal ? min(row + off, un.lk - 1) : un.lk - 1;  // highest permitted key

            float m_ref = -INFINITY;  // running max of raw scores q.k (reference for P~)
            float l = 0.0f;           // running sum of the unrounded P~: gives the LSE
            float corr = 0.0f;        // sum over tiles of (bf16(P~_max) - P~_max): l + corr normalises O
            for (int j = 0; j < n; ++j, ++ts) {
                int bs_entry = 0;  // issued before the wait, used after it
                if constexpr (BSPARSE) bs_entry = __ldg(bs_own + j);
                // warp-uniform outcome: the TMEM accesses below are warp-collective
                ok = __all_sync(0xffffffffu, mbar_wait(&bar_s[w], ts & 1, abort_flag, p.status));
                if (!ok) break;
                tc_fence_after();
                float s[kFwdBN];
                {
                    uint32_t r[32];
#pragma unroll
                    for (int c = 0; c < kFwdBN / 32; ++c) {
                        tmem_ld32(t_s + c * 32, r);
#pragma unroll
                        for (int x = 0; x < 32; ++x) s[c * 32 + x] = __uint_as_float(r[x]);
                    }
                    tmem_wait_ld();
                }
                int kv0 = j * kFwdBN;
                bool mine = true;  // block-sparse: this query block may see the tile
                if constexpr (BSPARSE) {
                    kv0 = (bs_entry & kBsEntryTile) * kFwdBN;
                    mine = !(bs_entry & kBsOwnMasked);
                }
                const int lim = mine ? limit : kv0 - 1;  // a tile it may not see is masked whole
                const bool need_mask = !mine || (p.causal && kv0 + kFwdBN - 1 > tile_first_row + off) ||
                                       (kv0 + kFwdBN > un.lk);
                if (need_mask) {
#pragma unroll
                    for (int c = 0; c < kFwdBN; ++c)
                        if (kv0 + c > lim) s[c] = -INFINITY;
                }
                // Row max: eight independent chains, then a tree.
                float mx;
                {
                    float ma[8];
#pragma unroll
                    for (int x = 0; x < 8; ++x) ma[x] = s[x];
#pragma unroll
                    for (int c = 8; c < kFwdBN; ++c) ma[c & 7] = fmaxf(ma[c & 7], s[c]);
                    mx = fmaxf(fmaxf(fmaxf(ma[0], ma[1]), fmaxf(ma[2], ma[3])),
                               fmaxf(fmaxf(ma[4], ma[5]), fmaxf(ma[6], ma[7])));
                }
                const float m_new = fmaxf(m_ref, mx);
                const bool want =
                    (m_ref == -INFINITY) ? (m_new != -INFINITY) : ((m_new - m_ref) * sl2 > kRescaleLog2);
                if (__any_sync(0xffffffffu, want)) {
                    const float alpha = (m_ref == -INFINITY) ? 0.0f : ex2_approx((m_ref - m_new) * sl2);
                    l *= alpha;
                    corr *= alpha;
                    m_ref = m_new;
                    if (j > 0) {
                        // O~ <- alpha O~ (warp-uniform branch, rare).  PV_{j-1} is complete:
                        // the commit that signalled S_j tracked every earlier MMA.
#pragma unroll 1
                        for (int c = 0; c < D / 32; ++c) {
                            uint32_t r0[32];
                            tmem_ld32(t_o + c * 32, r0);
                            tmem_wait_ld();
#pragma unroll
                            for (int x = 0; x < 32; ++x) r0[x] = __float_as_uint(__uint_as_float(r0[x]) * alpha);
                            tmem_st32(t_o + c * 32, r0);
                        }
                    }
                }
                const float mb = (m_ref == -INFINITY) ? 0.0f : m_ref * sl2;
                // P~ = exp2(s * scale*log2e - m * scale*log2e) in two halves of 64 keys;
                // each half is handed to the MMA as soon as it is in TMEM, so the
                // first half of PV runs while the second half is computed.
                // Packed fp32 pairs (FFMA2/FADD2) for the scale-subtract and the sum.
                const float2 sl2x2 = make_float2(sl2, sl2);
                const float2 nmb2 = make_float2(-mb, -mb);
                float2 ls2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    uint32_t pk[kFwdBN / 4];
#pragma unroll
                    for (int c = h * 64; c < h * 64 + 64; c += 2) {
                        const float2 x = __ffma2_rn(make_float2(s[c], s[c + 1]), sl2x2, nmb2);
                        // Masked keys hold s = -inf, so x = -inf and ex2 gives exactly +0:
                        // no select is needed (and none keeps a second copy of this loop).
                        const float p0 = ex2_approx(x.x);
                        const float p1 = ex2_approx(x.y);
                        ls2[(c >> 1) & 1] = __fadd2_rn(ls2[(c >> 1) & 1], make_float2(p0, p1));
                        pk[(c - h * 64) >> 1] = pack_bf16x2(p0, p1);
                    }
                    tmem_st16(t_s + h * 32, pk);
                    tmem_st16(t_s + h * 32 + 16, pk + 16);
                    tmem_wait_st();
                    tc_fence_before();
                    mbar_arrive(&bar_p[2 * w + h]);
                }
                {
                    const float2 t2 = __fadd2_rn(ls2[0], ls2[1]);
                    l += t2.x + t2.y;
                    // The tile's largest P~ dominates its row's rounding error: account
                    // for its bf16 rounding in the normaliser of O.
                    const float pmax = (mx == -INFINITY) ? 0.0f : ex2_approx(fmaf(mx, sl2, -mb));
                    corr += round_bf16(pmax) - pmax;
                }
            }
            if (!ok) break;

            // ---- epilogue: O = O~ / l, LSE = scale * m + ln l
            ok = __all_sync(0xffffffffu, mbar_wait(&bar_o[w], nunits & 1, abort_flag, p.status));
            if (!ok) break;
            ++nunits;
            tc_fence_after();
            // fp32 O of the batched and block-sparse kernels is stored directly from
            // registers; for that, O is read with the 16x256b shape: four consecutive
            // threads then hold 32 contiguous bytes of one row, so each store instruction
            // writes whole 32-byte sectors (eight rows x 32 bytes), with no staging and
            // no wait on the copy engine.  Other outputs go through the TMA-store path.
            const bool direct = !VARLEN && p.o_dtype == FA_DT_F32;
            uint32_t ov[D];
            if (direct) {
                // ov[(16h + c/8... ) ]: half h = lanes [16h, 16h + 16) of the warp, 64-column block b
#pragma unroll
                for (int h = 0; h < 2; ++h) {
#pragma unroll
                    for (int b = 0; b < D / 64; ++b) {
                        uint32_t r[32];
                        tmem_ld_16x256b_x8(t_o + (static_cast<uint32_t>(16 * h) << 16) + b * 64, r);
#pragma unroll
                        for (int x = 0; x < 32; ++x) ov[(h * (D / 64) + b) * 32 + x] = r[x];
                    }
                }
            } else {
#pragma unroll
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t r[32];
                    tmem_ld32(t_o + c * 32, r);
#pragma unroll
                    for (int x = 0; x < 32; ++x) ov[c * 32 + x] = r[x];
                }
            }
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(&bar_ofree[w]);  // O_w may now be overwritten by the next unit's PV
            if (direct) {
                // Rows held by this thread: rsub + 8k of the warp's 32 (k = 0..3: half h = k / 2,
                // upper 8 rows of the half when k is odd); their normalisers come from the
                // threads that own those rows.  Block-sparse rows that see no key store 0.
                const float den = l + corr;
                const bool empty_row = BSPARSE && !(den > 0.0f);
                const float inv_l = empty_row ? 0.0f : 1.0f / den;
                const int rsub = lane >> 2, cp = (lane & 3) * 2;
                float* obase = static_cast<float*>(p.o) +
                               (static_cast<size_t>(un.bh) * p.Lq + tile_first_row + wq * 32) * D;
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int rl = rsub + 8 * k;  // row within the warp's 32
                    const float inv = __shfl_sync(0xffffffffu, inv_l, rl);
                    const bool zero = __shfl_sync(0xffffffffu, empty_row ? 1 : 0, rl) != 0;
                    if (tile_first_row + wq * 32 + rl >= p.Lq) continue;
                    float* orow_k = obase + static_cast<size_t>(rl) * D + cp;
                    const int h = k >> 1, up = k & 1;
#pragma unroll
                    for (int b = 0; b < D / 64; ++b) {
#pragma unroll
                        for (int c = 0; c < 8; ++c) {
                            const int base = (h * (D / 64) + b) * 32 + 4 * c + 2 * up;
                            const float x0 = zero ? 0.0f : __uint_as_float(ov[base]) * inv;
                            const float x1 = zero ? 0.0f : __uint_as_float(ov[base + 1]) * inv;
                            st_global_v2f(orow_k + b * 64 + 8 * c, x0, x1);
                        }
                    }
                }
                if (row < un.lq) p.lse[static_cast<size_t>(un.bh) * p.Lq + row] = m_ref * p.scale + logf(l);
            } else {
                // O leaves through the copy engine: per 128-byte column chunk, each
                // thread writes its row's 128 bytes into the warp's 32-row stage in
                // the 128-byte-swizzled layout of the O tensor map (16-byte pieces
                // XOR row % 8: no bank conflicts), and one lane issues the tile store.
                // Rows past Lq are clipped by the copy engine.
                // Block-sparse: a row that may see no key has l = 0 and gets O = 0, LSE = -inf.
                // Its accumulator is cleared rather than scaled: the fully masked tile it ran
                // may hold non-finite V rows, and 0 * inf or 0 * NaN in the PV product is NaN.
                const float den = l + corr;
                const float inv_l = (BSPARSE && !(den > 0.0f)) ? 0.0f : 1.0f / den;
                if constexpr (BSPARSE) {
                    if (!(den > 0.0f)) {
#pragma unroll
                        for (int c = 0; c < D; ++c) ov[c] = 0u;
                    }
                }
                uint8_t* stg = smem + Lay::kStageOff + warp * 4096;
                const bool f32 = p.o_dtype == FA_DT_F32;
                const int n_chunks = f32 ? D / 32 : D / 64;
                // A packed sequence's last partial 32-row box would spill into the next
                // sequence's rows: its rows are written one by one instead.
                const bool by_rows = VARLEN && tile_first_row + wq * 32 + 32 > un.lq;
                const size_t tok_bytes = static_cast<size_t>(p.H) * D * (f32 ? 4 : 2);
                uint8_t* orow = static_cast<uint8_t*>(p.o) + static_cast<size_t>(un.q0 + row) * tok_bytes +
                                static_cast<size_t>(un.bh % p.H) * D * (f32 ? 4 : 2);
#pragma unroll
                for (int k = 0; k < D / 32; ++k) {
                    if (k >= n_chunks) break;
                    // the stage's previous tile store has finished reading it
                    if (!by_rows) {
                        if (lane == 0) bulk_wait_group_read0();
                        __syncwarp();
                    }
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                        uint4 v;
                        if (f32) {
                            const int c0 = k * 32 + q * 4;
                            v.x = __float_as_uint(__uint_as_float(ov[c0 + 0]) * inv_l);
                            v.y = __float_as_uint(__uint_as_float(ov[c0 + 1]) * inv_l);
                            v.z = __float_as_uint(__uint_as_float(ov[c0 + 2]) * inv_l);
                            v.w = __float_as_uint(__uint_as_float(ov[c0 + 3]) * inv_l);
                        } else {
                            const int c0 = (k * 64 + q * 8) & (D - 1);
                            v.x = pack_bf16x2(__uint_as_float(ov[c0 + 0]) * inv_l, __uint_as_float(ov[c0 + 1]) * inv_l);
                            v.y = pack_bf16x2(__uint_as_float(ov[c0 + 2]) * inv_l, __uint_as_float(ov[c0 + 3]) * inv_l);
                            v.z = pack_bf16x2(__uint_as_float(ov[c0 + 4]) * inv_l, __uint_as_float(ov[c0 + 5]) * inv_l);
                            v.w = pack_bf16x2(__uint_as_float(ov[c0 + 6]) * inv_l, __uint_as_float(ov[c0 + 7]) * inv_l);
                        }
                        if (by_rows) {
                            if (row < un.lq) *reinterpret_cast<uint4*>(orow + k * 128 + q * 16) = v;
                        } else {
                            *reinterpret_cast<uint4*>(stg + lane * 128 + ((q ^ (lane & 7)) << 4)) = v;
                        }
                    }
                    if (by_rows) continue;
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        if constexpr (VARLEN) {
                            tma_store_3d(&p.tm_o, stg, k * (f32 ? 32 : 64), un.bh % p.H, un.q0 + tile_first_row + wq * 32);
                        } else {
                            if (tile_first_row + wq * 32 < p.Lq)
                                tma_store_3d(&p.tm_o, stg, k * (f32 ? 32 : 64), tile_first_row + wq * 32, un.bh);
                        }
                        bulk_commit_group();
                    }
                }
                if (row < un.lq) {
                    const size_t li = VARLEN ? static_cast<size_t>(un.bh % p.H) * p.Lq + un.q0 + row
                                             : static_cast<size_t>(un.bh) * p.Lq + row;
                    p.lse[li] = m_ref * p.scale + logf(l);
                }
            }
        }
    }

    // O tile stores issued by this thread are complete before the CTA exits.
    if (warp < 8 && lane == 0) bulk_wait_group0();
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
    // Every producer of this launch has stopped claiming units once it reaches here;
    // the last CTA to finish returns the scheduler slot to zero for a later launch.
    if (threadIdx.x == 0 && p.sched) {
        __threadfence();
        if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
            atomicExch(p.sched, 0u);
            atomicExch(p.sched + 1, 0u);
        }
    }
}

// Block-sparse planning, one warp per 256-row unit (b*H + h, pair).  For each of the
// unit's two 128-row query blocks, a key block is seen when it lies inside the causal
// cut and the length bound and its mask byte is set.  Per 32 key blocks, one per lane,
// ballots and popcounts compact, in increasing order:
//   - the union list (key blocks either query block sees; bit 14 + w when block w does),
//     which the producer loads and the MMA issuer walks;
//   - each query block's own list, which its softmax warpgroup walks.
// A query block that exists but sees nothing still takes part in one entry (the union's
// first, or key block 0 when the union is empty), flagged kBsOwnMasked in its own list:
// its scores are all masked, and its rows get O = 0 and LSE = -inf.
constexpr int kBsPlanThreads = 256;

__global__ void __launch_bounds__(kBsPlanThreads) fa_bsparse_plan(const BsPlanParams q) {
    const long long unit = (static_cast<long long>(blockIdx.x) * kBsPlanThreads + threadIdx.x) >> 5;
    const int lane = threadIdx.x & 31;
    const long long n_units = static_cast<long long>(q.B) * q.H * q.n_pairs;
    if (unit >= n_units) return;  // warp-uniform
    const int bh = static_cast<int>(unit / q.n_pairs);
    const int pair = static_cast<int>(unit % q.n_pairs);
    const int b = bh / q.H, h = bh % q.H;
    const int off = q.Lk - q.Lq;  // causal: query i sits at key position i + off
    int n[2];  // key blocks within the causal cut and the length bound, per query block
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        const int first = pair * kFwdRowsPerCta + w * kFwdBM;
        if (first >= q.Lq) {
            n[w] = 0;
        } else if (q.causal) {
            const int last = min(first + kFwdBM - 1, q.Lq - 1);
            n[w] = min(q.tk, (last + off) / kFwdBN + 1);
        } else {
            n[w] = q.tk;
        }
    }
    // mask rows of the two query blocks (the second is only read when it exists: n[1] > 0)
    const uint8_t* m0 = q.mask + b * q.stride_b + h * q.stride_h + static_cast<long long>(2 * pair) * q.tk;
    const uint8_t* m1 = m0 + q.tk;
    uint16_t* out = q.list + unit * q.tk;
    uint16_t* own0 = q.own + 2 * unit * q.tk;
    uint16_t* own1 = own0 + q.tk;
    const unsigned below = (1u << lane) - 1u;
    int cnt = 0, c0 = 0, c1 = 0, last0 = -1, last1 = -1;
    const int n_max = max(n[0], n[1]);
    for (int base = 0; base < n_max; base += 32) {
        const int t = base + lane;
        const bool s0 = t < n[0] && m0[t] != 0;
        const bool s1 = t < n[1] && m1[t] != 0;
        const unsigned keep = __ballot_sync(0xffffffffu, s0 || s1);
        const unsigned k0 = __ballot_sync(0xffffffffu, s0);
        const unsigned k1 = __ballot_sync(0xffffffffu, s1);
        const int pos = cnt + __popc(keep & below);  // this lane's union index, if kept
        if (s0 || s1) out[pos] = static_cast<uint16_t>(t | (s0 ? 1 << 14 : 0) | (s1 ? 1 << 15 : 0));
        if (s0) own0[c0 + __popc(k0 & below)] = static_cast<uint16_t>(t);
        if (s1) own1[c1 + __popc(k1 & below)] = static_cast<uint16_t>(t);
        last0 = max(last0, __reduce_max_sync(0xffffffffu, s0 ? pos : -1));
        last1 = max(last1, __reduce_max_sync(0xffffffffu, s1 ? pos : -1));
        cnt += __popc(keep);
        c0 += __popc(k0);
        c1 += __popc(k1);
    }
    __syncwarp();  // the lists' writes are visible to lane 0 below
    if (lane == 0) {
        if (cnt == 0) {
            out[0] = 0;
            cnt = 1;
        }
        const int tile0 = out[0] & kBsEntryTile;
        if (c0 == 0) {  // query block 0 always exists
            out[0] = static_cast<uint16_t>(out[0] | (1 << 14));
            own0[0] = static_cast<uint16_t>(tile0 | kBsOwnMasked);
            c0 = 1;
            last0 = max(last0, 0);
        }
        if (n[1] > 0 && c1 == 0) {
            out[0] = static_cast<uint16_t>(out[0] | (1 << 15));
            own1[0] = static_cast<uint16_t>(tile0 | kBsOwnMasked);
            c1 = 1;
            last1 = max(last1, 0);
        }
        q.meta[unit] = make_int4(cnt, last0, n[1] > 0 ? last1 : -1, c0 | (c1 << 16));
    }
}

// The setmaxnreg split only works if the block was launched with at least as
// many registers as the split hands out; otherwise the increase would wait
// forever.  Refuse to launch a build whose register count does not cover it.
template <typename K>
cudaError_t check_register_split(K kernel) {
    cudaFuncAttributes a{};
    cudaError_t e = cudaFuncGetAttributes(&a, kernel);
    if (e != cudaSuccess) return e;
    const long long pool = static_cast<long long>(a.numRegs) * kFwdThreads;
    const long long need = 2LL * 128 * kFwdRegsSoftmax + 128LL * kFwdRegsOther;
    return pool >= need ? cudaSuccess : cudaErrorInvalidConfiguration;
}

}  // namespace

int fwd_smem_bytes(int d) { return d == 128 ? FwdLayout<128>::kBytes : FwdLayout<64>::kBytes; }

template <int D, bool VARLEN, bool BSPARSE>
cudaError_t launch_fwd_kernel(const FwdParams& p, int num_sms, cudaStream_t stream) {
    const long long pairs = VARLEN ? p.max_pairs : (p.Lq + kFwdRowsPerCta - 1) / kFwdRowsPerCta;
    const long long units = static_cast<long long>(p.B) * p.H * pairs;
    if (units == 0) return cudaSuccess;
    const dim3 grid(static_cast<unsigned>(units < num_sms ? units : num_sms));
    const int smem = fwd_smem_bytes(D);
    cudaError_t e;
    if ((e = check_register_split(fa_fwd_kernel<D, VARLEN, BSPARSE>)) != cudaSuccess) return e;
    e = cudaFuncSetAttribute(fa_fwd_kernel<D, VARLEN, BSPARSE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    fa_fwd_kernel<D, VARLEN, BSPARSE><<<grid, kFwdThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

cudaError_t launch_fwd(const FwdParams& p, int d, int num_sms, cudaStream_t stream) {
    return d == 128 ? launch_fwd_kernel<128, false, false>(p, num_sms, stream)
                    : launch_fwd_kernel<64, false, false>(p, num_sms, stream);
}

cudaError_t launch_fwd_varlen(const FwdParams& p, int d, int num_sms, cudaStream_t stream) {
    return d == 128 ? launch_fwd_kernel<128, true, false>(p, num_sms, stream)
                    : launch_fwd_kernel<64, true, false>(p, num_sms, stream);
}

cudaError_t launch_fwd_blocksparse(const BsPlanParams& plan, const FwdParams& p, int d, int num_sms,
                                   cudaStream_t stream) {
    const long long n_units = static_cast<long long>(plan.B) * plan.H * plan.n_pairs;
    if (n_units == 0) return cudaSuccess;
    const long long blocks = (n_units * 32 + kBsPlanThreads - 1) / kBsPlanThreads;
    fa_bsparse_plan<<<static_cast<unsigned>(blocks), kBsPlanThreads, 0, stream>>>(plan);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (d == 256) return launch_fwd256_blocksparse(p, num_sms, stream);
    return d == 128 ? launch_fwd_kernel<128, false, true>(p, num_sms, stream)
                    : launch_fwd_kernel<64, false, true>(p, num_sms, stream);
}

#ifdef FA_TEST_HOOKS
cudaError_t fwd_test_arm_skip_k() {
    const int one = 1;
    return cudaMemcpyToSymbol(g_test_skip_k, &one, sizeof(int));
}
#endif

size_t bs_workspace_bytes(int B, int H, int Lq, int Lk) {
    const size_t n_units = static_cast<size_t>(B) * H * ((Lq + kFwdRowsPerCta - 1) / kFwdRowsPerCta);
    const size_t tk = (static_cast<size_t>(Lk) + kFwdBN - 1) / kFwdBN;
    auto up = [](size_t x) { return (x + 255) & ~static_cast<size_t>(255); };
    // metadata, union lists, own lists (two per unit)
    return up(n_units * sizeof(int4)) + up(n_units * tk * sizeof(uint16_t)) + up(2 * n_units * tk * sizeof(uint16_t));
}

}  // namespace fa
