// Forward pass of exact attention for sm_100a at head dimension 256.
//
// The same blockwise method as the d <= 128 kernel (glossary "How it works";
// "What FlashAttention does instead"; "The Three Running Statistics"), with a
// tile shape chosen for d = 256, where a head's rows are twice as wide
// ("Basic Flash Attention Forward Pass" takes D as a free shape parameter):
//   - a work unit is ONE 128-row Q tile of one (b, h) (64 KB of Q);
//   - K and V stream in 64-key tiles (32 KB each) through two 2-stage rings,
//     so Q, the rings and the epilogue stages fit in 224 KB of shared memory;
//   - S = Q K^T (128 x 64) is double-buffered in TMEM (2 x 64 columns) next to
//     the 128 x 256 fp32 accumulator O (256 columns): 384 of 512 columns;
//   - two softmax warpgroups split every score row: warpgroup g owns keys
//     [32g, 32g + 32) of each tile, and thread (g, r) of both warpgroups works
//     on row r.  The partners exchange their partial row maxima through spare
//     TMEM columns of their (shared) lane, so both apply the same running max
//     and take the same rescaling decision; each keeps its own partial row sum
//     and rescales its own half of O's columns.  The partial sums are combined
//     once per unit, in the epilogue, where warpgroup g stores O's columns
//     [128g, 128g + 128).
//   warp 8      TMA producer: Q per unit, K_j and V_j through the rings.
//   warp 9      MMA issuer: S(j) = Q K_j^T (SS MMA, N = 64), then, once both
//               halves of P(j) are in TMEM, O += P(j) V_j (TS MMA, N = 256) and
//               S(j+2) into the buffer P(j) occupied.
//   warps 10-11 idle (registers go to the softmax warpgroups).
// Rescaling is deferred while the running max has grown by no more than 2^8
// (exp2 units), as in the d <= 128 kernel; a rescale waits for the PV MMA of
// the previous tile to finish, because S runs two tiles ahead of PV here.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fa_internal.h"
#include "ptx.cuh"

namespace fa {
namespace {

constexpr int kD = 256;
constexpr int kBM = 128;          // query rows per unit
constexpr int kBN = kFwd256BN;    // keys per K/V tile (64)
constexpr int kStages = 2;        // K and V ring depth
constexpr int kUnitRing = 4;
constexpr float kRescaleLog2 = 8.0f;

struct Lay256 {
    static constexpr int kQBox = kBM * 64 * 2;             // 16 KB: 128 rows x 64 bf16
    static constexpr int kKVBox = kBN * 64 * 2;            // 8 KB: 64 rows x 64 bf16
    static constexpr int kQBytes = kQBox * (kD / 64);      // 64 KB
    static constexpr int kKVBytes = kKVBox * (kD / 64);    // 32 KB
    static constexpr int kQOff = 0;
    static constexpr int kKOff = kQOff + kQBytes;
    static constexpr int kVOff = kKOff + kStages * kKVBytes;
    static constexpr int kStageOff = kVOff + kStages * kKVBytes;  // 8 warps x 4 KB epilogue stages
    static constexpr int kBarOff = kStageOff + 8 * 4096;
    // q, q_free, k[S], v[S], kfree[S], vfree[S], s[2], p[2][2], pv, o, ofree, x[4], drain, ufull[R], ufree[R]
    static constexpr int kNumBars = 2 + 4 * kStages + 2 + 4 + 3 + 4 + 1 + 2 * kUnitRing;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    // unit ring: 4 unit indices, then 4 decoded units (32 bytes each)
    static constexpr int kRingOff = kMiscOff + 16;
    static constexpr int kBytes = kRingOff + 16 + 128 + 1024;  // + alignment slack
};

// TMEM columns: S buffers [0, 64) and [64, 128); the partners' exchange slots
// [128, 132) (two parities x two warpgroups); O [256, 512).
constexpr uint32_t kColX = 128;
constexpr uint32_t kColO = 256;

// One work unit: (b*H + h), its first query row within the sequence, the 64-key tiles to
// visit, where its sequence lives (packed first rows and lengths; 0, 0, Lq, Lk for a
// batched call), and (block-sparse) the index of its query block's own key-block list.
struct __align__(16) Unit256 {
    int bh, i0, n;
    int q0, k0, lq, lk;
    int lst;
};

// Units in a fixed global order: the (b, h) pairs in groups of p.head_group heads
// whose K and V fit in L2 together; within a group, longest causal rows first
// (query tile index descending), heads interleaved.
__device__ __forceinline__ Unit256 unit256_of(const FwdParams& p, int u) {
    const int BH = p.B * p.H;
    const int n_qt = (p.Lq + kBM - 1) / kBM;
    const int G = p.head_group;
    const int grp = u / (G * n_qt);
    const int rem = u - grp * G * n_qt;
    const int gsz = min(G, BH - grp * G);
    Unit256 r;
    const int qt = n_qt - 1 - rem / gsz;
    r.bh = grp * G + rem % gsz;
    r.i0 = qt * kBM;
    const int n_all = (p.Lk + kBN - 1) / kBN;
    if (p.causal) {
        const int last = min(r.i0 + kBM - 1, p.Lq - 1) + (p.Lk - p.Lq);  // highest key any row may see
        r.n = min(n_all, last / kBN + 1);
    } else {
        r.n = n_all;
    }
    r.q0 = 0;
    r.k0 = 0;
    r.lq = p.Lq;
    r.lk = p.Lk;
    r.lst = 0;
    return r;
}

// Block-sparse: the batched unit order; the unit's 128-row query block visits the key
// blocks of its own list (planned before the launch for pairs of query blocks, at least
// one entry), each as two 64-key tiles.
__device__ __forceinline__ Unit256 unit256_of_bsparse(const FwdParams& p, int u) {
    Unit256 r = unit256_of(p, u);
    const int qb = r.i0 / kBM;
    const int n_pairs = (p.Lq + 2 * kBM - 1) / (2 * kBM);
    const int ui = r.bh * n_pairs + (qb >> 1);
    const int w = qb & 1;
    const int cnt = (__ldg(p.bs_meta + ui).w >> (16 * w)) & 0xffff;
    r.n = 2 * cnt;
    r.lst = 2 * ui + w;
    return r;
}

// Packed variable-length batch: unit u is (query tile, b*H + h) in a virtual space of
// p.max_pairs 128-row tiles per (b, h), longest causal rows first.  Units past a
// sequence's end are empty (no KV tiles).  A sequence whose offsets are out of range or
// decreasing, that is longer than max_pairs * 128 rows, that has queries but no keys, or
// (causal) more queries than keys is skipped and flagged FA_ERR_SEQLEN (once, from its
// tile-0 unit).
__device__ __forceinline__ Unit256 unit256_of_varlen(const FwdParams& p, int u) {
    const int BH = p.B * p.H;
    Unit256 r;
    const int qt = p.max_pairs - 1 - u / BH;
    r.bh = u % BH;
    r.i0 = qt * kBM;
    r.n = 0;
    r.lst = 0;
    const int b = r.bh / p.H;
    const int q0 = p.cu_q[b], q1 = p.cu_q[b + 1], k0 = p.cu_k[b], k1 = p.cu_k[b + 1];
    r.q0 = q0;
    r.k0 = k0;
    r.lq = q1 - q0;
    r.lk = k1 - k0;
    const bool bad = q0 < 0 || q1 < q0 || q1 > p.Lq || k0 < 0 || k1 < k0 || k1 > p.Lk ||
                     r.lq > p.max_pairs * kBM || (r.lq > 0 && r.lk == 0) || (p.causal && r.lq > r.lk);
    if (bad) {
        if (qt == 0) atomicCAS(p.status, 0, FA_ERR_SEQLEN);
        r.lq = 0;
        return r;
    }
    if (r.i0 < r.lq) {
        const int n_all = (r.lk + kBN - 1) / kBN;
        r.n = p.causal ? min(n_all, (min(r.i0 + kBM - 1, r.lq - 1) + r.lk - r.lq) / kBN + 1) : n_all;
    }
    return r;
}

__device__ __forceinline__ void tmem_st1(uint32_t taddr, float v) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(__float_as_uint(v))
                 : "memory");
}
__device__ __forceinline__ float tmem_ld1(uint32_t taddr) {
    uint32_t r;
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x1.b32 {%0}, [%1];" : "=r"(r) : "r"(taddr));
    return __uint_as_float(r);
}

template <bool VARLEN, bool BSPARSE>
__global__ void __launch_bounds__(kFwdThreads, 1) fa_fwd256_kernel(const __grid_constant__ FwdParams p) {
    using Lay = Lay256;
    constexpr int S = kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + Lay::kQOff;
    uint8_t* sK = smem + Lay::kKOff;
    uint8_t* sV = smem + Lay::kVOff;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
    uint64_t* bar_q = bars;               // Q landed
    uint64_t* bar_q_free = bars + 1;      // the unit's last S MMA is done with Q
    uint64_t* bar_k = bars + 2;           // [S]
    uint64_t* bar_v = bar_k + S;          // [S]
    uint64_t* bar_kfree = bar_v + S;      // [S]
    uint64_t* bar_vfree = bar_kfree + S;  // [S]
    uint64_t* bar_s = bar_vfree + S;      // [buffer]: S(j) in TMEM
    uint64_t* bar_p = bar_s + 2;          // [2 * buffer + g]: warpgroup g's half of P(j) in TMEM
    uint64_t* bar_pv = bar_p + 4;         // PV(j) done (one phase per tile)
    uint64_t* bar_o = bar_pv + 1;         // the unit's last PV is done
    uint64_t* bar_ofree = bar_o + 1;      // the epilogue has read O
    uint64_t* bar_x = bar_ofree + 1;      // [warp & 3]: partner exchange, one phase per exchange
    uint64_t* bar_drain = bar_x + 4;
    uint64_t* bar_ufull = bar_drain + 1;
    uint64_t* bar_ufree = bar_ufull + kUnitRing;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 4);
    volatile int* s_unit = reinterpret_cast<volatile int*>(smem + Lay::kRingOff);
    // The producer decodes each unit once (for a packed batch that reads the sequence's
    // offsets from global memory) and publishes it with the unit index.
    Unit256* s_units = reinterpret_cast<Unit256*>(smem + Lay::kRingOff + 16);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const int n_units = p.B * p.H * (VARLEN ? p.max_pairs : (p.Lq + kBM - 1) / kBM);

    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        mbar_init(bar_q_free, 1);
        for (int s = 0; s < S; ++s) {
            mbar_init(&bar_k[s], 1);
            mbar_init(&bar_v[s], 1);
            mbar_init(&bar_kfree[s], 1);
            mbar_init(&bar_vfree[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&bar_s[b], 1);
            mbar_init(&bar_p[2 * b], 128);
            mbar_init(&bar_p[2 * b + 1], 128);
        }
        mbar_init(bar_pv, 1);
        mbar_init(bar_o, 1);
        mbar_init(bar_ofree, 256);
        for (int x = 0; x < 4; ++x) mbar_init(&bar_x[x], 64);
        mbar_init(bar_drain, 1);
        for (int r = 0; r < kUnitRing; ++r) {
            mbar_init(&bar_ufull[r], 1);
            mbar_init(&bar_ufree[r], 1 + 8);  // MMA warp + 8 softmax warps
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

    if (warp >= 8) {
        asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kFwdRegsOther));
    }
    if (warp == 8) {
        // ================= TMA producer: Q, then K_j and V_j in order
        auto wait = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.status));
        };
        int kc = 0, nk = 0, nv = 0, nq = 0;
        unsigned claims = 0;
        bool ok = !*abort_flag;
        for (int it = 0; ok; ++it) {
            const int rs = it % kUnitRing;
            if (it >= kUnitRing && !(ok = wait(&bar_ufree[rs], ((it / kUnitRing) - 1) & 1))) break;
            int u;
            Unit256 un;
            for (;;) {  // a packed batch's virtual units past a sequence's end are skipped here
                unsigned int ticket = 0;
                if (p.sched) {
                    if (lane == 0) ticket = atomicAdd(p.sched, 1u);
                    ticket = __shfl_sync(0xffffffffu, ticket, 0);
                } else {
                    const unsigned G = gridDim.x, k = claims++;
                    ticket = k * G + ((k & 1u) ? G - 1u - blockIdx.x : blockIdx.x);
                }
                u = static_cast<int>(min(ticket, static_cast<unsigned>(n_units)));
                if (u >= n_units) break;
                if constexpr (VARLEN) un = unit256_of_varlen(p, u);
                else if constexpr (BSPARSE) un = unit256_of_bsparse(p, u);
                else un = unit256_of(p, u);
                if (!VARLEN || un.n > 0) break;
            }
            if (lane == 0) {
                s_unit[rs] = u;
                if (u < n_units) s_units[rs] = un;
                mbar_arrive(&bar_ufull[rs]);
            }
            __syncwarp();
            if (u >= n_units) break;
            if (nq > 0 && !(ok = wait(bar_q_free, (nq - 1) & 1))) break;
            mbar_arrive_expect_tx_w(bar_q, Lay::kQBytes);
            // batched maps are [B*H][L][d]; packed maps are [total][H][d]
            for (int b = 0; b < kD / 64; ++b)
                tma_load_3d_w(sQ + b * Lay::kQBox, &p.tm_q, bar_q, b * 64, VARLEN ? un.bh % p.H : un.i0,
                              VARLEN ? un.q0 + un.i0 : un.bh);
            ++nq;
            const uint16_t* own = BSPARSE ? p.bs_own + static_cast<size_t>(un.lst) * p.bs_tk : nullptr;
            for (int j = 0; j < un.n; ++j, ++kc) {
                const int s = kc % S;
                int ky = j * kBN;  // first key of the tile (batched and block-sparse maps)
                if constexpr (BSPARSE) ky = (__ldg(own + (j >> 1)) & kBsEntryTile) * (2 * kBN) + (j & 1) * kBN;
                if (kc >= S && !(ok = wait(&bar_kfree[s], ((kc / S) - 1) & 1))) break;
                mbar_arrive_expect_tx_w(&bar_k[s], Lay::kKVBytes);
                for (int b = 0; b < kD / 64; ++b)
                    tma_load_3d_w(sK + s * Lay::kKVBytes + b * Lay::kKVBox, &p.tm_k, &bar_k[s], b * 64,
                                  VARLEN ? un.bh % p.H : ky, VARLEN ? un.k0 + j * kBN : un.bh);
                ++nk;
                if (kc >= S && !(ok = wait(&bar_vfree[s], ((kc / S) - 1) & 1))) break;
                mbar_arrive_expect_tx_w(&bar_v[s], Lay::kKVBytes);
                for (int b = 0; b < kD / 64; ++b)
                    tma_load_3d_w(sV + s * Lay::kKVBytes + b * Lay::kKVBox, &p.tm_v, &bar_v[s], b * 64,
                                  VARLEN ? un.bh % p.H : ky, VARLEN ? un.k0 + j * kBN : un.bh);
                ++nv;
            }
        }
        // every copy issued here lands before the CTA exits (each barrier is at the
        // phase of its last copy)
        if (nq > 0) mbar_wait_drain(bar_q, (nq - 1) & 1, p.status);
        for (int t = max(0, nk - S); t < nk; ++t) mbar_wait_drain(&bar_k[t % S], (t / S) & 1, p.status);
        for (int t = max(0, nv - S); t < nv; ++t) mbar_wait_drain(&bar_v[t % S], (t / S) & 1, p.status);
    } else if (warp == 9) {
        // ================= MMA issuer
        auto wait = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.status));
        };
        constexpr uint32_t kIdescQK = idesc_bf16_f32(128, kBN, 0, 0);
        constexpr uint32_t kIdescPV = idesc_bf16_f32(128, kD, 0, 1);
        const uint32_t sQa = smem_u32(sQ), sKa = smem_u32(sK), sVa = smem_u32(sV);
        // S(j) = Q K_j^T into buffer b: 16 MMAs of K = 16 over the 256 columns
        auto issue_s = [&](int s, int b) {
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
                const uint32_t qoff = (kk >> 2) * Lay::kQBox + (kk & 3) * 32;
                const uint32_t koff = (kk >> 2) * Lay::kKVBox + (kk & 3) * 32;
                umma_ss_w(tmem_base + b * 64, smem_desc_sw128(sQa + qoff, 16, 1024),
                          smem_desc_sw128(sKa + s * Lay::kKVBytes + koff, 16, 1024), kIdescQK, kk > 0 ? 1u : 0u);
            }
            umma_commit_w(&bar_s[b]);
        };
        // O += P(j) V_j for keys [32h, 32h + 32) of the tile (P from TMEM, 2 MMAs of K = 16)
        auto issue_pv_half = [&](int s, int b, bool first, int h) {
#pragma unroll
            for (int k2 = 0; k2 < 2; ++k2) {
                const int kk = 2 * h + k2;  // 16-key step: V rows [16kk, 16kk + 16)
                const uint64_t bdesc = smem_desc_sw128(sVa + s * Lay::kKVBytes + kk * 2048, Lay::kKVBox, 1024);
                umma_ts_w(tmem_base + kColO, tmem_base + b * 64 + kk * 8, bdesc, kIdescPV,
                          (!first || kk > 0) ? 1u : 0u);
            }
        };
        int kc = 0, q_iter = 0, ts = 0, units = 0;
        bool ok = true;
        for (int it = 0; ok; ++it) {
            const int rs = it % kUnitRing;
            if (!(ok = wait(&bar_ufull[rs], (it / kUnitRing) & 1))) break;
            const int u = s_unit[rs];
            const int n = s_units[rs].n;  // read before the slot is handed back
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_ufree[rs]);
            if (u >= n_units) break;
            if (!(ok = wait(bar_q, q_iter & 1))) break;
            ++q_iter;
            // the first two S of the unit (buffers of tiles ts and ts + 1)
            for (int j = 0; ok && j < min(n, 2); ++j) {
                const int pos = kc + j;
                if (!(ok = wait(&bar_k[pos % S], (pos / S) & 1))) break;
                tc_fence_after();
                issue_s(pos % S, (ts + j) & 1);
                umma_commit_w(&bar_kfree[pos % S]);
                if (j == n - 1) umma_commit_w(bar_q_free);
            }
            for (int j = 0; ok && j < n; ++j) {
                const int pos = kc + j, s = pos % S, t = ts + j, b = t & 1;
                if (!(ok = wait(&bar_v[s], (pos / S) & 1))) break;
                if (j == 0 && units > 0) {
                    // O still holds the previous unit until its epilogue has read it
                    if (!(ok = wait(bar_ofree, (units - 1) & 1))) break;
                }
                for (int h = 0; ok && h < 2; ++h) {
                    if (!(ok = wait(&bar_p[2 * b + h], (t >> 1) & 1))) break;
                    tc_fence_after();
                    issue_pv_half(s, b, j == 0, h);
                }
                if (!ok) break;
                umma_commit_w(&bar_vfree[s]);
                umma_commit_w(bar_pv);
                if (j == n - 1) {
                    umma_commit_w(bar_o);
                    ++units;
                }
                if (j + 2 < n) {
                    // S(j+2) reuses the buffer P(j) sits in: it follows PV(j) in issue order
                    const int pos2 = pos + 2;
                    if (!(ok = wait(&bar_k[pos2 % S], (pos2 / S) & 1))) break;
                    tc_fence_after();
                    issue_s(pos2 % S, b);
                    umma_commit_w(&bar_kfree[pos2 % S]);
                    if (j + 2 == n - 1) umma_commit_w(bar_q_free);
                }
            }
            kc += n;
            ts += n;
        }
        umma_commit_w(bar_drain);
        mbar_wait_drain(bar_drain, 0, p.status);
    } else if (warp < 8) {
        // ================= softmax warpgroups: g = keys [32g, 32g + 32) of each tile
        asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kFwdRegsSoftmax));
        const int g = warp >> 2;
        const int wq = warp & 3;
        const int row_in_tile = wq * 32 + lane;
        const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t t_row = tmem_base + lane_bits;
        const float sl2 = p.scale_log2;
        uint64_t* xbar = &bar_x[wq];
        int xc = 0;      // exchanges with the partner thread so far
        int ts = 0;      // tiles consumed
        int units = 0;   // units finished
        bool ok = true;
        // Exchange one float with the partner thread (same row, other warpgroup)
        // through TMEM columns of the shared lane; bounded wait.
        auto exchange = [&](float mine, float& theirs) -> bool {
            const uint32_t base = t_row + kColX + 2 * (xc & 1);
            tmem_st1(base + g, mine);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(xbar);
            const bool good = __all_sync(0xffffffffu, mbar_wait(xbar, xc & 1, abort_flag, p.status));
            ++xc;
            if (!good) return false;
            tc_fence_after();
            theirs = tmem_ld1(base + (1 - g));
            tmem_wait_ld();
            return true;
        };
        for (int it = 0; ok; ++it) {
            const int rs = it % kUnitRing;
            ok = __all_sync(0xffffffffu, mbar_wait(&bar_ufull[rs], (it / kUnitRing) & 1, abort_flag, p.status));
            if (!ok) break;
            const int u = s_unit[rs];
            Unit256 un;  // read before the slot is handed back
            un.bh = s_units[rs].bh;
            un.i0 = s_units[rs].i0;
            un.n = s_units[rs].n;
            un.lst = BSPARSE ? s_units[rs].lst : 0;
            if constexpr (VARLEN) {
                un.q0 = s_units[rs].q0;
                un.lq = s_units[rs].lq;
                un.lk = s_units[rs].lk;
            } else {
                un.q0 = 0;
                un.lq = p.Lq;
                un.lk = p.Lk;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_ufree[rs]);
            if (u >= n_units) break;
            const int row = un.i0 + row_in_tile;  // within the sequence
            const int off = un.lk - un.lq;        // causal: query i sits at key position i + off
            const int limit = p.causal ? min(row + off, un.lk - 1) : un.lk - 1;  // highest permitted key
            float m_ref = -INFINITY;  // running max of raw scores (the same in both partners)
            float l = 0.0f;           // this thread's partial sum of the unrounded P~
            float corr = 0.0f;        // bf16 rounding of this half's largest P~, summed over tiles
            const uint16_t* own = BSPARSE ? p.bs_own + static_cast<size_t>(un.lst) * p.bs_tk : nullptr;
            for (int j = 0; j < un.n; ++j, ++ts) {
                const int b = ts & 1;
                int bs_entry = 0;  // issued before the wait, used after it
                if constexpr (BSPARSE) bs_entry = __ldg(own + (j >> 1));
                ok = __all_sync(0xffffffffu, mbar_wait(&bar_s[b], (ts >> 1) & 1, abort_flag, p.status));
                if (!ok) break;
                tc_fence_after();
                float s[32];
                {
                    uint32_t r[32];
                    tmem_ld32(t_row + b * 64 + g * 32, r);
                    tmem_wait_ld();
#pragma unroll
                    for (int x = 0; x < 32; ++x) s[x] = __uint_as_float(r[x]);
                }
                int kv0 = j * kBN + g * 32;
                bool mine = true;  // block-sparse: this query block may see the tile
                if constexpr (BSPARSE) {
                    kv0 = (bs_entry & kBsEntryTile) * (2 * kBN) + (j & 1) * kBN + g * 32;
                    mine = !(bs_entry & kBsOwnMasked);
                }
                const int lim = mine ? limit : kv0 - 1;  // a tile it may not see is masked whole
                if (kv0 + 31 > lim) {
#pragma unroll
                    for (int c = 0; c < 32; ++c)
                        if (kv0 + c > lim) s[c] = -INFINITY;
                }
                float mx;
                {
                    float ma[4];
#pragma unroll
                    for (int x = 0; x < 4; ++x) ma[x] = s[x];
#pragma unroll
                    for (int c = 4; c < 32; ++c) ma[c & 3] = fmaxf(ma[c & 3], s[c]);
                    mx = fmaxf(fmaxf(ma[0], ma[1]), fmaxf(ma[2], ma[3]));
                }
                // The exchange also orders both partners' score loads before either
                // writes P over the buffer (warpgroup 1's P lands on warpgroup 0's scores).
                float mx_other = -INFINITY;
                if (!(ok = __all_sync(0xffffffffu, exchange(mx, mx_other)))) break;
                const float mt = fmaxf(mx, mx_other);
                const float m_new = fmaxf(m_ref, mt);
                const bool want = (m_ref == -INFINITY) ? (m_new != -INFINITY) : ((m_new - m_ref) * sl2 > kRescaleLog2);
                if (__any_sync(0xffffffffu, want)) {
                    const float alpha = (m_ref == -INFINITY) ? 0.0f : ex2_approx((m_ref - m_new) * sl2);
                    l *= alpha;
                    corr *= alpha;
                    m_ref = m_new;
                    if (j > 0) {
                        // O <- alpha O on this warpgroup's 128 columns, once PV(j-1) is done
                        // (S runs two tiles ahead, so S(j) landing does not imply it).
                        ok = __all_sync(0xffffffffu, mbar_wait(bar_pv, (ts - 1) & 1, abort_flag, p.status));
                        if (!ok) break;
                        tc_fence_after();
#pragma unroll 1
                        for (int c = 0; c < 4; ++c) {
                            uint32_t r0[32];
                            const uint32_t ta = t_row + kColO + g * 128 + c * 32;
                            tmem_ld32(ta, r0);
                            tmem_wait_ld();
#pragma unroll
                            for (int x = 0; x < 32; ++x) r0[x] = __float_as_uint(__uint_as_float(r0[x]) * alpha);
                            tmem_st32(ta, r0);
                        }
                        tmem_wait_st();
                    }
                }
                const float mb = (m_ref == -INFINITY) ? 0.0f : m_ref * sl2;
                const float2 sl2x2 = make_float2(sl2, sl2);
                const float2 nmb2 = make_float2(-mb, -mb);
                float2 ls2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 32; c += 2) {
                    const float2 x = __ffma2_rn(make_float2(s[c], s[c + 1]), sl2x2, nmb2);
                    const float p0 = ex2_approx(x.x);  // masked keys: x = -inf, p = +0
                    const float p1 = ex2_approx(x.y);
                    ls2[(c >> 1) & 1] = __fadd2_rn(ls2[(c >> 1) & 1], make_float2(p0, p1));
                    pk[c >> 1] = pack_bf16x2(p0, p1);
                }
                // P for keys [32g, 32g + 32) goes to columns [16g, 16g + 16) of the buffer
                tmem_st16(t_row + b * 64 + g * 16, pk);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(&bar_p[2 * b + g]);
                const float2 t2 = __fadd2_rn(ls2[0], ls2[1]);
                l += t2.x + t2.y;
                const float pmax = (mx == -INFINITY) ? 0.0f : ex2_approx(fmaf(mx, sl2, -mb));
                corr += round_bf16(pmax) - pmax;
            }
            if (!ok) break;

            // ---- epilogue: both partners need l + corr of the whole row
            float l_other = 0.0f, c_other = 0.0f;
            if (!(ok = __all_sync(0xffffffffu, exchange(l, l_other)))) break;
            if (!(ok = __all_sync(0xffffffffu, exchange(corr, c_other)))) break;
            const float l_row = l + l_other;
            const float den = l_row + corr + c_other;
            // Block-sparse: a row that may see no key has l = 0 and gets O = 0, LSE = -inf.
            const bool empty_row = BSPARSE && !(den > 0.0f);
            const float inv = empty_row ? 0.0f : 1.0f / den;
            ok = __all_sync(0xffffffffu, mbar_wait(bar_o, units & 1, abort_flag, p.status));
            if (!ok) break;
            ++units;
            tc_fence_after();
            uint32_t ov[128];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t r[32];
                tmem_ld32(t_row + kColO + g * 128 + c * 32, r);
#pragma unroll
                for (int x = 0; x < 32; ++x) ov[c * 32 + x] = r[x];
            }
            tmem_wait_ld();
            tc_fence_before();
            mbar_arrive(bar_ofree);  // O may now be overwritten by the next unit's PV
            if constexpr (BSPARSE) {
                // Cleared rather than scaled: the fully masked tile such a row ran may hold
                // non-finite V rows, and 0 * inf or 0 * NaN in the PV product is NaN.
                if (empty_row) {
#pragma unroll
                    for (int c = 0; c < 128; ++c) ov[c] = 0u;
                }
            }
            uint8_t* stg = smem + Lay::kStageOff + warp * 4096;
            const bool f32 = p.o_dtype == FA_DT_F32;
            const int n_chunks = f32 ? 4 : 2;  // 128-byte column chunks of this warpgroup's 128 columns
            // A packed sequence's last partial 32-row box would spill into the next
            // sequence's rows: its rows are written one by one instead.
            const bool by_rows = VARLEN && un.i0 + wq * 32 + 32 > un.lq;
            uint8_t* orow = nullptr;
            if constexpr (VARLEN) {
                const size_t esz = f32 ? 4 : 2;
                orow = static_cast<uint8_t*>(p.o) + (static_cast<size_t>(un.q0 + row) * p.H + un.bh % p.H) * kD * esz +
                       static_cast<size_t>(g) * 128 * esz;
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (k >= n_chunks) break;
                if (!by_rows) {
                    if (lane == 0) bulk_wait_group_read0();  // the stage's previous store has read it
                    __syncwarp();
                }
#pragma unroll
                for (int q = 0; q < 8; ++q) {
                    uint4 v;
                    if (f32) {
                        const int c0 = k * 32 + q * 4;
                        v.x = __float_as_uint(__uint_as_float(ov[c0 + 0]) * inv);
                        v.y = __float_as_uint(__uint_as_float(ov[c0 + 1]) * inv);
                        v.z = __float_as_uint(__uint_as_float(ov[c0 + 2]) * inv);
                        v.w = __float_as_uint(__uint_as_float(ov[c0 + 3]) * inv);
                    } else {
                        const int c0 = (k * 64 + q * 8) & 127;
                        v.x = pack_bf16x2(__uint_as_float(ov[c0 + 0]) * inv, __uint_as_float(ov[c0 + 1]) * inv);
                        v.y = pack_bf16x2(__uint_as_float(ov[c0 + 2]) * inv, __uint_as_float(ov[c0 + 3]) * inv);
                        v.z = pack_bf16x2(__uint_as_float(ov[c0 + 4]) * inv, __uint_as_float(ov[c0 + 5]) * inv);
                        v.w = pack_bf16x2(__uint_as_float(ov[c0 + 6]) * inv, __uint_as_float(ov[c0 + 7]) * inv);
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
                        tma_store_3d(&p.tm_o, stg, g * 128 + k * (f32 ? 32 : 64), un.bh % p.H, un.q0 + un.i0 + wq * 32);
                    } else {
                        if (un.i0 + wq * 32 < p.Lq)
                            tma_store_3d(&p.tm_o, stg, g * 128 + k * (f32 ? 32 : 64), un.i0 + wq * 32, un.bh);
                    }
                    bulk_commit_group();
                }
            }
            // LSE: [B*H][Lq] for a batched call, [H][total_q] for a packed one
            if (g == 0 && row < un.lq) {
                const size_t li = VARLEN ? static_cast<size_t>(un.bh % p.H) * p.Lq + un.q0 + row
                                         : static_cast<size_t>(un.bh) * p.Lq + row;
                p.lse[li] = m_ref * p.scale + logf(l_row);
            }
        }
    }

    if (warp < 8 && lane == 0) bulk_wait_group0();
    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
    if (threadIdx.x == 0 && p.sched) {
        __threadfence();
        if (atomicAdd(p.sched + 1, 1u) == gridDim.x - 1) {
            atomicExch(p.sched, 0u);
            atomicExch(p.sched + 1, 0u);
        }
    }
}

template <bool VARLEN, bool BSPARSE>
cudaError_t launch_fwd256_kernel(const FwdParams& p, int num_sms, cudaStream_t stream) {
    const long long tiles = VARLEN ? p.max_pairs : (p.Lq + kBM - 1) / kBM;
    const long long units = static_cast<long long>(p.B) * p.H * tiles;
    if (units == 0) return cudaSuccess;
    const dim3 grid(static_cast<unsigned>(units < num_sms ? units : num_sms));
    cudaFuncAttributes a{};
    cudaError_t e = cudaFuncGetAttributes(&a, fa_fwd256_kernel<VARLEN, BSPARSE>);
    if (e != cudaSuccess) return e;
    // the setmaxnreg split must fit the registers the block is launched with
    if (static_cast<long long>(a.numRegs) * kFwdThreads < 2LL * 128 * kFwdRegsSoftmax + 128LL * kFwdRegsOther)
        return cudaErrorInvalidConfiguration;
    e = cudaFuncSetAttribute(fa_fwd256_kernel<VARLEN, BSPARSE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Lay256::kBytes);
    if (e != cudaSuccess) return e;
    fa_fwd256_kernel<VARLEN, BSPARSE><<<grid, kFwdThreads, Lay256::kBytes, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

int fwd256_smem_bytes() { return Lay256::kBytes; }

cudaError_t launch_fwd256(const FwdParams& p, int num_sms, cudaStream_t stream) {
    return launch_fwd256_kernel<false, false>(p, num_sms, stream);
}

// Packed batch: p.max_pairs is the number of 128-row query tiles of the longest sequence.
cudaError_t launch_fwd256_varlen(const FwdParams& p, int num_sms, cudaStream_t stream) {
    return launch_fwd256_kernel<true, false>(p, num_sms, stream);
}

// Block-sparse batch (the plan has run on the stream before): p.bs_* set.
cudaError_t launch_fwd256_blocksparse(const FwdParams& p, int num_sms, cudaStream_t stream) {
    return launch_fwd256_kernel<false, true>(p, num_sms, stream);
}

}  // namespace fa
