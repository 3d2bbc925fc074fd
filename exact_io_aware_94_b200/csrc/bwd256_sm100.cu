// Backward pass of exact attention for sm_100a at head dimension 256, by
// recomputation ("Backward Pass Efficiency": per-row statistics instead of
// stored matrices; glossary "How it works": intermediates are recomputed).
// The same formulas as the d <= 128 kernels (P = exp(scale q.k - LSE),
// dS = P o (dP - D), dV = P^T dO, dK = scale dS^T Q, dQ = scale dS K), with a
// shape chosen for the tensor-memory budget at d = 256: the dK and dV
// accumulators of a 128-key tile would need 512 columns by themselves.
//
//   fa_bwd_dkdv256  one CTA per (b, h, 128-key tile, half of d): K and V stay in
//                   shared memory; per 64-query tile, S^T = K Q^T and
//                   dP^T = V dO^T over all 256 columns (SS MMA, N = 64), one
//                   thread per key row forms P^T and dS^T (bf16, back into
//                   TMEM; warpgroup g takes queries [32g, 32g + 32)), then
//                   dV_h += P^T dO[:, h] and dK_h += dS^T Q[:, h] on this CTA's
//                   128 columns h (TS MMA).  TMEM: S^T 64, dP^T 64, dV_h 128,
//                   dK_h 128 columns.  The two halves recompute S^T and dP^T:
//                   6 GEMMs for the 5 of the formulas.
//   fa_bwd_dq256    one CTA per (b, h, 128-query tile): Q and dO stay in shared
//                   memory; per 64-key tile, S = Q K^T and dP = dO V^T, one
//                   thread per query row forms dS (bf16, into TMEM), then
//                   dQ += dS K (TS MMA, N = 256).  TMEM: S 64, dP 64, dQ 256.
// D = rowsum(dO o O) comes from the same pre-kernel as for d <= 128.  No
// atomics: the result is deterministic.  Each K/V (or Q/dO) tile is loaded once
// per use into a single stage; its next load waits until the MMAs reading it
// are done.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fa_internal.h"
#include "ptx.cuh"

namespace fa {
namespace {

constexpr int kD = 256;
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------- dK, dV (one half of d per CTA)
struct DkdvLay256 {
    static constexpr int kBig = 128 * 64 * 2;          // box: 128 rows x 64 bf16 (16 KB)
    static constexpr int kSmall = 64 * 64 * 2;         // box: 64 rows x 64 bf16 (8 KB)
    static constexpr int kKOff = 0;                    // K [128 keys][256], 4 boxes
    static constexpr int kVOff = kKOff + 4 * kBig;     // V
    static constexpr int kQStage = 4 * kSmall;         // Q [64 queries][256], 4 boxes
    static constexpr int kQOff = kVOff + 4 * kBig;     // 2 stages
    static constexpr int kGOff = kQOff + 2 * kQStage;  // dO, 1 stage
    static constexpr int kStatOff = kGOff + 4 * kSmall;  // per Q stage: lse2[64], dsum[64]
    static constexpr int kBarOff = kStatOff + 2 * 2 * 64 * 4;
    // kv, q[2], dO, qfree[2], dofree, s, dp, p, ds, acc, drain
    static constexpr int kNumBars = 13;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kBytes = kMiscOff + 16 + 1024;
};

__global__ void __launch_bounds__(kBwdThreads, 1) fa_bwd_dkdv256(const __grid_constant__ BwdParams p) {
    using Lay = DkdvLay256;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sK = smem + Lay::kKOff;
    uint8_t* sV = smem + Lay::kVOff;
    uint8_t* sQ = smem + Lay::kQOff;
    uint8_t* sG = smem + Lay::kGOff;
    float* sStat = reinterpret_cast<float*>(smem + Lay::kStatOff);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
    // Q tiles and their statistics are double-buffered: the next tile's copies and
    // statistic loads run while this tile's MMAs and elementwise work do.  (Without that,
    // each tile waited a full load after the previous tile's last MMA freed the buffer.)
    uint64_t* bar_kv = bars;         // K and V landed
    uint64_t* bar_q = bars + 1;      // [stage]: Q tile and its statistics landed
    uint64_t* bar_do = bars + 3;     // dO tile landed
    uint64_t* bar_qfree = bars + 4;  // [stage]: S^T and dK MMAs are done with the Q tile (and its statistics)
    uint64_t* bar_dofree = bars + 6; // dP^T and dV MMAs are done with the dO tile
    uint64_t* bar_s = bars + 7;
    uint64_t* bar_dp = bars + 8;
    uint64_t* bar_p = bars + 9;
    uint64_t* bar_ds = bars + 10;
    uint64_t* bar_acc = bars + 11;
    uint64_t* bar_drain = bars + 12;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int BH = p.B * p.H;
    const int half = static_cast<int>(blockIdx.x) & 1;   // columns [128 half, 128 half + 128) of dK, dV
    // small key tiles first (they see the most queries), in groups of heads whose Q and dO stay in L2
    int kt, bh;
    grouped_block(static_cast<int>(blockIdx.x) >> 1, BH, (p.Lk + 127) / 128, p.hg_kv, kt, bh);
    const int j0 = kt * 128;
    const int off = p.Lk - p.Lq;
    const int nq_all = (p.Lq + 63) / 64;
    const int qt0 = p.causal ? max(0, j0 - off) / 64 : 0;
    const int nq = nq_all - qt0;  // >= 1: the last query row sees every key

    // TMEM columns: S^T [0,64) dP^T [64,128) dV_h [128,256) dK_h [256,384)
    constexpr uint32_t kColS = 0, kColDP = 64, kColDV = 128, kColDK = 256;

    if (threadIdx.x == 0) {
        mbar_init(bar_kv, 1);
        for (int st = 0; st < 2; ++st) {
            mbar_init(&bar_q[st], 1 + 32);
            mbar_init(&bar_qfree[st], 1);
        }
        mbar_init(bar_do, 1);
        mbar_init(bar_dofree, 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_dp, 1);
        mbar_init(bar_p, 256);
        mbar_init(bar_ds, 256);
        mbar_init(bar_acc, 1);
        mbar_init(bar_drain, 1);
        *abort_flag = (atomicAdd(p.status, 0) == FA_ERR_TIMEOUT) ? 1 : 0;
        fence_barrier_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 8) {
        // ================= producer: K, V once; then Q (+ statistics) and dO per query tile
        auto wait = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.status));
        };
        int issued_q = 0, issued_do = 0;
        bool kv_issued = false;
        if (!*abort_flag) {
            mbar_arrive_expect_tx_w(bar_kv, 8 * Lay::kBig);
            for (int b = 0; b < 4; ++b) {
                tma_load_3d_w(sK + b * Lay::kBig, &p.tm_k, bar_kv, b * 64, j0, bh);
                tma_load_3d_w(sV + b * Lay::kBig, &p.tm_v, bar_kv, b * 64, j0, bh);
            }
            kv_issued = true;
            for (int t = 0; t < nq; ++t) {
                const int i0 = (qt0 + t) * 64;
                const int qs = t & 1;
                if (t >= 2 && !wait(&bar_qfree[qs], ((t >> 1) - 1) & 1)) break;
                mbar_arrive_expect_tx_w(&bar_q[qs], Lay::kQStage);
                for (int b = 0; b < 4; ++b)
                    tma_load_3d_w(sQ + qs * Lay::kQStage + b * Lay::kSmall, &p.tm_q64, &bar_q[qs], b * 64, i0, bh);
#pragma unroll
                for (int x = 0; x < 2; ++x) {
                    const int r = lane * 2 + x;
                    const int i = i0 + r;
                    const bool valid = i < p.Lq;
                    const size_t idx = static_cast<size_t>(bh) * p.Lq + i;
                    sStat[qs * 128 + r] = valid ? p.lse[idx] * kLog2e : INFINITY;  // P = 0 for rows past Lq
                    sStat[qs * 128 + 64 + r] = valid ? p.dsum[idx] : 0.0f;
                }
                mbar_arrive(&bar_q[qs]);
                ++issued_q;
                if (t > 0 && !wait(bar_dofree, (t - 1) & 1)) break;
                mbar_arrive_expect_tx_w(bar_do, 4 * Lay::kSmall);
                for (int b = 0; b < 4; ++b) tma_load_3d_w(sG + b * Lay::kSmall, &p.tm_do64, bar_do, b * 64, i0, bh);
                ++issued_do;
            }
        }
        // every copy issued here lands before the CTA exits
        if (kv_issued) mbar_wait_drain(bar_kv, 0, p.status);
        for (int t = (issued_q > 2 ? issued_q - 2 : 0); t < issued_q; ++t)
            mbar_wait_drain(&bar_q[t & 1], (t >> 1) & 1, p.status);
        if (issued_do > 0) mbar_wait_drain(bar_do, (issued_do - 1) & 1, p.status);
    } else if (warp == 9) {
        // ================= MMA issuer
        auto wait = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.status));
        };
        constexpr uint32_t kIdescSS = idesc_bf16_f32(128, 64, 0, 0);
        constexpr uint32_t kIdescTS = idesc_bf16_f32(128, 128, 0, 1);
        const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV), sQa = smem_u32(sQ), sGa = smem_u32(sG);
        // X^T = A B^T over all 256 columns: A = K or V [128 keys], B = Q or dO [64 queries]
        auto issue_ss = [&](uint32_t d_col, uint32_t a_base, uint32_t b_base) {
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
                umma_ss_w(tmem_base + d_col, smem_desc_sw128(a_base + (kk >> 2) * Lay::kBig + (kk & 3) * 32, 16, 1024),
                          smem_desc_sw128(b_base + (kk >> 2) * Lay::kSmall + (kk & 3) * 32, 16, 1024), kIdescSS,
                          kk > 0 ? 1u : 0u);
            }
        };
        // acc_h += X^T(bf16, TMEM) B[:, half]: K = 64 queries in 4 steps of 16; warpgroup g's 32
        // queries sit at TMEM columns [32g, 32g + 16) of the X^T region; B is MN-major over the
        // two 64-column boxes of this CTA's half.
        auto issue_ts = [&](uint32_t d_col, uint32_t a_col, uint32_t b_base, bool first) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t a = tmem_base + a_col + (kk >> 1) * 32 + (kk & 1) * 8;
                umma_ts_w(tmem_base + d_col, a,
                          smem_desc_sw128(b_base + (2 * half) * Lay::kSmall + kk * 2048, Lay::kSmall, 1024),
                          kIdescTS, (!first || kk > 0) ? 1u : 0u);
            }
        };
        bool ok = wait(bar_kv, 0);
        for (int t = 0; ok && t < nq; ++t) {
            // S^T(t) overwrites P^T(t-1) and dP^T(t) overwrites dS^T(t-1): both follow dK(t-1)
            const uint32_t sQt = sQa + (t & 1) * Lay::kQStage;
            if (!(ok = wait(&bar_q[t & 1], (t >> 1) & 1))) break;
            tc_fence_after();
            issue_ss(kColS, sKa, sQt);
            umma_commit_w(bar_s);
            if (!(ok = wait(bar_do, t & 1))) break;
            tc_fence_after();
            issue_ss(kColDP, sVa, sGa);
            umma_commit_w(bar_dp);
            if (!(ok = wait(bar_p, t & 1))) break;
            tc_fence_after();
            issue_ts(kColDV, kColS, sGa, t == 0);  // dV_h += P^T dO[:, h]
            umma_commit_w(bar_dofree);
            if (!(ok = wait(bar_ds, t & 1))) break;
            tc_fence_after();
            issue_ts(kColDK, kColDP, sQt, t == 0);  // dK_h += dS^T Q[:, h]
            umma_commit_w(&bar_qfree[t & 1]);
        }
        if (ok) umma_commit_w(bar_acc);
        umma_commit_w(bar_drain);
        mbar_wait_drain(bar_drain, 0, p.status);
    } else if (warp < 8) {
        // ================= elementwise: thread = key row, warpgroup g = queries [32g, 32g + 32)
        const int g = warp >> 2, wq = warp & 3;
        const int r = wq * 32 + lane;
        const int key = j0 + r;
        const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tS = tmem_base + lane_bits + kColS + g * 32;
        const uint32_t tDP = tmem_base + lane_bits + kColDP + g * 32;
        const float sl2 = p.scale_log2;
        bool ok = true;
        for (int t = 0; t < nq; ++t) {
            const int i0 = (qt0 + t) * 64 + g * 32;  // first query of this warpgroup's columns
            ok = __all_sync(0xffffffffu, mbar_wait(bar_s, t & 1, abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            float pr[32];
            {
                uint32_t u[32];
                tmem_ld32(tS, u);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) pr[x] = __uint_as_float(u[x]);
            }
            if (p.causal && (j0 + 127 > i0 + off)) {
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    if (key > i0 + c + off) pr[c] = -INFINITY;
            }
            // the statistics of tile t stay in place until its dK MMA is done
            const float4* lse4 = reinterpret_cast<const float4*>(sStat + (t & 1) * 128 + g * 32);
#pragma unroll
            for (int c4 = 0; c4 < 8; ++c4) {
                const float4 lv = lse4[c4];
                const float lc[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
                for (int x = 0; x < 4; ++x) pr[c4 * 4 + x] = ex2_approx(fmaf(pr[c4 * 4 + x], sl2, -lc[x]));
            }
            {
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) pk[c] = pack_bf16x2(pr[2 * c], pr[2 * c + 1]);
                tmem_st16(tS, pk);
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(bar_p);
            ok = __all_sync(0xffffffffu, mbar_wait(bar_dp, t & 1, abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            {
                uint32_t u[32], pk[16];
                tmem_ld32(tDP, u);
                tmem_wait_ld();
                const float4* d4 = reinterpret_cast<const float4*>(sStat + (t & 1) * 128 + 64 + g * 32);
#pragma unroll
                for (int c4 = 0; c4 < 8; ++c4) {
                    const float4 dv = d4[c4];
                    const int c = c4 * 4;
                    pk[c4 * 2] = pack_bf16x2(pr[c] * (__uint_as_float(u[c]) - dv.x),
                                             pr[c + 1] * (__uint_as_float(u[c + 1]) - dv.y));
                    pk[c4 * 2 + 1] = pack_bf16x2(pr[c + 2] * (__uint_as_float(u[c + 2]) - dv.z),
                                                 pr[c + 3] * (__uint_as_float(u[c + 3]) - dv.w));
                }
                tmem_st16(tDP, pk);
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(bar_ds);
        }
        // epilogue: dV_h = acc, dK_h = scale * acc; warpgroup g writes columns
        // [128 half + 64g, 128 half + 64g + 64)
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_acc, 0, abort_flag, p.status));
        if (ok) {
            tc_fence_after();
            const bool valid = key < p.Lk;
            const size_t rowoff = (static_cast<size_t>(bh) * p.Lk + key) * kD + half * 128 + g * 64;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const uint32_t col0 = (part == 0 ? kColDV : kColDK) + g * 64;
                __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(part == 0 ? p.dv : p.dk) + rowoff;
                const float mul = (part == 0) ? 1.0f : p.scale;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    uint32_t u[32];
                    tmem_ld32(tmem_base + lane_bits + col0 + c * 32, u);
                    tmem_wait_ld();
                    if (valid) {  // 32-byte stores
#pragma unroll
                        for (int x = 0; x < 2; ++x) {
                            uint32_t v8[8];
#pragma unroll
                            for (int y = 0; y < 8; ++y)
                                v8[y] = pack_bf16x2(__uint_as_float(u[16 * x + 2 * y]) * mul,
                                                    __uint_as_float(u[16 * x + 2 * y + 1]) * mul);
                            st_global_v8(dst + c * 32 + 16 * x, v8);
                        }
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

// ---------------------------------------------------------------- dQ
struct DqLay256 {
    static constexpr int kBig = 128 * 64 * 2;        // box: 128 rows x 64 bf16
    static constexpr int kSmall = 64 * 64 * 2;       // box: 64 rows x 64 bf16
    static constexpr int kQOff = 0;                  // Q [128 queries][256], 4 boxes
    static constexpr int kGOff = kQOff + 4 * kBig;   // dO
    static constexpr int kKStage = 4 * kSmall;      // K [64 keys][256], 4 boxes
    static constexpr int kKOff = kGOff + 4 * kBig;   // 2 stages
    static constexpr int kVOff = kKOff + 2 * kKStage; // V, 1 stage
    static constexpr int kBarOff = kVOff + 4 * kSmall;
    // qd, k[2], v, kfree[2], vfree, s, dp, dsr, acc, drain
    static constexpr int kNumBars = 12;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kBytes = kMiscOff + 16 + 1024;
};

__global__ void __launch_bounds__(kBwdThreads, 1) fa_bwd_dq256(const __grid_constant__ BwdParams p) {
    using Lay = DqLay256;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + Lay::kQOff;
    uint8_t* sG = smem + Lay::kGOff;
    uint8_t* sK = smem + Lay::kKOff;
    uint8_t* sV = smem + Lay::kVOff;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
    // K tiles are double-buffered: a K tile is held until its dQ MMAs, the last of its
    // key tile, so with one buffer the next tile's copy could only start after them.
    uint64_t* bar_qd = bars;         // Q and dO landed
    uint64_t* bar_k = bars + 1;      // [stage]: K tile landed
    uint64_t* bar_v = bars + 3;      // V tile landed
    uint64_t* bar_kfree = bars + 4;  // [stage]: S and dQ MMAs are done with the K tile
    uint64_t* bar_vfree = bars + 6;  // the dP MMAs are done with the V tile
    uint64_t* bar_s = bars + 7;
    uint64_t* bar_dp = bars + 8;
    uint64_t* bar_dsr = bars + 9;
    uint64_t* bar_acc = bars + 10;
    uint64_t* bar_drain = bars + 11;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int BH = p.B * p.H;
    const int nq_all = (p.Lq + 127) / 128;
    // long causal rows first, in groups of heads whose K and V stay in L2
    int t, bh;
    grouped_block(static_cast<int>(blockIdx.x), BH, nq_all, p.hg_q, t, bh);
    const int qt = nq_all - 1 - t;
    const int i0 = qt * 128;
    const int off = p.Lk - p.Lq;
    const int nk_all = (p.Lk + 63) / 64;
    const int nk = p.causal ? min(nk_all, (min(i0 + 127, p.Lq - 1) + off) / 64 + 1) : nk_all;

    // TMEM columns: S [0,64) dP [64,128) dQ [256,512)
    constexpr uint32_t kColS = 0, kColDP = 64, kColDQ = 256;

    if (threadIdx.x == 0) {
        mbar_init(bar_qd, 1);
        for (int st = 0; st < 2; ++st) {
            mbar_init(&bar_k[st], 1);
            mbar_init(&bar_kfree[st], 1);
        }
        mbar_init(bar_v, 1);
        mbar_init(bar_vfree, 1);
        mbar_init(bar_s, 1);
        mbar_init(bar_dp, 1);
        mbar_init(bar_dsr, 256);
        mbar_init(bar_acc, 1);
        mbar_init(bar_drain, 1);
        *abort_flag = (atomicAdd(p.status, 0) == FA_ERR_TIMEOUT) ? 1 : 0;
        fence_barrier_init();
    }
    if (warp == 9) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 8) {
        // ================= producer: Q and dO once; K_j and V_j per key tile
        auto wait = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.status));
        };
        int issued_k = 0, issued_v = 0;
        bool qd_issued = false;
        if (!*abort_flag) {
            mbar_arrive_expect_tx_w(bar_qd, 8 * Lay::kBig);
            for (int b = 0; b < 4; ++b) {
                tma_load_3d_w(sQ + b * Lay::kBig, &p.tm_q, bar_qd, b * 64, i0, bh);
                tma_load_3d_w(sG + b * Lay::kBig, &p.tm_do, bar_qd, b * 64, i0, bh);
            }
            qd_issued = true;
            for (int j = 0; j < nk; ++j) {
                const int ks = j & 1;
                if (j >= 2 && !wait(&bar_kfree[ks], ((j >> 1) - 1) & 1)) break;
                mbar_arrive_expect_tx_w(&bar_k[ks], Lay::kKStage);
                for (int b = 0; b < 4; ++b)
                    tma_load_3d_w(sK + ks * Lay::kKStage + b * Lay::kSmall, &p.tm_k64, &bar_k[ks], b * 64, j * 64, bh);
                ++issued_k;
                if (j > 0 && !wait(bar_vfree, (j - 1) & 1)) break;
                mbar_arrive_expect_tx_w(bar_v, 4 * Lay::kSmall);
                for (int b = 0; b < 4; ++b) tma_load_3d_w(sV + b * Lay::kSmall, &p.tm_v64, bar_v, b * 64, j * 64, bh);
                ++issued_v;
            }
        }
        if (qd_issued) mbar_wait_drain(bar_qd, 0, p.status);
        for (int j = (issued_k > 2 ? issued_k - 2 : 0); j < issued_k; ++j)
            mbar_wait_drain(&bar_k[j & 1], (j >> 1) & 1, p.status);
        if (issued_v > 0) mbar_wait_drain(bar_v, (issued_v - 1) & 1, p.status);
    } else if (warp == 9) {
        // ================= MMA issuer
        auto wait = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.status));
        };
        constexpr uint32_t kIdescSS = idesc_bf16_f32(128, 64, 0, 0);
        constexpr uint32_t kIdescTS = idesc_bf16_f32(128, kD, 0, 1);
        const uint32_t sQa = smem_u32(sQ), sGa = smem_u32(sG), sKa = smem_u32(sK), sVa = smem_u32(sV);
        // X = A B^T over all 256 columns: A = Q or dO [128 queries], B = K or V [64 keys]
        auto issue_ss = [&](uint32_t d_col, uint32_t a_base, uint32_t b_base) {
#pragma unroll
            for (int kk = 0; kk < kD / 16; ++kk) {
                umma_ss_w(tmem_base + d_col, smem_desc_sw128(a_base + (kk >> 2) * Lay::kBig + (kk & 3) * 32, 16, 1024),
                          smem_desc_sw128(b_base + (kk >> 2) * Lay::kSmall + (kk & 3) * 32, 16, 1024), kIdescSS,
                          kk > 0 ? 1u : 0u);
            }
        };
        bool ok = wait(bar_qd, 0);
        for (int j = 0; ok && j < nk; ++j) {
            // S(j) overwrites dS(j-1) and dP(j) overwrites dP(j-1): both follow dQ(j-1)
            const uint32_t sKj = sKa + (j & 1) * Lay::kKStage;
            if (!(ok = wait(&bar_k[j & 1], (j >> 1) & 1))) break;
            tc_fence_after();
            issue_ss(kColS, sQa, sKj);
            umma_commit_w(bar_s);
            if (!(ok = wait(bar_v, j & 1))) break;
            tc_fence_after();
            issue_ss(kColDP, sGa, sVa);
            umma_commit_w(bar_dp);
            umma_commit_w(bar_vfree);
            if (!(ok = wait(bar_dsr, j & 1))) break;
            tc_fence_after();
            // dQ += dS K: K = 64 keys in 4 steps of 16 (warpgroup g's 32 keys at TMEM columns
            // [32g, 32g + 16)); B = K tile, MN-major over its four 64-column boxes
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint32_t a = tmem_base + kColS + (kk >> 1) * 32 + (kk & 1) * 8;
                umma_ts_w(tmem_base + kColDQ, a, smem_desc_sw128(sKj + kk * 2048, Lay::kSmall, 1024), kIdescTS,
                          (j > 0 || kk > 0) ? 1u : 0u);
            }
            umma_commit_w(&bar_kfree[j & 1]);
        }
        if (ok) umma_commit_w(bar_acc);
        umma_commit_w(bar_drain);
        mbar_wait_drain(bar_drain, 0, p.status);
    } else if (warp < 8) {
        // ================= elementwise: thread = query row, warpgroup g = keys [32g, 32g + 32)
        const int g = warp >> 2, wq = warp & 3;
        const int r = wq * 32 + lane;
        const int row = i0 + r;
        const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tS = tmem_base + lane_bits + kColS + g * 32;
        const uint32_t tDP = tmem_base + lane_bits + kColDP + g * 32;
        const float sl2 = p.scale_log2;
        const bool row_valid = row < p.Lq;
        const size_t ridx = static_cast<size_t>(bh) * p.Lq + row;
        const float lse2 = row_valid ? p.lse[ridx] * kLog2e : INFINITY;
        const float dsum = row_valid ? p.dsum[ridx] : 0.0f;
        const int limit = p.causal ? min(row + off, p.Lk - 1) : p.Lk - 1;  // highest permitted key
        bool ok = true;
        for (int j = 0; j < nk; ++j) {
            const int k0 = j * 64 + g * 32;
            ok = __all_sync(0xffffffffu, mbar_wait(bar_s, j & 1, abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            float pr[32];
            {
                uint32_t u[32];
                tmem_ld32(tS, u);
                tmem_wait_ld();
#pragma unroll
                for (int x = 0; x < 32; ++x) pr[x] = __uint_as_float(u[x]);
            }
            if (k0 + 31 > limit) {
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    if (k0 + c > limit) pr[c] = -INFINITY;
            }
#pragma unroll
            for (int c = 0; c < 32; ++c) pr[c] = ex2_approx(fmaf(pr[c], sl2, -lse2));
            ok = __all_sync(0xffffffffu, mbar_wait(bar_dp, j & 1, abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            {
                uint32_t u[32], pk[16];
                tmem_ld32(tDP, u);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    pk[c] = pack_bf16x2(pr[2 * c] * (__uint_as_float(u[2 * c]) - dsum),
                                        pr[2 * c + 1] * (__uint_as_float(u[2 * c + 1]) - dsum));
                tmem_st16(tS, pk);  // dS over this thread's own scores
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(bar_dsr);
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_acc, 0, abort_flag, p.status));
        if (ok) {
            tc_fence_after();
            // warpgroup g writes columns [128g, 128g + 128) of dQ
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.dq) + ridx * kD + g * 128;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                uint32_t u[32];
                tmem_ld32(tmem_base + lane_bits + kColDQ + g * 128 + c * 32, u);
                tmem_wait_ld();
                if (row_valid) {  // 32-byte stores
#pragma unroll
                    for (int x = 0; x < 2; ++x) {
                        uint32_t v8[8];
#pragma unroll
                        for (int y = 0; y < 8; ++y)
                            v8[y] = pack_bf16x2(__uint_as_float(u[16 * x + 2 * y]) * p.scale,
                                                __uint_as_float(u[16 * x + 2 * y + 1]) * p.scale);
                        st_global_v8(dst + c * 32 + 16 * x, v8);
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 9) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 512);
    }
}

}  // namespace

// The dK/dV and dQ kernels at d = 256 (the D pre-kernel has run on `stream`).
cudaError_t launch_bwd256_main(const BwdParams& p, cudaStream_t stream) {
    const unsigned BH = static_cast<unsigned>(p.B) * p.H;
    cudaError_t e = cudaFuncSetAttribute(fa_bwd_dkdv256, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         DkdvLay256::kBytes);
    if (e != cudaSuccess) return e;
    fa_bwd_dkdv256<<<BH * ((p.Lk + 127) / 128) * 2, kBwdThreads, DkdvLay256::kBytes, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(fa_bwd_dq256, cudaFuncAttributeMaxDynamicSharedMemorySize, DqLay256::kBytes)) !=
        cudaSuccess)
        return e;
    fa_bwd_dq256<<<BH * ((p.Lq + 127) / 128), kBwdThreads, DqLay256::kBytes, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace fa
