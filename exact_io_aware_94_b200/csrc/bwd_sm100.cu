// Backward pass of exact attention for sm_100a, by recomputation.
//
// The pages keep only per-row statistics for the backward pass and recompute
// the probabilities instead of storing them ("Backward Pass Efficiency": D_i,
// l_i, m_i; glossary "How it works": intermediates are recomputed).  Here the
// saved statistic is LSE_i = m_i + ln l_i, so P_ij = exp(scale q_i.k_j - LSE_i).
// With dP = dO V^T, D_i = rowsum(dO o O), dS = P o (dP - D):
//     dV = P^T dO,   dK = scale dS^T Q,   dQ = scale dS K.
//
// Three kernels, no atomics (deterministic):
//   fa_bwd_dot   D_i = sum_c dO_ic O_ic                        (HBM-bound)
//   fa_bwd_dkdv  one CTA per (b, h, 128-key tile), loop over 128-row Q tiles:
//                S^T = K Q^T and dP^T = V dO^T (SS MMA into TMEM); one thread
//                per key row turns them into P^T and dS^T (bf16, written back
//                into TMEM); dV += P^T dO and dK += dS^T Q (TS MMA, A from TMEM).
//   fa_bwd_dq    one CTA per (b, h, 128-row Q tile), loop over 128-key tiles:
//                S = Q K^T (double-buffered) and dP = dO V^T; one thread per
//                query row forms dS (bf16, into TMEM); dQ += dS K (TS MMA).
// Each of the two heavy kernels has two elementwise warpgroups that split the
// 128 columns of every tile between them, a TMA producer warp and an MMA warp.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fa_internal.h"
#include "ptx.cuh"

namespace fa {
namespace {

constexpr float kLog2e = 1.4426950408889634f;

#ifdef FA_TEST_HOOKS
// One-shot fault (test build only): the next dK/dV CTA's K and V tiles are not
// loaded (neither the expected byte count nor the copies), so the MMA warp's
// wait for them runs out.
__device__ int g_test_skip_kv;
#endif

template <int D>
struct BwdTiles {
    static constexpr int kBoxBytes = 128 * 64 * 2;
    static constexpr int kBoxes = D / 64;
    static constexpr int kTileBytes = kBoxBytes * kBoxes;  // one 128-row bf16 tile
    static constexpr int kStages = (D == 128) ? 2 : 4;
};

// ---------------------------------------------------------------- D = rowsum(dO o O)
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_dot(BwdParams p) {
    constexpr int kLanes = D / 8;  // lanes per row, 8 elements each
    const long long rows = static_cast<long long>(p.B) * p.H * p.Lq;
    const long long row = (static_cast<long long>(blockIdx.x) * 256 + threadIdx.x) / kLanes;
    const int e0 = (threadIdx.x % kLanes) * 8;
    float acc = 0.0f;
    if (row < rows) {
        const uint4 g = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.dO) + row * D + e0);
        const float gf[8] = {__uint_as_float(g.x << 16), __uint_as_float(g.x & 0xFFFF0000u),
                             __uint_as_float(g.y << 16), __uint_as_float(g.y & 0xFFFF0000u),
                             __uint_as_float(g.z << 16), __uint_as_float(g.z & 0xFFFF0000u),
                             __uint_as_float(g.w << 16), __uint_as_float(g.w & 0xFFFF0000u)};
        if (p.o_dtype == FA_DT_F32) {
            const float4* o = reinterpret_cast<const float4*>(static_cast<const float*>(p.o) + row * D + e0);
            const float4 a = o[0], b = o[1];
            acc = gf[0] * a.x + gf[1] * a.y + gf[2] * a.z + gf[3] * a.w + gf[4] * b.x + gf[5] * b.y +
                  gf[6] * b.z + gf[7] * b.w;
        } else {
            const uint4 o = *reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.o) + row * D + e0);
            acc = gf[0] * __uint_as_float(o.x << 16) + gf[1] * __uint_as_float(o.x & 0xFFFF0000u) +
                  gf[2] * __uint_as_float(o.y << 16) + gf[3] * __uint_as_float(o.y & 0xFFFF0000u) +
                  gf[4] * __uint_as_float(o.z << 16) + gf[5] * __uint_as_float(o.z & 0xFFFF0000u) +
                  gf[6] * __uint_as_float(o.w << 16) + gf[7] * __uint_as_float(o.w & 0xFFFF0000u);
        }
    }
#pragma unroll
    for (int o = kLanes / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (row < rows && (threadIdx.x % kLanes) == 0) p.dsum[row] = acc;
}

// ---------------------------------------------------------------- dK, dV
template <int D>
struct DkdvLayout {
    using T = BwdTiles<D>;
    static constexpr int S = T::kStages;
    static constexpr int kKOff = 0;
    static constexpr int kVOff = kKOff + T::kTileBytes;
    static constexpr int kQOff = kVOff + T::kTileBytes;             // S stages
    static constexpr int kGOff = kQOff + S * T::kTileBytes;         // dO, S stages
    static constexpr int kStatOff = kGOff + S * T::kTileBytes;      // per stage: lse2[128], dsum[128]
    static constexpr int kBarOff = kStatOff + S * 2 * 128 * 4;
    // bars: kv, qd[S], empty[S], s, dp, p, ds, acc, drain, p (second half)
    static constexpr int kNumBars = 1 + 2 * S + 7;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kBytes = kMiscOff + 16 + 1024;
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) fa_bwd_dkdv(const __grid_constant__ BwdParams p) {
    using T = BwdTiles<D>;
    using Lay = DkdvLayout<D>;
    constexpr int S = Lay::S;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sK = smem + Lay::kKOff;
    uint8_t* sV = smem + Lay::kVOff;
    uint8_t* sQ = smem + Lay::kQOff;
    uint8_t* sG = smem + Lay::kGOff;
    float* sStat = reinterpret_cast<float*>(smem + Lay::kStatOff);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
    uint64_t* bar_kv = bars;
    uint64_t* bar_qd = bars + 1;
    uint64_t* bar_empty = bars + 1 + S;
    uint64_t* bar_s = bars + 1 + 2 * S;
    uint64_t* bar_dp = bar_s + 1;
    uint64_t* bar_p = bar_s + 2;
    uint64_t* bar_ds = bar_s + 3;
    uint64_t* bar_acc = bar_s + 4;
    uint64_t* bar_drain = bar_s + 5;
    // P^T is handed over in two halves of each warpgroup's 64 queries: bar_p for queries
    // [0, 32), bar_p2 for [32, 64).  dV's MMAs on the first half run while the second
    // half's exponentials are computed.
    uint64_t* bar_p2 = bar_s + 6;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int BH = p.B * p.H;
    // small key tiles first (they see the most queries), in groups of heads whose Q and dO stay in L2
    int kt, bh;
    grouped_block(static_cast<int>(blockIdx.x), BH, (p.Lk + 127) / 128, p.hg_kv, kt, bh);
    const int j0 = kt * 128;
    const int off = p.Lk - p.Lq;
    const int nq_all = (p.Lq + 127) / 128;
    const int qt0 = p.causal ? max(0, j0 - off) / 128 : 0;
    const int nq = nq_all - qt0;  // >= 1: the last query row sees every key

    // TMEM columns: S^T [0,128) dP^T [128,256) dV [256,256+D) dK [256+D,256+2D)
    constexpr uint32_t kColS = 0, kColDP = 128, kColDV = 256, kColDK = 256 + D;

    if (threadIdx.x == 0) {
        mbar_init(bar_kv, 1);
        for (int s = 0; s < S; ++s) {
            mbar_init(&bar_qd[s], 1 + 32);
            mbar_init(&bar_empty[s], 1);
        }
        mbar_init(bar_s, 1);
        mbar_init(bar_dp, 1);
        mbar_init(bar_p, 256);
        mbar_init(bar_p2, 256);
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
        // ================= producer: K, V once; then Q, dO, LSE, D per query tile
        int issued = 0;
        bool kv_skipped = false;  // test build: the K/V copies were never issued
        if (!*abort_flag) {
            if (lane == 0) {
                tma_prefetch_desc(&p.tm_q);
                tma_prefetch_desc(&p.tm_do);
#ifdef FA_TEST_HOOKS
                kv_skipped = atomicExch(&g_test_skip_kv, 0) != 0;
#endif
                if (!kv_skipped) {
                    mbar_arrive_expect_tx(bar_kv, 2 * T::kTileBytes);
                    for (int b = 0; b < T::kBoxes; ++b) {
                        tma_load_3d(sK + b * T::kBoxBytes, &p.tm_k, bar_kv, b * 64, j0, bh);
                        tma_load_3d(sV + b * T::kBoxBytes, &p.tm_v, bar_kv, b * 64, j0, bh);
                    }
                }
            }
            for (int t = 0; t < nq; ++t) {
                const int s = t % S;
                bool ok = true;
                if (t >= S) ok = mbar_wait(&bar_empty[s], ((t / S) - 1) & 1, abort_flag, p.status);
                if (!__all_sync(0xffffffffu, ok)) break;
                const int i0 = (qt0 + t) * 128;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&bar_qd[s], 2 * T::kTileBytes);
                    for (int b = 0; b < T::kBoxes; ++b) {
                        tma_load_3d(sQ + s * T::kTileBytes + b * T::kBoxBytes, &p.tm_q, &bar_qd[s], b * 64, i0, bh);
                        tma_load_3d(sG + s * T::kTileBytes + b * T::kBoxBytes, &p.tm_do, &bar_qd[s], b * 64, i0, bh);
                    }
                }
                float* st = sStat + s * 256;
#pragma unroll
                for (int x = 0; x < 4; ++x) {
                    const int r = lane * 4 + x;
                    const int i = i0 + r;
                    const bool valid = i < p.Lq;
                    const size_t idx = static_cast<size_t>(bh) * p.Lq + i;
                    st[r] = valid ? p.lse[idx] * kLog2e : INFINITY;  // P = 0 for rows past Lq
                    st[128 + r] = valid ? p.dsum[idx] : 0.0f;
                }
                mbar_arrive(&bar_qd[s]);
                issued = t + 1;
            }
        }
        // every copy issued here lands before the CTA exits (each barrier is at the
        // phase of its last copy)
        if (lane == 0 && issued > 0) {
            if (!kv_skipped) mbar_wait_drain(bar_kv, 0, p.status);
            for (int t = max(0, issued - S); t < issued; ++t) mbar_wait_drain(&bar_qd[t % S], (t / S) & 1, p.status);
        }
    } else if (warp == 9) {
        // ================= MMA issuer: the whole warp runs the loop (operands stay
        // warp-uniform), one lane chosen by elect.sync issues each MMA and commit
        auto wait = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.status));
        };
        {
            constexpr uint32_t kIdescSS = idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t kIdescTS = idesc_bf16_f32(128, D, 0, 1);
            const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV), sQa = smem_u32(sQ), sGa = smem_u32(sG);
            // S^T = K Q^T and dP^T = V dO^T for query tile t  (M = 128 keys, N = 128 queries, K = D)
            auto issue_st = [&](int t) {
                const int s = t % S;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * T::kBoxBytes + (kk & 3) * 32;
                    umma_ss_w(tmem_base + kColS, smem_desc_sw128(sKa + koff, 16, 1024),
                              smem_desc_sw128(sQa + s * T::kTileBytes + koff, 16, 1024), kIdescSS, kk > 0);
                }
                umma_commit_w(bar_s);
            };
            auto issue_dpt = [&](int t) {
                const int s = t % S;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * T::kBoxBytes + (kk & 3) * 32;
                    umma_ss_w(tmem_base + kColDP, smem_desc_sw128(sVa + koff, 16, 1024),
                              smem_desc_sw128(sGa + s * T::kTileBytes + koff, 16, 1024), kIdescSS, kk > 0);
                }
                umma_commit_w(bar_dp);
            };
            // Order per query tile t: dV(t), S^T(t+1), dK(t), dP^T(t+1).  S^T(t+1)
            // overwrites the columns of P^T(t), so it follows dV(t), and dP^T(t+1)
            // overwrites dS^T(t), so it follows dK(t); MMAs run in issue order.
            // The next S^T is then computed while the elementwise warps form dS(t).
            bool ok = wait(bar_kv, 0) && wait(&bar_qd[0], 0);
            if (ok && nq > 0) {
                tc_fence_after();
                issue_st(0);
                issue_dpt(0);
            }
            for (int t = 0; ok && t < nq; ++t) {
                const int s = t % S;
                const bool more = t + 1 < nq;
                // dV += P^T dO   (A = P^T from TMEM: queries 0-63 at cols [0,32), 64-127 at [64,96)),
                // 16 queries per MMA: kk = 0, 1, 4, 5 take the first half of each warpgroup's
                // queries (bar_p), kk = 2, 3, 6, 7 the second (bar_p2)
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    if (!(ok = wait(h == 0 ? bar_p : bar_p2, t & 1))) break;
                    tc_fence_after();
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const int kk = (i >> 1) * 4 + 2 * h + (i & 1);
                        const uint32_t a = tmem_base + kColS + (kk >> 2) * 64 + (kk & 3) * 8;
                        umma_ts_w(tmem_base + kColDV, a,
                                  smem_desc_sw128(sGa + s * T::kTileBytes + kk * 2048, T::kBoxBytes, 1024), kIdescTS,
                                  (t > 0 || kk > 0) ? 1u : 0u);
                    }
                }
                if (!ok) break;
                if (more) {
                    if (!(ok = wait(&bar_qd[(t + 1) % S], ((t + 1) / S) & 1))) break;
                    tc_fence_after();
                    issue_st(t + 1);
                }
                // dK += dS^T Q
                if (!(ok = wait(bar_ds, t & 1))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t a = tmem_base + kColDP + (kk >> 2) * 64 + (kk & 3) * 8;
                    umma_ts_w(tmem_base + kColDK, a,
                              smem_desc_sw128(sQa + s * T::kTileBytes + kk * 2048, T::kBoxBytes, 1024), kIdescTS,
                              (t > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit_w(&bar_empty[s]);
                if (more) issue_dpt(t + 1);
            }
            if (ok) umma_commit_w(bar_acc);
            umma_commit_w(bar_drain);
            mbar_wait_drain(bar_drain, 0, p.status);
        }
    } else {
        // ================= elementwise: thread = key row, warpgroup w = query columns [64w, 64w+64)
        const int w = warp >> 2, wq = warp & 3;
        const int r = wq * 32 + lane;
        const int key = j0 + r;
        const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t tS = tmem_base + lane_bits + kColS + w * 64;
        const uint32_t tDP = tmem_base + lane_bits + kColDP + w * 64;
        const float sl2 = p.scale_log2;
        bool ok = true;
        for (int t = 0; t < nq; ++t) {
            const int s = t % S;
            const int i0 = (qt0 + t) * 128 + w * 64;  // first query of this warpgroup's columns
            const float* lse2 = sStat + s * 256 + w * 64;
            const float* dsum = sStat + s * 256 + 128 + w * 64;
            ok = __all_sync(0xffffffffu, mbar_wait(bar_s, t & 1, abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            float pr[64];
            {
                uint32_t u[32];
                tmem_ld32(tS, u);
#pragma unroll
                for (int x = 0; x < 32; ++x) pr[x] = __uint_as_float(u[x]);
                tmem_ld32(tS + 32, u);
#pragma unroll
                for (int x = 0; x < 32; ++x) pr[32 + x] = __uint_as_float(u[x]);
                tmem_wait_ld();
            }
            // P^T = exp2(S^T * scale*log2e - LSE*log2e); causal: key > query + off -> 0.
            // Masked scores are set to -inf first, so the exponential gives exactly +0
            // with no select in its loop (the LSE of a valid row is finite; rows past
            // Lq carry +inf).
            if (p.causal && (j0 + 127 > i0 + off)) {
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    if (key > i0 + c + off) pr[c] = -INFINITY;
            }
            const float4* lse4 = reinterpret_cast<const float4*>(lse2);  // broadcast reads, 4 per load
#pragma unroll
            for (int h = 0; h < 2; ++h) {  // queries [32h, 32h + 32) of this warpgroup
#pragma unroll
                for (int c4 = 8 * h; c4 < 8 * h + 8; ++c4) {
                    const float4 lv = lse4[c4];
                    const float lc[4] = {lv.x, lv.y, lv.z, lv.w};
#pragma unroll
                    for (int x = 0; x < 4; ++x) pr[c4 * 4 + x] = ex2_approx(fmaf(pr[c4 * 4 + x], sl2, -lc[x]));
                }
                uint32_t pk[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) pk[c] = pack_bf16x2(pr[32 * h + 2 * c], pr[32 * h + 2 * c + 1]);
                tmem_st16(tS + 16 * h, pk);
                tmem_wait_st();
                tc_fence_before();
                mbar_arrive(h == 0 ? bar_p : bar_p2);
            }
            ok = __all_sync(0xffffffffu, mbar_wait(bar_dp, t & 1, abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            {
                const float4* d4 = reinterpret_cast<const float4*>(dsum);
                uint32_t u[32], pk[32];
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    tmem_ld32(tDP + 32 * h, u);
                    tmem_wait_ld();
#pragma unroll
                    for (int c4 = 0; c4 < 8; ++c4) {
                        const float4 dv = d4[h * 8 + c4];
                        const int c = h * 32 + c4 * 4;
                        pk[h * 16 + c4 * 2] = pack_bf16x2(pr[c] * (__uint_as_float(u[c4 * 4]) - dv.x),
                                                          pr[c + 1] * (__uint_as_float(u[c4 * 4 + 1]) - dv.y));
                        pk[h * 16 + c4 * 2 + 1] = pack_bf16x2(pr[c + 2] * (__uint_as_float(u[c4 * 4 + 2]) - dv.z),
                                                              pr[c + 3] * (__uint_as_float(u[c4 * 4 + 3]) - dv.w));
                    }
                }
                tmem_st32(tDP, pk);
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(bar_ds);
        }
        // epilogue: dV = acc, dK = scale * acc; warpgroup w writes columns [w*D/2, (w+1)*D/2)
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_acc, 0, abort_flag, p.status));
        if (ok) {
            tc_fence_after();
            const bool valid = key < p.Lk;
            const size_t rowoff = (static_cast<size_t>(bh) * p.Lk + key) * D;
#pragma unroll
            for (int part = 0; part < 2; ++part) {
                const uint32_t col0 = (part == 0 ? kColDV : kColDK) + w * (D / 2);
                __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(part == 0 ? p.dv : p.dk) + rowoff + w * (D / 2);
                const float mul = (part == 0) ? 1.0f : p.scale;
#pragma unroll
                for (int c = 0; c < D / 64; ++c) {
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
template <int D>
struct DqLayout {
    using T = BwdTiles<D>;
    static constexpr int S = T::kStages;
    static constexpr int kQOff = 0;
    static constexpr int kGOff = kQOff + T::kTileBytes;
    static constexpr int kKOff = kGOff + T::kTileBytes;  // S stages
    static constexpr int kVOff = kKOff + S * T::kTileBytes;
    static constexpr int kBarOff = kVOff + S * T::kTileBytes;
    // bars: qd, k[S], v[S], empty[S], s[2], dp, dsr, acc, drain
    static constexpr int kNumBars = 1 + 3 * S + 2 + 4;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kBytes = kMiscOff + 16 + 1024;
};

template <int D>
__global__ void __launch_bounds__(kBwdThreads, 1) fa_bwd_dq(const __grid_constant__ BwdParams p) {
    using T = BwdTiles<D>;
    using Lay = DqLayout<D>;
    constexpr int S = Lay::S;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + Lay::kQOff;
    uint8_t* sG = smem + Lay::kGOff;
    uint8_t* sK = smem + Lay::kKOff;
    uint8_t* sV = smem + Lay::kVOff;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
    uint64_t* bar_qd = bars;
    uint64_t* bar_k = bars + 1;
    uint64_t* bar_v = bars + 1 + S;
    uint64_t* bar_empty = bars + 1 + 2 * S;
    uint64_t* bar_s = bars + 1 + 3 * S;  // [2]
    uint64_t* bar_dp = bar_s + 2;
    uint64_t* bar_dsr = bar_s + 3;
    uint64_t* bar_acc = bar_s + 4;
    uint64_t* bar_drain = bar_s + 5;
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
    const int nk_all = (p.Lk + 127) / 128;
    const int nk = p.causal ? min(nk_all, (min(i0 + 127, p.Lq - 1) + off) / 128 + 1) : nk_all;

    // TMEM columns: S buffers [0,128) [128,256), dP [256,384), dQ [384,384+D)
    constexpr uint32_t kColDP = 256, kColDQ = 384;

    if (threadIdx.x == 0) {
        mbar_init(bar_qd, 1);
        for (int s = 0; s < S; ++s) {
            mbar_init(&bar_k[s], 1);
            mbar_init(&bar_v[s], 1);
            mbar_init(&bar_empty[s], 1);
        }
        mbar_init(&bar_s[0], 1);
        mbar_init(&bar_s[1], 1);
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
        // producer: whole warp, one elected lane issues each copy
        auto wait = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.status));
        };
        if (!*abort_flag) {
            if (lane == 0) {
                tma_prefetch_desc(&p.tm_k);
                tma_prefetch_desc(&p.tm_v);
            }
            mbar_arrive_expect_tx_w(bar_qd, 2 * T::kTileBytes);
            for (int b = 0; b < T::kBoxes; ++b) {
                tma_load_3d_w(sQ + b * T::kBoxBytes, &p.tm_q, bar_qd, b * 64, i0, bh);
                tma_load_3d_w(sG + b * T::kBoxBytes, &p.tm_do, bar_qd, b * 64, i0, bh);
            }
            int issued = 0;
            for (int j = 0; j < nk; ++j) {
                const int s = j % S;
                if (j >= S && !wait(&bar_empty[s], ((j / S) - 1) & 1)) break;
                mbar_arrive_expect_tx_w(&bar_k[s], T::kTileBytes);
                for (int b = 0; b < T::kBoxes; ++b)
                    tma_load_3d_w(sK + s * T::kTileBytes + b * T::kBoxBytes, &p.tm_k, &bar_k[s], b * 64, j * 128, bh);
                mbar_arrive_expect_tx_w(&bar_v[s], T::kTileBytes);
                for (int b = 0; b < T::kBoxes; ++b)
                    tma_load_3d_w(sV + s * T::kTileBytes + b * T::kBoxBytes, &p.tm_v, &bar_v[s], b * 64, j * 128, bh);
                issued = j + 1;
            }
            // every copy issued here lands before the CTA exits (each barrier is at
            // the phase of its last copy)
            mbar_wait_drain(bar_qd, 0, p.status);
            for (int j = max(0, issued - S); j < issued; ++j) {
                mbar_wait_drain(&bar_k[j % S], (j / S) & 1, p.status);
                mbar_wait_drain(&bar_v[j % S], (j / S) & 1, p.status);
            }
        }
    } else if (warp == 9) {
        // MMA issuer: whole warp, one elected lane issues (see the dK/dV kernel)
        auto wait = [&](uint64_t* bar, uint32_t parity) {
            return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, p.status));
        };
        {
            constexpr uint32_t kIdescSS = idesc_bf16_f32(128, 128, 0, 0);
            constexpr uint32_t kIdescTS = idesc_bf16_f32(128, D, 0, 1);
            const uint32_t sQa = smem_u32(sQ), sGa = smem_u32(sG), sKa = smem_u32(sK), sVa = smem_u32(sV);
            auto issue_s = [&](int j) {
                const int s = j % S;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * T::kBoxBytes + (kk & 3) * 32;
                    umma_ss_w(tmem_base + (j & 1) * 128, smem_desc_sw128(sQa + koff, 16, 1024),
                            smem_desc_sw128(sKa + s * T::kTileBytes + koff, 16, 1024), kIdescSS, kk > 0);
                }
                umma_commit_w(&bar_s[j & 1]);
            };
            auto issue_dp = [&](int j) {
                const int s = j % S;
#pragma unroll
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint32_t koff = (kk >> 2) * T::kBoxBytes + (kk & 3) * 32;
                    umma_ss_w(tmem_base + kColDP, smem_desc_sw128(sGa + koff, 16, 1024),
                            smem_desc_sw128(sVa + s * T::kTileBytes + koff, 16, 1024), kIdescSS, kk > 0);
                }
                umma_commit_w(bar_dp);
            };
            bool ok = wait(bar_qd, 0) && wait(&bar_k[0], 0);
            if (ok) {
                tc_fence_after();
                issue_s(0);
                ok = wait(&bar_v[0], 0);
                if (ok) {
                    tc_fence_after();
                    issue_dp(0);
                }
            }
            for (int j = 0; ok && j < nk; ++j) {
                const int s = j % S, s1 = (j + 1) % S;
                if (j + 1 < nk) {
                    if (!(ok = wait(&bar_k[s1], ((j + 1) / S) & 1))) break;
                    tc_fence_after();
                    issue_s(j + 1);
                }
                // dS_j ready in S buffer j&1 (and dP_j read): dQ += dS_j K_j
                if (!(ok = wait(bar_dsr, j & 1))) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint32_t a = tmem_base + (j & 1) * 128 + (kk >> 2) * 64 + (kk & 3) * 8;
                    umma_ts_w(tmem_base + kColDQ, a,
                            smem_desc_sw128(sKa + s * T::kTileBytes + kk * 2048, T::kBoxBytes, 1024), kIdescTS,
                            (j > 0 || kk > 0) ? 1u : 0u);
                }
                umma_commit_w(&bar_empty[s]);
                if (j + 1 < nk) {
                    if (!(ok = wait(&bar_v[s1], ((j + 1) / S) & 1))) break;
                    tc_fence_after();
                    issue_dp(j + 1);
                }
            }
            if (ok) umma_commit_w(bar_acc);
            umma_commit_w(bar_drain);
            mbar_wait_drain(bar_drain, 0, p.status);
        }
    } else {
        // ================= elementwise: thread = query row, warpgroup w = key columns [64w, 64w+64)
        const int w = warp >> 2, wq = warp & 3;
        const int r = wq * 32 + lane;
        const int row = i0 + r;
        const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
        const float sl2 = p.scale_log2;
        const bool row_valid = row < p.Lq;
        const size_t ridx = static_cast<size_t>(bh) * p.Lq + row;
        const float lse2 = row_valid ? p.lse[ridx] * kLog2e : INFINITY;
        const float dsum = row_valid ? p.dsum[ridx] : 0.0f;
        const int limit = p.causal ? min(row + off, p.Lk - 1) : p.Lk - 1;  // highest permitted key
        bool ok = true;
        for (int j = 0; j < nk; ++j) {
            const uint32_t tS = tmem_base + lane_bits + (j & 1) * 128 + w * 64;
            const int k0 = j * 128 + w * 64;
            ok = __all_sync(0xffffffffu, mbar_wait(&bar_s[j & 1], (j >> 1) & 1, abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            float pr[64];
            {
                uint32_t u[32];
                tmem_ld32(tS, u);
#pragma unroll
                for (int x = 0; x < 32; ++x) pr[x] = __uint_as_float(u[x]);
                tmem_ld32(tS + 32, u);
#pragma unroll
                for (int x = 0; x < 32; ++x) pr[32 + x] = __uint_as_float(u[x]);
                tmem_wait_ld();
            }
            // Masked keys (causal, or past Lk) become -inf before the exponential,
            // which then gives exactly +0 with no select in its loop.
            if (k0 + 63 > i0 + off || k0 + 64 > p.Lk) {
#pragma unroll
                for (int c = 0; c < 64; ++c)
                    if (k0 + c > limit) pr[c] = -INFINITY;
            }
#pragma unroll
            for (int c = 0; c < 64; ++c) pr[c] = ex2_approx(fmaf(pr[c], sl2, -lse2));
            ok = __all_sync(0xffffffffu, mbar_wait(bar_dp, j & 1, abort_flag, p.status));
            if (!ok) break;
            tc_fence_after();
            {
                const uint32_t tDP = tmem_base + lane_bits + kColDP + w * 64;
                uint32_t u[32], pk[32];
                tmem_ld32(tDP, u);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    pk[c] = pack_bf16x2(pr[2 * c] * (__uint_as_float(u[2 * c]) - dsum),
                                        pr[2 * c + 1] * (__uint_as_float(u[2 * c + 1]) - dsum));
                tmem_ld32(tDP + 32, u);
                tmem_wait_ld();
#pragma unroll
                for (int c = 0; c < 16; ++c)
                    pk[16 + c] = pack_bf16x2(pr[32 + 2 * c] * (__uint_as_float(u[2 * c]) - dsum),
                                             pr[32 + 2 * c + 1] * (__uint_as_float(u[2 * c + 1]) - dsum));
                tmem_st32(tS, pk);
                tmem_wait_st();
            }
            tc_fence_before();
            mbar_arrive(bar_dsr);
        }
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(bar_acc, 0, abort_flag, p.status));
        if (ok) {
            tc_fence_after();
            __nv_bfloat16* dst = static_cast<__nv_bfloat16*>(p.dq) + ridx * D + w * (D / 2);
#pragma unroll
            for (int c = 0; c < D / 64; ++c) {
                uint32_t u[32];
                tmem_ld32(tmem_base + lane_bits + kColDQ + w * (D / 2) + c * 32, u);
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

template <int D>
cudaError_t launch_bwd_d(const BwdParams& p, cudaStream_t stream) {
    const long long rows = static_cast<long long>(p.B) * p.H * p.Lq;
    const long long threads = rows * (D / 8);
    fa_bwd_dot<D><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const int BH = p.B * p.H;
    const int smem1 = DkdvLayout<D>::kBytes;
    if ((e = cudaFuncSetAttribute(fa_bwd_dkdv<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem1)) !=
        cudaSuccess)
        return e;
    fa_bwd_dkdv<D><<<static_cast<unsigned>(BH) * ((p.Lk + 127) / 128), kBwdThreads, smem1, stream>>>(p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int smem2 = DqLayout<D>::kBytes;
    if ((e = cudaFuncSetAttribute(fa_bwd_dq<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem2)) !=
        cudaSuccess)
        return e;
    fa_bwd_dq<D><<<static_cast<unsigned>(BH) * ((p.Lq + 127) / 128), kBwdThreads, smem2, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

#ifdef FA_TEST_HOOKS
cudaError_t bwd_test_arm_skip_kv() {
    const int one = 1;
    return cudaMemcpyToSymbol(g_test_skip_kv, &one, sizeof(int));
}
#endif

size_t bwd_workspace_bytes(int B, int H, int Lq) {
    const size_t n = static_cast<size_t>(B) * H * Lq * sizeof(float);
    return (n + 255) & ~size_t(255);
}

cudaError_t launch_bwd(const BwdParams& p, int d, cudaStream_t stream) {
    if (d == 256) {
        const long long threads = static_cast<long long>(p.B) * p.H * p.Lq * (256 / 8);
        fa_bwd_dot<256><<<static_cast<unsigned>((threads + 255) / 256), 256, 0, stream>>>(p);
        const cudaError_t e = cudaGetLastError();
        return e != cudaSuccess ? e : launch_bwd256_main(p, stream);
    }
    return d == 128 ? launch_bwd_d<128>(p, stream) : launch_bwd_d<64>(p, stream);
}

}  // namespace fa
