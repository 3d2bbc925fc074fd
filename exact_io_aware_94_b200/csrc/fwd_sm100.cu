// Forward pass of exact attention for sm_100a.
//
// Follows the blockwise method of the pages (glossary "How it works"; "What
// FlashAttention does instead"; "The Three Running Statistics"): for each
// query tile, stream K/V tiles through on-chip memory, compute the score tile,
// update the running max m and running sum l per row, rescale the unnormalised
// output O~ when the max moves, accumulate P~ V, and divide by l at the end.
//
// B200 mapping (one CTA = 256 query rows of one (b, h)):
//   warp 8      TMA producer: Q tiles once, then K_j / V_j into a smem ring.
//   warp 9      MMA issuer (one thread): S_w = Q_w K_j^T into TMEM (SS MMA),
//               O_w += P_w V_j with P_w read from TMEM (TS MMA).
//   warps 0-3   softmax warpgroup 0 (rows 0..127 of the CTA), warps 4-7
//               warpgroup 1 (rows 128..255).  One thread owns one row: it loads
//               its score row from TMEM, applies the mask, updates m and l,
//               rescales its O~ row in TMEM when needed, and writes bf16 P~
//               back over its score row for the PV MMA.
// TMEM (512 columns): S0 [0,128) S1 [128,256) O0 [256,256+d) O1 [256+d,256+2d).
//
// Rescaling is deferred while the running max has grown by no more than
// 2^kRescaleLog2 in exp2 units: O = O~ / l holds for any common reference
// value, so the result is unchanged; only overflow headroom is spent.
// O is normalised by the sum of the bf16-rounded P~ that the MMA consumes, so
// numerator and denominator use the same weights; the LSE uses the sum of the
// unrounded P~.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "fa_internal.h"
#include "ptx.cuh"

namespace fa {
namespace {

constexpr float kRescaleLog2 = 8.0f;

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
    // barriers: q, k[S], v[S], empty[S], s[2], p[2], o[2], drain
    static constexpr int kNumBars = 1 + 3 * kStages + 2 + 2 + 2 + 1;
    static constexpr int kMiscOff = kBarOff + kNumBars * 8;
    static constexpr int kBytes = kMiscOff + 16 + 1024;  // + tmem slot/abort + alignment slack
};

template <int D>
__global__ void __launch_bounds__(kFwdThreads, 1) fa_fwd_kernel(const __grid_constant__ FwdParams p) {
    using Lay = FwdLayout<D>;
    constexpr int S = Lay::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sQ = smem + Lay::kQOff;
    uint8_t* sK = smem + Lay::kKOff;
    uint8_t* sV = smem + Lay::kVOff;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
    uint64_t* bar_q = bars;
    uint64_t* bar_k = bars + 1;
    uint64_t* bar_v = bars + 1 + S;
    uint64_t* bar_empty = bars + 1 + 2 * S;
    uint64_t* bar_s = bars + 1 + 3 * S;
    uint64_t* bar_p = bar_s + 2;
    uint64_t* bar_o = bar_p + 2;
    uint64_t* bar_drain = bar_o + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + Lay::kMiscOff);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff + 4);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;

    // ---- work unit: (b*H + h, pair of 128-row Q tiles), longest causal rows first
    const int BH = p.B * p.H;
    const int n_pairs = (p.Lq + kFwdRowsPerCta - 1) / kFwdRowsPerCta;
    const int pair = n_pairs - 1 - static_cast<int>(blockIdx.x) / BH;
    const int bh = static_cast<int>(blockIdx.x) % BH;
    const int i0 = pair * kFwdRowsPerCta;
    const int n_kv_all = (p.Lk + kFwdBN - 1) / kFwdBN;
    const int off = p.Lk - p.Lq;  // causal: query i sits at key position i + off
    int n_kv[2];
#pragma unroll
    for (int w = 0; w < 2; ++w) {
        const int first = i0 + w * kFwdBM;
        if (first >= p.Lq) {
            n_kv[w] = 0;
        } else if (p.causal) {
            const int last = min(first + kFwdBM - 1, p.Lq - 1);
            n_kv[w] = min(n_kv_all, (last + off) / kFwdBN + 1);
        } else {
            n_kv[w] = n_kv_all;
        }
    }
    const int n_max = max(n_kv[0], n_kv[1]);

    // ---- setup
    if (threadIdx.x == 0) {
        mbar_init(bar_q, 1);
        for (int s = 0; s < S; ++s) {
            mbar_init(&bar_k[s], 1);
            mbar_init(&bar_v[s], 1);
            mbar_init(&bar_empty[s], 1);
        }
        for (int w = 0; w < 2; ++w) {
            mbar_init(&bar_s[w], 1);
            mbar_init(&bar_p[w], 4 * 32);
            mbar_init(&bar_o[w], 1);
        }
        mbar_init(bar_drain, 1);
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

    if (warp == 8) {
        // ================= TMA producer =================
        if (lane == 0 && !*abort_flag) {
            uint32_t q_bytes = 0;
#pragma unroll
            for (int w = 0; w < 2; ++w)
                if (n_kv[w] > 0) q_bytes += Lay::kTileBytes;
            if (q_bytes) {
                mbar_arrive_expect_tx(bar_q, q_bytes);
#pragma unroll
                for (int w = 0; w < 2; ++w) {
                    if (n_kv[w] == 0) continue;
                    for (int b = 0; b < Lay::kBoxes; ++b)
                        tma_load_3d(sQ + w * Lay::kTileBytes + b * Lay::kBoxBytes, &p.tm_q, bar_q, b * 64,
                                    i0 + w * kFwdBM, bh);
                }
            }
            int issued = 0;
            for (int j = 0; j < n_max; ++j) {
                const int s = j % S;
                if (j >= S && !mbar_wait(&bar_empty[s], ((j / S) - 1) & 1, abort_flag, p.status)) break;
                mbar_arrive_expect_tx(&bar_k[s], Lay::kTileBytes);
                for (int b = 0; b < Lay::kBoxes; ++b)
                    tma_load_3d(sK + s * Lay::kTileBytes + b * Lay::kBoxBytes, &p.tm_k, &bar_k[s], b * 64,
                                j * kFwdBN, bh);
                mbar_arrive_expect_tx(&bar_v[s], Lay::kTileBytes);
                for (int b = 0; b < Lay::kBoxes; ++b)
                    tma_load_3d(sV + s * Lay::kTileBytes + b * Lay::kBoxBytes, &p.tm_v, &bar_v[s], b * 64,
                                j * kFwdBN, bh);
                issued = j + 1;
            }
            if (*abort_flag) {
                // Let copies already in flight land before the CTA's smem goes away.
                if (q_bytes) mbar_wait_drain(bar_q, 0, p.status);
                for (int j = max(0, issued - S); j < issued; ++j) {
                    mbar_wait_drain(&bar_k[j % S], (j / S) & 1, p.status);
                    mbar_wait_drain(&bar_v[j % S], (j / S) & 1, p.status);
                }
            }
        }
    } else if (warp == 9) {
        // ================= MMA issuer =================
        if (lane == 0 && n_max > 0) {
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
                    umma_ss(t_s, a, b, kIdescQK, kk > 0 ? 1u : 0u);
                }
                umma_commit(&bar_s[w]);
            };
            auto issue_pv = [&](int w, int s, int j) {
                const uint32_t t_p = tmem_base + w * 128;
                const uint32_t t_o = tmem_base + 256 + w * D;
#pragma unroll
                for (int kk = 0; kk < kFwdBN / 16; ++kk) {
                    const uint64_t b =
                        smem_desc_sw128(sVa + s * Lay::kTileBytes + kk * 2048, Lay::kBoxBytes, 1024);
                    umma_ts(t_o, t_p + kk * 8, b, kIdescPV, (j > 0 || kk > 0) ? 1u : 0u);
                }
            };
            bool ok = mbar_wait(bar_q, 0, abort_flag, p.status) && mbar_wait(&bar_k[0], 0, abort_flag, p.status);
            if (ok) {
                tc_fence_after();
#pragma unroll
                for (int w = 0; w < 2; ++w)
                    if (n_kv[w] > 0) issue_s(w, 0);
            }
            for (int j = 0; ok && j < n_max; ++j) {
                const int s = j % S;
                const int s1 = (j + 1) % S;
                if (!mbar_wait(&bar_v[s], (j / S) & 1, abort_flag, p.status)) break;
                const bool more = (j + 1 < n_max);
                bool k_ready = false;
#pragma unroll
                for (int w = 0; w < 2; ++w) {
                    if (j < n_kv[w]) {
                        if (!(ok = mbar_wait(&bar_p[w], j & 1, abort_flag, p.status))) break;
                        tc_fence_after();
                        issue_pv(w, s, j);
                        if (j == n_kv[w] - 1) umma_commit(&bar_o[w]);
                    }
                    if (j + 1 < n_kv[w]) {
                        if (!k_ready) {
                            if (!(ok = mbar_wait(&bar_k[s1], ((j + 1) / S) & 1, abort_flag, p.status))) break;
                            tc_fence_after();
                            k_ready = true;
                        }
                        issue_s(w, s1);
                    }
                }
                (void)more;
                umma_commit(&bar_empty[s]);
            }
            // Drain: every MMA issued by this thread completes before TMEM is freed.
            umma_commit(bar_drain);
            mbar_wait_drain(bar_drain, 0, p.status);
        }
    } else {
        // ================= softmax warpgroups =================
        const int w = warp >> 2;
        const int wq = warp & 3;
        const int row_in_tile = wq * 32 + lane;
        const int row = i0 + w * kFwdBM + row_in_tile;
        const uint32_t lane_bits = static_cast<uint32_t>(wq * 32) << 16;
        const uint32_t t_s = tmem_base + lane_bits + w * 128;
        const uint32_t t_o = tmem_base + lane_bits + 256 + w * D;
        const float sl2 = p.scale_log2;
        const int tile_first_row = i0 + w * kFwdBM;
        const int n = (w == 0) ? n_kv[0] : n_kv[1];

        float m_ref = -INFINITY;  // running max of raw scores q.k (reference for P~)
        float l = 0.0f;           // running sum of P~ as rounded to bf16: normalises O
        float l_exact = 0.0f;     // running sum of P~ before rounding: gives the LSE
        bool ok = true;
        for (int j = 0; j < n; ++j) {
            // warp-uniform outcome: the TMEM accesses below are warp-collective
            ok = __all_sync(0xffffffffu, mbar_wait(&bar_s[w], j & 1, abort_flag, p.status));
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
            const int kv0 = j * kFwdBN;
            const bool need_mask =
                (p.causal && kv0 + kFwdBN - 1 > tile_first_row + off) || (kv0 + kFwdBN > p.Lk);
            if (need_mask) {
                const int limit = p.causal ? min(row + off, p.Lk - 1) : p.Lk - 1;
#pragma unroll
                for (int c = 0; c < kFwdBN; ++c)
                    if (kv0 + c > limit) s[c] = -INFINITY;
            }
            float mx;
            {
                float mp[8];
#pragma unroll
                for (int x = 0; x < 8; ++x) mp[x] = s[x];
#pragma unroll
                for (int c = 8; c < kFwdBN; ++c) mp[c & 7] = fmaxf(mp[c & 7], s[c]);
                mx = fmaxf(fmaxf(fmaxf(mp[0], mp[1]), fmaxf(mp[2], mp[3])),
                           fmaxf(fmaxf(mp[4], mp[5]), fmaxf(mp[6], mp[7])));
            }
            const float m_new = fmaxf(m_ref, mx);
            const bool want = (m_ref == -INFINITY) ? (m_new != -INFINITY) : ((m_new - m_ref) * sl2 > kRescaleLog2);
            if (__any_sync(0xffffffffu, want)) {
                const float alpha = (m_ref == -INFINITY) ? 0.0f : ex2_approx((m_ref - m_new) * sl2);
                l *= alpha;
                l_exact *= alpha;
                m_ref = m_new;
                if (j > 0) {
                    // Small chunks: the score row stays live in registers meanwhile.
#pragma unroll 1
                    for (int c = 0; c < D / 8; ++c) {
                        uint32_t r[8];
                        tmem_ld8(t_o + c * 8, r);
                        tmem_wait_ld();
#pragma unroll
                        for (int x = 0; x < 8; ++x) r[x] = __float_as_uint(__uint_as_float(r[x]) * alpha);
                        tmem_st8(t_o + c * 8, r);
                    }
                }
            }
            const float mb = (m_ref == -INFINITY) ? 0.0f : m_ref * sl2;
            uint32_t pk[kFwdBN / 2];
            float lp[4] = {0.f, 0.f, 0.f, 0.f};  // sums of the bf16-rounded P~ (what the MMA sees)
            float le[4] = {0.f, 0.f, 0.f, 0.f};  // sums of the unrounded P~ (for the LSE)
#pragma unroll
            for (int c = 0; c < kFwdBN / 2; ++c) {
                const float p0 = ex2_approx(fmaf(s[2 * c], sl2, -mb));
                const float p1 = ex2_approx(fmaf(s[2 * c + 1], sl2, -mb));
                pk[c] = pack_bf16x2(p0, p1);
                lp[c & 3] += bf16lo_to_f32(pk[c]) + bf16hi_to_f32(pk[c]);
                le[c & 3] += p0 + p1;
            }
            l += (lp[0] + lp[1]) + (lp[2] + lp[3]);
            l_exact += (le[0] + le[1]) + (le[2] + le[3]);
            tmem_st16(t_s + 0, pk + 0);
            tmem_st16(t_s + 16, pk + 16);
            tmem_st16(t_s + 32, pk + 32);
            tmem_st16(t_s + 48, pk + 48);
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(&bar_p[w]);
        }

        // ---- epilogue: O = O~ / l, LSE = scale * m + ln l
        if (n > 0 && ok) ok = __all_sync(0xffffffffu, mbar_wait(&bar_o[w], 0, abort_flag, p.status));
        if (n > 0 && ok) {
            tc_fence_after();
            const bool valid = row < p.Lq;
            const float inv_l = 1.0f / l;
            const size_t row_idx = static_cast<size_t>(bh) * p.Lq + row;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(t_o + c * 32, r);
                tmem_wait_ld();
                if (valid) {
                    if (p.o_dtype == FA_DT_F32) {
                        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(p.o) + row_idx * D + c * 32);
#pragma unroll
                        for (int x = 0; x < 8; ++x)
                            dst[x] = make_float4(__uint_as_float(r[4 * x]) * inv_l, __uint_as_float(r[4 * x + 1]) * inv_l,
                                                 __uint_as_float(r[4 * x + 2]) * inv_l,
                                                 __uint_as_float(r[4 * x + 3]) * inv_l);
                    } else {
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.o) + row_idx * D + c * 32);
#pragma unroll
                        for (int x = 0; x < 4; ++x) {
                            uint4 u;
                            u.x = pack_bf16x2(__uint_as_float(r[8 * x + 0]) * inv_l, __uint_as_float(r[8 * x + 1]) * inv_l);
                            u.y = pack_bf16x2(__uint_as_float(r[8 * x + 2]) * inv_l, __uint_as_float(r[8 * x + 3]) * inv_l);
                            u.z = pack_bf16x2(__uint_as_float(r[8 * x + 4]) * inv_l, __uint_as_float(r[8 * x + 5]) * inv_l);
                            u.w = pack_bf16x2(__uint_as_float(r[8 * x + 6]) * inv_l, __uint_as_float(r[8 * x + 7]) * inv_l);
                            dst[x] = u;
                        }
                    }
                }
            }
            if (valid) p.lse[row_idx] = m_ref * p.scale + logf(l_exact);
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

int fwd_smem_bytes(int d) { return d == 128 ? FwdLayout<128>::kBytes : FwdLayout<64>::kBytes; }

cudaError_t launch_fwd(const FwdParams& p, int d, cudaStream_t stream) {
    const int BH = p.B * p.H;
    const int n_pairs = (p.Lq + kFwdRowsPerCta - 1) / kFwdRowsPerCta;
    const dim3 grid(static_cast<unsigned>(BH) * static_cast<unsigned>(n_pairs));
    const int smem = fwd_smem_bytes(d);
    if (d == 128) {
        cudaError_t e = cudaFuncSetAttribute(fa_fwd_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        fa_fwd_kernel<128><<<grid, kFwdThreads, smem, stream>>>(p);
    } else {
        cudaError_t e = cudaFuncSetAttribute(fa_fwd_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        fa_fwd_kernel<64><<<grid, kFwdThreads, smem, stream>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace fa
