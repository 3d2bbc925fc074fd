// Paged decode with grouped key/value heads on the tensor cores (d = 64, 128).
//
// The attention is the same as fa_decode's ("What Is FlashAttention?", "What it
// changes for you": the cache of a generation lives in HBM and is read once;
// "The general lesson" names paged attention): per query head, the running max,
// running sum and unnormalised output of "The Three Running Statistics" over
// the keys [0, kv_len), split into 1,024-key chunks merged by fa_decode_combine.
//
// With H / Hkv query heads per key/value head, every K and V row a work item
// loads serves the whole group, and the per-key work is a small matrix product:
// S = Q_g K^T and O_g += P V with Q_g the group's G query rows.  They run as
// mma.sync m16n8k16 (bf16 in, fp32 accumulate) with the group's heads as the M
// rows (padded to 16 with zero rows), so the CUDA cores only do the exponentials:
//   - the S accumulator fragment of two 8-key tiles is exactly the A fragment of
//     P for the 16-key PV product, so P never leaves registers;
//   - K fragments come from shared memory by ldmatrix, V fragments by
//     ldmatrix.trans;
// A work item is (b, KV head, head group of G <= 16 heads, chunk).  Warp 8
// copies each 64-key stage of the item into a 4-stage ring with 2-D TMA loads of
// the page pools (one box per page block of min(page_size, 64) rows and per 64
// columns, looked up through the block table), counted on the stage's mbarrier
// by bytes.  The 128-byte swizzle the TMA applies keeps the eight rows of every
// 8x8 ldmatrix tile in distinct banks.  Compute warps 0-7 form two quads that take alternate
// stages; warp s of a quad handles keys [16s, 16s + 16) of the stage.  Each warp
// keeps its own running statistics per head (rescaling its accumulators only
// when a head's max grows by more than 2^8), and the eight warps merge them at
// the end of the item.  Every wait is bounded.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "fa_internal.h"
#include "ptx.cuh"

namespace fa {
namespace {

constexpr int kMmaStages = 4;
constexpr int kMmaStageKeys = 64;
constexpr int kMmaThreads = 288;  // 8 compute warps + 1 copy warp

#ifdef FA_TEST_HOOKS
// One-shot fault (test build only): the next stage the copy warp would fill gets
// no copies and no arrivals, so the compute warps' wait for it runs out.
__device__ int g_test_skip_stage_mma;
#endif

// A stage of K (or V) is D/64 boxes of [64 rows][128 bytes] as the TMA writes them
// with 128-byte swizzle: the 16-byte piece c of row r sits at piece c ^ (r % 8).
template <int D>
struct MmaLay {
    static constexpr int kBoxBytes = kMmaStageKeys * 128;
    static constexpr int kTileBytes = (D / 64) * kBoxBytes;     // 64 rows of K (or V)
    static constexpr int kKOff = 0;
    static constexpr int kVOff = kKOff + kMmaStages * kTileBytes;
    static constexpr int kRedOff = kVOff + kMmaStages * kTileBytes;  // [8 warps][16 heads][D] fp32
    static constexpr int kRedMOff = kRedOff + 8 * 16 * D * 4;        // [8][16] running max
    static constexpr int kRedLOff = kRedMOff + 8 * 16 * 4;           // [8][16] running sum
    static constexpr int kBarOff = kRedLOff + 8 * 16 * 4;
    // full[S], empty[S], merge[2]
    static constexpr int kMiscOff = kBarOff + (2 * kMmaStages + 2) * 8;
    static constexpr int kBytes = kMiscOff + 16 + 1024;  // + alignment slack
};

// Shared-memory address of row r, 16-byte piece c (8 bf16) of a swizzled stage.
template <int D>
__device__ __forceinline__ uint32_t swz(uint32_t stage, int r, int c) {
    return stage + (c >> 3) * MmaLay<D>::kBoxBytes + r * 128 + (((c & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr));
}
// D += A B for one m16n8k16 tile: A row-major 16x16 bf16 (4 regs), B col-major 16x8 (2 regs).
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D>
__global__ void __launch_bounds__(kMmaThreads, 1) fa_decode_paged_mma(const __grid_constant__ DecodeParams p, int G) {
    using Lay = MmaLay<D>;
    constexpr int S = kMmaStages;
    constexpr int KS = D / 16;  // 16-wide steps along d
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* sK = smem + Lay::kKOff;
    uint8_t* sV = smem + Lay::kVOff;
    float* red = reinterpret_cast<float*>(smem + Lay::kRedOff);
    float* red_m = reinterpret_cast<float*>(smem + Lay::kRedMOff);
    float* red_l = reinterpret_cast<float*>(smem + Lay::kRedLOff);
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
    uint64_t* empty = full + S;
    uint64_t* merge = empty + S;  // [0]: partials written, [1]: partials read
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < S; ++i) {
            mbar_init(&full[i], 1);   // the copy warp's expected-bytes arrival
            mbar_init(&empty[i], 4);  // the four warps of the quad that read the stage
        }
        mbar_init(&merge[0], 256);
        mbar_init(&merge[1], 256);
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    const int group = p.H / p.Hkv;
    const int n_hg = group / G;
    const int per_chunk = p.Hkv * n_hg;
    const int total = p.cum[p.B] * per_chunk;
    const int ps_mask = (1 << p.page_shift) - 1;
    const float sl2 = p.scale_log2;
    // item -> (b, kv head, head group, chunk); head groups of one chunk are adjacent
    auto decode_item = [&](int item, int& b, int& hkv, int& hg, int& chunk) {
        int lo = 0, hi = p.B;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (p.cum[mid] * per_chunk <= item) lo = mid; else hi = mid;
        }
        const int nb = p.cum[lo + 1] - p.cum[lo];
        const int local = item - p.cum[lo] * per_chunk;
        const int rem = local % (nb * n_hg);
        b = lo;
        hkv = local / (nb * n_hg);
        hg = rem % n_hg;
        chunk = rem / n_hg;
    };

    if (warp == 8) {
        // ---------------- copy warp
        int st = 0, skipped = -1;
        bool ok = true;
        for (int item = blockIdx.x; ok && item < total; item += gridDim.x) {
            int b, hkv, hg, chunk;
            decode_item(item, b, hkv, hg, chunk);
            const int start = chunk * kDecodeSplit;
            const int end = min(start + kDecodeSplit, p.lens[b]);
            const int* table = p.block_table + static_cast<size_t>(b) * p.max_blocks;
            for (int k0 = start; k0 < end; k0 += kMmaStageKeys, ++st) {
                const int s = st % S;
                if (st >= S) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&empty[s], ((st / S) - 1) & 1, abort_flag, p.status));
                    if (!ok) break;
                }
                bool skip = false;
#ifdef FA_TEST_HOOKS
                int armed = 0;
                if (lane == 0) armed = atomicExch(&g_test_skip_stage_mma, 0);
                skip = __shfl_sync(0xffffffffu, armed, 0) != 0;
                if (skip) skipped = st;
#endif
                if (skip) continue;
                const int n = min(kMmaStageKeys, end - k0);
                // The stage's valid rows in blocks of BR rows (each block inside one page, as
                // BR divides the page size and 64), each block one 2-D box per 64 columns.
                // Whole boxes arrive even for a short last block; the compute warps zero
                // the V rows past the chunk's end before using them.
                const int BR = p.pool_box_rows;
                const int nblk = (n + BR - 1) / BR;
                if (lane == 0) mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(nblk) * BR * D * 2 * 2);
                __syncwarp();
                for (int blk = lane; blk < nblk; blk += 32) {
                    const int key = k0 + blk * BR;
                    int pg = table[key >> p.page_shift];
                    pg = (static_cast<unsigned>(pg) < static_cast<unsigned>(p.num_pages)) ? pg : 0;  // flagged by the plan
                    const int row = (pg * p.Hkv + hkv) * (ps_mask + 1) + (key & ps_mask);
#pragma unroll
                    for (int bx = 0; bx < D / 64; ++bx) {
                        const int dst = s * Lay::kTileBytes + bx * Lay::kBoxBytes + blk * BR * 128;
                        tma_load_2d(sK + dst, &p.tm_kpool, &full[s], bx * 64, row);
                        tma_load_2d(sV + dst, &p.tm_vpool, &full[s], bx * 64, row);
                    }
                }
            }
        }
        // every copy issued here lands before the CTA's shared memory goes away (each
        // barrier waited on is at the phase of its last copies)
        for (int t = max(0, st - S); t < st; ++t)
            if (t != skipped) mbar_wait_drain(&full[t % S], (t / S) & 1, p.status);
    } else {
        // ---------------- compute warps: quad q takes stages st with st % 2 == q; warp sub of
        // the quad takes keys [16 sub, 16 sub + 16) of the stage
        const int quad = warp >> 2, sub = warp & 3;
        const int g = lane >> 2, t = lane & 3;  // fragment row (head) and column pair
        const uint32_t sKa = smem_u32(sK), sVa = smem_u32(sV);
        int st = 0;  // stages of the CTA so far (both quads count them all)
        bool ok = true;
        int mphase = 0;
        for (int item = blockIdx.x; ok && item < total; item += gridDim.x) {
            int b, hkv, hg, chunk;
            decode_item(item, b, hkv, hg, chunk);
            const int h0 = hkv * group + hg * G;
            const int start = chunk * kDecodeSplit;
            const int end = min(start + kDecodeSplit, p.lens[b]);
            // Q_g as the A operand, rows = heads (rows >= G and 8..15 are zero)
            uint32_t qa[KS][4];
            {
                const __nv_bfloat16* qrow = static_cast<const __nv_bfloat16*>(p.q) +
                                            (static_cast<size_t>(b) * p.H + h0 + g) * D;
#pragma unroll
                for (int kk = 0; kk < KS; ++kk) {
                    qa[kk][0] = g < G ? *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 2 * t) : 0u;
                    qa[kk][2] = g < G ? *reinterpret_cast<const uint32_t*>(qrow + kk * 16 + 8 + 2 * t) : 0u;
                    qa[kk][1] = 0u;
                    qa[kk][3] = 0u;
                }
            }
            float o[D / 8][4];
#pragma unroll
            for (int j = 0; j < D / 8; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.0f;
            float m = -INFINITY, l = 0.0f;  // this thread's head g; l is its lanes' partial sum
            const int n_st = (end - start + kMmaStageKeys - 1) / kMmaStageKeys;
            for (int i = 0; i < n_st; ++i, ++st) {
                if ((st & 1) != quad) continue;
                const int s = st % S;
                ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (st / S) & 1, abort_flag, p.status));
                if (!ok) break;
                const int kbase = start + i * kMmaStageKeys + sub * 16;  // first key of this warp
                const uint32_t kst = sKa + s * Lay::kTileBytes, vst = sVa + s * Lay::kTileBytes;
                if (kbase + 16 > end) {
                    // V rows past the chunk's end may hold anything (even NaN, which a zero
                    // probability would not cancel): this warp's such rows become zero
                    for (int e = lane; e < 16 * (D / 8); e += 32) {
                        const int r = e / (D / 8);
                        if (kbase + r >= end)
                            *reinterpret_cast<uint4*>(sV + (swz<D>(vst, sub * 16 + r, e % (D / 8)) - sVa)) =
                                make_uint4(0, 0, 0, 0);
                    }
                    __syncwarp();
                    fence_proxy_async_smem();  // before the stage's next TMA write
                }
                // S for keys kbase + [0, 8) and kbase + [8, 16)
                float sc[2][4];
#pragma unroll
                for (int n = 0; n < 2; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.0f;
#pragma unroll
                for (int kk = 0; kk < KS; kk += 2) {
#pragma unroll
                    for (int n = 0; n < 2; ++n) {
                        uint32_t bf[4];  // b0, b1 of step kk and of step kk + 1
                        ldsm_x4(swz<D>(kst, sub * 16 + n * 8 + (lane & 7), kk * 2 + (lane >> 3)), bf);
                        mma16816(sc[n], qa[kk], bf[0], bf[1]);
                        mma16816(sc[n], qa[kk + 1], bf[2], bf[3]);
                    }
                }
                // V fragments for all d tiles of this warp's 16 keys: read before releasing the stage
                // (the PV product below uses them after the softmax)
                // Mask keys at or past the chunk end; scores of padded rows are unused.
                float x[4] = {sc[0][0], sc[0][1], sc[1][0], sc[1][1]};  // keys 2t, 2t+1, 8+2t, 9+2t
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int key = kbase + (e >> 1) * 8 + 2 * t + (e & 1);
                    if (key >= end) x[e] = -INFINITY;
                }
                float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
                const float m_new = fmaxf(m, mx);
                const bool grow = (m == -INFINITY) ? (m_new != -INFINITY) : ((m_new - m) * sl2 > 8.0f);
                if (__any_sync(0xffffffffu, grow)) {
                    const float alpha = (m == -INFINITY) ? 0.0f : ex2_approx((m - m_new) * sl2);
                    l *= alpha;
#pragma unroll
                    for (int j = 0; j < D / 8; ++j) {
                        o[j][0] *= alpha;
                        o[j][1] *= alpha;
                    }
                    m = m_new;
                }
                const float mb = (m == -INFINITY) ? 0.0f : m * sl2;
                float pv[4];
#pragma unroll
                for (int e = 0; e < 4; ++e) pv[e] = ex2_approx(fmaf(x[e], sl2, -mb));  // masked: +0
                l += (pv[0] + pv[1]) + (pv[2] + pv[3]);
                uint32_t pa[4];
                pa[0] = pack_bf16x2(pv[0], pv[1]);  // row g, keys 2t, 2t+1
                pa[1] = 0u;                          // rows 8..15
                pa[2] = pack_bf16x2(pv[2], pv[3]);  // row g, keys 8+2t, 9+2t
                pa[3] = 0u;
                // O += P V: V tile of 16 keys as the B operand, two d tiles per ldmatrix
#pragma unroll
                for (int j = 0; j < D / 8; j += 2) {
                    uint32_t bf[4];  // b0, b1 of d tile j and of d tile j + 1
                    ldsm_x4_t(swz<D>(vst, sub * 16 + (lane & 7) + ((lane >> 3) & 1) * 8, j + (lane >> 4)), bf);
                    mma16816(o[j], pa, bf[0], bf[1]);
                    mma16816(o[j + 1], pa, bf[2], bf[3]);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
            }
            if (!ok) break;
            // ---- merge the eight warps' partials of each head
            l += __shfl_xor_sync(0xffffffffu, l, 1);
            l += __shfl_xor_sync(0xffffffffu, l, 2);
            if (g < G) {
                if (t == 0) {
                    red_m[warp * 16 + g] = m;
                    red_l[warp * 16 + g] = l;
                }
#pragma unroll
                for (int j = 0; j < D / 8; ++j) {
                    red[(warp * 16 + g) * D + j * 8 + 2 * t] = o[j][0];
                    red[(warp * 16 + g) * D + j * 8 + 2 * t + 1] = o[j][1];
                }
            }
            mbar_arrive(&merge[0]);
            ok = __all_sync(0xffffffffu, mbar_wait(&merge[0], mphase & 1, abort_flag, p.status));
            if (!ok) break;
            for (int e = threadIdx.x; e < G * D; e += 256) {
                const int hh = e / D, c = e % D;
                float M = -INFINITY;
                for (int w = 0; w < 8; ++w) M = fmaxf(M, red_m[w * 16 + hh]);
                float L = 0.0f, O = 0.0f;
                for (int w = 0; w < 8; ++w) {
                    const float mw = red_m[w * 16 + hh];
                    if (mw == -INFINITY) continue;
                    const float wt = ex2_approx((mw - M) * sl2);
                    L = fmaf(wt, red_l[w * 16 + hh], L);
                    O = fmaf(wt, red[(w * 16 + hh) * D + c], O);
                }
                const size_t slot = (static_cast<size_t>(b) * p.H + h0 + hh) * p.max_splits + chunk;
                p.part_o[slot * D + c] = O / L;
                if (c == 0) p.part_lse[slot] = M * p.scale + logf(L);
            }
            mbar_arrive(&merge[1]);  // the partials may be overwritten by the next item
            ok = __all_sync(0xffffffffu, mbar_wait(&merge[1], mphase & 1, abort_flag, p.status));
            ++mphase;
        }
    }
}

}  // namespace

// Largest head group <= 16 that divides H / Hkv.
int paged_mma_group(int group) {
    for (int g = 16; g > 1; g >>= 1)
        if (group % g == 0) return g;
    return 1;
}

cudaError_t launch_paged_mma_split(const DecodeParams& p, int d, int num_sms, cudaStream_t stream) {
    const int G = paged_mma_group(p.H / p.Hkv);
    const long long upper = static_cast<long long>(p.B) * p.Hkv * ((p.H / p.Hkv) / G) * p.max_splits;
    const int grid = static_cast<int>(std::min<long long>(upper, num_sms));
    if (grid == 0) return cudaSuccess;
    cudaError_t e;
    if (d == 128) {
        if ((e = cudaFuncSetAttribute(fa_decode_paged_mma<128>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      MmaLay<128>::kBytes)) != cudaSuccess)
            return e;
        fa_decode_paged_mma<128><<<grid, kMmaThreads, MmaLay<128>::kBytes, stream>>>(p, G);
    } else {
        if ((e = cudaFuncSetAttribute(fa_decode_paged_mma<64>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      MmaLay<64>::kBytes)) != cudaSuccess)
            return e;
        fa_decode_paged_mma<64><<<grid, kMmaThreads, MmaLay<64>::kBytes, stream>>>(p, G);
    }
    return cudaGetLastError();
}

#ifdef FA_TEST_HOOKS
cudaError_t paged_mma_test_arm_skip_stage() {
    const int one = 1;
    return cudaMemcpyToSymbol(g_test_skip_stage_mma, &one, sizeof(int));
}
#endif

}  // namespace fa
