// Single-query decode over a KV cache, split over the key axis.
//
// The decode phase reads the whole cache once per generated token and does
// about one FLOP per byte, so it is bound by HBM bandwidth ("What Is
// FlashAttention?", "What it changes for you": the cache lives in HBM).  The
// keys of each sequence are cut into fixed chunks of kDecodeSplit keys; every
// chunk of every (b, h) is an independent work item that streams its K and V
// rows with coalesced 128-bit loads, runs the running-max / running-sum
// recurrence of "The Three Running Statistics" over them, and writes a
// normalised partial output with its log-sum-exp.  A combine kernel merges the
// partials of each (b, h) with the same recurrence applied to whole chunks.
//
// Kernels:
//   fa_decode_plan     one CTA: clamps kv_lens to [0, cap] (flagging bad ones) and
//                      prefix-sums the chunk counts per sequence.
//   fa_decode_split    persistent CTAs over all (b, h, chunk) items.
//   fa_decode_combine  one CTA per (b, h): log-sum-exp merge of its chunks.
//
// Paged cache with grouped heads (fa_decode_paged): the same split and combine,
// with keys reached through a per-sequence block table of fixed-size pages and
// H / Hkv query heads sharing each key/value head ("What Is FlashAttention?",
// "The general lesson" names paged attention among the ways of moving less
// data).  A work item covers a group of query heads of one KV head, so every K
// and V row it loads serves the whole group.
//   fa_decode_paged_tma    persistent CTAs over (b, kv head, head group, chunk); a
//                          copy warp stages each 64-key slice of K and V into
//                          shared memory with bulk copies, 8 warps compute.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>

#include "fa_internal.h"
#include "ptx.cuh"

namespace fa {
namespace {

constexpr int kPlanThreads = 1024;

#ifdef FA_TEST_HOOKS
// One-shot fault (test build only): the next stage a paged-decode copy warp of
// the d = 256 kernel would fill gets neither its expected byte count nor its
// copies, so the compute warps' wait for it runs out.
__device__ int g_test_skip_stage;
#endif

__device__ __forceinline__ uint4 ld_stream_u4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ float ex2f_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Eight bf16 values packed in a uint4 -> float.
__device__ __forceinline__ void unpack8(const uint4& u, float (&f)[8]) {
    f[0] = __uint_as_float(u.x << 16);
    f[1] = __uint_as_float(u.x & 0xFFFF0000u);
    f[2] = __uint_as_float(u.y << 16);
    f[3] = __uint_as_float(u.y & 0xFFFF0000u);
    f[4] = __uint_as_float(u.z << 16);
    f[5] = __uint_as_float(u.z & 0xFFFF0000u);
    f[6] = __uint_as_float(u.w << 16);
    f[7] = __uint_as_float(u.w & 0xFFFF0000u);
}

__global__ void __launch_bounds__(kPlanThreads) fa_decode_plan(DecodeParams p) {
    __shared__ int part[kPlanThreads];
    const int t = threadIdx.x;
    const int per = (p.B + kPlanThreads - 1) / kPlanThreads;
    const int b0 = min(p.B, t * per), b1 = min(p.B, b0 + per);
    int local = 0;
    for (int b = b0; b < b1; ++b) {
        int n = p.kv_lens[b];
        if (n < 0 || n > p.cap) {
            atomicCAS(p.status, 0, FA_ERR_KV_LEN);
            n = n < 0 ? 0 : p.cap;
        }
        p.lens[b] = n;
        local += (n + kDecodeSplit - 1) / kDecodeSplit;
        if (p.block_table) {
            // every page a valid key will read must exist; the split kernel clamps bad ones
            const int nblk = (n + (1 << p.page_shift) - 1) >> p.page_shift;
            for (int blk = 0; blk < nblk; ++blk) {
                const int pg = p.block_table[static_cast<size_t>(b) * p.max_blocks + blk];
                if (pg < 0 || pg >= p.num_pages) atomicCAS(p.status, 0, FA_ERR_PAGE);
            }
        }
    }
    part[t] = local;
    __syncthreads();
    // inclusive scan over the per-thread counts (Hillis-Steele)
    for (int s = 1; s < kPlanThreads; s <<= 1) {
        const int add = (t >= s) ? part[t - s] : 0;
        __syncthreads();
        part[t] += add;
        __syncthreads();
    }
    int run = part[t] - local;  // exclusive prefix
    for (int b = b0; b < b1; ++b) {
        p.cum[b] = run;
        run += (p.lens[b] + kDecodeSplit - 1) / kDecodeSplit;
    }
    if (t == kPlanThreads - 1) p.cum[p.B] = part[t];
}

// D/8 lanes hold one key row (8 bf16 each); a warp covers 256/D keys per load.
template <int D>
__global__ void __launch_bounds__(kDecodeThreads, 3) fa_decode_split(DecodeParams p) {
    constexpr int kLanesPerKey = D / 8;
    constexpr int kGroupsPerWarp = 32 / kLanesPerKey;
    constexpr int kGroups = (kDecodeThreads / 32) * kGroupsPerWarp;  // key groups per CTA
    constexpr int kUnroll = 4;
    constexpr int kStep = kGroups * kUnroll;

    __shared__ float red_m[kGroups];
    __shared__ float red_l[kGroups];
    __shared__ float red_acc[kGroups][D];
    __shared__ int s_item[3];

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = warp * kGroupsPerWarp + lane / kLanesPerKey;  // key group of this thread
    const int e0 = (lane % kLanesPerKey) * 8;                  // first element of its slice
    const float sl2 = p.scale_log2;
    const int total = p.cum[p.B] * p.H;

    for (int item = blockIdx.x; item < total; item += gridDim.x) {
        if (threadIdx.x == 0) {
            // item -> (b, h, chunk): items are ordered by b, then h, then chunk
            int lo = 0, hi = p.B;  // find b with H*cum[b] <= item < H*cum[b+1]
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (p.cum[mid] * p.H <= item) lo = mid; else hi = mid;
            }
            const int nb = p.cum[lo + 1] - p.cum[lo];
            const int local = item - p.cum[lo] * p.H;
            s_item[0] = lo;
            s_item[1] = local / nb;
            s_item[2] = local % nb;
        }
        __syncthreads();
        const int b = s_item[0], h = s_item[1], chunk = s_item[2];
        const int len = p.lens[b];
        const int start = chunk * kDecodeSplit;
        const int end = min(start + kDecodeSplit, len);
        const size_t bh = static_cast<size_t>(b) * p.H + h;
        const __nv_bfloat16* kbase = static_cast<const __nv_bfloat16*>(p.k) + bh * p.cap * D + e0;
        const __nv_bfloat16* vbase = static_cast<const __nv_bfloat16*>(p.v) + bh * p.cap * D + e0;

        float qf[8];
        unpack8(*reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.q) + bh * D + e0), qf);

        float m = -INFINITY, l = 0.0f;
        float acc[8];
#pragma unroll
        for (int x = 0; x < 8; ++x) acc[x] = 0.0f;

        for (int base = start; base < end; base += kStep) {
            uint4 kr[kUnroll], vr[kUnroll];
            bool valid[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const int key = base + u * kGroups + g;
                valid[u] = key < end;
                kr[u] = valid[u] ? ld_stream_u4(kbase + static_cast<size_t>(key) * D) : make_uint4(0, 0, 0, 0);
                vr[u] = valid[u] ? ld_stream_u4(vbase + static_cast<size_t>(key) * D) : make_uint4(0, 0, 0, 0);
            }
            float s[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                float kf[8];
                unpack8(kr[u], kf);
                float dot = 0.0f;
#pragma unroll
                for (int x = 0; x < 8; ++x) dot = fmaf(qf[x], kf[x], dot);
#pragma unroll
                for (int o = kLanesPerKey / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
                s[u] = valid[u] ? dot : -INFINITY;
            }
            float mb = s[0];
#pragma unroll
            for (int u = 1; u < kUnroll; ++u) mb = fmaxf(mb, s[u]);
            const float m_new = fmaxf(m, mb);
            // m_new is -inf only while this group has seen no valid key: then
            // alpha = 0 and every p = 0, leaving l = 0 and acc = 0.
            const float m_use = (m_new == -INFINITY) ? 0.0f : m_new;
            const float alpha = (m == -INFINITY) ? 0.0f : ex2f_approx((m - m_use) * sl2);
            const float mbias = m_use * sl2;
            l *= alpha;
#pragma unroll
            for (int x = 0; x < 8; ++x) acc[x] *= alpha;
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                const float pu = ex2f_approx(fmaf(s[u], sl2, -mbias));  // 0 for invalid keys
                l += pu;
                float vf[8];
                unpack8(vr[u], vf);
#pragma unroll
                for (int x = 0; x < 8; ++x) acc[x] = fmaf(pu, vf[x], acc[x]);
            }
            m = m_new;
        }

        // merge the key groups of this CTA (same recurrence over whole groups)
        if (lane % kLanesPerKey == 0) {
            red_m[g] = m;
            red_l[g] = l;
        }
#pragma unroll
        for (int x = 0; x < 8; ++x) red_acc[g][e0 + x] = acc[x];
        __syncthreads();
        if (threadIdx.x < D) {
            const int c = threadIdx.x;
            float M = -INFINITY;
            for (int i = 0; i < kGroups; ++i) M = fmaxf(M, red_m[i]);
            float L = 0.0f, O = 0.0f;
            for (int i = 0; i < kGroups; ++i) {
                if (red_m[i] == -INFINITY) continue;
                const float w = ex2f_approx((red_m[i] - M) * sl2);
                L = fmaf(w, red_l[i], L);
                O = fmaf(w, red_acc[i][c], O);
            }
            const size_t slot = bh * p.max_splits + chunk;
            p.part_o[slot * D + c] = O / L;
            if (c == 0) p.part_lse[slot] = M * p.scale + logf(L);
        }
        __syncthreads();
    }
}

// Paged decode with grouped heads, K/V staged through shared memory.  A work
// item is (b, KV head, group of GG query heads, chunk): every K and V row it
// reads serves the whole group.  Warp 8 copies each 64-key stage of the item
// (page segments of K and V, valid rows only) with 1-D bulk copies into a ring
// of kPgStages<D> stages.  In warps 0-7, D/8 lanes hold one key row slice (8 bf16)
// and keep, per head, a running max, a running sum and an 8-wide accumulator:
// dot products and accumulation use packed FFMA2, and the accumulators are
// rescaled only when a head's max grows by more than 2^8 (O = acc / l holds for
// any common reference).  Bytes in flight are bounded by the ring (128 KB at
// d = 128), not by registers.  Every wait is bounded; an abort drains the
// copies in flight.
// ring depth: 4 stages of 64 keys (128 KB of K and V at d = 128); 2 at d = 256
template <int D>
constexpr int kPgStages = (D == 256) ? 2 : 4;
constexpr int kPgStageKeys = 64;
constexpr int kPgThreads = 288;  // 8 compute warps + 1 copy warp

template <int D, int GG>
struct PagedTmaLayout {
    static constexpr int kLanesPerKey = D / 8;
    static constexpr int kGroups = 8 * (32 / kLanesPerKey);
    static constexpr int kStageBytes = kPgStageKeys * D * 2;  // one of K or V
    static constexpr int kKOff = 0;
    static constexpr int kVOff = kKOff + kPgStages<D> * kStageBytes;
    static constexpr int kRedMOff = kVOff + kPgStages<D> * kStageBytes;
    static constexpr int kRedLOff = kRedMOff + GG * kGroups * 4;
    static constexpr int kRedAccOff = kRedLOff + GG * kGroups * 4;
    static constexpr int kBarOff = (kRedAccOff + GG * kGroups * D * 4 + 7) / 8 * 8;
    static constexpr int kMiscOff = kBarOff + 2 * kPgStages<D> * 8;
    static constexpr int kBytes = kMiscOff + 16 + 128;
};

__device__ __forceinline__ void named_bar_sync(int id, int threads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

template <int D, int GG>
__global__ void __launch_bounds__(kPgThreads, 1) fa_decode_paged_tma(DecodeParams p) {
    using Lay = PagedTmaLayout<D, GG>;
    constexpr int kLanesPerKey = Lay::kLanesPerKey;
    constexpr int kGroupsPerWarp = 32 / kLanesPerKey;
    constexpr int kGroups = Lay::kGroups;
    constexpr int kKeysPerGroup = kPgStageKeys / kGroups;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
    __nv_bfloat16* sk = reinterpret_cast<__nv_bfloat16*>(smem + Lay::kKOff);
    __nv_bfloat16* sv = reinterpret_cast<__nv_bfloat16*>(smem + Lay::kVOff);
    float* red_m = reinterpret_cast<float*>(smem + Lay::kRedMOff);    // [GG][kGroups]
    float* red_l = reinterpret_cast<float*>(smem + Lay::kRedLOff);    // [GG][kGroups]
    float* red_acc = reinterpret_cast<float*>(smem + Lay::kRedAccOff);  // [GG][kGroups][D]
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + Lay::kBarOff);
    uint64_t* empty = full + kPgStages<D>;
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + Lay::kMiscOff);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kPgStages<D>; ++i) {
            mbar_init(&full[i], 1);
            mbar_init(&empty[i], 8);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();

    const int group = p.H / p.Hkv;
    const int n_hg = group / GG;
    const int per_chunk = p.Hkv * n_hg;
    const int total = p.cum[p.B] * per_chunk;
    const int ps_mask = (1 << p.page_shift) - 1;
    const float sl2 = p.scale_log2;
    // item -> (b, kv head, head group, chunk); every warp decodes it the same way
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
        int st = 0;  // stages issued
        int skipped = -1;  // test build: a stage whose copies were never issued
        bool ok = true;
        for (int item = blockIdx.x; ok && item < total; item += gridDim.x) {
            int b, hkv, hg, chunk;
            decode_item(item, b, hkv, hg, chunk);
            const int start = chunk * kDecodeSplit;
            const int end = min(start + kDecodeSplit, p.lens[b]);
            const int* table = p.block_table + static_cast<size_t>(b) * p.max_blocks;
            for (int k0 = start; k0 < end; k0 += kPgStageKeys, ++st) {
                const int s = st % kPgStages<D>;
                if (st >= kPgStages<D>) {
                    ok = __all_sync(0xffffffffu, mbar_wait(&empty[s], ((st / kPgStages<D>) - 1) & 1, abort_flag, p.status));
                    if (!ok) break;
                }
                const int n = min(kPgStageKeys, end - k0);
                bool skip = false;
#ifdef FA_TEST_HOOKS
                int armed = 0;
                if (lane == 0) armed = atomicExch(&g_test_skip_stage, 0);
                skip = __shfl_sync(0xffffffffu, armed, 0) != 0;
                if (skip) skipped = st;
#endif
                if (lane == 0 && !skip) {
                    mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(n) * D * 2 * 2);
                    for (int key = k0; key < k0 + n;) {
                        int pg = table[key >> p.page_shift];
                        pg = (static_cast<unsigned>(pg) < static_cast<unsigned>(p.num_pages)) ? pg : 0;  // flagged by the plan
                        const int r0 = key & ps_mask;
                        const int seg = min(ps_mask + 1 - r0, k0 + n - key);
                        const size_t row = (static_cast<size_t>(pg) * p.Hkv + hkv) * (ps_mask + 1) + r0;
                        bulk_load(sk + (static_cast<size_t>(s) * kPgStageKeys + (key - k0)) * D,
                                  static_cast<const __nv_bfloat16*>(p.k) + row * D, static_cast<uint32_t>(seg) * D * 2,
                                  &full[s]);
                        bulk_load(sv + (static_cast<size_t>(s) * kPgStageKeys + (key - k0)) * D,
                                  static_cast<const __nv_bfloat16*>(p.v) + row * D, static_cast<uint32_t>(seg) * D * 2,
                                  &full[s]);
                        key += seg;
                    }
                }
                __syncwarp();
            }
        }
        // every copy issued here lands before the CTA's shared memory goes away
        // (each barrier is at the phase of its last copy)
        for (int t = max(0, st - kPgStages<D>); t < st; ++t)
            if (t != skipped) mbar_wait_drain(&full[t % kPgStages<D>], (t / kPgStages<D>) & 1, p.status);
    } else {
        // ---------------- compute warps 0-7
        const int g = warp * kGroupsPerWarp + lane / kLanesPerKey;
        const int e0 = (lane % kLanesPerKey) * 8;
        int st = 0;  // stages consumed
        bool ok = true;
        for (int item = blockIdx.x; ok && item < total; item += gridDim.x) {
            int b, hkv, hg, chunk;
            decode_item(item, b, hkv, hg, chunk);
            const int h0 = hkv * group + hg * GG;
            const int start = chunk * kDecodeSplit;
            const int end = min(start + kDecodeSplit, p.lens[b]);
            float2 q2[GG][4];
#pragma unroll
            for (int gg = 0; gg < GG; ++gg) {
                float qf[8];
                unpack8(*reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.q) +
                                                        (static_cast<size_t>(b) * p.H + h0 + gg) * D + e0),
                        qf);
#pragma unroll
                for (int i = 0; i < 4; ++i) q2[gg][i] = make_float2(qf[2 * i], qf[2 * i + 1]);
            }
            float m[GG], l[GG];
            float2 acc2[GG][4];
#pragma unroll
            for (int gg = 0; gg < GG; ++gg) {
                m[gg] = -INFINITY;
                l[gg] = 0.0f;
#pragma unroll
                for (int i = 0; i < 4; ++i) acc2[gg][i] = make_float2(0.0f, 0.0f);
            }
            for (int k0 = start; k0 < end; k0 += kPgStageKeys, ++st) {
                const int s = st % kPgStages<D>;
                ok = __all_sync(0xffffffffu, mbar_wait(&full[s], (st / kPgStages<D>) & 1, abort_flag, p.status));
                if (!ok) break;
                const int n = min(kPgStageKeys, end - k0);
                float sc[kKeysPerGroup][GG];
                uint4 vr[kKeysPerGroup];
#pragma unroll
                for (int u = 0; u < kKeysPerGroup; ++u) {
                    const int kl = u * kGroups + g;
                    const bool valid = kl < n;
                    const size_t off = (static_cast<size_t>(s) * kPgStageKeys + kl) * D + e0;
                    const uint4 kr = valid ? *reinterpret_cast<const uint4*>(sk + off) : make_uint4(0, 0, 0, 0);
                    vr[u] = valid ? *reinterpret_cast<const uint4*>(sv + off) : make_uint4(0, 0, 0, 0);
                    const float2 k2[4] = {make_float2(__uint_as_float(kr.x << 16), __uint_as_float(kr.x & 0xFFFF0000u)),
                                          make_float2(__uint_as_float(kr.y << 16), __uint_as_float(kr.y & 0xFFFF0000u)),
                                          make_float2(__uint_as_float(kr.z << 16), __uint_as_float(kr.z & 0xFFFF0000u)),
                                          make_float2(__uint_as_float(kr.w << 16), __uint_as_float(kr.w & 0xFFFF0000u))};
#pragma unroll
                    for (int gg = 0; gg < GG; ++gg) {
                        float2 d2 = __fmul2_rn(q2[gg][0], k2[0]);
#pragma unroll
                        for (int i = 1; i < 4; ++i) d2 = __ffma2_rn(q2[gg][i], k2[i], d2);
                        float dot = d2.x + d2.y;
#pragma unroll
                        for (int o = kLanesPerKey / 2; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
                        sc[u][gg] = valid ? dot : -INFINITY;
                    }
                }
                // the stage's rows are in registers: hand it back to the copy warp
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[s]);
                bool grow = false;
                float mb[GG];
#pragma unroll
                for (int gg = 0; gg < GG; ++gg) {
                    mb[gg] = sc[0][gg];
#pragma unroll
                    for (int u = 1; u < kKeysPerGroup; ++u) mb[gg] = fmaxf(mb[gg], sc[u][gg]);
                    grow |= (m[gg] == -INFINITY) ? (mb[gg] != -INFINITY) : ((mb[gg] - m[gg]) * sl2 > 8.0f);
                }
                if (__any_sync(0xffffffffu, grow)) {
#pragma unroll
                    for (int gg = 0; gg < GG; ++gg) {
                        const float m_new = fmaxf(m[gg], mb[gg]);
                        const float alpha = (m[gg] == -INFINITY) ? 0.0f : ex2f_approx((m[gg] - m_new) * sl2);
                        l[gg] *= alpha;
                        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
                        for (int i = 0; i < 4; ++i) acc2[gg][i] = __fmul2_rn(acc2[gg][i], a2);
                        m[gg] = m_new;
                    }
                }
#pragma unroll
                for (int u = 0; u < kKeysPerGroup; ++u) {
                    const float2 v2[4] = {make_float2(__uint_as_float(vr[u].x << 16), __uint_as_float(vr[u].x & 0xFFFF0000u)),
                                          make_float2(__uint_as_float(vr[u].y << 16), __uint_as_float(vr[u].y & 0xFFFF0000u)),
                                          make_float2(__uint_as_float(vr[u].z << 16), __uint_as_float(vr[u].z & 0xFFFF0000u)),
                                          make_float2(__uint_as_float(vr[u].w << 16), __uint_as_float(vr[u].w & 0xFFFF0000u))};
#pragma unroll
                    for (int gg = 0; gg < GG; ++gg) {
                        const float mbias = (m[gg] == -INFINITY) ? 0.0f : m[gg] * sl2;
                        const float pu = ex2f_approx(fmaf(sc[u][gg], sl2, -mbias));
                        l[gg] += pu;
                        const float2 p2 = make_float2(pu, pu);
#pragma unroll
                        for (int i = 0; i < 4; ++i) acc2[gg][i] = __ffma2_rn(p2, v2[i], acc2[gg][i]);
                    }
                }
            }
            if (!ok) break;
            // merge the key groups of the 8 compute warps, per head
#pragma unroll
            for (int gg = 0; gg < GG; ++gg) {
                if (lane % kLanesPerKey == 0) {
                    red_m[gg * kGroups + g] = m[gg];
                    red_l[gg * kGroups + g] = l[gg];
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    red_acc[(gg * kGroups + g) * D + e0 + 2 * i] = acc2[gg][i].x;
                    red_acc[(gg * kGroups + g) * D + e0 + 2 * i + 1] = acc2[gg][i].y;
                }
            }
            named_bar_sync(1, 256);
            for (int t = threadIdx.x; t < GG * D; t += 256) {
                const int gg = t / D, c = t % D;
                float M = -INFINITY;
                for (int i = 0; i < kGroups; ++i) M = fmaxf(M, red_m[gg * kGroups + i]);
                float L = 0.0f, O = 0.0f;
                for (int i = 0; i < kGroups; ++i) {
                    const float mi = red_m[gg * kGroups + i];
                    if (mi == -INFINITY) continue;
                    const float w = ex2f_approx((mi - M) * sl2);
                    L = fmaf(w, red_l[gg * kGroups + i], L);
                    O = fmaf(w, red_acc[(gg * kGroups + i) * D + c], O);
                }
                const size_t slot = (static_cast<size_t>(b) * p.H + h0 + gg) * p.max_splits + chunk;
                p.part_o[slot * D + c] = O / L;
                if (c == 0) p.part_lse[slot] = M * p.scale + logf(L);
            }
            named_bar_sync(1, 256);
        }
    }
}

template <int D>
__global__ void __launch_bounds__(D) fa_decode_combine(DecodeParams p) {
    const int bh = blockIdx.x;
    const int b = bh / p.H;
    const int c = threadIdx.x;
    const int n = (p.lens[b] + kDecodeSplit - 1) / kDecodeSplit;
    const size_t out = static_cast<size_t>(bh) * D + c;
    if (n == 0) {
        if (p.o_dtype == FA_DT_F32) static_cast<float*>(p.o)[out] = 0.0f;
        else static_cast<__nv_bfloat16*>(p.o)[out] = __float2bfloat16_rn(0.0f);
        if (c == 0) p.lse[bh] = -INFINITY;
        return;
    }
    const float* lse_s = p.part_lse + static_cast<size_t>(bh) * p.max_splits;
    const float* o_s = p.part_o + static_cast<size_t>(bh) * p.max_splits * D;
    float M = -INFINITY;
    for (int s = 0; s < n; ++s) M = fmaxf(M, lse_s[s]);
    float L = 0.0f, O = 0.0f;
    for (int s = 0; s < n; ++s) {
        const float w = __expf(lse_s[s] - M);
        L += w;
        O = fmaf(w, o_s[static_cast<size_t>(s) * D + c], O);
    }
    O /= L;
    if (p.o_dtype == FA_DT_F32) static_cast<float*>(p.o)[out] = O;
    else static_cast<__nv_bfloat16*>(p.o)[out] = __float2bfloat16_rn(O);
    if (c == 0) p.lse[bh] = M + logf(L);
}

template <int D, int GG>
cudaError_t launch_paged_tma(const DecodeParams& p, int num_sms, cudaStream_t stream) {
    const int n_hg = (p.H / p.Hkv) / GG;
    const long long upper = static_cast<long long>(p.B) * p.Hkv * n_hg * p.max_splits;
    const int grid = static_cast<int>(std::min<long long>(upper, num_sms));
    const int smem = PagedTmaLayout<D, GG>::kBytes;
    cudaError_t e = cudaFuncSetAttribute(fa_decode_paged_tma<D, GG>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    fa_decode_paged_tma<D, GG><<<grid, kPgThreads, smem, stream>>>(p);
    return cudaGetLastError();
}

// d = 64, 128 with pages of at least 8 rows: the tensor-core split kernel
// (decode_paged_mma.cu); otherwise the CUDA-core split kernel above.
template <int D>
cudaError_t launch_paged_d(const DecodeParams& p, int num_sms, cudaStream_t stream) {
    const int group = p.H / p.Hkv;
    cudaError_t e;
    if (D != 256 && p.pool_box_rows > 0) e = launch_paged_mma_split(p, D, num_sms, stream);
    else if (group % 4 == 0) e = launch_paged_tma<D, 4>(p, num_sms, stream);
    else if (group % 2 == 0) e = launch_paged_tma<D, 2>(p, num_sms, stream);
    else e = launch_paged_tma<D, 1>(p, num_sms, stream);
    if (e != cudaSuccess) return e;
    fa_decode_combine<D><<<p.B * p.H, D, 0, stream>>>(p);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_decode_paged(const DecodeParams& p, int d, int num_sms, cudaStream_t stream) {
    fa_decode_plan<<<1, kPlanThreads, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    if (d == 256) return launch_paged_d<256>(p, num_sms, stream);
    return d == 128 ? launch_paged_d<128>(p, num_sms, stream) : launch_paged_d<64>(p, num_sms, stream);
}

#ifdef FA_TEST_HOOKS
cudaError_t paged_test_arm_skip_stage() {
    const int one = 1;
    return cudaMemcpyToSymbol(g_test_skip_stage, &one, sizeof(int));
}
#endif

size_t decode_workspace_bytes(int B, int H, int cap, int d) {
    const size_t max_splits = (static_cast<size_t>(cap) + kDecodeSplit - 1) / kDecodeSplit;
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t bh = static_cast<size_t>(B) * H;
    return up(bh * max_splits * d * sizeof(float)) + up(bh * max_splits * sizeof(float)) +
           up(static_cast<size_t>(B) * sizeof(int)) + up((static_cast<size_t>(B) + 1) * sizeof(int));
}

void decode_carve_workspace(DecodeParams& p, void* ws, int B, int H, int cap, int d) {
    const size_t max_splits = (static_cast<size_t>(cap) + kDecodeSplit - 1) / kDecodeSplit;
    auto up = [](size_t x) { return (x + 255) & ~size_t(255); };
    const size_t bh = static_cast<size_t>(B) * H;
    uint8_t* w = static_cast<uint8_t*>(ws);
    p.part_o = reinterpret_cast<float*>(w);
    w += up(bh * max_splits * d * sizeof(float));
    p.part_lse = reinterpret_cast<float*>(w);
    w += up(bh * max_splits * sizeof(float));
    p.lens = reinterpret_cast<int*>(w);
    w += up(static_cast<size_t>(B) * sizeof(int));
    p.cum = reinterpret_cast<int*>(w);
    p.max_splits = static_cast<int>(max_splits);
}

cudaError_t launch_decode(const DecodeParams& p, int d, int num_sms, cudaStream_t stream) {
    fa_decode_plan<<<1, kPlanThreads, 0, stream>>>(p);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    const long long upper = static_cast<long long>(p.B) * p.H * p.max_splits;
    const int grid = static_cast<int>(std::min<long long>(upper, static_cast<long long>(num_sms) * 3));
    if (d == 256) {
        fa_decode_split<256><<<grid, kDecodeThreads, 0, stream>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        fa_decode_combine<256><<<p.B * p.H, 256, 0, stream>>>(p);
    } else if (d == 128) {
        fa_decode_split<128><<<grid, kDecodeThreads, 0, stream>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        fa_decode_combine<128><<<p.B * p.H, 128, 0, stream>>>(p);
    } else {
        fa_decode_split<64><<<grid, kDecodeThreads, 0, stream>>>(p);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        fa_decode_combine<64><<<p.B * p.H, 64, 0, stream>>>(p);
    }
    return cudaGetLastError();
}

}  // namespace fa
