// Exact per-token top-k select: radix select in shared memory, then an
// order-preserving compaction.
//
// For token t, keep the min(k, n_vis(t)) largest scores among rows j < n_vis(t);
// among equal scores the lower j wins; write the kept j in ascending order, then -1.
// This is the "authoritative long-prefill top-k rows" handed straight to attention
// in "perf(ds4): extend sparse prefill scheduling to 10K", Summary ("pass
// authoritative long-prefill top-k rows directly", "preserve ... selected-row
// order"); the tie rule and the ascending listing are this library's reading.
//
// One CTA per token. fp32 scores become order-preserving 32-bit keys (+0 and -0 map
// to the same key). 8-bit radix passes over the keys find the k-th largest key K and
// how many keys equal to K must be kept (`need`). The passes cover only the bits where
// the candidates' keys differ (a block-wide AND and OR while the keys load):
// integer-valued indexer scores in a narrow range share their top and bottom bits, so
// two passes usually replace four, and the first pass spreads the keys over many
// histogram bins instead of a few. The compaction then writes, in ascending j, every
// key > K and the first `need` keys == K.
//
// The keys sit in shared memory; after a block scan of per-thread counts each thread
// compacts a contiguous run of j.
//
// Explicit-mask form (a debug form of the same kernel, for the "explicit-mask versus
// analytic-mask" check of the page's Qualification section): when `vis_mask` is
// given, the candidates are the j < mask_cols whose mask byte for token t is set,
// instead of j < n_vis(t). Rows the mask hides get key 0, below every finite score,
// so they are never kept; with fewer than k candidates all of them are kept and the
// remaining slots hold -1. Scores must be finite.
#pragma once

#include "device_common.cuh"

namespace ds4sp {

__device__ __forceinline__ uint32_t order_key(float x) {
    uint32_t u = __float_as_uint(x);
    if (x == 0.f) u = 0u;                        // -0 ties with +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The select helpers below run on a group of THREADS threads that synchronise through
// `sync` (the whole block with __syncthreads, or a select group of the fused indexer
// with a named barrier); `tid` is the thread's index inside the group (0 .. THREADS-1),
// and the group starts on a warp boundary.
struct BlockSync {
    __device__ __forceinline__ void operator()() const { __syncthreads(); }
};

// Block-wide OR and AND of the candidates' keys and their count (every thread gets
// them): bits where OR and AND agree are the same in every candidate.
template <int THREADS, class Sync>
__device__ __forceinline__ void block_key_stats(uint32_t kor, uint32_t kand, uint32_t cand,
                                                uint32_t* w_or, uint32_t* w_and, uint32_t* w_cnt,
                                                uint32_t& all_or, uint32_t& all_and,
                                                uint32_t& n_cand, int tid, Sync sync) {
    const int lane = tid & 31, warp = tid >> 5;
    kor = __reduce_or_sync(0xffffffffu, kor);
    kand = __reduce_and_sync(0xffffffffu, kand);
    cand = __reduce_add_sync(0xffffffffu, cand);
    if (lane == 0) {
        w_or[warp] = kor;
        w_and[warp] = kand;
        w_cnt[warp] = cand;
    }
    sync();
    all_or = 0u;
    all_and = 0xffffffffu;
    n_cand = 0u;
#pragma unroll 4
    for (int w = 0; w < THREADS / 32; ++w) {
        all_or |= w_or[w];
        all_and &= w_and[w];
        n_cand += w_cnt[w];
    }
}

// Warp 0: in a 256-bin histogram find the digit where the count from the top first
// reaches `remaining`, and the count of the bins above it. Lane l owns bins 8l .. 8l+7.
__device__ __forceinline__ void radix_find_digit(const uint32_t* hist, uint32_t remaining,
                                                 uint32_t* s_digit, uint32_t* s_above) {
    const int lane = threadIdx.x & 31;
    uint32_t cnt[8], lane_sum = 0;
#pragma unroll
    for (int b = 0; b < 8; ++b) {
        cnt[b] = hist[8 * lane + b];
        lane_sum += cnt[b];
    }
    uint32_t suffix = lane_sum;                  // bins of lanes >= lane
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const uint32_t o = __shfl_down_sync(0xffffffffu, suffix, off);
        if (lane + off < 32) suffix += o;
    }
    uint32_t above = suffix - lane_sum;          // bins of lanes > lane
#pragma unroll
    for (int b = 7; b >= 0; --b) {
        if (above < remaining && above + cnt[b] >= remaining) {
            *s_digit = 8u * lane + b;
            *s_above = above;
        }
        above += cnt[b];
    }
}

// Radix select of the k-th largest candidate key (thr) and of how many keys equal to
// it to keep (need), for n_cand > k candidates whose keys have block-wide OR all_or and
// AND all_and. The 8-bit windows run from the highest bit where the candidates differ
// down to the lowest; bits above the first window are the common prefix, bits below
// the last are common too. The caller runs the passes:
//     RadixSelect<Sync> rs(all_or, all_and, k, tid, sync);
//     while (rs.active) {
//         rs.clear(hist, threads);                      // barrier inside
//         each key x with x != 0 && (x & rs.digits) == rs.prefix:
//             atomicAdd(&hist[(x >> rs.shift) & 255], 1)
//         rs.step(hist, &s_digit, &s_above);            // barriers inside
//     }
//     rs.thr, rs.need
template <class Sync>
struct RadixSelect {
    uint32_t all_or, digits, prefix, remaining, thr, need;
    int shift, lo_bit;
    bool active;
    int tid;
    Sync sync;

    __device__ __forceinline__ RadixSelect(uint32_t or_, uint32_t and_, uint32_t k, int tid_,
                                           Sync sync_)
        : all_or(or_), remaining(k), thr(or_), need(k), tid(tid_), sync(sync_) {
        const uint32_t diff = or_ ^ and_;
        active = diff != 0u;                     // all candidates equal: the first k
        const int hi_bit = active ? 31 - __clz(diff) : 0;
        lo_bit = active ? __ffs(diff) - 1 : 0;
        digits = hi_bit < 31 ? ~((2u << hi_bit) - 1u) : 0u;
        prefix = or_ & digits;
        shift = max(hi_bit - 7, 0);
    }
    __device__ __forceinline__ void clear(uint32_t* hist, int threads) const {
        for (int b = tid; b < 256; b += threads) hist[b] = 0;
        sync();
    }
    __device__ __forceinline__ void step(const uint32_t* hist, uint32_t* s_digit,
                                         uint32_t* s_above) {
        sync();                                  // the histogram is complete
        if (tid < 32) radix_find_digit(hist, remaining, s_digit, s_above);
        sync();
        prefix |= *s_digit << shift;
        digits |= 255u << shift;
        remaining -= *s_above;
        sync();                                  // s_digit / hist reused next pass
        if (shift <= lo_bit) {
            active = false;
            thr = prefix | (all_or & ((1u << shift) - 1u));
            need = remaining;
        } else {
            shift = max(shift - 8, 0);
        }
    }
};

// Exclusive block scan of a pair of counts packed as (hi << 32 | lo).
template <int THREADS, class Sync>
__device__ __forceinline__ unsigned long long block_exclusive_scan(unsigned long long v,
                                                                    unsigned long long* warp_tot,
                                                                    int tid, Sync sync) {
    const int lane = tid & 31, warp = tid >> 5;
    unsigned long long incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned long long o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_tot[warp] = incl;
    sync();
    unsigned long long before = 0;
    for (int w = 0; w < warp; ++w) before += warp_tot[w];
    return before + incl - v;
}

// One CTA per token. The 128-thread form is held to 32 registers (16 CTAs an SM) so that
// a 2,048-token band's CTAs run in one wave (148 x 16 >= 2,048) instead of 1.4 waves.
template <int THREADS>
__global__ void __launch_bounds__(THREADS, THREADS <= 128 ? 16 : 1)
topk_radix_kernel(const float* __restrict__ scores, int ld, int t0, int n_q, int k, int ratio,
                  const uint8_t* __restrict__ vis_mask, long long mask_ld, int mask_cols,
                  int32_t* __restrict__ topk) {
    // Keys are handled four at a time (16-byte loads and shared-memory accesses): the
    // row and the key array are 16-byte aligned and ld is a multiple of 4, so the
    // n4 = ceil(n/4) groups stay inside both; keys of j >= n are 0 (no candidate).
    extern __shared__ uint4 keys4[];             // [ld / 4]
    __shared__ uint32_t hist[256];
    __shared__ uint32_t s_digit, s_above;
    __shared__ uint32_t w_or[THREADS / 32], w_and[THREADS / 32], w_cnt[THREADS / 32];
    __shared__ unsigned long long warp_tot[THREADS / 32];

    const int i = blockIdx.x;
    const int t = t0 + i;
    grid_dependency_wait();                      // the scores are complete
    grid_dependents_launch();
    int32_t* out = topk + (size_t)i * k;
    const int tid = threadIdx.x;
    const float4* row4 = reinterpret_cast<const float4*>(scores + (size_t)i * ld);
    int n;                                       // keys examined: j < n
    int keep = k;                                // slots filled; the rest hold -1
    uint32_t kor = 0u, kand = 0xffffffffu, cand = 0u;   // over this thread's candidates
    auto take = [&](uint32_t key) {
        kor |= key;
        kand &= key;
        ++cand;
    };

    if (vis_mask == nullptr) {
        n = n_vis(t, ratio);
        if (n <= k) {                            // every visible row is kept
            for (int s = tid; s < k; s += THREADS) out[s] = s < n ? s : -1;
            return;
        }
        const int n4 = (n + 3) / 4;
        for (int x = tid; x < n4; x += THREADS) {
            const float4 v = row4[x];
            const int j = 4 * x;
            uint4 kk;
            kk.x = order_key(v.x);
            kk.y = j + 1 < n ? order_key(v.y) : 0u;
            kk.z = j + 2 < n ? order_key(v.z) : 0u;
            kk.w = j + 3 < n ? order_key(v.w) : 0u;
            keys4[x] = kk;
            take(kk.x);
            if (kk.y) take(kk.y);
            if (kk.z) take(kk.z);
            if (kk.w) take(kk.w);
        }
    } else {
        n = mask_cols;
        const uint8_t* mrow = vis_mask + (size_t)t * mask_ld;
        const int n4 = (n + 3) / 4;
        for (int x = tid; x < n4; x += THREADS) {
            const float4 v = row4[x];
            const float f[4] = {v.x, v.y, v.z, v.w};
            uint32_t kk[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int j = 4 * x + c;
                const bool vis = j < n && mrow[j] != 0;
                kk[c] = vis ? order_key(f[c]) : 0u;
                if (vis) take(kk[c]);
            }
            keys4[x] = make_uint4(kk[0], kk[1], kk[2], kk[3]);
        }
    }
    const int n4 = (n + 3) / 4;
    uint32_t all_or, all_and, n_cand;
    block_key_stats<THREADS>(kor, kand, cand, w_or, w_and, w_cnt, all_or, all_and, n_cand, tid,
                             BlockSync{});

    uint32_t thr = 0, need = 0;                  // without selection: every key > 0
    if (n_cand <= (uint32_t)k) {
        keep = (int)n_cand;                      // keep every candidate
    } else {
        RadixSelect<BlockSync> rs(all_or, all_and, (uint32_t)k, tid, BlockSync{});
        while (rs.active) {
            rs.clear(hist, THREADS);
            for (int x = tid; x < n4; x += THREADS) {
                const uint4 kk = keys4[x];
                const uint32_t q[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
                for (int c = 0; c < 4; ++c)
                    if (q[c] != 0u && (q[c] & rs.digits) == rs.prefix)
                        atomicAdd(&hist[(q[c] >> rs.shift) & 255u], 1u);
            }
            rs.step(hist, &s_digit, &s_above);
        }
        thr = rs.thr;                            // the k-th largest key
        need = rs.need;                          // keys == thr to keep, lowest j first
    }

    // Each thread compacts a contiguous run of key groups, in ascending j.
    const int per = (n4 + THREADS - 1) / THREADS;
    const int xb = min(n4, tid * per), xe = min(n4, xb + per);
    uint32_t gt = 0, eq = 0;
    for (int x = xb; x < xe; ++x) {
        const uint4 kk = keys4[x];
        gt += (kk.x > thr) + (kk.y > thr) + (kk.z > thr) + (kk.w > thr);
        eq += (kk.x == thr) + (kk.y == thr) + (kk.z == thr) + (kk.w == thr);
    }
    const unsigned long long before =
        block_exclusive_scan<THREADS>(((unsigned long long)gt << 32) | eq, warp_tot, tid, BlockSync{});
    const uint32_t gt_before = (uint32_t)(before >> 32), eq_before = (uint32_t)before;
    uint32_t pos = gt_before + min(eq_before, need), eq_rank = eq_before;
    for (int x = xb; x < xe; ++x) {
        const uint4 kk = keys4[x];
        const uint32_t q[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
        for (int c = 0; c < 4; ++c) {
            if (q[c] > thr) {
                out[pos++] = 4 * x + c;
            } else if (q[c] == thr) {
                if (eq_rank < need) out[pos++] = 4 * x + c;
                ++eq_rank;
            }
        }
    }
    for (int s = keep + tid; s < k; s += THREADS) out[s] = -1;
}

// ---------------------------------------------------------------- a cluster per token
//
// The same selection for calls of a few tokens with long rows (the verify form: one to
// five tokens, 30,720 candidates each), where one CTA per token would leave the GPU
// idle: a cluster of CL CTAs per token, CTA r holding the keys of j in [r c, r c + c),
// c = ceil(n / CL), in its shared memory. The OR/AND window, each radix pass's 256-bin
// histogram and the compaction's counts are combined across the cluster through
// distributed shared memory (each CTA reads its peers' words after a cluster barrier;
// every CTA derives the same digits from the same sums). Histograms alternate between
// two buffers, so one cluster barrier per pass suffices: a buffer is cleared only after
// the barrier that follows every peer's reads of it. Analytic visibility only.
template <int CL, int THREADS>
__global__ void __launch_bounds__(THREADS)
topk_cluster_kernel(const float* __restrict__ scores, int ld, int t0, int n_q, int k, int ratio,
                    int32_t* __restrict__ topk) {
    extern __shared__ uint32_t keys[];           // [c]
    __shared__ uint32_t hist[2][256];
    __shared__ uint32_t ghist[256];              // the cluster's sums of a pass
    __shared__ uint32_t s_word[4];               // this CTA's OR, AND; kept > thr, == thr
    __shared__ uint32_t s_all[4];                // the cluster's OR, AND; counts before this CTA
    __shared__ uint32_t s_digit, s_above;
    __shared__ uint32_t w_or[THREADS / 32], w_and[THREADS / 32], w_cnt[THREADS / 32];
    __shared__ unsigned long long warp_tot[THREADS / 32];

    const uint32_t rank = cluster_ctarank();
    const int i = blockIdx.x / CL;               // the launch's token (grid = n_q x CL)
    const int tid = threadIdx.x;
    grid_dependency_wait();                      // the scores are complete
    grid_dependents_launch();
    const int t = t0 + i;
    const int n = n_vis(t, ratio);
    int32_t* out = topk + (size_t)i * k;
    if (n <= k) {                                // the same in every CTA of the cluster
        if (rank == 0)
            for (int s = tid; s < k; s += THREADS) out[s] = s < n ? s : -1;
        return;
    }
    const int c = (n + CL - 1) / CL;
    const int jb = min(n, (int)rank * c), nl = min(n, jb + c) - jb;   // this CTA's keys
    const float* row = scores + (size_t)i * ld + jb;
    uint32_t kor = 0u, kand = 0xffffffffu, cand = 0u;
    for (int x = tid; x < nl; x += THREADS) {
        const uint32_t key = order_key(row[x]);
        keys[x] = key;
        kor |= key;
        kand &= key;
        ++cand;
    }
    uint32_t cta_or, cta_and, cta_cnt;
    block_key_stats<THREADS>(kor, kand, cand, w_or, w_and, w_cnt, cta_or, cta_and, cta_cnt, tid,
                             BlockSync{});
    if (tid == 0) {
        s_word[0] = cta_or;
        s_word[1] = cta_and;
    }
    cluster_sync();
    if (tid < 32) {
        uint32_t o = 0u, a = 0xffffffffu;
        if (tid < CL) {
            o = ld_cluster_u32(smem_u32(&s_word[0]), tid);
            a = ld_cluster_u32(smem_u32(&s_word[1]), tid);
        }
        o = __reduce_or_sync(0xffffffffu, o);
        a = __reduce_and_sync(0xffffffffu, a);
        if (tid == 0) {
            s_all[0] = o;
            s_all[1] = a;
        }
    }
    __syncthreads();
    const uint32_t all_or = s_all[0], all_and = s_all[1];

    // Radix passes over the bits where the token's candidates differ (as RadixSelect).
    uint32_t thr = all_or, need = (uint32_t)k;   // all candidates equal: the first k
    const uint32_t diff = all_or ^ all_and;
    if (diff != 0u) {
        const int hi_bit = 31 - __clz(diff), lo_bit = __ffs(diff) - 1;
        uint32_t digits = hi_bit < 31 ? ~((2u << hi_bit) - 1u) : 0u;
        uint32_t prefix = all_or & digits, remaining = (uint32_t)k;
        int shift = max(hi_bit - 7, 0);
        for (int pass = 0;; ++pass) {
            uint32_t* h = hist[pass & 1];
            for (int b = tid; b < 256; b += THREADS) h[b] = 0u;
            __syncthreads();
            for (int x = tid; x < nl; x += THREADS) {
                const uint32_t key = keys[x];
                if ((key & digits) == prefix) atomicAdd(&h[(key >> shift) & 255u], 1u);
            }
            cluster_sync();                      // every CTA's histogram of this pass
            for (int b = tid; b < 256; b += THREADS) {
                uint32_t sum = 0u;
#pragma unroll
                for (int r = 0; r < CL; ++r) sum += ld_cluster_u32(smem_u32(&h[b]), r);
                ghist[b] = sum;
            }
            __syncthreads();
            if (tid < 32) radix_find_digit(ghist, remaining, &s_digit, &s_above);
            __syncthreads();
            prefix |= s_digit << shift;
            digits |= 255u << shift;
            remaining -= s_above;
            if (shift <= lo_bit) {
                thr = prefix | (all_or & ((1u << shift) - 1u));
                need = remaining;
                break;
            }
            shift = max(shift - 8, 0);
        }
    }

    // Compaction in ascending j: this CTA's keys > thr and its share of the first
    // `need` keys == thr, after the counts of the CTAs before it.
    const int per = (nl + THREADS - 1) / THREADS;
    const int xb = min(nl, tid * per), xe = min(nl, xb + per);
    uint32_t gt = 0, eq = 0;
    for (int x = xb; x < xe; ++x) {
        const uint32_t key = keys[x];
        gt += key > thr;
        eq += key == thr;
    }
    const unsigned long long v = ((unsigned long long)gt << 32) | eq;
    const unsigned long long before = block_exclusive_scan<THREADS>(v, warp_tot, tid, BlockSync{});
    if (tid == THREADS - 1) {
        s_word[2] = (uint32_t)((before + v) >> 32);
        s_word[3] = (uint32_t)(before + v);
    }
    cluster_sync();                              // every CTA's counts
    if (tid < 32) {
        uint32_t g = 0u, e = 0u;
        if (tid < (int)rank) {
            g = ld_cluster_u32(smem_u32(&s_word[2]), tid);
            e = ld_cluster_u32(smem_u32(&s_word[3]), tid);
        }
        g = __reduce_add_sync(0xffffffffu, g);
        e = __reduce_add_sync(0xffffffffu, e);
        if (tid == 0) {
            s_all[2] = g;
            s_all[3] = e;
        }
    }
    __syncthreads();
    const uint32_t gt_before = s_all[2] + (uint32_t)(before >> 32);
    const uint32_t eq_before = s_all[3] + (uint32_t)before;
    uint32_t pos = gt_before + min(eq_before, need), eq_rank = eq_before;
    for (int x = xb; x < xe; ++x) {
        const uint32_t key = keys[x];
        if (key > thr) {
            if (pos < (uint32_t)k) out[pos] = jb + x;
            ++pos;
        } else if (key == thr) {
            if (eq_rank < need) {
                if (pos < (uint32_t)k) out[pos] = jb + x;
                ++pos;
            }
            ++eq_rank;
        }
    }
    cluster_sync();                              // no CTA leaves while a peer reads its words
}

}  // namespace ds4sp
