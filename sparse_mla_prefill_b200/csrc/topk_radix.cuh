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
// to the same key). Four 8-bit radix passes over the keys in shared memory find the
// k-th largest key K and how many keys equal to K must be kept (`need`). A block
// scan then writes, in ascending j, every key > K and the first `need` keys == K.
#pragma once

#include "device_common.cuh"

namespace ds4sp {

__device__ __forceinline__ uint32_t order_key(float x) {
    uint32_t u = __float_as_uint(x);
    if (x == 0.f) u = 0u;                        // -0 ties with +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive block scan of a pair of counts packed as (hi << 32 | lo).
template <int THREADS>
__device__ __forceinline__ unsigned long long block_exclusive_scan(unsigned long long v,
                                                                    unsigned long long* warp_tot) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    unsigned long long incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const unsigned long long o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
    }
    if (lane == 31) warp_tot[warp] = incl;
    __syncthreads();
    unsigned long long before = 0;
    for (int w = 0; w < warp; ++w) before += warp_tot[w];
    return before + incl - v;
}

template <int THREADS>
__global__ void __launch_bounds__(THREADS)
topk_radix_kernel(const float* __restrict__ scores, int ld, int t0, int n_q, int k, int ratio,
                  int32_t* __restrict__ topk) {
    extern __shared__ uint32_t keys[];           // [ld]
    __shared__ uint32_t hist[256];
    __shared__ uint32_t s_digit, s_above;
    __shared__ unsigned long long warp_tot[THREADS / 32];

    const int i = blockIdx.x;
    const int t = t0 + i;
    const int nv = n_vis(t, ratio);
    int32_t* out = topk + (size_t)i * k;
    const int tid = threadIdx.x;

    if (nv <= k) {                               // every visible row is kept
        for (int s = tid; s < k; s += THREADS) out[s] = s < nv ? s : -1;
        return;
    }
    const float* row = scores + (size_t)i * ld;
    for (int j = tid; j < nv; j += THREADS) keys[j] = order_key(row[j]);

    uint32_t prefix = 0, mask = 0, remaining = (uint32_t)k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int b = tid; b < 256; b += THREADS) hist[b] = 0;
        __syncthreads();
        for (int j = tid; j < nv; j += THREADS) {
            const uint32_t key = keys[j];
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid < 32) {
            // Lane l owns bins 8l .. 8l+7; find the digit where the count from the top
            // first reaches `remaining`.
            uint32_t cnt[8], lane_sum = 0;
#pragma unroll
            for (int b = 0; b < 8; ++b) {
                cnt[b] = hist[8 * tid + b];
                lane_sum += cnt[b];
            }
            uint32_t suffix = lane_sum;          // bins of lanes >= tid
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const uint32_t o = __shfl_down_sync(0xffffffffu, suffix, off);
                if (tid + off < 32) suffix += o;
            }
            uint32_t above = suffix - lane_sum;  // bins of lanes > tid
#pragma unroll
            for (int b = 7; b >= 0; --b) {
                if (above < remaining && above + cnt[b] >= remaining) {
                    s_digit = 8u * tid + b;
                    s_above = above;
                }
                above += cnt[b];
            }
        }
        __syncthreads();
        prefix |= s_digit << shift;
        mask |= 255u << shift;
        remaining -= s_above;
        __syncthreads();                         // s_digit / hist reused next pass
    }
    const uint32_t thr = prefix;                 // the k-th largest key
    const uint32_t need = remaining;             // keys == thr to keep, lowest j first

    const int per = (nv + THREADS - 1) / THREADS;
    const int jb = min(nv, tid * per), je = min(nv, jb + per);
    uint32_t gt = 0, eq = 0;
    for (int j = jb; j < je; ++j) {
        const uint32_t key = keys[j];
        gt += key > thr;
        eq += key == thr;
    }
    const unsigned long long before =
        block_exclusive_scan<THREADS>(((unsigned long long)gt << 32) | eq, warp_tot);
    const uint32_t gt_before = (uint32_t)(before >> 32), eq_before = (uint32_t)before;
    uint32_t pos = gt_before + min(eq_before, need), eq_rank = eq_before;
    for (int j = jb; j < je; ++j) {
        const uint32_t key = keys[j];
        if (key > thr) {
            out[pos++] = j;
        } else if (key == thr) {
            if (eq_rank < need) out[pos++] = j;
            ++eq_rank;
        }
    }
}

}  // namespace ds4sp
