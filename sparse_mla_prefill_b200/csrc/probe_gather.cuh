// Row-gather bandwidth probe: a measurement helper, not a step of the path.
//
// The attention kernel's traffic is a gather of 1152-byte latent rows chosen per token
// from a table that stays in L2 (the unique KV of a 10K prefill is 14.75 MB, well under
// the 126 MB L2). Its roofline against HBM bandwidth therefore says little about how
// close it runs to the memory system's limit for that access pattern. This kernel
// measures the limit directly: it reads rows of `row_bytes` at the given indices with
// 16-byte loads into registers, eight lanes per row, nine loads in flight per lane for
// a 1152-byte row, and folds everything into one word so that no load is dead.
#pragma once

#include "device_common.cuh"

namespace ds4sp {

constexpr int kProbeThreads = 512;

template <int CHUNKS_PER_LANE>
__global__ void __launch_bounds__(kProbeThreads)
probe_gather_kernel(const uint4* __restrict__ table, int row_chunks,
                    const int32_t* __restrict__ idx, int n, uint32_t* sink) {
    const int lane = threadIdx.x & 31, sub = lane & 7;
    const int group = (blockIdx.x * kProbeThreads + threadIdx.x) >> 3;   // one row per 8 lanes
    const int groups = gridDim.x * kProbeThreads / 8;
    uint32_t acc = 0;
    for (int r = group; r < n; r += groups) {
        const uint4* row = table + (size_t)idx[r] * row_chunks;
        uint4 v[CHUNKS_PER_LANE];
#pragma unroll
        for (int m = 0; m < CHUNKS_PER_LANE; ++m) {
            const int c = sub + 8 * m;
            v[m] = c < row_chunks ? __ldcg(row + c) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int m = 0; m < CHUNKS_PER_LANE; ++m) acc ^= v[m].x ^ v[m].y ^ v[m].z ^ v[m].w;
    }
    acc = __reduce_xor_sync(0xffffffffu, acc);
    if (lane == 0) atomicXor(sink, acc);
}

}  // namespace ds4sp
