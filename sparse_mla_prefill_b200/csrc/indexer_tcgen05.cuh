// Indexer scores on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// score(t, j) = sum_h w[t,h] * ReLU(q_idx[t,h,:] . k_idx[j,:]) for every compressed
// row j visible to t (4j+3 <= t). The pages name the indexer ("direct long-prefill
// top-k handoff", "perf(ds4): extend sparse prefill scheduling to 10K", Summary;
// "packed small-CM rocWMMA indexer", "perf(ds4): accelerate long context and add
// PFlash", Summary) without defining its score; this library fixes the formula above.
//
// Tile: D[j, (t,h)] = k_idx[j,:] . q_idx[t,h,:] with the 128 compressed rows of a tile
// as UMMA M and 256 (token, head) pairs as UMMA N, so each TMEM lane holds one row j
// and the head sum for a token runs along that lane's columns, inside one thread:
// no cross-lane reduction. K = D_i in steps of 16.
//
// Warp roles (192 threads): warp 0 issues TMA loads, warp 1 owns TMEM and issues
// the MMAs, warps 2-5 run the epilogue (ReLU, head weights, sum, store). Two TMEM
// accumulators (2 x 256 columns) let the epilogue of tile i overlap the MMAs of
// tile i+1. Every wait is bounded (device_common.cuh).
#pragma once

#include <cuda.h>

#include "device_common.cuh"

namespace ds4sp {

template <int D_I, int H_I>
struct IndexerTile {
    static constexpr int BM = 128;              // compressed rows per tile (UMMA M)
    static constexpr int BN = 256;              // (token, head) columns per tile (UMMA N)
    static constexpr int TB = BN / H_I;         // tokens per tile
    static constexpr int KSUB = D_I / 64;       // 128-byte K sub-tiles (64 fp16 each)
    static constexpr int A_SUB = BM * 128;      // bytes of one A sub-tile
    static constexpr int B_SUB = BN * 128;      // bytes of one B sub-tile
    static constexpr int A_STAGE = A_SUB * KSUB;
    static constexpr int B_BYTES = B_SUB * KSUB;
    static constexpr int STAGES = 4;
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int OFF_B = 0;
    static constexpr int OFF_A = B_BYTES;
    static constexpr int OFF_W = OFF_A + STAGES * A_STAGE;
    static constexpr int OFF_BAR = OFF_W + BN * 4;
    static constexpr int N_BARS = 2 * STAGES + 1 + 2 + 2 + 1;  // full, empty, b, tfull, tempty, done
    static constexpr int OFF_TMEM_PTR = OFF_BAR + N_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_TMEM_PTR + 16 + 1024;  // + alignment slack
    static constexpr uint32_t IDESC = umma_idesc_f16_f32(BM, BN);
    static_assert(D_I == 64 || D_I == 128, "D_i must be 64 or 128");
    static_assert(H_I >= 1 && H_I <= 64 && (BN % H_I) == 0, "H_i must divide 256 and be <= 64");
};

struct IndexerParams {
    const float* w;        // [n_q, H_i] fp32, row 0 = token t0
    float* scores;         // [n_q, ld] fp32 scratch
    uint32_t* status;      // device status word
    int t0, n_q, ld, ratio;
    int n_tb;              // token blocks of TB tokens
    int nsplit;            // j-tile ranges per token block
};

// Wait used only while draining at exit: ignores the abort flag, still bounded.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity, uint32_t* status) {
    bool abort = false;
    mbar_wait(bar, parity, status, abort);
}

template <int D_I, int H_I>
__global__ void __launch_bounds__(192, 1)
indexer_tcgen05_kernel(const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_q, IndexerParams p) {
    using C = IndexerTile<D_I, H_I>;
    // Heavy token blocks (later tokens see more rows) are launched first.
    const int unit = blockIdx.x;
    const int tb = p.n_tb - 1 - unit / p.nsplit;
    const int split = unit % p.nsplit;
    const int tok0 = p.t0 + tb * C::TB;                       // first token of the block
    const int tok_end = min(tok0 + C::TB, p.t0 + p.n_q);
    const int nv_last = n_vis(tok_end - 1, p.ratio);
    const int n_jt = (nv_last + C::BM - 1) / C::BM;
    const int chunk = (n_jt + p.nsplit - 1) / p.nsplit;
    const int jt_begin = split * chunk;
    const int n_tiles = min(n_jt, jt_begin + chunk) - jt_begin;
    if (n_tiles <= 0) return;                                 // uniform across the CTA

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t base = (raw_u32 + 1023u) & ~1023u;         // 128B-swizzle atoms need 1 KB alignment
    uint8_t* smem = smem_raw + (base - raw_u32);
    float* sw = reinterpret_cast<float*>(smem + C::OFF_W);
    const uint32_t bar0 = base + C::OFF_BAR;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (C::STAGES + s); };
    const uint32_t b_bar = bar0 + 8u * (2 * C::STAGES);
    auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * C::STAGES + 1 + b); };
    auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * C::STAGES + 3 + b); };
    const uint32_t done_bar = bar0 + 8u * (2 * C::STAGES + 5);
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_PTR);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

    if (threadIdx.x == 0) {
        for (int s = 0; s < C::STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(b_bar, 1);
        for (int b = 0; b < 2; ++b) {
            mbar_init(tfull_bar(b), 1);
            mbar_init(tempty_bar(b), 4);   // one arrive per epilogue warp
        }
        mbar_init(done_bar, 1);
        fence_mbar_init();
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_q);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_ptr), C::TMEM_COLS);
        tmem_relinquish();
    }
    // Head weights of this block's tokens, in column order (col = token*H_i + h).
    for (int c = threadIdx.x; c < C::BN; c += blockDim.x) {
        const int tl = c / H_I;
        sw[c] = (tok0 + tl < tok_end) ? p.w[(size_t)(tok0 - p.t0 + tl) * H_I + (c % H_I)] : 0.f;
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_ptr;

    bool abort = false;
    if (warp == 0) {
        if (lane == 0) {
            // B operand: the block's (token, head) rows of q_idx, loaded once.
            mbar_arrive_expect_tx(b_bar, C::B_BYTES);
            for (int ks = 0; ks < C::KSUB; ++ks)
                tma_load_2d(base + C::OFF_B + ks * C::B_SUB, &tmap_q, b_bar, ks * 64,
                            (tok0 - p.t0) * H_I);
            int issued[C::STAGES] = {};
            for (int it = 0; it < n_tiles; ++it) {
                const int s = it % C::STAGES;
                if (!mbar_wait(empty_bar(s), ((it / C::STAGES) & 1) ^ 1, p.status, abort)) break;
                mbar_arrive_expect_tx(full_bar(s), C::A_STAGE);
                for (int ks = 0; ks < C::KSUB; ++ks)
                    tma_load_2d(base + C::OFF_A + s * C::A_STAGE + ks * C::A_SUB, &tmap_k,
                                full_bar(s), ks * 64, (jt_begin + it) * C::BM);
                ++issued[s];
            }
            // Every bulk copy this CTA started must land before the CTA exits.
            mbar_drain(b_bar, 0, p.status);
            for (int s = 0; s < C::STAGES; ++s)
                if (issued[s]) mbar_drain(full_bar(s), (issued[s] - 1) & 1, p.status);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            if (mbar_wait(b_bar, 0, p.status, abort)) {
                for (int it = 0; it < n_tiles; ++it) {
                    const int s = it % C::STAGES, buf = it & 1;
                    if (!mbar_wait(tempty_bar(buf), ((it >> 1) & 1) ^ 1, p.status, abort)) break;
                    if (!mbar_wait(full_bar(s), (it / C::STAGES) & 1, p.status, abort)) break;
                    tc_fence_after();
                    const uint32_t d = tmem_base + buf * C::BN;
                    const uint32_t a0 = base + C::OFF_A + s * C::A_STAGE;
                    const uint32_t b0 = base + C::OFF_B;
#pragma unroll
                    for (int kk = 0; kk < D_I / 16; ++kk) {
                        // k16 step kk: sub-tile kk/4, 32-byte offset inside the 128-byte row
                        const uint32_t off = (kk % 4) * 32;
                        const uint64_t ad = umma_desc_sw128(a0 + (kk / 4) * C::A_SUB + off);
                        const uint64_t bd = umma_desc_sw128(b0 + (kk / 4) * C::B_SUB + off);
                        umma_f16(d, ad, bd, C::IDESC, kk > 0);
                    }
                    umma_commit(empty_bar(s));     // A stage free once these MMAs finish
                    umma_commit(tfull_bar(buf));   // accumulator ready for the epilogue
                }
            }
            // All MMAs issued by this thread must finish before TMEM is released.
            umma_commit(done_bar);
            mbar_drain(done_bar, 0, p.status);
        }
        __syncwarp();
    } else {
        // Epilogue: warp w reads TMEM lanes 32*(w%4) .. 32*(w%4)+31.
        const int quarter = warp & 3;
        const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16);
        for (int it = 0; it < n_tiles; ++it) {
            const int buf = it & 1;
            const bool ready = mbar_wait(tfull_bar(buf), (it >> 1) & 1, p.status, abort);
            if (!__all_sync(0xffffffffu, ready)) break;   // warp-uniform before .sync.aligned loads
            tc_fence_after();
            // Columns are (token, head) in token-major order, so one running sum
            // suffices: a token's sum is complete at its last head column.
            const int j = (jt_begin + it) * C::BM + quarter * 32 + lane;
            float acc = 0.f;
#pragma unroll
            for (int ch = 0; ch < C::BN / 32; ++ch) {
                uint32_t v[32];
                tmem_ld_x32(lane_addr + buf * C::BN + ch * 32, v);
                tmem_ld_wait();
                if (ch == C::BN / 32 - 1) {        // all of this buffer is in registers
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(tempty_bar(buf));
                }
#pragma unroll
                for (int c = 0; c < 32; ++c) {
                    const int col = ch * 32 + c;
                    acc = fmaf(sw[col], fmaxf(__uint_as_float(v[c]), 0.f), acc);
                    if (col % H_I == H_I - 1) {
                        const int t = tok0 + col / H_I;
                        if (t < tok_end && j < n_vis(t, p.ratio))
                            p.scores[(size_t)(t - p.t0) * p.ld + j] = acc;
                        acc = 0.f;
                    }
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace ds4sp
