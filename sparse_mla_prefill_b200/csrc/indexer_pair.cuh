// Indexer scores on a CTA pair: the same scores as indexer_tcgen05_kernel, with each
// tcgen05 MMA shared by the two CTAs of a 2-CTA cluster (cta_group::2).
//
// score(t, j) = sum_h w[t,h] * ReLU(q_idx[t,h,:] . k_idx[j,:]) for every compressed row j
// visible to t (4j+3 <= t); the score definition, the tile orientation (rows j as M,
// (token, head) pairs as N, the head sum along one TMEM lane) and the epilogue are those of
// indexer_tcgen05.cuh.
//
// Why a pair: one CTA's 128 x 256 x 16 MMA reads 4 KB of A and 8 KB of B from its shared
// memory per instruction, and that operand traffic, not the tensor pipe, set the single-CTA
// kernel's pace (a tile every ~1,400 cycles against ~1,090 of math, unchanged with every
// TMA load removed). A pair MMA is 256 x 256 x 16: CTA r holds the 128 rows of its j-tile
// (A) and columns 128r .. 128r+127 of the token block's q_idx (B), so each CTA reads 4 KB
// of A and 4 KB of B per instruction for the same math per SM.
//
// Work: units of (token block, pair of 128-row j-tiles 2p, 2p+1); CTA r of the pair
// takes j-tile 2p+r of each. Persistent pairs (one per two SMs) each take a contiguous
// share of about equal cost (cut on the host, as for the single-CTA kernel).
// Protocol (PTX ISA, tcgen05 with cta_group::2): both CTAs load their halves with TMA
// loads that complete on the leader's (rank 0) full barriers, which the leader's loaders
// arm for both CTAs' bytes; the leader's MMA warp issues the pair MMAs and commits them
// to the stage-free barriers of both CTAs at once; each CTA's epilogue reads its own TMEM
// rows and releases the accumulator on the leader's barrier. TMEM is allocated and freed
// by warp 1 of both CTAs. A cluster barrier at the end keeps both CTAs alive until
// neither can touch the other's shared memory. Every wait is bounded (device_common.cuh).
#pragma once

#include <cuda.h>

#include "device_common.cuh"
#include "indexer_tcgen05.cuh"

namespace ds4sp {

template <int D_I, int H_I>
struct PairTile {
    static constexpr int BM = 128;              // rows of one CTA's j-tile (pair M = 256)
    static constexpr int BN = 256;              // (token, head) columns of the pair MMA
    static constexpr int BN_HALF = BN / 2;      // columns held by one CTA
    static constexpr int TB = BN / H_I;         // tokens per token block
    static constexpr int KSUB = D_I / 64;       // 128-byte K sub-tiles
    static constexpr int A_SUB = BM * 128;
    static constexpr int A_STAGE = A_SUB * KSUB;
    static constexpr int B_SUB = BN_HALF * 128;
    static constexpr int B_BYTES = B_SUB * KSUB;  // one CTA's half of a q_idx block
    static constexpr int A_STAGES = KSUB == 2 ? 4 : 8;
    static constexpr int EPI_WARPS = 8;
    static constexpr int B_WARP = 2 + EPI_WARPS;
    static constexpr int THREADS = (3 + EPI_WARPS) * 32;
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int OFF_B = 0;                                   // two B buffers
    static constexpr int OFF_A = 2 * B_BYTES;
    static constexpr int OFF_W = OFF_A + A_STAGES * A_STAGE;          // two w buffers
    static constexpr int OFF_BAR = OFF_W + 2 * BN * 4;
    // afull[A_STAGES], aempty[A_STAGES], bfull[2], bempty[2], tempty[2], done
    static constexpr int N_BARS = 2 * A_STAGES + 2 + 2 + 2 + 1;
    static constexpr int OFF_TMEM_PTR = OFF_BAR + N_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_TMEM_PTR + 16 + 1024;
    static constexpr uint32_t IDESC = umma_idesc_f16_f32(2 * BM, BN);
    static_assert(D_I == 64 || D_I == 128, "D_i must be 64 or 128");
    static_assert(H_I >= 4 && H_I <= 64 && (BN % H_I) == 0, "H_i must be a power of two in [4, 64]");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

// Pair p's share: `count[p]` consecutive (token block, j-tile pair) items from token
// block start_tb[p], pair start_jt[p]; the fields of IndexerParams are reused with j-tile
// pairs in place of j-tiles.
__device__ __forceinline__ int pair_tiles(int tiles) { return (tiles + 1) / 2; }

struct PairWalk {
    int tb, jp, left;
    template <int TB>
    __device__ __forceinline__ bool next(const IndexerParams& p, IndexerUnit& w) {
        if (left <= 0) return false;
        int n = pair_tiles(block_tiles<TB>(p, tb));
        while (n - jp <= 0 && tb + 1 < p.n_tb) {
            ++tb;
            jp = 0;
            n = pair_tiles(block_tiles<TB>(p, tb));
        }
        if (n - jp <= 0) {
            left = 0;
            return false;
        }
        const int take = min(n - jp, left);
        w.tok0 = p.t0 + tb * TB;
        w.tok_end = min(w.tok0 + TB, p.t0 + p.n_q);
        w.jt_begin = jp;                         // in j-tile pairs
        w.n_tiles = take;
        left -= take;
        ++tb;
        jp = 0;
        return true;
    }
};

template <int D_I, int H_I>
__global__ void __launch_bounds__(PairTile<D_I, H_I>::THREADS, 1)
indexer_pair_kernel(const __grid_constant__ CUtensorMap tmap_k,
                    const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ IndexerParams p) {
    using C = PairTile<D_I, H_I>;
    const uint32_t rank = cluster_ctarank();     // 0: the leader
    const int pair = blockIdx.x / 2;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t base = (raw_u32 + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_u32);
    float* sw = reinterpret_cast<float*>(smem + C::OFF_W);
    const uint32_t bar0 = base + C::OFF_BAR;
    auto afull = [&](int s) { return bar0 + 8u * s; };
    auto aempty = [&](int s) { return bar0 + 8u * (C::A_STAGES + s); };
    auto bfull = [&](int i) { return bar0 + 8u * (2 * C::A_STAGES + i); };
    auto bempty = [&](int i) { return bar0 + 8u * (2 * C::A_STAGES + 2 + i); };
    auto tempty = [&](int i) { return bar0 + 8u * (2 * C::A_STAGES + 4 + i); };
    const uint32_t done_bar = bar0 + 8u * (2 * C::A_STAGES + 6);
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_PTR);
    constexpr uint16_t kBoth = 0x3;              // commit to both CTAs of the pair

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::A_STAGES; ++s) {
            mbar_init(afull(s), 1);              // leader: its loader's arm; both CTAs' bytes
            mbar_init(aempty(s), 1);             // the leader's commit
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(bfull(i), 1);
            mbar_init(bempty(i), 1);
            mbar_init(tempty(i), 2 * C::EPI_WARPS);   // leader: both CTAs' epilogue warps
        }
        mbar_init(done_bar, 1);
        fence_mbar_init();
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_q);
    }
    if (warp == 1) {
        tmem_alloc_pair(smem_u32(tmem_ptr), C::TMEM_COLS);
        tmem_relinquish_pair();
    }
    tc_fence_before();
    __syncthreads();
    // The peer's barriers must be initialised before either CTA arrives on or loads
    // into the other's.
    cluster_sync();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_ptr;
    grid_dependency_wait();
    grid_dependents_launch();
    const PairWalk walk0{p.start_tb[pair], p.start_jt[pair], p.count[pair]};

    bool abort = false;
    if (warp == C::B_WARP || warp == 0) {
        // ------------------------------------------------------------ TMA producers
        // Both CTAs load their halves; the leader arms its full barriers for both.
        if (warp == C::B_WARP && lane == 0) {
            int bi = 0;
            PairWalk wk = walk0;
            IndexerUnit w;
            while (!abort && wk.next<C::TB>(p, w)) {
                const int bb = bi & 1;
                if (!mbar_wait(bempty(bb), ((bi >> 1) & 1) ^ 1, p.wc, abort)) break;
                if (rank == 0) mbar_arrive_expect_tx(bfull(bb), 2 * C::B_BYTES);
                const uint32_t full = cluster_addr(bfull(bb), 0);
                for (int ks = 0; ks < C::KSUB; ++ks)
                    tma_load_2d_pair(base + C::OFF_B + bb * C::B_BYTES + ks * C::B_SUB, &tmap_q, full,
                                     ks * 64, (w.tok0 - p.t0) * H_I + (int)rank * C::BN_HALF);
                ++bi;
            }
            if (rank == 0)                       // both CTAs' copies land on these
                for (int i = 0; i < 2; ++i) {
                    const int issued = (bi + 1 - i) / 2;
                    if (issued) mbar_wait_drain(bfull(i), (issued - 1) & 1, p.wc);
                }
        } else if (warp == 0 && lane == 0) {
            int a_it = 0;
            PairWalk wk = walk0;
            IndexerUnit w;
            while (!abort && wk.next<C::TB>(p, w)) {
                for (int it = 0; it < w.n_tiles; ++it, ++a_it) {
                    const int s = a_it % C::A_STAGES;
                    if (!mbar_wait(aempty(s), ((a_it / C::A_STAGES) & 1) ^ 1, p.wc, abort)) break;
                    if (rank == 0) mbar_arrive_expect_tx(afull(s), 2 * C::A_STAGE);
                    const uint32_t full = cluster_addr(afull(s), 0);
                    const int jt = 2 * (w.jt_begin + it) + (int)rank;
#pragma unroll
                    for (int ks = 0; ks < C::KSUB; ++ks)
                        tma_load_2d_pair(base + C::OFF_A + s * C::A_STAGE + ks * C::A_SUB, &tmap_k, full,
                                         ks * 64, jt * C::BM);
                }
            }
            if (rank == 0)
                for (int s = 0; s < C::A_STAGES; ++s) {
                    const int issued = a_it > s ? (a_it - 1 - s) / C::A_STAGES + 1 : 0;
                    if (issued) mbar_wait_drain(afull(s), (issued - 1) & 1, p.wc);
                }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer (leader)
        if (rank == 0 && lane == 0) {
            const uint64_t a_desc0 = umma_desc_sw128(base + C::OFF_A);
            const uint64_t b_desc0 = umma_desc_sw128(base + C::OFF_B);
            int bi = 0, tc = 0;
            PairWalk wk = walk0;
            IndexerUnit w;
            while (!abort && wk.next<C::TB>(p, w)) {
                const int bb = bi & 1;
                if (!mbar_wait(bfull(bb), (bi >> 1) & 1, p.wc, abort)) break;
                const uint64_t b_desc = b_desc0 + (uint64_t)((bb * C::B_BYTES) >> 4);
                for (int it = 0; it < w.n_tiles; ++it, ++tc) {
                    const int buf = tc & 1, s = tc % C::A_STAGES;
                    if (!mbar_wait(tempty(buf), ((tc >> 1) & 1) ^ 1, p.wc, abort)) break;
                    if (!mbar_wait(afull(s), (tc / C::A_STAGES) & 1, p.wc, abort)) break;
                    tc_fence_after();
                    const uint32_t d = tmem_base + buf * C::BN;
                    const uint64_t a_desc = a_desc0 + (uint64_t)((s * C::A_STAGE) >> 4);
#pragma unroll
                    for (int ks = 0; ks < C::KSUB; ++ks)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)
                            umma_f16_pair(d, a_desc + (uint64_t)((ks * C::A_SUB + kk * 32) >> 4),
                                          b_desc + (uint64_t)((ks * C::B_SUB + kk * 32) >> 4), C::IDESC,
                                          ks > 0 || kk > 0);
                    // frees the A stage in both CTAs and tells both epilogues the tile is done
                    umma_commit_pair(aempty(s), kBoth);
                }
                umma_commit_pair(bempty(bb), kBoth);
                ++bi;
            }
            umma_commit_pair(done_bar, kBoth);
        }
        // TMEM is freed below only after the pair MMAs are done (both CTAs wait).
        if (lane == 0) mbar_wait_drain(done_bar, 0, p.wc);
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int e = warp - 2;                      // 0..7
        const int quarter = warp & 3;                // TMEM lanes 32*quarter .. +31
        const int half = e / 4;                      // columns 128*half .. +127
        const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16) + half * 128;
        const int col = e * 32 + lane;
        auto unit_weight = [&](const IndexerUnit& w) {
            const int tl = col / H_I;
            return (w.tok0 + tl < w.tok_end) ? p.w[(size_t)(w.tok0 - p.t0 + tl) * H_I + (col % H_I)]
                                             : 0.f;
        };
        int bi = 0, tc = 0;
        PairWalk wk = walk0;
        IndexerUnit w, w_nx;
        bool have = wk.next<C::TB>(p, w_nx);
        float w_next = have ? unit_weight(w_nx) : 0.f;
        while (have) {
            w = w_nx;
            const float w_this = w_next;
            have = wk.next<C::TB>(p, w_nx);
            w_next = have ? unit_weight(w_nx) : 0.f;
            float* swb = sw + (bi & 1) * C::BN;
            swb[col] = 0.5f * w_this;           // halved: see epilogue_half
            named_barrier(1, C::EPI_WARPS * 32);
            const float* wh = swb + half * 128;
            for (int it = 0; it < w.n_tiles; ++it, ++tc) {
                const int buf = tc & 1;
                const bool ready = mbar_wait(aempty(tc % C::A_STAGES), (tc / C::A_STAGES) & 1,
                                             p.wc, abort);
                if (!__all_sync(0xffffffffu, ready)) {
                    abort = true;
                    continue;
                }
                tc_fence_after();
                const int j = (2 * (w.jt_begin + it) + (int)rank) * C::BM + quarter * 32 + lane;
                const int t_first = w.tok0 + half * (128 / H_I);
                epilogue_tile<H_I>(
                    lane_addr + buf * C::BN, wh,
                    [&] {
                        // the leader may reuse this accumulator once both CTAs released it
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive_cluster(cluster_addr(tempty(buf), 0));
                    },
                    [&](int tk, float score) {
                        const int t = t_first + tk;
                        if (t < w.tok_end && p.ratio * (j + 1) <= t + 1)
                            p.scores[(size_t)(t - p.t0) * p.ld + j] = score;
                    });
            }
            ++bi;
        }
    }

    tc_fence_before();
    __syncthreads();
    // Neither CTA leaves while the other may still arrive on or load into its barriers.
    cluster_sync();
    tc_fence_after();
    // After a give-up a loader may have issued copies for a stage the leader never armed,
    // which no barrier here tracks: let them land (copies take microseconds) before the
    // shared memory is released.
    if (launch_gave_up(p.wc)) {
        const unsigned long long t_end = global_ns() + 50000ull;
        while (global_ns() < t_end) {
        }
    }
    if (warp == 1) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
}

}  // namespace ds4sp
