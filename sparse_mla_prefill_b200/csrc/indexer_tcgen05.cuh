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
// Work: the (block of 256/H_i tokens, 128-row j-tile) pairs a launch needs, in block
// order. Persistent CTAs (one per SM) each take a contiguous share of about equal cost
// (a tile, plus the q_idx load of each token block it starts) and process it as one
// unit per token block it touches.
// Warp roles (384 threads): warp 10 loads q_idx blocks into two B buffers, up to two
// units ahead; warp 0 streams whole k_idx tiles (one 64-dim TMA box per K sub-tile)
// into a ring of three (D_i = 128) or four (D_i = 64) stages (a third stage measured
// 2.4% faster than two: the L2 latency of a 32 KB tile needs two tiles of lead);
// warp 1 owns TMEM and issues the MMAs of even tiles, warp 11 those of odd tiles (so
// that one issuer's barrier waits, fences and commit between tiles overlap the other's
// MMAs, which a single issuer left as gaps in the tensor pipe); warps 2-9 run the epilogue (ReLU, head
// weights, sum, store), two warps per TMEM lane quarter, each on half of the columns,
// the second 64 of its columns loading from TMEM while the first 64 are reduced.
// Two TMEM accumulators (2 x 256 columns) let the epilogue of tile i overlap the MMAs
// of tile i+1.
// Every wait is bounded (device_common.cuh).
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
    static constexpr int A_SUB = BM * 128;      // bytes of one 64-dim A sub-tile
    static constexpr int A_STAGE = A_SUB * KSUB;  // one ring stage: a whole k_idx tile
    static constexpr int B_SUB = BN * 128;      // bytes of one B sub-tile
    static constexpr int B_BYTES = B_SUB * KSUB;
    static constexpr int B_BUFS = 2;                                  // q_idx block buffers
    static constexpr int A_STAGES = KSUB == 2 ? 3 : 4;
    static constexpr int EPI_WARPS = 8;
    static constexpr int B_WARP = 2 + EPI_WARPS;                      // q_idx loader
    static constexpr int MMA2_WARP = 3 + EPI_WARPS;                   // MMAs of odd tiles
    static constexpr int THREADS = (4 + EPI_WARPS) * 32;
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int OFF_B = 0;
    static constexpr int OFF_A = B_BUFS * B_BYTES;
    static constexpr int OFF_W = OFF_A + A_STAGES * A_STAGE;          // one unit's weights
    static constexpr int OFF_BAR = OFF_W + BN * 4;
    // afull[A_STAGES], aempty[A_STAGES], bfull[B_BUFS], bempty[B_BUFS], tempty[2], done
    static constexpr int N_BARS = 2 * A_STAGES + 2 * B_BUFS + 2 + 1;
    static constexpr int OFF_TMEM_PTR = OFF_BAR + N_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_TMEM_PTR + 16 + 1024;       // + alignment slack
    static constexpr uint32_t IDESC = umma_idesc_f16_f32(BM, BN);
    static_assert(D_I == 64 || D_I == 128, "D_i must be 64 or 128");
    static_assert(H_I >= 4 && H_I <= 64 && (BN % H_I) == 0, "H_i must be a power of two in [4, 64]");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

constexpr int kIndexerMaxGrid = 160;

struct IndexerParams {
    const float* w;        // [n_q, H_i] fp32, row 0 = token t0
    float* scores;         // [n_q, ld] fp32 scratch
    WaitCtl wc;            // bounded waits of this launch
    int t0, n_q, ld, ratio;
    int n_tb;              // token blocks of TB tokens
    // CTA b's share: count[b] consecutive (token block, j-tile) pairs from token block
    // start_tb[b], j-tile start_jt[b].
    uint16_t start_tb[kIndexerMaxGrid], start_jt[kIndexerMaxGrid], count[kIndexerMaxGrid];
};

// j-tiles (128 compressed rows each) that token block tb needs: those below n_vis of its
// last token.
template <int TB>
__device__ __forceinline__ int block_tiles(const IndexerParams& p, int tb) {
    const int t_last = p.t0 + min((tb + 1) * TB, p.n_q) - 1;
    return (n_vis(t_last, p.ratio) + 127) / 128;
}

// A unit: j-tiles jt_begin .. jt_begin+n_tiles-1 of one token block.
struct IndexerUnit {
    int tok0, tok_end, jt_begin, n_tiles;
    __device__ __forceinline__ int jt(int it) const { return jt_begin + it; }
};

// A CTA's share of the launch: `left` consecutive tiles of the list of all (token block,
// j-tile) pairs in block order, starting at tile jt of block tb. The walk cuts a share
// into one unit per token block it touches.
struct IndexerWalk {
    int tb, jt, left;
    template <int TB>
    __device__ __forceinline__ bool next(const IndexerParams& p, IndexerUnit& w) {
        if (left <= 0) return false;
        int n = block_tiles<TB>(p, tb);
        while (n - jt <= 0 && tb + 1 < p.n_tb) {
            ++tb;
            jt = 0;
            n = block_tiles<TB>(p, tb);
        }
        if (n - jt <= 0) {
            left = 0;
            return false;
        }
        const int take = min(n - jt, left);
        w.tok0 = p.t0 + tb * TB;
        w.tok_end = min(w.tok0 + TB, p.t0 + p.n_q);
        w.jt_begin = jt;
        w.n_tiles = take;
        left -= take;
        ++tb;
        jt = 0;
        return true;
    }
};

// acc.xy += a.xy * b.xy as one packed fp32x2 FMA (round-to-nearest per lane).
__device__ __forceinline__ void ffma2(float& acc_x, float& acc_y, float a_x, float a_y, float b_x,
                                      float b_y) {
    asm("{\n\t.reg .b64 ra, rb, rc;\n\t"
        "mov.b64 ra, {%2, %3};\n\t"
        "mov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%0, %1};\n\t"
        "fma.rn.f32x2 rc, ra, rb, rc;\n\t"
        "mov.b64 {%0, %1}, rc;\n\t}"
        : "+f"(acc_x), "+f"(acc_y)
        : "f"(a_x), "f"(a_y), "f"(b_x), "f"(b_y));
}

// Epilogue of one 64-column half of a warp's accumulator columns: the scores of its
// 64 / H_I tokens. The ReLU is taken as x + |x| = 2 ReLU(x), exact and on the FMA pipe,
// against head weights stored halved (0.5 w, exact), so every product equals
// w * ReLU(x) bit for bit (for |x| < 2^127 and w not subnormal). NP independent packed
// accumulators per token keep the FMA chains short. store(token of the half, score).
template <int H_I, class Store>
__device__ __forceinline__ void epilogue_half(const uint32_t (&vh)[2][32], const float* wh_half,
                                              Store store) {
    constexpr int TPH = 64 / H_I;
    constexpr int NP = H_I >= 16 ? 4 : H_I / 4;
#pragma unroll
    for (int tk = 0; tk < TPH; ++tk) {
        float acc[2 * NP];
#pragma unroll
        for (int i = 0; i < 2 * NP; ++i) acc[i] = 0.f;
#pragma unroll
        for (int c = tk * H_I; c < (tk + 1) * H_I; c += 4) {
            const float4 wv = *reinterpret_cast<const float4*>(wh_half + c);
            const int pr = (c / 4) % NP;
            const float x0 = __uint_as_float(vh[c / 32][c % 32]);
            const float x1 = __uint_as_float(vh[c / 32][c % 32 + 1]);
            const float x2 = __uint_as_float(vh[c / 32][c % 32 + 2]);
            const float x3 = __uint_as_float(vh[c / 32][c % 32 + 3]);
            ffma2(acc[2 * pr], acc[2 * pr + 1], wv.x, wv.y, x0 + fabsf(x0), x1 + fabsf(x1));
            ffma2(acc[2 * pr], acc[2 * pr + 1], wv.z, wv.w, x2 + fabsf(x2), x3 + fabsf(x3));
        }
#pragma unroll
        for (int i = 2; i < 2 * NP; i += 2) {
            acc[0] += acc[i];
            acc[1] += acc[i + 1];
        }
        store(tk, acc[0] + acc[1]);
    }
}

// A warp's 128 accumulator columns of one tile (lane = row j): the first 64 columns are
// loaded and, while they are turned into scores, the other 64 load; the accumulator is
// released (`release`) once both halves are in registers.
template <int H_I, class Release, class Store>
__device__ __forceinline__ void epilogue_tile(uint32_t taddr, const float* wh, Release release,
                                              Store store) {
    uint32_t va[2][32], vb[2][32];
    tmem_ld_x32(taddr, va[0]);
    tmem_ld_x32(taddr + 32, va[1]);
    tmem_ld_wait();
    tmem_ld_x32(taddr + 64, vb[0]);
    tmem_ld_x32(taddr + 96, vb[1]);
    constexpr int TPH = 64 / H_I;
    epilogue_half<H_I>(va, wh, [&](int tk, float s) { store(tk, s); });
    tmem_ld_wait();
    tmem_regs_after_wait(vb[0]);
    tmem_regs_after_wait(vb[1]);
    release();
    epilogue_half<H_I>(vb, wh + 64, [&](int tk, float s) { store(TPH + tk, s); });
}

template <int D_I, int H_I>
__global__ void __launch_bounds__(IndexerTile<D_I, H_I>::THREADS, 1)
indexer_tcgen05_kernel(const __grid_constant__ CUtensorMap tmap_k,
                       const __grid_constant__ CUtensorMap tmap_q, IndexerParams p) {
    using C = IndexerTile<D_I, H_I>;
    const int b = blockIdx.x;

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t base = (raw_u32 + 1023u) & ~1023u;         // 128B-swizzle atoms need 1 KB alignment
    uint8_t* smem = smem_raw + (base - raw_u32);
    float* sw = reinterpret_cast<float*>(smem + C::OFF_W);
    const uint32_t bar0 = base + C::OFF_BAR;
    auto afull = [&](int s) { return bar0 + 8u * s; };
    auto aempty = [&](int s) { return bar0 + 8u * (C::A_STAGES + s); };
    auto bfull = [&](int i) { return bar0 + 8u * (2 * C::A_STAGES + i); };
    auto bempty = [&](int i) { return bar0 + 8u * (2 * C::A_STAGES + C::B_BUFS + i); };
    auto tempty = [&](int i) { return bar0 + 8u * (2 * C::A_STAGES + 2 * C::B_BUFS + i); };
    const uint32_t done_bar = bar0 + 8u * (2 * C::A_STAGES + 2 * C::B_BUFS + 2);
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_PTR);

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::A_STAGES; ++s) {
            mbar_init(afull(s), 1);
            mbar_init(aempty(s), 1);
        }
        for (int i = 0; i < C::B_BUFS; ++i) {
            mbar_init(bfull(i), 1);
            mbar_init(bempty(i), 2);              // both MMA issuers, once per unit
        }
        for (int i = 0; i < 2; ++i) mbar_init(tempty(i), C::EPI_WARPS);  // one per epilogue warp
        mbar_init(done_bar, 2);
        fence_mbar_init();
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_q);
    }
    if (warp == 1) {
        tmem_alloc(smem_u32(tmem_ptr), C::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_ptr;
    // The prologue above (barriers, TMEM, descriptors) may overlap the previous kernel;
    // inputs are read and outputs written only after it has completed.
    grid_dependency_wait();
    grid_dependents_launch();
    // This CTA's share, as the host cut it.
    const IndexerWalk walk0{p.start_tb[b], p.start_jt[b], p.count[b]};

    bool abort = false;
    if (warp == C::B_WARP || warp == 0) {
        // ------------------------------------------------------------ TMA producers
        // The last warp loads the q_idx blocks (B) and runs up to two units ahead; warp 0
        // streams the k_idx tiles (A). Each waits only on the ring it fills.
        if (warp == C::B_WARP && lane == 0) {
            int bi = 0;
            int b_issued[C::B_BUFS] = {};
            IndexerWalk wk = walk0;
            IndexerUnit w;
            while (!abort && wk.next<C::TB>(p, w)) {
                const int bb = bi % C::B_BUFS;
                if (!mbar_wait(bempty(bb), ((bi / C::B_BUFS) & 1) ^ 1, p.wc, abort)) break;
                mbar_arrive_expect_tx(bfull(bb), C::B_BYTES);
                for (int ks = 0; ks < C::KSUB; ++ks)
                    tma_load_2d(base + C::OFF_B + bb * C::B_BYTES + ks * C::B_SUB, &tmap_q,
                                bfull(bb), ks * 64, (w.tok0 - p.t0) * H_I);
                ++b_issued[bb];
                ++bi;
            }
            // Every bulk copy this CTA started must land before the CTA exits (a drain
            // wait: the copies complete on their own, whatever the other roles did).
            for (int i = 0; i < C::B_BUFS; ++i)
                if (b_issued[i]) mbar_wait_drain(bfull(i), (b_issued[i] - 1) & 1, p.wc);
        } else if (warp == 0 && lane == 0) {
            int a_it = 0;
            int a_issued[C::A_STAGES] = {};
            IndexerWalk wk = walk0;
            IndexerUnit w;
            while (!abort && wk.next<C::TB>(p, w)) {
                for (int it = 0; it < w.n_tiles; ++it, ++a_it) {
                    const int s = a_it % C::A_STAGES;
                    if (!mbar_wait(aempty(s), ((a_it / C::A_STAGES) & 1) ^ 1, p.wc, abort))
                        break;
                    mbar_arrive_expect_tx(afull(s), C::A_STAGE);
#pragma unroll
                    for (int ks = 0; ks < C::KSUB; ++ks)
                        tma_load_2d(base + C::OFF_A + s * C::A_STAGE + ks * C::A_SUB, &tmap_k, afull(s),
                                    ks * 64, w.jt(it) * C::BM);
                    ++a_issued[s];
                }
            }
            for (int s = 0; s < C::A_STAGES; ++s)
                if (a_issued[s]) mbar_wait_drain(afull(s), (a_issued[s] - 1) & 1, p.wc);
        }
        __syncwarp();
    } else if (warp == 1 || warp == C::MMA2_WARP) {
        // ------------------------------------------------------------ MMA issuers
        // Two threads issue the MMAs, warp 1 those of even tiles and the last warp those
        // of odd tiles (each on its own accumulator buffer): while one waits on its next
        // tile's barriers, fences and commits, the other's MMAs keep the tensor pipe's
        // short queue filled.
        if (lane == 0) {
            const int par = warp == 1 ? 0 : 1;
            // Descriptors differ only in their start-address field (address >> 4 in the low
            // 14 bits), so each stage's is built once and offset per K step.
            const uint64_t a_desc0 = umma_desc_sw128(base + C::OFF_A);
            const uint64_t b_desc0 = umma_desc_sw128(base + C::OFF_B);
            int bi = 0, tc = 0;
            IndexerWalk wk = walk0;
            IndexerUnit w;
            while (!abort && wk.next<C::TB>(p, w)) {
                const int bb = bi % C::B_BUFS;
                if (!mbar_wait(bfull(bb), (bi / C::B_BUFS) & 1, p.wc, abort)) break;
                const uint64_t b_desc = b_desc0 + (uint64_t)((bb * C::B_BYTES) >> 4);
                for (int it = 0; it < w.n_tiles; ++it, ++tc) {
                    if ((tc & 1) != par) continue;       // the other issuer's tile
                    const int buf = tc & 1, s = tc % C::A_STAGES;
                    if (!mbar_wait(tempty(buf), ((tc >> 1) & 1) ^ 1, p.wc, abort)) break;
                    if (!mbar_wait(afull(s), (tc / C::A_STAGES) & 1, p.wc, abort)) break;
                    tc_fence_after();
                    const uint32_t d = tmem_base + buf * C::BN;
                    const uint64_t a_desc = a_desc0 + (uint64_t)((s * C::A_STAGE) >> 4);
#pragma unroll
                    for (int ks = 0; ks < C::KSUB; ++ks)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)   // k16 steps: 32 bytes into the 128-byte row
                            umma_f16(d, a_desc + (uint64_t)((ks * C::A_SUB + kk * 32) >> 4),
                                     b_desc + (uint64_t)((ks * C::B_SUB + kk * 32) >> 4), C::IDESC,
                                     ks > 0 || kk > 0);
                    // One commit: frees the A stage and tells the epilogue that the
                    // accumulator of this tile is complete.
                    umma_commit(aempty(s));
                }
                // B buffer free once both issuers' MMAs of the unit finish
                umma_commit(bempty(bb));
                ++bi;
            }
            // All MMAs issued by both threads must finish before TMEM is released (a
            // drain wait: committed MMAs complete on their own).
            umma_commit(done_bar);
            mbar_wait_drain(done_bar, 0, p.wc);
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------ epilogue
        const int e = warp - 2;                      // 0..7
        const int quarter = warp & 3;                // TMEM lanes 32*quarter .. +31
        const int half = e / 4;                      // columns 128*half .. +127
        const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16) + half * 128;
        // Head weight of column e*32+lane for a unit, read from global memory one unit
        // ahead so that its latency hides behind the previous unit's tiles.
        const int col = e * 32 + lane;
        auto unit_weight = [&](const IndexerUnit& w) {
            const int tl = col / H_I;
            return (w.tok0 + tl < w.tok_end) ? p.w[(size_t)(w.tok0 - p.t0 + tl) * H_I + (col % H_I)]
                                             : 0.f;
        };
        int bi = 0, tc = 0;
        IndexerWalk wk = walk0;
        IndexerUnit w, w_nx;
        bool have = wk.next<C::TB>(p, w_nx);
        float w_next = have ? unit_weight(w_nx) : 0.f;
        while (have) {
            w = w_nx;
            const float w_this = w_next;
            have = wk.next<C::TB>(p, w_nx);
            w_next = have ? unit_weight(w_nx) : 0.f;
            // Head weights of the unit's tokens, in column order (col = token*H_i + h).
            // One weight buffer: every epilogue warp is past the previous unit's tiles
            // before it is overwritten.
            if (bi > 0) named_barrier(1, C::EPI_WARPS * 32);
            sw[col] = 0.5f * w_this;            // halved: see epilogue_half
            named_barrier(1, C::EPI_WARPS * 32);
            const float* wh = sw + half * 128;
            // After a wait gives up this warp keeps walking the units (waits then return at
            // once) so that it still meets every named barrier of the epilogue warps.
            for (int it = 0; it < w.n_tiles; ++it, ++tc) {
                const int buf = tc & 1;
                // The tile's A-stage barrier completes when its MMAs do.
                const bool ready = mbar_wait(aempty(tc % C::A_STAGES), (tc / C::A_STAGES) & 1,
                                             p.wc, abort);
                if (!__all_sync(0xffffffffu, ready)) {           // warp-uniform skip
                    abort = true;
                    continue;
                }
                tc_fence_after();
                const int j = w.jt(it) * C::BM + quarter * 32 + lane;
                const int t_first = w.tok0 + half * (128 / H_I);
                epilogue_tile<H_I>(
                    lane_addr + buf * C::BN, wh,
                    [&] {
                        // the accumulator may be overwritten by the tile after next
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(tempty(buf));
                    },
                    [&](int tk, float score) {
                        const int t = t_first + tk;
                        // j < n_vis(t) = floor((t+1)/ratio)  <=>  ratio*(j+1) <= t+1
                        if (t < w.tok_end && p.ratio * (j + 1) <= t + 1)
                            p.scores[(size_t)(t - p.t0) * p.ld + j] = score;
                    });
            }
            ++bi;
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace ds4sp
