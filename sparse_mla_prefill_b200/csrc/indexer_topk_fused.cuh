// Indexer and top-k in one kernel: the scores never leave the SM.
//
// Same scores as indexer_tcgen05_kernel -- score(t, j) = sum_h w[t,h] *
// ReLU(q_idx[t,h,:] . k_idx[j,:]) for the rows j visible to t (4j+3 <= t), computed as
// D[j, (t,h)] tiles on the tensor cores with the ReLU and the head-weighted sum in the
// epilogue -- and the same selection as topk_radix_kernel: the min(k, n_vis(t)) largest
// scores, equal scores to the lower j, listed by ascending j, then -1. The pages hand
// the long-prefill top-k rows straight to attention ("pass authoritative long-prefill
// top-k rows directly", "perf(ds4): extend sparse prefill scheduling to 10K", Summary;
// "direct long-prefill top-k handoff", "perf(ds4): unify gfx1151 sparse-prefill stack",
// Composition); here the handoff goes one step further and the score rows themselves
// are never written to global memory.
//
// Work: a unit is one whole token block (256/H_i tokens) with all the 128-row j-tiles
// its last token needs, so a CTA ends a unit holding complete score rows. The host
// assigns the launch's token blocks to the persistent CTAs by longest-processing-time
// on their cost (tiles, plus the select), heaviest first.
// Per unit: the epilogue warps turn each tile's accumulator into order-preserving keys
// of the scores (the top-k kernel's mapping) in one of two shared-memory key buffers
// [tokens of the block][128 x tiles]; when the unit's last tile is done they hand the
// buffer to eight select warps and go on with the next unit's tiles. The select warps
// run the radix select of topk_radix.cuh, four groups of two warps on four tokens at
// once (each group with its own named barrier), write the tokens' indices and hand the
// buffer back. So the select of one unit overlaps the tensor-core work of the next.
// Warps: 0 streams k_idx tiles (TMA), 1 owns TMEM and issues the MMAs, 2 loads q_idx
// blocks into the single B buffer as soon as the previous unit's MMAs have read it, 3 is
// idle, 4-11 run the epilogue, 12-19 the select. setmaxnreg gives the epilogue warps
// most of the registers. Every wait is bounded (device_common.cuh).
#pragma once

#include <cuda.h>

#include "device_common.cuh"
#include "indexer_tcgen05.cuh"
#include "topk_radix.cuh"

namespace ds4sp {

template <int D_I, int H_I>
struct FusedTile {
    using T = IndexerTile<D_I, H_I>;
    static constexpr int BM = T::BM, BN = T::BN, TB = T::TB, KSUB = T::KSUB;
    static constexpr int A_SUB = T::A_SUB, A_STAGE = T::A_STAGE, B_SUB = T::B_SUB;
    static constexpr int B_BYTES = T::B_BYTES;
    static constexpr int A_STAGES = KSUB == 2 ? 2 : 4;           // k_idx ring
    static constexpr int A_WARP = 0, MMA_WARP = 1, B_WARP = 2;
    static constexpr int EPI_WARP0 = 4, EPI_WARPS = 8, EPI_THREADS = EPI_WARPS * 32;
    static constexpr int SEL_WARP0 = 12, SEL_WARPS = 8, SEL_ALL = SEL_WARPS * 32;
    static constexpr int THREADS = (SEL_WARP0 + SEL_WARPS) * 32;  // 640
    // Registers per thread: the launch's (THREADS x LAUNCH_REGS) is split by setmaxnreg
    // between the warpgroups; the host checks the built count before the first launch.
    static constexpr int LAUNCH_REGS = 96, CTRL_REGS = 40, EPI_REGS = 152, SEL_REGS = 64;
    static_assert(4 * 32 * CTRL_REGS + EPI_THREADS * EPI_REGS + SEL_ALL * SEL_REGS <=
                      THREADS * LAUNCH_REGS, "register split must fit the launch's registers");
    static constexpr int TMEM_COLS = 2 * BN;
    static constexpr int KEY_BYTES = 40 * 1024;                   // one of two key buffers
    static constexpr int OFF_B = 0;                               // one B buffer
    static constexpr int OFF_A = B_BYTES;
    static constexpr int OFF_KEYS = OFF_A + A_STAGES * A_STAGE;
    static constexpr int OFF_W = OFF_KEYS + 2 * KEY_BYTES;        // two w buffers
    static constexpr int OFF_SEL = OFF_W + 2 * BN * 4;            // select scratch
    // Per select group: hist[256], w_or/w_and/w_cnt[2], s_digit, s_above, warp_tot[2]
    // (8-byte aligned); after the groups, the abort flag.
    static constexpr int SEL_GROUPS = 4, SEL_THREADS = SEL_ALL / SEL_GROUPS;
    static constexpr int GROUP_SEL = 256 * 4 + 3 * 2 * 4 + 2 * 4 + 2 * 8;
    static constexpr int SEL_ABORT = SEL_GROUPS * GROUP_SEL;      // byte offset of the flag
    static constexpr int SEL_BYTES = SEL_ABORT + 16;
    static constexpr int OFF_BAR = OFF_SEL + SEL_BYTES;
    // afull[A_STAGES], aempty[A_STAGES], bfull, bempty, tempty[2], kfull[2], kempty[2], done
    static constexpr int N_BARS = 2 * A_STAGES + 1 + 1 + 2 + 2 + 2 + 1;
    static constexpr int OFF_TMEM_PTR = OFF_BAR + N_BARS * 8;
    static constexpr int SMEM_BYTES = OFF_TMEM_PTR + 16 + 1024;   // + alignment slack
    static constexpr uint32_t IDESC = T::IDESC;
    static constexpr int EPI_BAR = 1, SEL_BAR = 6;                // named barriers (2-5: groups)
    static_assert(GROUP_SEL % 8 == 0 && OFF_SEL % 8 == 0, "8-byte aligned select scratch");
    static_assert(SEL_THREADS == 64, "two warps per select group");
    static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
};

constexpr int kFusedMaxBlocks = 1024;     // token blocks of one launch

struct FusedParams {
    const float* w;        // [n_q, H_i] fp32, row 0 = token t0
    int32_t* topk;         // [n_q, k] int32 output, row 0 = token t0
    WaitCtl wc;
    int t0, n_q, k, ratio;
    int kld;               // key row stride (128 x the launch's largest tile count)
    // CTA b processes token blocks blk[first[b]] .. blk[first[b+1]-1], in that order.
    uint16_t first[kIndexerMaxGrid + 1];
    uint16_t blk[kFusedMaxBlocks];
};

// Named barrier of one select group: two select warps, barrier id 2 + group.
struct GroupSync {
    int id;
    __device__ __forceinline__ void operator()() const { named_barrier(id, 64); }
};

// Top-k of one token's key row (n candidates, n > k) by one select group of 64 threads:
// the radix select and compaction of topk_radix_kernel on keys already in shared memory.
// `sel` is the group's scratch; `tid` the thread's index in the group.
__device__ __forceinline__ void fused_select_row(const uint32_t* keys, int n, int k, int32_t* out,
                                                 uint8_t* sel, int tid, GroupSync sync) {
    constexpr int NT = 64;
    uint32_t* hist = reinterpret_cast<uint32_t*>(sel);
    uint32_t* w_or = hist + 256;
    uint32_t* w_and = w_or + 2;
    uint32_t* w_cnt = w_and + 2;
    uint32_t* s_digit = w_cnt + 2;
    uint32_t* s_above = s_digit + 1;
    unsigned long long* warp_tot = reinterpret_cast<unsigned long long*>(s_above + 1);
    // Keys four at a time (the row is 16-byte aligned with room to a multiple of 128
    // keys); j >= n holds stale keys of an earlier unit, read as 0 (no candidate).
    const int n4 = (n + 3) / 4;
    auto group = [&](int x) {
        uint4 kk = reinterpret_cast<const uint4*>(keys)[x];
        const int j = 4 * x;
        if (j + 1 >= n) kk.y = 0u;
        if (j + 2 >= n) kk.z = 0u;
        if (j + 3 >= n) kk.w = 0u;
        return kk;
    };
    uint32_t kor = 0u, kand = 0xffffffffu, cand = 0u;
    for (int x = tid; x < n4; x += NT) {
        const uint4 kk = group(x);
        const uint32_t q[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
        for (int c = 0; c < 4; ++c)
            if (q[c]) {
                kor |= q[c];
                kand &= q[c];
                ++cand;
            }
    }
    uint32_t all_or, all_and, n_cand;
    block_key_stats<NT>(kor, kand, cand, w_or, w_and, w_cnt, all_or, all_and, n_cand, tid, sync);
    RadixSelect<GroupSync> rs(all_or, all_and, (uint32_t)k, tid, sync);
    while (rs.active) {
        rs.clear(hist, NT);
        for (int x = tid; x < n4; x += NT) {
            const uint4 kk = group(x);
            const uint32_t q[4] = {kk.x, kk.y, kk.z, kk.w};
#pragma unroll
            for (int c = 0; c < 4; ++c)
                if (q[c] != 0u && (q[c] & rs.digits) == rs.prefix)
                    atomicAdd(&hist[(q[c] >> rs.shift) & 255u], 1u);
        }
        rs.step(hist, s_digit, s_above);
    }
    const uint32_t thr = rs.thr, need = rs.need;
    const int per = (n4 + NT - 1) / NT;
    const int xb = min(n4, tid * per), xe = min(n4, xb + per);
    uint32_t gt = 0, eq = 0;
    for (int x = xb; x < xe; ++x) {
        const uint4 kk = group(x);
        gt += (kk.x > thr) + (kk.y > thr) + (kk.z > thr) + (kk.w > thr);
        eq += (kk.x == thr) + (kk.y == thr) + (kk.z == thr) + (kk.w == thr);
    }
    const unsigned long long before =
        block_exclusive_scan<NT>(((unsigned long long)gt << 32) | eq, warp_tot, tid, sync);
    const uint32_t gt_before = (uint32_t)(before >> 32), eq_before = (uint32_t)before;
    uint32_t pos = gt_before + min(eq_before, need), eq_rank = eq_before;
    for (int x = xb; x < xe; ++x) {
        const uint4 kk = group(x);
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
    // exactly k entries were written (n > k); the scratch is reused by the next row
    sync();
}

template <int D_I, int H_I>
__global__ void __launch_bounds__(FusedTile<D_I, H_I>::THREADS, 1)
indexer_topk_fused_kernel(const __grid_constant__ CUtensorMap tmap_k,
                          const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ FusedParams p) {
    using C = FusedTile<D_I, H_I>;
    const int b = blockIdx.x;
    const int u_begin = p.first[b], u_end = p.first[b + 1];

    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t base = (raw_u32 + 1023u) & ~1023u;         // 128B-swizzle atoms need 1 KB alignment
    uint8_t* smem = smem_raw + (base - raw_u32);
    auto keys_of = [&](int ui) {
        return reinterpret_cast<uint32_t*>(smem + C::OFF_KEYS + (ui & 1) * C::KEY_BYTES);
    };
    float* sw = reinterpret_cast<float*>(smem + C::OFF_W);
    uint8_t* sel = smem + C::OFF_SEL;
    volatile uint32_t* sel_abort = reinterpret_cast<volatile uint32_t*>(sel + C::SEL_ABORT);
    const uint32_t bar0 = base + C::OFF_BAR;
    auto afull = [&](int s) { return bar0 + 8u * s; };
    auto aempty = [&](int s) { return bar0 + 8u * (C::A_STAGES + s); };
    const uint32_t bfull = bar0 + 8u * (2 * C::A_STAGES);
    const uint32_t bempty = bar0 + 8u * (2 * C::A_STAGES + 1);
    auto tempty = [&](int i) { return bar0 + 8u * (2 * C::A_STAGES + 2 + i); };
    auto kfull = [&](int i) { return bar0 + 8u * (2 * C::A_STAGES + 4 + i); };
    auto kempty = [&](int i) { return bar0 + 8u * (2 * C::A_STAGES + 6 + i); };
    const uint32_t done_bar = bar0 + 8u * (2 * C::A_STAGES + 8);
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + C::OFF_TMEM_PTR);

    // Token block tb of the launch: tokens [tok0, tok_end), j-tiles 0 .. n_tiles-1.
    auto unit_of = [&](int u, int& tok0, int& tok_end, int& n_tiles) {
        const int tb = p.blk[u];
        tok0 = p.t0 + tb * C::TB;
        tok_end = min(tok0 + C::TB, p.t0 + p.n_q);
        n_tiles = (n_vis(tok_end - 1, p.ratio) + C::BM - 1) / C::BM;
    };

    const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
    if (threadIdx.x == 0) {
        for (int s = 0; s < C::A_STAGES; ++s) {
            mbar_init(afull(s), 1);
            mbar_init(aempty(s), 1);
        }
        mbar_init(bfull, 1);
        mbar_init(bempty, 1);
        for (int i = 0; i < 2; ++i) {
            mbar_init(tempty(i), C::EPI_WARPS);
            mbar_init(kfull(i), C::EPI_WARPS);     // the epilogue warps hand a key buffer over
            mbar_init(kempty(i), C::SEL_WARPS);    // the select warps hand it back
        }
        mbar_init(done_bar, 1);
        *sel_abort = 0u;
        fence_mbar_init();
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_q);
    }
    if (warp == C::MMA_WARP) {
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

    bool abort = false;
    if (warp < C::EPI_WARP0) {
        regs_decrease<C::CTRL_REGS>();
        if (warp == C::B_WARP && lane == 0) {
            // ------------------------------------------------------------ q_idx loader
            int issued = 0;
            for (int u = u_begin; u < u_end && !abort; ++u) {
                int tok0, tok_end, n_tiles;
                unit_of(u, tok0, tok_end, n_tiles);
                // the single B buffer is free once the previous unit's MMAs have read it
                if (!mbar_wait(bempty, ((u - u_begin) & 1) ^ 1, p.wc, abort)) break;
                mbar_arrive_expect_tx(bfull, C::B_BYTES);
                for (int ks = 0; ks < C::KSUB; ++ks)
                    tma_load_2d(base + C::OFF_B + ks * C::B_SUB, &tmap_q, bfull, ks * 64,
                                (tok0 - p.t0) * H_I);
                ++issued;
            }
            // Every bulk copy this CTA started must land before the CTA exits.
            if (issued) mbar_wait_drain(bfull, (issued - 1) & 1, p.wc);
        } else if (warp == C::A_WARP && lane == 0) {
            // ------------------------------------------------------------ k_idx loader
            int a_it = 0;
            int a_issued[C::A_STAGES] = {};
            for (int u = u_begin; u < u_end && !abort; ++u) {
                int tok0, tok_end, n_tiles;
                unit_of(u, tok0, tok_end, n_tiles);
                for (int it = 0; it < n_tiles; ++it, ++a_it) {
                    const int s = a_it % C::A_STAGES;
                    if (!mbar_wait(aempty(s), ((a_it / C::A_STAGES) & 1) ^ 1, p.wc, abort)) break;
                    mbar_arrive_expect_tx(afull(s), C::A_STAGE);
#pragma unroll
                    for (int ks = 0; ks < C::KSUB; ++ks)
                        tma_load_2d(base + C::OFF_A + s * C::A_STAGE + ks * C::A_SUB, &tmap_k,
                                    afull(s), ks * 64, it * C::BM);
                    ++a_issued[s];
                }
            }
            for (int s = 0; s < C::A_STAGES; ++s)
                if (a_issued[s]) mbar_wait_drain(afull(s), (a_issued[s] - 1) & 1, p.wc);
        } else if (warp == C::MMA_WARP && lane == 0) {
            // ------------------------------------------------------------ MMA issuer
            const uint64_t a_desc0 = umma_desc_sw128(base + C::OFF_A);
            const uint64_t b_desc = umma_desc_sw128(base + C::OFF_B);
            int tc = 0;
            for (int u = u_begin; u < u_end && !abort; ++u) {
                int tok0, tok_end, n_tiles;
                unit_of(u, tok0, tok_end, n_tiles);
                if (!mbar_wait(bfull, (u - u_begin) & 1, p.wc, abort)) break;
                for (int it = 0; it < n_tiles; ++it, ++tc) {
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
                            umma_f16(d, a_desc + (uint64_t)((ks * C::A_SUB + kk * 32) >> 4),
                                     b_desc + (uint64_t)((ks * C::B_SUB + kk * 32) >> 4), C::IDESC,
                                     ks > 0 || kk > 0);
                    umma_commit(aempty(s));      // frees the A stage; the accumulator is final
                }
                umma_commit(bempty);             // B free once the unit's MMAs finish
            }
            umma_commit(done_bar);
            mbar_wait_drain(done_bar, 0, p.wc);
        }
        __syncwarp();
    } else if (warp < C::SEL_WARP0) {
        // ------------------------------------------------------------ epilogue
        regs_increase<C::EPI_REGS>();
        const int e = warp - C::EPI_WARP0;           // 0..7
        const int quarter = warp & 3;                // TMEM lanes 32*quarter .. +31
        const int half = e / 4;                      // columns 128*half .. +127
        const uint32_t lane_addr = tmem_base + ((uint32_t)(quarter * 32) << 16) + half * 128;
        const int col = e * 32 + lane;
        auto unit_weight = [&](int u) {
            int tok0, tok_end, n_tiles;
            unit_of(u, tok0, tok_end, n_tiles);
            const int tl = col / H_I;
            return (tok0 + tl < tok_end) ? p.w[(size_t)(tok0 - p.t0 + tl) * H_I + (col % H_I)] : 0.f;
        };
        int tc = 0;
        float w_next = u_begin < u_end ? unit_weight(u_begin) : 0.f;
        for (int u = u_begin; u < u_end; ++u) {
            const int ui = u - u_begin;
            int tok0, tok_end, n_tiles;
            unit_of(u, tok0, tok_end, n_tiles);
            const float w_this = w_next;
            w_next = u + 1 < u_end ? unit_weight(u + 1) : 0.f;
            float* swb = sw + (ui & 1) * C::BN;
            swb[col] = 0.5f * w_this;                // halved: see epilogue_half
            named_barrier(C::EPI_BAR, C::EPI_THREADS);
            const float* wh = swb + half * 128;
            uint32_t* keys = keys_of(ui);
            // this key buffer's previous unit (ui - 2) must be selected before it is rewritten
            if (!__all_sync(0xffffffffu, mbar_wait(kempty(ui & 1), ((ui >> 1) & 1) ^ 1, p.wc, abort))) {
                abort = true;
                *sel_abort = 1u;
            }
            for (int it = 0; it < n_tiles; ++it, ++tc) {
                const int buf = tc & 1;
                const bool ready = mbar_wait(aempty(tc % C::A_STAGES), (tc / C::A_STAGES) & 1,
                                             p.wc, abort);
                if (!__all_sync(0xffffffffu, ready)) {           // warp-uniform skip
                    abort = true;
                    *sel_abort = 1u;
                    continue;
                }
                tc_fence_after();
                const int j = it * C::BM + quarter * 32 + lane;
                const int tl_first = half * (128 / H_I);
                epilogue_tile<H_I>(
                    lane_addr + buf * C::BN, wh,
                    [&] {
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(tempty(buf));
                    },
                    [&](int tk, float score) {
                        const int tl = tl_first + tk, t = tok0 + tl;
                        if (t < tok_end && p.ratio * (j + 1) <= t + 1)
                            keys[tl * p.kld + j] = order_key(score);
                    });
            }
            // hand the unit's keys to the select warps (also after a give-up, so that they
            // are not left waiting; they read the abort flag first)
            __syncwarp();
            if (lane == 0) mbar_arrive(kfull(ui & 1));
        }
    } else {
        // ------------------------------------------------------------ select
        regs_decrease<C::SEL_REGS>();
        const int stid = threadIdx.x - C::SEL_WARP0 * 32;   // 0..255
        const int g = stid / C::SEL_THREADS, gtid = stid % C::SEL_THREADS;
        for (int u = u_begin; u < u_end; ++u) {
            const int ui = u - u_begin;
            int tok0, tok_end, n_tiles;
            unit_of(u, tok0, tok_end, n_tiles);
            const bool ready = mbar_wait(kfull(ui & 1), (ui >> 1) & 1, p.wc, abort);
            // The epilogue may raise the flag at any time: one reduction gives every select
            // warp the same answer, so that none is left alone at a group barrier.
            if (named_barrier_or(C::SEL_BAR, C::SEL_ALL, !ready || *sel_abort != 0u)) break;
            const uint32_t* keys = keys_of(ui);
            // The block's tokens, one per select group at a time (the groups run at once).
            for (int tl = g; tl < tok_end - tok0; tl += C::SEL_GROUPS) {
                const int t = tok0 + tl, n = n_vis(t, p.ratio);
                int32_t* out = p.topk + (size_t)(t - p.t0) * p.k;
                if (n <= p.k) {                     // every visible row is kept
                    for (int s = gtid; s < p.k; s += C::SEL_THREADS) out[s] = s < n ? s : -1;
                    continue;
                }
                fused_select_row(keys + tl * p.kld, n, p.k, out, sel + g * C::GROUP_SEL, gtid,
                                 GroupSync{2 + g});
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(kempty(ui & 1));     // the buffer may be rewritten
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == C::MMA_WARP) tmem_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace ds4sp
