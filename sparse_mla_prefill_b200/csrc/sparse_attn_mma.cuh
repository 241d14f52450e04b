// Streaming sparse MLA attention: 16 heads share every gathered latent row.
//
// For token t the attended rows are the selected compressed rows (top-k, ascending
// j) followed by the raw rows max(0, t-n_swa+1) .. t; one softmax runs over all of
// them. Key = the row's 576 dims, value = its first 512 dims. "perf(ds4): extend
// sparse prefill scheduling to 10K", Summary: "keep selected raw/compressed KV
// transport in F16, and stream each selected latent row once across sixteen ...
// heads". The per-token visibility (n_vis = (t+1)/4, window bounds) is computed
// here from t; no mask is stored.
//
// Persistent CTAs (one per SM) walk their tokens heaviest first. Warp 8 is the
// producer: while it issues one token's rows it prefetches the next token's top-k
// row into shared memory (4-byte cp.async), so resolving a row never waits on global
// memory. Per 32-row block each lane resolves one row (top-k entry or window
// position), checks it, and copies its 1152 bytes into a 4-stage shared-memory ring
// with one cp.async.bulk; an mbarrier per stage counts the bytes in. It runs ahead
// across token boundaries and also fetches each token's Q. Warps 0-7 consume, with
// the 16 heads as the M of mma.sync.m16n8k16:
//   S = Q . R^T  warp w: rows 8(w%4) .. +7 of the block, dims 288(w/4) .. +287, with
//                its half of Q held in registers; the two K halves meet in shared memory;
//   softmax      per-head block max across warps, online rescaling in fp32, P to
//                shared memory as fp16;
//   O += P . V   warp w owns value dims 64w .. 64w+63 over all 32 rows of the block.
// fp32 logits, max, sums and output; probabilities enter P . V as fp16.
// Waits are bounded; a wait that gives up is turned into an abort that all consumer
// warps take together at the next named barrier, so no warp is left waiting.
#pragma once

#include "device_common.cuh"

namespace ds4sp {
namespace attn {

constexpr int H = 16;
constexpr int DQK = 576;
constexpr int DV = 512;
constexpr int ROW_BYTES = DQK * 2;           // 1152
constexpr int BR = 32;                       // rows per block
constexpr int STAGES = 4;
constexpr int CWARPS = 8;                    // consumer warps
constexpr int THREADS = (CWARPS + 1) * 32;   // + one producer warp
constexpr int ROW_PITCH = ROW_BYTES + 16;    // 1168 B: staggers ldmatrix rows over banks
constexpr int STAGE_BYTES = BR * ROW_PITCH;
constexpr int P_PITCH = (BR + 8) * 2;        // fp16 probabilities, 80 B per head
constexpr int OFF_STAGE = 0;
constexpr int OFF_Q = OFF_STAGE + STAGES * STAGE_BYTES;
constexpr int OFF_P = OFF_Q + H * ROW_PITCH;
constexpr int OFF_SX = OFF_P + H * P_PITCH;            // S partials of the upper K half
constexpr int OFF_RED_MAX = OFF_SX + 4 * 32 * 16;
constexpr int OFF_RED_SUM = OFF_RED_MAX + 4 * H * 4;
constexpr int OFF_ROWOK = OFF_RED_SUM + 4 * H * 4;
constexpr int OFF_FLAG = OFF_ROWOK + STAGES * BR * 4;
constexpr int OFF_BAR = (OFF_FLAG + 16 + 7) / 8 * 8;
constexpr int N_BARS = 2 * STAGES + 2;                 // full, empty, q_full, q_empty
constexpr int OFF_IDX = (OFF_BAR + N_BARS * 8 + 15) / 16 * 16;  // two top-k rows (int32)
constexpr int MAX_TOPK = 4096;                          // top-k rows staged in shared memory
__host__ __device__ constexpr int smem_bytes(int k) { return OFF_IDX + 2 * ((k + 3) / 4 * 4) * 4; }
constexpr int CONSUMER_BAR = 1;                        // named barrier id of warps 0-7
static_assert(DV == CWARPS * 64, "each consumer warp owns 64 value dims");
static_assert(BR == 32, "one producer lane per row");
static_assert((OFF_Q % 16) == 0 && (ROW_PITCH % 16) == 0, "bulk copies need 16-byte alignment");

}  // namespace attn

struct AttnParams {
    const __half* q;       // [n_q, 16, 576], row 0 = token t0
    const __half* kv_raw;  // [>= t0+n_q, 576]
    const __half* kv_cmp;  // [>= n_vis(t0+n_q-1), 576]
    const int32_t* topk;   // [n_q, k]
    float* out;            // [n_q, 16, 512]
    uint32_t* status;
    int t0, n_q, k, n_swa, ratio;
    float scale_log2;      // softmax scale * log2(e)
};

struct TokenRows {
    int i, t, nv, nsel, s_lo, nrows, nblk;
};

__device__ __forceinline__ TokenRows token_rows(const AttnParams& p, int idx) {
    TokenRows r;
    r.i = p.n_q - 1 - idx;                        // heaviest (latest) tokens first
    r.t = p.t0 + r.i;
    r.nv = n_vis(r.t, p.ratio);
    r.nsel = min(p.k, r.nv);
    r.s_lo = max(0, r.t - p.n_swa + 1);
    r.nrows = r.nsel + (r.t - r.s_lo + 1);
    r.nblk = (r.nrows + attn::BR - 1) / attn::BR;
    return r;
}

__global__ void __launch_bounds__(attn::THREADS, 1) sparse_attn_mma_kernel(AttnParams p) {
    using namespace attn;
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    float* red_max = reinterpret_cast<float*>(smem + OFF_RED_MAX);
    float* red_sum = reinterpret_cast<float*>(smem + OFF_RED_SUM);
    int* rowok = reinterpret_cast<int*>(smem + OFF_ROWOK);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_FLAG);
    const uint32_t bar0 = sbase + OFF_BAR;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (STAGES + s); };
    const uint32_t qfull_bar = bar0 + 8u * (2 * STAGES);
    const uint32_t qempty_bar = bar0 + 8u * (2 * STAGES + 1);

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    if (tid == 0) {
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), CWARPS);
        }
        mbar_init(qfull_bar, 1);
        mbar_init(qempty_bar, CWARPS);
        *abort_flag = 0;
        fence_mbar_init();
    }
    __syncthreads();

    bool abort = false;
    if (warp == CWARPS) {
        // ------------------------------------------------------------ producer
        int it = 0, ntok = 0;
        int issued[STAGES] = {};
        bool q_issued = false;
        const int kpad = (p.k + 3) / 4 * 4;
        int* sidx = reinterpret_cast<int*>(smem + OFF_IDX);
        // Stage the selected entries of a token's top-k row in buffer `buf`.
        auto prefetch_idx = [&](int idx, int buf) {
            if (idx < p.n_q) {
                const TokenRows nx = token_rows(p, idx);
                const int32_t* src = p.topk + (size_t)nx.i * p.k;
                const uint32_t dst = sbase + OFF_IDX + buf * kpad * 4;
                for (int g = lane; g < nx.nsel; g += 32)
                    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst + 4 * g),
                                 "l"(src + g)
                                 : "memory");
            }
            cp_async_commit();
        };
        prefetch_idx(blockIdx.x, 0);
        for (int idx = blockIdx.x; idx < p.n_q && !abort; idx += gridDim.x, ++ntok) {
            const TokenRows tr = token_rows(p, idx);
            cp_async_wait<0>();                   // this token's top-k row is in shared memory
            __syncwarp();
            const int* tk = sidx + (ntok & 1) * kpad;
            prefetch_idx(idx + gridDim.x, (ntok + 1) & 1);   // lands while this token streams
            if (!__all_sync(0xffffffffu, mbar_wait(qempty_bar, (ntok & 1) ^ 1, p.status, abort))) {
                abort = true;                      // warp-uniform from here on
                break;
            }
            if (lane == 0) mbar_arrive_expect_tx(qfull_bar, H * ROW_BYTES);
            __syncwarp();
            if (lane < H)
                bulk_load(sbase + OFF_Q + lane * ROW_PITCH, p.q + ((size_t)tr.i * H + lane) * DQK,
                          ROW_BYTES, qfull_bar);
            q_issued = true;
            for (int blk = 0; blk < tr.nblk; ++blk, ++it) {
                const int s = it % STAGES;
                // Resolve this lane's row before waiting for the stage to free up.
                const int gr = blk * BR + lane;
                const __half* src = p.kv_raw + (size_t)tr.t * DQK;   // harmless stand-in
                int ok = 0;
                if (gr < tr.nsel) {
                    const int j = tk[gr];
                    if (j >= 0 && j < tr.nv) {
                        src = p.kv_cmp + (size_t)j * DQK;
                        ok = 1;
                    } else {
                        record_status(p.status, kStatusBounds);
                    }
                } else if (gr < tr.nrows) {
                    src = p.kv_raw + (size_t)(tr.s_lo + gr - tr.nsel) * DQK;
                    ok = 1;
                }
                if (!__all_sync(0xffffffffu,
                                mbar_wait(empty_bar(s), ((it / STAGES) & 1) ^ 1, p.status, abort))) {
                    abort = true;
                    break;
                }
                rowok[s * BR + lane] = ok;
                __syncwarp();
                if (lane == 0) mbar_arrive_expect_tx(full_bar(s), BR * ROW_BYTES);
                __syncwarp();
                bulk_load(sbase + OFF_STAGE + s * STAGE_BYTES + lane * ROW_PITCH, src, ROW_BYTES,
                          full_bar(s));
                ++issued[s];
            }
        }
        // Every copy started here must land before the CTA exits.
        cp_async_wait<0>();
        bool drain_abort = false;
        if (q_issued) mbar_wait(qfull_bar, (ntok - 1) & 1, p.status, drain_abort);
        for (int s = 0; s < STAGES; ++s) {
            drain_abort = false;
            if (issued[s]) mbar_wait(full_bar(s), (issued[s] - 1) & 1, p.status, drain_abort);
        }
    } else {
        // ------------------------------------------------------------ consumers
        const int g = lane / 4, c = lane % 4;     // mma fragment coordinates
        const int nt = warp & 3, kh = warp >> 2;  // S: n-tile (8 rows) and K half
        int it = 0, ntok = 0;
        for (int idx = blockIdx.x; idx < p.n_q; idx += gridDim.x, ++ntok) {
            const TokenRows tr = token_rows(p, idx);
            if (!mbar_wait(qfull_bar, ntok & 1, p.status, abort)) *abort_flag = 1;
            uint32_t qf[18][4];                   // this warp's K half of Q as A fragments
            {
                const int r = (lane & 7) + ((lane >> 3) & 1) * 8, kc = (lane >> 4) * 8;
#pragma unroll
                for (int kk = 0; kk < 18; ++kk)
                    ldsm_x4(sbase + OFF_Q + r * ROW_PITCH + ((18 * kh + kk) * 16 + kc) * 2,
                            qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3]);
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(qempty_bar);

            float o[8][4];
#pragma unroll
            for (int n = 0; n < 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
            float m_g = -INFINITY, m_g8 = -INFINITY;   // running max, heads g and g+8 (log2 units)
            float l_g = 0.f, l_g8 = 0.f;               // partial sums (K-half-0 warps only)

            for (int blk = 0; blk < tr.nblk; ++blk, ++it) {
                const int s = it % STAGES;
                if (!mbar_wait(full_bar(s), (it / STAGES) & 1, p.status, abort)) *abort_flag = 1;
                const uint32_t stage = sbase + OFF_STAGE + s * STAGE_BYTES;

                // ---- S partial over this warp's K half, two accumulator chains
                float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
                {
                    const uint32_t rowaddr = stage + (8 * nt + (lane & 7)) * ROW_PITCH +
                                             (lane >> 3) * 16 + kh * (ROW_BYTES / 2);
#pragma unroll
                    for (int k2 = 0; k2 < 9; ++k2) {
                        uint32_t b0, b1, b2, b3;
                        ldsm_x4(rowaddr + k2 * 64, b0, b1, b2, b3);
                        if (k2 & 1) {
                            mma_16816(a1, qf[2 * k2], b0, b1);
                            mma_16816(a1, qf[2 * k2 + 1], b2, b3);
                        } else {
                            mma_16816(a0, qf[2 * k2], b0, b1);
                            mma_16816(a0, qf[2 * k2 + 1], b2, b3);
                        }
                    }
                }
                float sv[4] = {a0[0] + a1[0], a0[1] + a1[1], a0[2] + a1[2], a0[3] + a1[3]};
                float4* sx = reinterpret_cast<float4*>(smem + OFF_SX) + nt * 32 + lane;
                if (kh == 1) *sx = make_float4(sv[0], sv[1], sv[2], sv[3]);
                named_barrier(CONSUMER_BAR, CWARPS * 32);
                if (*abort_flag) break;            // every consumer warp sees the same flag here

                const int r0 = 8 * nt + 2 * c;
                if (kh == 0) {
                    const float4 up = *sx;
                    const bool ok0 = rowok[s * BR + r0] != 0, ok1 = rowok[s * BR + r0 + 1] != 0;
                    sv[0] = ok0 ? (sv[0] + up.x) * p.scale_log2 : -INFINITY;
                    sv[1] = ok1 ? (sv[1] + up.y) * p.scale_log2 : -INFINITY;
                    sv[2] = ok0 ? (sv[2] + up.z) * p.scale_log2 : -INFINITY;
                    sv[3] = ok1 ? (sv[3] + up.w) * p.scale_log2 : -INFINITY;
                    float mx_g = fmaxf(sv[0], sv[1]), mx_g8 = fmaxf(sv[2], sv[3]);
#pragma unroll
                    for (int off = 1; off <= 2; off <<= 1) {
                        mx_g = fmaxf(mx_g, __shfl_xor_sync(0xffffffffu, mx_g, off));
                        mx_g8 = fmaxf(mx_g8, __shfl_xor_sync(0xffffffffu, mx_g8, off));
                    }
                    if (c == 0) {
                        red_max[nt * H + g] = mx_g;
                        red_max[nt * H + g + 8] = mx_g8;
                    }
                }
                named_barrier(CONSUMER_BAR, CWARPS * 32);

                // ---- online softmax (every warp derives the same running max)
                float bm_g = fmaxf(fmaxf(red_max[g], red_max[H + g]),
                                   fmaxf(red_max[2 * H + g], red_max[3 * H + g]));
                float bm_g8 = fmaxf(fmaxf(red_max[g + 8], red_max[H + g + 8]),
                                    fmaxf(red_max[2 * H + g + 8], red_max[3 * H + g + 8]));
                const float mn_g = fmaxf(m_g, bm_g), mn_g8 = fmaxf(m_g8, bm_g8);
                const float ref_g = mn_g == -INFINITY ? 0.f : mn_g;
                const float ref_g8 = mn_g8 == -INFINITY ? 0.f : mn_g8;
                const float alpha_g = fast_exp2(m_g - ref_g), alpha_g8 = fast_exp2(m_g8 - ref_g8);
                m_g = mn_g;
                m_g8 = mn_g8;
                if (kh == 0) {
                    const float p0 = fast_exp2(sv[0] - ref_g), p1 = fast_exp2(sv[1] - ref_g);
                    const float p2 = fast_exp2(sv[2] - ref_g8), p3 = fast_exp2(sv[3] - ref_g8);
                    l_g = l_g * alpha_g + p0 + p1;
                    l_g8 = l_g8 * alpha_g8 + p2 + p3;
                    uint8_t* pb = smem + OFF_P;
                    *reinterpret_cast<uint32_t*>(pb + g * P_PITCH + r0 * 2) = pack_half2(p0, p1);
                    *reinterpret_cast<uint32_t*>(pb + (g + 8) * P_PITCH + r0 * 2) = pack_half2(p2, p3);
                }
                named_barrier(CONSUMER_BAR, CWARPS * 32);

                // ---- O = alpha * O + P . V over value dims 64w .. 64w+63
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    o[n][0] *= alpha_g;
                    o[n][1] *= alpha_g;
                    o[n][2] *= alpha_g8;
                    o[n][3] *= alpha_g8;
                }
                {
                    const int ar = (lane & 7) + ((lane >> 3) & 1) * 8, hi = (lane >> 4) * 8;
#pragma unroll
                    for (int ks = 0; ks < BR / 16; ++ks) {
                        uint32_t a[4];
                        ldsm_x4(sbase + OFF_P + ar * P_PITCH + (ks * 16 + hi) * 2, a[0], a[1], a[2], a[3]);
                        const uint32_t vrow = stage + (ks * 16 + ar) * ROW_PITCH + (64 * warp + hi) * 2;
#pragma unroll
                        for (int np = 0; np < 4; ++np) {
                            uint32_t b0, b1, b2, b3;
                            ldsm_x4_trans(vrow + np * 32, b0, b1, b2, b3);
                            mma_16816(o[2 * np], a, b0, b1);
                            mma_16816(o[2 * np + 1], a, b2, b3);
                        }
                    }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_bar(s));
            }
            if (*abort_flag) break;

            // ---- normalise and store
            if (kh == 0) {
#pragma unroll
                for (int off = 1; off <= 2; off <<= 1) {
                    l_g += __shfl_xor_sync(0xffffffffu, l_g, off);
                    l_g8 += __shfl_xor_sync(0xffffffffu, l_g8, off);
                }
                if (c == 0) {
                    red_sum[nt * H + g] = l_g;
                    red_sum[nt * H + g + 8] = l_g8;
                }
            }
            named_barrier(CONSUMER_BAR, CWARPS * 32);
            const float L_g = red_sum[g] + red_sum[H + g] + red_sum[2 * H + g] + red_sum[3 * H + g];
            const float L_g8 = red_sum[g + 8] + red_sum[H + g + 8] + red_sum[2 * H + g + 8] +
                               red_sum[3 * H + g + 8];
            named_barrier(CONSUMER_BAR, CWARPS * 32);   // red_sum is rewritten by the next token
            const float inv_g = L_g > 0.f ? 1.f / L_g : 0.f;
            const float inv_g8 = L_g8 > 0.f ? 1.f / L_g8 : 0.f;
            float* ot = p.out + (size_t)tr.i * H * DV;
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                const int d = 64 * warp + 8 * n + 2 * c;
                *reinterpret_cast<float2*>(ot + g * DV + d) = make_float2(o[n][0] * inv_g, o[n][1] * inv_g);
                *reinterpret_cast<float2*>(ot + (g + 8) * DV + d) =
                    make_float2(o[n][2] * inv_g8, o[n][3] * inv_g8);
            }
        }
    }
    __syncthreads();
}

}  // namespace ds4sp
