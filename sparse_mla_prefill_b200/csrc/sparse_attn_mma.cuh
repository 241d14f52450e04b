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
// One CTA (8 warps) per token. Rows stream through shared memory in blocks of 64,
// gathered with 16-byte cp.async (two stages). The 16 heads are the M of
// mma.sync.m16n8k16:
//   S = Q . R^T  warp w computes the 8 rows 8w..8w+7 of the block over all 576 dims,
//                with Q held in registers as A fragments;
//   softmax      block max per head across warps through shared memory, online
//                rescaling in fp32, probabilities to shared memory as fp16;
//   O += P . V   warp w owns value dims 64w .. 64w+63 and reads P for all 64 rows.
// fp32 logits, max, sums and output; probabilities enter P . V as fp16.
#pragma once

#include "device_common.cuh"

namespace ds4sp {
namespace attn {

constexpr int H = 16;
constexpr int DQK = 576;
constexpr int DV = 512;
constexpr int BR = 64;                       // rows per block
constexpr int WARPS = 8;
constexpr int THREADS = WARPS * 32;
constexpr int ROW_PITCH = DQK * 2 + 16;      // 1168 B: staggers ldmatrix rows over banks
constexpr int CHUNKS = DQK * 2 / 16;         // 72 sixteen-byte chunks per row
constexpr int STAGES = 2;
constexpr int STAGE_BYTES = BR * ROW_PITCH;
constexpr int P_PITCH = (BR + 8) * 2;        // fp16 probabilities, 144 B per head
constexpr int OFF_STAGE = 0;
constexpr int OFF_Q = OFF_STAGE + STAGES * STAGE_BYTES;
constexpr int OFF_P = OFF_Q + H * ROW_PITCH;
constexpr int OFF_RED_MAX = OFF_P + H * P_PITCH;
constexpr int OFF_RED_SUM = OFF_RED_MAX + WARPS * H * 4;
constexpr int OFF_ROWOK = OFF_RED_SUM + WARPS * H * 4;
constexpr int SMEM_BYTES = OFF_ROWOK + STAGES * BR * 4;
static_assert(DV == WARPS * 64, "each warp owns 64 value dims");
static_assert(CHUNKS * 16 == DQK * 2, "row is a whole number of 16-byte chunks");

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

__global__ void __launch_bounds__(attn::THREADS, 1) sparse_attn_mma_kernel(AttnParams p) {
    using namespace attn;
    extern __shared__ __align__(16) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    float* red_max = reinterpret_cast<float*>(smem + OFF_RED_MAX);
    float* red_sum = reinterpret_cast<float*>(smem + OFF_RED_SUM);
    int* rowok = reinterpret_cast<int*>(smem + OFF_ROWOK);

    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int g = lane / 4, c = lane % 4;        // mma fragment coordinates

    const int i = p.n_q - 1 - (int)blockIdx.x;   // heavier (later) tokens first
    const int t = p.t0 + i;
    const int nv = n_vis(t, p.ratio);
    const int nsel = min(p.k, nv);
    const int s_lo = max(0, t - p.n_swa + 1);
    const int nrows = nsel + (t - s_lo + 1);
    const int nblk = (nrows + BR - 1) / BR;
    const int32_t* tk = p.topk + (size_t)i * p.k;

    // Loader mapping: 4 threads per row, 18 chunks each.
    const int ld_row = tid / 4, ld_part = tid % 4;
    auto issue_block = [&](int blk, int st) {
        const int gr = blk * BR + ld_row;
        const __half* src = p.kv_raw;
        bool ok = false;
        if (gr < nsel) {
            const int j = tk[gr];
            if (j >= 0 && j < nv) {
                src = p.kv_cmp + (size_t)j * DQK;
                ok = true;
            } else if (ld_part == 0) {
                record_status(p.status, kStatusBounds);
            }
        } else if (gr < nrows) {
            src = p.kv_raw + (size_t)(s_lo + gr - nsel) * DQK;
            ok = true;
        }
        const uint32_t dst = sbase + OFF_STAGE + st * STAGE_BYTES + ld_row * ROW_PITCH;
#pragma unroll
        for (int q = 0; q < CHUNKS / 4; ++q) {
            const int ch = ld_part + 4 * q;
            cp_async_16(dst + ch * 16, src + ch * 8, ok);
        }
        if (ld_part == 0) rowok[st * BR + ld_row] = ok;
    };

    // Q of this token -> shared memory, together with the first row block.
    {
        const __half* qt = p.q + (size_t)i * H * DQK;
        for (int x = tid; x < H * CHUNKS; x += THREADS) {
            const int h = x / CHUNKS, ch = x % CHUNKS;
            cp_async_16(sbase + OFF_Q + h * ROW_PITCH + ch * 16, qt + h * DQK + ch * 8, true);
        }
    }
    issue_block(0, 0);
    cp_async_commit();

    uint32_t qf[DQK / 16][4];                    // Q as A fragments, all 36 k-steps
    cp_async_wait<0>();
    __syncthreads();
    {
        const int r = (lane & 7) + ((lane >> 3) & 1) * 8, kc = (lane >> 4) * 8;
#pragma unroll
        for (int kk = 0; kk < DQK / 16; ++kk)
            ldsm_x4(sbase + OFF_Q + r * ROW_PITCH + (kk * 16 + kc) * 2, qf[kk][0], qf[kk][1],
                    qf[kk][2], qf[kk][3]);
    }
    float o[8][4];                               // O[16 heads, 64 dims of this warp]
#pragma unroll
    for (int n = 0; n < 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
    float m_g = -INFINITY, m_g8 = -INFINITY;     // running max, heads g and g+8 (log2 units)
    float l_g = 0.f, l_g8 = 0.f;                 // this thread's partial sums

    for (int blk = 0; blk < nblk; ++blk) {
        const int st = blk & 1;
        if (blk > 0) {
            cp_async_wait<0>();
            __syncthreads();
        }
        if (blk + 1 < nblk) issue_block(blk + 1, st ^ 1);
        cp_async_commit();
        const uint32_t stage = sbase + OFF_STAGE + st * STAGE_BYTES;

        // ---- S = Q . R^T for rows 8w .. 8w+7 of the block
        float s[4] = {0.f, 0.f, 0.f, 0.f};
        {
            const uint32_t rowaddr = stage + (8 * warp + (lane & 7)) * ROW_PITCH + (lane >> 3) * 16;
#pragma unroll
            for (int k2 = 0; k2 < DQK / 32; ++k2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(rowaddr + k2 * 64, b0, b1, b2, b3);
                mma_16816(s, qf[2 * k2], b0, b1);
                mma_16816(s, qf[2 * k2 + 1], b2, b3);
            }
        }
        const int r0 = 8 * warp + 2 * c;
        const bool ok0 = rowok[st * BR + r0] != 0, ok1 = rowok[st * BR + r0 + 1] != 0;
        s[0] = ok0 ? s[0] * p.scale_log2 : -INFINITY;
        s[1] = ok1 ? s[1] * p.scale_log2 : -INFINITY;
        s[2] = ok0 ? s[2] * p.scale_log2 : -INFINITY;
        s[3] = ok1 ? s[3] * p.scale_log2 : -INFINITY;
        float mx_g = fmaxf(s[0], s[1]), mx_g8 = fmaxf(s[2], s[3]);
#pragma unroll
        for (int off = 1; off <= 2; off <<= 1) {
            mx_g = fmaxf(mx_g, __shfl_xor_sync(0xffffffffu, mx_g, off));
            mx_g8 = fmaxf(mx_g8, __shfl_xor_sync(0xffffffffu, mx_g8, off));
        }
        if (c == 0) {
            red_max[warp * H + g] = mx_g;
            red_max[warp * H + g + 8] = mx_g8;
        }
        __syncthreads();

        // ---- online softmax
        float bm_g = -INFINITY, bm_g8 = -INFINITY;
#pragma unroll
        for (int w = 0; w < WARPS; ++w) {
            bm_g = fmaxf(bm_g, red_max[w * H + g]);
            bm_g8 = fmaxf(bm_g8, red_max[w * H + g + 8]);
        }
        const float mn_g = fmaxf(m_g, bm_g), mn_g8 = fmaxf(m_g8, bm_g8);
        const float ref_g = mn_g == -INFINITY ? 0.f : mn_g;
        const float ref_g8 = mn_g8 == -INFINITY ? 0.f : mn_g8;
        const float alpha_g = exp2f(m_g - ref_g), alpha_g8 = exp2f(m_g8 - ref_g8);
        const float p0 = exp2f(s[0] - ref_g), p1 = exp2f(s[1] - ref_g);
        const float p2 = exp2f(s[2] - ref_g8), p3 = exp2f(s[3] - ref_g8);
        l_g = l_g * alpha_g + p0 + p1;
        l_g8 = l_g8 * alpha_g8 + p2 + p3;
        m_g = mn_g;
        m_g8 = mn_g8;
        {
            uint8_t* pb = smem + OFF_P;
            *reinterpret_cast<uint32_t*>(pb + g * P_PITCH + r0 * 2) = pack_half2(p0, p1);
            *reinterpret_cast<uint32_t*>(pb + (g + 8) * P_PITCH + r0 * 2) = pack_half2(p2, p3);
        }
        __syncthreads();

        // ---- O = alpha * O + P . V over value dims 64w .. 64w+63
#pragma unroll
        for (int n = 0; n < 8; ++n) {
            o[n][0] *= alpha_g;
            o[n][1] *= alpha_g;
            o[n][2] *= alpha_g8;
            o[n][3] *= alpha_g8;
        }
        {
            const int ar = (lane & 7) + ((lane >> 3) & 1) * 8, akc = (lane >> 4) * 8;
            const int vr = (lane & 7) + ((lane >> 3) & 1) * 8, vdc = (lane >> 4) * 8;
#pragma unroll
            for (int ks = 0; ks < BR / 16; ++ks) {
                uint32_t a[4];
                ldsm_x4(sbase + OFF_P + ar * P_PITCH + (ks * 16 + akc) * 2, a[0], a[1], a[2], a[3]);
                const uint32_t vrow = stage + (ks * 16 + vr) * ROW_PITCH;
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_trans(vrow + (64 * warp + np * 16 + vdc) * 2, b0, b1, b2, b3);
                    mma_16816(o[2 * np], a, b0, b1);
                    mma_16816(o[2 * np + 1], a, b2, b3);
                }
            }
        }
    }

    // ---- normalise and store
#pragma unroll
    for (int off = 1; off <= 2; off <<= 1) {
        l_g += __shfl_xor_sync(0xffffffffu, l_g, off);
        l_g8 += __shfl_xor_sync(0xffffffffu, l_g8, off);
    }
    if (c == 0) {
        red_sum[warp * H + g] = l_g;
        red_sum[warp * H + g + 8] = l_g8;
    }
    __syncthreads();
    float L_g = 0.f, L_g8 = 0.f;
#pragma unroll
    for (int w = 0; w < WARPS; ++w) {
        L_g += red_sum[w * H + g];
        L_g8 += red_sum[w * H + g + 8];
    }
    const float inv_g = L_g > 0.f ? 1.f / L_g : 0.f;
    const float inv_g8 = L_g8 > 0.f ? 1.f / L_g8 : 0.f;
    float* ot = p.out + (size_t)i * H * DV;
#pragma unroll
    for (int n = 0; n < 8; ++n) {
        const int d = 64 * warp + 8 * n + 2 * c;
        *reinterpret_cast<float2*>(ot + g * DV + d) = make_float2(o[n][0] * inv_g, o[n][1] * inv_g);
        *reinterpret_cast<float2*>(ot + (g + 8) * DV + d) =
            make_float2(o[n][2] * inv_g8, o[n][3] * inv_g8);
    }
}

}  // namespace ds4sp
