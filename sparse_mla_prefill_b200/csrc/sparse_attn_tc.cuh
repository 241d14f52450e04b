// Sparse MLA attention with the logits on the 5th-generation tensor cores (tcgen05).
//
// The same computation as sparse_attn_mma_kernel -- for token t one softmax of the 16
// heads over the selected compressed rows (ascending j) followed by the window's raw
// rows, key = a row's 576 values, value = its first 512 ("stream each selected latent
// row once across sixteen ... heads", "perf(ds4): extend sparse prefill scheduling to
// 10K", Summary) -- in the form with KV rows as the MMA's M and heads as its N: a unit
// is 128 gathered rows, and S = R . Q^T (M = 128 rows, N = 16 heads, K = 576) is one
// chain of 36 tcgen05.mma.kind::f16 instructions issued by one thread into a 16-column
// fp32 accumulator in TMEM, so the tensor core computes the logits asynchronously while
// the other warps run.
//
// Warps: 0-3 gather (each token's top-k row and Q, then per unit 128 rows with 16-byte
// cp.async straight into the 128-byte-swizzled K-major layout the MMA descriptors read:
// nine 64-value slabs of 128 rows x 128 bytes); warp 4 owns TMEM and issues the MMAs;
// warps 5-8 take one row each of S from TMEM (tcgen05.ld, the warp's lane quarter), run
// an exact online softmax over the unit (per-head maxima combined in shared memory, O
// and the sums rescaled when a head's maximum rises), write P as fp16, and compute
// O += P . V with mma.sync.m16n8k16 (heads as M), each warp owning 128 value dims, V
// read from the same row tile. The row tile (147 KB) is single-buffered: the next
// unit's gather starts when the consumers have finished this unit's P . V.
// Every wait is bounded (device_common.cuh); a consumer that gives up raises a flag that
// the consumer warps read after their next barrier.
#pragma once

#include "device_common.cuh"
#include "sparse_attn_mma.cuh"

namespace ds4sp {
namespace tcattn {

constexpr int M = 128;                         // rows per unit (UMMA M)
constexpr int NH = attn::H;                    // heads (UMMA N)
constexpr int SLABS = attn::DQK / 64;          // 9 slabs of 64 values (128 bytes)
constexpr int SLAB_R = M * 128;                // one slab of the row tile: 16 KB
constexpr int TILE = SLABS * SLAB_R;           // 147,456 bytes
constexpr int SLAB_Q = NH * 128;               // one slab of Q: 2 KB
constexpr int QBYTES = SLABS * SLAB_Q;         // 18,432 bytes
constexpr int P_PITCH = (M + 8) * 2;           // fp16 P row of one head, padded
constexpr int PWARPS = 4, MWARP = 4, CWARPS = 4;
constexpr int CWARP0 = PWARPS + 1;             // consumer warps 5..8
constexpr int THREADS = (PWARPS + 1 + CWARPS) * 32;
constexpr int PTHREADS = PWARPS * 32, CTHREADS = CWARPS * 32;
constexpr int PRODUCER_BAR = 1, CONSUMER_BAR = 2;
constexpr int OFF_TILE = 0;
constexpr int OFF_Q = OFF_TILE + TILE;
constexpr int OFF_P = OFF_Q + QBYTES;
constexpr int OFF_RED = OFF_P + NH * P_PITCH;                 // [CWARPS][NH] maxima, then sums
constexpr int OFF_FLAG = OFF_RED + 2 * CWARPS * NH * 4;
constexpr int OFF_BAR = OFF_FLAG + 16;                        // q_full q_empty t_full t_empty s_full done
constexpr int OFF_TMEM = OFF_BAR + 6 * 8;
constexpr int OFF_IDX = OFF_TMEM + 16;                        // two staged top-k rows
constexpr uint32_t IDESC = umma_idesc_f16_f32(M, NH);
__host__ __device__ constexpr int smem_bytes(int k) {
    return OFF_IDX + 2 * ((k + 3) / 4 * 4) * 4 + 1024;        // + 1 KB alignment slack
}
static_assert(OFF_Q % 1024 == 0 && OFF_TILE % 1024 == 0, "swizzle atoms need 1 KB alignment");
static_assert(OFF_IDX % 16 == 0, "16-byte aligned index rows");
static_assert(smem_bytes(attn::MAX_TOPK) <= 227 * 1024, "shared memory budget");

// Byte offset of 16-byte chunk `ch` (0..71) of row `r` in a K-major tile of `rows_slab`
// bytes per slab: slab ch/8, 8-row atoms of 1024 bytes, chunk index XOR (row & 7) -- the
// 128-byte swizzle the UMMA shared-memory descriptor (umma_desc_sw128) expects.
__device__ __forceinline__ uint32_t sw128_off(int r, int ch, int slab_bytes) {
    return (ch >> 3) * slab_bytes + (r >> 3) * 1024 + (r & 7) * 128 + (((ch & 7) ^ (r & 7)) << 4);
}

}  // namespace tcattn

__global__ void __launch_bounds__(tcattn::THREADS, 1) sparse_attn_tc_kernel(AttnParams p) {
    using namespace tcattn;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_u32 = smem_u32(smem_raw);
    const uint32_t base = (raw_u32 + 1023u) & ~1023u;
    uint8_t* smem = smem_raw + (base - raw_u32);
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int kpad = (p.k + 3) / 4 * 4;
    const uint32_t bar0 = base + OFF_BAR;
    const uint32_t q_full = bar0, q_empty = bar0 + 8, t_full = bar0 + 16, t_empty = bar0 + 24,
                   s_full = bar0 + 32, done_bar = bar0 + 40;
    uint32_t* tmem_ptr = reinterpret_cast<uint32_t*>(smem + OFF_TMEM);
    volatile int* cflag = reinterpret_cast<volatile int*>(smem + OFF_FLAG);
    auto idx_buf = [&](int m) { return reinterpret_cast<int*>(smem + OFF_IDX) + (m & 1) * kpad; };

    if (tid == 0) {
        mbar_init(q_full, PTHREADS);     // the producers' copy arrivals
        mbar_init(q_empty, 1);           // MMA commit after a token's last unit
        mbar_init(t_full, PTHREADS);
        mbar_init(t_empty, CWARPS);      // one arrival per consumer warp
        mbar_init(s_full, 1);            // MMA commit per unit
        mbar_init(done_bar, 1);
        *cflag = 0;
        fence_mbar_init();
    }
    if (warp == MWARP) {
        tmem_alloc(smem_u32(tmem_ptr), 32);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_ptr;
    grid_dependency_wait();
    grid_dependents_launch();

    // This CTA's tokens, heaviest (latest) first.
    auto token_of = [&](int m, TokenRows& tr) {
        const int idx = blockIdx.x + m * gridDim.x;
        if (idx >= p.n_q) return false;
        tr = token_rows_of(p, p.n_q - 1 - idx);
        return true;
    };
    // Row gr of token tr: a selected compressed row (checked) or a window row.
    auto resolve = [&](const TokenRows& tr, const int* tk, int gr, bool& cmp, long long& src) {
        cmp = false;
        src = 0;
        if (gr >= tr.nrows) return false;
        if (gr < tr.nsel) {
            const int j = tk[gr];
            cmp = true;
            src = j;
            if (p.vis_mask == nullptr) return j >= 0 && j < tr.nv;
            return j >= 0 && j < p.mask_cols && p.vis_mask[(size_t)tr.t * p.mask_ld + j] != 0;
        }
        src = tr.s_lo + gr - tr.nsel;
        return true;
    };

    bool abort = false;
    if (warp < PWARPS) {
        // ================================================================ producers
        const int ptid = tid;
        int ui = 0;                              // units gathered so far
        TokenRows tr;
        for (int m = 0; token_of(m, tr); ++m) {
            // Q and the top-k row of token m; Q is free once the previous token's MMAs ran.
            if (!abort && !__all_sync(0xffffffffu, mbar_wait(q_empty, (m & 1) ^ 1, p.wc, abort)))
                abort = true;
            if (!abort) {
                int* tk = idx_buf(m);
                const int32_t* src = p.topk + (size_t)tr.i * p.k;
                for (int e = ptid; e < tr.nsel; e += PTHREADS)
                    asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(tk + e)),
                                 "l"(src + e)
                                 : "memory");
                cp_async_commit();
                const __half* qt = p.q + (size_t)tr.i * NH * attn::DQK;
                for (int e = ptid; e < NH * attn::CH; e += PTHREADS) {
                    const int r = e / attn::CH, ch = e % attn::CH;
                    cp_async_16(base + OFF_Q + sw128_off(r, ch, SLAB_Q), qt + r * attn::DQK + ch * 8, true);
                }
                cp_async_commit();
                cp_async_arrive_noinc(q_full);
                cp_async_wait<1>();              // this thread's top-k entries have landed
            }
            named_barrier(PRODUCER_BAR, PTHREADS);   // every producer sees the whole row
            const int* tk = idx_buf(m);
            const int nu = (tr.nrows + M - 1) / M;
            for (int u = 0; u < nu; ++u, ++ui) {
                if (!abort &&
                    !__all_sync(0xffffffffu, mbar_wait(t_empty, (ui & 1) ^ 1, p.wc, abort)))
                    abort = true;
                if (abort) continue;
#pragma unroll 1
                for (int pass = 0; pass < M / 32; ++pass) {
                    const int r = 32 * pass + 8 * warp + (lane >> 2);
                    bool cmp;
                    long long srow;
                    const bool ok = resolve(tr, tk, u * M + r, cmp, srow);
                    if (!ok && u * M + r < tr.nsel && (lane & 3) == 0) {
                        const int j = tk[u * M + r];
                        if (!(p.vis_mask != nullptr && (j == -1 || (j >= 0 && j < p.mask_cols))))
                            record_status(p.wc.status, kStatusBounds);
                    }
                    const __half* row = ok ? (cmp ? p.kv_cmp : p.kv_raw) + (size_t)srow * attn::DQK
                                           : p.kv_raw + (size_t)tr.t * attn::DQK;   // valid stand-in
#pragma unroll
                    for (int i = 0; i < 18; ++i) {
                        const int ch = (lane & 3) + 4 * i;
                        cp_async_16(base + OFF_TILE + sw128_off(r, ch, SLAB_R), row + ch * 8, ok);
                    }
                }
                cp_async_arrive_noinc(t_full);
            }
        }
        cp_async_wait<0>();
    } else if (warp == MWARP) {
        // ================================================================ MMA issuer
        if (lane == 0) {
            const uint64_t a0 = umma_desc_sw128(base + OFF_TILE);
            const uint64_t b0 = umma_desc_sw128(base + OFF_Q);
            int ui = 0;
            TokenRows tr;
            for (int m = 0; !abort && token_of(m, tr); ++m) {
                if (!mbar_wait(q_full, m & 1, p.wc, abort)) break;
                const int nu = (tr.nrows + M - 1) / M;
                for (int u = 0; u < nu; ++u, ++ui) {
                    if (!mbar_wait(t_full, ui & 1, p.wc, abort)) break;
                    tc_fence_after();
#pragma unroll
                    for (int s = 0; s < SLABS; ++s)
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk)   // k16 steps: 32 bytes into a 128-byte row
                            umma_f16(tmem_base, a0 + (uint64_t)((s * SLAB_R + kk * 32) >> 4),
                                     b0 + (uint64_t)((s * SLAB_Q + kk * 32) >> 4), IDESC,
                                     s > 0 || kk > 0);
                    umma_commit(s_full);
                }
                if (abort) break;
                umma_commit(q_empty);            // Q may be overwritten once these finish
            }
            umma_commit(done_bar);
            mbar_wait_drain(done_bar, 0, p.wc);
        }
        __syncwarp();
    } else {
        // ================================================================ consumers
        const int cw = warp - CWARP0;            // value dims 128cw .. 128cw+127
        const int qd = warp & 3;                 // TMEM lane quarter: rows 32qd .. 32qd+31
        const int r = 32 * qd + lane;            // this thread's row of each unit
        const int g = lane / 4, c = lane % 4;    // mma fragment coordinates
        const int ar = (lane & 7) + ((lane >> 3) & 1) * 8, hi = lane >> 4;
        float* red_max = reinterpret_cast<float*>(smem + OFF_RED);
        float* red_sum = red_max + CWARPS * NH;
        uint8_t* pbuf = smem + OFF_P;
        const uint32_t pbase = base + OFF_P;
        int ui = 0;
        TokenRows tr;
        for (int m = 0; token_of(m, tr); ++m) {
            float o[16][4];
#pragma unroll
            for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
            float mrun[NH], lpart[NH];
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                mrun[h] = -INFINITY;
                lpart[h] = 0.f;
            }
            const int* tk = idx_buf(m);
            const int nu = (tr.nrows + M - 1) / M;
            bool stop = false;
            for (int u = 0; u < nu; ++u, ++ui) {
                const bool ok = mbar_wait(t_full, ui & 1, p.wc, abort) &&
                                mbar_wait(s_full, ui & 1, p.wc, abort);
                if (!__all_sync(0xffffffffu, ok)) *cflag = 1;
                tc_fence_after();
                bool cmp;
                long long srow;
                const bool valid = resolve(tr, tk, u * M + r, cmp, srow);
                uint32_t sv[NH];
                tmem_ld_x16(tmem_base + ((uint32_t)(32 * qd) << 16), sv);
                tmem_ld_wait();
                float lg[NH];
#pragma unroll
                for (int h = 0; h < NH; ++h) lg[h] = valid ? __uint_as_float(sv[h]) * p.scale_log2 : -INFINITY;
                // per-head maximum of the unit: the warp's 32 rows, then the four warps
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    float v = lg[h];
#pragma unroll
                    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
                    if (lane == 0) red_max[cw * NH + h] = v;
                }
                named_barrier(CONSUMER_BAR, CTHREADS);        // A: maxima in place
                if (*cflag) {                                 // every consumer warp sees it
                    stop = true;
                    break;
                }
                float alpha[NH];
#pragma unroll
                for (int h = 0; h < NH; ++h) {
                    float mu = red_max[h];
#pragma unroll
                    for (int w2 = 1; w2 < CWARPS; ++w2) mu = fmaxf(mu, red_max[w2 * NH + h]);
                    const float mnew = fmaxf(mrun[h], mu);
                    alpha[h] = mnew == -INFINITY ? 1.f : fast_exp2(mrun[h] - mnew);
                    const float pr = mnew == -INFINITY ? 0.f : fast_exp2(lg[h] - mnew);
                    lpart[h] = lpart[h] * alpha[h] + pr;
                    mrun[h] = mnew;
                    *reinterpret_cast<__half*>(pbuf + h * P_PITCH + r * 2) = __float2half_rn(pr);
                }
                float a_g = 1.f, a_g8 = 1.f;          // the rescale of this lane's two heads
#pragma unroll
                for (int h = 0; h < NH / 2; ++h)
                    if (g == h) {
                        a_g = alpha[h];
                        a_g8 = alpha[h + NH / 2];
                    }
#pragma unroll
                for (int n = 0; n < 16; ++n) {
                    o[n][0] *= a_g;
                    o[n][1] *= a_g;
                    o[n][2] *= a_g8;
                    o[n][3] *= a_g8;
                }
                named_barrier(CONSUMER_BAR, CTHREADS);        // B: P complete
                // O += P . V over this warp's 128 value dims, the unit's 128 rows
#pragma unroll 2
                for (int ks = 0; ks < M / 16; ++ks) {
                    uint32_t a[4];
                    ldsm_x4(pbase + ar * P_PITCH + (ks * 16 + hi * 8) * 2, a[0], a[1], a[2], a[3]);
                    const int vr = ks * 16 + ar;
#pragma unroll
                    for (int np = 0; np < 8; ++np) {
                        uint32_t b0, b1, b2, b3;
                        const int vch = 16 * cw + 2 * np + hi;
                        ldsm_x4_trans(base + OFF_TILE + sw128_off(vr, vch, SLAB_R), b0, b1, b2, b3);
                        mma_16816(o[2 * np], a, b0, b1);
                        mma_16816(o[2 * np + 1], a, b2, b3);
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(t_empty);          // rows, S and P may be reused
            }
            if (stop) break;
            // token end: sums over all rows, then O / sum
#pragma unroll
            for (int h = 0; h < NH; ++h) {
                float v = lpart[h];
#pragma unroll
                for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
                if (lane == 0) red_sum[cw * NH + h] = v;
            }
            named_barrier(CONSUMER_BAR, CTHREADS);
            float L_g = 0.f, L_g8 = 0.f;
#pragma unroll
            for (int w2 = 0; w2 < CWARPS; ++w2) {
                L_g += red_sum[w2 * NH + g];
                L_g8 += red_sum[w2 * NH + g + 8];
            }
            const float inv_g = L_g > 0.f ? 1.f / L_g : 0.f, inv_g8 = L_g8 > 0.f ? 1.f / L_g8 : 0.f;
            float* ot = p.out + (size_t)tr.i * NH * attn::DV;
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                const int d = 128 * cw + 8 * n + 2 * c;
                *reinterpret_cast<float2*>(ot + g * attn::DV + d) = make_float2(o[n][0] * inv_g, o[n][1] * inv_g);
                *reinterpret_cast<float2*>(ot + (g + 8) * attn::DV + d) =
                    make_float2(o[n][2] * inv_g8, o[n][3] * inv_g8);
            }
            named_barrier(CONSUMER_BAR, CTHREADS);            // the sums are read before reuse
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == MWARP) tmem_dealloc(tmem_base, 32);
}

}  // namespace ds4sp
