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
// Persistent CTAs (one per SM) walk their tokens heaviest first as a flat sequence of
// units: per token, one unit holding its Q (16 rows), then its rows in blocks of 32.
// Units stream through a 5-slot shared-memory ring with one mbarrier pair per slot.
//   * Warps 8-11 produce. They stage each token's top-k row in shared memory one
//     token ahead, resolve and check every row, and copy it in 16-byte chunks with
//     cp.async; cp.async.mbarrier.arrive.noinc lets the slot's barrier count the copies
//     without the producer waiting for them. Each producer warp also publishes which of
//     its 8 rows are valid. Producers never take part in the consumers' barriers.
//   * Warps 0-7 consume, with the 16 heads as the M of mma.sync.m16n8k16. Warp w owns
//     row tile nt = w%4 (8 rows) and K half kh = w/4 (288 dims) of S = Q . R^T, Q held
//     in registers; the two K halves meet in shared memory. A round takes two
//     consecutive row units of a token (64 rows: two row tiles per warp) when it can.
//     Softmax runs against a running reference max that is raised only when a round's
//     max exceeds it by more than 2^8 (probabilities stay <= 256, fine in fp16): a round
//     normally needs two consumer barriers; raising the reference rescales O, the sums
//     and that round's P in every warp. O += P . V: warp w owns value dims 64w .. 64w+63.
// Rows are stored unpadded with their 16-byte chunks XOR-swizzled, which keeps the
// producers' copies and the consumers' ldmatrix reads free of bank conflicts.
// fp32 logits, sums and output; P enters P . V as fp16; exponentials on ex2.approx.
// Every wait is bounded; a consumer that gives up sets a flag that all consumer warps
// read at their next barrier, so none is left waiting.
#pragma once

#include "device_common.cuh"

namespace ds4sp {
namespace attn {

constexpr int H = 16;
constexpr int DQK = 576;
constexpr int DV = 512;
constexpr int ROW = DQK * 2;                  // 1152 bytes per latent row
constexpr int CH = ROW / 16;                  // 72 sixteen-byte chunks per row
constexpr int BR = 32;                        // rows per unit
constexpr int NS = 5;                         // ring slots
constexpr int CWARPS = 8;                     // consumer warps
constexpr int PWARPS = 4;                     // producer warps
constexpr int CTHREADS = CWARPS * 32;
constexpr int PTHREADS = PWARPS * 32;
constexpr int THREADS = CTHREADS + PTHREADS;
constexpr int CONSUMER_BAR = 1;               // named barriers
constexpr int PRODUCER_BAR = 2;
// Registers per thread: the kernel is built for LAUNCH_REGS (one CTA of THREADS per
// SM); producers hand part of theirs to the consumers with setmaxnreg. The host checks
// the built count before the first launch: a split above the launch's total would
// leave the consumers' setmaxnreg.inc waiting.
constexpr int LAUNCH_REGS = 168;
constexpr int CONSUMER_REGS = 224;
constexpr int PRODUCER_REGS = 56;
static_assert(CWARPS * 32 * CONSUMER_REGS + PWARPS * 32 * PRODUCER_REGS <= THREADS * LAUNCH_REGS,
              "register split must fit the launch's registers");
constexpr float HEADROOM = 8.f;               // log2 units a block may exceed the reference
constexpr int SLOT = BR * ROW;
constexpr int P_PITCH = (2 * BR + 8) * 2;     // fp16 probabilities of two units, 144 B per head
constexpr int IDX_BUFS = 2;                   // producers' top-k rows: this token, the next
constexpr int OFF_RING = 0;
constexpr int OFF_P = OFF_RING + NS * SLOT;
constexpr int OFF_SX = OFF_P + H * P_PITCH;   // S partials of the upper K half, two units
constexpr int OFF_REF = OFF_SX + 2 * 4 * 32 * 16;  // per row tile: reference used for its P
constexpr int OFF_RED_SUM = OFF_REF + 4 * H * 4;
constexpr int OFF_FLAGS = OFF_RED_SUM + 4 * H * 4;   // raised[2], abort, pad
constexpr int OFF_MASK = OFF_FLAGS + 16;             // row-validity bits per slot
constexpr int OFF_BAR = OFF_MASK + 32;               // full[NS], empty[NS]
constexpr int OFF_IDX = OFF_BAR + 2 * NS * 8;
constexpr int MAX_TOPK = 2048;
__host__ __device__ constexpr int smem_bytes(int k) {
    return OFF_IDX + IDX_BUFS * ((k + 3) / 4 * 4) * 4;
}
static_assert(DV == CWARPS * 64, "each consumer warp owns 64 value dims");
static_assert(CH % 8 == 0 && BR * CH == PTHREADS * 18, "producer chunk split");
static_assert(smem_bytes(MAX_TOPK) <= 227 * 1024, "shared memory budget");

// 16-byte chunk swizzle: eight consecutive rows put one chunk in eight different bank
// groups (ldmatrix), and rows 2m, 2m+1 put an aligned group of four chunks in
// complementary halves (a quarter warp's cp.async).
__device__ __forceinline__ int swz(int row) { return ((row & 1) << 2) | ((row >> 1) & 3); }
__device__ __forceinline__ uint32_t chunk_addr(uint32_t slot, int row, int chunk) {
    return slot + row * ROW + ((chunk ^ swz(row)) << 4);
}

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

// Position in a CTA's flat unit sequence: token number n (the CTA's n-th token), unit u
// (0 = Q, 1.. = row blocks).
struct UnitCursor {
    int n, idx, u;
    TokenRows tr;
    bool valid;
    __device__ __forceinline__ void start(const AttnParams& p) {
        n = 0;
        idx = blockIdx.x;
        u = 0;
        valid = idx < p.n_q;
        if (valid) tr = token_rows(p, idx);
    }
    __device__ __forceinline__ void advance(const AttnParams& p) {
        if (!valid) return;
        if (++u > tr.nblk) {
            u = 0;
            ++n;
            idx += gridDim.x;
            valid = idx < p.n_q;
            if (valid) tr = token_rows(p, idx);
        }
    }
};

__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

__global__ void __launch_bounds__(attn::THREADS, 1) sparse_attn_mma_kernel(AttnParams p) {
    using namespace attn;
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int kpad = (p.k + 3) / 4 * 4;
    volatile int* flags = reinterpret_cast<volatile int*>(smem + OFF_FLAGS);  // raised[2], abort
    volatile uint32_t* rowmask = reinterpret_cast<volatile uint32_t*>(smem + OFF_MASK);
    const uint32_t bar0 = sbase + OFF_BAR;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (NS + s); };

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) {
            mbar_init(full_bar(s), PTHREADS + PWARPS);   // noinc copy arrivals + mask writers
            mbar_init(empty_bar(s), CWARPS);
        }
        flags[0] = flags[1] = flags[2] = 0;
        fence_mbar_init();
    }
    __syncthreads();

    bool abort = false;
    if (warp >= CWARPS) {
        // ================================================================ producers
        regs_decrease<PRODUCER_REGS>();
        const int ptid = tid - CTHREADS, pw = warp - CWARPS;
        auto stage_idx = [&](int n) {             // top-k row of the CTA's token number n
            const int idx = blockIdx.x + n * gridDim.x;
            if (idx >= p.n_q) return;
            const TokenRows nx = token_rows(p, idx);
            const int32_t* src = p.topk + (size_t)nx.i * p.k;
            const uint32_t dst = sbase + OFF_IDX + (n % IDX_BUFS) * kpad * 4;
            for (int e = ptid; e < nx.nsel; e += PTHREADS)
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst + 4 * e),
                             "l"(src + e)
                             : "memory");
        };
        stage_idx(0);
        cp_async_commit();
        cp_async_wait<0>();
        named_barrier(PRODUCER_BAR, PTHREADS);
        UnitCursor cu;
        cu.start(p);
        for (int uc = 0; cu.valid; ++uc, cu.advance(p)) {
            const int s = uc % NS;
            if (!__all_sync(0xffffffffu,
                            mbar_wait(empty_bar(s), ((uc / NS) & 1) ^ 1, p.status, abort)))
                break;
            const uint32_t dst = sbase + OFF_RING + s * SLOT;
            if (cu.u == 0) {
                // Q of the token, and the next token's top-k row one token ahead.
                stage_idx(cu.n + 1);
                const __half* qt = p.q + (size_t)cu.tr.i * H * DQK;
#pragma unroll
                for (int m = 0; m < H * CH / PTHREADS; ++m) {
                    const int e = ptid + m * PTHREADS, r = e / CH, ch = e % CH;
                    cp_async_16(chunk_addr(dst, r, ch), qt + r * DQK + ch * 8, true);
                }
                cp_async_commit();
                cp_async_arrive_noinc(full_bar(s));
                __syncwarp();
                if (lane == 0) mbar_arrive(full_bar(s));
                // This token's top-k row (staged one token earlier) must be in shared
                // memory, for every producer thread, before its row units are resolved.
                cp_async_wait<1>();
                named_barrier(PRODUCER_BAR, PTHREADS);
                continue;
            }
            const int* tk = reinterpret_cast<const int*>(smem + OFF_IDX) + (cu.n % IDX_BUFS) * kpad;
            const int r = 8 * pw + (lane >> 2);   // this lane's row of the unit
            const int gr = (cu.u - 1) * BR + r;
            const __half* row = p.kv_raw + (size_t)cu.tr.t * DQK;   // valid stand-in
            bool ok = false;
            if (gr < cu.tr.nsel) {
                const int j = tk[gr];
                if (j >= 0 && j < cu.tr.nv) {
                    row = p.kv_cmp + (size_t)j * DQK;
                    ok = true;
                } else if ((lane & 3) == 0) {
                    record_status(p.status, kStatusBounds);
                }
            } else if (gr < cu.tr.nrows) {
                row = p.kv_raw + (size_t)(cu.tr.s_lo + gr - cu.tr.nsel) * DQK;
                ok = true;
            }
#pragma unroll
            for (int m = 0; m < 18; ++m) {
                const int ch = (lane & 3) + 4 * m;
                cp_async_16(chunk_addr(dst, r, ch), row + ch * 8, ok);   // zero-filled if masked
            }
            cp_async_arrive_noinc(full_bar(s));
            const uint32_t bits = __ballot_sync(0xffffffffu, ok && (lane & 3) == 0);
            if (lane == 0) {
                uint32_t m8 = 0;
#pragma unroll
                for (int i = 0; i < 8; ++i) m8 |= ((bits >> (4 * i)) & 1u) << i;
                reinterpret_cast<volatile uint8_t*>(rowmask + s)[pw] = (uint8_t)m8;
                mbar_arrive(full_bar(s));         // release: the mask byte is visible with the slot
            }
        }
        cp_async_wait<0>();
    } else {
        // ================================================================ consumers
        regs_increase<CONSUMER_REGS>();
        // A round consumes the Q unit of a token, or one or two consecutive row units of
        // the same token (64 rows): two row tiles per warp between the same two barriers.
        float* ref_tile = reinterpret_cast<float*>(smem + OFF_REF);
        float* red_sum = reinterpret_cast<float*>(smem + OFF_RED_SUM);
        const int g = lane / 4, c = lane % 4;    // mma fragment coordinates
        const int nt = warp & 3, kh = warp >> 2; // S: row tile and K half of this warp
        const int r0 = 8 * nt + 2 * c;           // S columns of this lane: unit rows r0, r0+1
        const int rr8 = 8 * nt + (lane & 7);     // S: this lane's ldmatrix row
        const int ar = (lane & 7) + ((lane >> 3) & 1) * 8, hi = lane >> 4;
        uint32_t qf[18][4];
        float o[8][4];
        float m_g = -INFINITY, m_g8 = -INFINITY; // reference max, heads g and g+8 (log2 units)
        float l_g = 0.f, l_g8 = 0.f;             // partial sums (K-half-0 warps only)
        auto wait_full = [&](int q) {
            if (!__all_sync(0xffffffffu, mbar_wait(full_bar(q % NS), (q / NS) & 1, p.status, abort)))
                flags[2] = 1;
        };
        UnitCursor cu;
        cu.start(p);
        int rr = 0;                               // row rounds
        int q = 0;                                // next unit of the ring
        while (cu.valid) {
            const uint32_t slot_a = sbase + OFF_RING + (q % NS) * SLOT;
            if (cu.u == 0) {
                wait_full(q);
#pragma unroll
                for (int kk = 0; kk < 18; ++kk)
                    ldsm_x4(chunk_addr(slot_a, ar, 36 * kh + 2 * kk + hi), qf[kk][0], qf[kk][1],
                            qf[kk][2], qf[kk][3]);
#pragma unroll
                for (int n = 0; n < 8; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
                m_g = m_g8 = -INFINITY;
                l_g = l_g8 = 0.f;
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_bar(q % NS));
                ++q;
                cu.advance(p);
                continue;
            }
            const bool two = cu.u < cu.tr.nblk;   // a second row unit of this token follows
            const bool last = cu.u + (two ? 1 : 0) == cu.tr.nblk;
            const uint32_t slot_b = sbase + OFF_RING + ((q + 1) % NS) * SLOT;
            wait_full(q);
            if (two) wait_full(q + 1);

            // ---- S partials over this warp's K half: unit A and unit B interleaved
            float aa[2][4] = {}, ab[2][4] = {};
#pragma unroll
            for (int k2 = 0; k2 < 9; ++k2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(chunk_addr(slot_a, rr8, 36 * kh + 4 * k2 + (lane >> 3)), b0, b1, b2, b3);
                mma_16816(aa[0], qf[2 * k2], b0, b1);
                mma_16816(aa[1], qf[2 * k2 + 1], b2, b3);
                if (two) {
                    ldsm_x4(chunk_addr(slot_b, rr8, 36 * kh + 4 * k2 + (lane >> 3)), b0, b1, b2, b3);
                    mma_16816(ab[0], qf[2 * k2], b0, b1);
                    mma_16816(ab[1], qf[2 * k2 + 1], b2, b3);
                }
            }
            float sa[4], sb[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                sa[e] = aa[0][e] + aa[1][e];
                sb[e] = ab[0][e] + ab[1][e];
            }
            float4* sx = reinterpret_cast<float4*>(smem + OFF_SX) + nt * 32 + lane;
            if (kh == 1) {
                sx[0] = make_float4(sa[0], sa[1], sa[2], sa[3]);
                if (two) sx[128] = make_float4(sb[0], sb[1], sb[2], sb[3]);
            }
            named_barrier(CONSUMER_BAR, CTHREADS);    // A: S halves meet
            if (flags[2]) break;                       // every consumer warp sees the same flag

            float ref_g = m_g, ref_g8 = m_g8;
            if (kh == 0) {
                const float4 ua = sx[0];
                const uint32_t ma = rowmask[q % NS];
                const bool a0 = (ma >> r0) & 1u, a1 = (ma >> (r0 + 1)) & 1u;
                sa[0] = a0 ? (sa[0] + ua.x) * p.scale_log2 : -INFINITY;
                sa[1] = a1 ? (sa[1] + ua.y) * p.scale_log2 : -INFINITY;
                sa[2] = a0 ? (sa[2] + ua.z) * p.scale_log2 : -INFINITY;
                sa[3] = a1 ? (sa[3] + ua.w) * p.scale_log2 : -INFINITY;
                if (two) {
                    const float4 ub = sx[128];
                    const uint32_t mb = rowmask[(q + 1) % NS];
                    const bool b0 = (mb >> r0) & 1u, b1 = (mb >> (r0 + 1)) & 1u;
                    sb[0] = b0 ? (sb[0] + ub.x) * p.scale_log2 : -INFINITY;
                    sb[1] = b1 ? (sb[1] + ub.y) * p.scale_log2 : -INFINITY;
                    sb[2] = b0 ? (sb[2] + ub.z) * p.scale_log2 : -INFINITY;
                    sb[3] = b1 ? (sb[3] + ub.w) * p.scale_log2 : -INFINITY;
                } else {
                    sb[0] = sb[1] = sb[2] = sb[3] = -INFINITY;
                }
                float mx_g = fmaxf(fmaxf(sa[0], sa[1]), fmaxf(sb[0], sb[1]));
                float mx_g8 = fmaxf(fmaxf(sa[2], sa[3]), fmaxf(sb[2], sb[3]));
#pragma unroll
                for (int off = 1; off <= 2; off <<= 1) {
                    mx_g = fmaxf(mx_g, __shfl_xor_sync(0xffffffffu, mx_g, off));
                    mx_g8 = fmaxf(mx_g8, __shfl_xor_sync(0xffffffffu, mx_g8, off));
                }
                // Keep the running reference unless these tiles exceed it by the headroom.
                if (mx_g > m_g + HEADROOM) ref_g = mx_g;
                if (mx_g8 > m_g8 + HEADROOM) ref_g8 = mx_g8;
                const float rg = ref_g == -INFINITY ? 0.f : ref_g;
                const float rg8 = ref_g8 == -INFINITY ? 0.f : ref_g8;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    sa[e] = fast_exp2(sa[e] - (e < 2 ? rg : rg8));
                    sb[e] = fast_exp2(sb[e] - (e < 2 ? rg : rg8));
                }
                uint8_t* pb = smem + OFF_P;
                *reinterpret_cast<uint32_t*>(pb + g * P_PITCH + r0 * 2) = pack_half2(sa[0], sa[1]);
                *reinterpret_cast<uint32_t*>(pb + (g + 8) * P_PITCH + r0 * 2) = pack_half2(sa[2], sa[3]);
                *reinterpret_cast<uint32_t*>(pb + g * P_PITCH + (BR + r0) * 2) = pack_half2(sb[0], sb[1]);
                *reinterpret_cast<uint32_t*>(pb + (g + 8) * P_PITCH + (BR + r0) * 2) =
                    pack_half2(sb[2], sb[3]);
                if (c == 0) {
                    ref_tile[nt * H + g] = ref_g;
                    ref_tile[nt * H + g + 8] = ref_g8;
                }
                if (ref_g != m_g || ref_g8 != m_g8) flags[rr & 1] = 1;
            }
            named_barrier(CONSUMER_BAR, CTHREADS);    // B: P and the tiles' references visible
            const bool raise = flags[rr & 1] != 0;    // the same in every consumer thread
            if (tid == 0) flags[(rr + 1) & 1] = 0;    // next round's flag; its writers follow A

            if (raise) {                              // rare: raise the reference, rescale
                const float M_g = fmaxf(fmaxf(ref_tile[g], ref_tile[H + g]),
                                        fmaxf(ref_tile[2 * H + g], ref_tile[3 * H + g]));
                const float M_g8 = fmaxf(fmaxf(ref_tile[g + 8], ref_tile[H + g + 8]),
                                         fmaxf(ref_tile[2 * H + g + 8], ref_tile[3 * H + g + 8]));
                const float Mg = M_g == -INFINITY ? 0.f : M_g, Mg8 = M_g8 == -INFINITY ? 0.f : M_g8;
                const float alpha_g = fast_exp2(m_g - Mg), alpha_g8 = fast_exp2(m_g8 - Mg8);
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    o[n][0] *= alpha_g;
                    o[n][1] *= alpha_g;
                    o[n][2] *= alpha_g8;
                    o[n][3] *= alpha_g8;
                }
                if (kh == 0) {
                    const float rg = ref_g == -INFINITY ? 0.f : ref_g;
                    const float rg8 = ref_g8 == -INFINITY ? 0.f : ref_g8;
                    const float beta_g = fast_exp2(rg - Mg), beta_g8 = fast_exp2(rg8 - Mg8);
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        sa[e] *= e < 2 ? beta_g : beta_g8;
                        sb[e] *= e < 2 ? beta_g : beta_g8;
                    }
                    l_g *= alpha_g;
                    l_g8 *= alpha_g8;
                    uint8_t* pb = smem + OFF_P;
                    *reinterpret_cast<uint32_t*>(pb + g * P_PITCH + r0 * 2) = pack_half2(sa[0], sa[1]);
                    *reinterpret_cast<uint32_t*>(pb + (g + 8) * P_PITCH + r0 * 2) =
                        pack_half2(sa[2], sa[3]);
                    *reinterpret_cast<uint32_t*>(pb + g * P_PITCH + (BR + r0) * 2) =
                        pack_half2(sb[0], sb[1]);
                    *reinterpret_cast<uint32_t*>(pb + (g + 8) * P_PITCH + (BR + r0) * 2) =
                        pack_half2(sb[2], sb[3]);
                }
                m_g = M_g;
                m_g8 = M_g8;
                named_barrier(CONSUMER_BAR, CTHREADS);   // rescaled P visible
            }
            if (kh == 0) {
                l_g += (sa[0] + sa[1]) + (sb[0] + sb[1]);
                l_g8 += (sa[2] + sa[3]) + (sb[2] + sb[3]);
            }
            ++rr;

            // ---- O += P . V over value dims 64w .. 64w+63, 32 or 64 rows
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
                if (ks >= 2 && !two) break;
                uint32_t a[4];
                ldsm_x4(sbase + OFF_P + ar * P_PITCH + (ks * 16 + hi * 8) * 2, a[0], a[1], a[2], a[3]);
                const uint32_t vslot = ks < 2 ? slot_a : slot_b;
                const int vr = (ks & 1) * 16 + ar;
#pragma unroll
                for (int np = 0; np < 4; ++np) {
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_trans(chunk_addr(vslot, vr, 8 * warp + 2 * np + hi), b0, b1, b2, b3);
                    mma_16816(o[2 * np], a, b0, b1);
                    mma_16816(o[2 * np + 1], a, b2, b3);
                }
            }
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(empty_bar(q % NS));
                if (two) mbar_arrive(empty_bar((q + 1) % NS));
            }

            if (last) {
                // ---- last block of the token: normalise and store
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
                named_barrier(CONSUMER_BAR, CTHREADS);
                const float L_g = red_sum[g] + red_sum[H + g] + red_sum[2 * H + g] + red_sum[3 * H + g];
                const float L_g8 = red_sum[g + 8] + red_sum[H + g + 8] + red_sum[2 * H + g + 8] +
                                   red_sum[3 * H + g + 8];
                const float inv_g = L_g > 0.f ? 1.f / L_g : 0.f;
                const float inv_g8 = L_g8 > 0.f ? 1.f / L_g8 : 0.f;
                float* ot = p.out + (size_t)cu.tr.i * H * DV;
#pragma unroll
                for (int n = 0; n < 8; ++n) {
                    const int d = 64 * warp + 8 * n + 2 * c;
                    *reinterpret_cast<float2*>(ot + g * DV + d) =
                        make_float2(o[n][0] * inv_g, o[n][1] * inv_g);
                    *reinterpret_cast<float2*>(ot + (g + 8) * DV + d) =
                        make_float2(o[n][2] * inv_g8, o[n][3] * inv_g8);
                }
            }
            q += two ? 2 : 1;
            cu.advance(p);
            if (two) cu.advance(p);
        }
    }
    __syncthreads();
}

}  // namespace ds4sp
