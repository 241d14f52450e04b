// Streaming sparse MLA attention: 16 heads share every gathered latent row.
//
// For token t the attended rows are the selected compressed rows (top-k, ascending
// j) followed by the raw rows max(0, t-n_swa+1) .. t; one softmax runs over all of
// them. Key = the row's 576 dims, value = its first 512 dims. "perf(ds4): extend
// sparse prefill scheduling to 10K", Summary: "keep selected raw/compressed KV
// transport in F16, and stream each selected latent row once across sixteen ...
// heads". The per-token visibility (n_vis = (t+1)/4, window bounds) is computed
// here from t; no mask is stored. (A debug form takes the compressed rows' visibility
// from a stored mask instead, for the page's "explicit-mask versus analytic-mask"
// check, Qualification section: see AttnParams::vis_mask.)
//
// Persistent CTAs (one per SM) take every gridDim-th token, heaviest first. A token
// is a sequence of units: one unit holding its Q (16 rows), then its rows in blocks of
// 32. Two consumer groups work on different tokens at once (group g takes the CTA's
// tokens g, g+2, ...), so one group's softmax and barriers overlap the other group's
// tensor-core work. The two groups' unit sequences are merged, one unit of each in
// turn, into one stream through a 5-slot shared-memory ring with an mbarrier pair
// per slot; producers and both groups walk the same merged order.
//   * Warps 8-11 produce (8-15 for the quantized caches, whose dequantization needs the
//     extra warps). They stage each token's top-k row in shared memory one
//     token ahead per group, resolve and check every row, and copy it in 16-byte chunks
//     with cp.async; cp.async.mbarrier.arrive.noinc lets the slot's barrier count the
//     copies without the producer waiting for them. Each producer warp also publishes
//     which of its rows are valid. Producers never take part in the consumers'
//     barriers, and setmaxnreg moves most of their registers to the consumers.
//   * Warps 4g .. 4g+3 form consumer group g, with the 16 heads as the M of
//     mma.sync.m16n8k16. Group warp w (kh = w/2, rh = w%2) computes the partial
//     S = Q . R^T of rows 16rh .. 16rh+15 over K half kh (288 dims), Q's half held in
//     registers; the halves meet in shared memory and warp w completes and
//     normalises the 8-row tile 2rh+kh. Softmax runs against a running reference max
//     that is raised only when a tile's max exceeds it by more than 2^8 (probabilities
//     stay <= 256, fine in fp16): a unit normally needs two group barriers; raising the
//     reference rescales O, the sums and that unit's P. O += P . V: group warp w owns
//     value dims 128w .. 128w+127.
// Rows are stored unpadded with their 16-byte chunks XOR-swizzled, which keeps the
// producers' copies and the consumers' ldmatrix reads free of bank conflicts.
// fp32 logits, sums and output; P enters P . V as fp16 (or, in the fp32-staged
// instantiation, as the sum of two fp16 terms hi + lo, lo = fp16(p - hi), at twice the
// P . V tensor work); exponentials on ex2.approx (or exp2f in the precise instantiation).
// Every wait is bounded; a consumer that gives up sets its group's flag, which the
// group's warps read after their next barrier, so none is left waiting.
#pragma once

#include "device_common.cuh"
#include "quant_kv.cuh"

namespace ds4sp {
namespace attn {

constexpr int H = 16;
constexpr int DQK = 576;
constexpr int DV = 512;
constexpr int ROW = DQK * 2;                  // 1152 bytes per latent row
constexpr int CH = ROW / 16;                  // 72 sixteen-byte chunks per row
constexpr int BR = 32;                        // rows per unit
constexpr int NS = 5;                         // ring slots
constexpr int GROUPS = 2;                     // consumer groups, each on its own token
constexpr int GWARPS = 4;                     // warps per consumer group
constexpr int CWARPS = GROUPS * GWARPS;       // consumer warps
constexpr int GTHREADS = GWARPS * 32;
constexpr int CTHREADS = CWARPS * 32;
constexpr int PRODUCER_BAR = 1;               // named barriers; group g uses GROUP_BAR + g
constexpr int GROUP_BAR = 2;
// Registers per thread: the kernel is built for Roles<KVF>::LAUNCH_REGS (one CTA per
// SM); producers hand part of theirs to the consumers with setmaxnreg. The host checks
// the built count before the first launch: a split above the launch's total would
// leave the consumers' setmaxnreg.inc waiting.
constexpr float HEADROOM = 8.f;               // log2 units a tile may exceed the reference
constexpr int SLOT = BR * ROW;
constexpr int P_PITCH = (BR + 8) * 2;         // fp16 probabilities of one unit, 80 B per head
constexpr int IDX_BUFS = 2;                   // per group: top-k rows of this token, the next
// Per-group areas.
constexpr int P_BYTES = H * P_PITCH;
constexpr int X_BYTES = 4 * 32 * 16;          // S partials passed between the K halves
constexpr int REF_BYTES = 4 * H * 4;          // per S tile: reference used for its P
constexpr int RED_BYTES = GWARPS * H * 4;     // per warp: softmax sums of a finished token
constexpr int FLAG_BYTES = 16;                // raised[2], abort, pad
constexpr int G_BYTES = 2 * P_BYTES + X_BYTES + REF_BYTES + RED_BYTES + FLAG_BYTES;
constexpr int G_P = 0, G_PLO = P_BYTES, G_X = 2 * P_BYTES, G_REF = G_X + X_BYTES,
              G_RED = G_REF + REF_BYTES, G_FLAGS = G_RED + RED_BYTES;
constexpr int MAX_TOPK = 2048;
constexpr int SMEM_LIMIT = 227 * 1024;
constexpr int ROWV = DV * 2;                  // 1024 bytes: a separate value row

// Shared-memory layout of the kernel for a cache format: NS ring slots of BR rows, each
// row 1152 bytes (key = the row's 576 values; value = its first 512), or, for the
// "Q8 K / Q4 V" format whose keys and values differ, a 1152-byte key row plus a
// 1024-byte value row (the value rows of a slot follow its key rows); then the groups'
// areas, the row-validity bits, the barriers and the staged top-k rows.
template <int KVF>
struct RingLayout {
    static constexpr bool SPLIT = KVF == kFmtQ8Q4;
    // Q8_0 and Q4_0 rows are staged: the producers copy a unit's quantized rows into one
    // of two staging buffers a unit ahead and dequantize from there into the ring.
    static constexpr bool STAGED = KVF == kFmtQ8 || KVF == kFmtQ4;
    static constexpr int NS_ = SPLIT ? 3 : KVF == kFmtQ8 ? 4 : NS;
    static constexpr int VOFF = BR * ROW;                   // value rows within a slot
    static constexpr int SLOT_ = SPLIT ? BR * (ROW + ROWV) : SLOT;
    static constexpr int QROW = STAGED ? quant_row_bytes(KVF, DQK) : 0;   // a stored row
    static constexpr int STAGE = BR * QROW;                 // one staging buffer
    static constexpr int OFF_RING = 0;
    static constexpr int OFF_GROUP = OFF_RING + NS_ * SLOT_;
    // Row-validity bytes per slot: one per producer warp (four, or eight for the
    // quantized formats' eight producer warps).
    static constexpr int MASK_STRIDE = STAGED || SPLIT ? 8 : 4;
    static constexpr int OFF_MASK = OFF_GROUP + GROUPS * G_BYTES;
    static constexpr int OFF_BAR = OFF_MASK + 8 * MASK_STRIDE;      // full[NS_], empty[NS_]
    static constexpr int OFF_STAGE = OFF_BAR + 2 * NS_ * 8;
    static constexpr int OFF_IDX = OFF_STAGE + 2 * STAGE;
    __host__ __device__ static constexpr int smem_bytes(int k) {
        return OFF_IDX + GROUPS * IDX_BUFS * ((k + 3) / 4 * 4) * 4;
    }
    // the largest top_k whose staged rows fit
    static constexpr int MAX_K = (SMEM_LIMIT - OFF_IDX) / (GROUPS * IDX_BUFS * 4) / 4 * 4 < MAX_TOPK
                                     ? (SMEM_LIMIT - OFF_IDX) / (GROUPS * IDX_BUFS * 4) / 4 * 4
                                     : MAX_TOPK;
    static_assert(NS_ <= 8, "row-validity bytes for at most 8 slots");
    static_assert(G_BYTES % 16 == 0 && OFF_GROUP % 16 == 0, "16-byte aligned group areas");
    static_assert(smem_bytes(MAX_K) <= SMEM_LIMIT, "shared memory budget");
};
__host__ __device__ constexpr int smem_bytes(int k) { return RingLayout<kFmtF16>::smem_bytes(k); }

// Producer warps of a cache format: four (eight rows of the unit each, four lanes a row)
// for fp16 rows and the split format; eight (four rows each, eight lanes a row) for the
// staged Q8_0 / Q4_0 rows, whose dequantization is the producers' limit. The register
// split keeps the launch's 64K registers: consumers 224 / producers 56 at 384 threads,
// 200 / 56 at 512.
template <int KVF>
struct Roles {
    // producer warps: eight for the quantized formats, whose producers dequantize
    static constexpr int PW = RingLayout<KVF>::STAGED || RingLayout<KVF>::SPLIT ? 8 : 4;
    static constexpr int PT = PW * 32;
    static constexpr int THREADS = CTHREADS + PT;
    static constexpr int RPW = BR / PW;          // rows per producer warp
    static constexpr int LPR = 32 / RPW;         // lanes per row
    static constexpr int LPR_LOG2 = LPR == 8 ? 3 : 2;
    static constexpr int LAUNCH_REGS = 65536 / THREADS / 8 * 8;
    static constexpr int PREGS = 56;
    static constexpr int CREGS = (THREADS * LAUNCH_REGS - PT * PREGS) / CTHREADS / 8 * 8;
    static_assert(CREGS <= 224 && CWARPS * 32 * CREGS + PT * PREGS <= THREADS * LAUNCH_REGS,
                  "register split must fit the launch's registers");
    static_assert(RPW * PW == BR && LPR * RPW == 32 && (1 << LPR_LOG2) == LPR,
                  "whole rows per producer warp");
    static_assert(CH % LPR == 0, "a row's chunks split evenly over its lanes");
    static_assert(PW == RingLayout<KVF>::MASK_STRIDE, "one row-validity byte per producer warp");
};
static_assert(DV == GWARPS * 128, "each group warp owns 128 value dims");
static_assert(CH % 8 == 0, "whole 128-byte swizzle groups per row");
static_assert(RingLayout<kFmtF16>::MAX_K == MAX_TOPK, "fp16 ring holds top_k up to 2048");

// 16-byte chunk swizzle: eight consecutive rows put one chunk in eight different bank
// groups (ldmatrix), and rows 2m, 2m+1 put an aligned group of four chunks in
// complementary halves (a quarter warp's cp.async).
__device__ __forceinline__ int swz(int row) { return ((row & 1) << 2) | ((row >> 1) & 3); }
__device__ __forceinline__ uint32_t chunk_addr(uint32_t slot, int row, int chunk) {
    return slot + row * ROW + ((chunk ^ swz(row)) << 4);
}
// The same swizzle for rows of `pitch` bytes (a multiple of 128) from `base`.
__device__ __forceinline__ uint32_t chunk_addr_p(uint32_t base, int row, int chunk, int pitch) {
    return base + row * pitch + ((chunk ^ swz(row)) << 4);
}

}  // namespace attn

struct AttnParams {
    const __half* q;       // [n_q, 16, 576], row 0 = token t0
    const __half* kv_raw;  // [>= t0+n_q, 576]
    const __half* kv_cmp;  // [>= n_vis(t0+n_q-1), 576]
    const int32_t* topk;   // [n_q, k]
    float* out;            // [n_q, 16, 512]
    WaitCtl wc;            // bounded waits of this launch; wc.status also takes index errors
    int t0, n_q, k, n_swa, ratio;
    float scale_log2;      // softmax scale * log2(e)
    // Optional: a region the next kernel will read (the next band's indexer queries);
    // once a CTA's producers have issued their last copy they ask L2 to fetch this CTA's
    // slice of it, while the consumers finish. NULL or 0 bytes: nothing.
    const char* prefetch;
    long long prefetch_bytes;
    // Split mode (few tokens): when `split` is set, a work item is one 32-row unit of a
    // token rather than the whole token, items come in token order (the units of token
    // 0, then token 1, ...), and each item writes its unnormalised O with its reference
    // max and softmax sum to part_o / part_ml for attn_merge_kernel.
    int split, n_items;
    float* part_o;         // [n_items, 16, 512]
    float* part_ml;        // [n_items, 2, 16]: reference max (log2 units), sum
    // Explicit-mask form (debug): when set, a top-k entry j is attended iff
    // 0 <= j < mask_cols and vis_mask[t * mask_ld + j] != 0, in place of j < n_vis(t);
    // -1 entries and entries the mask hides are dropped without a status bit (the
    // top-k of this form pads with -1 when the mask leaves fewer than k rows).
    const uint8_t* vis_mask;
    long long mask_ld;
    int mask_cols;
    // Quantized cache (kernel instantiations with KVF != 0): kv_raw and kv_cmp hold rows
    // of quant_row_bytes(KVF, 576) bytes, which the producers dequantize into the ring.
    int kv_row_bytes;
};

// A work item: the token (i, t and its rows) and the run of its 32-row units it covers,
// units u0 .. u0+nblk-1 (0-based) of the token's nrows rows.
struct TokenRows {
    int i, t, nv, nsel, s_lo, nrows, nblk, u0, item;
};

__device__ __forceinline__ TokenRows token_rows_of(const AttnParams& p, int i) {
    TokenRows r;
    r.i = i;
    r.t = p.t0 + i;
    r.nv = n_vis(r.t, p.ratio);
    r.nsel = min(p.k, r.nv);
    r.s_lo = max(0, r.t - p.n_swa + 1);
    r.nrows = r.nsel + (r.t - r.s_lo + 1);
    r.nblk = (r.nrows + attn::BR - 1) / attn::BR;
    r.u0 = 0;
    r.item = i;
    return r;
}

__device__ __forceinline__ TokenRows token_rows(const AttnParams& p, int idx) {
    if (!p.split) return token_rows_of(p, p.n_q - 1 - idx);   // heaviest (latest) first
    // Item idx is unit (idx - units of tokens before) of the token that holds it.
    int i = 0, before = 0;
    TokenRows r = token_rows_of(p, 0);
    while (before + r.nblk <= idx && i + 1 < p.n_q) {
        before += r.nblk;
        r = token_rows_of(p, ++i);
    }
    r.u0 = idx - before;
    r.nblk = 1;
    r.item = idx;
    return r;
}

// One consumer group's position: its m-th token (the CTA's token number g + 2m),
// unit u of it (0 = Q, 1.. = row blocks).
struct GroupCursor {
    int m, idx, u;
    TokenRows tr;
    bool valid;
    __device__ __forceinline__ void start(const AttnParams& p, int g) {
        m = 0;
        idx = blockIdx.x + g * gridDim.x;
        u = 0;
        valid = idx < p.n_items;
        if (valid) tr = token_rows(p, idx);
    }
    __device__ __forceinline__ void advance(const AttnParams& p) {
        if (++u > tr.nblk) {
            u = 0;
            ++m;
            idx += attn::GROUPS * gridDim.x;
            valid = idx < p.n_items;
            if (valid) tr = token_rows(p, idx);
        }
    }
};

// The ring's unit order: one unit of each group in turn while both have units left,
// then the remaining group's units. `turn` is the group of the current unit. (Two named
// cursors rather than an array indexed by `turn`, which would live in local memory.)
struct MergedCursor {
    GroupCursor c0, c1;
    int turn;
    __device__ __forceinline__ void start(const AttnParams& p) {
        c0.start(p, 0);
        c1.start(p, 1);
        turn = c0.valid ? 0 : 1;
    }
    __device__ __forceinline__ const GroupCursor& group(int g) const { return g ? c1 : c0; }
    __device__ __forceinline__ bool valid() const { return turn ? c1.valid : c0.valid; }
    __device__ __forceinline__ void advance(const AttnParams& p) {
        if (turn) {
            c1.advance(p);
            if (c0.valid) turn = 0;
        } else {
            c0.advance(p);
            if (c1.valid) turn = 1;
        }
    }
};

__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

// Producer side of a quantized cache: this lane's blocks of one stored row part (lane l
// of the row's LPR takes blocks l, l+LPR, l+2*LPR, ...), loaded as 16-byte words,
// dequantized to fp16 and stored as four 16-byte chunks per block into ring row r of
// `pitch` bytes from `base`; a masked row stores zeros. FMT is Q8_0 or Q4_0 and NB the
// part's blocks.
template <int FMT, int NB, int LPR>
__device__ __forceinline__ void dequant_part_to_ring(const uint8_t* rowq, bool ok, uint32_t base,
                                                     int pitch, int r, int sub) {
    using attn::chunk_addr_p;
    constexpr int CB = quant_code_bytes(FMT, NB * kQBlock);
    constexpr int W = FMT == kFmtQ8 ? 2 : 1;             // 16-byte words per block
    constexpr int BATCH = FMT == kFmtQ8 ? 2 : 3;         // blocks whose loads fly together
    if (!ok) {
        for (int m = sub; m < NB; m += LPR)
#pragma unroll
            for (int k = 0; k < 4; ++k) st_shared_v4(chunk_addr_p(base, r, 4 * m + k, pitch), make_uint4(0, 0, 0, 0));
        return;
    }
    for (int m0 = sub; m0 < NB; m0 += LPR * BATCH) {
        uint4 c[BATCH][W];
        __half2 d2[BATCH];
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
            const int m = m0 + LPR * i;
            if (m < NB) {
                const uint4* src = reinterpret_cast<const uint4*>(rowq + m * 16 * W);
#pragma unroll
                for (int h = 0; h < W; ++h) c[i][h] = __ldg(src + h);
                d2[i] = __half2half2(*reinterpret_cast<const __half*>(rowq + CB + 2 * m));
            }
        }
#pragma unroll
        for (int i = 0; i < BATCH; ++i) {
            const int m = m0 + LPR * i;
            if (m >= NB) continue;
            if constexpr (FMT == kFmtQ8) {
                st_shared_v4(chunk_addr_p(base, r, 4 * m + 0, pitch), dequant_q8_chunk(c[i][0].x, c[i][0].y, d2[i]));
                st_shared_v4(chunk_addr_p(base, r, 4 * m + 1, pitch), dequant_q8_chunk(c[i][0].z, c[i][0].w, d2[i]));
                st_shared_v4(chunk_addr_p(base, r, 4 * m + 2, pitch), dequant_q8_chunk(c[i][1].x, c[i][1].y, d2[i]));
                st_shared_v4(chunk_addr_p(base, r, 4 * m + 3, pitch), dequant_q8_chunk(c[i][1].z, c[i][1].w, d2[i]));
            } else {
                const uint4 w = c[i][0];
                const uint32_t M = 0x0F0F0F0Fu;
                st_shared_v4(chunk_addr_p(base, r, 4 * m + 0, pitch), dequant_q4_chunk(w.x & M, w.y & M, d2[i]));
                st_shared_v4(chunk_addr_p(base, r, 4 * m + 1, pitch), dequant_q4_chunk(w.z & M, w.w & M, d2[i]));
                st_shared_v4(chunk_addr_p(base, r, 4 * m + 2, pitch),
                             dequant_q4_chunk((w.x >> 4) & M, (w.y >> 4) & M, d2[i]));
                st_shared_v4(chunk_addr_p(base, r, 4 * m + 3, pitch),
                             dequant_q4_chunk((w.z >> 4) & M, (w.w >> 4) & M, d2[i]));
            }
        }
    }
}

// Staged quantized rows (Q8_0, Q4_0). Lane `sub` of a row's LPR copies the code bytes of
// blocks sub, sub+LPR, ... and, for sub < 3, one 16-byte piece of the scales, to the same
// byte offsets of a staging row; it later dequantizes the same blocks (its own copies,
// plus the scales its row's lanes copied, once the warp has synchronised).
template <int FMT, int LPR>
__device__ __forceinline__ void stage_row_copy(const uint8_t* rowq, uint32_t srow, int sub) {
    constexpr int NB = attn::DQK / kQBlock;
    constexpr int CB = quant_code_bytes(FMT, attn::DQK);
    constexpr int W = FMT == kFmtQ8 ? 2 : 1;
    for (int m = sub; m < NB; m += LPR)
#pragma unroll
        for (int h = 0; h < W; ++h) cp_async_16(srow + (m * W + h) * 16, rowq + (m * W + h) * 16, true);
    if (sub < 3) cp_async_16(srow + CB + 16 * sub, rowq + CB + 16 * sub, true);
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr));
    return v;
}

__device__ __forceinline__ uint32_t ld_shared_u16(uint32_t addr) {
    unsigned short v;
    asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(addr));
    return v;
}

// Lane `sub` of the row's LPR: blocks sub, sub+LPR, ... of the staged row into ring row r.
template <int FMT, int LPR>
__device__ __forceinline__ void dequant_staged_to_ring(uint32_t srow, bool ok, uint32_t dst, int r,
                                                       int sub) {
    using attn::chunk_addr;
    constexpr int NB = attn::DQK / kQBlock;
    constexpr int CB = quant_code_bytes(FMT, attn::DQK);
    for (int m = sub; m < NB; m += LPR) {
        if (!ok) {
#pragma unroll
            for (int k = 0; k < 4; ++k) st_shared_v4(chunk_addr(dst, r, 4 * m + k), make_uint4(0, 0, 0, 0));
            continue;
        }
        const unsigned short dbits = (unsigned short)ld_shared_u16(srow + CB + 2 * m);
        const __half2 d2 = __half2half2(__ushort_as_half(dbits));
        if constexpr (FMT == kFmtQ8) {
            const uint4 c0 = ld_shared_v4(srow + 32 * m), c1 = ld_shared_v4(srow + 32 * m + 16);
            st_shared_v4(chunk_addr(dst, r, 4 * m + 0), dequant_q8_chunk(c0.x, c0.y, d2));
            st_shared_v4(chunk_addr(dst, r, 4 * m + 1), dequant_q8_chunk(c0.z, c0.w, d2));
            st_shared_v4(chunk_addr(dst, r, 4 * m + 2), dequant_q8_chunk(c1.x, c1.y, d2));
            st_shared_v4(chunk_addr(dst, r, 4 * m + 3), dequant_q8_chunk(c1.z, c1.w, d2));
        } else {
            const uint4 w = ld_shared_v4(srow + 16 * m);
            const uint32_t M = 0x0F0F0F0Fu;
            st_shared_v4(chunk_addr(dst, r, 4 * m + 0), dequant_q4_chunk(w.x & M, w.y & M, d2));
            st_shared_v4(chunk_addr(dst, r, 4 * m + 1), dequant_q4_chunk(w.z & M, w.w & M, d2));
            st_shared_v4(chunk_addr(dst, r, 4 * m + 2), dequant_q4_chunk((w.x >> 4) & M, (w.y >> 4) & M, d2));
            st_shared_v4(chunk_addr(dst, r, 4 * m + 3), dequant_q4_chunk((w.z >> 4) & M, (w.w >> 4) & M, d2));
        }
    }
}

// A stored row of the cache format into ring row r of the slot at `dst` (this lane's
// blocks: lane `sub` of the row's LPR).
template <int KVF, int LPR>
__device__ __forceinline__ void dequant_row_to_ring(const uint8_t* rowq, bool ok, uint32_t dst,
                                                    int r, int sub) {
    using namespace attn;
    constexpr int NB = DQK / kQBlock;                        // 18 key blocks
    if constexpr (KVF == kFmtQ8Q4) {
        dequant_part_to_ring<kFmtQ8, NB, LPR>(rowq, ok, dst, ROW, r, sub);
        dequant_part_to_ring<kFmtQ4, DV / kQBlock, LPR>(rowq + quant_row_bytes(kFmtQ8, DQK), ok,
                                                        dst + RingLayout<KVF>::VOFF, ROWV, r, sub);
    } else {
        dequant_part_to_ring<KVF, NB, LPR>(rowq, ok, dst, ROW, r, sub);
    }
}

// PRECISE selects exp2f for the softmax exponentials instead of ex2.approx; PSPLIT the
// fp32-staged probabilities; KVF the cache format (kFmtF16, or a quantized one whose rows
// the producers dequantize).
template <bool PRECISE, bool PSPLIT, int KVF>
__global__ void __launch_bounds__(attn::Roles<KVF>::THREADS, 1) sparse_attn_mma_kernel(AttnParams p) {
    using namespace attn;
    using L = RingLayout<KVF>;
    using R = Roles<KVF>;
    auto exp2_ = [](float x) { return PRECISE ? exp2f(x) : fast_exp2(x); };
    extern __shared__ __align__(128) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
    const int kpad = (p.k + 3) / 4 * 4;
    // Row validity of each slot: byte w of the slot's MASK_STRIDE holds producer warp w's
    // rows, row RPW*w + i in bit i (so with eight rows a warp, bit r of the slot's word).
    volatile uint8_t* rowmask = reinterpret_cast<volatile uint8_t*>(smem + L::OFF_MASK);
    const uint32_t bar0 = sbase + L::OFF_BAR;
    auto full_bar = [&](int s) { return bar0 + 8u * s; };
    auto empty_bar = [&](int s) { return bar0 + 8u * (L::NS_ + s); };

    if (tid == 0) {
        for (int s = 0; s < L::NS_; ++s) {
            mbar_init(full_bar(s), R::PT + R::PW);       // noinc copy arrivals + mask writers
            mbar_init(empty_bar(s), GWARPS);             // the owning group's warps
        }
        for (int g = 0; g < GROUPS; ++g) {
            volatile int* f = reinterpret_cast<volatile int*>(smem + L::OFF_GROUP + g * G_BYTES + G_FLAGS);
            f[0] = f[1] = f[2] = 0;
        }
        fence_mbar_init();
    }
    __syncthreads();
    // Global memory only after the previous kernel of the stream has completed (the
    // prologue above may overlap it when launched as a programmatic dependent).
    grid_dependency_wait();
    grid_dependents_launch();

    bool abort = false;
    if (warp >= CWARPS) {
        // ================================================================ producers
        regs_decrease<R::PREGS>();
        const int ptid = tid - CTHREADS, pw = warp - CWARPS;
        const int sub = lane & (R::LPR - 1);      // this lane's part of its row
        auto idx_buf = [&](int g, int m) { return L::OFF_IDX + (g * IDX_BUFS + (m & 1)) * kpad * 4; };
        auto stage_idx = [&](int g, int m) {      // top-k row of group g's m-th token
            const int idx = blockIdx.x + (g + GROUPS * m) * gridDim.x;
            if (idx >= p.n_items) return;
            const TokenRows nx = token_rows(p, idx);
            const int32_t* src = p.topk + (size_t)nx.i * p.k;
            const uint32_t dst = sbase + idx_buf(g, m);
            for (int e = ptid; e < nx.nsel; e += R::PT)
                asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(dst + 4 * e),
                             "l"(src + e)
                             : "memory");
        };
        stage_idx(0, 0);
        stage_idx(1, 0);
        cp_async_commit();
        cp_async_wait<0>();
        named_barrier(PRODUCER_BAR, R::PT);
        // Row r of group g's current unit: a selected compressed row (index checked; with
        // `report`, an out-of-range entry sets the status word) or a window row.
        auto resolve_row = [&](int g, const GroupCursor& cu, int r, long long& src_row, bool& cmp,
                               bool report) {
            const int* tk = reinterpret_cast<const int*>(smem + idx_buf(g, cu.m));
            const int gr = (cu.tr.u0 + cu.u - 1) * BR + r;
            src_row = 0;
            cmp = false;
            if (gr < cu.tr.nsel) {
                const int j = tk[gr];
                if (p.vis_mask == nullptr) {
                    if (j >= 0 && j < cu.tr.nv) {
                        src_row = j;
                        cmp = true;
                        return true;
                    }
                    if (report && sub == 0) record_status(p.wc.status, kStatusBounds);
                    return false;
                }
                if (j >= 0 && j < p.mask_cols) {
                    if (p.vis_mask[(size_t)cu.tr.t * p.mask_ld + j] != 0) {
                        src_row = j;
                        cmp = true;
                        return true;
                    }
                    return false;
                }
                if (j != -1 && report && sub == 0) record_status(p.wc.status, kStatusBounds);
                return false;
            }
            if (gr < cu.tr.nrows) {
                src_row = cu.tr.s_lo + gr - cu.tr.nsel;
                return true;
            }
            return false;
        };
        auto stage_buf = [&](int uc) { return sbase + L::OFF_STAGE + (uc & 1) * L::STAGE; };
        // Staged formats: copy the rows of the unit after `uc` (if it is a row unit) into
        // the other staging buffer; this lane's row and blocks only.
        auto stage_next = [&](const MergedCursor& at, int uc) {
            MergedCursor nx = at;
            nx.advance(p);
            if (nx.valid()) {
                const GroupCursor cn = nx.group(nx.turn);
                if (cn.u != 0) {
                    const int r = R::RPW * pw + (lane >> R::LPR_LOG2);
                    long long src_row;
                    bool cmp;
                    if (resolve_row(nx.turn, cn, r, src_row, cmp, false)) {
                        const uint8_t* base_q = reinterpret_cast<const uint8_t*>(cmp ? p.kv_cmp : p.kv_raw);
                        stage_row_copy<KVF == kFmtQ8 ? kFmtQ8 : kFmtQ4, R::LPR>(
                            base_q + (size_t)src_row * p.kv_row_bytes, stage_buf(uc + 1) + r * L::QROW,
                            sub);
                    }
                }
            }
            cp_async_commit();
        };
        MergedCursor mc;
        mc.start(p);
        // A producer warp whose wait gives up stops copying but keeps walking the units
        // (its waits then return at once), so that it still meets every producer barrier
        // that the other producer warps reach.
        for (int uc = 0; mc.valid(); ++uc, mc.advance(p)) {
            const int s = uc % L::NS_;
            if (!abort &&
                !__all_sync(0xffffffffu, mbar_wait<true>(empty_bar(s), ((uc / L::NS_) & 1) ^ 1, p.wc, abort)))
                abort = true;                      // the whole warp gives up together
            const uint32_t dst = sbase + L::OFF_RING + s * L::SLOT_;
            const GroupCursor cu = mc.group(mc.turn);
            if (cu.u == 0) {
                if (!abort) {
                    // Q of the token, and the group's next top-k row one token ahead.
                    stage_idx(mc.turn, cu.m + 1);
                    const __half* qt = p.q + (size_t)cu.tr.i * H * DQK;
#pragma unroll
                    for (int m = 0; m < (H * CH + R::PT - 1) / R::PT; ++m) {
                        const int e = ptid + m * R::PT, r = e / CH, ch = e % CH;
                        if (H * CH % R::PT == 0 || e < H * CH)
                            cp_async_16(chunk_addr(dst, r, ch), qt + r * DQK + ch * 8, true);
                    }
                    cp_async_commit();
                    cp_async_arrive_noinc(full_bar(s));
                    __syncwarp();
                    if (lane == 0) mbar_arrive(full_bar(s));
                    // This token's top-k row (staged at the group's previous Q unit, an
                    // earlier commit group) must be in shared memory, for every producer
                    // thread, before its row units are resolved.
                    cp_async_wait<1>();
                }
                named_barrier(PRODUCER_BAR, R::PT);
                if constexpr (L::STAGED)
                    if (!abort) stage_next(mc, uc);   // the top-k rows it needs are in place
                continue;
            }
            if (abort) continue;
            const int r = R::RPW * pw + (lane >> R::LPR_LOG2);   // this lane's row of the unit
            long long src_row = 0;
            bool cmp = false;
            const bool ok = resolve_row(mc.turn, cu, r, src_row, cmp, true);
            if constexpr (L::STAGED) {
                // this unit's rows were copied to staging[uc & 1] one unit ago; copy the next
                // unit's rows to the other buffer, then dequantize this one into the slot
                cp_async_wait<0>();
                __syncwarp();
                stage_next(mc, uc);
                dequant_staged_to_ring<KVF, R::LPR>(stage_buf(uc) + r * L::QROW, ok, dst, r, sub);
                mbar_arrive(full_bar(s));          // release: this thread's stores are visible
            } else if constexpr (KVF == kFmtF16) {
                const __half* row = ok ? (cmp ? p.kv_cmp : p.kv_raw) + (size_t)src_row * DQK
                                       : p.kv_raw + (size_t)cu.tr.t * DQK;   // valid stand-in
#pragma unroll
                for (int m = 0; m < CH / R::LPR; ++m) {
                    const int ch = sub + R::LPR * m;
                    cp_async_16(chunk_addr(dst, r, ch), row + ch * 8, ok);   // zero-filled if masked
                }
                cp_async_arrive_noinc(full_bar(s));
            } else {
                const uint8_t* base_q = reinterpret_cast<const uint8_t*>(cmp ? p.kv_cmp : p.kv_raw);
                dequant_row_to_ring<KVF, R::LPR>(base_q + (size_t)src_row * p.kv_row_bytes, ok, dst, r, sub);
                mbar_arrive(full_bar(s));          // release: this thread's stores are visible
            }
            const uint32_t bits = __ballot_sync(0xffffffffu, ok && sub == 0);
            if (lane == 0) {
                uint32_t m8 = 0;
#pragma unroll
                for (int i = 0; i < R::RPW; ++i) m8 |= ((bits >> (R::LPR * i)) & 1u) << i;
                rowmask[L::MASK_STRIDE * s + pw] = (uint8_t)m8;
                mbar_arrive(full_bar(s));         // release: the mask byte is visible with the slot
            }
            if constexpr (L::STAGED) __syncwarp();   // staging[uc & 1] is read before its reuse
        }
        if (p.prefetch_bytes > 0 && !abort) {
            // This CTA's slice of the region, in 16-byte-aligned pieces of up to 32 KB,
            // spread over the producer warps' first lanes.
            const long long per = (p.prefetch_bytes / gridDim.x + 15) / 16 * 16;
            const long long lo = per * blockIdx.x;
            const long long hi = min(p.prefetch_bytes, lo + per);
            if (lane == 0)
                for (long long off = lo + (long long)pw * 32768; off < hi; off += R::PW * 32768LL)
                    prefetch_l2(p.prefetch + off, (uint32_t)min(32768LL, hi - off));
        }
        cp_async_wait<0>();
    } else {
        // ================================================================ consumers
        regs_increase<R::CREGS>();
        const int grp = warp / GWARPS, gw = warp % GWARPS;
        const int gbar = GROUP_BAR + grp;
        uint8_t* garea = smem + L::OFF_GROUP + grp * G_BYTES;
        const uint32_t pbase = sbase + L::OFF_GROUP + grp * G_BYTES + G_P;
        const uint32_t plobase = sbase + L::OFF_GROUP + grp * G_BYTES + G_PLO;
        float4* xbuf = reinterpret_cast<float4*>(garea + G_X);
        float* ref_tile = reinterpret_cast<float*>(garea + G_REF);
        float* red_sum = reinterpret_cast<float*>(garea + G_RED);
        volatile int* flags = reinterpret_cast<volatile int*>(garea + G_FLAGS);  // raised[2], abort
        const int g = lane / 4, c = lane % 4;    // mma fragment coordinates
        const int kh = gw >> 1, rh = gw & 1;     // S: K half, row half (rows 16rh .. 16rh+15)
        const int own = 2 * rh + kh;             // the 8-row S tile this warp completes
        const int give = 2 * rh + (kh ^ 1);      // the partner's tile
        const int r0 = 8 * own + 2 * c;          // S columns of this lane: unit rows r0, r0+1
        const int rlo = 16 * rh + (lane & 7);    // S: this lane's ldmatrix row, first tile
        const int ar = (lane & 7) + ((lane >> 3) & 1) * 8, hi = lane >> 4;
        uint32_t qf[18][4];
        float o[16][4];
        float m_g = -INFINITY, m_g8 = -INFINITY; // reference max, heads g and g+8 (log2 units)
        float l_g = 0.f, l_g8 = 0.f;             // this warp's share of the softmax sums
        auto wait_full = [&](int q) {
            if (!__all_sync(0xffffffffu, mbar_wait<true>(full_bar(q % L::NS_), (q / L::NS_) & 1, p.wc, abort)))
                flags[2] = 1;
        };
        MergedCursor mc;
        mc.start(p);
        int rr = 0;                               // this group's row units
        for (int q = 0; mc.valid(); ++q, mc.advance(p)) {
            if (mc.turn != grp) continue;         // the other group's unit
            const GroupCursor cu = mc.group(grp);
            const uint32_t slot = sbase + L::OFF_RING + (q % L::NS_) * L::SLOT_;
            wait_full(q);
            if (cu.u == 0) {
#pragma unroll
                for (int kk = 0; kk < 18; ++kk)
                    ldsm_x4(chunk_addr(slot, ar, 36 * kh + 2 * kk + hi), qf[kk][0], qf[kk][1],
                            qf[kk][2], qf[kk][3]);
#pragma unroll
                for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;
                m_g = m_g8 = -INFINITY;
                l_g = l_g8 = 0.f;
                __syncwarp();
                if (lane == 0) mbar_arrive(empty_bar(q % L::NS_));
                continue;
            }

            // ---- S partials over this warp's K half, both 8-row tiles of its row half
            float aa[2][4] = {}, ab[2][4] = {};
#pragma unroll
            for (int k2 = 0; k2 < 9; ++k2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(chunk_addr(slot, rlo, 36 * kh + 4 * k2 + (lane >> 3)), b0, b1, b2, b3);
                mma_16816(aa[0], qf[2 * k2], b0, b1);
                mma_16816(aa[1], qf[2 * k2 + 1], b2, b3);
                ldsm_x4(chunk_addr(slot, rlo + 8, 36 * kh + 4 * k2 + (lane >> 3)), b0, b1, b2, b3);
                mma_16816(ab[0], qf[2 * k2], b0, b1);
                mma_16816(ab[1], qf[2 * k2 + 1], b2, b3);
            }
            float s4[4], sg[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const float lo = aa[0][e] + aa[1][e], up = ab[0][e] + ab[1][e];
                s4[e] = kh == 0 ? lo : up;        // partial of the own tile
                sg[e] = kh == 0 ? up : lo;        // partial of the partner's tile
            }
            xbuf[give * 32 + lane] = make_float4(sg[0], sg[1], sg[2], sg[3]);
            named_barrier(gbar, GTHREADS);        // A: S halves meet
            if (flags[2]) break;                  // every warp of the group sees the same flag

            {
                const float4 u = xbuf[own * 32 + lane];
                bool v0, v1;
                if constexpr (R::RPW == 8) {
                    const uint32_t mk =
                        *reinterpret_cast<const volatile uint32_t*>(rowmask + 4 * (q % L::NS_));
                    v0 = (mk >> r0) & 1u;
                    v1 = (mk >> (r0 + 1)) & 1u;
                } else {
                    const volatile uint8_t* mb = rowmask + L::MASK_STRIDE * (q % L::NS_);
                    v0 = (mb[r0 / R::RPW] >> (r0 % R::RPW)) & 1u;
                    v1 = (mb[(r0 + 1) / R::RPW] >> ((r0 + 1) % R::RPW)) & 1u;
                }
                s4[0] = v0 ? (s4[0] + u.x) * p.scale_log2 : -INFINITY;
                s4[1] = v1 ? (s4[1] + u.y) * p.scale_log2 : -INFINITY;
                s4[2] = v0 ? (s4[2] + u.z) * p.scale_log2 : -INFINITY;
                s4[3] = v1 ? (s4[3] + u.w) * p.scale_log2 : -INFINITY;
            }
            float mx_g = fmaxf(s4[0], s4[1]), mx_g8 = fmaxf(s4[2], s4[3]);
#pragma unroll
            for (int off = 1; off <= 2; off <<= 1) {
                mx_g = fmaxf(mx_g, __shfl_xor_sync(0xffffffffu, mx_g, off));
                mx_g8 = fmaxf(mx_g8, __shfl_xor_sync(0xffffffffu, mx_g8, off));
            }
            // Keep the running reference unless this tile exceeds it by the headroom.
            float ref_g = m_g, ref_g8 = m_g8;
            if (mx_g > m_g + HEADROOM) ref_g = mx_g;
            if (mx_g8 > m_g8 + HEADROOM) ref_g8 = mx_g8;
            {
                const float rg = ref_g == -INFINITY ? 0.f : ref_g;
                const float rg8 = ref_g8 == -INFINITY ? 0.f : ref_g8;
#pragma unroll
                for (int e = 0; e < 4; ++e) s4[e] = exp2_(s4[e] - (e < 2 ? rg : rg8));
            }
            uint8_t* pb = garea + G_P + r0 * 2;
            *reinterpret_cast<uint32_t*>(pb + g * P_PITCH) = pack_half2(s4[0], s4[1]);
            *reinterpret_cast<uint32_t*>(pb + (g + 8) * P_PITCH) = pack_half2(s4[2], s4[3]);
            // fp32-staged: the fp16 remainder lo = p - fp16(p) beside P.
            auto store_lo = [&](const float (&v)[4]) {
                uint8_t* pl = garea + G_PLO + r0 * 2;
                *reinterpret_cast<uint32_t*>(pl + g * P_PITCH) =
                    pack_half2(v[0] - __half2float(__float2half_rn(v[0])),
                               v[1] - __half2float(__float2half_rn(v[1])));
                *reinterpret_cast<uint32_t*>(pl + (g + 8) * P_PITCH) =
                    pack_half2(v[2] - __half2float(__float2half_rn(v[2])),
                               v[3] - __half2float(__float2half_rn(v[3])));
            };
            if constexpr (PSPLIT) store_lo(s4);
            if (c == 0) {
                ref_tile[own * H + g] = ref_g;
                ref_tile[own * H + g + 8] = ref_g8;
            }
            if (ref_g != m_g || ref_g8 != m_g8) flags[rr & 1] = 1;
            named_barrier(gbar, GTHREADS);        // B: P and the tiles' references visible
            const bool raise = flags[rr & 1] != 0;   // the same in every warp of the group
            if (gw == 0 && lane == 0) flags[(rr + 1) & 1] = 0;   // next unit's; writers follow A

            if (raise) {                          // rare: raise the reference, rescale
                float M_g = -INFINITY, M_g8 = -INFINITY;
#pragma unroll
                for (int t = 0; t < 4; ++t) {
                    M_g = fmaxf(M_g, ref_tile[t * H + g]);
                    M_g8 = fmaxf(M_g8, ref_tile[t * H + g + 8]);
                }
                const float Mg = M_g == -INFINITY ? 0.f : M_g, Mg8 = M_g8 == -INFINITY ? 0.f : M_g8;
                const float alpha_g = exp2_(m_g - Mg), alpha_g8 = exp2_(m_g8 - Mg8);
#pragma unroll
                for (int n = 0; n < 16; ++n) {
                    o[n][0] *= alpha_g;
                    o[n][1] *= alpha_g;
                    o[n][2] *= alpha_g8;
                    o[n][3] *= alpha_g8;
                }
                l_g *= alpha_g;
                l_g8 *= alpha_g8;
                const float rg = ref_g == -INFINITY ? 0.f : ref_g;
                const float rg8 = ref_g8 == -INFINITY ? 0.f : ref_g8;
                const float beta_g = exp2_(rg - Mg), beta_g8 = exp2_(rg8 - Mg8);
#pragma unroll
                for (int e = 0; e < 4; ++e) s4[e] *= e < 2 ? beta_g : beta_g8;
                *reinterpret_cast<uint32_t*>(pb + g * P_PITCH) = pack_half2(s4[0], s4[1]);
                *reinterpret_cast<uint32_t*>(pb + (g + 8) * P_PITCH) = pack_half2(s4[2], s4[3]);
                if constexpr (PSPLIT) store_lo(s4);
                m_g = M_g;
                m_g8 = M_g8;
                named_barrier(gbar, GTHREADS);    // rescaled P visible
            }
            l_g += s4[0] + s4[1];
            l_g8 += s4[2] + s4[3];
            ++rr;

            // ---- O += P . V over value dims 128gw .. 128gw+127, 32 rows
#pragma unroll
            for (int ks = 0; ks < 2; ++ks) {
                uint32_t a[4];
                ldsm_x4(pbase + ar * P_PITCH + (ks * 16 + hi * 8) * 2, a[0], a[1], a[2], a[3]);
                uint32_t al[4];
                if constexpr (PSPLIT)
                    ldsm_x4(plobase + ar * P_PITCH + (ks * 16 + hi * 8) * 2, al[0], al[1], al[2],
                            al[3]);
                const int vr = ks * 16 + ar;
#pragma unroll
                for (int np = 0; np < 8; ++np) {
                    uint32_t b0, b1, b2, b3;
                    const int vch = 16 * gw + 2 * np + hi;
                    const uint32_t vaddr = L::SPLIT ? chunk_addr_p(slot + L::VOFF, vr, vch, ROWV)
                                                    : chunk_addr(slot, vr, vch);
                    ldsm_x4_trans(vaddr, b0, b1, b2, b3);
                    if constexpr (PSPLIT) {
                        mma_16816(o[2 * np], al, b0, b1);
                        mma_16816(o[2 * np + 1], al, b2, b3);
                    }
                    mma_16816(o[2 * np], a, b0, b1);
                    mma_16816(o[2 * np + 1], a, b2, b3);
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(empty_bar(q % L::NS_));

            if (cu.u == cu.tr.nblk) {
                // ---- last unit of the token: normalise and store
#pragma unroll
                for (int off = 1; off <= 2; off <<= 1) {
                    l_g += __shfl_xor_sync(0xffffffffu, l_g, off);
                    l_g8 += __shfl_xor_sync(0xffffffffu, l_g8, off);
                }
                if (c == 0) {
                    red_sum[gw * H + g] = l_g;
                    red_sum[gw * H + g + 8] = l_g8;
                }
                named_barrier(gbar, GTHREADS);
                float L_g = 0.f, L_g8 = 0.f;
#pragma unroll
                for (int w = 0; w < GWARPS; ++w) {
                    L_g += red_sum[w * H + g];
                    L_g8 += red_sum[w * H + g + 8];
                }
                if (p.split) {
                    // Unnormalised O of this unit, with the reference it is relative to.
                    float* po = p.part_o + (size_t)cu.tr.item * H * DV;
#pragma unroll
                    for (int n = 0; n < 16; ++n) {
                        const int d = 128 * gw + 8 * n + 2 * c;
                        *reinterpret_cast<float2*>(po + g * DV + d) = make_float2(o[n][0], o[n][1]);
                        *reinterpret_cast<float2*>(po + (g + 8) * DV + d) = make_float2(o[n][2], o[n][3]);
                    }
                    if (gw == 0 && c == 0) {
                        float* ml = p.part_ml + (size_t)cu.tr.item * 2 * H;
                        ml[g] = m_g;
                        ml[g + 8] = m_g8;
                        ml[H + g] = L_g;
                        ml[H + g + 8] = L_g8;
                    }
                    continue;
                }
                const float inv_g = L_g > 0.f ? 1.f / L_g : 0.f;
                const float inv_g8 = L_g8 > 0.f ? 1.f / L_g8 : 0.f;
                float* ot = p.out + (size_t)cu.tr.i * H * DV;
#pragma unroll
                for (int n = 0; n < 16; ++n) {
                    const int d = 128 * gw + 8 * n + 2 * c;
                    *reinterpret_cast<float2*>(ot + g * DV + d) =
                        make_float2(o[n][0] * inv_g, o[n][1] * inv_g);
                    *reinterpret_cast<float2*>(ot + (g + 8) * DV + d) =
                        make_float2(o[n][2] * inv_g8, o[n][3] * inv_g8);
                }
            }
        }
    }
    __syncthreads();
}

// Split mode, second step: token i's output from its units' partial results (items
// first .. first+cnt-1): with M = the largest reference of a head, each unit's O and
// sum are scaled by 2^(m - M) before they are added; O / sum is the token's output.
// The units are added in order, so the result does not depend on how many tokens the
// call held. One CTA of 128 threads per (token, head), four value dims per thread.
namespace attn {
constexpr int SPLIT_MAX_TOKENS = 36;          // split mode: at most this many tokens,
constexpr int SPLIT_MAX_UNITS = 64;           // each with at most this many 32-row units
}  // namespace attn

struct MergeParams {
    const float* part_o;
    const float* part_ml;
    float* out;
    int n_q;
    int first[attn::SPLIT_MAX_TOKENS + 1];      // token i's items: first[i] .. first[i+1]-1
};

__global__ void __launch_bounds__(128) attn_merge_kernel(const MergeParams mp) {
    using namespace attn;
    __shared__ float wgt[SPLIT_MAX_UNITS];      // per unit: 2^(m - M) / L for this head
    __shared__ float red[2][4];
    const int i = blockIdx.x / H, h = blockIdx.x % H;
    grid_dependency_wait();                      // the partial results are complete
    grid_dependents_launch();
    if (i >= mp.n_q) return;
    const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
    const int first = mp.first[i], cnt = min(mp.first[i + 1] - first, SPLIT_MAX_UNITS);
    // Largest reference of the head over the units (threads 0 .. cnt-1 hold one each).
    const float m = tid < cnt ? mp.part_ml[(size_t)(first + tid) * 2 * H + h] : -INFINITY;
    float mx = m;
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) red[0][warp] = mx;
    __syncthreads();
    const float M = fmaxf(fmaxf(red[0][0], red[0][1]), fmaxf(red[0][2], red[0][3]));
    const float Mr = M == -INFINITY ? 0.f : M;
    const float a = tid < cnt ? exp2f(m - Mr) : 0.f;
    float l = tid < cnt ? mp.part_ml[(size_t)(first + tid) * 2 * H + H + h] * a : 0.f;
    // Sum of the scaled unit sums in unit order: gather them, then one thread adds.
    if (tid < cnt) wgt[tid] = l;
    __syncthreads();
    if (tid == 0) {
        float L = 0.f;
        for (int s2 = 0; s2 < cnt; ++s2) L += wgt[s2];
        red[1][0] = L > 0.f ? 1.f / L : 0.f;
    }
    __syncthreads();
    if (tid < cnt) wgt[tid] = a * red[1][0];
    __syncthreads();
    const float* src = mp.part_o + (size_t)first * H * DV + h * DV + 4 * tid;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 4
    for (int s2 = 0; s2 < cnt; ++s2) {
        const float4 v = *reinterpret_cast<const float4*>(src + (size_t)s2 * H * DV);
        const float w = wgt[s2];
        acc.x += v.x * w;
        acc.y += v.y * w;
        acc.z += v.z * w;
        acc.w += v.w * w;
    }
    *reinterpret_cast<float4*>(mp.out + ((size_t)i * H + h) * DV + 4 * tid) = acc;
}

}  // namespace ds4sp
