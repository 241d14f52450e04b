// C ABI of libds4sp (declared in include/ds4sp.h): argument checks, band order,
// workspace sizing, TMA descriptors and kernel launches. Everything the path
// computes runs in the kernels included below; this file only validates and launches.
#include <cuda.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <mutex>
#include <new>
#include <string>
#include <utility>
#include <vector>

#include "ds4sp.h"
#include "indexer_tcgen05.cuh"
#include "indexer_topk_fused.cuh"
#include "indexer_pair.cuh"
#include "probe_gather.cuh"
#include "sparse_attn_mma.cuh"
#include "sparse_attn_tc.cuh"
#include "topk_radix.cuh"

using namespace ds4sp;

namespace {

thread_local std::string g_last_error;

ds4sp_status fail(ds4sp_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
ds4sp_status fail(ds4sp_status s, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return s;
}

ds4sp_status cuda_fail(cudaError_t e, const char* what) {
    return fail(DS4SP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

constexpr int kMaxTopkCandidates = 51200;  // top-k keeps a token's row in shared memory
constexpr int kTopkCluster = 8;            // CTAs per token in topk_cluster_kernel
constexpr int kHostStep = 1024;            // ds4sp_prefill_host: tokens per copy/compute step
constexpr int kHostTail = 256;             // ds4sp_prefill_host: tokens of the last step at most

enum Kind { kIndexer = 0, kTopk = 1, kAttn = 2 };

struct TimedLaunch {
    int kind;
    cudaEvent_t start, stop;
};

}  // namespace

struct ds4sp_handle {
    ds4sp_config cfg;
    int device = 0;
    int sm_count = 148;
    // Device words: [0] the status word ds4sp_device_status reads, [1] the abort word of
    // the kernels' bounded waits (see WaitCtl).
    uint32_t* d_status = nullptr;
    uint32_t epoch = 0;                                  // of the last launch
    unsigned long long wait_limit_ns = kWaitLimitNs;     // ds4sp_debug_set_wait_limit_ns
    cudaEvent_t last = nullptr;
    int next_band = 0;
    int fail_launches = 0;
    bool profiling = false;
    std::vector<TimedLaunch> timed;
    std::vector<cudaEvent_t> event_pool;
    bool smem_set[3] = {false, false, false};
    // ds4sp_prefill_host: copy streams (in, out) and per-step events, made on first use.
    cudaStream_t copy_in = nullptr, copy_out = nullptr;
    std::vector<cudaEvent_t> step_in, step_done;
    cudaEvent_t host_start = nullptr, host_end = nullptr;
    // Split-mode attention partials (few tokens): capacity in 32-row units.
    int split_cap = 0;
    float* part_o = nullptr;
    float* part_ml = nullptr;
    // ds4sp_debug_set_mask: explicit visibility mask [mask_rows, mask_cols], or NULL.
    const uint8_t* mask = nullptr;
    int mask_rows = 0, mask_cols = 0;
};

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// An NVTX range around each entry point that queues work, named after it, so that a
// profiler's timeline shows the library's calls (no cost without a profiler attached).
struct TraceRange {
    explicit TraceRange(const char* name) { nvtxRangePushA(name); }
    ~TraceRange() { nvtxRangePop(); }
    TraceRange(const TraceRange&) = delete;
    TraceRange& operator=(const TraceRange&) = delete;
};

int nvis(int t, int ratio) { return (t + 1) / ratio; }

// The bounded-wait settings of the handle's next launch, with a fresh epoch.
WaitCtl next_wait(ds4sp_handle* h) {
    if (++h->epoch == 0) h->epoch = 1;   // epoch 0 would match a cleared abort word
    return WaitCtl{h->d_status, h->d_status + 1, h->epoch, h->wait_limit_ns};
}

constexpr int kMaxDevices = 64;

// cudaFuncSetAttribute(kernel, max dynamic shared memory) once per (device, kernel): the
// attribute belongs to the device's copy of the function.
ds4sp_status set_smem_once(ds4sp_handle* h, const void* fn, int bytes, int slot, const char* what,
                           int launch_regs = 0) {
    static std::mutex mu;
    static bool done[kMaxDevices][32] = {};
    if (h->device < 0 || h->device >= kMaxDevices || slot < 0 || slot >= 32)
        return fail(DS4SP_ERR_UNSUPPORTED, "device %d", h->device);
    std::lock_guard<std::mutex> lock(mu);
    if (done[h->device][slot]) return DS4SP_OK;
    const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) return cuda_fail(e, what);
    if (launch_regs) {   // a setmaxnreg split that assumes this launch register count
        cudaFuncAttributes fa;
        const cudaError_t ea = cudaFuncGetAttributes(&fa, fn);
        if (ea != cudaSuccess) return cuda_fail(ea, what);
        if (fa.numRegs != launch_regs)
            return fail(DS4SP_ERR_UNSUPPORTED, "%s: kernel built with %d registers, not %d", what,
                        fa.numRegs, launch_regs);
    }
    done[h->device][slot] = true;
    return DS4SP_OK;
}

// Slot of an indexer instantiation in set_smem_once's table: D_i in {64, 128} x H_i in
// {4, 8, 16, 32, 64}.
constexpr int indexer_slot(int d_idx, int h_idx) {
    return (d_idx == 128 ? 5 : 0) + (h_idx == 4 ? 0 : h_idx == 8 ? 1 : h_idx == 16 ? 2 : h_idx == 32 ? 3 : 4);
}
// Slots 0-9: indexer_tcgen05_kernel; 10-19 (tables of 32): the fused kernel; 20-29: the
// CTA-pair indexer.
constexpr int fused_slot(int d_idx, int h_idx) { return 10 + indexer_slot(d_idx, h_idx); }
constexpr int pair_slot(int d_idx, int h_idx) { return 20 + indexer_slot(d_idx, h_idx); }

int score_ld(int t_last, int ratio) {
    const int nv = nvis(t_last, ratio);
    return ((nv > 0 ? nv : 1) + 3) / 4 * 4;
}

// Shared memory of the streaming attention kernel for a cache format and top_k, and the
// largest top_k that format's layout holds.
int attn_smem_bytes(int kvf, int k) {
    switch (kvf) {
        case kFmtQ8: return attn::RingLayout<kFmtQ8>::smem_bytes(k);
        case kFmtQ4: return attn::RingLayout<kFmtQ4>::smem_bytes(k);
        case kFmtQ8Q4: return attn::RingLayout<kFmtQ8Q4>::smem_bytes(k);
        default: return attn::RingLayout<kFmtF16>::smem_bytes(k);
    }
}
int attn_max_topk(int kvf) {
    switch (kvf) {
        case kFmtQ8: return attn::RingLayout<kFmtQ8>::MAX_K;
        case kFmtQ4: return attn::RingLayout<kFmtQ4>::MAX_K;
        case kFmtQ8Q4: return attn::RingLayout<kFmtQ8Q4>::MAX_K;
        default: return attn::RingLayout<kFmtF16>::MAX_K;
    }
}

// Bytes of one row of kv_raw / kv_cmp in the handle's cache format.
int kv_row_bytes_of(const ds4sp_config& c) {
    return c.kv_format == 0 ? c.d_qk * 2 : quant_row_bytes(c.kv_format, c.d_qk);
}

float scale_of(const ds4sp_config& c) {
    return c.softmax_scale > 0.f ? c.softmax_scale : 1.0f / std::sqrt((float)c.d_qk);
}

#define DS4SP_TRY(x)                      \
    do {                                  \
        const ds4sp_status s_ = (x);      \
        if (s_ != DS4SP_OK) return s_;    \
    } while (0)

cudaEvent_t pooled_event(ds4sp_handle* h) {
    if (!h->event_pool.empty()) {
        cudaEvent_t e = h->event_pool.back();
        h->event_pool.pop_back();
        return e;
    }
    cudaEvent_t e = nullptr;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    return e;
}

// Runs `launch` on `stream`, honouring the fault-injection counter and recording
// timing events when profiling is on.
template <class F>
ds4sp_status launch(ds4sp_handle* h, int kind, cudaStream_t stream, F&& f) {
    if (h->fail_launches > 0) {
        --h->fail_launches;
        return fail(DS4SP_ERR_CUDA, "launch suppressed by ds4sp_debug_fail_launches");
    }
    TimedLaunch tl{kind, nullptr, nullptr};
    if (h->profiling) {
        tl.start = pooled_event(h);
        tl.stop = pooled_event(h);
        if (!tl.start || !tl.stop) return fail(DS4SP_ERR_CUDA, "cudaEventCreate failed");
        cudaEventRecord(tl.start, stream);
    }
    f();
    const cudaError_t e = cudaGetLastError();
    if (h->profiling) {
        cudaEventRecord(tl.stop, stream);
        h->timed.push_back(tl);
    }
    if (e != cudaSuccess) return cuda_fail(e, "kernel launch");
    return DS4SP_OK;
}

// A kernel launch on `stream`, as a programmatic dependent of the previous kernel when
// `dependent` is set (the kernels wait for that kernel before touching global memory,
// so only their launch and prologue overlap its tail). Launch errors are also left for
// cudaGetLastError.
template <class... KArgs, class... Args>
void launch_k(bool dependent, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
              cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t lc = {};
    lc.gridDim = grid;
    lc.blockDim = block;
    lc.dynamicSmemBytes = smem;
    lc.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = dependent ? 1 : 0;
    cudaLaunchKernelEx(&lc, kernel, std::forward<Args>(args)...);
}

// The same with thread-block clusters of `cluster` CTAs along x.
template <class... KArgs, class... Args>
void launch_k_cluster(bool dependent, int cluster, void (*kernel)(KArgs...), dim3 grid, dim3 block,
                      size_t smem, cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t lc = {};
    lc.gridDim = grid;
    lc.blockDim = block;
    lc.dynamicSmemBytes = smem;
    lc.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = cluster;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    lc.attrs = attr;
    lc.numAttrs = dependent ? 2 : 1;
    cudaLaunchKernelEx(&lc, kernel, std::forward<Args>(args)...);
}

// ---------------------------------------------------------------- TMA descriptors

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (EncodeTiledFn) nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// 2-D fp16 row-major [rows, cols] map with a (64 x box_rows) box and 128-byte swizzle.
bool make_tmap_2d(CUtensorMap* m, const void* base, int cols, int rows, int box_rows) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1u, 1u};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---------------------------------------------------------------- launchers

template <int D_I, int H_I>
ds4sp_status launch_indexer(ds4sp_handle* h, const void* q_idx, const void* k_idx, const float* w,
                            int t0, int n_q, float* scores, int ld, cudaStream_t stream) {
    using C = IndexerTile<D_I, H_I>;
    const int ratio = h->cfg.ratio;
    const int t_last = t0 + n_q - 1;
    const int n_rows = nvis(t_last, ratio);
    if (n_rows == 0) return DS4SP_OK;  // no token of the range sees a compressed row
    CUtensorMap tk, tq;
    if (!make_tmap_2d(&tk, k_idx, D_I, n_rows, C::BM) ||
        !make_tmap_2d(&tq, q_idx, D_I, n_q * H_I, C::BN))
        return fail(DS4SP_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    DS4SP_TRY(set_smem_once(h, reinterpret_cast<const void*>(indexer_tcgen05_kernel<D_I, H_I>),
                            C::SMEM_BYTES, indexer_slot(D_I, H_I), "cudaFuncSetAttribute(indexer)"));
    IndexerParams p;
    p.w = w;
    p.scores = scores;
    p.wc = next_wait(h);
    p.t0 = t0;
    p.n_q = n_q;
    p.ld = ld;
    p.ratio = ratio;
    p.n_tb = (n_q + C::TB - 1) / C::TB;
    // Persistent CTAs, one per SM, each taking an equal contiguous share of the launch's
    // tiles (token block x 128-row j-tile, in block order); no CTA without a tile.
    auto block_tiles = [&](int tb) {
        return (nvis(t0 + std::min((tb + 1) * C::TB, n_q) - 1, ratio) + C::BM - 1) / C::BM;
    };
    long long tiles = 0;
    for (int tb = 0; tb < p.n_tb; ++tb) tiles += block_tiles(tb);
    if (tiles == 0) return DS4SP_OK;
    if (tiles > (1 << 30) || p.n_tb > 65535)
        return fail(DS4SP_ERR_UNSUPPORTED, "indexer launch of %lld tiles", tiles);
    const int grid = (int)std::min<long long>(tiles, std::min(h->sm_count, kIndexerMaxGrid));
    if ((tiles + p.n_tb) / grid + 2 > 65535)     // a share's tile count must fit 16 bits
        return fail(DS4SP_ERR_UNSUPPORTED, "indexer launch of %lld tiles", tiles);
    {
        // Cut the tile list into `grid` contiguous shares of about equal cost: one per
        // tile, plus kLoadCost for the first tile of each token block (its q_idx block
        // load). Every share gets at least one tile.
        constexpr double kLoadCost = 1.0;
        const double total_cost = (double)tiles + kLoadCost * p.n_tb;
        int b = 0, tb = 0, jt = 0, nb = block_tiles(0);
        long long left_tiles = tiles;
        double cost = 0.0;
        p.start_tb[0] = 0;
        p.start_jt[0] = 0;
        int count = 0;
        while (left_tiles > 0) {
            while (jt >= nb) {                    // next token block with tiles
                ++tb;
                jt = 0;
                nb = block_tiles(tb);
            }
            cost += 1.0 + (jt == 0 ? kLoadCost : 0.0);
            ++count;
            ++jt;
            --left_tiles;
            const double target = total_cost * (b + 1) / grid;
            // Close share b at its cost target, but leave a tile for every later share.
            if (b + 1 < grid && (cost >= target || left_tiles == grid - 1 - b)) {
                p.count[b] = (uint16_t)count;
                ++b;
                count = 0;
                while (jt >= nb && left_tiles > 0) {
                    ++tb;
                    jt = 0;
                    nb = block_tiles(tb);
                }
                p.start_tb[b] = (uint16_t)tb;
                p.start_jt[b] = (uint16_t)jt;
            }
        }
        p.count[b] = (uint16_t)count;
        if (b != grid - 1) return fail(DS4SP_ERR_CUDA, "indexer partition: %d of %d shares", b + 1, grid);
    }
    return launch(h, kIndexer, stream, [&] {
        launch_k(h->cfg.dependent_launch != 0, indexer_tcgen05_kernel<D_I, H_I>, grid, C::THREADS,
                 C::SMEM_BYTES, stream, tk, tq, p);
    });
}

// The CTA-pair indexer (indexer_pair_kernel): items are (token block, pair of j-tiles),
// cut into contiguous shares of about equal cost, one per pair of CTAs (a 2-CTA cluster).
template <int D_I, int H_I>
ds4sp_status launch_indexer_pair(ds4sp_handle* h, const void* q_idx, const void* k_idx,
                                 const float* w, int t0, int n_q, float* scores, int ld,
                                 cudaStream_t stream) {
    using C = PairTile<D_I, H_I>;
    const int ratio = h->cfg.ratio;
    const int n_rows = nvis(t0 + n_q - 1, ratio);
    if (n_rows == 0) return DS4SP_OK;
    CUtensorMap tk, tq;
    if (!make_tmap_2d(&tk, k_idx, D_I, n_rows, C::BM) ||
        !make_tmap_2d(&tq, q_idx, D_I, n_q * H_I, C::BN_HALF))
        return fail(DS4SP_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    DS4SP_TRY(set_smem_once(h, reinterpret_cast<const void*>(indexer_pair_kernel<D_I, H_I>),
                            C::SMEM_BYTES, pair_slot(D_I, H_I), "cudaFuncSetAttribute(indexer pairs)"));
    IndexerParams p;
    p.w = w;
    p.scores = scores;
    p.wc = next_wait(h);
    p.t0 = t0;
    p.n_q = n_q;
    p.ld = ld;
    p.ratio = ratio;
    p.n_tb = (n_q + C::TB - 1) / C::TB;
    auto block_items = [&](int tb) {
        const int tiles = (nvis(t0 + std::min((tb + 1) * C::TB, n_q) - 1, ratio) + C::BM - 1) / C::BM;
        return (tiles + 1) / 2;
    };
    long long items = 0;
    for (int tb = 0; tb < p.n_tb; ++tb) items += block_items(tb);
    if (items == 0) return DS4SP_OK;
    const int pairs = (int)std::min<long long>(items, std::min(h->sm_count / 2, kIndexerMaxGrid));
    if (items > (1 << 30) || p.n_tb > 65535 || (items + p.n_tb) / pairs + 2 > 65535)
        return fail(DS4SP_ERR_UNSUPPORTED, "indexer launch of %lld tile pairs", items);
    {
        // Contiguous shares of about equal cost: one per item, plus kLoadCost for the first
        // item of each token block (its q_idx load). Every share gets at least one item.
        constexpr double kLoadCost = 1.0;
        const double total_cost = (double)items + kLoadCost * p.n_tb;
        int b = 0, tb = 0, jp = 0, nb = block_items(0);
        long long left = items;
        double cost = 0.0;
        p.start_tb[0] = 0;
        p.start_jt[0] = 0;
        int count = 0;
        while (left > 0) {
            while (jp >= nb) {
                ++tb;
                jp = 0;
                nb = block_items(tb);
            }
            cost += 1.0 + (jp == 0 ? kLoadCost : 0.0);
            ++count;
            ++jp;
            --left;
            const double target = total_cost * (b + 1) / pairs;
            if (b + 1 < pairs && (cost >= target || left == pairs - 1 - b)) {
                p.count[b] = (uint16_t)count;
                ++b;
                count = 0;
                while (jp >= nb && left > 0) {
                    ++tb;
                    jp = 0;
                    nb = block_items(tb);
                }
                p.start_tb[b] = (uint16_t)tb;
                p.start_jt[b] = (uint16_t)jp;
            }
        }
        p.count[b] = (uint16_t)count;
        if (b != pairs - 1) return fail(DS4SP_ERR_CUDA, "indexer partition: %d of %d shares", b + 1, pairs);
    }
    return launch(h, kIndexer, stream, [&] {
        launch_k_cluster(h->cfg.dependent_launch != 0, 2, indexer_pair_kernel<D_I, H_I>, 2 * pairs,
                         C::THREADS, C::SMEM_BYTES, stream, tk, tq, p);
    });
}

template <int D_I>
ds4sp_status dispatch_indexer_h(ds4sp_handle* h, const void* q_idx, const void* k_idx,
                                const float* w, int t0, int n_q, float* scores, int ld,
                                cudaStream_t s) {
    if (h->cfg.indexer_kernel == 1) {
        switch (h->cfg.n_idx_heads) {
            case 4: return launch_indexer_pair<D_I, 4>(h, q_idx, k_idx, w, t0, n_q, scores, ld, s);
            case 8: return launch_indexer_pair<D_I, 8>(h, q_idx, k_idx, w, t0, n_q, scores, ld, s);
            case 16: return launch_indexer_pair<D_I, 16>(h, q_idx, k_idx, w, t0, n_q, scores, ld, s);
            case 32: return launch_indexer_pair<D_I, 32>(h, q_idx, k_idx, w, t0, n_q, scores, ld, s);
            case 64: return launch_indexer_pair<D_I, 64>(h, q_idx, k_idx, w, t0, n_q, scores, ld, s);
        }
        return fail(DS4SP_ERR_UNSUPPORTED, "n_idx_heads %d", h->cfg.n_idx_heads);
    }
    switch (h->cfg.n_idx_heads) {
        case 4: return launch_indexer<D_I, 4>(h, q_idx, k_idx, w, t0, n_q, scores, ld, s);
        case 8: return launch_indexer<D_I, 8>(h, q_idx, k_idx, w, t0, n_q, scores, ld, s);
        case 16: return launch_indexer<D_I, 16>(h, q_idx, k_idx, w, t0, n_q, scores, ld, s);
        case 32: return launch_indexer<D_I, 32>(h, q_idx, k_idx, w, t0, n_q, scores, ld, s);
        case 64: return launch_indexer<D_I, 64>(h, q_idx, k_idx, w, t0, n_q, scores, ld, s);
    }
    return fail(DS4SP_ERR_UNSUPPORTED, "n_idx_heads %d", h->cfg.n_idx_heads);
}

// Indexer and top-k in one launch (indexer_topk_fused_kernel), when the call qualifies:
// no explicit mask, some token sees a compressed row, the key rows of a token block fit
// one of the kernel's two 40 KB key buffers (2,560 rows, a 10,240-token context, at 64
// index heads) and the launch has at most kFusedMaxBlocks token blocks.
// Returns DS4SP_ERR_UNSUPPORTED (with nothing launched) when it does not qualify.
template <int D_I, int H_I>
ds4sp_status launch_fused(ds4sp_handle* h, const void* q_idx, const void* k_idx, const float* w,
                          int t0, int n_q, int32_t* topk, cudaStream_t stream) {
    using C = FusedTile<D_I, H_I>;
    const int ratio = h->cfg.ratio, k = h->cfg.top_k;
    const int n_rows = nvis(t0 + n_q - 1, ratio);
    const int n_tb = (n_q + C::TB - 1) / C::TB;
    const int max_tiles = (n_rows + C::BM - 1) / C::BM;
    const int kld = C::BM * max_tiles;
    if (h->mask || n_rows == 0 || n_tb > kFusedMaxBlocks ||
        (long long)C::TB * kld * 4 > C::KEY_BYTES)
        return DS4SP_ERR_UNSUPPORTED;
    CUtensorMap tk, tq;
    if (!make_tmap_2d(&tk, k_idx, D_I, n_rows, C::BM) ||
        !make_tmap_2d(&tq, q_idx, D_I, n_q * H_I, C::BN))
        return fail(DS4SP_ERR_CUDA, "cuTensorMapEncodeTiled failed");
    DS4SP_TRY(set_smem_once(h, reinterpret_cast<const void*>(indexer_topk_fused_kernel<D_I, H_I>),
                            C::SMEM_BYTES, fused_slot(D_I, H_I),
                            "cudaFuncSetAttribute(fused indexer)", C::LAUNCH_REGS));
    FusedParams p;
    p.w = w;
    p.topk = topk;
    p.wc = next_wait(h);
    p.t0 = t0;
    p.n_q = n_q;
    p.k = k;
    p.ratio = ratio;
    p.kld = kld;
    // Longest-processing-time assignment of the token blocks to the persistent CTAs: cost
    // = the block's tiles plus 1.5 tiles per token that needs a select (n_vis > k), kept
    // in half tiles so that it is an integer; blocks go heaviest first (ties: the later
    // block first) to the least loaded CTA (ties: the lower CTA). Block costs never fall
    // with the block index in a launch, so the heaviest-first order is usually the
    // reverse block order and the sort is skipped.
    const int grid = std::min(n_tb, std::min(h->sm_count, kIndexerMaxGrid));
    struct Item { int cost, tb; };
    Item items[kFusedMaxBlocks];
    bool ascending = true;
    const int t_sel = ratio * (k + 1) - 1;      // tokens t >= t_sel see more than k rows
    for (int tb = 0; tb < n_tb; ++tb) {
        const int tok0 = t0 + tb * C::TB, tok_end = std::min(tok0 + C::TB, t0 + n_q);
        const int tiles = (nvis(tok_end - 1, ratio) + C::BM - 1) / C::BM;
        const int sel = std::max(0, tok_end - std::max(tok0, t_sel));
        items[tb] = {2 * tiles + 3 * sel, tb};
        if (tb && items[tb].cost < items[tb - 1].cost) ascending = false;
    }
    if (ascending)
        std::reverse(items, items + n_tb);
    else
        std::sort(items, items + n_tb, [](const Item& x, const Item& y) {
            return x.cost != y.cost ? x.cost > y.cost : x.tb > y.tb;
        });
    struct Load { long long load; int cta; };
    Load heap[kIndexerMaxGrid];                 // a min-heap of the CTAs' loads
    for (int c = 0; c < grid; ++c) heap[c] = {0, c};
    auto later = [](const Load& x, const Load& y) {
        return x.load != y.load ? x.load > y.load : x.cta > y.cta;
    };
    uint16_t cta_of[kFusedMaxBlocks];
    int count[kIndexerMaxGrid] = {};
    for (int u = 0; u < n_tb; ++u) {
        std::pop_heap(heap, heap + grid, later);
        Load& top = heap[grid - 1];
        cta_of[u] = (uint16_t)top.cta;
        ++count[top.cta];
        top.load += items[u].cost;
        std::push_heap(heap, heap + grid, later);
    }
    int pos[kIndexerMaxGrid];
    int u_total = 0;
    for (int c = 0; c < grid; ++c) {
        p.first[c] = (uint16_t)u_total;
        pos[c] = u_total;
        u_total += count[c];
    }
    p.first[grid] = (uint16_t)u_total;
    for (int u = 0; u < n_tb; ++u) p.blk[pos[cta_of[u]]++] = (uint16_t)items[u].tb;
    return launch(h, kIndexer, stream, [&] {
        launch_k(h->cfg.dependent_launch != 0, indexer_topk_fused_kernel<D_I, H_I>, grid, C::THREADS,
                 C::SMEM_BYTES, stream, tk, tq, p);
    });
}

template <int D_I>
ds4sp_status dispatch_fused_h(ds4sp_handle* h, const void* q_idx, const void* k_idx,
                              const float* w, int t0, int n_q, int32_t* topk, cudaStream_t s) {
    switch (h->cfg.n_idx_heads) {
        case 4: return launch_fused<D_I, 4>(h, q_idx, k_idx, w, t0, n_q, topk, s);
        case 8: return launch_fused<D_I, 8>(h, q_idx, k_idx, w, t0, n_q, topk, s);
        case 16: return launch_fused<D_I, 16>(h, q_idx, k_idx, w, t0, n_q, topk, s);
        case 32: return launch_fused<D_I, 32>(h, q_idx, k_idx, w, t0, n_q, topk, s);
        case 64: return launch_fused<D_I, 64>(h, q_idx, k_idx, w, t0, n_q, topk, s);
    }
    return fail(DS4SP_ERR_UNSUPPORTED, "n_idx_heads %d", h->cfg.n_idx_heads);
}

ds4sp_status launch_topk(ds4sp_handle* h, const float* scores, int ld, int t0, int n_q,
                         int32_t* topk, cudaStream_t stream) {
    const int k = h->cfg.top_k, ratio = h->cfg.ratio;
    // Explicit-mask form: candidates only among the columns this call's scores cover.
    const int mcols = h->mask ? std::min(h->mask_cols, nvis(t0 + n_q - 1, ratio)) : 0;
    const uint8_t* vm = h->mask;
    const long long mld = h->mask_cols;
    const bool big = ld > 4096;
    if (!h->smem_set[kTopk]) {
        cudaError_t e = cudaFuncSetAttribute(topk_radix_kernel<128>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kMaxTopkCandidates * 4 + 64);
        if (e == cudaSuccess)
            e = cudaFuncSetAttribute(topk_radix_kernel<1024>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     kMaxTopkCandidates * 4 + 64);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(topk)");
        h->smem_set[kTopk] = true;
    }
    const size_t smem = (size_t)ld * 4;
    const bool pdl = h->cfg.dependent_launch != 0;
    // A few tokens with long rows (the verify form): a cluster of kTopkCluster CTAs per
    // token shares each row, so that the launch covers more than a handful of SMs.
    const int n_max = nvis(t0 + n_q - 1, ratio);
    if (!vm && n_max > 4096 && (long long)n_q * kTopkCluster <= 2LL * h->sm_count) {
        const size_t csmem = (size_t)((n_max + kTopkCluster - 1) / kTopkCluster) * 4;
        return launch(h, kTopk, stream, [&] {
            launch_k_cluster(pdl, kTopkCluster, topk_cluster_kernel<kTopkCluster, 512>,
                             n_q * kTopkCluster, 512, csmem, stream, scores, ld, t0, n_q, k, ratio,
                             topk);
        });
    }
    return launch(h, kTopk, stream, [&] {
        if (big)
            launch_k(pdl, topk_radix_kernel<1024>, n_q, 1024, smem, stream, scores, ld, t0, n_q, k,
                     ratio, vm, mld, mcols, topk);
        else
            launch_k(pdl, topk_radix_kernel<128>, n_q, 128, smem, stream, scores, ld, t0, n_q, k,
                     ratio, vm, mld, mcols, topk);
    });
}

ds4sp_status launch_attn(ds4sp_handle* h, const void* q, const void* kv_raw, const void* kv_cmp,
                         const int32_t* topk, int t0, int n_q, float* out, cudaStream_t stream,
                         const void* prefetch = nullptr, size_t prefetch_bytes = 0) {
    const int kvf = h->cfg.kv_format;
    const bool tc = h->cfg.attn_kernel == 1;
    const int smem = tc ? tcattn::smem_bytes(h->cfg.top_k) : attn_smem_bytes(kvf, h->cfg.top_k);
    if (!h->smem_set[kAttn]) {
        // Every instantiation (fast or precise exponentials x fp16 or fp32-staged P, and
        // the two quantized-cache forms), once per handle.
        const void* fns[7] = {
            reinterpret_cast<const void*>(sparse_attn_mma_kernel<false, false, kFmtF16>),
            reinterpret_cast<const void*>(sparse_attn_mma_kernel<true, false, kFmtF16>),
            reinterpret_cast<const void*>(sparse_attn_mma_kernel<false, true, kFmtF16>),
            reinterpret_cast<const void*>(sparse_attn_mma_kernel<true, true, kFmtF16>),
            reinterpret_cast<const void*>(sparse_attn_mma_kernel<false, false, kFmtQ8>),
            reinterpret_cast<const void*>(sparse_attn_mma_kernel<false, false, kFmtQ4>),
            reinterpret_cast<const void*>(sparse_attn_mma_kernel<false, false, kFmtQ8Q4>)};
        const int fmt_of[7] = {kFmtF16, kFmtF16, kFmtF16, kFmtF16, kFmtQ8, kFmtQ4, kFmtQ8Q4};
        auto launch_regs = [](int fmt) {
            return fmt == kFmtQ8 ? attn::Roles<kFmtQ8>::LAUNCH_REGS
                   : fmt == kFmtQ4 ? attn::Roles<kFmtQ4>::LAUNCH_REGS
                   : fmt == kFmtQ8Q4 ? attn::Roles<kFmtQ8Q4>::LAUNCH_REGS
                                     : attn::Roles<kFmtF16>::LAUNCH_REGS;
        };
        for (int fi = 0; fi < 7; ++fi) {
            const void* fn = fns[fi];
            const int max_smem = attn_smem_bytes(fmt_of[fi], attn_max_topk(fmt_of[fi]));
            const cudaError_t e = cudaFuncSetAttribute(fn, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                       max_smem);
            if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attention)");
            cudaFuncAttributes fa;
            const cudaError_t ea = cudaFuncGetAttributes(&fa, fn);
            if (ea != cudaSuccess) return cuda_fail(ea, "cudaFuncGetAttributes(attention)");
            if (fa.numRegs != launch_regs(fmt_of[fi]))   // the warp roles' register split assumes it
                return fail(DS4SP_ERR_UNSUPPORTED, "attention kernel built with %d registers, not %d",
                            fa.numRegs, launch_regs(fmt_of[fi]));
        }
        const cudaError_t e = cudaFuncSetAttribute(sparse_attn_tc_kernel,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                   tcattn::smem_bytes(attn::MAX_TOPK));
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(attention, tcgen05)");
        h->smem_set[kAttn] = true;
    }
    AttnParams p;
    p.q = static_cast<const __half*>(q);
    p.kv_raw = static_cast<const __half*>(kv_raw);
    p.kv_cmp = static_cast<const __half*>(kv_cmp);
    p.topk = topk;
    p.out = out;
    p.wc = next_wait(h);
    p.t0 = t0;
    p.n_q = n_q;
    p.k = h->cfg.top_k;
    p.n_swa = h->cfg.n_swa;
    p.ratio = h->cfg.ratio;
    p.scale_log2 = scale_of(h->cfg) * 1.4426950408889634f;
    // Explicit-mask form: entries only among the compressed rows this call may read.
    p.vis_mask = h->mask;
    p.mask_ld = h->mask_cols;
    p.mask_cols = h->mask ? std::min(h->mask_cols, nvis(t0 + n_q - 1, h->cfg.ratio)) : 0;
    p.kv_row_bytes = kv_row_bytes_of(h->cfg);
    // Few tokens: one work item per 32-row unit, then a merge per token. The decision
    // and each token's units depend only on the token, so a token's result is the same
    // in every call that takes this path.
    MergeParams mp{};
    p.split = 0;
    p.n_items = n_q;
    if (!tc && n_q <= attn::SPLIT_MAX_TOKENS && h->split_cap > 0) {
        int items = 0;
        bool fits = true;
        for (int i = 0; i < n_q; ++i) {
            const int t = t0 + i, nsel = std::min(h->cfg.top_k, nvis(t, h->cfg.ratio));
            const int nrows = nsel + (t - std::max(0, t - h->cfg.n_swa + 1) + 1);
            const int nblk = (nrows + attn::BR - 1) / attn::BR;
            mp.first[i] = items;
            items += nblk;
            fits = fits && nblk <= attn::SPLIT_MAX_UNITS;
        }
        mp.first[n_q] = items;
        if (fits && items <= h->split_cap && items > n_q) {
            p.split = 1;
            p.n_items = items;
            p.part_o = h->part_o;
            p.part_ml = h->part_ml;
            mp.part_o = h->part_o;
            mp.part_ml = h->part_ml;
            mp.out = out;
            mp.n_q = n_q;
        }
    }
    // The region must start 16-byte aligned; its length is cut to a multiple of 16.
    const bool pf = prefetch && aligned16(prefetch) && prefetch_bytes >= 16;
    p.prefetch = pf ? static_cast<const char*>(prefetch) : nullptr;
    p.prefetch_bytes = pf ? (long long)(prefetch_bytes / 16 * 16) : 0;
    return launch(h, kAttn, stream, [&] {
        // persistent: one CTA per SM, each walking its share of the work items
        const int grid = std::min(p.n_items, h->sm_count);
        const dim3 g(grid), b(attn::Roles<kFmtF16>::THREADS);
        const dim3 bs(attn::Roles<kFmtQ8>::THREADS);   // the quantized formats' eight producer warps
        static_assert(attn::Roles<kFmtQ8>::THREADS == attn::Roles<kFmtQ4>::THREADS &&
                          attn::Roles<kFmtQ8Q4>::THREADS == attn::Roles<kFmtQ8>::THREADS,
                      "block shapes per format");
        const bool pdl = h->cfg.dependent_launch != 0;
        if (tc) {
            launch_k(pdl, sparse_attn_tc_kernel, g, dim3(tcattn::THREADS), smem, stream, p);
        } else if (h->cfg.kv_format == kFmtQ8) {
            launch_k(pdl, sparse_attn_mma_kernel<false, false, kFmtQ8>, g, bs, smem, stream, p);
        } else if (h->cfg.kv_format == kFmtQ4) {
            launch_k(pdl, sparse_attn_mma_kernel<false, false, kFmtQ4>, g, bs, smem, stream, p);
        } else if (h->cfg.kv_format == kFmtQ8Q4) {
            launch_k(pdl, sparse_attn_mma_kernel<false, false, kFmtQ8Q4>, g, bs, smem, stream, p);
        } else {
            switch (2 * h->cfg.pv_mode + h->cfg.exp_mode) {
                case 0: launch_k(pdl, sparse_attn_mma_kernel<false, false, kFmtF16>, g, b, smem, stream, p); break;
                case 1: launch_k(pdl, sparse_attn_mma_kernel<true, false, kFmtF16>, g, b, smem, stream, p); break;
                case 2: launch_k(pdl, sparse_attn_mma_kernel<false, true, kFmtF16>, g, b, smem, stream, p); break;
                default: launch_k(pdl, sparse_attn_mma_kernel<true, true, kFmtF16>, g, b, smem, stream, p); break;
            }
        }
        if (p.split) launch_k(pdl, attn_merge_kernel, n_q * attn::H, 128, 0, stream, mp);
    });
}

ds4sp_status check_handle(const ds4sp_handle* h) {
    if (!h) return fail(DS4SP_ERR_INVALID_ARG, "null handle");
    return DS4SP_OK;
}

ds4sp_status check_range(const ds4sp_handle* h, int t0, int n_q) {
    if (t0 < 0 || n_q < 0 || (long long)t0 + n_q > h->cfg.max_tokens)
        return fail(DS4SP_ERR_INVALID_ARG, "token range [%d, %d+%d) outside [0, %d)", t0, t0, n_q,
                    h->cfg.max_tokens);
    if (h->mask && (long long)t0 + n_q > h->mask_rows)
        return fail(DS4SP_ERR_INVALID_ARG, "token range [%d, %d+%d) outside the mask's %d rows",
                    t0, t0, n_q, h->mask_rows);
    return DS4SP_OK;
}

ds4sp_status check_ptr(const void* p, const char* name) {
    if (!p) return fail(DS4SP_ERR_INVALID_ARG, "%s is null", name);
    if (!aligned16(p)) return fail(DS4SP_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
    return DS4SP_OK;
}


ds4sp_status record_last(ds4sp_handle* h, cudaStream_t stream) {
    // Not while the stream is being captured into a graph: the record would belong to
    // the graph, and ds4sp_destroy could not wait on it (replays are the caller's to
    // finish before destroy).
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(stream, &cs) != cudaSuccess)
        return cuda_fail(cudaGetLastError(), "cudaStreamIsCapturing");
    if (cs != cudaStreamCaptureStatusNone) return DS4SP_OK;
    const cudaError_t e = cudaEventRecord(h->last, stream);
    return e == cudaSuccess ? DS4SP_OK : cuda_fail(e, "cudaEventRecord");
}

ds4sp_status indexer_topk_impl(ds4sp_handle* h, const void* q_idx, const void* k_idx,
                               const float* w, int t0, int n_q, int32_t* topk, void* ws,
                               size_t ws_bytes, cudaStream_t stream) {
    DS4SP_TRY(check_range(h, t0, n_q));
    if (n_q == 0) return DS4SP_OK;
    const int k = h->cfg.top_k;
    if (k == 0) return DS4SP_OK;  // nothing to select, nothing to write
    const int t_last = t0 + n_q - 1;
    DS4SP_TRY(check_ptr(q_idx, "q_idx"));
    if (nvis(t_last, h->cfg.ratio) > 0) DS4SP_TRY(check_ptr(k_idx, "k_idx"));
    DS4SP_TRY(check_ptr(w, "w"));
    DS4SP_TRY(check_ptr(topk, "topk"));
    DS4SP_TRY(check_ptr(ws, "ws"));
    if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
        return fail(DS4SP_ERR_INVALID_ARG, "ws is not 256-byte aligned");
    if (nvis(t_last, h->cfg.ratio) > kMaxTopkCandidates)
        return fail(DS4SP_ERR_UNSUPPORTED, "%d candidate rows exceed the top-k limit %d",
                    nvis(t_last, h->cfg.ratio), kMaxTopkCandidates);
    const size_t need = ds4sp_workspace_bytes(h, t0, n_q);
    if (ws_bytes < need)
        return fail(DS4SP_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
    if (h->cfg.topk_mode == 1) {
        // Fused indexer + top-k where the call qualifies, else the two kernels below.
        const ds4sp_status fs =
            h->cfg.d_idx == 64 ? dispatch_fused_h<64>(h, q_idx, k_idx, w, t0, n_q, topk, stream)
                               : dispatch_fused_h<128>(h, q_idx, k_idx, w, t0, n_q, topk, stream);
        if (fs == DS4SP_OK) return record_last(h, stream);
        if (fs != DS4SP_ERR_UNSUPPORTED) return fs;
    }
    const int ld = score_ld(t_last, h->cfg.ratio);
    float* scores = static_cast<float*>(ws);
    const ds4sp_status s =
        h->cfg.d_idx == 64
            ? dispatch_indexer_h<64>(h, q_idx, k_idx, w, t0, n_q, scores, ld, stream)
            : dispatch_indexer_h<128>(h, q_idx, k_idx, w, t0, n_q, scores, ld, stream);
    DS4SP_TRY(s);
    DS4SP_TRY(launch_topk(h, scores, ld, t0, n_q, topk, stream));
    return record_last(h, stream);
}

ds4sp_status sparse_attn_impl(ds4sp_handle* h, const void* q, const void* kv_raw,
                              const void* kv_cmp, const int32_t* topk, int t0, int n_q,
                              float* out, cudaStream_t stream, const void* prefetch = nullptr,
                              size_t prefetch_bytes = 0) {
    DS4SP_TRY(check_range(h, t0, n_q));
    if (n_q == 0) return DS4SP_OK;
    DS4SP_TRY(check_ptr(q, "q"));
    DS4SP_TRY(check_ptr(kv_raw, "kv_raw"));
    DS4SP_TRY(check_ptr(out, "out"));
    if (h->cfg.top_k > 0) {
        DS4SP_TRY(check_ptr(topk, "topk"));
        if (nvis(t0 + n_q - 1, h->cfg.ratio) > 0) DS4SP_TRY(check_ptr(kv_cmp, "kv_cmp"));
    }
    DS4SP_TRY(launch_attn(h, q, kv_raw, kv_cmp, topk, t0, n_q, out, stream, prefetch,
                          prefetch_bytes));
    return record_last(h, stream);
}

// Steps 1-3 for tokens [t0, t0+n_q) on whole-sequence base pointers (q, q_idx, w,
// topk, out are offset here to row t0; the KV tensors are used as given).
ds4sp_status prefill_range(ds4sp_handle* h, int t0, int n_q, const void* q, const void* q_idx,
                           const float* w, const void* kv_raw, const void* kv_cmp,
                           const void* k_idx, int32_t* topk, float* out, void* ws,
                           size_t ws_bytes, cudaStream_t s, const void* prefetch,
                           size_t prefetch_bytes) {
    const ds4sp_config& c = h->cfg;
    auto* qh = static_cast<const __half*>(q) + (size_t)t0 * c.n_heads * c.d_qk;
    auto* qi = static_cast<const __half*>(q_idx) + (size_t)t0 * c.n_idx_heads * c.d_idx;
    const float* wt = w + (size_t)t0 * c.n_idx_heads;
    int32_t* tk = c.top_k > 0 ? topk + (size_t)t0 * c.top_k : nullptr;
    float* ot = out + (size_t)t0 * c.n_heads * c.d_v;
    if (c.top_k > 0) DS4SP_TRY(indexer_topk_impl(h, qi, k_idx, wt, t0, n_q, tk, ws, ws_bytes, s));
    return sparse_attn_impl(h, qh, kv_raw, kv_cmp, tk, t0, n_q, ot, s, prefetch, prefetch_bytes);
}

}  // namespace

extern "C" {

ds4sp_status ds4sp_create(const ds4sp_config* cfg, ds4sp_handle** out) {
    if (!out) return fail(DS4SP_ERR_INVALID_ARG, "out is null");
    *out = nullptr;
    if (!cfg) return fail(DS4SP_ERR_INVALID_ARG, "cfg is null");
    const ds4sp_config& c = *cfg;
    if (c.n_heads != 16 || c.d_qk != 576 || c.d_v != 512 || c.ratio != 4)
        return fail(DS4SP_ERR_UNSUPPORTED, "supported: n_heads 16, d_qk 576, d_v 512, ratio 4");
    if (c.d_idx != 64 && c.d_idx != 128)
        return fail(DS4SP_ERR_UNSUPPORTED, "d_idx %d (supported: 64, 128)", c.d_idx);
    if (c.n_idx_heads < 4 || c.n_idx_heads > 64 || (c.n_idx_heads & (c.n_idx_heads - 1)))
        return fail(DS4SP_ERR_UNSUPPORTED, "n_idx_heads %d (supported: 4, 8, 16, 32, 64)",
                    c.n_idx_heads);
    if (c.top_k > attn::MAX_TOPK)
        return fail(DS4SP_ERR_UNSUPPORTED, "top_k %d (supported: up to %d)", c.top_k, attn::MAX_TOPK);
    if (c.top_k < 0 || c.n_swa < 1 || c.band < 1 || c.max_tokens < 1 || c.max_tokens > (1 << 24) ||
        !(c.softmax_scale == c.softmax_scale))
        return fail(DS4SP_ERR_INVALID_ARG, "top_k >= 0, n_swa >= 1, band >= 1, "
                                           "1 <= max_tokens <= 2^24 and a finite scale required");
    if (c.exp_mode != 0 && c.exp_mode != 1)
        return fail(DS4SP_ERR_INVALID_ARG, "exp_mode %d (0 = ex2.approx, 1 = exp2f)", c.exp_mode);
    if (c.pv_mode != 0 && c.pv_mode != 1)
        return fail(DS4SP_ERR_INVALID_ARG, "pv_mode %d (0 = fp16 P, 1 = fp32-staged P)", c.pv_mode);
    if (c.topk_mode != 0 && c.topk_mode != 1)
        return fail(DS4SP_ERR_INVALID_ARG, "topk_mode %d (0 = separate top-k, 1 = fused)", c.topk_mode);
    if (c.attn_kernel != 0 && c.attn_kernel != 1)
        return fail(DS4SP_ERR_INVALID_ARG, "attn_kernel %d (0 = mma.sync streaming, 1 = tcgen05 logits)",
                    c.attn_kernel);
    if (c.indexer_kernel != 0 && c.indexer_kernel != 1)
        return fail(DS4SP_ERR_INVALID_ARG, "indexer_kernel %d (0 = one CTA per tile, 1 = CTA pairs)",
                    c.indexer_kernel);
    if (c.attn_kernel == 1 && (c.kv_format != 0 || c.exp_mode != 0 || c.pv_mode != 0))
        return fail(DS4SP_ERR_UNSUPPORTED, "attn_kernel 1 runs fp16 rows with exp_mode 0 and pv_mode 0");
    if (c.dependent_launch != 0 && c.dependent_launch != 1)
        return fail(DS4SP_ERR_INVALID_ARG, "dependent_launch %d (0 or 1)", c.dependent_launch);
    if (c.kv_format < 0 || c.kv_format > 3)
        return fail(DS4SP_ERR_INVALID_ARG, "kv_format %d (0 = fp16, 1 = Q8_0, 2 = Q4_0, 3 = Q8 K / Q4 V)",
                    c.kv_format);
    if (c.kv_format >= 1 && c.kv_format <= 3 && c.top_k > attn_max_topk(c.kv_format))
        return fail(DS4SP_ERR_UNSUPPORTED, "kv_format %d supports top_k up to %d", c.kv_format,
                    attn_max_topk(c.kv_format));
    if (c.kv_format != 0 && (c.exp_mode != 0 || c.pv_mode != 0))
        return fail(DS4SP_ERR_UNSUPPORTED, "a quantized cache runs with exp_mode 0 and pv_mode 0");
    ds4sp_handle* h = new (std::nothrow) ds4sp_handle();
    if (!h) return fail(DS4SP_ERR_INVALID_ARG, "out of host memory");
    h->cfg = c;
    cudaError_t e = cudaGetDevice(&h->device);
    if (e == cudaSuccess)
        e = cudaDeviceGetAttribute(&h->sm_count, cudaDevAttrMultiProcessorCount, h->device);
    if (e == cudaSuccess) e = cudaMalloc(&h->d_status, 2 * sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaMemset(h->d_status, 0, 2 * sizeof(uint32_t));
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&h->last, cudaEventDisableTiming);
    // Partials of split-mode attention (calls of few tokens): two 32-row units per SM.
    if (e == cudaSuccess) {
        h->split_cap = 2 * h->sm_count;
        e = cudaMalloc(&h->part_o, (size_t)h->split_cap * c.n_heads * c.d_v * sizeof(float));
        if (e == cudaSuccess)
            e = cudaMalloc(&h->part_ml, (size_t)h->split_cap * 2 * c.n_heads * sizeof(float));
    }
    if (e != cudaSuccess) {
        ds4sp_destroy(h);
        return cuda_fail(e, "ds4sp_create");
    }
    *out = h;
    return DS4SP_OK;
}

ds4sp_status ds4sp_destroy(ds4sp_handle* h) {
    if (!h) return DS4SP_OK;
    ds4sp_status s = DS4SP_OK;
    if (h->last && cudaEventSynchronize(h->last) != cudaSuccess)
        s = fail(DS4SP_ERR_CUDA, "pending work failed before destroy");
    for (auto& tl : h->timed) {
        cudaEventSynchronize(tl.stop);
        cudaEventDestroy(tl.start);
        cudaEventDestroy(tl.stop);
    }
    for (auto e : h->event_pool) cudaEventDestroy(e);
    if (h->copy_in && cudaStreamSynchronize(h->copy_in) != cudaSuccess)
        s = fail(DS4SP_ERR_CUDA, "pending copies failed before destroy");
    if (h->copy_out && cudaStreamSynchronize(h->copy_out) != cudaSuccess)
        s = fail(DS4SP_ERR_CUDA, "pending copies failed before destroy");
    for (auto e : h->step_in) cudaEventDestroy(e);
    for (auto e : h->step_done) cudaEventDestroy(e);
    if (h->host_start) cudaEventDestroy(h->host_start);
    if (h->host_end) cudaEventDestroy(h->host_end);
    if (h->copy_in) cudaStreamDestroy(h->copy_in);
    if (h->copy_out) cudaStreamDestroy(h->copy_out);
    if (h->last) cudaEventDestroy(h->last);
    if (h->d_status) cudaFree(h->d_status);
    if (h->part_o) cudaFree(h->part_o);
    if (h->part_ml) cudaFree(h->part_ml);
    delete h;
    return s;
}

size_t ds4sp_workspace_bytes(const ds4sp_handle* h, int t0, int n_q) {
    if (!h || t0 < 0 || n_q <= 0 || (long long)t0 + n_q > h->cfg.max_tokens) return 0;
    const int ld = score_ld(t0 + n_q - 1, h->cfg.ratio);
    const size_t bytes = (size_t)n_q * ld * sizeof(float);
    return (bytes + 255) / 256 * 256;
}

ds4sp_status ds4sp_indexer_topk(ds4sp_handle* h, const void* q_idx, const void* k_idx,
                                const float* w, int t0, int n_q, int32_t* topk, void* ws,
                                size_t ws_bytes, void* stream) {
    const TraceRange trace("ds4sp_indexer_topk");
    DS4SP_TRY(check_handle(h));
    return indexer_topk_impl(h, q_idx, k_idx, w, t0, n_q, topk, ws, ws_bytes,
                             static_cast<cudaStream_t>(stream));
}

ds4sp_status ds4sp_sparse_attn(ds4sp_handle* h, const void* q, const void* kv_raw,
                               const void* kv_cmp, const int32_t* topk, int t0, int n_q,
                               float* out, void* stream) {
    const TraceRange trace("ds4sp_sparse_attn");
    DS4SP_TRY(check_handle(h));
    return sparse_attn_impl(h, q, kv_raw, kv_cmp, topk, t0, n_q, out,
                            static_cast<cudaStream_t>(stream));
}

ds4sp_status ds4sp_prefill_band(ds4sp_handle* h, int b, int n_tokens, const void* q,
                                const void* q_idx, const float* w, const void* kv_raw,
                                const void* kv_cmp, const void* k_idx, int32_t* topk,
                                float* out, void* ws, size_t ws_bytes, void* stream) {
    const TraceRange trace("ds4sp_prefill_band");
    DS4SP_TRY(check_handle(h));
    const ds4sp_config& c = h->cfg;
    if (n_tokens < 1 || n_tokens > c.max_tokens)
        return fail(DS4SP_ERR_INVALID_ARG, "n_tokens %d outside [1, %d]", n_tokens, c.max_tokens);
    if (b < 0 || (long long)b * c.band >= n_tokens)
        return fail(DS4SP_ERR_INVALID_ARG, "band %d outside the %d-token sequence", b, n_tokens);
    if (b != h->next_band)
        return fail(DS4SP_ERR_ORDER, "band %d called, band %d expected next", b, h->next_band);
    DS4SP_TRY(check_ptr(q, "q"));
    DS4SP_TRY(check_ptr(q_idx, "q_idx"));
    DS4SP_TRY(check_ptr(w, "w"));
    DS4SP_TRY(check_ptr(kv_raw, "kv_raw"));
    DS4SP_TRY(check_ptr(out, "out"));
    const int t0 = b * c.band;
    const int n_q = std::min(c.band, n_tokens - t0);
    if (c.top_k > 0) {
        DS4SP_TRY(check_ptr(topk, "topk"));
        if (nvis(t0 + n_q - 1, c.ratio) > 0) {   // some token of the band sees a compressed row
            DS4SP_TRY(check_ptr(kv_cmp, "kv_cmp"));
            DS4SP_TRY(check_ptr(k_idx, "k_idx"));
        }
    }
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    if (c.top_k > 0 && ws_bytes < ds4sp_workspace_bytes(h, t0, n_q))
        return fail(DS4SP_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes,
                    ds4sp_workspace_bytes(h, t0, n_q));
    // The next band's indexer queries (read first thing by its indexer) are brought into
    // L2 at the tail of this band's attention.
    const int t1 = t0 + n_q, n_next = std::min(c.band, n_tokens - t1);
    const void* pf = nullptr;
    size_t pf_bytes = 0;
    if (c.top_k > 0 && n_next > 0) {
        pf = static_cast<const __half*>(q_idx) + (size_t)t1 * c.n_idx_heads * c.d_idx;
        pf_bytes = (size_t)n_next * c.n_idx_heads * c.d_idx * 2;
    }
    DS4SP_TRY(prefill_range(h, t0, n_q, q, q_idx, w, kv_raw, kv_cmp, k_idx, topk, out, ws,
                            ws_bytes, s, pf, pf_bytes));
    h->next_band = b + 1;
    return DS4SP_OK;
}

ds4sp_status ds4sp_prefill_host(ds4sp_handle* h, int n_tokens, const ds4sp_io* host,
                                const ds4sp_io* dev, void* ws, size_t ws_bytes, void* stream) {
    const TraceRange trace("ds4sp_prefill_host");
    DS4SP_TRY(check_handle(h));
    if (!host || !dev) return fail(DS4SP_ERR_INVALID_ARG, "host or dev is null");
    const ds4sp_config& c = h->cfg;
    if (n_tokens < 1 || n_tokens > c.max_tokens)
        return fail(DS4SP_ERR_INVALID_ARG, "n_tokens %d outside [1, %d]", n_tokens, c.max_tokens);
    const bool sel = c.top_k > 0;
    const int n_c = nvis(n_tokens - 1, c.ratio);   // compressed rows the last token sees
    for (const ds4sp_io* io : {host, dev}) {
        const char* side = io == host ? "host" : "dev";
        if (!io->q || !io->q_idx || !io->w || !io->kv_raw || !io->out)
            return fail(DS4SP_ERR_INVALID_ARG, "%s: null q, q_idx, w, kv_raw or out", side);
        if (n_c > 0 && sel && (!io->kv_cmp || !io->k_idx))
            return fail(DS4SP_ERR_INVALID_ARG, "%s: null kv_cmp or k_idx", side);
    }
    if (sel && !dev->topk) return fail(DS4SP_ERR_INVALID_ARG, "dev: null topk");
    const int n_bands = (n_tokens + c.band - 1) / c.band;
    const size_t need = ds4sp_workspace_bytes(h, (n_bands - 1) * c.band,
                                              n_tokens - (n_bands - 1) * c.band);
    if (sel && ws_bytes < need)
        return fail(DS4SP_ERR_WORKSPACE, "workspace %zu bytes < %zu needed", ws_bytes, need);
    if (sel) {
        DS4SP_TRY(check_ptr(dev->topk, "dev: topk"));
        DS4SP_TRY(check_ptr(ws, "ws"));
    }
    for (const void* p : {static_cast<const void*>(dev->q), static_cast<const void*>(dev->q_idx),
                          static_cast<const void*>(dev->w), static_cast<const void*>(dev->kv_raw),
                          static_cast<const void*>(dev->out)})
        DS4SP_TRY(check_ptr(p, "dev tensor"));

    // Steps of about kHostStep tokens inside each band, in order: band b's tokens
    // [b*band, (b+1)*band) are cut into steps; a step's copies in, its compute and its
    // copies out are queued on three streams, so that copies in, compute and copies out
    // of neighbouring steps overlap and only the last step's output copy trails.
    // A remainder small enough for the few-token attention path joins the step before
    // it, so that no step takes that path unless its whole band does (the device path
    // then takes it too): every token sees the same kernels as in ds4sp_prefill_band.
    struct Step { int band, t0, n; };
    std::vector<Step> steps;
    for (int b = 0; b < n_bands; ++b) {
        const int t0 = b * c.band, t1 = std::min(n_tokens, t0 + c.band);
        for (int u = t0; u < t1;) {
            const int left = t1 - u;
            const int n = left - kHostStep <= attn::SPLIT_MAX_TOKENS ? left : kHostStep;
            steps.push_back({b, u, n});
            u += n;
        }
    }
    // Only the last step's compute and copy out trail the copies in (the link is the
    // bound): cut the last kHostTail tokens into a step of their own.
    if (steps.back().n - kHostTail > attn::SPLIT_MAX_TOKENS) {
        Step& last = steps.back();
        last.n -= kHostTail;
        steps.push_back({last.band, last.t0 + last.n, kHostTail});
    }
    const int n_steps = (int)steps.size();

    cudaError_t e = cudaSuccess;
    if (!h->copy_in) e = cudaStreamCreateWithFlags(&h->copy_in, cudaStreamNonBlocking);
    if (e == cudaSuccess && !h->copy_out)
        e = cudaStreamCreateWithFlags(&h->copy_out, cudaStreamNonBlocking);
    if (e == cudaSuccess && !h->host_start)
        e = cudaEventCreateWithFlags(&h->host_start, cudaEventDisableTiming);
    if (e == cudaSuccess && !h->host_end)
        e = cudaEventCreateWithFlags(&h->host_end, cudaEventDisableTiming);
    while (e == cudaSuccess && (int)h->step_in.size() < n_steps) {
        cudaEvent_t a = nullptr, b = nullptr;
        e = cudaEventCreateWithFlags(&a, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&b, cudaEventDisableTiming);
        if (e != cudaSuccess) {
            if (a) cudaEventDestroy(a);
            break;
        }
        h->step_in.push_back(a);
        h->step_done.push_back(b);
    }
    if (e != cudaSuccess) return cuda_fail(e, "ds4sp_prefill_host: streams/events");

    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    // Copies start after whatever the caller queued on `stream` before this call.
    e = cudaEventRecord(h->host_start, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(h->copy_in, h->host_start, 0);
    if (e != cudaSuccess) return cuda_fail(e, "ds4sp_prefill_host: ordering");

    const size_t q_row = (size_t)c.n_heads * c.d_qk * 2, qi_row = (size_t)c.n_idx_heads * c.d_idx * 2;
    const size_t w_row = (size_t)c.n_idx_heads * 4, kv_row = (size_t)kv_row_bytes_of(c);
    const size_t ki_row = (size_t)c.d_idx * 2, o_row = (size_t)c.n_heads * c.d_v * 4;
    const size_t tk_row = (size_t)c.top_k * 4;
    auto h2d = [&](const void* dst, const void* src, size_t off, size_t bytes) {
        if (bytes == 0) return cudaSuccess;
        return cudaMemcpyAsync(static_cast<char*>(const_cast<void*>(dst)) + off,
                               static_cast<const char*>(src) + off, bytes,
                               cudaMemcpyHostToDevice, h->copy_in);
    };
    auto d2h = [&](void* dst, const void* src, size_t off, size_t bytes) {
        if (bytes == 0) return cudaSuccess;
        return cudaMemcpyAsync(static_cast<char*>(dst) + off, static_cast<const char*>(src) + off,
                               bytes, cudaMemcpyDeviceToHost, h->copy_out);
    };
    // Inputs: per step, its token rows and the KV rows it is the first to need.
    int raw_done = 0, cmp_done = 0;
    for (int i = 0; i < n_steps && e == cudaSuccess; ++i) {
        const int t0 = steps[i].t0, n = steps[i].n, t1 = t0 + n;
        e = h2d(dev->q, host->q, t0 * q_row, n * q_row);
        if (e == cudaSuccess && sel) e = h2d(dev->q_idx, host->q_idx, t0 * qi_row, n * qi_row);
        if (e == cudaSuccess && sel) e = h2d(dev->w, host->w, t0 * w_row, n * w_row);
        if (e == cudaSuccess) e = h2d(dev->kv_raw, host->kv_raw, raw_done * kv_row, (t1 - raw_done) * kv_row);
        raw_done = t1;
        const int cmp_need = sel ? nvis(t1 - 1, c.ratio) : 0;
        if (e == cudaSuccess && cmp_need > cmp_done) {
            e = h2d(dev->kv_cmp, host->kv_cmp, cmp_done * kv_row, (cmp_need - cmp_done) * kv_row);
            if (e == cudaSuccess)
                e = h2d(dev->k_idx, host->k_idx, cmp_done * ki_row, (cmp_need - cmp_done) * ki_row);
            cmp_done = cmp_need;
        }
        if (e == cudaSuccess) e = cudaEventRecord(h->step_in[i], h->copy_in);
    }
    if (e != cudaSuccess) return cuda_fail(e, "ds4sp_prefill_host: copies in");

    // Compute, step by step in band order, each after its inputs; outputs copied back
    // step by step.
    h->next_band = 0;
    for (int i = 0; i < n_steps; ++i) {
        const int t0 = steps[i].t0, n = steps[i].n;
        e = cudaStreamWaitEvent(s, h->step_in[i], 0);
        if (e != cudaSuccess) return cuda_fail(e, "ds4sp_prefill_host: wait for inputs");
        DS4SP_TRY(prefill_range(h, t0, n, dev->q, dev->q_idx, dev->w, dev->kv_raw, dev->kv_cmp,
                                dev->k_idx, dev->topk, dev->out, ws, ws_bytes, s, nullptr, 0));
        if (i + 1 == n_steps || steps[i + 1].band != steps[i].band)
            h->next_band = steps[i].band + 1;
        e = cudaEventRecord(h->step_done[i], s);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(h->copy_out, h->step_done[i], 0);
        if (e == cudaSuccess) e = d2h(host->out, dev->out, t0 * o_row, n * o_row);
        if (e == cudaSuccess && sel && host->topk)
            e = d2h(host->topk, dev->topk, t0 * tk_row, n * tk_row);
        if (e != cudaSuccess) return cuda_fail(e, "ds4sp_prefill_host: copies out");
    }
    // `stream` completes only after the last copy out.
    e = cudaEventRecord(h->host_end, h->copy_out);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, h->host_end, 0);
    if (e != cudaSuccess) return cuda_fail(e, "ds4sp_prefill_host: ordering");
    return record_last(h, s);
}

ds4sp_status ds4sp_reset(ds4sp_handle* h, int next_band) {
    DS4SP_TRY(check_handle(h));
    if (next_band < 0) return fail(DS4SP_ERR_INVALID_ARG, "next_band %d < 0", next_band);
    h->next_band = next_band;
    return DS4SP_OK;
}

int ds4sp_next_band(const ds4sp_handle* h) { return h ? h->next_band : -1; }

ds4sp_status ds4sp_device_status(ds4sp_handle* h, void* stream, uint32_t* bits) {
    DS4SP_TRY(check_handle(h));
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    uint32_t word = 0;
    cudaError_t e = cudaStreamSynchronize(s);
    if (e == cudaSuccess) e = cudaMemcpy(&word, h->d_status, sizeof(word), cudaMemcpyDeviceToHost);
    // Both words: the status and the launch give-up word (a replayed graph reuses its
    // launches' epochs, which a stale give-up word would match).
    if (e == cudaSuccess) e = cudaMemset(h->d_status, 0, 2 * sizeof(uint32_t));
    if (e != cudaSuccess) return cuda_fail(e, "ds4sp_device_status");
    if (bits) *bits = word;
    if (word) return fail(DS4SP_ERR_DEVICE_BOUNDS, "device status word 0x%x", word);
    return DS4SP_OK;
}

ds4sp_status ds4sp_profile_enable(ds4sp_handle* h, int enable) {
    DS4SP_TRY(check_handle(h));
    h->profiling = enable != 0;
    return DS4SP_OK;
}

ds4sp_status ds4sp_profile_read(ds4sp_handle* h, double ms[3], int launches[3]) {
    DS4SP_TRY(check_handle(h));
    if (!ms || !launches) return fail(DS4SP_ERR_INVALID_ARG, "null output");
    for (int k = 0; k < 3; ++k) {
        ms[k] = 0.0;
        launches[k] = 0;
    }
    ds4sp_status st = DS4SP_OK;
    for (auto& tl : h->timed) {
        float m = 0.f;
        cudaError_t e = cudaEventSynchronize(tl.stop);
        if (e == cudaSuccess) e = cudaEventElapsedTime(&m, tl.start, tl.stop);
        if (e != cudaSuccess && st == DS4SP_OK) st = cuda_fail(e, "ds4sp_profile_read");
        ms[tl.kind] += m;
        launches[tl.kind] += 1;
        h->event_pool.push_back(tl.start);
        h->event_pool.push_back(tl.stop);
    }
    h->timed.clear();
    return st;
}

ds4sp_status ds4sp_debug_fail_launches(ds4sp_handle* h, int n) {
    DS4SP_TRY(check_handle(h));
    if (n < 0) return fail(DS4SP_ERR_INVALID_ARG, "n < 0");
    h->fail_launches = n;
    return DS4SP_OK;
}

ds4sp_status ds4sp_debug_set_wait_limit_ns(ds4sp_handle* h, long long ns) {
    DS4SP_TRY(check_handle(h));
    h->wait_limit_ns = ns < 0 ? kWaitLimitNs : (unsigned long long)ns;
    return DS4SP_OK;
}

ds4sp_status ds4sp_debug_set_mask(ds4sp_handle* h, const uint8_t* mask, int rows, int cols) {
    DS4SP_TRY(check_handle(h));
    if (mask == nullptr) {
        h->mask = nullptr;
        h->mask_rows = h->mask_cols = 0;
        return DS4SP_OK;
    }
    if (rows < 1 || cols < 1) return fail(DS4SP_ERR_INVALID_ARG, "mask of %d x %d", rows, cols);
    h->mask = mask;
    h->mask_rows = rows;
    h->mask_cols = cols;
    return DS4SP_OK;
}

int ds4sp_kv_row_bytes(int kv_format, int dims) {
    if (kv_format < kFmtQ8 || kv_format > kFmtQ8Q4 || dims < kQBlock || dims % kQBlock || dims > 4096)
        return 0;
    if (kv_format == kFmtQ8Q4 && dims < kValueDims) return 0;
    return quant_row_bytes(kv_format, dims);
}

ds4sp_status ds4sp_quantize_kv(const void* x, int rows, int dims, int kv_format, void* out,
                               void* stream) {
    const TraceRange trace("ds4sp_quantize_kv");
    const int rb = ds4sp_kv_row_bytes(kv_format, dims);
    if (rb == 0)
        return fail(DS4SP_ERR_INVALID_ARG, "kv_format %d with %d dims (1 = Q8_0 or 2 = Q4_0, "
                    "dims a multiple of 32 up to 4096)", kv_format, dims);
    if (rows < 0) return fail(DS4SP_ERR_INVALID_ARG, "rows %d", rows);
    if (rows == 0) return DS4SP_OK;
    DS4SP_TRY(check_ptr(x, "x"));
    DS4SP_TRY(check_ptr(out, "out"));
    const cudaStream_t st = static_cast<cudaStream_t>(stream);
    // (format, values, byte offset) of each part of a stored row
    struct Part { int fmt, dims, off; };
    Part parts[2] = {{kv_format, dims, 0}, {0, 0, 0}};
    int n_parts = 1;
    if (kv_format == kFmtQ8Q4) {
        parts[0] = {kFmtQ8, dims, 0};
        parts[1] = {kFmtQ4, kValueDims, quant_row_bytes(kFmtQ8, dims)};
        n_parts = 2;
    }
    for (int i = 0; i < n_parts; ++i) {
        const long long n = (long long)rows * (parts[i].dims / kQBlock);
        const int threads = 256;
        const long long grid = (n + threads - 1) / threads;
        if (grid > 0x7fffffffLL) return fail(DS4SP_ERR_INVALID_ARG, "%d rows is too many", rows);
        quantize_rows_kernel<<<(unsigned)grid, threads, 0, st>>>(
            static_cast<const __half*>(x), dims, rows, parts[i].dims, parts[i].fmt,
            static_cast<uint8_t*>(out), rb, parts[i].off);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) return cuda_fail(e, "quantize launch");
    }
    return DS4SP_OK;
}

ds4sp_status ds4sp_probe_gather(const void* table, int table_rows, int row_bytes,
                                const int32_t* idx, int n, uint32_t* sink, int grid, void* stream) {
    const TraceRange trace("ds4sp_probe_gather");
    if (row_bytes < 16 || row_bytes % 16 != 0 || row_bytes > 16 * 8 * 9)
        return fail(DS4SP_ERR_INVALID_ARG, "row_bytes %d (a multiple of 16, at most 1152)", row_bytes);
    if (table_rows < 1 || n < 0 || grid < 1 || grid > 65535)
        return fail(DS4SP_ERR_INVALID_ARG, "table_rows %d, n %d, grid %d", table_rows, n, grid);
    if (n == 0) return DS4SP_OK;
    DS4SP_TRY(check_ptr(table, "table"));
    DS4SP_TRY(check_ptr(idx, "idx"));
    if (!sink || (reinterpret_cast<uintptr_t>(sink) & 3u))
        return fail(DS4SP_ERR_INVALID_ARG, "sink is null or not 4-byte aligned");
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    probe_gather_kernel<9><<<grid, kProbeThreads, 0, s>>>(static_cast<const uint4*>(table),
                                                          row_bytes / 16, idx, n, sink);
    const cudaError_t e = cudaGetLastError();
    return e == cudaSuccess ? DS4SP_OK : cuda_fail(e, "probe_gather launch");
}

const char* ds4sp_status_string(ds4sp_status s) {
    switch (s) {
        case DS4SP_OK: return "ok";
        case DS4SP_ERR_INVALID_ARG: return "invalid argument";
        case DS4SP_ERR_UNSUPPORTED: return "unsupported shape";
        case DS4SP_ERR_ORDER: return "band out of order";
        case DS4SP_ERR_WORKSPACE: return "workspace too small";
        case DS4SP_ERR_CUDA: return "CUDA error";
        case DS4SP_ERR_DEVICE_BOUNDS: return "device index or wait check failed";
    }
    return "unknown status";
}

const char* ds4sp_last_error(void) { return g_last_error.c_str(); }

}  // extern "C"

// ---------------------------------------------------------------------------------
// Indexer + top-k without any device allocation.
//
// The score scratch of ds4sp_indexer_topk_noalloc lives in the fixed-size array below,
// which the library image carries: every GPU that loads the library holds these 8 MiB
// (plus one status word) until the process exits. In host code `g_static_scores` is only
// a host-side stand-in for the symbol, not a device address; the device address comes
// from cudaGetSymbolAddress, looked up once per device with that device current.
// ---------------------------------------------------------------------------------

namespace {

constexpr size_t kStaticScoreFloats = size_t(1) << 21;   // 8 MiB of fp32 scores

__device__ __align__(256) float g_static_scores[kStaticScoreFloats];
__device__ __align__(256) uint32_t g_static_status[4];

struct StaticScratch {
    float* scores = nullptr;
    uint32_t* status = nullptr;   // [0] status word, [1] abort word of the bounded waits
    int device = 0;
    int sm_count = 0;
    bool ready = false;
};

StaticScratch g_static[kMaxDevices];
std::atomic<uint32_t> g_static_epoch{0};
std::mutex g_static_mu;

// Device addresses of the static arrays on the current device (set-up on first use).
ds4sp_status static_scratch(StaticScratch* out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices) return fail(DS4SP_ERR_UNSUPPORTED, "device %d", dev);
    std::lock_guard<std::mutex> lock(g_static_mu);
    StaticScratch& s = g_static[dev];
    if (!s.ready) {
        e = cudaGetSymbolAddress(reinterpret_cast<void**>(&s.scores), g_static_scores);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scores)");
        e = cudaGetSymbolAddress(reinterpret_cast<void**>(&s.status), g_static_status);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
        e = cudaDeviceGetAttribute(&s.sm_count, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
        s.device = dev;
        s.ready = true;
    }
    *out = s;
    return DS4SP_OK;
}

ds4sp_status check_static_config(const ds4sp_config* cfg) {
    if (!cfg) return fail(DS4SP_ERR_INVALID_ARG, "cfg is null");
    const ds4sp_config& c = *cfg;
    if (c.n_heads != 16 || c.d_qk != 576 || c.d_v != 512 || c.ratio != 4)
        return fail(DS4SP_ERR_UNSUPPORTED, "supported: n_heads 16, d_qk 576, d_v 512, ratio 4");
    if (c.d_idx != 64 && c.d_idx != 128)
        return fail(DS4SP_ERR_UNSUPPORTED, "d_idx %d (supported: 64, 128)", c.d_idx);
    if (c.n_idx_heads < 4 || c.n_idx_heads > 64 || (c.n_idx_heads & (c.n_idx_heads - 1)))
        return fail(DS4SP_ERR_UNSUPPORTED, "n_idx_heads %d (supported: 4, 8, 16, 32, 64)",
                    c.n_idx_heads);
    if (c.top_k < 0 || c.top_k > attn::MAX_TOPK || c.max_tokens < 1 || c.max_tokens > (1 << 24))
        return fail(DS4SP_ERR_INVALID_ARG, "0 <= top_k <= %d and 1 <= max_tokens <= 2^24 required",
                    attn::MAX_TOPK);
    if (c.indexer_kernel != 0 && c.indexer_kernel != 1)
        return fail(DS4SP_ERR_INVALID_ARG, "indexer_kernel %d (0 or 1)", c.indexer_kernel);
    return DS4SP_OK;
}

}  // namespace

extern "C" ds4sp_status ds4sp_indexer_topk_noalloc(const ds4sp_config* cfg, const void* q_idx,
                                                   const void* k_idx, const float* w, int t0,
                                                   int n_q, int32_t* topk, void* stream) {
    const TraceRange trace("ds4sp_indexer_topk_noalloc");
    DS4SP_TRY(check_static_config(cfg));
    if (t0 < 0 || n_q < 0 || (long long)t0 + n_q > cfg->max_tokens)
        return fail(DS4SP_ERR_INVALID_ARG, "token range [%d, %d+%d) outside [0, %d)", t0, t0, n_q,
                    cfg->max_tokens);
    if (n_q == 0 || cfg->top_k == 0) return DS4SP_OK;
    const int ld = score_ld(t0 + n_q - 1, cfg->ratio);
    if ((size_t)n_q * ld > kStaticScoreFloats)
        return fail(DS4SP_ERR_WORKSPACE,
                    "%d tokens x %d score columns exceed the static scratch of %zu floats (8 MiB)",
                    n_q, ld, kStaticScoreFloats);
    const int t_last = t0 + n_q - 1;
    DS4SP_TRY(check_ptr(q_idx, "q_idx"));
    if (nvis(t_last, cfg->ratio) > 0) DS4SP_TRY(check_ptr(k_idx, "k_idx"));
    DS4SP_TRY(check_ptr(w, "w"));
    DS4SP_TRY(check_ptr(topk, "topk"));
    if (nvis(t_last, cfg->ratio) > kMaxTopkCandidates)
        return fail(DS4SP_ERR_UNSUPPORTED, "%d candidate rows exceed the top-k limit %d",
                    nvis(t_last, cfg->ratio), kMaxTopkCandidates);
    StaticScratch sc;
    DS4SP_TRY(static_scratch(&sc));
    const cudaStream_t s = static_cast<cudaStream_t>(stream);
    // A handle on the stack carries the launch settings; it owns no device memory. Its
    // status and abort words are the library's static ones; each call takes fresh wait
    // epochs, so a give-up in an earlier call never shortens this call's waits.
    ds4sp_handle tmp;
    tmp.cfg = *cfg;
    tmp.device = sc.device;
    tmp.d_status = sc.status;
    tmp.sm_count = sc.sm_count;
    tmp.epoch = g_static_epoch.fetch_add(16);
    // The status word is internal to this entry point; clear it once the arguments
    // have passed every check.
    const cudaError_t e = cudaMemsetAsync(sc.status, 0, sizeof(uint32_t), s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(status)");
    ds4sp_status st = cfg->d_idx == 64
             ? dispatch_indexer_h<64>(&tmp, q_idx, k_idx, w, t0, n_q, sc.scores, ld, s)
             : dispatch_indexer_h<128>(&tmp, q_idx, k_idx, w, t0, n_q, sc.scores, ld, s);
    if (st != DS4SP_OK) return st;
    return launch_topk(&tmp, sc.scores, ld, t0, n_q, topk, s);
}
