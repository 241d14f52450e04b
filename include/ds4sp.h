/*
 * ds4sp.h -- C ABI of libds4sp: DS4 sparse-prefill attention on NVIDIA B200 (sm_100a).
 *
 * Per query token t the library runs three steps:
 *   1. indexer:   score(t, j) = sum_h w[t,h] * ReLU(q_idx[t,h,:] . k_idx[j,:])
 *                 for every compressed row j visible to t (4j + 3 <= t);
 *   2. top-k:     keep the min(k, n_vis(t)) best rows, equal scores to the lower j,
 *                 listed by ascending j, unused slots -1;
 *   3. attention: one softmax of 16 query heads over the selected compressed rows
 *                 and the raw rows max(0, t-n_swa+1) .. t; key = all 576 dims of a
 *                 row, value = its first 512 dims.
 * Tokens are processed in 2048-token bands in chronological order.
 *
 * Sources: "perf(ds4): extend sparse prefill scheduling to 10K", Summary (five
 * 2,048-token bands up to a 10,240-token frontier; ratio-4 causal visibility derived
 * in the kernel instead of a stored quadratic mask; top-k rows handed directly to
 * attention; F16 transport of selected rows; each selected latent row streamed once
 * across sixteen heads; chronological state commit) and Qualification (ratio-4
 * boundary formula; explicit-mask versus analytic-mask oracle). The pages do not
 * define the indexer score, the tie rule or the window; this library fixes them as
 * written above.
 *
 * Conventions for every entry point
 *   - Tensors are caller-owned device memory, contiguous and row-major, and every
 *     pointer is 16-byte aligned. fp16 means IEEE binary16; fp32 means IEEE binary32.
 *   - Per-token tensors (q, q_idx, w, topk, out) start at token t0: row 0 is token t0.
 *     KV tensors (kv_raw, kv_cmp, k_idx) are whole-sequence base pointers holding at
 *     least max_tokens (raw) or max_tokens/4 (compressed) rows.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy default
 *     stream). The library launches kernels only; it never allocates or frees caller
 *     memory, copies it only in ds4sp_prefill_host (between the caller's host and
 *     device buffers), and never synchronises the caller's stream except where stated.
 *   - Argument, shape, order and workspace errors are returned before any launch.
 *     A failed launch returns DS4SP_ERR_CUDA. Index checks inside the kernels never
 *     fault: an out-of-range index is skipped and recorded in a device status word
 *     that ds4sp_device_status() reads.
 *   - No C++ exception crosses this ABI. A handle is not thread-safe; use one handle
 *     per host thread, or serialise calls.
 */
#ifndef DS4SP_H
#define DS4SP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct ds4sp_handle ds4sp_handle; /* opaque, owned by the library */

typedef enum {
    DS4SP_OK = 0,
    DS4SP_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, bad range or size */
    DS4SP_ERR_UNSUPPORTED = 2,   /* shape outside what the kernels implement */
    DS4SP_ERR_ORDER = 3,         /* band called out of chronological order */
    DS4SP_ERR_WORKSPACE = 4,     /* workspace smaller than ds4sp_workspace_bytes() */
    DS4SP_ERR_CUDA = 5,          /* a CUDA call or kernel launch failed */
    DS4SP_ERR_DEVICE_BOUNDS = 6, /* a kernel met an out-of-range index or gave up a wait */
} ds4sp_status;

/* Model and schedule constants, fixed at ds4sp_create. Supported: n_heads = 16,
 * d_qk = 576, d_v = 512, ratio = 4, d_idx in {64, 128}, n_idx_heads a power of two
 * in [4, 64], 0 <= top_k <= 2048, n_swa >= 1, band >= 1, 1 <= max_tokens <= 2^24;
 * a token may see at most 51,200 compressed rows (top-k keeps a row in shared memory). */
typedef struct {
    int n_heads;         /* query heads sharing each latent row (16) */
    int d_qk;            /* latent row width used as key: 512 latent + 64 rope (576) */
    int d_v;             /* leading dims of the row used as value (512) */
    int ratio;           /* raw tokens per compressed row (4) */
    int n_idx_heads;     /* indexer heads H_i */
    int d_idx;           /* indexer head dim D_i */
    int top_k;           /* compressed rows kept per token, k */
    int n_swa;           /* raw-row sliding window, inclusive of the token itself */
    int band;            /* tokens per band (2048) */
    int max_tokens;      /* sequence length T the KV buffers hold */
    float softmax_scale; /* <= 0 selects 1/sqrt(d_qk) */
    int exp_mode;        /* softmax exponentials: 0 = ex2.approx (about 2^-22 relative
                            error), 1 = exp2f (CUDA's precise function; measured the
                            faster of the two in the streaming kernel, and the Python
                            binding's default where the configuration allows it: fp16
                            rows, attn_kernel 0); other values are DS4SP_ERR_INVALID_ARG */
    int pv_mode;         /* probabilities entering P . V: 0 = one fp16 term (default),
                            1 = fp32-staged: P = hi + lo, two fp16 terms (hi = fp16(p),
                            lo = fp16(p - hi)), about 22 significant bits, at twice the
                            P . V tensor work ("FP32-staged streaming MLA" of "perf(ds4):
                            unify gfx1151 sparse-prefill stack", Validation completed);
                            other values are DS4SP_ERR_INVALID_ARG */
    int topk_mode;       /* steps 1-2: 0 = the indexer writes fp32 scores to the caller's
                            workspace and a top-k kernel reads them back; 1 = one fused
                            kernel keeps each token block's scores in shared memory and
                            selects there, so no score reaches global memory. A call takes
                            the fused kernel when no explicit mask is set and a token
                            block's score rows fit one of its two 40 KB key buffers
                            (256/n_idx_heads tokens x 128 x ceil(n_vis(last token)/128) x 4
                            bytes, e.g. up to 2,560 visible rows -- a 10,240-token context
                            -- at 64 indexer heads) in a call of at most 1,024 token
                            blocks; otherwise the two kernels run. Indices are
                            the same bits either way; 1 is the faster prefill and
                            the Python binding's default. Other values are
                            DS4SP_ERR_INVALID_ARG */
    int kv_format;       /* storage of kv_raw and kv_cmp: 0 = fp16 rows of 576 values
                            (1152 bytes); 1 = Q8_0 and 2 = Q4_0 quantized rows (one row
                            is key and value), 3 = "Q8 K / Q4 V" rows (the Q8_0 row of the
                            576 values is the key, the Q4_0 row of the first 512 the
                            value), of ds4sp_kv_row_bytes(kv_format, 576) bytes (624, 336,
                            912), as ds4sp_quantize_kv writes them. The attention
                            dequantizes the rows it gathers (value d*q or d*(n-8), rounded
                            once to fp16) and otherwise computes as for fp16 rows; the
                            indexer keys (k_idx) stay fp16. Quantized formats need
                            exp_mode 0 and pv_mode 0, and top_k <= 1012 (format 2) or
                            824 (format 3) (else DS4SP_ERR_UNSUPPORTED); other values are DS4SP_ERR_INVALID_ARG
                            ("Q4_0 K/V cache" and "Q8 K / Q4 V", "perf(ds4): extend sparse
                            prefill scheduling to 10K", Production workflow and the
                            clean-head validation; the pages name the formats without
                            defining them) */
    int dependent_launch; /* 1 = launch each kernel as a programmatic dependent of the
                            kernel before it on the stream: its launch and prologue
                            (barrier set-up, tensor-memory allocation) overlap that
                            kernel's last wave, and it touches global memory only once
                            that kernel has completed, so results are the same bits.
                            0 = plain stream order. Other values are
                            DS4SP_ERR_INVALID_ARG */
    int attn_kernel;     /* step 3's kernel: 0 = streaming kernel on mma.sync (32-row units
                            through a 5-slot ring, default); 1 = logits on the tcgen05
                            tensor cores: units of 128 gathered rows as the MMA's M and the
                            16 heads as its N, S = R . Q^T accumulated in TMEM, softmax from
                            TMEM, P . V on mma.sync (an alternative to the streaming
                            form, as the pages time a grouped path against the streaming
                            one: "perf(ds4): unify gfx1151 sparse-prefill stack",
                            Validation completed). 1 needs kv_format 0, exp_mode 0 and
                            pv_mode 0 (else DS4SP_ERR_UNSUPPORTED) and does not take the
                            few-token split. Other values are DS4SP_ERR_INVALID_ARG */
    int indexer_kernel;  /* step 1's kernel in the two-kernel form (topk_mode 0, or a call
                            the fused kernel does not take): 0 = one CTA per tile, each
                            tcgen05 MMA 128 rows x 256 (token, head) columns; 1 = CTA pairs
                            (2-CTA clusters): each MMA 256 rows x 256 columns shared by the
                            pair (cta_group::2), CTA r holding the rows of its j-tile and
                            columns 128r .. 128r+127 of the q_idx block. The same scores
                            either way. Other values are DS4SP_ERR_INVALID_ARG */
} ds4sp_config;

/* Validate cfg and create a handle bound to the current CUDA device. The handle owns
 * two device words (the status word and the abort word of the kernels' bounded waits),
 * the partial-result buffer of few-token attention calls
 * (2 x SMs x 16 x 512 fp32 plus 2 x SMs x 32 fp32: about 9.7 MB on a 148-SM B200) and
 * some host state. *out is NULL on error. */
ds4sp_status ds4sp_create(const ds4sp_config* cfg, ds4sp_handle** out);

/* Wait for every launch this handle made (it records an event after each call), then
 * free the handle's own memory. Caller memory is never touched. NULL is accepted. */
ds4sp_status ds4sp_destroy(ds4sp_handle* h);

/* Bytes of scratch ds4sp_indexer_topk needs for query tokens [t0, t0+n_q): the fp32
 * score rows [n_q, ld] with ld = n_vis(t0+n_q-1) rounded up to 4 floats. Returns 0 for
 * an invalid handle or range. The scratch is caller-owned, 256-byte aligned, and may
 * be reused as soon as the call's kernels have run. */
size_t ds4sp_workspace_bytes(const ds4sp_handle* h, int t0, int n_q);

/* Steps 1-2 for tokens [t0, t0+n_q).
 *   q_idx [n_q, H_i, D_i] fp16, k_idx [max_tokens/4, D_i] fp16, w [n_q, H_i] fp32,
 *   topk  [n_q, top_k] int32 (output; may be NULL when top_k == 0),
 *   ws    scratch of ws_bytes >= ds4sp_workspace_bytes(h, t0, n_q).
 * Scores are fp32, accumulated from fp16 products on the tensor cores; integer-valued
 * inputs with |score| < 2^24 therefore give exact scores and exact indices. */
ds4sp_status ds4sp_indexer_topk(ds4sp_handle* h, const void* q_idx, const void* k_idx,
                                const float* w, int t0, int n_q, int32_t* topk,
                                void* ws, size_t ws_bytes, void* stream);

/* Step 3 for tokens [t0, t0+n_q).
 *   q [n_q, 16, 576] fp16, kv_raw [max_tokens, 576] fp16, kv_cmp [max_tokens/4, 576]
 *   fp16, topk [n_q, top_k] int32 as written by ds4sp_indexer_topk (entries
 *   0 .. min(k, n_vis(t))-1 hold visible rows), out [n_q, 16, 512] fp32 (output).
 * Rows are fp16; logits, softmax and accumulation are fp32; probabilities enter the
 * value product as fp16 (pv_mode 0) or as two fp16 terms (pv_mode 1). Calls of at most
 * 36 tokens whose tokens attend at most 64 x 32 rows each, and that fit the handle's
 * partial buffer, spread each token's rows over the GPU 32 at a time and merge the
 * partial softmax results per token in a second kernel (each unit's O and sum rescaled
 * to the largest reference max, added in unit order): a token's result then depends
 * only on the token, not on the other tokens of the call. Such calls use the handle's
 * partial buffer, so two of them must not run concurrently on one handle. */
ds4sp_status ds4sp_sparse_attn(ds4sp_handle* h, const void* q, const void* kv_raw,
                               const void* kv_cmp, const int32_t* topk, int t0, int n_q,
                               float* out, void* stream);

/* Steps 1-3 for band b, tokens [b*band, min((b+1)*band, n_tokens)). Bands must come in
 * order: b must equal the handle's next band (0 after create or ds4sp_reset), else
 * DS4SP_ERR_ORDER; on success the next band becomes b+1. All tensor arguments are
 * whole-sequence base pointers: q [n_tokens,16,576], q_idx [n_tokens,H_i,D_i],
 * w [n_tokens,H_i], topk [n_tokens,top_k], out [n_tokens,16,512]; KV as above.
 * n_tokens <= max_tokens. ws_bytes >= ds4sp_workspace_bytes(h, b*band, band-length). */
ds4sp_status ds4sp_prefill_band(ds4sp_handle* h, int b, int n_tokens, const void* q,
                                const void* q_idx, const float* w, const void* kv_raw,
                                const void* kv_cmp, const void* k_idx, int32_t* topk,
                                float* out, void* ws, size_t ws_bytes, void* stream);

/* Whole-sequence tensors of one prefill, by role (all row-major, layouts as for
 * ds4sp_prefill_band). As inputs of ds4sp_prefill_host they live in host memory (pinned
 * memory lets the copies run asynchronously; pageable memory works but serialises the
 * copies); as its device buffers they live on the handle's device. topk may be NULL
 * in the host set (indices are then not copied back); with top_k = 0 it is unused. */
typedef struct ds4sp_io {
    const void* q;        /* [n_tokens, 16, 576] fp16 */
    const void* q_idx;    /* [n_tokens, H_i, D_i] fp16 */
    const float* w;       /* [n_tokens, H_i] fp32 */
    const void* kv_raw;   /* [n_tokens, 576] fp16 */
    const void* kv_cmp;   /* [n_tokens/4, 576] fp16 */
    const void* k_idx;    /* [n_tokens/4, D_i] fp16 */
    int32_t* topk;        /* [n_tokens, top_k] int32 (output) */
    float* out;           /* [n_tokens, 16, 512] fp32 (output) */
} ds4sp_io;

/* A whole n_tokens prefill from host memory to host memory: every band in order, as
 * ds4sp_prefill_band does, with the transfers overlapped. Each band is taken in steps of
 * about 1,024 tokens, in token order. A step's rows of q, q_idx and w, and the KV,
 * compressed-KV and index-key rows it is the first step to need, are copied in on a
 * copy stream of the handle; the step computes (steps 1-3 for its tokens) on `stream`
 * once they have arrived; its rows of out (and topk) go back on a second copy stream of
 * the handle, so copies in, compute and copies out of neighbouring steps run at the
 * same time and only the last step's copy out trails. Every token's result is the same
 * bits as in ds4sp_prefill_band (a token's indices and output do not depend on the
 * other tokens of a call). The pages commit bands in order ("perf(ds4): extend sparse
 * prefill scheduling to 10K", Summary); this entry point is the host side of that loop.
 *   host  inputs and outputs in host memory; dev  device buffers of the same shapes
 *   (all of them required, including topk when top_k > 0), overwritten by the call;
 *   ws    device scratch of ws_bytes >= ds4sp_workspace_bytes(h, t0, band) for every
 *   band (the largest is the last band's).
 * Resets the handle's band order to 0 and leaves it at the band after the last. All
 * work is ordered after work already queued on `stream`, and the call returns without
 * waiting: host->out (and host->topk) hold the result once `stream` has completed. The
 * host buffers must stay valid and unchanged until then. Errors as for
 * ds4sp_prefill_band; a failed copy returns DS4SP_ERR_CUDA. */
ds4sp_status ds4sp_prefill_host(ds4sp_handle* h, int n_tokens, const ds4sp_io* host,
                                const ds4sp_io* dev, void* ws, size_t ws_bytes, void* stream);

/* Set the band the next ds4sp_prefill_band call must name (resume or restart). */
ds4sp_status ds4sp_reset(ds4sp_handle* h, int next_band);

/* The band the next ds4sp_prefill_band call must name, or -1 for a NULL handle. */
int ds4sp_next_band(const ds4sp_handle* h);

/* Synchronise `stream`, then read and clear the handle's device status word:
 * DS4SP_OK, or DS4SP_ERR_DEVICE_BOUNDS if a kernel skipped an out-of-range index or
 * gave up a bounded wait since the last read. *bits (may be NULL) receives the raw
 * word: bit 0 = index out of range, bit 1 = wait gave up. It also clears the word
 * through which the CTAs of a launch that gave up tell one another.
 *
 * CUDA graphs: ds4sp_indexer_topk, ds4sp_sparse_attn and ds4sp_prefill_band may be
 * captured into a graph (stream capture) once each has run outside the capture with
 * the same configuration (the first call sets kernel attributes). A replay launches
 * the captured kernels with their captured arguments; after a replay that gave up a
 * wait, call this function before the next replay. ds4sp_destroy does not wait for
 * replays: finish them (synchronise their stream) before destroying the handle. */
ds4sp_status ds4sp_device_status(ds4sp_handle* h, void* stream, uint32_t* bits);

/* Per-kernel timing. When enabled, the handle records CUDA events around each of its
 * kernels on the launch stream. ds4sp_profile_read synchronises those events and
 * returns, per kernel kind (0 = indexer, 1 = top-k, 2 = attention), the summed
 * milliseconds and launch counts since the last read; then it clears them. */
ds4sp_status ds4sp_profile_enable(ds4sp_handle* h, int enable);
ds4sp_status ds4sp_profile_read(ds4sp_handle* h, double ms[3], int launches[3]);

/* Host-side fault injection for tests: the next n kernel launches of this handle are
 * not made, and the call that would make them returns DS4SP_ERR_CUDA. */
ds4sp_status ds4sp_debug_fail_launches(ds4sp_handle* h, int n);

/* Bounded waits, for tests of the give-up path. Every pipeline wait inside the kernels
 * (one role waiting for another through a shared-memory barrier) gives up after a limit,
 * by default 1,000,000,000 ns (about one second); the kernel then records bit 1 of the
 * status word, every other wait of the same launch gives up at once, and the launch
 * returns with its outputs undefined. Waits for copies and tensor-core work a thread
 * issued itself, before the memory they write is released, keep the default limit
 * whatever is set here (they complete on their own). A give-up in one launch does not
 * shorten the waits of later launches.
 *   ns  the limit for this handle's later launches, in nanoseconds; 0 = give up at the
 *       first wait that is not already complete; negative = back to the default. */
ds4sp_status ds4sp_debug_set_wait_limit_ns(ds4sp_handle* h, long long ns);

/* Explicit-mask visibility, a debug form of the path for the "explicit-mask versus
 * analytic-mask" oracle check ("perf(ds4): extend sparse prefill scheduling to 10K",
 * Qualification). While a mask is set, the top-k and the attention take the visibility
 * of compressed rows from it instead of the ratio-4 formula:
 *   mask  device pointer, uint8 [rows, cols], row-major, caller-owned; mask[t*cols + j]
 *         != 0 means compressed row j is visible to absolute token t. It must stay valid
 *         until the calls that use it have completed.
 *   top-k      the candidates of token t are the j < min(cols, n_vis(t_last)) whose byte
 *              is set (t_last = the call's last token); fewer than k: all of them,
 *              ascending, then -1.
 *   attention  a top-k entry j is attended iff 0 <= j < min(cols, n_vis(t_last)) and
 *              its byte is set; -1 entries and hidden rows are dropped silently; other
 *              out-of-range entries set the status word's index bit.
 * The indexer, the window of raw rows and the work partition are unchanged; the score
 * columns j >= n_vis(t) are not computed, so a mask that shows such a row selects on an
 * undefined score (the check then fails, which is its purpose). With the mask that the
 * formula defines, every output is bit-identical to the analytic path.
 * mask = NULL clears it (rows and cols are then ignored). Calls whose tokens reach past
 * `rows` return DS4SP_ERR_INVALID_ARG before any launch. rows, cols >= 1 otherwise. */
ds4sp_status ds4sp_debug_set_mask(ds4sp_handle* h, const uint8_t* mask, int rows, int cols);

/* Steps 1-2 like ds4sp_indexer_topk, for callers that cannot allocate device memory.
 * The pages have no counterpart to this entry point; it exists for the host side only.
 * Some callers cannot call cudaMalloc: a framework whose allocator reserves all device
 * memory up front (a raw cudaMalloc then fails or splits its pool), or a latency-bound
 * loop where cudaMalloc/cudaFree would synchronise the device. This entry point needs
 * no handle and no workspace, and calls no cudaMalloc, cudaFree or allocating library
 * routine. Its score scratch is a fixed 8 MiB array inside the library (2^21 fp32
 * scores); every GPU that loads the library holds that array until the process exits.
 *   cfg     the same configuration ds4sp_create takes (validated the same way; this
 *           entry point always runs the two-kernel form, whatever cfg->topk_mode says);
 *   q_idx, k_idx, w, t0, n_q, topk, stream  as for ds4sp_indexer_topk.
 * n_q * ld must be <= 2^21, with ld = n_vis(t0+n_q-1) rounded up to 4 (for example, a
 * 2048-token band whose last token sees up to 1024 rows, or up to 5 tokens at a
 * 122,880-token context); larger ranges return DS4SP_ERR_WORKSPACE. Every argument error
 * is returned before any work is queued.
 * The first call on a device looks up the array's device address (cudaGetSymbolAddress)
 * with that device current; make that first call before any stream capture. All calls
 * share the one array, which keeps the last call's scores: calls whose kernels overlap on
 * the GPU (other streams, other threads) race on it, so serialise them. Device-side index
 * and wait checks of this path are recorded in a library-internal word that each call
 * clears; they are not reported to the caller. */
ds4sp_status ds4sp_indexer_topk_noalloc(const ds4sp_config* cfg, const void* q_idx,
                                        const void* k_idx, const float* w, int t0, int n_q,
                                        int32_t* topk, void* stream);

/* Quantized KV rows. The pages run their model on a quantized cache ("Q4_0 K/V cache",
 * "Q8 K / Q4 V"; "perf(ds4): extend sparse prefill scheduling to 10K", Production
 * workflow and the clean-head validation) without defining the formats; this library
 * reads them as blocks of 32 values with one fp16 scale d each:
 *   Q8_0 (kv_format 1)  codes q in [-127, 127], value d*q, d = max|x| / 127;
 *   Q4_0 (kv_format 2)  codes n in [0, 15], value d*(n-8), d = m / -8, m the block's
 *                       first value of largest magnitude.
 * Codes are decided in fp32 (x / d, IEEE division, rounded half to even, clamped). A row
 * is stored as its codes (Q8_0: one byte each; Q4_0: byte b of a block holds value b in
 * the low nibble and value b+16 in the high nibble), then its fp16 scales, then zeros up
 * to a multiple of 16 bytes. In formats 1 and 2 one latent row is key and value, so a
 * cache stores each 576-wide row once; format 3 ("Q8 K / Q4 V") stores the Q8_0 row of
 * the 576 values (the key) followed by the Q4_0 row of its first 512 (the value).
 *
 * ds4sp_kv_row_bytes: bytes of one stored row of `dims` values (a multiple of 32, at most
 * 4096; at least 512 for format 3) in kv_format 1, 2 or 3, or 0 for anything else.
 * ds4sp_quantize_kv: quantize x [rows, dims] fp16 (device) into out [rows,
 * ds4sp_kv_row_bytes(kv_format, dims)] bytes (device, caller-owned). Asynchronous on
 * `stream`; argument errors are returned before the launch. */
int ds4sp_kv_row_bytes(int kv_format, int dims);
ds4sp_status ds4sp_quantize_kv(const void* x, int rows, int dims, int kv_format, void* out,
                               void* stream);

/* Measurement helper, not a step of the path: the bandwidth ceiling of the attention
 * kernel's access pattern. Reads n rows of row_bytes (a multiple of 16, at most 1152)
 * from `table` [table_rows, row_bytes] at the row indices idx[0..n) (each in
 * [0, table_rows); the caller guarantees it, the kernel does not check), with 16-byte
 * loads into registers, and XORs every word into *sink (4 bytes, device memory) so that
 * no load is dead. Timing it with events around the call gives bytes/s for random row
 * gathers: with an L2-resident table (such as the KV of a 10K prefill, 14.75 MB) it is
 * the L2-to-SM gather ceiling that the attention kernel's rows are served under.
 * grid = CTAs of 512 threads (a multiple of the SM count is best). Asynchronous on
 * `stream`; argument errors are returned before the launch. */
ds4sp_status ds4sp_probe_gather(const void* table, int table_rows, int row_bytes,
                                const int32_t* idx, int n, uint32_t* sink, int grid, void* stream);

/* Static description of a status code. */
const char* ds4sp_status_string(ds4sp_status s);

/* Details of the most recent error on the calling host thread ("" if none). */
const char* ds4sp_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* DS4SP_H */
