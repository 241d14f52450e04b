"""CPU oracle for DS4 sparse-prefill attention (indexer -> top-k -> streaming MLA).

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. The CUDA library never
calls it, and it shares no code with the CUDA library: it imports NumPy only.

Everything is plain NumPy in float64 (int64 for the exact score variant), one
query token at a time, in the order the method states, with no blocking, fusion
or reordering. A reader can check each function against its definition:

* Visibility -- "perf(ds4): extend sparse prefill scheduling to 10K", Summary
  ("derive long ratio-4 causal visibility ... instead of retaining ... its
  quadratic score mask") and Qualification ("the ratio-4 boundary formula";
  "explicit-mask versus analytic-mask ... oracle"). Compressed row j summarises
  tokens 4j..4j+3 and is visible to token t once all four are in the past,
  i.e. 4j+3 <= t.
* Indexer score -- the pages name the indexer ("direct long-prefill top-k
  handoff", "packed small-CM rocWMMA indexer") but never define its score. This
  library fixes it as score(t, j) = sum_h w[t,h] * ReLU(q_idx[t,h,:] . k_idx[j,:]).
* Top-k -- "perf(ds4): extend sparse prefill scheduling to 10K", Summary ("pass
  authoritative long-prefill top-k rows directly", "preserve ... selected-row
  order"). Keep the min(k, n_vis(t)) largest scores among visible rows; equal
  scores go to the lower j; the kept rows are listed in ascending j, and unused
  slots hold -1.
* Explicit-mask top-k -- same page, Qualification ("explicit-mask versus
  analytic-mask" oracle): the same selection with the candidates read from a
  stored mask row instead of the formula (``topk_row_masked``).
* Attention -- same page, Summary ("keep selected raw/compressed KV transport in
  F16, and stream each selected latent row once across sixteen ... heads").
  One 576-wide latent row per position serves as key (all 576 dims) and value
  (first 512 dims) for all 16 query heads. The attended set is the selected
  compressed rows plus the raw rows of the sliding window max(0, t-n_swa+1)..t,
  under one softmax with scale ``scale`` (default 1/sqrt(576)).
* Bands -- same page, Summary ("independent 2K attention bands, and
  chronological state commit"): bands are scheduling units; running band after
  band gives the one-shot result.

* Quantized KV rows -- "perf(ds4): extend sparse prefill scheduling to 10K",
  Production workflow ("Q4_0 K/V cache") and its clean-head validation ("Q8 K / Q4
  V"). The pages name the formats without defining them; this library reads them as
  block formats of 32 values with one fp16 scale d each: Q8_0 stores q in [-127, 127]
  with value d*q, d = max|x|/127; Q4_0 stores n in [0, 15] with value d*(n-8), d =
  m/-8 where m is the block's first value of largest magnitude. Codes are decided in
  fp32 (x / d rounded half to even), the value is d*q exactly. One latent row serves as
  key and value, so a Q8_0 or Q4_0 cache stores each 576-wide row once
  (``quantize_rows``, ``dequantize_rows``, ``prefill_tokens_quant``). The "Q8 K / Q4 V"
  form keeps keys and values at different precisions: a stored row is the Q8_0 row of
  all 576 values (the key) followed by the Q4_0 row of its first 512 (the value), and
  attention takes logits from the first and values from the second
  (``attention_token_kv``).

Parity pins (tests/test_oracle_*.py) tie each function to something other than
itself: an explicit mask, exact int64 arithmetic, the ReLU identities
relu(x)-relu(-x)=x and relu(x)+relu(-x)=|x|, brute-force loops, dense masked
attention and torch's causal scaled_dot_product_attention.
"""
from __future__ import annotations

import math
from typing import Dict, Iterable, List, Optional, Sequence

import numpy as np

RATIO = 4


# --------------------------------------------------------------------------
# Visibility (ratio-4 causal visibility, no stored mask)
# --------------------------------------------------------------------------

def n_vis(t: int, ratio: int = RATIO) -> int:
    """Number of compressed rows visible to token t: rows j with ratio*j + ratio-1 <= t."""
    return (t + 1) // ratio


def is_visible(t: int, j: int, ratio: int = RATIO) -> bool:
    """Compressed row j (tokens ratio*j .. ratio*j+ratio-1) is visible to t iff its last token <= t."""
    return ratio * j + ratio - 1 <= t


def explicit_visibility_mask(T: int, n_c: int, ratio: int = RATIO) -> np.ndarray:
    """The quadratic mask the pages removed, built from the row-coverage definition.

    M[t, j] is True iff every token that compressed row j covers
    (ratio*j .. ratio*j+ratio-1) is <= t. Used only to check ``n_vis``.
    """
    m = np.zeros((T, n_c), dtype=bool)
    for t in range(T):
        for j in range(n_c):
            covered = range(ratio * j, ratio * j + ratio)
            m[t, j] = all(s <= t for s in covered)
    return m


def n_sel(t: int, k: int, ratio: int = RATIO) -> int:
    """Rows the top-k keeps for token t: all visible rows when fewer than k exist."""
    return min(k, n_vis(t, ratio))


def window(t: int, n_swa: int) -> np.ndarray:
    """Raw rows of token t's sliding window: max(0, t-n_swa+1) .. t inclusive."""
    return np.arange(max(0, t - n_swa + 1), t + 1, dtype=np.int64)


# --------------------------------------------------------------------------
# Indexer
# --------------------------------------------------------------------------

def indexer_scores_token(q_idx_t: np.ndarray, k_idx: np.ndarray, w_t: np.ndarray,
                         t: int, ratio: int = RATIO) -> np.ndarray:
    """Scores of token t against its visible compressed rows, float64.

    q_idx_t [H_i, D_i], k_idx [N_c, D_i], w_t [H_i] -> [n_vis(t)].
    dots[h, j] = q_idx_t[h] . k_idx[j]; score[j] = sum_h w_t[h] * max(dots[h, j], 0).
    """
    nv = n_vis(t, ratio)
    q = np.asarray(q_idx_t, dtype=np.float64)
    k = np.asarray(k_idx[:nv], dtype=np.float64)
    w = np.asarray(w_t, dtype=np.float64)
    dots = q @ k.T                       # [H_i, n_vis]
    return w @ np.maximum(dots, 0.0)     # [n_vis]


def indexer_scores_token_exact(q_idx_t: np.ndarray, k_idx: np.ndarray, w_t: np.ndarray,
                               t: int, ratio: int = RATIO) -> np.ndarray:
    """The same score in int64 arithmetic, for integer-valued inputs (exact by construction)."""
    nv = n_vis(t, ratio)
    q = np.asarray(q_idx_t, dtype=np.float64)
    k = np.asarray(k_idx[:nv], dtype=np.float64)
    w = np.asarray(w_t, dtype=np.float64)
    for a in (q, k, w):
        if not np.all(a == np.round(a)):
            raise ValueError("exact scores need integer-valued inputs")
    qi, ki, wi = q.astype(np.int64), k.astype(np.int64), w.astype(np.int64)
    dots = qi @ ki.T
    return wi @ np.maximum(dots, 0)


def indexer_scores(q_idx: np.ndarray, k_idx: np.ndarray, w: np.ndarray, t0: int,
                   ratio: int = RATIO, exact: bool = False) -> List[np.ndarray]:
    """Scores for query tokens t0 .. t0+n_q-1; entry i holds token t0+i's n_vis values."""
    f = indexer_scores_token_exact if exact else indexer_scores_token
    return [f(q_idx[i], k_idx, w[i], t0 + i, ratio) for i in range(q_idx.shape[0])]


# --------------------------------------------------------------------------
# Top-k selection
# --------------------------------------------------------------------------

def topk_row(scores: np.ndarray, k: int) -> np.ndarray:
    """Top-k of one token's score row: ascending j, ties to the lower j, -1 padded to k.

    Candidates are ordered by (score descending, j ascending); the first
    min(k, len(scores)) are kept and then listed by ascending j.
    """
    nv = len(scores)
    out = np.full(k, -1, dtype=np.int32)
    m = min(k, nv)
    if m == 0:
        return out
    j = np.arange(nv)
    order = np.lexsort((j, -np.asarray(scores, dtype=np.float64)))  # last key is primary
    kept = np.sort(order[:m])
    out[:m] = kept
    return out


def topk(scores: Sequence[np.ndarray], k: int) -> np.ndarray:
    """Stack ``topk_row`` over tokens: [n_q, k] int32."""
    return np.stack([topk_row(s, k) for s in scores]) if len(scores) else np.zeros((0, k), np.int32)


def topk_row_masked(scores: np.ndarray, visible: np.ndarray, k: int) -> np.ndarray:
    """Top-k of one token when visibility comes from a stored mask row, not the formula.

    The explicit-mask form of the selection ("perf(ds4): extend sparse prefill
    scheduling to 10K", Qualification: "explicit-mask versus analytic-mask"):
    the candidates are the j with visible[j] set; among them the same order as
    ``topk_row`` applies (score descending, then j ascending), the first
    min(k, #candidates) are kept and listed by ascending j, -1 padded to k.
    ``scores`` must cover every visible j (visible rows past its end raise).
    """
    visible = np.asarray(visible, dtype=bool)
    cand = np.flatnonzero(visible)
    if len(cand) and cand[-1] >= len(scores):
        raise ValueError("a visible row has no score")
    out = np.full(k, -1, dtype=np.int32)
    m = min(k, len(cand))
    if m == 0:
        return out
    s = np.asarray(scores, dtype=np.float64)[cand]
    order = np.lexsort((cand, -s))                      # last key is primary
    out[:m] = np.sort(cand[order[:m]])
    return out


# --------------------------------------------------------------------------
# Sparse MLA attention
# --------------------------------------------------------------------------

def default_scale(d_qk: int) -> float:
    return 1.0 / math.sqrt(d_qk)


def attended_rows(t: int, topk_t: np.ndarray, kv_raw: np.ndarray, kv_cmp: np.ndarray,
                  n_swa: int) -> np.ndarray:
    """Rows token t attends, in order: selected compressed rows (as listed), then window rows."""
    sel = topk_t[topk_t >= 0]
    return np.concatenate([np.asarray(kv_cmp[sel], dtype=np.float64),
                           np.asarray(kv_raw[window(t, n_swa)], dtype=np.float64)], axis=0)


def attention_token(q_t: np.ndarray, rows: np.ndarray, scale: float, d_v: int) -> np.ndarray:
    """Softmax attention of 16 heads over a shared set of latent rows, float64.

    q_t [H, d_qk], rows [R, d_qk] -> [H, d_v]. logits = scale * q_t @ rows^T;
    stable softmax over the rows; output = P @ rows[:, :d_v].
    """
    q = np.asarray(q_t, dtype=np.float64)
    logits = scale * (q @ rows.T)                      # [H, R]
    logits = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ rows[:, :d_v]


def sparse_mla_attention(q: np.ndarray, kv_raw: np.ndarray, kv_cmp: np.ndarray,
                         topk_idx: np.ndarray, t0: int, n_swa: int,
                         scale: Optional[float] = None, d_v: int = 512) -> np.ndarray:
    """Attention output for query tokens t0 .. t0+n_q-1: [n_q, H, d_v] float64."""
    n_q, H, d_qk = q.shape
    sc = default_scale(d_qk) if scale is None else scale
    out = np.zeros((n_q, H, d_v), dtype=np.float64)
    for i in range(n_q):
        rows = attended_rows(t0 + i, topk_idx[i], kv_raw, kv_cmp, n_swa)
        out[i] = attention_token(q[i], rows, sc, d_v)
    return out


# --------------------------------------------------------------------------
# Quantized KV rows (Q8_0, Q4_0)
# --------------------------------------------------------------------------

QBLOCK = 32
Q8_0, Q4_0, Q8K_Q4V = 1, 2, 3


def quantize_block_q8_0(x: np.ndarray):
    """One block of 32 values -> (codes int8 [32], scale as fp16).

    d = max|x| / 127 in fp32, stored as fp16; q = x / d in fp32, rounded half to even,
    clamped to [-127, 127]. An all-zero block has d = 0 and q = 0."""
    x = np.asarray(x, dtype=np.float32)
    amax = np.float32(np.max(np.abs(x)))
    d16 = np.float16(amax / np.float32(127.0))
    if d16 == 0:
        return np.zeros(QBLOCK, np.int8), np.float16(0.0)
    q = np.rint(x / np.float32(d16))
    return np.clip(q, -127, 127).astype(np.int8), d16


def quantize_block_q4_0(x: np.ndarray):
    """One block of 32 values -> (codes uint8 [32] in 0..15, scale as fp16).

    m = the first value of largest magnitude, d = m / -8 in fp32, stored as fp16;
    n = x / d in fp32 rounded half to even, plus 8, clamped to [0, 15]; value d*(n-8).
    An all-zero block has d = 0 and n = 8."""
    x = np.asarray(x, dtype=np.float32)
    i = int(np.argmax(np.abs(x)))            # first index of the largest magnitude
    d16 = np.float16(x[i] / np.float32(-8.0))
    if d16 == 0:
        return np.full(QBLOCK, 8, np.uint8), np.float16(0.0)
    n = np.rint(x / np.float32(d16)) + np.float32(8.0)
    return np.clip(n, 0, 15).astype(np.uint8), d16


def quantize_rows(x: np.ndarray, fmt: int):
    """Rows [R, D] (D a multiple of 32) -> (codes [R, D], scales fp16 [R, D/32])."""
    x = np.asarray(x, dtype=np.float32)
    R, Dm = x.shape
    f = quantize_block_q8_0 if fmt == Q8_0 else quantize_block_q4_0
    codes = np.zeros((R, Dm), np.int8 if fmt == Q8_0 else np.uint8)
    scales = np.zeros((R, Dm // QBLOCK), np.float16)
    for r in range(R):
        for b in range(Dm // QBLOCK):
            codes[r, b * QBLOCK:(b + 1) * QBLOCK], scales[r, b] = f(x[r, b * QBLOCK:(b + 1) * QBLOCK])
    return codes, scales


def dequantize_rows(codes: np.ndarray, scales: np.ndarray, fmt: int) -> np.ndarray:
    """Values of quantized rows in float64: d*q (Q8_0) or d*(n-8) (Q4_0)."""
    d = np.repeat(np.asarray(scales, np.float64), QBLOCK, axis=1)
    q = np.asarray(codes, np.float64)
    return d * (q if fmt == Q8_0 else q - 8.0)


def quant_row_bytes(fmt: int, dims: int) -> int:
    """Bytes of one stored row: codes, then the fp16 scales, padded to 16 bytes (for
    Q8K_Q4V: the Q8_0 row of the `dims` values, then the Q4_0 row of the first 512)."""
    if fmt == Q8K_Q4V:
        return quant_row_bytes(Q8_0, dims) + quant_row_bytes(Q4_0, 512)
    code_bytes = dims if fmt == Q8_0 else dims // 2
    raw = code_bytes + 2 * (dims // QBLOCK)
    return (raw + 15) // 16 * 16


def pack_rows(codes: np.ndarray, scales: np.ndarray, fmt: int) -> np.ndarray:
    """The stored row layout, uint8 [R, quant_row_bytes]: Q8_0 codes as bytes, or Q4_0
    codes two per byte (byte b of a block holds value b in its low nibble and value
    b+16 in its high nibble), then the scales as little-endian fp16, then zeros."""
    R, Dm = codes.shape
    out = np.zeros((R, quant_row_bytes(fmt, Dm)), np.uint8)
    if fmt == Q8_0:
        out[:, :Dm] = codes.astype(np.int8).view(np.uint8)
        cb = Dm
    else:
        blk = codes.reshape(R, Dm // QBLOCK, QBLOCK).astype(np.uint8)
        out[:, :Dm // 2] = (blk[:, :, :16] | (blk[:, :, 16:] << 4)).reshape(R, Dm // 2)
        cb = Dm // 2
    out[:, cb:cb + 2 * (Dm // QBLOCK)] = np.ascontiguousarray(
        scales.astype("<f2")).view(np.uint8).reshape(R, -1)
    return out


def unpack_rows(packed: np.ndarray, fmt: int, dims: int):
    """Inverse of pack_rows: (codes, scales)."""
    packed = np.asarray(packed, np.uint8)
    R = packed.shape[0]
    nb = dims // QBLOCK
    if fmt == Q8_0:
        codes = packed[:, :dims].view(np.int8).copy()
        cb = dims
    else:
        b = packed[:, :dims // 2].reshape(R, nb, 16)
        codes = np.concatenate([b & 15, b >> 4], axis=2).reshape(R, dims)
        cb = dims // 2
    scales = np.ascontiguousarray(packed[:, cb:cb + 2 * nb]).view("<f2").astype(np.float16)
    return codes, scales


def cache_rows(rows: np.ndarray, fmt: int, d_v: int = 512) -> np.ndarray:
    """The stored bytes of rows [R, dims] in cache format `fmt`: pack_rows of the
    quantized rows (Q8_0, Q4_0), or for Q8K_Q4V the Q8_0 row of all values followed by
    the Q4_0 row of the first d_v."""
    rows = np.asarray(rows)
    if fmt == Q8K_Q4V:
        return np.concatenate([pack_rows(*quantize_rows(rows, Q8_0), Q8_0),
                               pack_rows(*quantize_rows(rows[:, :d_v], Q4_0), Q4_0)], axis=1)
    return pack_rows(*quantize_rows(rows, fmt), fmt)


def kv_values(rows: np.ndarray, fmt: int, d_v: int = 512):
    """(key rows [R, 576], value rows [R, d_v]) in float64 as a cache of format `fmt`
    holds them: Q8_0 / Q4_0 dequantize one row that serves as both; Q8K_Q4V takes the key
    from the Q8_0 row and the value from the Q4_0 row of the first d_v values."""
    if fmt == Q8K_Q4V:
        k = dequantize_rows(*quantize_rows(rows, Q8_0), Q8_0)
        v = dequantize_rows(*quantize_rows(np.asarray(rows)[:, :d_v], Q4_0), Q4_0)
        return k, v
    deq = dequantize_rows(*quantize_rows(rows, fmt), fmt)
    return deq, deq[:, :d_v]


def attention_token_kv(q_t: np.ndarray, krows: np.ndarray, vrows: np.ndarray,
                       scale: float) -> np.ndarray:
    """Softmax attention of 16 heads over shared rows with separate keys and values,
    float64: logits = scale * q_t @ krows^T, stable softmax over the rows, P @ vrows."""
    q = np.asarray(q_t, dtype=np.float64)
    logits = scale * (q @ np.asarray(krows, np.float64).T)
    logits = logits - logits.max(axis=1, keepdims=True)
    p = np.exp(logits)
    p = p / p.sum(axis=1, keepdims=True)
    return p @ np.asarray(vrows, np.float64)


def prefill_tokens_quant(inputs: Dict[str, np.ndarray], tokens: Iterable[int], top_k: int,
                         n_swa: int, fmt: int, q_start: int = 0, scale: Optional[float] = None,
                         d_v: int = 512, ratio: int = RATIO) -> Dict[str, np.ndarray]:
    """The whole path with a quantized KV cache: kv_raw and kv_cmp are quantized row by
    row and attention reads the values the cache holds (kv_values); the indexer keys
    are unchanged. Per token: indexer scores -> top-k -> the attended key rows and value
    rows (selected compressed rows, then the window) -> attention_token_kv."""
    tokens = list(tokens)
    q, q_idx, w = inputs["q"], inputs["q_idx"], inputs["w"]
    k_raw, v_raw = kv_values(inputs["kv_raw"], fmt, d_v)
    k_cmp, v_cmp = kv_values(inputs["kv_cmp"], fmt, d_v)
    sc = default_scale(q.shape[2]) if scale is None else scale
    idx = np.zeros((len(tokens), top_k), dtype=np.int32)
    out = np.zeros((len(tokens), q.shape[1], d_v), dtype=np.float64)
    for n, t in enumerate(tokens):
        i = t - q_start
        s_t = indexer_scores_token(q_idx[i], inputs["k_idx"], w[i], t, ratio)
        idx[n] = topk_row(s_t, top_k)
        krows = attended_rows(t, idx[n], k_raw, k_cmp, n_swa)
        vrows = attended_rows(t, idx[n], v_raw, v_cmp, n_swa)
        out[n] = attention_token_kv(q[i], krows, vrows, sc)
    return {"tokens": np.asarray(tokens, dtype=np.int64), "topk": idx, "out": out}


# --------------------------------------------------------------------------
# Whole path over bands
# --------------------------------------------------------------------------

def prefill_tokens(inputs: Dict[str, np.ndarray], tokens: Iterable[int], top_k: int,
                   n_swa: int, q_start: int = 0, scale: Optional[float] = None,
                   d_v: int = 512, ratio: int = RATIO) -> Dict[str, np.ndarray]:
    """indexer -> top-k -> attention for the listed absolute token positions.

    Per-token arrays in ``inputs`` (q, q_idx, w) start at position ``q_start``.
    Each token's result depends only on that token's inputs and the resident
    KV, so any subset can be computed on its own (used for sampled parity).
    """
    tokens = list(tokens)
    q, q_idx, w = inputs["q"], inputs["q_idx"], inputs["w"]
    kv_raw, kv_cmp, k_idx = inputs["kv_raw"], inputs["kv_cmp"], inputs["k_idx"]
    d_qk = q.shape[2]
    sc = default_scale(d_qk) if scale is None else scale
    idx = np.zeros((len(tokens), top_k), dtype=np.int32)
    out = np.zeros((len(tokens), q.shape[1], d_v), dtype=np.float64)
    for n, t in enumerate(tokens):
        i = t - q_start
        s = indexer_scores_token(q_idx[i], k_idx, w[i], t, ratio)
        idx[n] = topk_row(s, top_k)
        rows = attended_rows(t, idx[n], kv_raw, kv_cmp, n_swa)
        out[n] = attention_token(q[i], rows, sc, d_v)
    return {"tokens": np.asarray(tokens, dtype=np.int64), "topk": idx, "out": out}


def prefill_bands(inputs: Dict[str, np.ndarray], T: int, top_k: int, n_swa: int,
                  band: int = 2048, scale: Optional[float] = None, d_v: int = 512,
                  ratio: int = RATIO) -> Dict[str, np.ndarray]:
    """Run the whole path band by band, in chronological order, over tokens 0 .. T-1.

    Band b covers tokens [b*band, min((b+1)*band, T)). Each band reads the
    resident KV only, so the concatenation equals the one-shot result.
    """
    parts = []
    for b0 in range(0, T, band):
        parts.append(prefill_tokens(inputs, range(b0, min(b0 + band, T)), top_k, n_swa,
                                    0, scale, d_v, ratio))
    return {"topk": np.concatenate([p["topk"] for p in parts]),
            "out": np.concatenate([p["out"] for p in parts])}
