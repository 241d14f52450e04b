"""Plant a plausible mistake in a private copy of the oracle (CPU only) and check
that the pins catch it. This shows the pins constrain every step of the oracle."""
import importlib.util
import os

import numpy as np
import pytest

import oracle_pins as P

ORACLE_SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                          "oracle", "ds4sp_oracle.py")


def fresh_oracle():
    spec = importlib.util.spec_from_file_location("oracle_mutant", ORACLE_SRC)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _mut_visibility_first_token(o):
    o.n_vis = lambda t, ratio=4: (t + ratio) // ratio          # row visible at its first token


def _mut_no_relu(o):
    def f(q, k, w, t, ratio=4):
        nv = o.n_vis(t, ratio)
        return np.asarray(w, float) @ (np.asarray(q, float) @ np.asarray(k[:nv], float).T)
    o.indexer_scores_token = f


def _mut_relu_after_head_sum(o):
    def f(q, k, w, t, ratio=4):
        nv = o.n_vis(t, ratio)
        return np.maximum(np.asarray(w, float) @ (np.asarray(q, float) @ np.asarray(k[:nv], float).T), 0)
    o.indexer_scores_token = f


def _mut_unweighted_heads(o):
    def f(q, k, w, t, ratio=4):
        nv = o.n_vis(t, ratio)
        return np.maximum(np.asarray(q, float) @ np.asarray(k[:nv], float).T, 0).sum(axis=0)
    o.indexer_scores_token = f


def _mut_ties_to_higher_j(o):
    def f(scores, k):
        nv = len(scores)
        out = np.full(k, -1, dtype=np.int32)
        m = min(k, nv)
        if m:
            order = np.lexsort((-np.arange(nv), -np.asarray(scores, float)))
            out[:m] = np.sort(order[:m])
        return out
    o.topk_row = f


def _mut_score_order_listing(o):
    def f(scores, k):
        nv = len(scores)
        out = np.full(k, -1, dtype=np.int32)
        m = min(k, nv)
        if m:
            out[:m] = np.lexsort((np.arange(nv), -np.asarray(scores, float)))[:m]
        return out
    o.topk_row = f


def _mut_value_last_dims(o):
    def f(q_t, rows, scale, d_v):
        logits = scale * (np.asarray(q_t, float) @ rows.T)
        p = np.exp(logits - logits.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        return p @ rows[:, -d_v:]
    o.attention_token = f


def _mut_window_excludes_self(o):
    o.window = lambda t, n_swa: np.arange(max(0, t - n_swa), t, dtype=np.int64)


def _mut_scale_ignored(o):
    orig = o.attention_token
    o.attention_token = lambda q_t, rows, scale, d_v: orig(q_t, rows, 1.0, d_v)


def _mut_dedup_window(o):
    # Drops raw rows whose index coincides with a selected compressed row index.
    orig = o.attended_rows
    def f(t, topk_t, kv_raw, kv_cmp, n_swa):
        sel = topk_t[topk_t >= 0]
        win = [s for s in o.window(t, n_swa) if s not in set(sel.tolist())]
        return np.concatenate([np.asarray(kv_cmp[sel], float), np.asarray(kv_raw[win], float)])
    o.attended_rows = f


def _mut_masked_ignores_mask(o):
    o.topk_row_masked = lambda scores, visible, k: o.topk_row(scores, k)


def _mut_masked_ties_by_candidate_rank(o):
    # Breaks ties by the position in the candidate list reversed (a higher j first).
    def f(scores, visible, k):
        cand = np.flatnonzero(np.asarray(visible, bool))
        out = np.full(k, -1, dtype=np.int32)
        m = min(k, len(cand))
        if m:
            order = np.lexsort((-cand, -np.asarray(scores, float)[cand]))
            out[:m] = np.sort(cand[order[:m]])
        return out
    o.topk_row_masked = f


def _prefill_with(o, attend_pos, q_row):
    """prefill_tokens rebuilt with a planted offset mistake: `attend_pos(t, i)` is the
    position handed to attended_rows, `q_row(t, i)` the per-token row read."""
    def f(inputs, tokens, top_k, n_swa, q_start=0, scale=None, d_v=512, ratio=4):
        tokens = list(tokens)
        q, q_idx, w = inputs["q"], inputs["q_idx"], inputs["w"]
        sc = o.default_scale(q.shape[2]) if scale is None else scale
        idx = np.zeros((len(tokens), top_k), dtype=np.int32)
        out = np.zeros((len(tokens), q.shape[1], d_v))
        for n, t in enumerate(tokens):
            i = t - q_start
            r = q_row(t, i)
            idx[n] = o.topk_row(o.indexer_scores_token(q_idx[r], inputs["k_idx"], w[r], t, ratio), top_k)
            rows = o.attended_rows(attend_pos(t, i), idx[n], inputs["kv_raw"], inputs["kv_cmp"], n_swa)
            out[n] = o.attention_token(q[r], rows, sc, d_v)
        return {"tokens": np.asarray(tokens, dtype=np.int64), "topk": idx, "out": out}
    return f


def _mut_prefill_window_at_row(o):
    # The attended rows taken at the token's row i = t - q_start instead of its position t.
    o.prefill_tokens = _prefill_with(o, lambda t, i: i, lambda t, i: i)


def _mut_prefill_inputs_at_position(o):
    # Per-token inputs read at the position t instead of the row t - q_start.
    o.prefill_tokens = _prefill_with(o, lambda t, i: t, lambda t, i: t)


def _mut_q8_round_half_away(o):
    orig = o.quantize_block_q8_0
    def f(x):
        x = np.asarray(x, np.float32)
        _, d16 = orig(x)
        if d16 == 0:
            return np.zeros(32, np.int8), d16
        q = np.sign(x) * np.floor(np.abs(x / np.float32(d16)) + 0.5)
        return np.clip(q, -127, 127).astype(np.int8), d16
    o.quantize_block_q8_0 = f


def _mut_q4_scale_sign(o):
    def f(x):
        x = np.asarray(x, np.float32)
        i = int(np.argmax(np.abs(x)))
        d16 = np.float16(x[i] / np.float32(8.0))
        if d16 == 0:
            return np.full(32, 8, np.uint8), d16
        return np.clip(np.rint(x / np.float32(d16)) + 8, 0, 15).astype(np.uint8), d16
    o.quantize_block_q4_0 = f


def _mut_q4_last_extreme(o):
    def f(x):
        x = np.asarray(x, np.float32)
        a = np.abs(x)
        i = int(len(a) - 1 - np.argmax(a[::-1]))          # the last largest magnitude
        d16 = np.float16(x[i] / np.float32(-8.0))
        if d16 == 0:
            return np.full(32, 8, np.uint8), d16
        return np.clip(np.rint(x / np.float32(d16)) + 8, 0, 15).astype(np.uint8), d16
    o.quantize_block_q4_0 = f


def _mut_q4_adjacent_nibbles(o):
    orig_pack, orig_unpack = o.pack_rows, o.unpack_rows
    def pack(codes, scales, fmt):
        out = orig_pack(codes, scales, fmt)
        if fmt == o.Q4_0:
            R, Dm = codes.shape
            c = codes.astype(np.uint8).reshape(R, Dm // 2, 2)
            out[:, :Dm // 2] = c[:, :, 0] | (c[:, :, 1] << 4)
        return out
    def unpack(packed, fmt, dims):
        codes, scales = orig_unpack(packed, fmt, dims)
        if fmt == o.Q4_0:
            b = np.asarray(packed, np.uint8)[:, :dims // 2]
            codes = np.stack([b & 15, b >> 4], axis=2).reshape(b.shape[0], dims)
        return codes, scales
    o.pack_rows, o.unpack_rows = pack, unpack


def _mut_q4_no_offset(o):
    def f(codes, scales, fmt):
        d = np.repeat(np.asarray(scales, np.float64), 32, axis=1)
        return d * np.asarray(codes, np.float64)
    o.dequantize_rows = f


def _mut_split_values_from_keys(o):
    # The Q8 K / Q4 V cache read with the values taken from the Q8_0 key rows.
    orig = o.kv_values
    def f(rows, fmt, d_v=512):
        k, v = orig(rows, fmt, d_v)
        return (k, k[:, :d_v]) if fmt == o.Q8K_Q4V else (k, v)
    o.kv_values = f


def _mut_kv_attention_values_from_keys(o):
    o.attention_token_kv = lambda q_t, krows, vrows, scale: o.attention_token(q_t, krows, scale, 512)


MUTATIONS = [
    (_mut_visibility_first_token, [P.pin_visibility_mask, P.pin_visibility_golden]),
    (_mut_no_relu, [P.pin_scores_exact, P.pin_scores_relu_identities, P.pin_scores_bruteforce]),
    (_mut_relu_after_head_sum, [P.pin_scores_relu_identities, P.pin_scores_bruteforce]),
    (_mut_unweighted_heads, [P.pin_scores_relu_identities, P.pin_scores_bruteforce]),
    (_mut_ties_to_higher_j, [P.pin_topk_golden, P.pin_topk_bruteforce]),
    (_mut_score_order_listing, [P.pin_topk_golden, P.pin_topk_bruteforce]),
    (_mut_masked_ignores_mask, [P.pin_topk_masked_bruteforce]),
    (_mut_masked_ties_by_candidate_rank, [P.pin_topk_masked_bruteforce]),
    (_mut_value_last_dims, [P.pin_attention_sdpa_causal, P.pin_attention_closed_forms]),
    (_mut_window_excludes_self, [P.pin_attention_sdpa_causal, P.pin_attention_sdpa_window]),
    (_mut_scale_ignored, [P.pin_attention_sdpa_causal, P.pin_attention_bruteforce]),
    (_mut_dedup_window, [P.pin_attention_dense_mask, P.pin_attention_closed_forms]),
    (_mut_prefill_window_at_row, [P.pin_prefill_tokens_composition]),
    (_mut_prefill_inputs_at_position, [P.pin_prefill_tokens_composition]),
    (_mut_q8_round_half_away, [P.pin_quant_golden]),
    (_mut_q4_scale_sign, [P.pin_quant_golden, P.pin_quant_properties]),
    (_mut_q4_last_extreme, [P.pin_quant_golden]),
    (_mut_q4_adjacent_nibbles, [P.pin_quant_golden, P.pin_quant_dequant_bruteforce]),
    (_mut_q4_no_offset, [P.pin_quant_dequant_bruteforce, P.pin_quant_properties,
                         P.pin_quant_path_reduces_to_fp16]),
    (_mut_split_values_from_keys, [P.pin_quant_kv_split_composition]),
    (_mut_kv_attention_values_from_keys, [P.pin_attention_kv_sdpa]),
]


def test_offset_harness_without_mistake_passes():
    """The rebuilt prefill_tokens used by the offset mutations passes the pin when given
    the right offsets, so those mutations fail for their planted mistake alone."""
    o = fresh_oracle()
    o.prefill_tokens = _prefill_with(o, lambda t, i: t, lambda t, i: i)
    P.pin_prefill_tokens_composition(o)


@pytest.mark.parametrize("mutate,pins", MUTATIONS, ids=[m[0].__name__ for m in MUTATIONS])
def test_planted_mistake_is_caught(mutate, pins):
    o = fresh_oracle()
    for p in pins:            # the unmutated copy passes these pins
        p(o)
    mutate(o)
    caught = []
    for p in pins:
        try:
            with np.errstate(all="ignore"):
                p(o)
        except (AssertionError, ValueError, IndexError):
            caught.append(p.__name__)
    assert caught, f"{mutate.__name__} slipped past {[p.__name__ for p in pins]}"
