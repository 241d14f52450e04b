"""Pins that tie the CPU oracle to something other than itself.

Each ``pin_*`` takes the oracle module as ``o`` and raises AssertionError when
the oracle disagrees with an independent fact: a hand-worked fixture, an
explicit mask built from the row-coverage definition, exact integer
arithmetic, a ReLU identity, brute-force scalar loops, dense masked attention
or torch's causal scaled_dot_product_attention. ``test_oracle_pins.py`` runs
them on the real oracle; ``test_oracle_mutations.py`` runs them on copies with a
planted mistake and expects at least one to fail.
"""
from __future__ import annotations

import math
import os

import numpy as np
import torch

from sparse_mla_prefill_b200.inputs import generate_small

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _np(inputs):
    return {k: v.numpy() for k, v in inputs.items()}


# ----------------------------------------------------------------- visibility

def pin_visibility_mask(o, n_c: int = 12):
    """n_vis(t) equals the row count of a mask built from row coverage, and the rows form a prefix."""
    T = 4 * n_c + 8
    mask = np.zeros((T, n_c), dtype=bool)
    for t in range(T):
        for j in range(n_c):
            mask[t, j] = max(4 * j, 4 * j + 1, 4 * j + 2, 4 * j + 3) <= t
    assert np.array_equal(o.explicit_visibility_mask(T, n_c), mask)
    for t in range(T):
        nv = min(o.n_vis(t), n_c)
        assert nv == int(mask[t].sum()), (t, nv, int(mask[t].sum()))
        assert mask[t, :nv].all() and not mask[t, nv:].any()
        for j in range(n_c):
            assert o.is_visible(t, j) == bool(mask[t, j])


def pin_visibility_golden(o):
    with open(os.path.join(GOLDEN, "visibility_ratio4.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            t, nv, rows = line.split()
            t, nv = int(t), int(nv)
            assert o.n_vis(t) == nv, (t, o.n_vis(t), nv)
            want = [] if rows == "-" else [int(x) for x in rows.split(",")]
            got = [j for j in range(nv + 3) if o.is_visible(t, j)]
            assert got == want, (t, got, want)


# -------------------------------------------------------------------- indexer

def _indexer_case(T=96, H_i=4, D_i=64, seed=11):
    return _np(generate_small(T, H_i, D_i, seed))


def pin_scores_exact(o, inp=None, tokens=None):
    """float64 scores equal exact int64 scores (integer-valued inputs)."""
    inp = inp or _indexer_case()
    tokens = range(inp["q_idx"].shape[0]) if tokens is None else tokens
    for t in tokens:
        f = o.indexer_scores_token(inp["q_idx"][t], inp["k_idx"], inp["w"][t], t)
        e = o.indexer_scores_token_exact(inp["q_idx"][t], inp["k_idx"], inp["w"][t], t)
        assert f.shape == e.shape == (o.n_vis(t),)
        assert np.array_equal(f, e.astype(np.float64)), t


def pin_scores_relu_identities(o, inp=None, tokens=None):
    """relu(x)-relu(-x) = x and relu(x)+relu(-x) = |x| give two closed forms.

    s(q) - s(-q) = sum_h w_h (q_h . k_j)   and   s(q) + s(-q) = sum_h w_h |q_h . k_j|,
    each a single matrix product with no ReLU; together they fix s(q).
    """
    inp = inp or _indexer_case()
    tokens = range(inp["q_idx"].shape[0]) if tokens is None else tokens
    k = inp["k_idx"].astype(np.float64)
    for t in tokens:
        q = inp["q_idx"][t].astype(np.float64)
        w = inp["w"][t].astype(np.float64)
        nv = o.n_vis(t)
        sp = o.indexer_scores_token(q, k, w, t)
        sm = o.indexer_scores_token(-q, k, w, t)
        x = q @ k[:nv].T
        assert np.array_equal(sp - sm, w @ x), t
        assert np.array_equal(sp + sm, w @ np.abs(x)), t


def pin_scores_bruteforce(o):
    """Pure-Python loops over (h, d) on a tiny case."""
    inp = _indexer_case(T=24, H_i=3, D_i=5, seed=5)
    q, k, w = inp["q_idx"], inp["k_idx"], inp["w"]
    for t in range(24):
        got = o.indexer_scores_token(q[t], k, w[t], t)
        want = []
        for j in range(k.shape[0]):
            if 4 * j + 3 > t:
                continue
            s = 0.0
            for h in range(q.shape[1]):
                dot = 0.0
                for d in range(q.shape[2]):
                    dot += float(q[t, h, d]) * float(k[j, d])
                s += float(w[t, h]) * (dot if dot > 0 else 0.0)
            want.append(s)
        assert got.tolist() == want, (t, got.tolist(), want)


# ---------------------------------------------------------------------- top-k

def pin_topk_golden(o):
    with open(os.path.join(GOLDEN, "topk_ties.txt")) as f:
        lines = [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]
    scores = np.array([float(x) for x in lines[0].split(":")[1].split()])
    for ln in lines[1:]:
        k, row = ln.split("|")
        want = [int(x) for x in row.split()]
        got = o.topk_row(scores, int(k)).tolist()
        assert got == want, (k, got, want)


def _topk_brute(scores, k):
    cands = sorted(range(len(scores)), key=lambda j: (-scores[j], j))[:min(k, len(scores))]
    cands.sort()
    return cands + [-1] * (k - len(cands))


def pin_topk_bruteforce(o, trials: int = 300, seed: int = 3):
    """Brute force by sorted() plus the defining properties, on rows rich in ties."""
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        n = int(rng.integers(0, 70))
        k = int(rng.integers(0, 40))
        scores = rng.integers(-3, 6, n).astype(np.float64) * float(rng.choice([1.0, 0.5, 1e3]))
        got = o.topk_row(scores, k)
        assert got.dtype == np.int32 and got.shape == (k,)
        assert got.tolist() == _topk_brute(scores.tolist(), k), (scores.tolist(), k)
        m = min(k, n)
        sel = got[:m]
        assert (got[m:] == -1).all() and (np.diff(sel) > 0).all()
        rest = np.setdiff1d(np.arange(n), sel)
        if m and len(rest):
            assert scores[sel].min() >= scores[rest].max()
            thr = scores[sel].min()
            if (scores[rest] == thr).any():
                assert sel[scores[sel] == thr].max() < rest[scores[rest] == thr].min()


def pin_topk_masked_bruteforce(o, trials: int = 300, seed: int = 4):
    """Explicit-mask selection: brute force over the mask's candidates, hidden rows never
    kept, and the formula's own mask row gives the prefix selection."""
    rng = np.random.default_rng(seed)
    for _ in range(trials):
        n = int(rng.integers(0, 70))
        k = int(rng.integers(0, 40))
        scores = rng.integers(-3, 6, n).astype(np.float64) * float(rng.choice([1.0, 0.5, 1e3]))
        vis = rng.random(n + int(rng.integers(0, 4))) < rng.choice([0.2, 0.6, 1.0])
        vis[n:] = False                            # rows past the scores are never visible
        got = o.topk_row_masked(scores, vis, k)
        cand = [j for j in range(n) if vis[j]]
        want = sorted(sorted(cand, key=lambda j: (-scores[j], j))[:min(k, len(cand))])
        assert got.dtype == np.int32 and got.shape == (k,)
        assert got.tolist() == want + [-1] * (k - len(want)), (scores.tolist(), vis.tolist(), k)
        assert all(vis[j] for j in got if j >= 0)
    # The ratio-4 mask row of token t (rows 4j+3 <= t) reduces to the prefix selection.
    scores = rng.integers(0, 4, 40).astype(np.float64)
    for t in (0, 3, 17, 90, 170):
        row = np.array([4 * j + 3 <= t for j in range(40)])
        nv = int(row.sum())
        got = o.topk_row_masked(scores, row, 8).tolist()
        want = sorted(sorted(range(nv), key=lambda j: (-scores[j], j))[:min(8, nv)])
        assert got == want + [-1] * (8 - len(want)), (t, got)


# ------------------------------------------------------------------ attention

def _attn_case(T=48, n_c=None, seed=21):
    g = torch.Generator("cpu").manual_seed(seed)
    n_c = T // 4 if n_c is None else n_c
    q = torch.randn(T, 16, 576, generator=g).half().double().numpy()
    kv_raw = torch.randn(T, 576, generator=g).half().double().numpy()
    kv_cmp = torch.randn(n_c, 576, generator=g).half().double().numpy()
    return q, kv_raw, kv_cmp


def pin_attention_sdpa_causal(o, T: int = 48):
    """k = 0 and n_swa >= T reduce to causal attention with one shared KV head."""
    q, kv_raw, kv_cmp = _attn_case(T)
    scale = 1.0 / 24.0
    got = o.sparse_mla_attention(q, kv_raw, kv_cmp, np.zeros((T, 0), np.int32), 0, T, scale)
    Q = torch.from_numpy(q).permute(1, 0, 2)[None]                 # [1,16,T,576]
    K = torch.from_numpy(kv_raw)[None, None].expand(1, 16, T, 576)
    V = torch.from_numpy(kv_raw[:, :512])[None, None].expand(1, 16, T, 512)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True, scale=scale)
    ref = ref[0].permute(1, 0, 2).numpy()
    assert got.shape == ref.shape
    assert np.abs(got - ref).max() < 1e-12, np.abs(got - ref).max()


def pin_attention_sdpa_window(o, T: int = 48, n_swa: int = 7):
    """k = 0 reduces to sliding-window attention over raw rows (banded boolean mask)."""
    q, kv_raw, kv_cmp = _attn_case(T, seed=22)
    scale = 0.05
    got = o.sparse_mla_attention(q, kv_raw, kv_cmp, np.zeros((T, 0), np.int32), 0, n_swa, scale)
    t = torch.arange(T)
    allowed = (t[None, :] <= t[:, None]) & (t[None, :] > t[:, None] - n_swa)
    Q = torch.from_numpy(q).permute(1, 0, 2)[None]
    K = torch.from_numpy(kv_raw)[None, None].expand(1, 16, T, 576)
    V = torch.from_numpy(kv_raw[:, :512])[None, None].expand(1, 16, T, 512)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=allowed, scale=scale)
    ref = ref[0].permute(1, 0, 2).numpy()
    assert np.abs(got - ref).max() < 1e-12, np.abs(got - ref).max()


def pin_attention_dense_mask(o, T: int = 64, n_swa: int = 9):
    """With k >= n_vis(t) for every t the output is dense masked attention over
    [all compressed rows ; all raw rows], whatever the indexer scores are."""
    q, kv_raw, kv_cmp = _attn_case(T, seed=23)
    n_c = kv_cmp.shape[0]
    k = n_c
    scale = 1.0 / 24.0
    # Any scores: selection keeps every visible row because k >= n_vis.
    rng = np.random.default_rng(0)
    idx = np.stack([o.topk_row(rng.standard_normal(o.n_vis(t)), k) for t in range(T)])
    got = o.sparse_mla_attention(q, kv_raw, kv_cmp, idx, 0, n_swa, scale)
    keys = np.concatenate([kv_cmp, kv_raw])                      # [n_c + T, 576]
    for t in range(T):
        cmp_ok = np.array([4 * j + 3 <= t for j in range(n_c)])
        raw_ok = np.array([t - n_swa < s <= t for s in range(T)])
        ok = np.concatenate([cmp_ok, raw_ok])
        logits = scale * (q[t] @ keys.T)
        logits[:, ~ok] = -np.inf
        p = np.exp(logits - logits.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        ref = p @ keys[:, :512]
        assert np.abs(got[t] - ref).max() < 1e-12, t


def pin_attention_bruteforce(o, tokens=(0, 3, 9, 30, 47)):
    """Scalar loops with math.exp for a few tokens of a small case (k=5, n_swa=6)."""
    T, k, n_swa = 48, 5, 6
    q, kv_raw, kv_cmp = _attn_case(T, seed=24)
    rng = np.random.default_rng(1)
    idx = np.stack([o.topk_row(rng.integers(0, 4, o.n_vis(t)).astype(float), k) for t in range(T)])
    scale = 1.0 / 24.0
    got = o.sparse_mla_attention(q, kv_raw, kv_cmp, idx, 0, n_swa, scale)
    for t in tokens:
        rows = [kv_cmp[j] for j in idx[t] if j >= 0]
        rows += [kv_raw[s] for s in range(max(0, t - n_swa + 1), t + 1)]
        for h in range(16):
            logits = [scale * sum(float(a) * float(b) for a, b in zip(q[t, h], r)) for r in rows]
            mx = max(logits)
            e = [math.exp(x - mx) for x in logits]
            z = sum(e)
            for d in range(0, 512, 37):
                want = sum(ei * float(r[d]) for ei, r in zip(e, rows)) / z
                assert abs(got[t, h, d] - want) < 1e-12, (t, h, d)


def pin_attention_closed_forms(o):
    """scale = 0 gives the plain mean of the attended rows' values; token 0 alone
    attends only raw row 0, so its output is that row's first 512 values."""
    T, k, n_swa = 40, 4, 5
    q, kv_raw, kv_cmp = _attn_case(T, seed=25)
    rng = np.random.default_rng(2)
    idx = np.stack([o.topk_row(rng.standard_normal(o.n_vis(t)), k) for t in range(T)])
    got0 = o.sparse_mla_attention(q, kv_raw, kv_cmp, idx, 0, n_swa, 0.0)
    for t in range(T):
        nsel = min(k, (t + 1) // 4)
        members = [kv_cmp[j] for j in idx[t][:nsel]] + [kv_raw[s] for s in range(max(0, t - n_swa + 1), t + 1)]
        want = np.mean(np.stack(members)[:, :512], axis=0)
        assert np.abs(got0[t] - want[None, :]).max() < 1e-12, t
    got = o.sparse_mla_attention(q, kv_raw, kv_cmp, idx, 0, n_swa, 1.0 / 24.0)
    assert np.abs(got[0] - kv_raw[0, :512][None, :]).max() < 1e-12


# ---------------------------------------------------------------------- bands

def pin_bands_equal_oneshot(o):
    """Band-by-band equals one pass over all tokens, exactly."""
    inp = _np(generate_small(160, 4, 64, seed=31))
    one = o.prefill_tokens(inp, range(160), top_k=8, n_swa=12)
    bands = o.prefill_bands(inp, 160, top_k=8, n_swa=12, band=64)
    assert np.array_equal(one["topk"], bands["topk"])
    assert np.array_equal(one["out"], bands["out"])


def pin_prefill_tokens_composition(o, T: int = 120, s: int = 37):
    """The whole path for a shuffled subset of tokens whose per-token inputs start at
    q_start = s > 0 equals the pinned steps called one by one on the full arrays:
    topk_row(indexer_scores_token(q_idx[t], k_idx, w[t], t)), then sparse_mla_attention
    of token t alone (t0 = t). This fixes the offset between a token's position t and
    its row t - s in the per-token arrays, and the order in which the steps compose."""
    full = _np(generate_small(T, 4, 64, seed=41))
    sliced = dict(full)
    for name in ("q", "q_idx", "w"):
        sliced[name] = full[name][s:]
    rng = np.random.default_rng(6)
    toks = [int(t) for t in rng.permutation(np.arange(s, T))[:40]]
    k, n_swa = 6, 9
    got = o.prefill_tokens(sliced, toks, top_k=k, n_swa=n_swa, q_start=s)
    assert got["tokens"].tolist() == toks
    assert got["topk"].shape == (len(toks), k) and got["out"].shape == (len(toks), 16, 512)
    for n, t in enumerate(toks):
        sc = o.indexer_scores_token(full["q_idx"][t], full["k_idx"], full["w"][t], t)
        idx = o.topk_row(sc, k)
        assert np.array_equal(got["topk"][n], idx), t
        want = o.sparse_mla_attention(full["q"][t:t + 1], full["kv_raw"], full["kv_cmp"],
                                      idx[None], t, n_swa)
        assert np.array_equal(got["out"][n], want[0]), t


# ------------------------------------------------------------ quantized KV rows

def pin_quant_golden(o):
    """Hand-derived blocks: half-to-even rounding, clamping, the first-largest-magnitude
    rule of Q4_0, the scale rounded to fp16, and the Q4_0 nibble order."""
    with open(os.path.join(GOLDEN, "quant_blocks.txt")) as f:
        lines = [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]
    for ln in lines:
        kind, xs, cs, sc = [part.strip() for part in ln.split("|")]
        x = np.zeros(32, np.float32)
        vals = [float(v) for v in xs.split()]
        x[:len(vals)] = vals
        fmt = o.Q8_0 if kind == "q8" else o.Q4_0
        f = o.quantize_block_q8_0 if fmt == o.Q8_0 else o.quantize_block_q4_0
        codes, d16 = f(x)
        assert float(d16) == float(sc), (ln, float(d16))
        if kind == "q4bytes":
            packed = o.pack_rows(codes[None].astype(np.uint8), np.array([[d16]], np.float16), fmt)
            want = [int(v, 16) for v in cs.split()]
            assert packed[0, :16].tolist() == want, (packed[0, :16].tolist(), want)
            continue
        want = [int(v) for v in cs.split()]
        zero_code = 0 if fmt == o.Q8_0 else 8
        want = want + [zero_code] * (32 - len(want))
        assert codes.astype(int).tolist() == want, (ln, codes.tolist())


def _dequant_loops(packed, fmt, dims):
    """Pure-Python reading of the stored row layout, element by element."""
    import struct
    nb = dims // 32
    code_bytes = dims if fmt == 1 else dims // 2
    out = []
    for row in packed.tolist():
        raw = bytes(row)
        vals = []
        for b in range(nb):
            d = struct.unpack("<e", raw[code_bytes + 2 * b: code_bytes + 2 * b + 2])[0]
            for i in range(32):
                if fmt == 1:
                    q = struct.unpack("b", raw[32 * b + i: 32 * b + i + 1])[0]
                    vals.append(d * q)
                else:
                    byte = raw[16 * b + (i % 16)]
                    n = (byte & 15) if i < 16 else (byte >> 4)
                    vals.append(d * (n - 8))
        out.append(vals)
    return np.array(out, dtype=np.float64)


def pin_quant_dequant_bruteforce(o, seed: int = 12):
    """dequantize_rows(unpack_rows(bytes)) equals a byte-by-byte loop over the layout,
    on random codes and scales, for both formats and both row widths."""
    rng = np.random.default_rng(seed)
    for fmt in (o.Q8_0, o.Q4_0):
        for dims in (576, 512):
            R = 3
            nb = dims // 32
            packed = np.zeros((R, o.quant_row_bytes(fmt, dims)), np.uint8)
            cb = dims if fmt == o.Q8_0 else dims // 2
            packed[:, :cb] = rng.integers(0, 256, (R, cb), dtype=np.uint8)
            if fmt == o.Q8_0:                  # -128 is not a code
                packed[:, :cb][packed[:, :cb] == 128] = 129
            scales = (rng.standard_normal((R, nb)) * 0.1).astype("<f2")
            packed[:, cb:cb + 2 * nb] = scales.view(np.uint8).reshape(R, -1)
            got = o.dequantize_rows(*o.unpack_rows(packed, fmt, dims), fmt)
            want = _dequant_loops(packed, fmt, dims)
            assert got.shape == (R, dims) and np.array_equal(got, want), (fmt, dims)


def pin_quant_properties(o, seed: int = 13):
    """Codes in range; Q8_0 error <= d/2; the largest magnitude maps to +-127 (Q8_0) or
    to 0 (Q4_0, the first one); Q4_0 error <= d/2 wherever |x/d| <= 7.5; pack/unpack
    round trip."""
    rng = np.random.default_rng(seed)
    x = (rng.standard_normal((6, 576)) * rng.choice([0.01, 1.0, 40.0], (6, 1))).astype(np.float16)
    x[0, :32] = 0                                          # an all-zero block
    for fmt in (o.Q8_0, o.Q4_0):
        codes, scales = o.quantize_rows(x, fmt)
        c2, s2 = o.unpack_rows(o.pack_rows(codes, scales, fmt), fmt, 576)
        assert np.array_equal(codes, c2) and np.array_equal(scales, s2)
        deq = o.dequantize_rows(codes, scales, fmt)
        d = np.repeat(np.abs(scales.astype(np.float64)), 32, axis=1)
        xf = x.astype(np.float64)
        assert np.all(deq[0, :32] == 0)
        if fmt == o.Q8_0:
            assert codes.min() >= -127 and codes.max() <= 127
            assert np.all(np.abs(xf - deq) <= d * (0.5 + 1e-3))
            blk = np.abs(xf).reshape(6, 18, 32).argmax(axis=2)
            top = np.take_along_axis(codes.astype(int).reshape(6, 18, 32), blk[..., None], 2)
            assert np.all((np.abs(top) == 127) | (scales.reshape(6, 18, 1) == 0))
        else:
            assert codes.min() >= 0 and codes.max() <= 15
            inside = np.abs(xf) <= 7.5 * d
            assert np.all(np.abs(xf - deq)[inside] <= d[inside] * (0.5 + 1e-3))
            blk = np.abs(xf).reshape(6, 18, 32).argmax(axis=2)
            top = np.take_along_axis(codes.astype(int).reshape(6, 18, 32), blk[..., None], 2)
            assert np.all((top == 0) | (scales.reshape(6, 18, 1) == 0))


def pin_quant_path_reduces_to_fp16(o, T: int = 64):
    """When every cache value is already d * integer with the block's extreme at the
    code limit, quantizing loses nothing: the quantized path equals prefill_tokens on
    the original cache, exactly, for both formats."""
    rng = np.random.default_rng(14)
    base = _np(generate_small(T, 4, 64, seed=42))
    for fmt, lim in ((o.Q8_0, 127), (o.Q4_0, 8)):
        inp = dict(base)
        for name, rows in (("kv_raw", T), ("kv_cmp", T // 4)):
            d = np.float16(2.0 ** -6)
            q = rng.integers(-lim + 1, lim, (rows, 576)).astype(np.float64)
            q[:, ::32] = -lim                             # each block's first value is the extreme
            inp[name] = (q * float(d)).astype(np.float16)
        toks = list(range(0, T, 5))
        a = o.prefill_tokens_quant(inp, toks, top_k=4, n_swa=5, fmt=fmt)
        b = o.prefill_tokens(inp, toks, top_k=4, n_swa=5)
        assert np.array_equal(a["topk"], b["topk"]) and np.array_equal(a["out"], b["out"]), fmt


def _sdpa_rows(q_t, krows, vrows, scale):
    """torch scaled_dot_product_attention in float64: 16 heads over one set of rows."""
    Q = torch.from_numpy(np.asarray(q_t, np.float64))[None, :, None, :]          # [1,16,1,576]
    K = torch.from_numpy(np.asarray(krows, np.float64))[None, None].expand(1, 16, -1, -1)
    V = torch.from_numpy(np.asarray(vrows, np.float64))[None, None].expand(1, 16, -1, -1)
    return torch.nn.functional.scaled_dot_product_attention(Q, K, V, scale=scale)[0, :, 0].numpy()


def pin_attention_kv_sdpa(o):
    """Separate keys and values: attention_token_kv equals torch SDPA with distinct K and V,
    and with V = the keys' first 512 values it equals attention_token."""
    q, kv_raw, kv_cmp = _attn_case(40, seed=26)
    rng = np.random.default_rng(3)
    krows = kv_raw[:37]
    vrows = rng.standard_normal((37, 512))
    got = o.attention_token_kv(q[5], krows, vrows, 0.06)
    assert np.abs(got - _sdpa_rows(q[5], krows, vrows, 0.06)).max() < 1e-12
    same = o.attention_token_kv(q[6], krows, krows[:, :512], 1.0 / 24.0)
    assert np.abs(same - o.attention_token(q[6], krows, 1.0 / 24.0, 512)).max() < 1e-13


def pin_quant_kv_split_composition(o, T: int = 48):
    """The Q8 K / Q4 V path for every token equals, built here step by step: keys from
    the Q8_0 rows, values from the Q4_0 rows of the first 512 values, the token's
    selected compressed rows then its window, and torch SDPA over them."""
    inp = _np(generate_small(T, 4, 64, seed=43))
    k, n_swa = 5, 7
    got = o.prefill_tokens_quant(inp, range(T), top_k=k, n_swa=n_swa, fmt=o.Q8K_Q4V)
    kq = {n: o.dequantize_rows(*o.quantize_rows(inp[n], o.Q8_0), o.Q8_0) for n in ("kv_raw", "kv_cmp")}
    vq = {n: o.dequantize_rows(*o.quantize_rows(inp[n][:, :512], o.Q4_0), o.Q4_0)
          for n in ("kv_raw", "kv_cmp")}
    for t in range(T):
        idx = o.topk_row(o.indexer_scores_token(inp["q_idx"][t], inp["k_idx"], inp["w"][t], t), k)
        assert np.array_equal(got["topk"][t], idx), t
        sel = [j for j in idx if j >= 0]
        win = list(range(max(0, t - n_swa + 1), t + 1))
        krows = np.concatenate([kq["kv_cmp"][sel], kq["kv_raw"][win]])
        vrows = np.concatenate([vq["kv_cmp"][sel], vq["kv_raw"][win]])
        want = _sdpa_rows(inp["q"][t], krows, vrows, 1.0 / 24.0)
        assert np.abs(got["out"][t] - want).max() < 1e-12, t


def pin_cache_rows_layout(o):
    """The stored row of each cache format read back part by part (unpack_rows at the
    part's byte offset, dequantize_rows) gives the key and value rows kv_values uses, and
    its length is quant_row_bytes."""
    rng = np.random.default_rng(15)
    x = (rng.standard_normal((5, 576)) * 2).astype(np.float16)
    for fmt in (o.Q8_0, o.Q4_0, o.Q8K_Q4V):
        packed = o.cache_rows(x, fmt)
        assert packed.shape == (5, o.quant_row_bytes(fmt, 576)), fmt
        k, v = o.kv_values(x, fmt)
        if fmt == o.Q8K_Q4V:
            kb = o.quant_row_bytes(o.Q8_0, 576)
            k2 = o.dequantize_rows(*o.unpack_rows(packed[:, :kb], o.Q8_0, 576), o.Q8_0)
            v2 = o.dequantize_rows(*o.unpack_rows(packed[:, kb:], o.Q4_0, 512), o.Q4_0)
        else:
            k2 = o.dequantize_rows(*o.unpack_rows(packed, fmt, 576), fmt)
            v2 = k2[:, :512]
        assert np.array_equal(k, k2) and np.array_equal(v, v2), fmt


ALL_PINS = [
    pin_visibility_mask, pin_visibility_golden,
    pin_scores_exact, pin_scores_relu_identities, pin_scores_bruteforce,
    pin_topk_golden, pin_topk_bruteforce, pin_topk_masked_bruteforce,
    pin_attention_sdpa_causal, pin_attention_sdpa_window, pin_attention_dense_mask,
    pin_attention_bruteforce, pin_attention_closed_forms,
    pin_bands_equal_oneshot, pin_prefill_tokens_composition,
    pin_quant_golden, pin_quant_dequant_bruteforce, pin_quant_properties,
    pin_quant_path_reduces_to_fp16, pin_attention_kv_sdpa, pin_quant_kv_split_composition,
    pin_cache_rows_layout,
]


def failing_pins(o):
    """Names of the pins the given oracle fails (used by the mutation tests)."""
    bad = []
    for p in ALL_PINS:
        try:
            p(o)
        except (AssertionError, ValueError, IndexError):
            bad.append(p.__name__)
    return bad
