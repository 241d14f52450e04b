"""CUDA path vs the CPU oracle on the same seeded inputs, through the C ABI.

Top-k indices must match bit for bit; attention within max-abs 2e-3 and NMSE 1e-6
of the float64 oracle. Small workloads are compared on every token; the 8K and
10K prefills run whole (as the benchmark times them) and are compared on band
edges plus a seeded random sample of tokens.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import (assert_attention_close, handle_for, oracle_tokens, run_prefill,
                        run_range, sample_tokens, to_device)
from sparse_mla_prefill_b200 import build as B
from sparse_mla_prefill_b200 import ds4sp as D
from sparse_mla_prefill_b200.inputs import Workload, generate, generate_small, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    B.build()
    D.load_library()


def _np(inp):
    return {k: v.numpy() for k, v in inp.items()}


@pytest.mark.parametrize("name", ["tiny", "band"])
def test_whole_workload(name):
    wl = workload(name)
    inp = generate(wl)
    with handle_for(wl) as h:
        topk, out = run_prefill(h, to_device(inp), wl.T, wl.top_k)
    ref = oracle.prefill_bands(_np(inp), wl.T, wl.top_k, wl.n_swa, band=wl.band)
    assert np.array_equal(topk.cpu().numpy(), ref["topk"])
    assert_attention_close(out.cpu().numpy(), ref["out"], name)


@pytest.mark.parametrize("name", ["8k", "10k"])
def test_full_size_sampled(name):
    wl = workload(name)
    inp = generate(wl)
    with handle_for(wl) as h:
        topk, out = run_prefill(h, to_device(inp), wl.T, wl.top_k)
    toks = sample_tokens(wl.T, wl.band, 48, seed=wl.seed)
    ref = oracle_tokens(_np(inp), toks, wl)
    got_topk = topk.cpu().numpy()[toks]
    assert np.array_equal(got_topk, ref["topk"])
    assert_attention_close(out.cpu().numpy()[toks], ref["out"], name)
    # properties that hold for every token at any size
    tk = topk.cpu().numpy()
    nsel = np.minimum(wl.top_k, (np.arange(wl.T) + 1) // 4)
    valid = tk >= 0
    assert np.array_equal(valid.sum(1), nsel)
    assert ((~valid) | (tk < ((np.arange(wl.T) + 1) // 4)[:, None])).all()
    assert np.isfinite(out.cpu().numpy()).all()


def test_verify_widths_bit_identical_across_widths():
    wl = workload("verify")
    inp = generate(wl)                       # per-token tensors: the last 5 positions
    dev = to_device(inp)
    npi = _np(inp)
    T = wl.T
    ref = oracle_tokens(npi, range(T - 5, T), wl, q_start=T - 5)
    results = {}
    with handle_for(wl) as h:
        for q in range(1, 6):
            sl = {k: (v[5 - q:].contiguous() if k in ("q", "q_idx", "w") else v) for k, v in dev.items()}
            topk, out = run_range(h, sl, T - q, q, wl.top_k)
            results[q] = (topk.cpu().numpy(), out.cpu().numpy())
            assert np.array_equal(results[q][0], ref["topk"][5 - q:]), q
            assert_attention_close(results[q][1], ref["out"][5 - q:], f"verify q={q}")
    # the same token gives the same bits whatever the width
    for q in range(1, 6):
        assert np.array_equal(results[q][0][-1], results[5][0][-1])
        assert np.array_equal(results[q][1][-1], results[5][1][-1])


def test_split_tokens_equal_across_call_sizes():
    """Split-mode attention of the 5-token verify step (100 units of 32 rows, fewer than
    the SMs) and of an 8-token call (160 units, more than the SMs, so a CTA takes two):
    the tokens both calls hold get the same top-k and output bits."""
    wl = workload("verify")
    inp = generate(wl)
    dev = to_device(inp)
    T = wl.T
    with handle_for(wl) as h:
        # the last 8 tokens: per-token tensors of the verify workload hold 5, so widen them
        # with 3 earlier tokens' copies of the same draws (positions differ, values repeat)
        sl8 = {k: (torch.cat([v[:3], v]).contiguous() if k in ("q", "q_idx", "w") else v)
               for k, v in dev.items()}
        tk8, out8 = run_range(h, sl8, T - 8, 8, wl.top_k)
        tk5, out5 = run_range(h, dev, T - 5, 5, wl.top_k)
    assert torch.equal(tk8[3:], tk5)
    assert torch.equal(out8[3:], out5)


def test_band_path_equals_one_shot_bitwise():
    wl = workload("band", T=2048 + 700, band=1024)
    inp = generate_small(wl.T, wl.H_i, wl.D_i, seed=9)
    dev = to_device(inp)
    with handle_for(wl) as h:
        tk_b, out_b = run_prefill(h, dev, wl.T, wl.top_k)
        tk_o, out_o = run_range(h, dev, 0, wl.T, wl.top_k)
    assert torch.equal(tk_b, tk_o)
    assert torch.equal(out_b, out_o)


EDGE_CASES = [
    # T, H_i, D_i, k, n_swa, band, scale      ragged bands / tails / degenerate windows
    (300, 8, 64, 24, 40, 128, 0.0),
    (515, 16, 128, 40, 7, 512, 0.0),
    (200, 32, 128, 64, 200, 2048, 0.0),      # k >= n_vis everywhere, window >= T: dense
    (130, 64, 64, 0, 130, 64, 0.0),          # no compressed rows: causal attention
    (97, 4, 64, 5, 1, 32, 0.03),             # window of one raw row, explicit scale
    (1, 4, 64, 4, 4, 2048, 0.0),             # one token
    (3, 4, 64, 4, 2, 2048, 0.0),             # no token sees a compressed row
    (700, 64, 128, 512, 128, 2048, 0.0),     # k > n_vis for every token
]


@pytest.mark.parametrize("T,H_i,D_i,k,n_swa,band,scale", EDGE_CASES)
def test_edge_cases(T, H_i, D_i, k, n_swa, band, scale):
    wl = Workload("edge", T=T, H_i=H_i, D_i=D_i, top_k=k, n_swa=n_swa, seed=T, band=band)
    inp = generate_small(T, H_i, D_i, seed=T + 1)
    with handle_for(wl, softmax_scale=scale) as h:
        topk, out = run_prefill(h, to_device(inp), T, k)
    ref = oracle_tokens(_np(inp), range(T), wl, scale=scale if scale > 0 else None)
    if k > 0:
        assert np.array_equal(topk.cpu().numpy(), ref["topk"])
    assert_attention_close(out.cpu().numpy(), ref["out"], f"edge T={T}")


@pytest.mark.parametrize("T,k,band,tail", [(600, 16, 256, None), (16400, 64, 2048, 3)])
def test_all_scores_equal(T, k, band, tail):
    """Zero index weights make every score 0, so every candidate key is the same: the
    select's all-keys-equal path must keep the k lowest rows (ties to the lower j). A
    600-token prefill (256-thread top-k) and the last 3 tokens of a 16,400-token context
    (rows of 4,100 scores: the 1,024-thread top-k, and few-token attention)."""
    wl = Workload("ties", T=T, H_i=4, D_i=64, top_k=k, n_swa=16, seed=T, band=band)
    inp = generate_small(T, 4, 64, seed=T + 2, weight_max=0)
    if tail is None:
        toks = list(range(T))
        with handle_for(wl) as h:
            topk, out = run_prefill(h, to_device(inp), T, k)
    else:
        t0 = T - tail
        toks = list(range(t0, T))
        dev = to_device({n: (v[t0:] if n in ("q", "q_idx", "w") else v) for n, v in inp.items()})
        with handle_for(wl) as h:
            topk, out = run_range(h, dev, t0, tail, k)
    ref = oracle_tokens(_np(inp), toks, wl)
    nv = (np.asarray(toks) + 1) // 4
    assert (ref["topk"][nv >= k] == np.arange(k)).all()      # the lowest k rows
    assert np.array_equal(topk.cpu().numpy(), ref["topk"])
    assert_attention_close(out.cpu().numpy(), ref["out"], f"equal scores T={T}")


def _dim0_scores(T, seed, dim0):
    """Inputs whose index score of row j is dim0[j] for every token: one index head with
    weight 1 whose query picks the key's first dimension (dim0 >= 0)."""
    inp = generate_small(T, 4, 64, seed=seed)
    k_idx = torch.zeros(T // 4, 64)
    k_idx[:, 0] = dim0
    q_idx = torch.zeros(T, 4, 64)
    q_idx[:, 0, 0] = 1.0
    w = torch.zeros(T, 4)
    w[:, 0] = 1.0
    inp.update(k_idx=k_idx.half(), q_idx=q_idx.half(), w=w)
    return inp


@pytest.mark.parametrize("case", ["ties", "near_equal"])
def test_topk_radix_candidate_list(case):
    """The radix select gathers the chosen bucket's keys into a list once a pass leaves at
    most 512 of them and runs the later passes over the list. "ties": rows 0..599 score 3
    and the rest 0, so a token that sees more than 512 rows never gets a small enough
    bucket (every pass scans all keys) and one that sees fewer is listed after the first
    pass; "near_equal": rows 0..599 score 1024 + j and the rest 1, so the first pass's
    bucket holds up to 600 keys and the list forms at the second pass. Indices must equal
    the oracle's (ties to the lower j)."""
    T, k = 3000, 64
    n_c = T // 4
    j = torch.arange(n_c, dtype=torch.float32)
    dim0 = torch.where(j < 600, torch.full_like(j, 3.0), torch.zeros_like(j)) if case == "ties" \
        else torch.where(j < 600, 1024.0 + j, torch.ones_like(j))
    inp = _dim0_scores(T, 21, dim0)
    wl = Workload(case, T=T, H_i=4, D_i=64, top_k=k, n_swa=16, seed=21)
    toks = sorted(set(range(0, T, 7)) | set(range(T - 8, T)) | {2047, 2400, 2403})
    with handle_for(wl) as h:
        topk, out = run_range(h, to_device(inp), 0, T, k)
    ref = oracle_tokens(_np(inp), toks, wl)
    got = topk.cpu().numpy()[toks]
    assert np.array_equal(got, ref["topk"])
    assert_attention_close(out.cpu().numpy()[toks], ref["out"], case)


def test_causal_reduction_against_sdpa():
    """k = 0 and n_swa >= T: the CUDA path equals causal attention (torch SDPA, float64)."""
    T = 160
    wl = Workload("causal", T=T, H_i=4, D_i=64, top_k=0, n_swa=T, seed=0)
    inp = generate_small(T, 4, 64, seed=77)
    with handle_for(wl) as h:
        _, out = run_prefill(h, to_device(inp), T, 0)
    q = inp["q"].double().permute(1, 0, 2)[None]
    kv = inp["kv_raw"].double()
    ref = torch.nn.functional.scaled_dot_product_attention(
        q, kv[None, None].expand(1, 16, T, 576), kv[None, None, :, :512].expand(1, 16, T, 512),
        is_causal=True, scale=1.0 / 24.0)[0].permute(1, 0, 2).numpy()
    assert_attention_close(out.cpu().numpy(), ref, "causal")
