"""Attention with the logits on tcgen05 (attn_kernel 1) against the oracle, through the C ABI.

The variant gathers 128 rows per unit into the 128-byte-swizzled K-major layout,
computes S = R . Q^T on the tensor cores into TMEM (rows as M = 128, the 16 heads as
N = 16), runs the softmax from TMEM and P . V on mma.sync. Its indices come from the same
indexer and top-k, so they must equal the oracle's bit for bit; its attention output
must meet the same bar as the streaming kernel (max-abs 2e-3, NMSE 1e-6 against the
float64 oracle): fp16 rows and probabilities, fp32 logits, softmax and accumulation.
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
def test_whole_workload_tc(name):
    wl = workload(name)
    inp = generate(wl)
    with handle_for(wl, attn_kernel=1) as h:
        topk, out = run_prefill(h, to_device(inp), wl.T, wl.top_k)
    ref = oracle.prefill_bands(_np(inp), wl.T, wl.top_k, wl.n_swa, band=wl.band)
    assert np.array_equal(topk.cpu().numpy(), ref["topk"])
    assert_attention_close(out.cpu().numpy(), ref["out"], f"tc {name}")


def test_10k_sampled_tc():
    wl = workload("10k")
    inp = generate(wl)
    with handle_for(wl, attn_kernel=1) as h:
        topk, out = run_prefill(h, to_device(inp), wl.T, wl.top_k)
    toks = sample_tokens(wl.T, wl.band, 32, seed=41)
    ref = oracle_tokens(_np(inp), toks, wl)
    assert np.array_equal(topk.cpu().numpy()[toks], ref["topk"])
    assert_attention_close(out.cpu().numpy()[toks], ref["out"], "tc 10k")
    assert np.isfinite(out.cpu().numpy()).all()


@pytest.mark.parametrize("T,H_i,D_i,k,n_swa,band,scale", [
    (300, 8, 64, 24, 40, 128, 0.0),          # ragged bands, units of < 128 rows
    (700, 64, 128, 512, 128, 2048, 0.0),     # k > n_vis: up to 303 rows, 3 units
    (97, 4, 64, 5, 1, 32, 0.03),             # window of one row, explicit scale
    (130, 64, 64, 0, 130, 64, 0.0),          # no compressed rows: causal attention
])
def test_edge_cases_tc(T, H_i, D_i, k, n_swa, band, scale):
    wl = Workload("edge", T=T, H_i=H_i, D_i=D_i, top_k=k, n_swa=n_swa, seed=T, band=band)
    inp = generate_small(T, H_i, D_i, seed=T + 21)
    with handle_for(wl, attn_kernel=1, softmax_scale=scale) as h:
        topk, out = run_prefill(h, to_device(inp), T, k)
    ref = oracle_tokens(_np(inp), range(T), wl, scale=scale if scale > 0 else None)
    if k > 0:
        assert np.array_equal(topk.cpu().numpy(), ref["topk"])
    assert_attention_close(out.cpu().numpy(), ref["out"], f"tc edge T={T}")


def test_verify_width_tc():
    """The last 3 tokens of the 122,880-token context (640 rows each, five units)."""
    wl = workload("verify")
    inp = generate(wl)
    q = 3
    sl = {k: (v[5 - q:].contiguous() if k in ("q", "q_idx", "w") else v) for k, v in inp.items()}
    with handle_for(wl, attn_kernel=1) as h:
        topk, out = run_range(h, to_device(sl), wl.T - q, q, wl.top_k)
    ref = oracle_tokens(_np(sl), range(wl.T - q, wl.T), wl, q_start=wl.T - q)
    assert np.array_equal(topk.cpu().numpy(), ref["topk"])
    assert_attention_close(out.cpu().numpy(), ref["out"], "tc verify")


def test_formula_mask_bit_identical_tc():
    """The explicit-mask form with the formula's own mask gives the analytic path's bits."""
    wl = workload("tiny")
    inp = to_device(generate(wl))
    with handle_for(wl, attn_kernel=1) as h:
        tk_a, out_a = run_prefill(h, inp, wl.T, wl.top_k)
        t = torch.arange(wl.T)[:, None]
        j = torch.arange(wl.T // 4)[None, :]
        mask = (4 * j + 3 <= t).to(torch.uint8).cuda()
        D.ds4sp_debug_set_mask(h, mask)
        tk_m, out_m = run_prefill(h, inp, wl.T, wl.top_k)
        D.ds4sp_debug_set_mask(h, None)
    assert torch.equal(tk_a, tk_m)
    assert torch.equal(out_a, out_m)
