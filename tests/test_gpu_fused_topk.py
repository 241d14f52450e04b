"""Fused indexer + top-k (topk_mode 1) against the oracle and against the two-kernel
path (topk_mode 0), through the C ABI.

The fused kernel keeps each token block's scores in shared memory and selects there;
the two-kernel path writes the scores to the workspace and reads them back. Both take
the same selection decisions on the same exact integer scores, so their indices must
be the same bits on every token, and both must equal the oracle's. Covered: whole
256-token (4 indexer heads: 64-token blocks) and 2048-token workloads, the full 8K and
10K prefills on every token, ragged bands and blocks, k >= n_vis, all scores equal,
and the calls the fused kernel does not take (rows longer than its key buffer, an
explicit mask), which must fall back to the two kernels with the same results.
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


def _both(wl, dev, **kw):
    res = {}
    for mode in (0, 1):
        with handle_for(wl, topk_mode=mode, **kw) as h:
            res[mode] = run_prefill(h, dev, wl.T, wl.top_k)
    return res


@pytest.mark.parametrize("name", ["tiny", "band"])
def test_whole_workload_fused(name):
    wl = workload(name)
    inp = generate(wl)
    res = _both(wl, to_device(inp))
    ref = oracle.prefill_bands(_np(inp), wl.T, wl.top_k, wl.n_swa, band=wl.band)
    assert np.array_equal(res[1][0].cpu().numpy(), ref["topk"])
    assert torch.equal(res[1][0], res[0][0])
    assert torch.equal(res[1][1], res[0][1])          # same indices -> same attention bits
    assert_attention_close(res[1][1].cpu().numpy(), ref["out"], name)


@pytest.mark.parametrize("name", ["8k", "10k"])
def test_full_prefill_fused_every_token(name):
    wl = workload(name)
    inp = generate(wl)
    res = _both(wl, to_device(inp))
    assert torch.equal(res[1][0], res[0][0])          # every token, bit for bit
    assert torch.equal(res[1][1], res[0][1])
    toks = sample_tokens(wl.T, wl.band, 24, seed=wl.seed + 100)
    ref = oracle_tokens(_np(inp), toks, wl)
    assert np.array_equal(res[1][0].cpu().numpy()[toks], ref["topk"])
    assert_attention_close(res[1][1].cpu().numpy()[toks], ref["out"], name)


@pytest.mark.parametrize("T,H_i,D_i,k,n_swa,band", [
    (300, 8, 64, 24, 40, 128),      # ragged bands, 32-token blocks
    (515, 16, 128, 40, 7, 512),     # ragged last block
    (2050, 64, 128, 100, 16, 1000), # 4-token blocks, ragged band of 50 tokens
    (200, 32, 128, 64, 200, 2048),  # k >= n_vis everywhere
    (3, 4, 64, 4, 2, 2048),         # no token sees a compressed row
])
def test_edge_cases_fused(T, H_i, D_i, k, n_swa, band):
    wl = Workload("edge", T=T, H_i=H_i, D_i=D_i, top_k=k, n_swa=n_swa, seed=T, band=band)
    inp = generate_small(T, H_i, D_i, seed=T + 11)
    res = _both(wl, to_device(inp))
    ref = oracle_tokens(_np(inp), range(T), wl)
    assert np.array_equal(res[1][0].cpu().numpy(), ref["topk"])
    assert torch.equal(res[1][0], res[0][0])
    assert_attention_close(res[1][1].cpu().numpy(), ref["out"], f"fused edge T={T}")


def test_all_scores_equal_fused():
    """Zero index weights: every key equal, the k lowest rows win (ties to the lower j)."""
    T, k = 512, 16                   # 128 rows at most: inside the fused kernel's key buffer
    wl = Workload("ties", T=T, H_i=4, D_i=64, top_k=k, n_swa=16, seed=T, band=256)
    inp = generate_small(T, 4, 64, seed=T + 2, weight_max=0)
    res = _both(wl, to_device(inp))
    ref = oracle_tokens(_np(inp), range(T), wl)
    nv = (np.arange(T) + 1) // 4
    assert (ref["topk"][nv >= k] == np.arange(k)).all()
    assert np.array_equal(res[1][0].cpu().numpy(), ref["topk"])


def test_fallback_for_long_rows():
    """The last 3 tokens of a 16,400-token context see 4,100 rows: more than the fused
    kernel's key buffer holds at 64 indexer heads, so the call runs the two kernels."""
    T, tail, k = 16400, 3, 64
    wl = Workload("long", T=T, H_i=64, D_i=128, top_k=k, n_swa=16, seed=T, band=2048)
    inp = generate_small(T, 64, 128, seed=T + 5)
    t0 = T - tail
    dev = to_device({n: (v[t0:] if n in ("q", "q_idx", "w") else v) for n, v in inp.items()})
    with handle_for(wl, topk_mode=1) as h:
        topk, out = run_range(h, dev, t0, tail, k)
    ref = oracle_tokens(_np(inp), range(t0, T), wl)
    assert np.array_equal(topk.cpu().numpy(), ref["topk"])
    assert_attention_close(out.cpu().numpy(), ref["out"], "long rows")
