"""The indexer's fp32 scores against the oracle's exact integer scores, bit for bit.

ds4sp_indexer_topk leaves the scores of its call in the caller's workspace, rows of
ld = n_vis(t_last) rounded up to 4 floats, one row per token. With integer-valued
indexer inputs every score is an integer below 2^24, so the fp32 value is exact
whatever the summation order; each defined column j < n_vis(t) of every token must
have the bits of oracle.indexer_scores_token_exact (int64 arithmetic) converted to
fp32. Columns j >= n_vis(t) are not defined and are not read. (The handles here use
topk_mode 0, the path that writes the scores; the fused path keeps them on chip and is
checked through its indices in test_gpu_fused_topk.py.) Both indexer kernels are run:
one CTA per tcgen05 tile (indexer_kernel 0) and CTA pairs sharing each MMA (1).
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import handle_for, to_device
from sparse_mla_prefill_b200 import build as B
from sparse_mla_prefill_b200 import ds4sp as D
from sparse_mla_prefill_b200.inputs import generate, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    B.build()
    D.load_library()


def _scores_of_call(h, dev, t0, n_q, top_k):
    need = D.ds4sp_workspace_bytes(h, t0, n_q)
    ws = torch.full((need,), 0xFF, dtype=torch.uint8, device="cuda")   # NaN bit patterns
    topk = torch.empty((n_q, top_k), dtype=torch.int32, device="cuda")
    D.ds4sp_indexer_topk(h, dev["q_idx"], dev["k_idx"], dev["w"], t0, n_q, topk, ws)
    torch.cuda.synchronize()
    st, bits = D.ds4sp_device_status(h)
    assert st == D.OK, f"device status {bits:#x}"
    nv_last = (t0 + n_q) // 4
    ld = (max(nv_last, 1) + 3) // 4 * 4
    return ws[:n_q * ld * 4].view(torch.float32).view(n_q, ld).cpu().numpy()


def _check_rows(scores, inp, t0, n_q):
    q_idx, k_idx, w = inp["q_idx"].numpy(), inp["k_idx"].numpy(), inp["w"].numpy()
    for i in range(n_q):
        t = t0 + i
        exact = oracle.indexer_scores_token_exact(q_idx[i], k_idx, w[i], t)
        assert exact.shape == (oracle.n_vis(t),)
        assert np.abs(exact).max(initial=0) < 2 ** 24
        got = scores[i, :len(exact)]
        want = exact.astype(np.float32)
        if not np.array_equal(got.view(np.uint32), want.view(np.uint32)):
            bad = np.flatnonzero(got.view(np.uint32) != want.view(np.uint32))
            raise AssertionError(f"token {t}: {len(bad)} scores differ, first j={bad[0]} "
                                 f"got {got[bad[0]]} want {want[bad[0]]}")


def _check_rows_sampled(scores, inp, t0, toks):
    for t in toks:
        i = t - t0
        _check_rows(scores[i:i + 1], {"q_idx": inp["q_idx"][i:i + 1], "k_idx": inp["k_idx"],
                                      "w": inp["w"][i:i + 1]}, t, 1)


@pytest.mark.parametrize("indexer_kernel", [0, 1])
@pytest.mark.parametrize("name", ["tiny", "band"])
def test_scores_every_token(name, indexer_kernel):
    """Every token of the 256-token (4 x 64 indexer) and 2048-token (64 x 128) workloads."""
    wl = workload(name)
    inp = generate(wl)
    with handle_for(wl, topk_mode=0, indexer_kernel=indexer_kernel) as h:
        scores = _scores_of_call(h, to_device(inp), 0, wl.T, wl.top_k)
    _check_rows(scores, inp, 0, wl.T)


@pytest.mark.parametrize("indexer_kernel", [0, 1])
@pytest.mark.parametrize("q", [1, 5])
def test_scores_verify_width(q, indexer_kernel):
    """The last q tokens of the 122,880-token context: rows of up to 30,720 scores."""
    wl = workload("verify")
    inp = generate(wl)                     # per-token tensors of the last 5 positions
    sl = {k: (v[5 - q:].contiguous() if k in ("q", "q_idx", "w") else v) for k, v in inp.items()}
    with handle_for(wl, topk_mode=0, indexer_kernel=indexer_kernel) as h:
        scores = _scores_of_call(h, to_device(sl), wl.T - q, q, wl.top_k)
    _check_rows(scores, sl, wl.T - q, q)


@pytest.mark.parametrize("indexer_kernel", [0, 1])
def test_scores_10k_last_band_sampled(indexer_kernel):
    """The last band of the 10K prefill (rows of 2,048-2,560 scores): 48 tokens, among
    them the band's first and last and both ends of a token block."""
    wl = workload("10k")
    inp = generate(wl)
    t0, n = 8192, 2048
    sl = {k: (v[t0:t0 + n].contiguous() if k in ("q", "q_idx", "w") else v) for k, v in inp.items()}
    with handle_for(wl, topk_mode=0, indexer_kernel=indexer_kernel) as h:
        scores = _scores_of_call(h, to_device(sl), t0, n, wl.top_k)
    rng = np.random.default_rng(5)
    toks = sorted({t0, t0 + 3, t0 + 4, t0 + n - 1, *rng.integers(t0, t0 + n, 44).tolist()})
    _check_rows_sampled(scores, sl, t0, toks)
