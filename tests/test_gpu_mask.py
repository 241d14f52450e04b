"""Explicit-mask versus analytic visibility ("perf(ds4): extend sparse prefill
scheduling to 10K", Qualification: an explicit-mask versus analytic-mask oracle whose
streaming-attention output is bit-identical).

The same kernels take the compressed rows' visibility from a stored uint8 mask
(ds4sp_debug_set_mask) instead of the ratio-4 formula. With the mask the oracle
builds from the row-coverage definition, the indices and the attention output must
be bit-identical to the analytic path. With a stricter mask (rows hidden at random)
the selection must follow the mask exactly (the oracle's explicit-mask top-k) and the
attention must drop every row the mask hides: this shows the mask is really read.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import assert_attention_close, handle_for, run_prefill, run_range, to_device
from sparse_mla_prefill_b200 import build as B
from sparse_mla_prefill_b200 import ds4sp as D
from sparse_mla_prefill_b200.inputs import generate, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    B.build()
    D.load_library()


def _np(inp):
    return {k: v.numpy() for k, v in inp.items()}


def _dev_mask(m: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(m.astype(np.uint8))).cuda()


def _bits(x: torch.Tensor) -> torch.Tensor:
    return x.contiguous().view(torch.int32)


def _stricter_mask(T: int, n_c: int, seed: int, hide: float = 0.3) -> np.ndarray:
    rng = np.random.default_rng(seed)
    return oracle.explicit_visibility_mask(T, n_c) & (rng.random((T, n_c)) >= hide)


@pytest.mark.parametrize("name,T", [("tiny", None), ("band", None), ("band", 4096)])
def test_formula_mask_is_bit_identical(name, T):
    wl = workload(name) if T is None else workload(name, T=T)   # 4096: two bands
    inp = generate(wl)
    dev = to_device(inp)
    mask = oracle.explicit_visibility_mask(wl.T, inp["kv_cmp"].shape[0])
    with handle_for(wl) as h:
        tk_a, out_a = run_prefill(h, dev, wl.T, wl.top_k)
        D.ds4sp_reset(h, 0)
        D.ds4sp_debug_set_mask(h, _dev_mask(mask))
        tk_m, out_m = run_prefill(h, dev, wl.T, wl.top_k)
        D.ds4sp_debug_set_mask(h, None)
        D.ds4sp_reset(h, 0)
        tk_b, out_b = run_prefill(h, dev, wl.T, wl.top_k)   # cleared: the formula again
    assert torch.equal(tk_a, tk_m)
    assert torch.equal(_bits(out_a), _bits(out_m))
    assert torch.equal(tk_a, tk_b) and torch.equal(_bits(out_a), _bits(out_b))


@pytest.mark.parametrize("name", ["tiny", "band"])
def test_stricter_mask_follows_the_mask(name):
    wl = workload(name)
    inp = generate(wl)
    npi = _np(inp)
    n_c = inp["kv_cmp"].shape[0]
    mask = _stricter_mask(wl.T, n_c, seed=wl.seed + 100)
    with handle_for(wl) as h:
        D.ds4sp_debug_set_mask(h, _dev_mask(mask))
        tk, out = run_prefill(h, to_device(inp), wl.T, wl.top_k)
    scores = oracle.indexer_scores(npi["q_idx"], npi["k_idx"], npi["w"], 0)
    want = np.stack([oracle.topk_row_masked(scores[t], mask[t], wl.top_k) for t in range(wl.T)])
    got = tk.cpu().numpy()
    assert np.array_equal(got, want)
    # some tokens keep fewer than k rows although more than k are visible by the formula
    nv = (np.arange(wl.T) + 1) // 4
    short = ((got >= 0).sum(1) < wl.top_k) & (nv > wl.top_k)
    assert short.any()
    ref = oracle.sparse_mla_attention(npi["q"], npi["kv_raw"], npi["kv_cmp"], want, 0, wl.n_swa)
    assert_attention_close(out.cpu().numpy(), ref, name + " masked")


def test_masked_attention_drops_hidden_rows():
    """The analytic top-k fed to the masked attention: rows the mask hides are dropped."""
    wl = workload("band")
    inp = generate(wl)
    npi = _np(inp)
    dev = to_device(inp)
    mask = _stricter_mask(wl.T, inp["kv_cmp"].shape[0], seed=7)
    with handle_for(wl) as h:
        tk, _ = run_range(h, dev, 0, wl.T, wl.top_k)
        D.ds4sp_debug_set_mask(h, _dev_mask(mask))
        out = torch.full((wl.T, 16, 512), float("nan"), dtype=torch.float32, device="cuda")
        D.ds4sp_sparse_attn(h, dev["q"], dev["kv_raw"], dev["kv_cmp"], tk, 0, wl.T, out)
        torch.cuda.synchronize()
        st, bits = D.ds4sp_device_status(h)
    assert st == D.OK, f"device status bits {bits:#x}"
    tk_np = tk.cpu().numpy()
    rows = np.arange(wl.T)[:, None]
    kept = np.where((tk_np >= 0) & mask[rows, np.maximum(tk_np, 0)], tk_np, -1)
    assert (kept != tk_np).any()
    ref = oracle.sparse_mla_attention(npi["q"], npi["kv_raw"], npi["kv_cmp"], kept, 0, wl.n_swa)
    assert_attention_close(out.cpu().numpy(), ref, "analytic top-k, masked attention")


def test_mask_shorter_than_the_call_is_rejected():
    wl = workload("tiny")
    inp = generate(wl)
    dev = to_device(inp)
    mask = oracle.explicit_visibility_mask(wl.T - 1, inp["kv_cmp"].shape[0])
    with handle_for(wl) as h:
        D.ds4sp_debug_set_mask(h, _dev_mask(mask))
        topk = torch.empty((wl.T, wl.top_k), dtype=torch.int32, device="cuda")
        ws = torch.empty(max(D.ds4sp_workspace_bytes(h, 0, wl.T), 256), dtype=torch.uint8,
                         device="cuda")
        with pytest.raises(D.Ds4spError) as e:
            D.ds4sp_indexer_topk(h, dev["q_idx"], dev["k_idx"], dev["w"], 0, wl.T, topk, ws)
        assert e.value.status == D.ERR_INVALID_ARG
        # a call inside the mask's rows runs
        D.ds4sp_indexer_topk(h, dev["q_idx"], dev["k_idx"], dev["w"], 0, wl.T - 1, topk, ws)
        lib = D.load_library()
        m = _dev_mask(mask)
        assert lib.ds4sp_debug_set_mask(h.ptr, m.data_ptr(), 0, m.shape[1]) == D.ERR_INVALID_ARG
        assert lib.ds4sp_debug_set_mask(h.ptr, m.data_ptr(), m.shape[0], -1) == D.ERR_INVALID_ARG
        torch.cuda.synchronize()


def test_mask_wide_rows_few_tokens():
    """Rows longer than 4,096 scores (the 1,024-thread top-k) and a few-token call (split
    attention with the merge): the last 5 tokens of a 16,400-token context."""
    wl = workload("verify", T=16400, seed=11)
    inp = generate(wl)
    npi = _np(inp)
    n_c = inp["kv_cmp"].shape[0]
    t0, n_q = wl.q_start, wl.verify_q
    t = np.arange(wl.T)[:, None]
    j = np.arange(n_c)[None, :]
    mask = 4 * j + 3 <= t                                   # the formula's mask
    rng = np.random.default_rng(5)
    mask[t0:] &= rng.random((n_q, n_c)) >= 0.3              # the query rows: stricter
    with handle_for(wl) as h:
        D.ds4sp_debug_set_mask(h, _dev_mask(mask))
        tk, out = run_range(h, to_device(inp), t0, n_q, wl.top_k)
    scores = oracle.indexer_scores(npi["q_idx"], npi["k_idx"], npi["w"], t0)
    want = np.stack([oracle.topk_row_masked(scores[i], mask[t0 + i], wl.top_k)
                     for i in range(n_q)])
    assert np.array_equal(tk.cpu().numpy(), want)
    ref = oracle.sparse_mla_attention(npi["q"], npi["kv_raw"], npi["kv_cmp"], want, t0, wl.n_swa)
    assert_attention_close(out.cpu().numpy(), ref, "wide rows, masked")
