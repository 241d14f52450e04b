"""Host-side error paths with a live handle. Each bad call must return its status
before launching anything; the in-kernel index check must skip and report an
out-of-range top-k entry without faulting (the bad index is never dereferenced)."""
import numpy as np
import pytest
import torch

from gpu_common import handle_for, run_prefill, to_device
from sparse_mla_prefill_b200 import build as B
from sparse_mla_prefill_b200 import ds4sp as D
from sparse_mla_prefill_b200.inputs import Workload, generate_small

pytestmark = pytest.mark.gpu

WL = Workload("err", T=600, H_i=8, D_i=64, top_k=32, n_swa=16, seed=0, band=256)


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    B.build()
    D.load_library()


@pytest.fixture()
def setup():
    inp = to_device(generate_small(WL.T, WL.H_i, WL.D_i, seed=5))
    h = handle_for(WL)
    topk = torch.zeros((WL.T, WL.top_k), dtype=torch.int32, device="cuda")
    out = torch.zeros((WL.T, 16, 512), dtype=torch.float32, device="cuda")
    ws = D.band_workspace(h, WL.T, "cuda")
    yield h, inp, topk, out, ws
    D.ds4sp_destroy(h)


def _band(h, b, inp, topk, out, ws, n_tokens=WL.T):
    D.ds4sp_prefill_band(h, b, n_tokens, inp["q"], inp["q_idx"], inp["w"], inp["kv_raw"],
                         inp["kv_cmp"], inp["k_idx"], topk, out, ws)


def _status_of(fn):
    with pytest.raises(D.Ds4spError) as e:
        fn()
    return e.value.status


def test_band_order_enforced(setup):
    h, inp, topk, out, ws = setup
    assert D.ds4sp_next_band(h) == 0
    assert _status_of(lambda: _band(h, 1, inp, topk, out, ws)) == D.ERR_ORDER
    torch.cuda.synchronize()
    assert out.abs().sum().item() == 0            # nothing launched
    _band(h, 0, inp, topk, out, ws)
    assert D.ds4sp_next_band(h) == 1
    assert _status_of(lambda: _band(h, 0, inp, topk, out, ws)) == D.ERR_ORDER
    _band(h, 1, inp, topk, out, ws)
    _band(h, 2, inp, topk, out, ws)
    assert _status_of(lambda: _band(h, 3, inp, topk, out, ws)) == D.ERR_INVALID_ARG  # past the end
    D.ds4sp_reset(h, 1)                            # resume from band 1
    _band(h, 1, inp, topk, out, ws)


def test_small_workspace_rejected(setup):
    h, inp, topk, out, ws = setup
    need = D.ds4sp_workspace_bytes(h, 0, 256)
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    assert _status_of(lambda: D.ds4sp_indexer_topk(h, inp["q_idx"], inp["k_idx"], inp["w"], 0,
                                                   256, topk, small)) == D.ERR_WORKSPACE
    assert _status_of(lambda: _band(h, 0, inp, topk, out, small)) == D.ERR_WORKSPACE


def test_misaligned_and_out_of_range(setup):
    h, inp, topk, out, ws = setup
    q_off = inp["q"].view(-1)[1:1 + 256 * 16 * 576]       # 2-byte offset
    assert _status_of(lambda: D.ds4sp_sparse_attn(h, q_off, inp["kv_raw"], inp["kv_cmp"], topk,
                                                  0, 256, out)) == D.ERR_INVALID_ARG
    assert _status_of(lambda: D.ds4sp_sparse_attn(h, inp["q"], inp["kv_raw"], inp["kv_cmp"], topk,
                                                  500, 200, out)) == D.ERR_INVALID_ARG
    assert _status_of(lambda: D.ds4sp_sparse_attn(h, inp["q"], inp["kv_raw"], inp["kv_cmp"], topk,
                                                  -1, 4, out)) == D.ERR_INVALID_ARG
    ws_off = ws[16:]                                       # 16-byte aligned, not 256
    assert _status_of(lambda: D.ds4sp_indexer_topk(h, inp["q_idx"], inp["k_idx"], inp["w"], 0, 8,
                                                   topk, ws_off)) == D.ERR_INVALID_ARG


def test_empty_range_is_a_no_op(setup):
    h, inp, topk, out, ws = setup
    D.ds4sp_indexer_topk(h, inp["q_idx"], inp["k_idx"], inp["w"], 10, 0, topk, ws)
    D.ds4sp_sparse_attn(h, inp["q"], inp["kv_raw"], inp["kv_cmp"], topk, 10, 0, out)
    torch.cuda.synchronize()
    assert out.abs().sum().item() == 0


def test_injected_launch_failure(setup):
    h, inp, topk, out, ws = setup
    D.ds4sp_debug_fail_launches(h, 1)
    assert _status_of(lambda: D.ds4sp_sparse_attn(h, inp["q"], inp["kv_raw"], inp["kv_cmp"], topk,
                                                  0, 64, out)) == D.ERR_CUDA
    torch.cuda.synchronize()
    assert out.abs().sum().item() == 0
    D.ds4sp_sparse_attn(h, inp["q"], inp["kv_raw"], inp["kv_cmp"], topk, 0, 64, out)  # recovers
    torch.cuda.synchronize()
    assert torch.isfinite(out[:64]).all()


def test_bad_topk_index_is_skipped_and_reported(setup):
    h, inp, topk, out, ws = setup
    t0, n_q = 400, 8                     # n_vis(t) = 100 .. 102 here, so 32 rows selected
    tk = torch.arange(WL.top_k, dtype=torch.int32, device="cuda").repeat(n_q, 1)
    tk[0, 5] = 10 ** 6                   # beyond every buffer
    tk[1, 0] = -1                        # a hole inside the selected slots
    tk[2, 31] = 101                      # not yet visible to token 400 (n_vis = 100)
    o = torch.zeros((n_q, 16, 512), dtype=torch.float32, device="cuda")
    D.ds4sp_sparse_attn(h, inp["q"][t0:t0 + n_q], inp["kv_raw"], inp["kv_cmp"], tk, t0, n_q, o)
    st, bits = D.ds4sp_device_status(h)
    assert st == D.ERR_DEVICE_BOUNDS and bits & 1
    assert torch.isfinite(o).all()
    st, bits = D.ds4sp_device_status(h)  # read clears the word
    assert st == D.OK and bits == 0


@pytest.mark.parametrize("topk_mode", [0, 1])
def test_profile_counts_launches(setup, topk_mode):
    """Three bands: three launches of each kernel, or, with the fused indexer + top-k,
    three of it (timed as the indexer) and none of the separate top-k."""
    _, inp, topk, out, _ = setup
    with handle_for(WL, topk_mode=topk_mode) as h:
        ws = D.band_workspace(h, WL.T, "cuda")
        D.ds4sp_profile_enable(h, True)
        D.prefill(h, inp, WL.T, topk, out, ws)
        prof = D.ds4sp_profile_read(h)
        n_topk = 3 if topk_mode == 0 else 0
        assert prof["indexer"][1] == 3 and prof["topk"][1] == n_topk and prof["attention"][1] == 3
        assert all(ms > 0 for ms, n in prof.values() if n > 0)
        assert all(n == 0 for _, n in D.ds4sp_profile_read(h).values())
        D.ds4sp_profile_enable(h, False)


def test_destroy_waits_for_work_in_flight():
    inp = to_device(generate_small(WL.T, WL.H_i, WL.D_i, seed=6))
    h = handle_for(WL)
    topk = torch.zeros((WL.T, WL.top_k), dtype=torch.int32, device="cuda")
    out = torch.zeros((WL.T, 16, 512), dtype=torch.float32, device="cuda")
    ws = D.band_workspace(h, WL.T, "cuda")
    D.prefill(h, inp, WL.T, topk, out, ws)
    D.ds4sp_destroy(h)                   # returns after the handle's last event
    assert torch.isfinite(out).all()
