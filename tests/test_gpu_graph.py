"""The library's calls inside a CUDA graph: a captured verify step (indexer + top-k +
split attention with its merge) and a captured band of the 2048-token workload, replayed,
give the same bits as the same calls launched directly, and leave the device status
clean."""
import pytest
import torch

from gpu_common import handle_for, to_device
from sparse_mla_prefill_b200 import build as B
from sparse_mla_prefill_b200 import ds4sp as D
from sparse_mla_prefill_b200.inputs import generate, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    B.build()
    D.load_library()


def _step(h, sl, t0, n, topk, out, ws):
    """sl: the per-token tensors (q, q_idx, w) start at token t0; the KV is whole."""
    D.ds4sp_indexer_topk(h, sl["q_idx"], sl["k_idx"], sl["w"], t0, n, topk, ws)
    D.ds4sp_sparse_attn(h, sl["q"], sl["kv_raw"], sl["kv_cmp"], topk, t0, n, out)


def _direct_and_replayed(wl, sl, t0, n, **kw):
    with handle_for(wl, **kw) as h:
        ws = torch.empty(max(D.ds4sp_workspace_bytes(h, t0, n), 256), dtype=torch.uint8,
                         device="cuda")
        topk = torch.full((n, wl.top_k), -7, dtype=torch.int32, device="cuda")
        out = torch.full((n, 16, 512), 7.0, dtype=torch.float32, device="cuda")
        _step(h, sl, t0, n, topk, out, ws)
        torch.cuda.synchronize()
        ref_topk, ref_out = topk.clone(), out.clone()
        topk.fill_(-7)
        out.fill_(7.0)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            _step(h, sl, t0, n, topk, out, ws)
        torch.cuda.synchronize()
        assert (topk == -7).all()                  # capture launches nothing
        for _ in range(3):
            g.replay()
        torch.cuda.synchronize()
        st, bits = D.ds4sp_device_status(h)
        assert st == D.OK, hex(bits)
        del g
        return (ref_topk, ref_out), (topk, out)


@pytest.mark.parametrize("q", [1, 3, 5])
def test_verify_step_in_a_graph(q):
    wl = workload("verify")
    dev = to_device(generate(wl))             # per-token tensors: the last 5 tokens
    sl = {k: (v[5 - q:].contiguous() if k in ("q", "q_idx", "w") else v) for k, v in dev.items()}
    (rt, ro), (gt, go) = _direct_and_replayed(wl, sl, wl.T - q, q)
    assert torch.equal(gt, rt)
    assert torch.equal(go, ro)


@pytest.mark.parametrize("topk_mode", [0, 1])
def test_band_in_a_graph(topk_mode):
    wl = workload("band")
    dev = to_device(generate(wl))
    (rt, ro), (gt, go) = _direct_and_replayed(wl, dev, 0, wl.T, topk_mode=topk_mode)
    assert torch.equal(gt, rt)
    assert torch.equal(go, ro)


def test_verify_graph_replays_follow_new_inputs():
    """A verify step (q = 5: indexer, top-k, split attention and its merge) captured once
    and replayed while the queries change in place: every replay gives the bits of a
    direct call on that replay's inputs (nothing of an earlier replay is reused)."""
    wl = workload("verify")
    dev = to_device(generate(wl))
    q = 5
    t0 = wl.T - q
    sl = {k: (v.clone() if k in ("q", "q_idx", "w") else v) for k, v in dev.items()}
    gen = torch.Generator(device="cuda").manual_seed(11)
    with handle_for(wl) as h:
        ws = torch.empty(max(D.ds4sp_workspace_bytes(h, t0, q), 256), dtype=torch.uint8,
                         device="cuda")
        topk = torch.empty((q, wl.top_k), dtype=torch.int32, device="cuda")
        out = torch.empty((q, 16, 512), dtype=torch.float32, device="cuda")
        g = torch.cuda.CUDAGraph()
        _step(h, sl, t0, q, topk, out, ws)             # warm-up outside the capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g):
            _step(h, sl, t0, q, topk, out, ws)
        torch.cuda.synchronize()
        for r in range(4):
            # new queries in the captured buffers (the rows and index keys stay)
            sl["q"].copy_((torch.randn(sl["q"].shape, generator=gen, device="cuda") * 0.5).half())
            g.replay()
            torch.cuda.synchronize()
            got_t, got_o = topk.clone(), out.clone()
            ref_t = torch.empty_like(topk)
            ref_o = torch.empty_like(out)
            _step(h, sl, t0, q, ref_t, ref_o, ws)
            torch.cuda.synchronize()
            assert torch.equal(got_t, ref_t), r
            assert torch.equal(got_o, ref_o), r
        st, bits = D.ds4sp_device_status(h)
        assert st == D.OK, hex(bits)
        del g
