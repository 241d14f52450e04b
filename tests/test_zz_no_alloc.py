"""ds4sp_indexer_topk_noalloc: indexer + top-k for callers that cannot allocate device
memory (a framework that reserves all device memory for its own allocator, or a loop
that cannot afford the device synchronisation cudaMalloc/cudaFree may cause).

The entry point takes no handle and no workspace: its score scratch is a fixed 8 MiB
array inside the library. These checks call it through the C ABI twice in a row, on
two different token ranges, and compare each result with ds4sp_indexer_topk (the
entry point with a caller-owned workspace). Indices must match bit for bit, the same
bar as every other index comparison here. A range larger than the array is rejected
before any launch.
"""
import pytest
import torch

from sparse_mla_prefill_b200 import build as B
from sparse_mla_prefill_b200 import ds4sp as D
from sparse_mla_prefill_b200.inputs import generate, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    B.build()
    D.load_library()


def _cfg(wl):
    return D.make_config(n_idx_heads=wl.H_i, d_idx=wl.D_i, top_k=wl.top_k, n_swa=wl.n_swa,
                         max_tokens=wl.T, band=wl.band)


def _with_workspace(wl, dev, t0, n_q):
    topk = torch.full((n_q, wl.top_k), -7, dtype=torch.int32, device="cuda")
    with D.ds4sp_create(_cfg(wl)) as h:
        ws = torch.empty(D.ds4sp_workspace_bytes(h, t0, n_q), dtype=torch.uint8, device="cuda")
        D.ds4sp_indexer_topk(h, dev["q_idx"][t0:t0 + n_q], dev["k_idx"], dev["w"][t0:t0 + n_q],
                             t0, n_q, topk, ws)
        torch.cuda.synchronize()
        assert D.ds4sp_device_status(h)[0] == D.OK
    return topk


def _static(wl, dev, t0, n_q):
    topk = torch.full((n_q, wl.top_k), -9, dtype=torch.int32, device="cuda")
    D.ds4sp_indexer_topk_noalloc(_cfg(wl), dev["q_idx"][t0:t0 + n_q], dev["k_idx"],
                                 dev["w"][t0:t0 + n_q], t0, n_q, topk)
    torch.cuda.synchronize()
    return topk


def test_static_scratch_matches_workspace_path_on_two_calls():
    # first call: the whole 2048-token band workload (2048 x 512 scores)
    wl1 = workload("band")
    dev1 = {k: v.cuda() for k, v in generate(wl1).items()}
    got1 = _static(wl1, dev1, 0, wl1.T)
    assert torch.equal(got1, _with_workspace(wl1, dev1, 0, wl1.T))

    # second call, straight after: band 1 of the 8K prefill, 2048 tokens x 1024 scores,
    # which fills the 2^21-float array exactly and overwrites the first call's scores
    wl2 = workload("8k")
    dev2 = {k: v.cuda() for k, v in generate(wl2).items()}
    got2 = _static(wl2, dev2, 2048, 2048)
    assert torch.equal(got2, _with_workspace(wl2, dev2, 2048, 2048))
    assert (got2 >= 0).all()                  # every token of that band selects 512 rows

    # the first range again gives the same bits (no state survives between calls)
    assert torch.equal(_static(wl1, dev1, 0, wl1.T), got1)


def test_range_beyond_static_scratch_is_rejected():
    wl = workload("8k")
    dev = {k: v.cuda() for k, v in generate(wl).items()}
    topk = torch.zeros((2048, wl.top_k), dtype=torch.int32, device="cuda")
    with pytest.raises(D.Ds4spError) as e:
        D.ds4sp_indexer_topk_noalloc(_cfg(wl), dev["q_idx"][4096:6144], dev["k_idx"],
                                     dev["w"][4096:6144], 4096, 2048, topk)
    assert e.value.status == D.ERR_WORKSPACE
    assert "static scratch" in str(e.value)
    torch.cuda.synchronize()
    assert (topk == 0).all()                  # rejected before any launch
