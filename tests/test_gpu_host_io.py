"""ds4sp_prefill_host: the whole prefill from pinned host buffers to host buffers, in
steps of about 1,024 tokens with the copies overlapped, must give exactly what the
device-resident band path gives (same kernels, same inputs), including an uneven last
band, small remainders, no top-k, and a call queued behind other work on the stream."""
import numpy as np
import pytest
import torch

from gpu_common import handle_for, run_prefill, to_device
from sparse_mla_prefill_b200 import build as B
from sparse_mla_prefill_b200 import ds4sp as D
from sparse_mla_prefill_b200.inputs import Workload, generate_small

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    B.build()
    D.load_library()


def _host_run(h, host, T, top_k, stream=None):
    dev = {k: torch.empty_like(v, device="cuda") for k, v in host.items()}
    topk = torch.empty((T, top_k), dtype=torch.int32, device="cuda") if top_k > 0 else None
    out = torch.empty((T, 16, 512), dtype=torch.float32, device="cuda")
    ws = D.band_workspace(h, T, "cuda")
    out_h = torch.full((T, 16, 512), float("nan"), dtype=torch.float32).pin_memory()
    topk_h = torch.full((T, top_k), -7, dtype=torch.int32).pin_memory() if top_k > 0 else None
    D.prefill_host(h, host, dev, T, topk, out, ws, out_h, stream=stream, topk_host=topk_h)
    (stream or torch.cuda.current_stream()).synchronize()
    st, bits = D.ds4sp_device_status(h)
    assert st == D.OK, f"device status bits {bits:#x}"
    return topk_h, out_h


@pytest.mark.parametrize("T,top_k,band", [(600, 32, 256), (1024, 64, 256), (300, 0, 128),
                                          (2048, 128, 2048),
                                          # 1,024-token steps: a 40-token last step,
                                          # an 18-token remainder folded into the step
                                          # before it, a 20-token band (few-token
                                          # attention on both paths)
                                          (3112, 64, 2048), (3090, 128, 2048),
                                          (2068, 32, 2048)])
def test_host_path_matches_device_path(T, top_k, band):
    wl = Workload("host", T=T, H_i=8, D_i=64, top_k=top_k, n_swa=32, seed=3, band=band)
    inp = generate_small(T, wl.H_i, wl.D_i, seed=11)
    host = {k: v.contiguous().pin_memory() for k, v in inp.items()}
    h = handle_for(wl)
    try:
        topk_d, out_d = run_prefill(h, to_device(inp), T, top_k)
        topk_h, out_h = _host_run(h, host, T, top_k)
        assert D.ds4sp_next_band(h) == (T + band - 1) // band
    finally:
        D.ds4sp_destroy(h)
    assert np.array_equal(out_h.numpy(), out_d.cpu().numpy())
    if top_k > 0:
        assert np.array_equal(topk_h.numpy(), topk_d.cpu().numpy())


def test_host_path_orders_after_queued_work():
    """Host inputs are read only after earlier work on the stream: a device->host copy
    queued first fills the pinned q the call then reads."""
    T = 512
    wl = Workload("host", T=T, H_i=8, D_i=64, top_k=32, n_swa=32, seed=3, band=256)
    inp = generate_small(T, wl.H_i, wl.D_i, seed=12)
    host = {k: v.contiguous().pin_memory() for k, v in inp.items()}
    q_dev = host["q"].cuda()
    host["q"].zero_()                      # wrong until the queued copy restores it
    s = torch.cuda.Stream()
    h = handle_for(wl)
    try:
        topk_d, out_d = run_prefill(h, to_device(inp), T, wl.top_k)
        torch.cuda.current_stream().synchronize()
        with torch.cuda.stream(s):
            torch.cuda._sleep(20_000_000)  # keep the stream busy before the copy
            host["q"].copy_(q_dev, non_blocking=True)
        _, out_h = _host_run(h, host, T, wl.top_k, stream=s)
    finally:
        D.ds4sp_destroy(h)
    assert np.array_equal(out_h.numpy(), out_d.cpu().numpy())


def test_host_path_rejects_bad_arguments():
    T = 256
    wl = Workload("host", T=T, H_i=8, D_i=64, top_k=32, n_swa=32, seed=3, band=128)
    inp = generate_small(T, wl.H_i, wl.D_i, seed=13)
    host = {k: v.contiguous().pin_memory() for k, v in inp.items()}
    dev = to_device(inp)
    h = handle_for(wl)
    try:
        out = torch.empty((T, 16, 512), dtype=torch.float32, device="cuda")
        out_h = torch.empty((T, 16, 512), dtype=torch.float32).pin_memory()
        ws = D.band_workspace(h, T, "cuda")
        with pytest.raises(D.Ds4spError) as e:        # top-k buffer missing on the device
            D.ds4sp_prefill_host(h, T, host, None, out_h, dev, None, out, ws)
        assert e.value.status == D.ERR_INVALID_ARG
        topk = torch.empty((T, wl.top_k), dtype=torch.int32, device="cuda")
        with pytest.raises(D.Ds4spError) as e:        # too many tokens
            D.ds4sp_prefill_host(h, T + 1, host, None, out_h, dev, topk, out, ws)
        assert e.value.status == D.ERR_INVALID_ARG
        small = torch.empty(16, dtype=torch.uint8, device="cuda")
        with pytest.raises(D.Ds4spError) as e:        # workspace too small
            D.ds4sp_prefill_host(h, T, host, None, out_h, dev, topk, out, small)
        assert e.value.status == D.ERR_WORKSPACE
    finally:
        D.ds4sp_destroy(h)
