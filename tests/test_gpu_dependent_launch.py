"""Programmatic dependent launch (dependent_launch 1) changes when kernels start, not what
they compute: every kernel waits for its predecessor before it touches global memory.
The whole 10K prefill, a verify width (few-token attention and its merge kernel) and the
fused top-k must give the same bits with it on and off."""
import pytest
import torch

from gpu_common import handle_for, run_prefill, run_range, to_device
from sparse_mla_prefill_b200 import build as B
from sparse_mla_prefill_b200 import ds4sp as D
from sparse_mla_prefill_b200.inputs import generate, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    B.build()
    D.load_library()


@pytest.mark.parametrize("topk_mode", [0, 1])
def test_prefill_same_bits_with_and_without_dependent_launch(topk_mode):
    wl = workload("10k")
    dev = to_device(generate(wl))
    res = []
    for dl in (0, 1):
        with handle_for(wl, dependent_launch=dl, topk_mode=topk_mode) as h:
            res.append(run_prefill(h, dev, wl.T, wl.top_k))
    assert torch.equal(res[0][0], res[1][0])
    assert torch.equal(res[0][1], res[1][1])


def test_verify_width_same_bits_with_and_without_dependent_launch():
    wl = workload("verify")
    inp = generate(wl)
    sl = to_device({k: (v[1:].contiguous() if k in ("q", "q_idx", "w") else v) for k, v in inp.items()})
    res = []
    for dl in (0, 1):
        with handle_for(wl, dependent_launch=dl) as h:
            res.append(run_range(h, sl, wl.T - 4, 4, wl.top_k))
    assert torch.equal(res[0][0], res[1][0])
    assert torch.equal(res[0][1], res[1][1])
