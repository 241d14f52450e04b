"""The kernels' bounded waits give up, report it, and leave the handle usable.

Every pipeline wait inside the kernels has a limit (about one second by default). A
test cannot make a healthy pipeline stall, so it lowers the limit instead:
ds4sp_debug_set_wait_limit_ns(h, 0) makes every wait give up at its first miss. The
2048-token band then runs with waits that give up, in both top-k forms (the fused
indexer + top-k kernel and the two-kernel form): the calls must return, the kernels
must end (the test would hang otherwise), the status word must carry bit 1 (a wait gave
up), and once the default limit is back the next prefill must give the same bits as
the one before, which is itself checked against the oracle on a sample of tokens.
"""
import numpy as np
import pytest
import torch

from gpu_common import (assert_attention_close, handle_for, oracle_tokens, run_prefill,
                        sample_tokens, to_device)
from sparse_mla_prefill_b200 import build as B
from sparse_mla_prefill_b200 import ds4sp as D
from sparse_mla_prefill_b200.inputs import generate, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    B.build()
    D.load_library()


@pytest.mark.parametrize("topk_mode", [0, 1])
def test_wait_give_up_is_reported_and_the_handle_recovers(topk_mode):
    wl = workload("band")
    inp = generate(wl)
    dev = to_device(inp)
    with handle_for(wl, topk_mode=topk_mode) as h:
        topk1, out1 = run_prefill(h, dev, wl.T, wl.top_k)          # asserts status 0
        toks = sample_tokens(wl.T, wl.band, 32, seed=11)
        ref = oracle_tokens({k: v.numpy() for k, v in inp.items()}, toks, wl)
        assert np.array_equal(topk1.cpu().numpy()[toks], ref["topk"])
        assert_attention_close(out1.cpu().numpy()[toks], ref["out"], "before")

        D.ds4sp_debug_set_wait_limit_ns(h, 0)
        topk2 = torch.full_like(topk1, -7)
        out2 = torch.zeros_like(out1)
        ws = D.band_workspace(h, wl.T, "cuda")
        D.prefill(h, dev, wl.T, topk2, out2, ws)                    # returns: launches only
        torch.cuda.synchronize()                                    # and the kernels end
        st, bits = D.ds4sp_device_status(h)
        assert st == D.ERR_DEVICE_BOUNDS and bits & 2, (st, bits)
        st, bits = D.ds4sp_device_status(h)                         # the read cleared it
        assert st == D.OK and bits == 0

        D.ds4sp_debug_set_wait_limit_ns(h, -1)
        topk3, out3 = run_prefill(h, dev, wl.T, wl.top_k)          # asserts status 0
        assert torch.equal(topk3, topk1)
        assert torch.equal(out3, out1)
