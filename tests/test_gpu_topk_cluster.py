"""Top-k of a few tokens with long rows (topk_cluster_kernel: a cluster of CTAs per token,
the histograms and counts combined through distributed shared memory) against the
oracle: indices bit for bit, and the attention that follows them."""
import numpy as np
import pytest

import oracle
from gpu_common import assert_attention_close, handle_for, oracle_tokens, run_range, to_device
from sparse_mla_prefill_b200 import build as B
from sparse_mla_prefill_b200 import ds4sp as D
from sparse_mla_prefill_b200.inputs import Workload, generate_small

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    B.build()
    D.load_library()


def _np(inp):
    return {k: v.numpy() for k, v in inp.items()}


@pytest.mark.parametrize("T,q,k,weight_max", [
    (20000, 1, 512, 3),      # 4,999 candidates
    (20000, 4, 64, 3),       # four tokens, small k
    (24577, 3, 1000, 3),     # ragged per-CTA ranges
    (20000, 2, 512, 0),      # every score equal: the k lowest rows
])
def test_few_tokens_long_rows(T, q, k, weight_max):
    wl = Workload("long", T=T, H_i=64, D_i=128, top_k=k, n_swa=16, seed=T + q, band=2048)
    inp = generate_small(T, 64, 128, seed=T + 3 * q, weight_max=weight_max)
    t0 = T - q
    dev = to_device({n: (v[t0:] if n in ("q", "q_idx", "w") else v) for n, v in inp.items()})
    with handle_for(wl) as h:
        topk, out = run_range(h, dev, t0, q, k)
    ref = oracle_tokens(_np(inp), range(t0, T), wl)
    assert np.array_equal(topk.cpu().numpy(), ref["topk"])
    if weight_max == 0:
        assert (ref["topk"] == np.arange(k)).all()
    assert_attention_close(out.cpu().numpy(), ref["out"], f"cluster top-k T={T} q={q}")
