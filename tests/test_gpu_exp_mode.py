"""Softmax exponentials: ex2.approx (exp_mode 0) against CUDA's exp2f (exp_mode 1, the
binding's default for fp16 rows). Both
must meet the attention tolerance against the float64 oracle on the band workload,
select the same rows, and differ from each other by no more than the tolerance; the
precise mode must not be less accurate than the fast one by more than rounding noise.
The measured errors of both are printed for the report."""
import numpy as np
import pytest

import oracle
from gpu_common import assert_attention_close, handle_for, run_prefill, to_device
from sparse_mla_prefill_b200 import build as B
from sparse_mla_prefill_b200 import ds4sp as D
from sparse_mla_prefill_b200.inputs import generate, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    B.build()
    D.load_library()


def test_fast_and_precise_exponentials():
    wl = workload("band")
    inp = generate(wl)
    dev = to_device(inp)
    ref = oracle.prefill_bands({k: v.numpy() for k, v in inp.items()}, wl.T, wl.top_k,
                               wl.n_swa, band=wl.band)
    outs, errs = {}, {}
    for mode in (0, 1):
        with handle_for(wl, exp_mode=mode) as h:
            topk, out = run_prefill(h, dev, wl.T, wl.top_k)
        assert np.array_equal(topk.cpu().numpy(), ref["topk"]), mode
        outs[mode] = out.cpu().numpy()
        errs[mode] = assert_attention_close(outs[mode], ref["out"], f"exp_mode {mode}")
    print(f"\nexp_mode 0 (ex2.approx): max_abs {errs[0][0]:.3e} nmse {errs[0][1]:.3e}; "
          f"exp_mode 1 (exp2f): max_abs {errs[1][0]:.3e} nmse {errs[1][1]:.3e}")
    assert errs[1][1] <= errs[0][1] * 1.5 + 1e-12
    assert_attention_close(outs[1], outs[0].astype(np.float64), "exp_mode 1 vs 0")
