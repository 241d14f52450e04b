"""The CPU oracle against its pins (no GPU)."""
import numpy as np
import pytest

import oracle
import oracle_pins as P
from sparse_mla_prefill_b200.inputs import generate, workload


@pytest.mark.parametrize("pin", P.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(pin):
    pin(oracle)


def test_scores_exact_on_tiny_workload():
    inp = {k: v.numpy() for k, v in generate(workload("tiny")).items()}
    P.pin_scores_exact(oracle, inp)
    P.pin_scores_relu_identities(oracle, inp, tokens=range(0, 256, 7))


def test_scores_exact_on_band_workload_sample():
    inp = {k: v.numpy() for k, v in generate(workload("band")).items()}
    toks = [0, 3, 4, 7, 511, 1024, 2046, 2047]
    P.pin_scores_exact(oracle, inp, toks)
    P.pin_scores_relu_identities(oracle, inp, toks)


def test_scores_fit_fp32_exactly():
    # |score| <= H_i * 3 * (9 * D_i) at the largest workload; below 2**24 every
    # integer is exact in fp32, so any summation order gives the same bits.
    wl = workload("10k")
    assert wl.H_i * 3 * 9 * wl.D_i < 2 ** 24


def test_topk_edge_cases():
    assert oracle.topk_row(np.array([]), 4).tolist() == [-1, -1, -1, -1]
    assert oracle.topk_row(np.array([1.0, 2.0]), 0).tolist() == []
    assert oracle.topk_row(np.zeros(10), 3).tolist() == [0, 1, 2]
    assert oracle.topk_row(np.array([-1.0, -5.0, -1.0]), 2).tolist() == [0, 2]
    assert oracle.topk_row(np.array([3.0, 1.0, 2.0]), 5).tolist() == [0, 1, 2, -1, -1]


def test_n_sel_and_window_edges():
    assert [oracle.n_sel(t, 2) for t in range(12)] == [0, 0, 0, 1, 1, 1, 1, 2, 2, 2, 2, 2]
    assert oracle.window(0, 128).tolist() == [0]
    assert oracle.window(5, 3).tolist() == [3, 4, 5]
    assert oracle.window(5, 100).tolist() == list(range(6))
