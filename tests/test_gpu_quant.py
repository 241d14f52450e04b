"""Quantized KV cache (kv_format 1 = Q8_0, 2 = Q4_0, 3 = Q8 K / Q4 V) through the C ABI.

ds4sp_quantize_kv must write the oracle's bytes exactly: codes are decided in fp32 on
both sides (IEEE division, half-to-even rounding, the first extreme of Q4_0), and the
layout is fixed. The attention over a quantized cache is compared with
oracle.prefill_tokens_quant (float64 over the exact dequantized values d*q): indices bit
for bit (the indexer does not read the cache), attention within max-abs 2e-3 and NMSE
1e-6. The kernel rounds each dequantized value once to fp16 for the tensor cores, a
relative error of at most 2^-11 per key and value element; with fp16 probabilities
already giving errors near 5e-4 max-abs on these workloads, the same bar holds (the
extra logit error is about scale * sqrt(576) * 2^-12 = 2.4e-4 relative).
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_common import assert_attention_close, handle_for, run_prefill, sample_tokens, to_device
from sparse_mla_prefill_b200 import build as B
from sparse_mla_prefill_b200 import ds4sp as D
from sparse_mla_prefill_b200.inputs import generate, workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_ok):
    B.build()
    D.load_library()


def _special_rows():
    """Rows that hit the rounding ties, the clamps, zero blocks and equal extremes."""
    r = np.zeros((4, 576), np.float32)
    r[0, :8] = [127, -127, 63.5, -63.5, 0.5, 1.5, -0.5, 2.49]
    r[0, 32:36] = [-3, 1.5, 0.75, 0.01]
    r[1, :7] = [-8, 7, 3.5, 2.5, -0.5, 8, 0.25]
    r[1, 32:36] = [4, -2, 1, 0.3]
    r[2, 64:96] = np.arange(32) * 0.25 - 4        # ties at every other step
    r[3] = np.tile([1e-4, -3e-5, 65504, -65504], 144)
    return r.astype(np.float16)


@pytest.mark.parametrize("fmt", [1, 2, 3])
@pytest.mark.parametrize("dims", [576, 512])
def test_quantize_bytes_match_oracle(fmt, dims):
    x = np.concatenate([_special_rows()[:, :dims],
                        generate(workload("band"))["kv_raw"].numpy()[:300, :dims]])
    got = D.ds4sp_quantize_kv(torch.from_numpy(x).cuda(), fmt).cpu().numpy()
    want = oracle.cache_rows(x, fmt)
    assert got.shape == want.shape == (x.shape[0], oracle.quant_row_bytes(fmt, dims))
    if not np.array_equal(got, want):
        bad = np.argwhere(got != want)
        raise AssertionError(f"{len(bad)} bytes differ, first at {bad[0].tolist()}")


def _quantized(dev, fmt):
    q = dict(dev)
    q["kv_raw"] = D.ds4sp_quantize_kv(dev["kv_raw"], fmt)
    q["kv_cmp"] = D.ds4sp_quantize_kv(dev["kv_cmp"], fmt)
    return q


@pytest.mark.parametrize("fmt", [1, 2, 3])
@pytest.mark.parametrize("name", ["tiny", "band"])
def test_quantized_cache_parity(name, fmt):
    wl = workload(name)
    inp = generate(wl)
    dev = _quantized(to_device(inp), fmt)
    with handle_for(wl, kv_format=fmt) as h:
        topk, out = run_prefill(h, dev, wl.T, wl.top_k)
    npi = {k: v.numpy() for k, v in inp.items()}
    ref = oracle.prefill_tokens_quant(npi, range(wl.T), wl.top_k, wl.n_swa, fmt)
    assert np.array_equal(topk.cpu().numpy(), ref["topk"])
    assert_attention_close(out.cpu().numpy(), ref["out"], f"{name} kv_format {fmt}")


def test_quantized_cache_10k_sampled():
    wl = workload("10k")
    inp = generate(wl)
    dev = _quantized(to_device(inp), 2)
    with handle_for(wl, kv_format=2) as h:
        topk, out = run_prefill(h, dev, wl.T, wl.top_k)
    toks = sample_tokens(wl.T, wl.band, 24, seed=31)
    npi = {k: v.numpy() for k, v in inp.items()}
    ref = oracle.prefill_tokens_quant(npi, toks, wl.top_k, wl.n_swa, 2)
    assert np.array_equal(topk.cpu().numpy()[toks], ref["topk"])
    assert_attention_close(out.cpu().numpy()[toks], ref["out"], "10k Q4_0")


def test_quantized_cache_host_path_equals_device_path():
    """ds4sp_prefill_host copies quantized KV rows (336 bytes at Q4_0) and must give the
    device path's bits."""
    wl = workload("band", T=4096)
    g = torch.Generator().manual_seed(77)
    inp = {"q": torch.randn(4096, 16, 576, generator=g).half(),
           "kv_raw": torch.randn(4096, 576, generator=g).half(),
           "kv_cmp": torch.randn(1024, 576, generator=g).half(),
           "q_idx": torch.randint(-3, 4, (4096, 64, 128), generator=g).half(),
           "k_idx": torch.randint(-3, 4, (1024, 128), generator=g).half(),
           "w": torch.randint(0, 4, (4096, 64), generator=g).float()}
    dev = _quantized(to_device(inp), 2)
    with handle_for(wl, kv_format=2) as h:
        topk_d, out_d = run_prefill(h, dev, wl.T, wl.top_k)
        host = {k: v.cpu().pin_memory() for k, v in dev.items()}
        dev2 = {k: torch.empty_like(v) for k, v in dev.items()}
        topk2 = torch.empty_like(topk_d)
        out2 = torch.empty_like(out_d)
        out_h = torch.empty(out_d.shape, dtype=torch.float32).pin_memory()
        ws = D.band_workspace(h, wl.T, "cuda")
        D.prefill_host(h, host, dev2, wl.T, topk2, out2, ws, out_h)
        torch.cuda.synchronize()
        assert D.ds4sp_device_status(h)[0] == D.OK
    assert torch.equal(topk2, topk_d)
    assert torch.equal(out_h, out_d.cpu())


def test_quantized_cache_10k_sampled_split_format():
    """Q8 K / Q4 V on the 10K prefill (its 3-slot ring): sampled tokens against the oracle."""
    wl = workload("10k")
    inp = generate(wl)
    dev = _quantized(to_device(inp), 3)
    with handle_for(wl, kv_format=3) as h:
        topk, out = run_prefill(h, dev, wl.T, wl.top_k)
    toks = sample_tokens(wl.T, wl.band, 16, seed=33)
    npi = {k: v.numpy() for k, v in inp.items()}
    ref = oracle.prefill_tokens_quant(npi, toks, wl.top_k, wl.n_swa, 3)
    assert np.array_equal(topk.cpu().numpy()[toks], ref["topk"])
    assert_attention_close(out.cpu().numpy()[toks], ref["out"], "10k Q8 K / Q4 V")


def test_quantized_format_limits():
    wl = workload("tiny")
    with pytest.raises(D.Ds4spError) as e:
        handle_for(wl, kv_format=1, pv_mode=1)
    assert e.value.status == D.ERR_UNSUPPORTED
    with pytest.raises(D.Ds4spError) as e:
        handle_for(workload("tiny", top_k=1000), kv_format=3)
    assert e.value.status == D.ERR_UNSUPPORTED
    assert D.ds4sp_kv_row_bytes(3, 576) == 912 and D.ds4sp_kv_row_bytes(3, 256) == 0


@pytest.mark.parametrize("fmt", [1, 2, 3])
def test_quantized_cache_few_tokens(fmt):
    """A call of three tokens (the split attention: one work item per 32-row unit, then
    the per-token merge) over each quantized cache, against the oracle."""
    from gpu_common import run_range
    wl = workload("band")
    inp = generate(wl)
    q = 3
    t0 = wl.T - q
    dev = _quantized(to_device({n: (v[t0:] if n in ("q", "q_idx", "w") else v)
                                for n, v in inp.items()}), fmt)
    with handle_for(wl, kv_format=fmt) as h:
        topk, out = run_range(h, dev, t0, q, wl.top_k)
    npi = {k: v.numpy() for k, v in inp.items()}
    ref = oracle.prefill_tokens_quant(npi, range(t0, wl.T), wl.top_k, wl.n_swa, fmt)
    assert np.array_equal(topk.cpu().numpy(), ref["topk"])
    assert_attention_close(out.cpu().numpy(), ref["out"], f"few tokens kv_format {fmt}")
