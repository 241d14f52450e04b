"""Host-side pieces of bench.py, on CPU: the algorithmic byte and FLOP counts behind the
roofline (against closed forms), the sampled parity check (passes on the oracle's own
result, fails on a planted error), the rule that an ncu traffic figure is used only
for the kernel sources it was captured on, and that every configuration the bench times
is one the library accepts."""
import hashlib

import numpy as np

import bench
import oracle
from sparse_mla_prefill_b200.inputs import generate, workload


def test_algorithmic_counts_match_closed_forms():
    # T = 10240 = 4q, q = 2560: sum_t floor((t+1)/4) = sum_{m=1}^{4q} floor(m/4) = 2q^2 - q.
    q = 2560
    sum_vis = 2 * q * q - q
    # selected rows: floor(m/4) summed for m = 1 .. 2047 (below k = 512), then 512 for
    # each of the 8,193 tokens with m >= 2048; window rows: 1 + ... + 128, then 128 each.
    sel = (2 * 512 * 512 - 512) - 512 + 512 * (10240 - 2047)
    win = 128 * 129 // 2 + 128 * (10240 - 128)
    rows = sel + win
    a = bench.algorithmic(workload("10k"))
    assert a["rows"] == rows == 6_020_672
    assert a["indexer_flops"] == 2 * 64 * 128 * sum_vis == 214_706_421_760
    assert a["attention_bytes"] == 1152 * rows + (16 * 576 * 2 + 16 * 512 * 4 + 4 * 512) * 10240
    assert a["attention_bytes"] == 7_481_073_664
    assert a["attention_flops"] == 2 * 16 * (576 + 512) * rows
    assert a["topk_bytes"] == 4 * sum_vis + 4 * 512 * 10240 == 73_390_080


def test_sampled_parity_passes_the_oracle_and_catches_errors():
    wl = workload("tiny")
    inp = {k: v.numpy() for k, v in generate(wl).items()}
    line, ref = bench.cpu_oracle_sample(wl, 64, inp, return_result=True)
    assert line["kind"] == "oracle" and line["value"] > 0
    full = oracle.prefill_bands(inp, wl.T, wl.top_k, wl.n_swa, band=wl.band)
    out = full["out"].astype(np.float32)
    ok = bench.sampled_parity(ref, full["topk"], out)
    assert ok["pass"] and ok["topk_bit_exact"] and ok["tokens"] == len(ref["tokens"])
    bad = out.copy()
    bad[ref["tokens"][5], 3, 7] += 0.01                  # one element off by 1e-2
    assert not bench.sampled_parity(ref, full["topk"], bad)["pass"]
    tk = full["topk"].copy()
    t = int(ref["tokens"][-1])
    tk[t, 0], tk[t, 1] = tk[t, 1], tk[t, 0]             # same set, wrong order
    r = bench.sampled_parity(ref, tk, out)
    assert not r["topk_bit_exact"] and not r["pass"]


def test_traffic_figure_needs_matching_kernel_sources(tmp_path, monkeypatch):
    root = tmp_path / "repo"
    csrc = root / "sparse_mla_prefill_b200" / "csrc"
    (root / "profiles").mkdir(parents=True)
    csrc.mkdir(parents=True)
    for f in ("sparse_attn_mma.cuh", "device_common.cuh"):
        (csrc / f).write_text(f"// {f}\n")
    sha = hashlib.sha256(b"".join((csrc / f).read_bytes()
                                  for f in ("sparse_attn_mma.cuh", "device_common.cuh")))
    prof = root / "profiles" / "sparse_attn_mma_kernel_10k_band4.md"
    prof.write_text(f"kernel_source_sha256: {sha.hexdigest()[:16]}\n"
                    "traffic_bytes_per_launch: 123456\n")
    monkeypatch.setattr(bench, "ROOT", str(root))
    assert bench.attention_traffic() == 123456
    (csrc / "sparse_attn_mma.cuh").write_text("// changed\n")
    assert bench.attention_traffic() is None


def test_every_variant_is_an_accepted_configuration():
    """Each configuration bench.py times (the headline, the two-kernel pass and every
    entry of VARIANTS) passes ds4sp_create's checks. Without a GPU, create reports a
    CUDA error once the configuration is accepted and a validation status otherwise."""
    import ctypes

    from sparse_mla_prefill_b200 import ds4sp as D
    lib = D.load_library()
    wl = workload("10k")
    base = dict(n_idx_heads=wl.H_i, d_idx=wl.D_i, top_k=wl.top_k, n_swa=wl.n_swa,
                max_tokens=wl.T, band=wl.band)
    configs = [("headline", {}), ("two-kernel pass", dict(topk_mode=0))] + list(bench.VARIANTS)
    for name, modes in configs:
        cfg = D.make_config(**base, **modes)
        out = ctypes.c_void_p()
        st = lib.ds4sp_create(ctypes.byref(cfg), ctypes.byref(out))
        assert st not in (D.ERR_INVALID_ARG, D.ERR_UNSUPPORTED), (name, modes, st)
        if st == D.OK:                       # a GPU is present: the handle is real
            lib.ds4sp_destroy(out)
