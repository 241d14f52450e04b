"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare it with the CPU oracle on the same seeded inputs."""
from __future__ import annotations

from typing import Dict, Iterable, Optional

import numpy as np
import torch

import oracle
from sparse_mla_prefill_b200 import ds4sp as D
from sparse_mla_prefill_b200.inputs import Workload

# Attention tolerance (fp16 rows and probabilities, fp32 accumulation) against the
# float64 oracle, over all compared elements.
MAX_ABS = 2e-3
NMSE = 1e-6


def to_device(inputs: Dict[str, torch.Tensor]) -> Dict[str, torch.Tensor]:
    return {k: v.cuda().contiguous() for k, v in inputs.items()}


def handle_for(wl: Workload, max_tokens: Optional[int] = None, **kw) -> D.Handle:
    cfg = D.make_config(n_idx_heads=wl.H_i, d_idx=wl.D_i, top_k=wl.top_k, n_swa=wl.n_swa,
                        max_tokens=max_tokens or wl.T, band=wl.band, **kw)
    return D.ds4sp_create(cfg)


def run_prefill(h: D.Handle, dev: Dict[str, torch.Tensor], T: int, top_k: int):
    """All bands through ds4sp_prefill_band; returns (topk, out) on the device."""
    topk = torch.full((T, top_k), -7, dtype=torch.int32, device="cuda") if top_k > 0 else None
    out = torch.full((T, 16, 512), float("nan"), dtype=torch.float32, device="cuda")
    ws = D.band_workspace(h, T, "cuda")
    D.prefill(h, dev, T, topk, out, ws)
    torch.cuda.synchronize()
    st, bits = D.ds4sp_device_status(h)
    assert st == D.OK, f"device status bits {bits:#x}"
    return topk, out


def run_range(h: D.Handle, dev: Dict[str, torch.Tensor], t0: int, n_q: int, top_k: int):
    """ds4sp_indexer_topk + ds4sp_sparse_attn on tokens [t0, t0+n_q); per-token
    device tensors in ``dev`` start at token t0."""
    topk = torch.full((n_q, top_k), -7, dtype=torch.int32, device="cuda") if top_k > 0 else None
    out = torch.full((n_q, 16, 512), float("nan"), dtype=torch.float32, device="cuda")
    if top_k > 0:
        ws = torch.empty(max(D.ds4sp_workspace_bytes(h, t0, n_q), 256), dtype=torch.uint8,
                         device="cuda")
        D.ds4sp_indexer_topk(h, dev["q_idx"], dev["k_idx"], dev["w"], t0, n_q, topk, ws)
    D.ds4sp_sparse_attn(h, dev["q"], dev["kv_raw"], dev["kv_cmp"], topk, t0, n_q, out)
    torch.cuda.synchronize()
    st, bits = D.ds4sp_device_status(h)
    assert st == D.OK, f"device status bits {bits:#x}"
    return topk, out


def oracle_tokens(inputs_np: Dict[str, np.ndarray], tokens: Iterable[int], wl: Workload,
                  q_start: int = 0, scale: Optional[float] = None):
    return oracle.prefill_tokens(inputs_np, tokens, wl.top_k, wl.n_swa, q_start=q_start,
                                 scale=scale)


def assert_attention_close(got: np.ndarray, ref: np.ndarray, what: str = ""):
    got = np.asarray(got, dtype=np.float64)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = got - ref
    max_abs = float(np.abs(err).max()) if err.size else 0.0
    nmse = float((err ** 2).sum() / max((ref ** 2).sum(), 1e-300)) if err.size else 0.0
    assert max_abs <= MAX_ABS and nmse <= NMSE, f"{what}: max_abs {max_abs:.3e} nmse {nmse:.3e}"
    return max_abs, nmse


def sample_tokens(T: int, band: int, n_random: int, seed: int):
    """Band edges, the first tokens and a seeded random sample."""
    rng = np.random.default_rng(seed)
    edges = {0, 1, 2, 3, 4, 7, T - 1}
    for b0 in range(0, T, band):
        edges |= {b0, b0 + 1, min(T - 1, b0 + band - 1)}
    picks = set(rng.choice(T, size=min(n_random, T), replace=False).tolist())
    return sorted(t for t in edges | picks if 0 <= t < T)
