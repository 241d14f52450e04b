"""Seeded synthetic inputs for DS4 sparse-prefill attention.

This module is shared by the CUDA path, the tests and the CPU oracle. It holds
shapes and random draws only: none of the method's arithmetic (no visibility,
no scores, no selection, no softmax) lives here.

Shapes and value distributions follow the workloads of "perf(ds4): extend
sparse prefill scheduling to 10K" (Summary: ratio-4 compressed rows, 2,048-token
bands up to a 10,240-token frontier, F16 latent rows streamed across sixteen
heads) and "perf(ds4): accelerate long context and add PFlash" (Summary:
verifier widths 2..5 at a 122,880-token context). The pages run real prompts;
these seeded tensors stand in for them:

* ``q``      [n_q, 16, 576]  fp16, N(0, 1)      query heads, 512 latent + 64 rope
* ``kv_raw`` [T, 576]        fp16, N(0, 1)      raw latent rows, one per token
* ``kv_cmp`` [T/4, 576]      fp16, N(0, 1)      ratio-4 compressed latent rows
* ``q_idx``  [n_q, H_i, D_i] fp16, integers in [-3, 3]   indexer queries
* ``k_idx``  [T/4, D_i]      fp16, integers in [-3, 3]   indexer keys
* ``w``      [n_q, H_i]      fp32, integers in [0, 3]    indexer head weights

Draw order is fixed (q, kv_raw, kv_cmp, q_idx, k_idx, w) from one
``torch.Generator('cpu')`` seeded with the workload's seed, so every consumer
sees identical bytes. Integer-valued indexer inputs make every indexer score an
exact integer below 2**24, so scores are exact in fp32 whatever the summation
order, and top-k indices can be compared bit for bit.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Dict, Optional

import torch

N_HEADS = 16
D_QK = 576
D_V = 512
RATIO = 4
BAND = 2048


@dataclass(frozen=True)
class Workload:
    """One synthetic workload.

    ``T`` is the number of resident KV tokens. Query tokens are ``[q_start, T)``:
    the whole sequence for prefill workloads, the last ``verify_q`` tokens for
    the long-context verify workload.
    """

    name: str
    T: int
    H_i: int
    D_i: int
    top_k: int
    n_swa: int
    seed: int
    verify_q: Optional[int] = None  # query width for the verify workload
    n_heads: int = N_HEADS
    d_qk: int = D_QK
    d_v: int = D_V
    ratio: int = RATIO
    band: int = BAND

    @property
    def n_c(self) -> int:
        return self.T // self.ratio

    @property
    def q_start(self) -> int:
        return self.T - self.verify_q if self.verify_q else 0

    @property
    def n_q(self) -> int:
        return self.T - self.q_start

    @property
    def n_bands(self) -> int:
        return (self.T + self.band - 1) // self.band


# Per-token tensors of the verify workload are drawn for the last VERIFY_MAX_Q
# positions; width q uses the last q of them.
VERIFY_MAX_Q = 5

WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", T=256, H_i=4, D_i=64, top_k=16, n_swa=32, seed=0),
    "band": Workload("band", T=2048, H_i=64, D_i=128, top_k=128, n_swa=128, seed=1),
    "8k": Workload("8k", T=8192, H_i=64, D_i=128, top_k=512, n_swa=128, seed=2),
    "10k": Workload("10k", T=10240, H_i=64, D_i=128, top_k=512, n_swa=128, seed=3),
    "verify": Workload("verify", T=122880, H_i=64, D_i=128, top_k=512, n_swa=128,
                       seed=4, verify_q=VERIFY_MAX_Q),
}


def workload(name: str, **overrides) -> Workload:
    """Return a named workload, optionally with fields replaced (for edge cases)."""
    w = WORKLOADS[name]
    return replace(w, **overrides) if overrides else w


def generate(wl: Workload) -> Dict[str, torch.Tensor]:
    """Draw the workload's tensors on the CPU in the fixed order.

    Per-token tensors cover query tokens ``[q_start, T)``. For the verify
    workload they are drawn for the last ``VERIFY_MAX_Q`` positions whatever
    ``verify_q`` is, so every width sees the same bytes for the same token.
    """
    g = torch.Generator("cpu").manual_seed(wl.seed)
    n_draw = VERIFY_MAX_Q if wl.verify_q else wl.T
    q = torch.randn(n_draw, wl.n_heads, wl.d_qk, generator=g).half()
    kv_raw = torch.randn(wl.T, wl.d_qk, generator=g).half()
    kv_cmp = torch.randn(wl.n_c, wl.d_qk, generator=g).half()
    q_idx = torch.randint(-3, 4, (n_draw, wl.H_i, wl.D_i), generator=g).half()
    k_idx = torch.randint(-3, 4, (wl.n_c, wl.D_i), generator=g).half()
    w = torch.randint(0, 4, (n_draw, wl.H_i), generator=g).float()
    if wl.verify_q:
        keep = slice(n_draw - wl.verify_q, n_draw)
        q, q_idx, w = q[keep].contiguous(), q_idx[keep].contiguous(), w[keep].contiguous()
    return {"q": q, "kv_raw": kv_raw, "kv_cmp": kv_cmp, "q_idx": q_idx,
            "k_idx": k_idx, "w": w}


def generate_small(T: int, H_i: int, D_i: int, seed: int, n_heads: int = N_HEADS,
                   d_qk: int = D_QK, ratio: int = RATIO,
                   index_range: int = 3, weight_max: int = 3) -> Dict[str, torch.Tensor]:
    """Same recipe at arbitrary small sizes, for edge-case and ragged-tail tests."""
    g = torch.Generator("cpu").manual_seed(seed)
    n_c = T // ratio
    return {
        "q": torch.randn(T, n_heads, d_qk, generator=g).half(),
        "kv_raw": torch.randn(T, d_qk, generator=g).half(),
        "kv_cmp": torch.randn(n_c, d_qk, generator=g).half(),
        "q_idx": torch.randint(-index_range, index_range + 1, (T, H_i, D_i), generator=g).half(),
        "k_idx": torch.randint(-index_range, index_range + 1, (n_c, D_i), generator=g).half(),
        "w": torch.randint(0, weight_max + 1, (T, H_i), generator=g).float(),
    }
