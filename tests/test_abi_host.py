"""The C-ABI library builds, loads and exports every declared symbol; argument
checks that need no device run on the CPU."""
import ctypes
import subprocess

import pytest

from sparse_mla_prefill_b200 import build as B
from sparse_mla_prefill_b200 import ds4sp as D


@pytest.fixture(scope="module")
def lib():
    B.build()
    return D.load_library()


def test_library_exports_every_header_symbol(lib):
    names = D.header_symbols()
    assert len(names) >= 14
    nm = subprocess.run(["nm", "-D", "--defined-only", B.LIB], capture_output=True, text=True).stdout
    exported = {ln.split()[-1] for ln in nm.splitlines() if ln.strip()}
    for n in names:
        assert n in exported, n
        assert hasattr(lib, n), n
    # the binding wraps each of them under the same name
    for n in names:
        assert callable(getattr(D, n)), n


def test_build_targets_sm100a_only():
    flags = " ".join(B.NVCC_FLAGS)
    assert "arch=compute_100a,code=sm_100a" in flags
    assert "sm_90" not in flags and "compute_90" not in flags


def _cfg(**kw):
    base = dict(n_idx_heads=64, d_idx=128, top_k=512, n_swa=128, max_tokens=10240)
    base.update(kw)
    return D.make_config(**base)


@pytest.mark.parametrize("kw,status", [
    (dict(n_heads=8), D.ERR_UNSUPPORTED),
    (dict(d_qk=512), D.ERR_UNSUPPORTED),
    (dict(d_v=576), D.ERR_UNSUPPORTED),
    (dict(ratio=2), D.ERR_UNSUPPORTED),
    (dict(d_idx=96), D.ERR_UNSUPPORTED),
    (dict(n_idx_heads=48), D.ERR_UNSUPPORTED),
    (dict(n_idx_heads=2), D.ERR_UNSUPPORTED),
    (dict(top_k=-1), D.ERR_INVALID_ARG),
    (dict(top_k=2049), D.ERR_UNSUPPORTED),
    (dict(n_swa=0), D.ERR_INVALID_ARG),
    (dict(band=0), D.ERR_INVALID_ARG),
    (dict(max_tokens=0), D.ERR_INVALID_ARG),
    (dict(max_tokens=(1 << 24) + 1), D.ERR_INVALID_ARG),
    (dict(softmax_scale=float("nan")), D.ERR_INVALID_ARG),
    (dict(exp_mode=2), D.ERR_INVALID_ARG),
    (dict(pv_mode=2), D.ERR_INVALID_ARG),
    (dict(pv_mode=-1), D.ERR_INVALID_ARG),
    (dict(topk_mode=2), D.ERR_INVALID_ARG),
    (dict(kv_format=4), D.ERR_INVALID_ARG),
    (dict(kv_format=1, exp_mode=1), D.ERR_UNSUPPORTED),
    (dict(kv_format=3, top_k=900), D.ERR_UNSUPPORTED),
    (dict(dependent_launch=2), D.ERR_INVALID_ARG),
    (dict(attn_kernel=2), D.ERR_INVALID_ARG),
    (dict(indexer_kernel=2), D.ERR_INVALID_ARG),
    (dict(attn_kernel=1, kv_format=2), D.ERR_UNSUPPORTED),
])
def test_create_rejects_bad_config_before_touching_the_device(lib, kw, status):
    out = ctypes.c_void_p(123)
    st = lib.ds4sp_create(ctypes.byref(_cfg(**kw)), ctypes.byref(out))
    assert st == status
    assert out.value is None
    assert lib.ds4sp_last_error()


def test_binding_defaults():
    """make_config's defaults: the fused indexer + top-k, and exp2f for the softmax where
    the configuration runs it (fp16 rows on the streaming kernel), else ex2.approx, so
    that every default configuration is one ds4sp_create accepts."""
    base = dict(n_idx_heads=64, d_idx=128, top_k=512, n_swa=128, max_tokens=10240)
    c = D.make_config(**base)
    assert c.topk_mode == 1 and c.exp_mode == 1 and c.pv_mode == 0 and c.kv_format == 0
    for kv in (1, 2, 3):
        assert D.make_config(**base, kv_format=kv).exp_mode == 0
    assert D.make_config(**base, attn_kernel=1).exp_mode == 0
    assert D.make_config(**base, exp_mode=0).exp_mode == 0          # explicit wins
    assert D.make_config(**base, topk_mode=0).topk_mode == 0


def test_null_handle_paths(lib):
    assert lib.ds4sp_destroy(None) == D.OK
    assert lib.ds4sp_workspace_bytes(None, 0, 10) == 0
    assert lib.ds4sp_next_band(None) == -1
    assert lib.ds4sp_reset(None, 0) == D.ERR_INVALID_ARG
    assert lib.ds4sp_create(None, None) == D.ERR_INVALID_ARG
    for fn in ("ds4sp_profile_enable", "ds4sp_debug_fail_launches"):
        assert getattr(lib, fn)(None, 1) == D.ERR_INVALID_ARG
    io = D.ds4sp_io()
    assert lib.ds4sp_prefill_host(None, 16, ctypes.byref(io), ctypes.byref(io), None, 0,
                                  None) == D.ERR_INVALID_ARG
    assert lib.ds4sp_debug_set_mask(None, None, 0, 0) == D.ERR_INVALID_ARG
    assert lib.ds4sp_debug_set_mask(None, 256, 16, 4) == D.ERR_INVALID_ARG


def test_status_strings(lib):
    for s in range(7):
        assert D.ds4sp_status_string(s)
    assert D.ds4sp_status_string(99) == "unknown status"


def test_missing_library_fails_loudly(tmp_path):
    with pytest.raises(D.Ds4spError):
        D.load_library(str(tmp_path / "libds4sp.so"))
