"""Python binding of libds4sp (include/ds4sp.h): argument marshalling only.

Each ``ds4sp_*`` function here calls the C entry point of the same name with the
data pointers of torch tensors and the current CUDA stream. Every step of the
path runs in the library's kernels; there is no fallback. If the library is
missing the first call raises ``Ds4spError``.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Dict, List, Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libds4sp.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "ds4sp.h")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_ORDER, ERR_WORKSPACE, ERR_CUDA, ERR_DEVICE_BOUNDS = range(7)


class Ds4spError(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: {detail} (status {status})")
        self.status = status


class ds4sp_config(ctypes.Structure):
    _fields_ = [("n_heads", ctypes.c_int), ("d_qk", ctypes.c_int), ("d_v", ctypes.c_int),
                ("ratio", ctypes.c_int), ("n_idx_heads", ctypes.c_int), ("d_idx", ctypes.c_int),
                ("top_k", ctypes.c_int), ("n_swa", ctypes.c_int), ("band", ctypes.c_int),
                ("max_tokens", ctypes.c_int), ("softmax_scale", ctypes.c_float),
                ("exp_mode", ctypes.c_int), ("pv_mode", ctypes.c_int),
                ("topk_mode", ctypes.c_int), ("kv_format", ctypes.c_int),
                ("dependent_launch", ctypes.c_int), ("attn_kernel", ctypes.c_int),
                ("indexer_kernel", ctypes.c_int)]


class ds4sp_io(ctypes.Structure):
    _fields_ = [("q", ctypes.c_void_p), ("q_idx", ctypes.c_void_p), ("w", ctypes.c_void_p),
                ("kv_raw", ctypes.c_void_p), ("kv_cmp", ctypes.c_void_p), ("k_idx", ctypes.c_void_p),
                ("topk", ctypes.c_void_p), ("out", ctypes.c_void_p)]


_lib: Optional[ctypes.CDLL] = None
_vp, _i32, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t

_SIGS = {
    "ds4sp_create": (_i32, [ctypes.POINTER(ds4sp_config), ctypes.POINTER(_vp)]),
    "ds4sp_destroy": (_i32, [_vp]),
    "ds4sp_workspace_bytes": (_sz, [_vp, _i32, _i32]),
    "ds4sp_indexer_topk": (_i32, [_vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp, _sz, _vp]),
    "ds4sp_sparse_attn": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _vp, _vp]),
    "ds4sp_prefill_band": (_i32, [_vp, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                  _vp, _sz, _vp]),
    "ds4sp_prefill_host": (_i32, [_vp, _i32, ctypes.POINTER(ds4sp_io), ctypes.POINTER(ds4sp_io),
                                  _vp, _sz, _vp]),
    "ds4sp_reset": (_i32, [_vp, _i32]),
    "ds4sp_next_band": (_i32, [_vp]),
    "ds4sp_device_status": (_i32, [_vp, _vp, ctypes.POINTER(ctypes.c_uint32)]),
    "ds4sp_profile_enable": (_i32, [_vp, _i32]),
    "ds4sp_profile_read": (_i32, [_vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(_i32)]),
    "ds4sp_debug_fail_launches": (_i32, [_vp, _i32]),
    "ds4sp_debug_set_mask": (_i32, [_vp, _vp, _i32, _i32]),
    "ds4sp_debug_set_wait_limit_ns": (_i32, [_vp, ctypes.c_longlong]),
    "ds4sp_indexer_topk_noalloc": (_i32, [ctypes.POINTER(ds4sp_config), _vp, _vp, _vp, _i32,
                                          _i32, _vp, _vp]),
    "ds4sp_kv_row_bytes": (_i32, [_i32, _i32]),
    "ds4sp_quantize_kv": (_i32, [_vp, _i32, _i32, _i32, _vp, _vp]),
    "ds4sp_probe_gather": (_i32, [_vp, _i32, _i32, _vp, _i32, _vp, _i32, _vp]),
    "ds4sp_status_string": (ctypes.c_char_p, [_i32]),
    "ds4sp_last_error": (ctypes.c_char_p, []),
}


def header_symbols(path: str = HEADER) -> List[str]:
    """Function names declared in include/ds4sp.h."""
    with open(path) as f:
        text = f.read()
    return sorted(set(re.findall(r"\b(ds4sp_[a-z_]+)\s*\(", text)))


def load_library(path: Optional[str] = None) -> ctypes.CDLL:
    """Load libds4sp.so (LIB_PATH unless a path is given) and declare every signature.
    Raises if it is missing."""
    global _lib
    path = LIB_PATH if path is None else path
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise Ds4spError(ERR_CUDA, "load_library",
                         f"{path} is missing; build it with python -m sparse_mla_prefill_b200.build")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    if path == LIB_PATH:
        _lib = lib
    return lib


def _check(status: int, where: str) -> None:
    if status != OK:
        lib = load_library()
        detail = lib.ds4sp_last_error().decode() or lib.ds4sp_status_string(status).decode()
        raise Ds4spError(status, where, detail)


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None) -> Optional[int]:
    if t is None:
        return None
    if not t.is_cuda:
        raise Ds4spError(ERR_INVALID_ARG, name, "tensor must be on a CUDA device")
    if not t.is_contiguous():
        raise Ds4spError(ERR_INVALID_ARG, name, "tensor must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise Ds4spError(ERR_INVALID_ARG, name, f"dtype {t.dtype}, expected {dtype}")
    return t.data_ptr()


def _kv_dtype(t) -> torch.dtype:
    """KV tensors are fp16 rows, or uint8 rows of a quantized cache (kv_format 1, 2)."""
    return torch.uint8 if t is not None and t.dtype == torch.uint8 else torch.float16


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


# ------------------------------------------------------------------ handle

class Handle:
    """Owns one ds4sp_handle*; destroy() (or garbage collection) releases it."""

    def __init__(self, ptr: int, cfg: ds4sp_config):
        self.ptr = ptr
        self.cfg = cfg
        self.mask = None       # tensor set by ds4sp_debug_set_mask, kept alive here

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        ds4sp_destroy(self)

    def __del__(self):
        try:
            if self.ptr:
                ds4sp_destroy(self)
        except Exception:
            pass


def make_config(n_idx_heads: int, d_idx: int, top_k: int, n_swa: int, max_tokens: int,
                band: int = 2048, softmax_scale: float = 0.0, n_heads: int = 16, d_qk: int = 576,
                d_v: int = 512, ratio: int = 4, exp_mode: Optional[int] = None,
                pv_mode: int = 0, topk_mode: int = 1, kv_format: int = 0,
                dependent_launch: int = 1, attn_kernel: int = 0,
                indexer_kernel: int = 0) -> ds4sp_config:
    """A ds4sp_config in field order. exp_mode: 0 = ex2.approx, 1 = exp2f for the
    softmax (unset: 1 where the configuration supports it, fp16 rows on the streaming
    kernel, where it measured faster; else 0); pv_mode: 0 = fp16 probabilities in P . V, 1 = fp32-staged (hi + lo fp16);
    topk_mode: 1 (the default) = fused indexer + top-k where the call qualifies, 0 =
    scores in the workspace and a separate top-k kernel; kv_format: 0 = fp16 KV rows, 1 = Q8_0,
    2 = Q4_0, 3 = Q8 K / Q4 V quantized rows (ds4sp_quantize_kv); dependent_launch:
    1 = each kernel a programmatic dependent of the one before it, 0 = plain order;
    attn_kernel: 0 = mma.sync streaming attention, 1 = logits on tcgen05 (TMEM);
    indexer_kernel: 0 = one CTA per tcgen05 tile, 1 = CTA pairs sharing each MMA."""
    if exp_mode is None:
        exp_mode = 1 if kv_format == 0 and attn_kernel == 0 else 0
    return ds4sp_config(n_heads, d_qk, d_v, ratio, n_idx_heads, d_idx, top_k, n_swa, band,
                        max_tokens, softmax_scale, exp_mode, pv_mode, topk_mode, kv_format,
                        dependent_launch, attn_kernel, indexer_kernel)


def ds4sp_create(cfg: ds4sp_config) -> Handle:
    lib = load_library()
    out = ctypes.c_void_p()
    _check(lib.ds4sp_create(ctypes.byref(cfg), ctypes.byref(out)), "ds4sp_create")
    return Handle(out.value, cfg)


def ds4sp_destroy(h: Handle) -> None:
    lib = load_library()
    ptr, h.ptr = h.ptr, None
    if ptr:
        _check(lib.ds4sp_destroy(ptr), "ds4sp_destroy")


def ds4sp_workspace_bytes(h: Handle, t0: int, n_q: int) -> int:
    return int(load_library().ds4sp_workspace_bytes(h.ptr, t0, n_q))


def ds4sp_indexer_topk(h: Handle, q_idx, k_idx, w, t0: int, n_q: int, topk, ws, stream=None):
    lib = load_library()
    _check(lib.ds4sp_indexer_topk(h.ptr, _ptr(q_idx, "q_idx", torch.float16),
                                  _ptr(k_idx, "k_idx", torch.float16),
                                  _ptr(w, "w", torch.float32), t0, n_q,
                                  _ptr(topk, "topk", torch.int32), _ptr(ws, "ws"),
                                  ws.numel() * ws.element_size() if ws is not None else 0,
                                  _stream(stream)), "ds4sp_indexer_topk")


def ds4sp_indexer_topk_noalloc(cfg: ds4sp_config, q_idx, k_idx, w, t0: int, n_q: int, topk,
                               stream=None):
    """Indexer + top-k with the library's fixed 8 MiB score scratch: no handle, no
    workspace, no device allocation (see include/ds4sp.h)."""
    lib = load_library()
    _check(lib.ds4sp_indexer_topk_noalloc(ctypes.byref(cfg), _ptr(q_idx, "q_idx", torch.float16),
                                          _ptr(k_idx, "k_idx", torch.float16),
                                          _ptr(w, "w", torch.float32), t0, n_q,
                                          _ptr(topk, "topk", torch.int32), _stream(stream)),
           "ds4sp_indexer_topk_noalloc")


def ds4sp_sparse_attn(h: Handle, q, kv_raw, kv_cmp, topk, t0: int, n_q: int, out, stream=None):
    lib = load_library()
    _check(lib.ds4sp_sparse_attn(h.ptr, _ptr(q, "q", torch.float16),
                                 _ptr(kv_raw, "kv_raw", _kv_dtype(kv_raw)),
                                 _ptr(kv_cmp, "kv_cmp", _kv_dtype(kv_cmp)),
                                 _ptr(topk, "topk", torch.int32), t0, n_q,
                                 _ptr(out, "out", torch.float32), _stream(stream)),
           "ds4sp_sparse_attn")


def ds4sp_prefill_band(h: Handle, b: int, n_tokens: int, q, q_idx, w, kv_raw, kv_cmp, k_idx,
                       topk, out, ws, stream=None):
    lib = load_library()
    _check(lib.ds4sp_prefill_band(h.ptr, b, n_tokens, _ptr(q, "q", torch.float16),
                                  _ptr(q_idx, "q_idx", torch.float16),
                                  _ptr(w, "w", torch.float32),
                                  _ptr(kv_raw, "kv_raw", _kv_dtype(kv_raw)),
                                  _ptr(kv_cmp, "kv_cmp", _kv_dtype(kv_cmp)),
                                  _ptr(k_idx, "k_idx", torch.float16),
                                  _ptr(topk, "topk", torch.int32),
                                  _ptr(out, "out", torch.float32), _ptr(ws, "ws"),
                                  ws.numel() * ws.element_size() if ws is not None else 0,
                                  _stream(stream)), "ds4sp_prefill_band")


def ds4sp_reset(h: Handle, next_band: int) -> None:
    _check(load_library().ds4sp_reset(h.ptr, next_band), "ds4sp_reset")


def ds4sp_next_band(h: Handle) -> int:
    return int(load_library().ds4sp_next_band(h.ptr))


def ds4sp_device_status(h: Handle, stream=None) -> Tuple[int, int]:
    """(status, raw bits) after synchronising the stream; does not raise on a set bit."""
    bits = ctypes.c_uint32(0)
    st = load_library().ds4sp_device_status(h.ptr, _stream(stream), ctypes.byref(bits))
    if st not in (OK, ERR_DEVICE_BOUNDS):
        _check(st, "ds4sp_device_status")
    return st, bits.value


def ds4sp_profile_enable(h: Handle, enable: bool) -> None:
    _check(load_library().ds4sp_profile_enable(h.ptr, int(enable)), "ds4sp_profile_enable")


def ds4sp_profile_read(h: Handle) -> Dict[str, Tuple[float, int]]:
    ms = (ctypes.c_double * 3)()
    n = (ctypes.c_int * 3)()
    _check(load_library().ds4sp_profile_read(h.ptr, ms, n), "ds4sp_profile_read")
    return {k: (ms[i], n[i]) for i, k in enumerate(("indexer", "topk", "attention"))}


def ds4sp_debug_fail_launches(h: Handle, n: int) -> None:
    _check(load_library().ds4sp_debug_fail_launches(h.ptr, n), "ds4sp_debug_fail_launches")


def ds4sp_debug_set_wait_limit_ns(h: Handle, ns: int) -> None:
    """Limit of the kernels' pipeline waits for this handle's later launches (ns; 0 =
    give up at the first miss; negative = back to the default of about one second)."""
    _check(load_library().ds4sp_debug_set_wait_limit_ns(h.ptr, int(ns)),
           "ds4sp_debug_set_wait_limit_ns")


def ds4sp_debug_set_mask(h: Handle, mask: Optional[torch.Tensor]) -> None:
    """Explicit-mask visibility: ``mask`` is uint8 [rows, cols] on the device (row t,
    column j: compressed row j visible to token t), or None to return to the formula.
    The handle keeps a reference to the tensor while it is set."""
    lib = load_library()
    if mask is None:
        _check(lib.ds4sp_debug_set_mask(h.ptr, None, 0, 0), "ds4sp_debug_set_mask")
        h.mask = None
        return
    if mask.dim() != 2:
        raise Ds4spError(ERR_INVALID_ARG, "mask", "mask must be 2-D [rows, cols]")
    _check(lib.ds4sp_debug_set_mask(h.ptr, _ptr(mask, "mask", torch.uint8), mask.shape[0],
                                    mask.shape[1]), "ds4sp_debug_set_mask")
    h.mask = mask


def ds4sp_kv_row_bytes(kv_format: int, dims: int) -> int:
    return int(load_library().ds4sp_kv_row_bytes(kv_format, dims))


def ds4sp_quantize_kv(x, kv_format: int, out=None, stream=None):
    """Quantize fp16 rows x [rows, dims] (device) into the stored row layout; returns
    ``out`` (uint8 [rows, ds4sp_kv_row_bytes(kv_format, dims)], allocated if None)."""
    rows, dims = x.shape
    rb = ds4sp_kv_row_bytes(kv_format, dims)
    if out is None:
        out = torch.empty((rows, max(rb, 16)), dtype=torch.uint8, device=x.device)
    _check(load_library().ds4sp_quantize_kv(_ptr(x, "x", torch.float16), rows, dims, kv_format,
                                            _ptr(out, "out", torch.uint8), _stream(stream)),
           "ds4sp_quantize_kv")
    return out


def ds4sp_probe_gather(table, idx, sink, grid: int, stream=None) -> None:
    """Row-gather bandwidth probe (measurement helper): reads table[idx[i]] for every i
    (table [rows, row_bytes/2] fp16 or any 2-D tensor with 16-byte-multiple rows) and
    XORs the words into sink (int32 [1])."""
    row_bytes = table.shape[1] * table.element_size()
    _check(load_library().ds4sp_probe_gather(_ptr(table, "table"), table.shape[0], row_bytes,
                                             _ptr(idx, "idx", torch.int32), idx.numel(),
                                             _ptr(sink, "sink", torch.int32), grid,
                                             _stream(stream)), "ds4sp_probe_gather")


def ds4sp_status_string(status: int) -> str:
    return load_library().ds4sp_status_string(status).decode()


def ds4sp_last_error() -> str:
    return load_library().ds4sp_last_error().decode()


# ------------------------------------------------------------------ whole prefill

def band_workspace(h: Handle, n_tokens: int, device) -> torch.Tensor:
    """Scratch large enough for every band of an n_tokens prefill (uint8, 256-aligned)."""
    band = h.cfg.band
    need = max([ds4sp_workspace_bytes(h, b0, min(band, n_tokens - b0))
                for b0 in range(0, n_tokens, band)] + [256])
    return torch.empty(need, dtype=torch.uint8, device=device)


def prefill(h: Handle, inputs: Dict[str, torch.Tensor], n_tokens: int,
            topk: torch.Tensor, out: torch.Tensor, ws: torch.Tensor, stream=None) -> None:
    """All bands of an n_tokens prefill, in order, on device-resident tensors."""
    ds4sp_reset(h, 0)
    for b in range((n_tokens + h.cfg.band - 1) // h.cfg.band):
        ds4sp_prefill_band(h, b, n_tokens, inputs["q"], inputs["q_idx"], inputs["w"],
                           inputs["kv_raw"], inputs["kv_cmp"], inputs["k_idx"], topk, out, ws,
                           stream)


def _io(t: Dict[str, torch.Tensor], topk: Optional[torch.Tensor], out: torch.Tensor,
        pinned: bool) -> ds4sp_io:
    def ptr(name, x, dtype):
        if x is None:
            return None
        if pinned and x.is_cuda:
            raise ValueError(f"{name}: expected a host tensor")
        if not pinned and not x.is_cuda:
            raise ValueError(f"{name}: expected a device tensor")
        if x.dtype != dtype or not x.is_contiguous():
            raise ValueError(f"{name}: expected a contiguous {dtype} tensor")
        return x.data_ptr()
    f16, f32, i32 = torch.float16, torch.float32, torch.int32
    kvt = t["kv_raw"].dtype if t["kv_raw"].dtype == torch.uint8 else f16   # quantized rows
    return ds4sp_io(ptr("q", t["q"], f16), ptr("q_idx", t["q_idx"], f16), ptr("w", t["w"], f32),
                    ptr("kv_raw", t["kv_raw"], kvt), ptr("kv_cmp", t.get("kv_cmp"), kvt),
                    ptr("k_idx", t.get("k_idx"), f16), ptr("topk", topk, i32), ptr("out", out, f32))


def ds4sp_prefill_host(h: Handle, n_tokens: int, host: Dict[str, torch.Tensor],
                       host_topk: Optional[torch.Tensor], host_out: torch.Tensor,
                       dev: Dict[str, torch.Tensor], dev_topk: Optional[torch.Tensor],
                       dev_out: torch.Tensor, ws: Optional[torch.Tensor], stream=None) -> None:
    lib = load_library()
    hio, dio = _io(host, host_topk, host_out, True), _io(dev, dev_topk, dev_out, False)
    _check(lib.ds4sp_prefill_host(h.ptr, n_tokens, ctypes.byref(hio), ctypes.byref(dio),
                                  _ptr(ws, "ws"),
                                  ws.numel() * ws.element_size() if ws is not None else 0,
                                  _stream(stream)), "ds4sp_prefill_host")


def prefill_host(h: Handle, host: Dict[str, torch.Tensor], dev: Dict[str, torch.Tensor],
                 n_tokens: int, topk: torch.Tensor, out: torch.Tensor, ws: torch.Tensor,
                 out_host: torch.Tensor, stream=None, topk_host: Optional[torch.Tensor] = None) -> None:
    """Prefill from host (pinned) inputs into a host output through ds4sp_prefill_host:
    per band, inputs copied in, computed, output copied back, the three overlapped across
    bands. ``dev``, ``topk`` and ``out`` are the device buffers. Asynchronous on the
    stream."""
    s = torch.cuda.current_stream() if stream is None else stream
    ds4sp_prefill_host(h, n_tokens, host, topk_host, out_host, dev, topk, out, ws, s)
