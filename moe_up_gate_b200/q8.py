"""Thin Python binding of libq8 (include/q8.h): argument marshalling only.

Every step of the path runs in the CUDA kernels of libq8.so; this module
allocates outputs and workspaces with torch (device memory), passes raw
pointers and the current torch CUDA stream through ctypes, and raises
``Q8Error`` on any non-OK status.  There is no CPU path: without the built
library or a CUDA device the calls fail loudly.
"""
from __future__ import annotations

import ctypes
import os
import threading
from dataclasses import dataclass

import torch

from . import build as _build

QK = 32
_lock = threading.Lock()
_lib = None

STATUS = {0: "Q8_OK", 1: "Q8_E_NULL", 2: "Q8_E_SHAPE", 3: "Q8_E_ALIGN", 4: "Q8_E_BAD_ID",
          5: "Q8_E_UNSUPPORTED", 6: "Q8_E_CUDA", 7: "Q8_E_WORKSPACE"}


class Q8Error(RuntimeError):
    def __init__(self, status: int, where: str, detail: str):
        super().__init__(f"{where}: {STATUS.get(status, status)}: {detail}")
        self.status = status
        self.name = STATUS.get(status, str(status))


class _Tensor(ctypes.Structure):
    _fields_ = [("qs", ctypes.c_void_p), ("d", ctypes.c_void_p), ("k", ctypes.c_int64),
                ("rows", ctypes.c_int64), ("n_mat", ctypes.c_int64), ("ld_d", ctypes.c_int64),
                ("mat_stride", ctypes.c_int64)]


class _GemvDesc(ctypes.Structure):
    _fields_ = [("W", _Tensor), ("x", ctypes.c_void_p), ("y", ctypes.c_void_p)]


EXPORTS = ["q8_scale_stride", "q8_pack", "q8_pack_up_gate", "q8_quantize_row", "q8_gemv",
           "q8_gemv_batched", "q8_moe_workspace_size", "q8_moe_up_gate_swiglu", "q8_mul_mat_id", "q8_moe_combine",
           "q8_moe_ffn_workspace_size", "q8_moe_ffn", "q8_check", "q8_debug_block_dots",
           "q8_status_string", "q8_last_error", "q8_moe_group",
           "q8_moe_up_gate_swiglu_pregrouped", "q8_mul_mat_id_pregrouped",
           "q8_moe_up_gate_swiglu_noalloc", "q8_moe_up_gate_swiglu_fp32", "q8_mul_mat_id_fp32",
           "q8_reset_errors", "q8_debug_wait_timeout", "q8_route"]


def lib_path() -> str:
    return _build.LIB


def load(auto_build: bool = True):
    """Load libq8.so (building it with nvcc first if it is missing or stale)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if auto_build and not _build.up_to_date():
            _build.build()
        if not os.path.exists(_build.LIB):
            raise RuntimeError(f"libq8.so is not built ({_build.LIB}); run "
                               "python -m moe_up_gate_b200.build")
        L = ctypes.CDLL(_build.LIB)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
        st = ctypes.c_int
        P = ctypes.POINTER
        sig = {
            "q8_scale_stride": (i64, [i64]),
            "q8_pack": (st, [vp, i64, i64, vp, vp, i64, vp]),
            "q8_pack_up_gate": (st, [vp, vp, i64, i64, i64, vp, vp, i64, vp]),
            "q8_quantize_row": (st, [vp, i64, i64, vp, vp, vp]),
            "q8_gemv": (st, [P(_Tensor), vp, vp, i64, vp, vp]),
            "q8_gemv_batched": (st, [P(_GemvDesc), i32, i64, vp]),
            "q8_moe_workspace_size": (sz, [i64, i32, i64]),
            "q8_moe_up_gate_swiglu": (st, [P(_Tensor), vp, vp, i64, vp, i32, vp, vp, vp, vp, vp,
                                           vp, sz, vp]),
            "q8_mul_mat_id": (st, [P(_Tensor), vp, vp, i32, i64, vp, i32, vp, vp, sz, vp]),
            "q8_moe_combine": (st, [vp, vp, i64, i32, i64, vp, vp]),
            "q8_moe_ffn_workspace_size": (sz, [i64, i32, i64, i64, i64]),
            "q8_moe_ffn": (st, [P(_Tensor), P(_Tensor), vp, i64, vp, vp, i32, vp, vp, sz, vp]),
            "q8_check": (st, [vp, vp]),
            "q8_debug_block_dots": (st, [P(_Tensor), i64, vp, i64, vp, vp, vp]),
            "q8_moe_group": (st, [vp, i64, i32, i64, vp, sz, vp]),
            "q8_moe_up_gate_swiglu_pregrouped": (st, [P(_Tensor), vp, vp, i64, i32, vp, vp, vp,
                                                      vp, vp, vp, sz, vp]),
            "q8_mul_mat_id_pregrouped": (st, [P(_Tensor), vp, vp, i32, i64, i32, vp, vp, sz,
                                              vp]),
            "q8_moe_up_gate_swiglu_noalloc": (st, [P(_Tensor), vp, vp, i64, vp, i32, vp, vp, vp,
                                                   vp, vp, vp]),
            "q8_moe_up_gate_swiglu_fp32": (st, [P(_Tensor), vp, i64, vp, i32, vp, vp, vp]),
            "q8_mul_mat_id_fp32": (st, [P(_Tensor), vp, i32, i64, vp, i32, vp, vp, vp]),
            "q8_reset_errors": (st, []),
            "q8_route": (st, [vp, vp, i64, i64, i64, i32, vp, vp, vp, vp]),
            "q8_debug_wait_timeout": (st, [i32, i64, vp, vp]),
            "q8_status_string": (ctypes.c_char_p, [st]),
            "q8_last_error": (ctypes.c_char_p, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
        return _lib


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _call(name, *args):
    L = load()
    rc = getattr(L, name)(*args)
    if rc != 0:
        raise Q8Error(rc, name, L.q8_last_error().decode(errors="replace"))


# --------------------------------------------------------------------------
# packed weights
# --------------------------------------------------------------------------
@dataclass
class Q8Tensor:
    """A packed Q8_0 weight tensor on the device (or a view of one).

    qs: int8 storage; d: float16 storage holding the fp16 scales; element
    (m, r, i) at qs[(m*mat_stride + r)*k + i] relative to ``qs_offset`` bytes,
    scale (m, r, b) at d[(m*mat_stride + r)*ld_d + b] relative to ``d_offset``."""
    qs: torch.Tensor
    d: torch.Tensor
    k: int
    rows: int
    n_mat: int
    ld_d: int
    mat_stride: int
    qs_offset: int = 0
    d_offset: int = 0

    def c(self) -> _Tensor:
        return _Tensor(self.qs.data_ptr() + self.qs_offset, self.d.data_ptr() + self.d_offset,
                       self.k, self.rows, self.n_mat, self.ld_d, self.mat_stride)

    def row_view(self, first_row: int, rows: int) -> "Q8Tensor":
        """Rows [first_row, first_row + rows) of every matrix, without a copy (view_3d)."""
        return Q8Tensor(self.qs, self.d, self.k, rows, self.n_mat, self.ld_d, self.mat_stride,
                        self.qs_offset + first_row * self.k,
                        self.d_offset + first_row * self.ld_d * 2)

    def gate(self) -> "Q8Tensor":
        return self.row_view(0, self.rows // 2)

    def up(self) -> "Q8Tensor":
        return self.row_view(self.rows // 2, self.rows // 2)

    @property
    def nbytes_q8(self) -> int:
        """Algorithmic bytes: 34 per 32 weights of the viewed rows."""
        return self.n_mat * self.rows * self.k // QK * 34


def scale_stride(k: int) -> int:
    return int(load().q8_scale_stride(k))


def pack(w: torch.Tensor, stream=None) -> Q8Tensor:
    """fp32 weights [rows, k] or [n_mat, rows, k] (CUDA) -> packed Q8_0 tensor."""
    assert w.is_cuda and w.dtype == torch.float32
    w = w.contiguous()
    if w.dim() == 2:
        n_mat, rows, k = 1, w.shape[0], w.shape[1]
    else:
        n_mat, rows, k = w.shape
    ld = scale_stride(k)
    if ld == 0:
        raise Q8Error(2, "pack", f"k={k} must be a positive multiple of 32")
    qs = torch.empty((n_mat * rows, k), dtype=torch.int8, device=w.device)
    d = torch.empty((n_mat * rows, ld), dtype=torch.float16, device=w.device)
    _call("q8_pack", _ptr(w), n_mat * rows, k, _ptr(qs), _ptr(d), ld, _stream(stream))
    return Q8Tensor(qs, d, k, rows, n_mat, ld, rows)


def pack_up_gate(w_gate: torch.Tensor, w_up: torch.Tensor, stream=None) -> Q8Tensor:
    """Separate fp32 gate and up weights, [n_ff, k] or [n_mat, n_ff, k] each (CUDA)
    -> the combined packed up/gate tensor (gate rows first in every matrix)."""
    assert w_gate.is_cuda and w_gate.dtype == torch.float32 and w_up.shape == w_gate.shape
    assert w_up.is_cuda and w_up.dtype == torch.float32
    w_gate, w_up = w_gate.contiguous(), w_up.contiguous()
    if w_gate.dim() == 2:
        n_mat, n_ff, k = 1, w_gate.shape[0], w_gate.shape[1]
    else:
        n_mat, n_ff, k = w_gate.shape
    ld = scale_stride(k)
    if ld == 0:
        raise Q8Error(2, "pack_up_gate", f"k={k} must be a positive multiple of 32")
    qs = torch.empty((n_mat * 2 * n_ff, k), dtype=torch.int8, device=w_gate.device)
    d = torch.empty((n_mat * 2 * n_ff, ld), dtype=torch.float16, device=w_gate.device)
    _call("q8_pack_up_gate", _ptr(w_gate), _ptr(w_up), n_mat, n_ff, k, _ptr(qs), _ptr(d), ld,
          _stream(stream))
    return Q8Tensor(qs, d, k, 2 * n_ff, n_mat, ld, 2 * n_ff)


def quantize_row(x: torch.Tensor, stream=None):
    """fp32 [n_rows, k] -> (qs int8 [n_rows, k], d float16 [n_rows, k/32])."""
    assert x.is_cuda and x.dtype == torch.float32
    x = x.contiguous()
    k = x.shape[-1]
    n = x.numel() // k
    qs = torch.empty(x.shape, dtype=torch.int8, device=x.device)
    d = torch.empty(x.shape[:-1] + (k // QK,), dtype=torch.float16, device=x.device)
    _call("q8_quantize_row", _ptr(x), n, k, _ptr(qs), _ptr(d), _stream(stream))
    return qs, d


def gemv(W: Q8Tensor, xq: torch.Tensor, xd: torch.Tensor, y: torch.Tensor | None = None,
         stream=None) -> torch.Tensor:
    n_tok = xq.numel() // W.k
    if y is None:
        y = torch.empty((n_tok, W.rows), dtype=torch.float32, device=xq.device)
    _call("q8_gemv", ctypes.byref(W.c()), _ptr(xq), _ptr(xd), n_tok, _ptr(y), _stream(stream))
    return y


def gemv_batched(problems, n_tok: int = 1, stream=None):
    """problems: list of (Q8Tensor, x fp32 [n_tok, k], y fp32 [n_tok, rows]) on the device."""
    arr = (_GemvDesc * len(problems))()
    for i, (W, x, y) in enumerate(problems):
        arr[i] = _GemvDesc(W.c(), x.data_ptr(), y.data_ptr())
    _call("q8_gemv_batched", arr, len(problems), n_tok, _stream(stream))


def moe_workspace(n_tok: int, n_used: int, n_mat: int, device="cuda") -> torch.Tensor:
    nbytes = int(load().q8_moe_workspace_size(n_tok, n_used, n_mat))
    return torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)


def moe_up_gate_swiglu(W: Q8Tensor, xq, xd, ids=None, want_hq=True, want_gu=False, ws=None,
                       out=None, stream=None):
    """Fused up/gate + SwiGLU.  Returns dict with h [n_tok, n_used, n_ff] (+ hq, hd, g, u)."""
    n_tok = xq.shape[0]
    n_used = 1 if ids is None else ids.shape[1]
    n_ff = W.rows // 2
    dev = xq.device
    o = out or {}
    h = o.get("h")
    if h is None:
        h = torch.empty((n_tok, n_used, n_ff), dtype=torch.float32, device=dev)
    hq = hd = g = u = None
    if want_hq:
        hq = o.get("hq")
        hd = o.get("hd")
        if hq is None:
            hq = torch.empty((n_tok, n_used, n_ff), dtype=torch.int8, device=dev)
            hd = torch.empty((n_tok, n_used, n_ff // QK), dtype=torch.float16, device=dev)
    if want_gu:
        g = torch.empty_like(h)
        u = torch.empty_like(h)
    if ids is not None and ws is None:
        ws = moe_workspace(n_tok, n_used, W.n_mat, dev)
    _call("q8_moe_up_gate_swiglu", ctypes.byref(W.c()), _ptr(xq), _ptr(xd), n_tok, _ptr(ids),
          n_used, _ptr(h), _ptr(hq), _ptr(hd), _ptr(g), _ptr(u), _ptr(ws),
          0 if ws is None else ws.numel(), _stream(stream))
    return dict(h=h, hq=hq, hd=hd, g=g, u=u, ws=ws)


def moe_up_gate_swiglu_noalloc(W: Q8Tensor, xq, xd, ids, h, hq=None, hd=None, g=None, u=None,
                               stream=None):
    """Routed up/gate + SwiGLU into caller-provided outputs, with no workspace
    (the grouping tables live in libq8's built-in device scratch)."""
    _call("q8_moe_up_gate_swiglu_noalloc", ctypes.byref(W.c()), _ptr(xq), _ptr(xd),
          xq.shape[0], _ptr(ids), ids.shape[1], _ptr(h), _ptr(hq), _ptr(hd), _ptr(g), _ptr(u),
          _stream(stream))
    return h


def moe_up_gate_swiglu_fp32(W: Q8Tensor, x, ids=None, h=None, err_word=None, stream=None):
    """Up/gate + SwiGLU from fp32 x (quantized in the kernel), small batches, no workspace."""
    n_tok = x.shape[0]
    n_used = 1 if ids is None else ids.shape[1]
    if h is None:
        h = torch.empty((n_tok, n_used, W.rows // 2), dtype=torch.float32, device=x.device)
    _call("q8_moe_up_gate_swiglu_fp32", ctypes.byref(W.c()), _ptr(x), n_tok, _ptr(ids), n_used,
          _ptr(h), _ptr(err_word), _stream(stream))
    return h


def mul_mat_id_fp32(W: Q8Tensor, a, ids, a_per_slot: bool, y=None, err_word=None, stream=None):
    """mul_mat_id from fp32 activations (quantized in the kernel), small batches."""
    n_tok, n_used = ids.shape
    if y is None:
        y = torch.empty((n_tok, n_used, W.rows), dtype=torch.float32, device=a.device)
    _call("q8_mul_mat_id_fp32", ctypes.byref(W.c()), _ptr(a), 1 if a_per_slot else 0, n_tok,
          _ptr(ids), n_used, _ptr(y), _ptr(err_word), _stream(stream))
    return y


def mul_mat_id(W: Q8Tensor, aq, ad, ids, a_per_slot: bool, ws=None, y=None, stream=None):
    n_tok, n_used = ids.shape
    dev = aq.device
    if y is None:
        y = torch.empty((n_tok, n_used, W.rows), dtype=torch.float32, device=dev)
    if ws is None:
        ws = moe_workspace(n_tok, n_used, W.n_mat, dev)
    _call("q8_mul_mat_id", ctypes.byref(W.c()), _ptr(aq), _ptr(ad), 1 if a_per_slot else 0,
          n_tok, _ptr(ids), n_used, _ptr(y), _ptr(ws), ws.numel(), _stream(stream))
    return y


def moe_group(ids, n_mat: int, ws=None, stream=None):
    """Expert grouping tables for ids [n_tok, n_used] into ws (allocated if None)."""
    n_tok, n_used = ids.shape
    if ws is None:
        ws = moe_workspace(n_tok, n_used, n_mat, ids.device)
    _call("q8_moe_group", _ptr(ids), n_tok, n_used, n_mat, _ptr(ws), ws.numel(), _stream(stream))
    return ws


def moe_up_gate_swiglu_pregrouped(W: Q8Tensor, xq, xd, n_used: int, ws, h, hq=None, hd=None,
                                  g=None, u=None, stream=None):
    _call("q8_moe_up_gate_swiglu_pregrouped", ctypes.byref(W.c()), _ptr(xq), _ptr(xd),
          xq.shape[0], n_used, _ptr(h), _ptr(hq), _ptr(hd), _ptr(g), _ptr(u), _ptr(ws),
          ws.numel(), _stream(stream))
    return h


def mul_mat_id_pregrouped(W: Q8Tensor, aq, ad, n_tok: int, n_used: int, a_per_slot: bool, ws,
                          y, stream=None):
    _call("q8_mul_mat_id_pregrouped", ctypes.byref(W.c()), _ptr(aq), _ptr(ad),
          1 if a_per_slot else 0, n_tok, n_used, _ptr(y), _ptr(ws), ws.numel(), _stream(stream))
    return y


def moe_combine(y, route_w, out=None, stream=None):
    n_tok, n_used, n_out = y.shape
    if out is None:
        out = torch.empty((n_tok, n_out), dtype=torch.float32, device=y.device)
    _call("q8_moe_combine", _ptr(y), _ptr(route_w), n_tok, n_used, n_out, _ptr(out),
          _stream(stream))
    return out


def moe_ffn_workspace(n_tok, n_used, n_mat, n_embd, n_ff, device="cuda") -> torch.Tensor:
    nbytes = int(load().q8_moe_ffn_workspace_size(n_tok, n_used, n_mat, n_embd, n_ff))
    return torch.zeros(nbytes, dtype=torch.uint8, device=device)  # zero before first use


def moe_ffn(up_gate: Q8Tensor, down: Q8Tensor, x, ids=None, route_w=None, ws=None, out=None,
            stream=None):
    n_tok = x.shape[0]
    n_used = 1 if ids is None else ids.shape[1]
    if ws is None:
        ws = moe_ffn_workspace(n_tok, n_used, up_gate.n_mat, up_gate.k, up_gate.rows // 2,
                               x.device)
    if out is None:
        out = torch.empty((n_tok, up_gate.k), dtype=torch.float32, device=x.device)
    _call("q8_moe_ffn", ctypes.byref(up_gate.c()), ctypes.byref(down.c()), _ptr(x), n_tok,
          _ptr(ids), _ptr(route_w), n_used, _ptr(out), _ptr(ws), ws.numel(), _stream(stream))
    return out


def check(ws, stream=None):
    _call("q8_check", _ptr(ws), _stream(stream))


def route(w_router, x, n_used: int, want_logits=False, ids=None, route_w=None, stream=None):
    """Router: fp32 w_router [n_exp, n_embd], x [n_tok, n_embd] -> (ids int32
    [n_tok, n_used], route_w fp32 [n_tok, n_used][, logits fp64 [n_tok, n_exp]])."""
    n_tok, n_embd = x.shape
    n_exp = w_router.shape[0]
    if ids is None:
        ids = torch.empty((n_tok, n_used), dtype=torch.int32, device=x.device)
    if route_w is None:
        route_w = torch.empty((n_tok, n_used), dtype=torch.float32, device=x.device)
    logits = (torch.empty((n_tok, n_exp), dtype=torch.float64, device=x.device)
              if want_logits else None)
    _call("q8_route", _ptr(w_router), _ptr(x), n_tok, n_embd, n_exp, n_used, _ptr(ids),
          _ptr(route_w), _ptr(logits), _stream(stream))
    return (ids, route_w, logits) if want_logits else (ids, route_w)


def reset_errors():
    """Clear the wait-timeout flags q8_check reports (no kernel may be running)."""
    _call("q8_reset_errors")


def debug_wait_timeout(kind: int, limit_ns: int, bar=None, stream=None):
    """Test hook: one bounded wait that must give up after limit_ns (kind 0: a
    shared-memory ring wait; kind 1: the grid barrier, bar = 2 zeroed int32 words)."""
    _call("q8_debug_wait_timeout", kind, limit_ns, _ptr(bar), _stream(stream))


def debug_block_dots(W: Q8Tensor, mat: int, rows: torch.Tensor, xq: torch.Tensor, stream=None):
    isum = torch.empty((rows.numel(), W.k // QK), dtype=torch.int32, device=xq.device)
    _call("q8_debug_block_dots", ctypes.byref(W.c()), mat, _ptr(rows), rows.numel(), _ptr(xq),
          _ptr(isum), _stream(stream))
    return isum
