"""Plain CPU oracle for the Q8_0 decode path and the fused MoE up/gate + SwiGLU step.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference leg may import this package.  The
product library (``moe_up_gate_b200``) never imports it, and this package never
imports the product library: the two share no code.

The Q8_0 arithmetic lives in ``q8_oracle.c`` (plain scalar C, fp64 sums, exact
int32 block dots); this module builds it with gcc, marshals numpy arrays into
it through ctypes and returns numpy arrays.  The router (``router_logits``,
``route``), the step before the path, is plain numpy and Python here.  Layouts are the canonical dense
ones: a Q8_0 tensor is ``qs`` int8 ``[..., rows, k]`` plus ``d`` uint16 (fp16
bits) ``[..., rows, k // 32]``.

Method sources (web pages): "GPUなしで13年前のXeon上でGemma 4 26Bを毎秒5トークンで
実行する" (news.hada.io), sections 「非AVX2ビルドで壊れていた演算パス」 and
「3段階で構成された修正」; "narray-llm" README, section "Llama 2 110M を int8
(Q8_0) で".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "q8_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
           "-fno-fast-math", "-Wall"]

_lock = threading.Lock()
_lib = None

QK = 32


def build(force: bool = False) -> str:
    """Compile q8_oracle.c into liboracle.so next to it (gcc). Returns the path."""
    with _lock:
        if (not force and os.path.exists(_LIB_PATH)
                and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
            return _LIB_PATH
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *_CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB_PATH)
        return _LIB_PATH


def _p(a, ct):
    return a.ctypes.data_as(ctypes.POINTER(ct))


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB_PATH)
        i64, i32 = ctypes.c_int64, ctypes.c_int32
        P = ctypes.POINTER
        L.oracle_fp16_from_fp32.argtypes = [ctypes.c_float]
        L.oracle_fp16_from_fp32.restype = ctypes.c_uint16
        L.oracle_fp32_from_fp16.argtypes = [ctypes.c_uint16]
        L.oracle_fp32_from_fp16.restype = ctypes.c_float
        L.oracle_fp16_from_fp32_n.argtypes = [P(ctypes.c_float), i64, P(ctypes.c_uint16)]
        L.oracle_fp16_from_fp32_n.restype = None
        L.oracle_fp32_from_fp16_n.argtypes = [P(ctypes.c_uint16), i64, P(ctypes.c_float)]
        L.oracle_fp32_from_fp16_n.restype = None
        L.oracle_quantize_rows.argtypes = [P(ctypes.c_float), i64, i64, P(ctypes.c_int8),
                                           P(ctypes.c_uint16)]
        L.oracle_quantize_rows.restype = ctypes.c_int
        L.oracle_block_dot.argtypes = [P(ctypes.c_int8), P(ctypes.c_int8)]
        L.oracle_block_dot.restype = i32
        L.oracle_row_block_dots.argtypes = [P(ctypes.c_int8), P(ctypes.c_int8), i64, P(i32)]
        L.oracle_row_block_dots.restype = None
        L.oracle_gemv.argtypes = [P(ctypes.c_int8), P(ctypes.c_uint16), i64, i64,
                                  P(ctypes.c_int8), P(ctypes.c_uint16), i64, P(ctypes.c_double)]
        L.oracle_gemv.restype = None
        L.oracle_silu.argtypes = [ctypes.c_double]
        L.oracle_silu.restype = ctypes.c_double
        L.oracle_up_gate_swiglu.argtypes = [P(ctypes.c_int8), P(ctypes.c_uint16), i64, i64, i64,
                                            P(ctypes.c_int8), P(ctypes.c_uint16), i64,
                                            ctypes.c_void_p, i64, ctypes.c_void_p,
                                            ctypes.c_void_p, P(ctypes.c_double)]
        L.oracle_up_gate_swiglu.restype = ctypes.c_int
        L.oracle_swiglu.argtypes = [P(ctypes.c_double), P(ctypes.c_double), i64,
                                    P(ctypes.c_double)]
        L.oracle_swiglu.restype = None
        L.oracle_mul_mat_id.argtypes = [P(ctypes.c_int8), P(ctypes.c_uint16), i64, i64, i64,
                                        P(ctypes.c_int8), P(ctypes.c_uint16), ctypes.c_int, i64,
                                        P(i32), i64, P(ctypes.c_double)]
        L.oracle_mul_mat_id.restype = ctypes.c_int
        L.oracle_combine.argtypes = [P(ctypes.c_double), P(ctypes.c_float), i64, i64, i64,
                                     P(ctypes.c_double)]
        L.oracle_combine.restype = None
        L.oracle_dequant_fp64_matmul.argtypes = [P(ctypes.c_int8), P(ctypes.c_uint16), i64, i64,
                                                 P(ctypes.c_int8), P(ctypes.c_uint16), i64,
                                                 P(ctypes.c_double)]
        L.oracle_dequant_fp64_matmul.restype = None
        L.oracle_moe_ffn.argtypes = [P(ctypes.c_int8), P(ctypes.c_uint16), P(ctypes.c_int8),
                                     P(ctypes.c_uint16), i64, i64, i64, P(ctypes.c_float), i64,
                                     ctypes.c_void_p, ctypes.c_void_p, i64,
                                     P(ctypes.c_int8), P(ctypes.c_uint16), P(ctypes.c_double),
                                     P(ctypes.c_float), P(ctypes.c_int8), P(ctypes.c_uint16),
                                     P(ctypes.c_double), P(ctypes.c_double)]
        L.oracle_moe_ffn.restype = ctypes.c_int
        L.oracle_set_num_threads.argtypes = [ctypes.c_int]
        L.oracle_set_num_threads.restype = None
        L.oracle_get_max_threads.argtypes = []
        L.oracle_get_max_threads.restype = ctypes.c_int
        _lib = L
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a, dtype=dtype)
    return a


def _vp(a):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def set_num_threads(n: int) -> None:
    lib().oracle_set_num_threads(int(n))


def max_threads() -> int:
    return int(lib().oracle_get_max_threads())


# --------------------------------------------------------------------------
# fp16
# --------------------------------------------------------------------------
def fp16_from_fp32(f: float) -> int:
    """IEEE binary16 bits of fp32 value f (round to nearest even, subnormals kept)."""
    return int(lib().oracle_fp16_from_fp32(float(np.float32(f))))


def fp32_from_fp16(h: int) -> float:
    return float(lib().oracle_fp32_from_fp16(int(h) & 0xFFFF))


def fp32_from_fp16_array(d: np.ndarray) -> np.ndarray:
    """Element-wise fp32_from_fp16 over an array of fp16 bit patterns."""
    d = _c(d, np.uint16)
    out = np.empty(d.shape, dtype=np.float32)
    lib().oracle_fp32_from_fp16_n(_p(d, ctypes.c_uint16), d.size, _p(out, ctypes.c_float))
    return out


def fp16_from_fp32_array(f: np.ndarray) -> np.ndarray:
    """Element-wise fp16_from_fp32 over an fp32 array; returns uint16 bit patterns."""
    f = _c(f, np.float32)
    out = np.empty(f.shape, dtype=np.uint16)
    lib().oracle_fp16_from_fp32_n(_p(f, ctypes.c_float), f.size, _p(out, ctypes.c_uint16))
    return out


# --------------------------------------------------------------------------
# quantize / dots
# --------------------------------------------------------------------------
def quantize_rows(x: np.ndarray):
    """x fp32 [..., k] -> (q int8 [..., k], d uint16 [..., k/32]) by the Q8_0 rule."""
    x = _c(x, np.float32)
    k = x.shape[-1]
    if k % QK:
        raise ValueError("k must be a multiple of 32")
    n = x.size // k if k else 0
    q = np.empty(x.shape, dtype=np.int8)
    d = np.empty(x.shape[:-1] + (k // QK,), dtype=np.uint16)
    rc = lib().oracle_quantize_rows(_p(x, ctypes.c_float), n, k, _p(q, ctypes.c_int8),
                                    _p(d, ctypes.c_uint16))
    if rc:
        raise ArithmeticError("quantized value outside [-127, 127]")
    return q, d


def block_dot(a: np.ndarray, b: np.ndarray) -> int:
    a = _c(a, np.int8)
    b = _c(b, np.int8)
    assert a.size == QK and b.size == QK
    return int(lib().oracle_block_dot(_p(a, ctypes.c_int8), _p(b, ctypes.c_int8)))


def row_block_dots(qw_row: np.ndarray, qx_row: np.ndarray) -> np.ndarray:
    qw_row = _c(qw_row, np.int8)
    qx_row = _c(qx_row, np.int8)
    k = qw_row.size
    out = np.empty(k // QK, dtype=np.int32)
    lib().oracle_row_block_dots(_p(qw_row, ctypes.c_int8), _p(qx_row, ctypes.c_int8), k,
                                _p(out, ctypes.c_int32))
    return out


def gemv(wq, wd, xq, xd) -> np.ndarray:
    """W [rows, k] Q8_0, x [n_tok, k] Q8_0 -> y fp64 [n_tok, rows]."""
    wq = _c(wq, np.int8)
    wd = _c(wd, np.uint16)
    xq = _c(xq, np.int8).reshape(-1, wq.shape[-1])
    xd = _c(xd, np.uint16).reshape(xq.shape[0], -1)
    rows, k = wq.shape[-2], wq.shape[-1]
    n_tok = xq.shape[0]
    y = np.empty((n_tok, rows), dtype=np.float64)
    lib().oracle_gemv(_p(wq, ctypes.c_int8), _p(wd, ctypes.c_uint16), rows, k,
                      _p(xq, ctypes.c_int8), _p(xd, ctypes.c_uint16), n_tok,
                      _p(y, ctypes.c_double))
    return y


def silu(z: float) -> float:
    return float(lib().oracle_silu(float(z)))


def up_gate_swiglu(wq, wd, xq, xd, ids=None, want_gu=False):
    """up_gate [n_exp, 2*n_ff, n_embd] Q8_0; x [n_tok, n_embd] Q8_0; ids [n_tok, n_used] or None.

    Returns h fp64 [n_tok, n_used, n_ff] (and g, u when want_gu)."""
    wq = _c(wq, np.int8)
    wd = _c(wd, np.uint16)
    if wq.ndim == 2:
        wq = wq[None]
        wd = wd[None]
    n_exp, two_ff, n_embd = wq.shape
    n_ff = two_ff // 2
    xq = _c(xq, np.int8).reshape(-1, n_embd)
    xd = _c(xd, np.uint16).reshape(xq.shape[0], -1)
    n_tok = xq.shape[0]
    if ids is None:
        n_used = 1
        idp = None
    else:
        ids = _c(ids, np.int32).reshape(n_tok, -1)
        n_used = ids.shape[1]
        idp = ids
    h = np.empty((n_tok, n_used, n_ff), dtype=np.float64)
    g = np.empty_like(h) if want_gu else None
    u = np.empty_like(h) if want_gu else None
    rc = lib().oracle_up_gate_swiglu(_p(wq, ctypes.c_int8), _p(wd, ctypes.c_uint16), n_exp, n_ff,
                                     n_embd, _p(xq, ctypes.c_int8), _p(xd, ctypes.c_uint16),
                                     n_tok, _vp(idp), n_used, _vp(g), _vp(u),
                                     _p(h, ctypes.c_double))
    if rc:
        raise ValueError("expert id out of range")
    return (h, g, u) if want_gu else h


def mul_mat_id(wq, wd, aq, ad, ids, a_per_slot: bool):
    """W [n_mat, rows, k]; a [n_tok, n_used, k] (per slot) or [n_tok, k]; ids [n_tok, n_used].

    Returns y fp64 [n_tok, n_used, rows]."""
    wq = _c(wq, np.int8)
    wd = _c(wd, np.uint16)
    n_mat, rows, k = wq.shape
    ids = _c(ids, np.int32)
    n_tok, n_used = ids.shape
    aq = _c(aq, np.int8)
    ad = _c(ad, np.uint16)
    y = np.empty((n_tok, n_used, rows), dtype=np.float64)
    rc = lib().oracle_mul_mat_id(_p(wq, ctypes.c_int8), _p(wd, ctypes.c_uint16), n_mat, rows, k,
                                 _p(aq, ctypes.c_int8), _p(ad, ctypes.c_uint16),
                                 1 if a_per_slot else 0, n_tok, _p(ids, ctypes.c_int32), n_used,
                                 _p(y, ctypes.c_double))
    if rc:
        raise ValueError("expert id out of range")
    return y


def swiglu(g, u) -> np.ndarray:
    """h = silu(g) * u elementwise in fp64 (the C oracle's silu)."""
    g = _c(g, np.float64)
    u = _c(u, np.float64)
    assert g.shape == u.shape
    h = np.empty_like(g)
    lib().oracle_swiglu(_p(g, ctypes.c_double), _p(u, ctypes.c_double), g.size,
                        _p(h, ctypes.c_double))
    return h


def up_gate_swiglu_split(gq, gd, uq, ud, xq, xd, ids=None, want_gu=False):
    """The path with separate gate and up weights (page "GPUなしで13年前のXeon上で
    Gemma 4 26Bを毎秒5トークンで実行する", section 「3段階で構成された修正」):
    g = mul_mat_id(W_gate, x), u = mul_mat_id(W_up, x), h = silu(g) * u.

    gate, up: [n_exp, n_ff, n_embd] Q8_0 each ([n_ff, n_embd] for a dense
    layer); x [n_tok, n_embd] Q8_0; ids [n_tok, n_used] or None (dense: every
    token uses matrix 0).  Returns h fp64 [n_tok, n_used, n_ff] (and g, u
    when want_gu)."""
    gq, gd, uq, ud = (_c(gq, np.int8), _c(gd, np.uint16), _c(uq, np.int8), _c(ud, np.uint16))
    if gq.ndim == 2:
        gq, gd, uq, ud = gq[None], gd[None], uq[None], ud[None]
    assert gq.shape == uq.shape and gd.shape == ud.shape
    n_embd = gq.shape[2]
    xq = _c(xq, np.int8).reshape(-1, n_embd)
    xd = _c(xd, np.uint16).reshape(xq.shape[0], -1)
    n_tok = xq.shape[0]
    ids = (np.zeros((n_tok, 1), np.int32) if ids is None
           else _c(ids, np.int32).reshape(n_tok, -1))
    g = mul_mat_id(gq, gd, xq, xd, ids, a_per_slot=False)
    u = mul_mat_id(uq, ud, xq, xd, ids, a_per_slot=False)
    h = swiglu(g, u)
    return (h, g, u) if want_gu else h


def combine(y, p) -> np.ndarray:
    """y [n_tok, n_used, n_out] (fp64), p [n_tok, n_used] fp32 -> out fp64 [n_tok, n_out]."""
    y = _c(y, np.float64)
    p = _c(p, np.float32)
    n_tok, n_used, n_out = y.shape
    out = np.empty((n_tok, n_out), dtype=np.float64)
    lib().oracle_combine(_p(y, ctypes.c_double), _p(p, ctypes.c_float), n_tok, n_used, n_out,
                         _p(out, ctypes.c_double))
    return out


def dequant_fp64_matmul(wq, wd, xq, xd) -> np.ndarray:
    wq = _c(wq, np.int8)
    wd = _c(wd, np.uint16)
    rows, k = wq.shape
    xq = _c(xq, np.int8).reshape(-1, k)
    xd = _c(xd, np.uint16).reshape(xq.shape[0], -1)
    y = np.empty((xq.shape[0], rows), dtype=np.float64)
    lib().oracle_dequant_fp64_matmul(_p(wq, ctypes.c_int8), _p(wd, ctypes.c_uint16), rows, k,
                                     _p(xq, ctypes.c_int8), _p(xd, ctypes.c_uint16), xq.shape[0],
                                     _p(y, ctypes.c_double))
    return y


def moe_ffn(ugq, ugd, dnq, dnd, x, ids=None, p=None):
    """Whole step from fp32 x: quantize -> up_gate+SwiGLU -> fp32 h -> quantize -> down -> combine.

    ugq [n_exp, 2*n_ff, n_embd], dnq [n_exp, n_embd, n_ff].  ids/p [n_tok, n_used] or None (dense).
    Returns dict with out fp64 [n_tok, n_embd] and the intermediates."""
    ugq = _c(ugq, np.int8)
    ugd = _c(ugd, np.uint16)
    dnq = _c(dnq, np.int8)
    dnd = _c(dnd, np.uint16)
    if ugq.ndim == 2:
        ugq, ugd, dnq, dnd = ugq[None], ugd[None], dnq[None], dnd[None]
    n_exp, two_ff, n_embd = ugq.shape
    n_ff = two_ff // 2
    x = _c(x, np.float32).reshape(-1, n_embd)
    n_tok = x.shape[0]
    if ids is None:
        n_used = 1
    else:
        ids = _c(ids, np.int32).reshape(n_tok, -1)
        n_used = ids.shape[1]
    if p is not None:
        p = _c(p, np.float32).reshape(n_tok, n_used)
    xq = np.empty((n_tok, n_embd), np.int8)
    xd = np.empty((n_tok, n_embd // QK), np.uint16)
    h = np.empty((n_tok, n_used, n_ff), np.float64)
    hf = np.empty((n_tok, n_used, n_ff), np.float32)
    hq = np.empty((n_tok, n_used, n_ff), np.int8)
    hd = np.empty((n_tok, n_used, n_ff // QK), np.uint16)
    y = np.empty((n_tok, n_used, n_embd), np.float64)
    out = np.empty((n_tok, n_embd), np.float64)
    rc = lib().oracle_moe_ffn(_p(ugq, ctypes.c_int8), _p(ugd, ctypes.c_uint16),
                              _p(dnq, ctypes.c_int8), _p(dnd, ctypes.c_uint16), n_exp, n_embd,
                              n_ff, _p(x, ctypes.c_float), n_tok, _vp(ids), _vp(p), n_used,
                              _p(xq, ctypes.c_int8), _p(xd, ctypes.c_uint16),
                              _p(h, ctypes.c_double), _p(hf, ctypes.c_float),
                              _p(hq, ctypes.c_int8), _p(hd, ctypes.c_uint16),
                              _p(y, ctypes.c_double), _p(out, ctypes.c_double))
    if rc:
        raise ValueError("oracle_moe_ffn: bad id or quantization range")
    return dict(out=out, xq=xq, xd=xd, h=h, hf=hf, hq=hq, hd=hd, y=y)


# --------------------------------------------------------------------------
# Router (the step before the path: ids and routing weights from logits).
# The pages name MoE routing only as a run-time option ("CPU-aware MoE
# routing"); the reading here is the plain top-k router: fp32 router weights
# (not quantized), logits in fp64, the n_used largest logits per token in
# descending order with equal logits taken by ascending expert index, and the
# routing weights a softmax over the selected logits only.  Plain numpy and
# Python loops: test infrastructure for small cases.
# --------------------------------------------------------------------------
def router_logits(w_router, x) -> np.ndarray:
    """w_router fp32 [n_exp, n_embd], x fp32 [n_tok, n_embd] -> logits fp64 [n_tok, n_exp]."""
    w = np.asarray(w_router, dtype=np.float64)
    xx = np.asarray(x, dtype=np.float64).reshape(-1, w.shape[1])
    return xx @ w.T


def route(logits, n_used: int):
    """logits [n_tok, n_exp] -> (ids int32 [n_tok, n_used], p fp64 [n_tok, n_used]).

    ids[t] lists the n_used experts with the largest logits, largest first;
    equal logits go by ascending expert index.  p[t] = softmax of the selected
    logits (the largest subtracted before exp)."""
    lg = np.asarray(logits, dtype=np.float64)
    n_tok, n_exp = lg.shape
    assert 1 <= n_used <= n_exp
    ids = np.empty((n_tok, n_used), np.int32)
    p = np.empty((n_tok, n_used), np.float64)
    for t in range(n_tok):
        order = sorted(range(n_exp), key=lambda e: (-lg[t, e], e))[:n_used]
        sel = lg[t, order]
        ex = np.exp(sel - sel[0])
        ids[t] = order
        p[t] = ex / ex.sum()
    return ids, p
