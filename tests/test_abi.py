"""The C-ABI library loads, exports every entry point include/q8.h declares, and
rejects bad arguments on the host before launching anything (CPU only: no call
here reaches a kernel, so no GPU is needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "q8.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(q8_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def q8():
    from moe_up_gate_b200 import q8 as m
    m.load()
    return m


def test_header_declares_the_path():
    names = _declared()
    for must in ("q8_pack", "q8_quantize_row", "q8_gemv", "q8_moe_up_gate_swiglu",
                 "q8_mul_mat_id"):
        assert must in names


def test_every_declared_symbol_is_exported(q8):
    lib = q8.load()
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    assert sorted(q8.EXPORTS) == _declared()


def test_scale_stride(q8):
    lib = q8.load()
    assert lib.q8_scale_stride(704) == 24      # 22 scales padded to a multiple of 8
    assert lib.q8_scale_stride(768) == 24
    assert lib.q8_scale_stride(4096) == 128
    assert lib.q8_scale_stride(48) == 0
    assert lib.q8_scale_stride(0) == 0


def test_status_strings(q8):
    lib = q8.load()
    for code in range(8):
        assert lib.q8_status_string(code)
    assert b"unknown" in lib.q8_status_string(99)


FAKE = ctypes.c_void_p(0x10000)      # aligned, non-NULL, never dereferenced
FAKE_ODD = ctypes.c_void_p(0x10001)


def _tensor(q8, k=64, rows=32, n_mat=1, ld_d=None, mat_stride=None, qs=FAKE, d=FAKE):
    ld = (k // 32 + 7) // 8 * 8 if ld_d is None else ld_d
    return q8._Tensor(qs.value if qs else None, d.value if d else None, k, rows, n_mat, ld,
                      rows if mat_stride is None else mat_stride)


def test_quantize_row_validation(q8):
    lib = q8.load()
    assert lib.q8_quantize_row(None, 1, 32, FAKE, FAKE, None) == 1           # NULL
    assert lib.q8_quantize_row(FAKE, 1, 48, FAKE, FAKE, None) == 2           # k % 32
    assert lib.q8_quantize_row(FAKE, 0, 32, FAKE, FAKE, None) == 2           # n_rows
    assert lib.q8_quantize_row(FAKE, 1, 32768, FAKE, FAKE, None) == 2        # k > max
    assert lib.q8_quantize_row(FAKE_ODD, 1, 32, FAKE, FAKE, None) == 3       # alignment
    assert b"16-byte" in lib.q8_last_error()


def test_pack_validation(q8):
    lib = q8.load()
    assert lib.q8_pack(FAKE, 4, 64, FAKE, FAKE, 1, None) == 3                # ld_d < k/32
    assert lib.q8_pack(FAKE, 4, 64, FAKE, FAKE, 4, None) == 3                # ld_d % 8
    assert lib.q8_pack(FAKE, 4, 63, FAKE, FAKE, 8, None) == 2


def test_pack_up_gate_validation(q8):
    lib = q8.load()
    assert lib.q8_pack_up_gate(FAKE, None, 2, 64, 64, FAKE, FAKE, 8, None) == 1       # NULL
    assert lib.q8_pack_up_gate(FAKE, FAKE, 0, 64, 64, FAKE, FAKE, 8, None) == 2       # n_mat
    assert lib.q8_pack_up_gate(FAKE, FAKE, 2, 48, 64, FAKE, FAKE, 8, None) == 2       # n_ff % 32
    assert lib.q8_pack_up_gate(FAKE, FAKE, 2, 64, 63, FAKE, FAKE, 8, None) == 2       # k % 32
    assert lib.q8_pack_up_gate(FAKE, FAKE, 2, 64, 64, FAKE, FAKE, 4, None) == 3       # ld_d % 8
    assert lib.q8_pack_up_gate(FAKE_ODD, FAKE, 2, 64, 64, FAKE, FAKE, 8, None) == 3   # alignment
    assert b"16-byte" in lib.q8_last_error()


def test_gemv_validation(q8):
    lib = q8.load()
    W = _tensor(q8)
    assert lib.q8_gemv(None, FAKE, FAKE, 1, FAKE, None) == 1
    assert lib.q8_gemv(ctypes.byref(_tensor(q8, qs=None)), FAKE, FAKE, 1, FAKE, None) == 1
    assert lib.q8_gemv(ctypes.byref(_tensor(q8, n_mat=2)), FAKE, FAKE, 1, FAKE, None) == 2
    assert lib.q8_gemv(ctypes.byref(_tensor(q8, ld_d=2)), FAKE, FAKE, 1, FAKE, None) == 3
    assert lib.q8_gemv(ctypes.byref(_tensor(q8, mat_stride=8)), FAKE, FAKE, 1, FAKE, None) == 2
    assert lib.q8_gemv(ctypes.byref(W), FAKE_ODD, FAKE, 1, FAKE, None) == 3
    assert lib.q8_gemv(ctypes.byref(W), FAKE, FAKE, 0, FAKE, None) == 2


def test_routed_validation(q8):
    lib = q8.load()
    W = _tensor(q8, k=64, rows=64, n_mat=4)
    ws_need = lib.q8_moe_workspace_size(3, 2, 4)
    assert ws_need >= 256 and ws_need % 256 == 0
    # workspace missing / too small / misaligned
    assert lib.q8_mul_mat_id(ctypes.byref(W), FAKE, FAKE, 1, 3, FAKE, 2, FAKE, None, 0,
                             None) == 7
    assert lib.q8_mul_mat_id(ctypes.byref(W), FAKE, FAKE, 1, 3, FAKE, 2, FAKE, FAKE,
                             ws_need - 1, None) == 7
    assert lib.q8_mul_mat_id(ctypes.byref(W), FAKE, FAKE, 1, 3, FAKE, 2, FAKE,
                             ctypes.c_void_p(0x10010), ws_need, None) == 7
    # ids required for mul_mat_id; n_used limits
    assert lib.q8_mul_mat_id(ctypes.byref(W), FAKE, FAKE, 1, 3, None, 2, FAKE, FAKE, ws_need,
                             None) == 1
    assert lib.q8_mul_mat_id(ctypes.byref(W), FAKE, FAKE, 1, 3, FAKE, 33, FAKE, FAKE, 1 << 20,
                             None) == 2
    # up_gate: rows must be 2*n_ff with n_ff % 32 == 0; dense needs n_mat == 1
    bad_rows = _tensor(q8, k=64, rows=96, n_mat=4)
    assert lib.q8_moe_up_gate_swiglu(ctypes.byref(bad_rows), FAKE, FAKE, 3, FAKE, 2, FAKE, None,
                                     None, None, None, FAKE, ws_need, None) == 2
    assert lib.q8_moe_up_gate_swiglu(ctypes.byref(W), FAKE, FAKE, 3, None, 1, FAKE, None, None,
                                     None, None, None, 0, None) == 2
    # hq and hd go together
    assert lib.q8_moe_up_gate_swiglu(ctypes.byref(W), FAKE, FAKE, 3, FAKE, 2, FAKE, FAKE, None,
                                     None, None, FAKE, ws_need, None) == 1
    # too many experts for the grouping kernel: unsupported, not a silent fallback
    big = _tensor(q8, k=64, rows=64, n_mat=5000)
    assert lib.q8_mul_mat_id(ctypes.byref(big), FAKE, FAKE, 1, 3, FAKE, 2, FAKE, FAKE, 1 << 30,
                             None) == 5


def test_ffn_validation(q8):
    lib = q8.load()
    ug = _tensor(q8, k=64, rows=64, n_mat=4)
    dn = _tensor(q8, k=32, rows=64, n_mat=4)
    need = lib.q8_moe_ffn_workspace_size(2, 2, 4, 64, 32)
    assert need > 0
    # ids without route_w
    assert lib.q8_moe_ffn(ctypes.byref(ug), ctypes.byref(dn), FAKE, 2, FAKE, None, 2, FAKE, FAKE,
                          need, None) == 1
    # down of the wrong shape
    bad = _tensor(q8, k=64, rows=64, n_mat=4)
    assert lib.q8_moe_ffn(ctypes.byref(ug), ctypes.byref(bad), FAKE, 2, FAKE, FAKE, 2, FAKE,
                          FAKE, need, None) == 2
    assert lib.q8_moe_ffn(ctypes.byref(ug), ctypes.byref(dn), FAKE, 2, FAKE, FAKE, 2, FAKE, FAKE,
                          need - 256, None) == 7


def test_gemv_batched_validation(q8):
    lib = q8.load()
    arr = (q8._GemvDesc * 2)()
    arr[0] = q8._GemvDesc(_tensor(q8), FAKE.value, FAKE.value)
    arr[1] = q8._GemvDesc(_tensor(q8, n_mat=3), FAKE.value, FAKE.value)
    assert lib.q8_gemv_batched(arr, 2, 1, None) == 2
    assert lib.q8_gemv_batched(arr, 0, 1, None) == 2
    assert lib.q8_gemv_batched(arr, 129, 1, None) == 2
    arr[1] = q8._GemvDesc(_tensor(q8), FAKE_ODD.value, FAKE.value)
    assert lib.q8_gemv_batched(arr, 2, 1, None) == 3


def test_wait_hook_validation(q8):
    lib = q8.load()
    assert lib.q8_debug_wait_timeout(2, 5_000_000, None, None) == 2     # kind
    assert lib.q8_debug_wait_timeout(0, 10, None, None) == 2            # limit below 1 us
    assert lib.q8_debug_wait_timeout(0, 10**11, None, None) == 2        # limit above 10 s
    assert lib.q8_debug_wait_timeout(1, 5_000_000, None, None) == 1     # no barrier words
    assert lib.q8_debug_wait_timeout(1, 5_000_000, FAKE_ODD, None) == 3


def test_noalloc_scratch_capacity(q8):
    # 128 experts, 8 per token: the grouping tables of 1982 tokens fit the
    # built-in 64 KiB scratch, those of 1983 do not
    lib = q8.load()
    assert lib.q8_moe_workspace_size(1982, 8, 128) <= 65536
    assert lib.q8_moe_workspace_size(1983, 8, 128) > 65536


def test_route_validation(q8):
    lib = q8.load()
    ok = dict(n_tok=2, n_embd=64, n_exp=16, n_used=4)

    def call(w=FAKE, x=FAKE, ids=FAKE, rw=FAKE, lg=None, **kw):
        a = dict(ok, **kw)
        return lib.q8_route(w, x, a["n_tok"], a["n_embd"], a["n_exp"], a["n_used"], ids, rw, lg,
                            None)

    assert call(w=None) == 1
    assert call(ids=None) == 1
    assert call(n_tok=0) == 2
    assert call(n_embd=62) == 2                 # not a multiple of 4
    assert call(n_exp=0) == 2
    assert call(n_exp=1025) == 2                # above Q8_ROUTE_MAX_EXP
    assert call(n_used=17, n_exp=16) == 2       # more than the experts
    assert call(n_used=33, n_exp=64) == 2       # above Q8_MAX_USED
    assert call(x=FAKE_ODD) == 3
    assert call(lg=ctypes.c_void_p(0x10004)) == 3  # logits 8-byte aligned
    # the longest rows with the most experts fit one token per cluster, so no
    # valid shape is refused for its shared-memory plan
