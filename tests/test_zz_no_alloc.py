"""The allocation-free entry point q8_moe_up_gate_swiglu_noalloc.

Some callers cannot call cudaMalloc (or any allocating routine) where they run
the MoE step -- inside an allocator hook, in a plugin whose host forbids device
allocation, or in a loop that must not touch the allocator -- so libq8 offers a
variant of the routed up/gate + SwiGLU call that takes no workspace and keeps
its expert-grouping tables in a built-in device array.  The tests call it
through the C ABI twice in a row (different token counts and routing ids, so the
second call starts from the first call's leftover scratch contents) and check
each result against the workspace-taking entry point q8_moe_up_gate_swiglu,
within the parity tolerances the other tests use; one case routes 32 tokens to
one expert so that the tensor-core kernel reads its tables from the built-in
scratch.  This file is collected last.
"""
import ctypes

import numpy as np
import pytest
import torch

from helpers import S_norm, TOL, bits, canon_d, host
from moe_up_gate_b200 import q8, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _inputs(n_tok, seed):
    shape = synth.MoeShape(n_embd=2816, n_ff=704, n_exp=128, n_used=8)
    t = synth.moe_layer_tensors(seed, 0, shape, n_tok, 1.0)
    UG = q8.pack(t["up_gate"].to(DEV))
    xq, xd = q8.quantize_row(t["x"].to(DEV))
    return UG, xq, xd, t["ids"].to(DEV)


def test_noalloc_matches_workspace_entry_on_two_calls():
    lib = q8.load()
    for n_tok, seed in ((16, 71), (5, 72)):
        UG, xq, xd, ids = _inputs(n_tok, seed)
        ref = q8.moe_up_gate_swiglu(UG, xq, xd, ids, want_hq=True, want_gu=True)
        n_used, n_ff = 8, 704
        h = torch.full((n_tok, n_used, n_ff), float("nan"), device=DEV)
        g = torch.full_like(h, float("nan"))
        u = torch.full_like(h, float("nan"))
        hq = torch.zeros((n_tok, n_used, n_ff), dtype=torch.int8, device=DEV)
        hd = torch.zeros((n_tok, n_used, n_ff // 32), dtype=torch.float16, device=DEV)
        rc = lib.q8_moe_up_gate_swiglu_noalloc(
            ctypes.byref(UG.c()), ctypes.c_void_p(xq.data_ptr()), ctypes.c_void_p(xd.data_ptr()),
            n_tok, ctypes.c_void_p(ids.data_ptr()), n_used, ctypes.c_void_p(h.data_ptr()),
            ctypes.c_void_p(hq.data_ptr()), ctypes.c_void_p(hd.data_ptr()),
            ctypes.c_void_p(g.data_ptr()), ctypes.c_void_p(u.data_ptr()),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == 0, lib.q8_last_error()
        torch.cuda.synchronize()
        # g and u: the matmul tolerance 1e-5 * sum|w x| per output
        wq = host(UG.qs).reshape(128, 2 * n_ff, 2816)
        wd = canon_d(UG.d, 2816).reshape(128, 2 * n_ff, 88)
        xqh, xdh, idh = host(xq), bits(xd), host(ids)
        for t in range(n_tok):
            for s in range(n_used):
                e = idh[t, s]
                Sg = S_norm(wq[e, :n_ff], wd[e, :n_ff], xqh[t:t + 1], xdh[t:t + 1])[0]
                Su = S_norm(wq[e, n_ff:], wd[e, n_ff:], xqh[t:t + 1], xdh[t:t + 1])[0]
                assert np.all(np.abs(host(g)[t, s] - host(ref["g"])[t, s]) <= TOL * Sg)
                assert np.all(np.abs(host(u)[t, s] - host(ref["u"])[t, s]) <= TOL * Su)
        # h: the SwiGLU tolerance; hq/hd: the quantized stages are bit-exact
        hr = host(ref["h"]).astype(np.float64)
        assert np.all(np.abs(host(h) - hr) <= TOL * (np.abs(hr) + 1e-30))
        assert np.array_equal(host(hq), host(ref["hq"]))
        assert np.array_equal(bits(hd), bits(ref["hd"]))


def _noalloc(lib, UG, xq, xd, ids, h, hq, hd):
    n_tok, n_used = ids.shape
    return lib.q8_moe_up_gate_swiglu_noalloc(
        ctypes.byref(UG.c()), ctypes.c_void_p(xq.data_ptr()), ctypes.c_void_p(xd.data_ptr()),
        n_tok, ctypes.c_void_p(ids.data_ptr()), n_used, ctypes.c_void_p(h.data_ptr()),
        ctypes.c_void_p(hq.data_ptr()), ctypes.c_void_p(hd.data_ptr()), None, None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def test_noalloc_tensor_core_branch():
    """Without the g/u taps, experts with >= 4 routed rows go to the
    tensor-core kernel, which reads the tensor-core list and the pair lists
    from the built-in scratch: slot 0 of all 32 tokens names expert 0.  Two
    calls in a row with different ids; each equals the workspace entry point
    bit for bit (the same kernels on the same tables)."""
    lib = q8.load()
    n_used, n_ff = 8, 704
    for n_tok, seed in ((32, 74), (48, 75)):
        UG, xq, xd, ids = _inputs(n_tok, seed)
        ids = ids.clone()
        for t in range(n_tok):  # expert 0 in slot 0 of every token, ids still distinct
            row = [e for e in ids[t].tolist() if e != 0][: n_used - 1]
            ids[t] = torch.tensor([0] + row, dtype=torch.int32, device=DEV)
        counts = torch.bincount(ids.flatten().long(), minlength=128)
        assert int(counts[0]) == n_tok >= 4
        ref = q8.moe_up_gate_swiglu(UG, xq, xd, ids, want_hq=True)
        h = torch.full((n_tok, n_used, n_ff), float("nan"), device=DEV)
        hq = torch.zeros((n_tok, n_used, n_ff), dtype=torch.int8, device=DEV)
        hd = torch.zeros((n_tok, n_used, n_ff // 32), dtype=torch.float16, device=DEV)
        assert _noalloc(lib, UG, xq, xd, ids, h, hq, hd) == 0, lib.q8_last_error()
        torch.cuda.synchronize()
        assert torch.equal(h, ref["h"])
        assert torch.equal(hq, ref["hq"]) and torch.equal(hd, ref["hd"])


def test_noalloc_rejects_calls_beyond_the_scratch():
    lib = q8.load()
    UG, xq, xd, ids = _inputs(1, 73)
    big_ids = torch.zeros((1984, 8), dtype=torch.int32, device=DEV)
    rc = lib.q8_moe_up_gate_swiglu_noalloc(
        ctypes.byref(UG.c()), ctypes.c_void_p(xq.data_ptr()), ctypes.c_void_p(xd.data_ptr()),
        1984, ctypes.c_void_p(big_ids.data_ptr()), 8, ctypes.c_void_p(xq.data_ptr()), None, None,
        None, None, None)
    assert rc == 7  # Q8_E_WORKSPACE: nothing launched
    assert b"scratch" in lib.q8_last_error()
