"""The pins are sharp enough: plausible mistakes planted in a copy of the oracle fail them.

Each case copies oracle/q8_oracle.c to a temporary directory, applies one
textual mistake (a tie rule, a constant, a swapped half, a dropped block, a
wrong index, a sign), compiles it with gcc and runs the relevant pins against
the mutant.  The committed oracle is never modified.  CPU only.
"""
import importlib.util
import json
import os
import shutil
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "q8_oracle.c")
GOLDEN = os.path.join(ROOT, "tests", "golden", "q8_worked_blocks.json")


def _load_mutant(tmp_path, old, new):
    src = open(SRC).read()
    assert old in src, old
    d = tmp_path / "oracle_mutant"
    d.mkdir()
    shutil.copy(os.path.join(ROOT, "oracle", "__init__.py"), d / "__init__.py")
    (d / "q8_oracle.c").write_text(src.replace(old, new, 1))
    spec = importlib.util.spec_from_file_location("oracle_mutant", d / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


def _worked_blocks_pass(m):
    g = json.load(open(GOLDEN))
    for blk in g["blocks"].values():
        q, d = m.quantize_rows(np.array(blk["x"], np.float32))
        if list(q) != blk["q"] or int(d[0]) != int(blk["d_bits"], 16):
            return False
    return True


def _fp16_pass(m):
    h = np.arange(0, 0x7C00, dtype=np.uint32).astype(np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).astype(np.uint16).view(np.float16).astype(np.float64)
    mid = ((lo + hi) / 2).astype(np.float32)
    return np.array_equal(m.fp16_from_fp32_array(mid), mid.astype(np.float16).view(np.uint16))


def _deq(q, d):
    return q.astype(np.float64) * np.repeat(d.view(np.float16).astype(np.float64), 32, axis=-1)


def _gemv_pass(m):
    rng = np.random.default_rng(5)
    x = (rng.standard_normal((9, 96)) * 0.02).astype(np.float32)
    a = rng.standard_normal((2, 96)).astype(np.float32)
    wq, wd = m.quantize_rows(x)
    xq, xd = m.quantize_rows(a)
    y = m.gemv(wq, wd, xq, xd)
    ref = _deq(xq, xd) @ _deq(wq, wd).T
    return bool(np.all(np.abs(y - ref) <= 1e-12 * (np.abs(_deq(xq, xd)) @ np.abs(_deq(wq, wd)).T)))


def _halves_pass(m):
    rng = np.random.default_rng(9)
    n_ff, n_embd = 32, 64
    ugq, ugd = m.quantize_rows((rng.standard_normal((2, 2 * n_ff, n_embd)) * 0.02).astype(np.float32))
    xq, xd = m.quantize_rows(rng.standard_normal((2, n_embd)).astype(np.float32))
    ids = np.array([[1], [0]], np.int32)
    h, g, u = m.up_gate_swiglu(ugq, ugd, xq, xd, ids, want_gu=True)
    for t in range(2):
        e = ids[t, 0]
        gg = m.gemv(ugq[e, :n_ff], ugd[e, :n_ff], xq[t:t + 1], xd[t:t + 1])[0]
        uu = m.gemv(ugq[e, n_ff:], ugd[e, n_ff:], xq[t:t + 1], xd[t:t + 1])[0]
        if not (np.array_equal(g[t, 0], gg) and np.array_equal(u[t, 0], uu)):
            return False
        if not np.allclose(h[t, 0], gg / (1 + np.exp(-gg)) * uu, rtol=1e-12, atol=1e-15):
            return False
    return True


def _combine_pass(m):
    rng = np.random.default_rng(61)
    y = rng.standard_normal((3, 8, 16))
    p = rng.random((3, 8)).astype(np.float32)
    return np.allclose(m.combine(y, p), np.einsum("tk,tkr->tr", p.astype(np.float64), y),
                       rtol=1e-14, atol=1e-14)


MUTANTS = [
    ("ties to even", "float r = roundf(v);", "float r = rintf(v);", _worked_blocks_pass),
    ("scale 1/128", "float d32 = amax / 127.0f;", "float d32 = amax / 128.0f;", _worked_blocks_pass),
    ("fp16 ties away", "(rest == 0x1000u && (keep & 1u))", "(rest == 0x1000u)", _fp16_pass),
    ("dropped block", "for (int64_t b = 0; b < k / QK; ++b) {\n        int32_t isum",
     "for (int64_t b = 1; b < k / QK; ++b) {\n        int32_t isum", _gemv_pass),
    ("swapped halves", "double gv = oracle_row_dot(we + r * n_embd, de + r * nb,",
     "double gv = oracle_row_dot(we + (n_ff + r) * n_embd, de + (n_ff + r) * nb,", _halves_pass),
    ("silu sign", "return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));", _halves_pass),
    ("combine index", "s += (double)p[t * n_used + k]", "s += (double)p[k]", _combine_pass),
]


@pytest.mark.parametrize("name,old,new,check", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new, check):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    import oracle
    assert check(oracle), "the committed oracle must pass the pin"
    mutant = _load_mutant(tmp_path, old, new)
    try:
        caught = not check(mutant)
    except (ArithmeticError, ValueError):  # the mutant's own range checks fired
        caught = True
    assert caught, f"pin did not catch planted mistake: {name}"
