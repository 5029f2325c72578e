"""Pins for the oracle's fp16 conversion and Q8_0 quantizer (CPU only).

What pins what:
  * fp16 <-> fp32: numpy's float16 conversion (a library routine implementing
    the same IEEE-754 round-to-nearest-even with subnormals) over every fp16
    value, every rounding tie between consecutive fp16 values and its
    neighbours, and a stride through all fp32 bit patterns; plus closed forms
    at the range edges.
  * quantizer: the hand-worked blocks in tests/golden/q8_worked_blocks.json
    (one of them fails any ties-to-even rounding), and properties the Q8_0
    definition fixes for any input: |q| <= 127, the largest-magnitude element
    maps to +-127, the dequantization error bound |x - d32*q| <= d32/2 (plus
    rounding slack), odd symmetry, invariance under power-of-two scaling.
"""
import json
import os

import numpy as np
import pytest

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "q8_worked_blocks.json")


def _np_fp16_bits(f32: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        return np.asarray(f32, dtype=np.float32).astype(np.float16).view(np.uint16)


def test_fp16_to_fp32_all_values(orc):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = orc.fp32_from_fp16_array(h)
    ref = h.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_fp16_round_trip_all_finite(orc):
    h = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    f = h.view(np.float16).astype(np.float32)
    ok = np.isfinite(f)
    back = orc.fp16_from_fp32_array(f[ok])
    assert np.array_equal(back, h[ok])


def test_fp32_to_fp16_ties_and_neighbours(orc):
    # every midpoint between consecutive non-negative fp16 values, +-3 fp32 ulps
    h = np.arange(0, 0x7C00, dtype=np.uint32).astype(np.uint16)
    lo = h.view(np.float16).astype(np.float64)
    hi = (h + 1).astype(np.uint16).view(np.float16).astype(np.float64)
    mid = ((lo + hi) / 2).astype(np.float32)  # exact in fp32 (needs <= 12 bits)
    assert np.array_equal(mid.astype(np.float64), (lo + hi) / 2)
    bits = mid.view(np.uint32).astype(np.int64)
    cands = np.concatenate([bits + dlt for dlt in range(-3, 4)])
    cands = cands[(cands >= 0) & (cands < 0x7F800000)].astype(np.uint32)
    f = cands.view(np.float32)
    f = np.concatenate([f, -f])
    assert np.array_equal(orc.fp16_from_fp32_array(f), _np_fp16_bits(f))


def test_fp32_to_fp16_strided_all_patterns(orc):
    bits = np.arange(0, 2**32, 4093, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[~np.isnan(f)]
    assert np.array_equal(orc.fp16_from_fp32_array(f), _np_fp16_bits(f))


@pytest.mark.parametrize("value,bits", [
    (65504.0, 0x7BFF),          # largest finite fp16
    (65519.996, 0x7BFF),        # just below the tie with 65536 -> stays finite
    (65520.0, 0x7C00),          # tie between 65504 and 65536: even -> infinity
    (2.0 ** -14, 0x0400),       # smallest normal
    (2.0 ** -24, 0x0001),       # smallest subnormal
    (2.0 ** -25, 0x0000),       # tie between 0 and 2^-24: even -> 0
    (1.5 * 2.0 ** -25, 0x0001),
    (3 * 2.0 ** -25, 0x0002),   # tie between 1 and 2 ulps: even -> 2
    (-1.0, 0xBC00),
    (1.0 / 3.0, 0x3555),
])
def test_fp32_to_fp16_closed_forms(orc, value, bits):
    assert orc.fp16_from_fp32(value) == bits


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


@pytest.mark.parametrize("name", ["A", "B", "C", "D", "E"])
def test_worked_blocks(orc, name):
    blk = _golden()["blocks"][name]
    x = np.array(blk["x"], dtype=np.float32)
    q, d = orc.quantize_rows(x)
    assert list(q) == blk["q"]
    assert int(d[0]) == int(blk["d_bits"], 16)


def test_worked_dot_a_c(orc):
    g = _golden()
    qa, da = orc.quantize_rows(np.array(g["blocks"]["A"]["x"], np.float32))
    qc, dc = orc.quantize_rows(np.array(g["blocks"]["C"]["x"], np.float32))
    assert orc.block_dot(qa, qc) == g["dots"]["A.C"]["isum"]
    # y = d_A * d_C * isum with d_A = 0.1259765625 = 129/1024, d_C = 129/16384 (exact fp16 values)
    y = orc.gemv(qa[None], da[None], qc[None], dc[None])[0, 0]
    assert y == (129 / 1024) * (129 / 16384) * -16129


def _rand_rows(rng, n, k, scale):
    return (rng.standard_normal((n, k)) * scale).astype(np.float32)


@pytest.mark.parametrize("scale", [1.0, 0.02, 1e-4, 300.0])
def test_quantize_properties(orc, scale):
    rng = np.random.default_rng(7)
    x = _rand_rows(rng, 64, 256, scale)
    x[3, 32:64] = 0.0                    # an all-zero block
    x[5, 0:32] = -x[5, 0:32]
    q, d = orc.quantize_rows(x)
    assert q.dtype == np.int8 and np.all(np.abs(q.astype(np.int32)) <= 127)
    xb = x.reshape(64, 8, 32).astype(np.float64)
    qb = q.reshape(64, 8, 32).astype(np.int32)
    amax = np.abs(xb).max(axis=2)
    d32 = (amax.astype(np.float32) / np.float32(127)).astype(np.float64)
    # the stored scale is the fp16 rounding of amax/127
    assert np.array_equal(d, _np_fp16_bits(d32.astype(np.float32)))
    # the element of largest magnitude maps to +-127 (unless the block is zero)
    idx = np.abs(xb).argmax(axis=2)
    top = np.take_along_axis(qb, idx[..., None], axis=2)[..., 0]
    nz = amax > 0
    assert np.all(np.abs(top[nz]) == 127)
    assert np.all(qb[~nz] == 0)
    # dequantization error of round-to-nearest with the fp32 scale
    err = np.abs(xb - d32[..., None] * qb)
    assert np.all(err <= d32[..., None] * (0.5 + 1e-5))
    # odd symmetry: quantize(-x) = -quantize(x), same scale
    qn, dn = orc.quantize_rows(-x)
    assert np.array_equal(qn, -q) and np.array_equal(dn, d)


def test_quantize_power_of_two_scaling(orc):
    rng = np.random.default_rng(11)
    x = _rand_rows(rng, 16, 128, 1.0)
    q1, _ = orc.quantize_rows(x)
    for e in (-6, -1, 3, 9):
        q2, _ = orc.quantize_rows(x * np.float32(2.0 ** e))
        assert np.array_equal(q1, q2)


def test_quantize_rejects_bad_k(orc):
    with pytest.raises(ValueError):
        orc.quantize_rows(np.zeros((2, 48), np.float32))
