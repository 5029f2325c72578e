"""The arithmetic identities the tensor-core epilogue relies on to scale an
int32 Q8_0 block sum v by an fp16 block scale d (the weight row's d_w) with
one fused multiply-add (csrc/q8_tc.cu, "Block scaling"):

  1. adding v to the bit pattern of M = 1.5 * 2^23 gives the fp32 value M + v
     exactly, for every |v| < 2^22 (a block sum is at most 32 * 128 * 128);
  2. M * d is exact in fp32 for every finite fp16 value d, so -M * d costs
     one exact multiply;
  3. hence fma(M + v, d, -M * d) = v * d rounded once to fp32, the same
     value as the plain product fp32(v) * d.

Checked exhaustively over the fp16 values and over a sweep of v, with the
fused multiply-add emulated exactly in fp64 (the operands' product needs at
most 24 + 11 significant bits, well inside fp64's 53)."""
import numpy as np

M = np.float32(12582912.0)  # 1.5 * 2^23
M_BITS = 0x4B400000


def _all_finite_fp16():
    h = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16).view(np.float16)
    return h[np.isfinite(h)].astype(np.float32)


def test_biased_bits_are_exact():
    v = np.concatenate([np.arange(-(1 << 22) + 1, -(1 << 22) + 4097),
                        np.arange(-70000, 70001, 7),
                        np.arange((1 << 22) - 4096, 1 << 22)]).astype(np.int64)
    x = (np.int64(M_BITS) + v).astype(np.uint32).view(np.float32)
    assert np.array_equal(x.astype(np.float64), np.float64(M) + v.astype(np.float64))
    # the largest block sum magnitude stays inside the exact range
    assert 32 * 128 * 128 < (1 << 22)


def test_magic_times_fp16_scale_is_exact():
    d = _all_finite_fp16()
    exact = np.float64(M) * d.astype(np.float64)
    assert np.array_equal((M * d).astype(np.float64), exact)


def test_fused_form_equals_single_rounding():
    d = _all_finite_fp16()
    d = d[d != 0]
    rng = np.random.default_rng(5)
    for v in [0, 1, -1, 127, -128, 4095, -4096, 524288, -524288,
              *rng.integers(-(1 << 19), 1 << 19, size=24).tolist()]:
        x = np.float64(M) + v                                 # M + v, exact in fp32
        nm = -(np.float64(M) * d.astype(np.float64))         # -M * d, exact in fp32
        fused = (x * d.astype(np.float64) + nm).astype(np.float32)   # one rounding
        plain = np.float32(v) * d                             # fp32(v) * d_x
        assert np.array_equal(fused, plain), v
