"""GPU parity of the Q8_0 quantizer, the weight packer and the block dot (P1, P2).

Every case draws its inputs once (moe_up_gate_b200.synth), runs the CUDA path
through the C ABI and the oracle on the same numbers, and requires int8 quants,
fp16 scales and int32 block dots to be bit-exact.
"""
import json
import os

import numpy as np
import pytest
import torch

import oracle
from helpers import bits, canon_d, host
from moe_up_gate_b200 import q8, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "q8_worked_blocks.json")


@pytest.mark.parametrize("n_rows,k,std", [(1, 32, 1.0), (3, 64, 1.0), (33, 704, 0.02),
                                          (7, 2816, 1e-3), (5, 14336, 1.0), (130, 768, 1e-4),
                                          (2, 4096, 300.0)])
def test_quantize_row_bit_exact(n_rows, k, std):
    x = synth.normal((n_rows, k), seed=100 + n_rows + k, std=std)
    qs, d = q8.quantize_row(x.to(DEV))
    rq, rd = oracle.quantize_rows(x.numpy())
    assert np.array_equal(host(qs), rq)
    assert np.array_equal(bits(d), rd)


def test_quantize_special_values():
    x = torch.zeros((6, 64), dtype=torch.float32)
    x[1, :32] = 1.0
    x[2, :] = 1e-3                       # subnormal fp16 scale
    x[3, 5] = -7.5                       # one non-zero element
    x[4, :32] = torch.arange(32) - 16.0
    x[5, :] = 1e-30                      # scale underflows to fp16 zero
    qs, d = q8.quantize_row(x.to(DEV))
    rq, rd = oracle.quantize_rows(x.numpy())
    assert np.array_equal(host(qs), rq) and np.array_equal(bits(d), rd)


def test_worked_blocks_on_gpu():
    g = json.load(open(GOLDEN))
    for name, blk in g["blocks"].items():
        x = torch.tensor(blk["x"], dtype=torch.float32).reshape(1, 32)
        qs, d = q8.quantize_row(x.to(DEV))
        assert host(qs)[0].tolist() == blk["q"], name
        assert int(bits(d)[0, 0]) == int(blk["d_bits"], 16), name


@pytest.mark.parametrize("n_mat,rows,k", [(1, 33, 64), (3, 64, 704), (2, 40, 2816)])
def test_pack_bit_exact(n_mat, rows, k):
    w = synth.normal((n_mat, rows, k), seed=200 + rows, std=0.02)
    W = q8.pack(w.to(DEV))
    assert W.ld_d % 8 == 0 and W.ld_d >= k // 32
    rq, rd = oracle.quantize_rows(w.numpy().reshape(-1, k))
    assert np.array_equal(host(W.qs), rq)
    d_all = bits(W.d)
    assert np.array_equal(d_all[:, : k // 32], rd)
    assert np.all(d_all[:, k // 32:] == 0)          # padding scales are zero


def test_block_dots_bit_exact():
    k = 2816
    w = synth.normal((2, 50, k), seed=301, std=0.02)
    x = synth.normal((1, k), seed=302)
    W = q8.pack(w.to(DEV))
    xq, xd = q8.quantize_row(x.to(DEV))
    rows = torch.tensor([0, 7, 49, 13], dtype=torch.int64, device=DEV)
    got = host(q8.debug_block_dots(W, 1, rows, xq))
    wq = host(W.qs).reshape(2, 50, k)
    xqh = host(xq)[0]
    for i, r in enumerate([0, 7, 49, 13]):
        assert np.array_equal(got[i], oracle.row_block_dots(wq[1, r], xqh))
    # an out-of-range row index reads nothing and reports INT32_MIN
    bad = torch.tensor([50, -1], dtype=torch.int64, device=DEV)
    assert np.all(host(q8.debug_block_dots(W, 1, bad, xq)) == np.iinfo(np.int32).min)
