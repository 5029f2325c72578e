"""GPU parity of the batch-1 Q8_0 GEMV and the batched GEMV (P3), plus
determinism and the no-unwritten-output (poison) check."""
import numpy as np
import pytest
import torch

import oracle
from helpers import S_norm, assert_p3, bits, canon_d, host
from moe_up_gate_b200 import q8, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(rows, k, n_tok, seed):
    w = synth.normal((rows, k), seed=seed, std=0.02)
    x = synth.normal((n_tok, k), seed=seed + 1)
    W = q8.pack(w.to(DEV))
    xq, xd = q8.quantize_row(x.to(DEV))
    return w, x, W, xq, xd


def _oracle_y(W, xq, xd):
    wq = host(W.qs)
    wd = canon_d(W.d, W.k)
    y = oracle.gemv(wq, wd, host(xq), bits(xd))
    return y, S_norm(wq, wd, host(xq), bits(xd))


@pytest.mark.parametrize("rows,k,n_tok", [(1, 32, 1), (3, 64, 1), (33, 96, 2), (768, 768, 1),
                                          (1000, 2048, 3), (37, 14336, 1), (130, 704, 5),
                                          (64, 2816, 8), (45, 768, 9), (20, 256, 17)])
def test_gemv_p3(rows, k, n_tok):
    w, x, W, xq, xd = _case(rows, k, n_tok, seed=rows * 7 + k + n_tok)
    y = q8.gemv(W, xq, xd)
    ref, S = _oracle_y(W, xq, xd)
    assert_p3(host(y), ref, S, f"gemv {rows}x{k} T={n_tok}")


def test_gemv_deterministic_and_fully_written():
    w, x, W, xq, xd = _case(333, 2048, 3, seed=11)
    y1 = torch.full((3, 333), float("nan"), device=DEV)
    y2 = torch.full((3, 333), float("nan"), device=DEV)
    q8.gemv(W, xq, xd, y=y1)
    q8.gemv(W, xq, xd, y=y2)
    assert not torch.isnan(y1).any()
    assert torch.equal(y1.view(torch.int32), y2.view(torch.int32))


def test_gemv_batched_matches_quantize_then_gemv():
    shapes = [(768, 768), (2048, 768), (768, 2048), (37, 96), (1000, 32)]
    probs, refs = [], []
    for i, (rows, k) in enumerate(shapes):
        w = synth.normal((rows, k), seed=500 + i, std=0.02)
        x = synth.normal((2, k), seed=600 + i)
        W = q8.pack(w.to(DEV))
        xd_ = x.to(DEV)
        y = torch.full((2, rows), float("nan"), device=DEV)
        probs.append((W, xd_, y))
        refs.append((W, x))
    q8.gemv_batched(probs, n_tok=2)
    torch.cuda.synchronize()
    for (W, x), (_, xdev, y) in zip(refs, probs):
        rq, rd = oracle.quantize_rows(x.numpy())
        wq = host(W.qs)
        wd = canon_d(W.d, W.k)
        ref = oracle.gemv(wq, wd, rq, rd)
        assert_p3(host(y), ref, S_norm(wq, wd, rq, rd), "gemv_batched")
        # same bits as the two-call path
        xq, xd = q8.quantize_row(xdev)
        y2 = q8.gemv(W, xq, xd)
        assert torch.equal(y.view(torch.int32), y2.view(torch.int32))


@pytest.mark.parametrize("n_tok", [1, 3])
def test_gemv_batched_long_rows(n_tok):
    """Rows too long for the raw slot (k > 4096): every CTA quantizes the
    fp32 activations from global memory with eight threads per block; the
    short problem of the same launch then stages that way too.  P3 against
    the oracle and the same bits as quantize + q8_gemv."""
    shapes = [(300, 14336), (70, 8192), (768, 768)]
    probs, refs = [], []
    for i, (rows, k) in enumerate(shapes):
        w = synth.normal((rows, k), seed=700 + i, std=0.02)
        x = synth.normal((n_tok, k), seed=800 + i)
        W = q8.pack(w.to(DEV))
        y = torch.full((n_tok, rows), float("nan"), device=DEV)
        probs.append((W, x.to(DEV), y))
        refs.append((W, x))
    q8.gemv_batched(probs, n_tok=n_tok)
    torch.cuda.synchronize()
    for (W, x), (_, xdev, y) in zip(refs, probs):
        rq, rd = oracle.quantize_rows(x.numpy())
        wq = host(W.qs)
        wd = canon_d(W.d, W.k)
        ref = oracle.gemv(wq, wd, rq, rd)
        assert_p3(host(y), ref, S_norm(wq, wd, rq, rd), f"gemv_batched k={W.k}")
        xq, xd = q8.quantize_row(xdev)
        assert np.array_equal(host(xq), rq) and np.array_equal(bits(xd), rd)
        y2 = q8.gemv(W, xq, xd)
        assert torch.equal(y.view(torch.int32), y2.view(torch.int32))


def test_gemv_on_row_view():
    """A row view (offset rows of one matrix) reads exactly those rows."""
    w, x, W, xq, xd = _case(96, 128, 1, seed=77)
    V = W.row_view(32, 40)
    y = host(q8.gemv(V, xq, xd))
    full = host(q8.gemv(W, xq, xd))
    assert np.array_equal(y, full[:, 32:72])

