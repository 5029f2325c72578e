"""GPU parity of the int8 tensor-core (tcgen05) path, which serves experts with
at least 4 routed rows in the workspace (grouped) calls: the fused up/gate +
SwiGLU, the mul_mat_id down projection and the whole step at a large batch.

Its per-block int32 dots are exact like the dp4a path's; only the fp32
accumulation order differs, so outputs are held to the oracle with the P3
bound (matmul outputs) and, for h = silu(g) * u, with the bound that P3 on g
and u implies: |dh| <= 1.2 |u| dg + |silu(g)| du + 1e-6 |h|.
"""
import numpy as np
import pytest
import torch

import oracle
from helpers import S_norm, TOL, assert_p3, bits, canon_d, host
from moe_up_gate_b200 import q8, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _w_host(W):
    return (host(W.qs).reshape(W.n_mat, W.mat_stride, W.k),
            canon_d(W.d, W.k).reshape(W.n_mat, W.mat_stride, W.k // 32))


def _ids_skewed(n_tok, n_exp, n_used, hot, seed):
    """Routing ids whose first `hot` experts take most tokens (distinct per token)."""
    g = torch.Generator().manual_seed(seed)
    rows = []
    for t in range(n_tok):
        if t % 4 != 3:  # three quarters of the tokens route to the hot experts
            first = torch.randperm(hot, generator=g)[: min(n_used, hot)].tolist()
        else:
            first = []
        rest = [e for e in torch.randperm(n_exp, generator=g).tolist() if e not in first]
        rows.append((first + rest)[:n_used])
    return torch.tensor(rows, dtype=torch.int32)


def _check_h(UG, xq, xd, ids, h):
    wq, wd = _w_host(UG)
    xqh, xdh = host(xq), bits(xd)
    idh = host(ids)
    h_ref, g_ref, u_ref = oracle.up_gate_swiglu(wq, wd, xqh, xdh, idh, want_gu=True)
    n_tok, n_used, n_ff = h_ref.shape
    hh = host(h).astype(np.float64)
    worst = 0.0
    for t in range(n_tok):
        for s in range(n_used):
            e = idh[t, s]
            Sg = S_norm(wq[e, :n_ff], wd[e, :n_ff], xqh[t:t + 1], xdh[t:t + 1])[0]
            Su = S_norm(wq[e, n_ff:], wd[e, n_ff:], xqh[t:t + 1], xdh[t:t + 1])[0]
            g, u = g_ref[t, s], u_ref[t, s]
            sg = g / (1 + np.exp(-g))
            bound = TOL * (1.2 * np.abs(u) * Sg + np.abs(sg) * Su) + 1e-6 * np.abs(h_ref[t, s]) + 1e-30
            err = np.abs(hh[t, s] - h_ref[t, s])
            assert np.all(err <= bound), (t, s, float((err / bound).max()))
            worst = max(worst, float((err / bound).max()))
    return worst


@pytest.mark.parametrize("n_exp,n_ff,n_embd,n_tok,n_used,hot", [
    (4, 64, 256, 40, 2, 4),       # every expert >= 16 rows: tensor cores only
    (2, 128, 512, 80, 1, 2),      # > 32 rows per expert: several passes per tile
    (16, 64, 2816, 64, 2, 2),     # two hot experts on the tensor cores, the rest dp4a
    (8, 128, 1024, 48, 2, 1),     # 5..11 rows on most experts: padded 16-column passes
])
def test_tc_up_gate(n_exp, n_ff, n_embd, n_tok, n_used, hot):
    shape = synth.MoeShape(n_embd=n_embd, n_ff=n_ff, n_exp=n_exp, n_used=n_used)
    t = synth.moe_layer_tensors(700 + n_exp, 0, shape, n_tok, 1.0)
    UG = q8.pack(t["up_gate"].to(DEV))
    ids = _ids_skewed(n_tok, n_exp, n_used, hot, seed=n_exp).to(DEV)
    xq, xd = q8.quantize_row(t["x"].to(DEV))
    r = q8.moe_up_gate_swiglu(UG, xq, xd, ids, want_hq=True)
    _check_h(UG, xq, xd, ids, r["h"])
    rq, _ = oracle.quantize_rows(host(r["h"]).reshape(-1, n_ff))
    assert np.array_equal(host(r["hq"]).reshape(-1, n_ff), rq)
    # deterministic
    r2 = q8.moe_up_gate_swiglu(UG, xq, xd, ids)
    assert torch.equal(r["h"], r2["h"])


@pytest.mark.parametrize("n_mat,rows,k,n_tok,n_used,hot", [
    (4, 200, 704, 40, 2, 4),      # a ragged last row tile, k with a half K chunk
    (3, 256, 2816, 50, 1, 3),
    (8, 128, 128, 72, 2, 2),
    (4, 128, 224, 40, 2, 4),      # an odd block count: the gather by plain loads
    (8, 256, 704, 48, 2, 1),      # 5..11 rows on most experts: padded 16-column passes
])
def test_tc_mul_mat_id(n_mat, rows, k, n_tok, n_used, hot):
    w = synth.normal((n_mat, rows, k), seed=801 + k, std=0.02)
    W = q8.pack(w.to(DEV))
    ids = _ids_skewed(n_tok, n_mat, n_used, hot, seed=rows).to(DEV)
    a = synth.normal((n_tok * n_used, k), seed=802 + k)
    aq, ad = q8.quantize_row(a.to(DEV))
    y = torch.full((n_tok, n_used, rows), float("nan"), device=DEV)
    q8.mul_mat_id(W, aq, ad, ids, a_per_slot=True, y=y)
    wq, wd = _w_host(W)
    aqh = host(aq).reshape(n_tok, n_used, k)
    adh = bits(ad).reshape(n_tok, n_used, k // 32)
    ref = oracle.mul_mat_id(wq, wd, aqh, adh, host(ids), True)
    yh = host(y)
    idh = host(ids)
    assert not np.isnan(yh).any()
    for t_ in range(n_tok):
        for s in range(n_used):
            e = idh[t_, s]
            S = S_norm(wq[e], wd[e], aqh[t_, s][None], adh[t_, s][None])[0]
            assert_p3(yh[t_, s], ref[t_, s], S, "tc mul_mat_id")


def test_tc_and_dp4a_agree():
    """The same call through the tensor cores (workspace path) and through dp4a
    (small-batch fp32 path) agree within the P3 bound on g/u-derived h."""
    shape = synth.MoeShape(n_embd=2816, n_ff=704, n_exp=8, n_used=2)
    t = synth.moe_layer_tensors(731, 0, shape, 48, 1.0)
    UG = q8.pack(t["up_gate"].to(DEV))
    DN = q8.pack(t["down"].to(DEV))
    ids = _ids_skewed(48, 8, 2, 3, seed=5).to(DEV)
    x = t["x"].to(DEV)
    xq, xd = q8.quantize_row(x)
    h_tc = q8.moe_up_gate_swiglu(UG, xq, xd, ids, want_hq=True)
    h_dp = q8.moe_up_gate_swiglu_fp32(UG, x, ids)
    _check_h(UG, xq, xd, ids, h_tc["h"])
    _check_h(UG, xq, xd, ids, h_dp)
    y_tc = q8.mul_mat_id(DN, h_tc["hq"].reshape(-1, 704), h_tc["hd"].reshape(-1, 22), ids, True)
    y_dp = q8.mul_mat_id_fp32(DN, h_tc["h"].reshape(-1, 704), ids, True)
    # the same quantized h feeds both: P3 against each other, twice the bound
    wq, wd = _w_host(DN)
    hq = host(h_tc["hq"]).reshape(48, 2, 704)
    hd = bits(h_tc["hd"]).reshape(48, 2, 22)
    idh = host(ids)
    for t_ in range(48):
        for s in range(2):
            e = idh[t_, s]
            S = S_norm(wq[e], wd[e], hq[t_, s][None], hd[t_, s][None])[0]
            assert np.all(np.abs(host(y_tc)[t_, s] - host(y_dp)[t_, s]) <= 2 * TOL * S + 1e-30)


def test_large_batch_ffn_step_sampled():
    """A Gemma-4-26B-A4B-shaped layer at 256 tokens (2048 routed pairs): the
    whole step takes the workspace path (grouping kernel, tensor cores for
    experts with >= 4 rows).  Sampled tokens are checked stage by stage
    against the oracle."""
    shape = synth.MOE_LAYER
    t = synth.moe_layer_tensors(5, 0, shape, 256, synth.W_STD, device=DEV)
    UG = q8.pack(t["up_gate"])
    DN = q8.pack(t["down"])
    x, ids, p = t["x"], t["ids"].to(DEV), t["p"].to(DEV)
    out = q8.moe_ffn(UG, DN, x, ids, p)
    xq, xd = q8.quantize_row(x)
    r = q8.moe_up_gate_swiglu(UG, xq, xd, ids, want_hq=True)
    y = q8.mul_mat_id(DN, r["hq"].reshape(-1, 704), r["hd"].reshape(-1, 22), ids, True)
    assert torch.equal(out, q8.moe_combine(y, p))
    counts = torch.bincount(ids.flatten().long(), minlength=128)
    assert int((counts >= 4).sum()) > 0, "the seeded batch has tensor-core experts"
    # oracle on sampled tokens (the oracle quantizes the fp32 weights itself)
    ugq, ugd = oracle.quantize_rows(t["up_gate"].cpu().numpy())
    dnq, dnd = oracle.quantize_rows(t["down"].cpu().numpy())
    assert np.array_equal(ugq.reshape(-1, 2816), host(UG.qs))
    idh = host(ids)
    for tok in (0, 77, 255):
        sub_ids = idh[tok:tok + 1]
        hr, gr, ur = oracle.up_gate_swiglu(ugq, ugd, host(xq)[tok:tok + 1], bits(xd)[tok:tok + 1],
                                           sub_ids, want_gu=True)
        hh = host(r["h"])[tok]
        for s in range(8):
            e = sub_ids[0, s]
            Sg = S_norm(ugq[e, :704], ugd[e, :704], host(xq)[tok:tok + 1], bits(xd)[tok:tok + 1])[0]
            Su = S_norm(ugq[e, 704:], ugd[e, 704:], host(xq)[tok:tok + 1], bits(xd)[tok:tok + 1])[0]
            g, u = gr[0, s], ur[0, s]
            sg = g / (1 + np.exp(-g))
            bound = TOL * (1.2 * np.abs(u) * Sg + np.abs(sg) * Su) + 1e-6 * np.abs(hr[0, s]) + 1e-30
            assert np.all(np.abs(hh[s] - hr[0, s]) <= bound)
        hq_t = host(r["hq"])[tok]
        hd_t = bits(r["hd"])[tok]
        yr = oracle.mul_mat_id(dnq, dnd, hq_t[None], hd_t[None], sub_ids, True)
        for s in range(8):
            e = sub_ids[0, s]
            S = S_norm(dnq[e], dnd[e], hq_t[s][None], hd_t[s][None])[0]
            assert_p3(host(y)[tok, s], yr[0, s], S, "down")


@pytest.mark.parametrize("rows,k,n_tok", [(300, 704, 16), (128, 2816, 16), (77, 256, 32),
                                          (256, 4096, 21), (130, 160, 19)])
def test_tc_dense_gemv(rows, k, n_tok):
    """Dense matmuls with 16..32 activation rows run on the tensor cores (one
    pass over W): P3 against the oracle, every output written."""
    w = synth.normal((rows, k), seed=811 + k + n_tok, std=0.02)
    W = q8.pack(w.to(DEV))
    a = synth.normal((n_tok, k), seed=812 + k)
    aq, ad = q8.quantize_row(a.to(DEV))
    y = torch.full((n_tok, rows), float("nan"), device=DEV)
    q8.gemv(W, aq, ad, y=y)
    wq, wd = host(W.qs), canon_d(W.d, k)
    ref = oracle.gemv(wq, wd, host(aq), bits(ad))
    assert not torch.isnan(y).any()
    assert_p3(host(y), ref, S_norm(wq, wd, host(aq), bits(ad)), "tc dense gemv")


@pytest.mark.parametrize("n_ff,n_embd,n_tok", [(128, 512, 16), (64, 2816, 24), (192, 1024, 32)])
def test_tc_dense_up_gate(n_ff, n_embd, n_tok):
    """Dense up/gate + SwiGLU with 16..32 rows on the tensor cores: h against
    the oracle (the bound P3 on g and u implies), hq by the oracle's quantizer
    (P5), and the fp32 entry point gives the same bits."""
    shape = synth.MoeShape(n_embd=n_embd, n_ff=n_ff, n_exp=1, n_used=1)
    t = synth.moe_layer_tensors(820 + n_tok, 0, shape, n_tok, 1.0)
    UG = q8.pack(t["up_gate"].to(DEV))
    x = t["x"].to(DEV)
    xq, xd = q8.quantize_row(x)
    r = q8.moe_up_gate_swiglu(UG, xq, xd, None, want_hq=True)
    ids0 = torch.zeros((n_tok, 1), dtype=torch.int32)
    _check_h(UG, xq, xd, ids0, r["h"])
    rq, _ = oracle.quantize_rows(host(r["h"]).reshape(-1, n_ff))
    assert np.array_equal(host(r["hq"]).reshape(-1, n_ff), rq)
    h32 = q8.moe_up_gate_swiglu_fp32(UG, x, None)
    assert torch.equal(h32, r["h"])


def test_tc_dense_ffn_equals_chain():
    """The dense feed-forward step at 16 tokens (both matmuls on the tensor
    cores) equals quantize -> up/gate -> GEMV bitwise."""
    shape = synth.MoeShape(n_embd=512, n_ff=256, n_exp=1, n_used=1)
    t = synth.moe_layer_tensors(840, 0, shape, 16, 1.0)
    UG = q8.pack(t["up_gate"].to(DEV))
    DN = q8.pack(t["down"].to(DEV))
    x = t["x"].to(DEV)
    out = q8.moe_ffn(UG, DN, x)
    xq, xd = q8.quantize_row(x)
    r = q8.moe_up_gate_swiglu(UG, xq, xd, None, want_hq=True)
    y = q8.gemv(DN, r["hq"].reshape(16, 256), r["hd"].reshape(16, 8))
    assert torch.equal(out, y)
