"""Pins for the oracle's block dot, GEMV, up_gate + SwiGLU, mul_mat_id and combine (CPU only).

What pins what:
  * block dot: numpy integer dot (library) on random and extreme int8 blocks.
  * GEMV / row dot: brute force -- dequantize both operands to fp64 with
    numpy's float16 (pinned in test_oracle_quant) and multiply with numpy's
    float64 matmul -- on tiny shapes; and the oracle's own dequant-then-fp64
    routine.  Agreement within 1e-12 of sum|w*x|.
  * up_gate + SwiGLU: numpy composition per routed pair; the invariant that the
    combined weight splits exactly into a gate half (rows 0..n_ff-1) and an up
    half (rows n_ff..2n_ff-1), i.e. g and u equal GEMVs on the two slices (the
    news.hada.io article, section 「3段階で構成された修正」: two view_3d slices,
    mul_mat_id on each, fused_mul_unary(gate, up, SILU)); swapping the halves
    changes h; silu closed forms.
  * mul_mat_id: routing selects exactly the named experts (marker expert test,
    perturbation of an unnamed expert leaves the output bitwise unchanged);
    per-pair numpy.
  * split gate/up weights: bitwise the combined op on the concatenated rows,
    g and u against numpy, gate/up not interchangeable, silu closed forms.
  * combine: numpy einsum.
  * invariants: dense op == one expert with every id 0; permuting tokens
    permutes outputs bitwise.
"""
import numpy as np
import pytest

QK = 32


def _deq(q, d):
    q = np.asarray(q)
    d = np.asarray(d, dtype=np.uint16)
    scale = d.view(np.float16).astype(np.float64)
    return q.astype(np.float64) * np.repeat(scale, QK, axis=-1)


def _qrand(orc, rng, shape, std):
    x = (rng.standard_normal(shape) * std).astype(np.float32)
    return orc.quantize_rows(x)


def _S(wq, wd, xq, xd):
    """sum_b |d_w d_x| sum_i |q_w q_x| per (token, row): the tolerance normaliser."""
    return np.abs(_deq(xq, xd)) @ np.abs(_deq(wq, wd)).T


def test_block_dot_vs_numpy(orc):
    rng = np.random.default_rng(1)
    for _ in range(200):
        a = rng.integers(-128, 128, 32).astype(np.int8)
        b = rng.integers(-128, 128, 32).astype(np.int8)
        assert orc.block_dot(a, b) == int(a.astype(np.int64) @ b.astype(np.int64))
    ext = np.full(32, -128, np.int8)
    assert orc.block_dot(ext, ext) == 32 * 128 * 128
    assert orc.block_dot(np.full(32, 127, np.int8), np.full(32, -127, np.int8)) == -32 * 127 * 127


@pytest.mark.parametrize("rows,k,n_tok", [(1, 32, 1), (3, 64, 2), (33, 96, 5), (17, 32, 17)])
def test_gemv_brute_force(orc, rows, k, n_tok):
    rng = np.random.default_rng(rows * 1000 + k + n_tok)
    wq, wd = _qrand(orc, rng, (rows, k), 0.02)
    xq, xd = _qrand(orc, rng, (n_tok, k), 1.0)
    y = orc.gemv(wq, wd, xq, xd)
    ref = _deq(xq, xd) @ _deq(wq, wd).T
    S = _S(wq, wd, xq, xd)
    assert np.all(np.abs(y - ref) <= 1e-12 * S + 1e-300)
    y2 = orc.dequant_fp64_matmul(wq, wd, xq, xd)
    assert np.all(np.abs(y - y2) <= 1e-12 * S + 1e-300)


def test_row_block_dots(orc):
    rng = np.random.default_rng(3)
    wq, _ = _qrand(orc, rng, (1, 128), 0.02)
    xq, _ = _qrand(orc, rng, (1, 128), 1.0)
    isum = orc.row_block_dots(wq[0], xq[0])
    ref = (wq[0].astype(np.int64).reshape(4, 32) * xq[0].astype(np.int64).reshape(4, 32)).sum(1)
    assert np.array_equal(isum, ref)


def test_silu_closed_forms(orc):
    assert orc.silu(0.0) == 0.0
    for z in (0.3, 1.7, 5.0, 12.0):
        # silu(z) - silu(-z) = z * (sigmoid(z) + sigmoid(-z)) = z
        assert abs((orc.silu(z) - orc.silu(-z)) - z) <= 1e-15 * abs(z)
    assert abs(orc.silu(40.0) - 40.0) < 1e-12
    assert abs(orc.silu(1.0) - 1.0 / (1.0 + np.exp(-1.0))) < 1e-16


def _moe_inputs(orc, seed, n_exp, n_ff, n_embd, n_tok, n_used):
    rng = np.random.default_rng(seed)
    ugq, ugd = _qrand(orc, rng, (n_exp, 2 * n_ff, n_embd), 0.02)
    xq, xd = _qrand(orc, rng, (n_tok, n_embd), 1.0)
    ids = np.stack([rng.permutation(n_exp)[:n_used] for _ in range(n_tok)]).astype(np.int32)
    return ugq, ugd, xq, xd, ids


@pytest.mark.parametrize("n_exp,n_ff,n_embd,n_tok,n_used", [(5, 64, 96, 3, 2), (2, 32, 64, 4, 2),
                                                            (4, 96, 32, 7, 3)])
def test_up_gate_vs_numpy(orc, n_exp, n_ff, n_embd, n_tok, n_used):
    ugq, ugd, xq, xd, ids = _moe_inputs(orc, 5, n_exp, n_ff, n_embd, n_tok, n_used)
    h, g, u = orc.up_gate_swiglu(ugq, ugd, xq, xd, ids, want_gu=True)
    xdq = _deq(xq, xd)
    for t in range(n_tok):
        for s in range(n_used):
            e = ids[t, s]
            W = _deq(ugq[e], ugd[e])
            gr = W[:n_ff] @ xdq[t]
            ur = W[n_ff:] @ xdq[t]
            Sg = np.abs(W[:n_ff]) @ np.abs(xdq[t])
            Su = np.abs(W[n_ff:]) @ np.abs(xdq[t])
            assert np.all(np.abs(g[t, s] - gr) <= 1e-12 * Sg)
            assert np.all(np.abs(u[t, s] - ur) <= 1e-12 * Su)
            href = gr / (1.0 + np.exp(-gr)) * ur
            assert np.allclose(h[t, s], href, rtol=1e-10, atol=1e-12 * (Sg * Su).max())


def test_up_gate_halves_split_exactly(orc):
    n_exp, n_ff, n_embd, n_tok, n_used = 3, 64, 64, 4, 2
    ugq, ugd, xq, xd, ids = _moe_inputs(orc, 9, n_exp, n_ff, n_embd, n_tok, n_used)
    h, g, u = orc.up_gate_swiglu(ugq, ugd, xq, xd, ids, want_gu=True)
    for t in range(n_tok):
        for s in range(n_used):
            e = ids[t, s]
            gg = orc.gemv(ugq[e, :n_ff], ugd[e, :n_ff], xq[t:t + 1], xd[t:t + 1])[0]
            uu = orc.gemv(ugq[e, n_ff:], ugd[e, n_ff:], xq[t:t + 1], xd[t:t + 1])[0]
            assert np.array_equal(g[t, s], gg) and np.array_equal(u[t, s], uu)
    # the same through mul_mat_id on the two slices (the unfused chain)
    gate_q, gate_d = ugq[:, :n_ff], ugd[:, :n_ff]
    up_q, up_d = ugq[:, n_ff:], ugd[:, n_ff:]
    g2 = orc.mul_mat_id(gate_q, gate_d, xq, xd, ids, a_per_slot=False)
    u2 = orc.mul_mat_id(up_q, up_d, xq, xd, ids, a_per_slot=False)
    assert np.array_equal(g2, g) and np.array_equal(u2, u)
    # swapping the halves changes h
    sw_q = np.concatenate([up_q, gate_q], axis=1)
    sw_d = np.concatenate([up_d, gate_d], axis=1)
    h_sw = orc.up_gate_swiglu(sw_q, sw_d, xq, xd, ids)
    assert not np.allclose(h_sw, h)
    # which half is gate: a constant up half (q = 1, d = 1.0) makes u = sum of x
    c_q = ugq.copy()
    c_d = ugd.copy()
    c_q[:, n_ff:] = 1
    c_d[:, n_ff:] = 0x3C00
    hc, gc, uc = orc.up_gate_swiglu(c_q, c_d, xq, xd, ids, want_gu=True)
    xs = _deq(xq, xd).sum(axis=1)
    for t in range(n_tok):
        assert np.allclose(uc[t], xs[t], rtol=1e-12, atol=1e-12)
        assert np.allclose(hc[t], gc[t] / (1 + np.exp(-gc[t])) * xs[t], rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("n_exp,n_ff,n_embd,n_tok,n_used", [(4, 64, 96, 3, 2), (1, 32, 64, 5, 1)])
def test_split_weights_path(orc, n_exp, n_ff, n_embd, n_tok, n_used):
    """Separate gate and up tensors (two mul_mat_id, then silu(g) * u): bitwise
    the combined-tensor op on their row concatenation; g and u against numpy;
    gate and up not interchangeable; the dense form is expert 0 for every token."""
    rng = np.random.default_rng(40 + n_exp)
    gq, gd = _qrand(orc, rng, (n_exp, n_ff, n_embd), 0.02)
    uq, ud = _qrand(orc, rng, (n_exp, n_ff, n_embd), 0.02)
    xq, xd = _qrand(orc, rng, (n_tok, n_embd), 1.0)
    ids = np.stack([rng.permutation(n_exp)[:n_used] for _ in range(n_tok)]).astype(np.int32)
    h, g, u = orc.up_gate_swiglu_split(gq, gd, uq, ud, xq, xd, ids, want_gu=True)
    ugq = np.concatenate([gq, uq], axis=1)
    ugd = np.concatenate([gd, ud], axis=1)
    hc, gc, uc = orc.up_gate_swiglu(ugq, ugd, xq, xd, ids, want_gu=True)
    assert np.array_equal(h, hc) and np.array_equal(g, gc) and np.array_equal(u, uc)
    xdq = _deq(xq, xd)
    for t in range(n_tok):
        for s in range(n_used):
            e = ids[t, s]
            Wg, Wu = _deq(gq[e], gd[e]), _deq(uq[e], ud[e])
            gr, ur = Wg @ xdq[t], Wu @ xdq[t]
            assert np.all(np.abs(g[t, s] - gr) <= 1e-12 * (np.abs(Wg) @ np.abs(xdq[t])))
            assert np.all(np.abs(u[t, s] - ur) <= 1e-12 * (np.abs(Wu) @ np.abs(xdq[t])))
            assert np.allclose(h[t, s], gr / (1.0 + np.exp(-gr)) * ur, rtol=1e-10, atol=1e-15)
    assert not np.allclose(orc.up_gate_swiglu_split(uq, ud, gq, gd, xq, xd, ids), h)
    if n_exp == 1:
        assert np.array_equal(orc.up_gate_swiglu_split(gq[0], gd[0], uq[0], ud[0], xq, xd), h)


def test_swiglu_elementwise(orc):
    g = np.array([0.0, 1.0, -1.0, 30.0, -30.0, 2.5], np.float64)
    u = np.array([3.0, 2.0, 2.0, 0.5, 4.0, -1.0], np.float64)
    h = orc.swiglu(g, u)
    assert h[0] == 0.0
    assert abs(h[1] - 2.0 * 0.7310585786300049) < 1e-15      # silu(1) = 1 / (1 + e^-1)
    assert abs(h[2] - 2.0 * -0.2689414213699951) < 1e-15     # silu(-1) = -1 / (1 + e)
    # far tails: silu(30) = 30 / (1 + e^-30) ~ 30, silu(-30) = -30 / (1 + e^30) ~ -2.8e-12
    assert abs(h[3] / (0.5 * 30.0 / (1.0 + np.exp(-30.0))) - 1.0) < 1e-15
    assert abs(h[4] / (4.0 * -30.0 / (1.0 + np.exp(30.0))) - 1.0) < 1e-14
    assert np.allclose(h, g / (1.0 + np.exp(-g)) * u, rtol=1e-15, atol=0)


def test_dense_equals_single_expert(orc):
    rng = np.random.default_rng(21)
    n_ff, n_embd, n_tok = 64, 96, 5
    ugq, ugd = _qrand(orc, rng, (1, 2 * n_ff, n_embd), 0.02)
    xq, xd = _qrand(orc, rng, (n_tok, n_embd), 1.0)
    hd = orc.up_gate_swiglu(ugq, ugd, xq, xd, None)
    h0 = orc.up_gate_swiglu(ugq, ugd, xq, xd, np.zeros((n_tok, 1), np.int32))
    assert np.array_equal(hd, h0)


def test_routing_selects_named_experts(orc):
    n_exp, n_ff, n_embd, n_tok, n_used = 6, 32, 64, 8, 2
    ugq, ugd, xq, xd, ids = _moe_inputs(orc, 31, n_exp, n_ff, n_embd, n_tok, n_used)
    marker = int(ids[2, 1])
    z_q = np.zeros_like(ugq)
    z_q[marker] = ugq[marker]
    h = orc.up_gate_swiglu(z_q, ugd, xq, xd, ids)
    nz = np.any(h != 0, axis=2)
    assert np.array_equal(nz, ids == marker)
    # perturbing an expert no token names leaves everything bitwise unchanged
    unused = [e for e in range(n_exp) if e not in set(ids.ravel().tolist())]
    h_ref = orc.up_gate_swiglu(ugq, ugd, xq, xd, ids)
    if unused:
        p_q = ugq.copy()
        p_q[unused[0]] = -p_q[unused[0]]
        assert np.array_equal(orc.up_gate_swiglu(p_q, ugd, xq, xd, ids), h_ref)
    # out-of-range ids are an error
    bad = ids.copy()
    bad[0, 0] = n_exp
    with pytest.raises(ValueError):
        orc.up_gate_swiglu(ugq, ugd, xq, xd, bad)


def test_token_permutation(orc):
    n_exp, n_ff, n_embd, n_tok, n_used = 4, 32, 64, 6, 2
    ugq, ugd, xq, xd, ids = _moe_inputs(orc, 41, n_exp, n_ff, n_embd, n_tok, n_used)
    perm = np.random.default_rng(0).permutation(n_tok)
    h = orc.up_gate_swiglu(ugq, ugd, xq, xd, ids)
    hp = orc.up_gate_swiglu(ugq, ugd, xq[perm], xd[perm], ids[perm])
    assert np.array_equal(hp, h[perm])


def test_mul_mat_id_vs_numpy(orc):
    rng = np.random.default_rng(51)
    n_mat, rows, k, n_tok, n_used = 5, 33, 64, 4, 3
    wq, wd = _qrand(orc, rng, (n_mat, rows, k), 0.02)
    aq, ad = _qrand(orc, rng, (n_tok, n_used, k), 1.0)
    ids = np.stack([rng.permutation(n_mat)[:n_used] for _ in range(n_tok)]).astype(np.int32)
    y = orc.mul_mat_id(wq, wd, aq, ad, ids, a_per_slot=True)
    for t in range(n_tok):
        for s in range(n_used):
            W = _deq(wq[ids[t, s]], wd[ids[t, s]])
            a = _deq(aq[t, s], ad[t, s])
            S = np.abs(W) @ np.abs(a)
            assert np.all(np.abs(y[t, s] - W @ a) <= 1e-12 * S)
    # a marker matrix: zero every matrix except one; only its slots are non-zero
    marker = int(ids[1, 0])
    z = np.zeros_like(wq)
    z[marker] = wq[marker]
    yz = orc.mul_mat_id(z, wd, aq, ad, ids, a_per_slot=True)
    assert np.array_equal(np.any(yz != 0, axis=2), ids == marker)


def test_combine_vs_numpy(orc):
    rng = np.random.default_rng(61)
    y = rng.standard_normal((3, 8, 40))
    p = rng.random((3, 8)).astype(np.float32)
    out = orc.combine(y, p)
    ref = np.einsum("tk,tkr->tr", p.astype(np.float64), y)
    assert np.allclose(out, ref, rtol=1e-14, atol=1e-14)
    # one-hot weights select one slot exactly
    oh = np.zeros((3, 8), np.float32)
    oh[:, 5] = 1.0
    assert np.array_equal(orc.combine(y, oh), y[:, 5])


def test_moe_ffn_dense_and_routed_agree(orc):
    """The whole step: dense (no ids) equals one expert with id 0 and weight 1."""
    rng = np.random.default_rng(71)
    n_ff, n_embd, n_tok = 64, 96, 3
    ugq, ugd = _qrand(orc, rng, (1, 2 * n_ff, n_embd), 0.02)
    dnq, dnd = _qrand(orc, rng, (1, n_embd, n_ff), 0.02)
    x = rng.standard_normal((n_tok, n_embd)).astype(np.float32)
    a = orc.moe_ffn(ugq, ugd, dnq, dnd, x)
    b = orc.moe_ffn(ugq, ugd, dnq, dnd, x, np.zeros((n_tok, 1), np.int32),
                    np.ones((n_tok, 1), np.float32))
    assert np.array_equal(a["out"], b["out"])
    # stages: xq is the quantizer's, hq the quantizer on fp32(h), out the down GEMV of hq
    xq, xd = orc.quantize_rows(x)
    assert np.array_equal(a["xq"], xq) and np.array_equal(a["xd"], xd)
    hq, hd = orc.quantize_rows(a["h"].astype(np.float32).reshape(n_tok, n_ff))
    assert np.array_equal(a["hq"].reshape(n_tok, n_ff), hq)
    ref = _deq(hq, hd) @ _deq(dnq[0], dnd[0]).T
    S = np.abs(_deq(hq, hd)) @ np.abs(_deq(dnq[0], dnd[0])).T
    assert np.all(np.abs(a["out"] - ref) <= 1e-12 * S)
