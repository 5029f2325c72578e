"""GPU parity of the fused MoE up/gate + SwiGLU step, mul_mat_id, the combine
and the whole feed-forward step (P3-P5), with the invariants the method fixes:
the combined weight splits exactly into gate and up halves, routing selects
exactly the named experts, dense == one expert with id 0, token order only
permutes outputs, two runs are bitwise equal, every output is written; and the
device-side id validation (no GPU fault: bad pairs are skipped and reported)."""
import numpy as np
import pytest
import torch

import oracle
from helpers import S_norm, TOL, assert_p3, bits, canon_d, host
from moe_up_gate_b200 import q8, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _layer(n_exp, n_ff, n_embd, n_tok, n_used, seed, x_std=1.0):
    shape = synth.MoeShape(n_embd=n_embd, n_ff=n_ff, n_exp=n_exp, n_used=n_used)
    t = synth.moe_layer_tensors(seed, 0, shape, n_tok, x_std)
    UG = q8.pack(t["up_gate"].to(DEV))
    DN = q8.pack(t["down"].to(DEV))
    ids = None if t["ids"] is None else t["ids"].to(DEV)
    p = None if t["p"] is None else t["p"].to(DEV)
    return t, UG, DN, ids, p


def _w_host(W):
    return (host(W.qs).reshape(W.n_mat, W.mat_stride, W.k),
            canon_d(W.d, W.k).reshape(W.n_mat, W.mat_stride, W.k // 32))


def _check_up_gate(UG, xq, xd, ids, r):
    """P3 on g and u, P4 on h, P5 on hq against the oracle."""
    wq, wd = _w_host(UG)
    xqh, xdh = host(xq), bits(xd)
    idh = None if ids is None else host(ids)
    h_ref, g_ref, u_ref = oracle.up_gate_swiglu(wq, wd, xqh, xdh, idh, want_gu=True)
    n_tok, n_used, n_ff = g_ref.shape
    g, u, h = host(r["g"]), host(r["u"]), host(r["h"])
    for t in range(n_tok):
        for s in range(n_used):
            e = 0 if idh is None else idh[t, s]
            Sg = S_norm(wq[e, :n_ff], wd[e, :n_ff], xqh[t:t + 1], xdh[t:t + 1])[0]
            Su = S_norm(wq[e, n_ff:], wd[e, n_ff:], xqh[t:t + 1], xdh[t:t + 1])[0]
            assert_p3(g[t, s], g_ref[t, s], Sg, "gate")
            assert_p3(u[t, s], u_ref[t, s], Su, "up")
    gd, ud = g.astype(np.float64), u.astype(np.float64)
    sw = gd / (1.0 + np.exp(-gd)) * ud
    assert np.all(np.abs(h - sw) <= TOL * (np.abs(sw) + 1e-30)), "P4 SwiGLU"
    rq, rd = oracle.quantize_rows(h.reshape(-1, n_ff))
    assert np.array_equal(host(r["hq"]).reshape(-1, n_ff), rq), "P5 hq"
    assert np.array_equal(bits(r["hd"]).reshape(-1, n_ff // 32), rd), "P5 hd"
    return h_ref


@pytest.mark.parametrize("n_exp,n_ff,n_embd,n_tok,n_used", [
    (5, 64, 96, 3, 2), (8, 32, 64, 1, 8), (16, 96, 704, 9, 4), (128, 64, 2816, 1, 8),
    (4, 32, 32, 33, 2), (128, 704, 2816, 2, 8)])
def test_up_gate_routed(n_exp, n_ff, n_embd, n_tok, n_used):
    t, UG, DN, ids, p = _layer(n_exp, n_ff, n_embd, n_tok, n_used, seed=n_exp + n_tok)
    xq, xd = q8.quantize_row(t["x"].to(DEV))
    r = q8.moe_up_gate_swiglu(UG, xq, xd, ids, want_hq=True, want_gu=True)
    _check_up_gate(UG, xq, xd, ids, r)


@pytest.mark.parametrize("n_exp,n_ff,n_embd,n_tok,n_used", [(6, 64, 128, 5, 3), (1, 96, 256, 4, 1)])
def test_separate_gate_up_weights(n_exp, n_ff, n_embd, n_tok, n_used):
    """Separate gate and up weights packed by q8_pack_up_gate: bitwise the pack
    of their row concatenation; the fused step on it passes P3-P5, and its
    oracle value is the oracle's separate-weights path (two mul_mat_id, then
    silu(g) * u) on the separately quantized halves."""
    wg = synth.normal((n_exp, n_ff, n_embd), seed=500 + n_exp, std=0.02)
    wu = synth.normal((n_exp, n_ff, n_embd), seed=600 + n_exp, std=0.02)
    P = q8.pack_up_gate(wg.to(DEV), wu.to(DEV))
    C = q8.pack(torch.cat([wg, wu], dim=1).to(DEV))
    assert torch.equal(P.qs, C.qs)
    assert torch.equal(P.d.view(torch.int16), C.d.view(torch.int16))
    xq, xd = q8.quantize_row(synth.normal((n_tok, n_embd), seed=700 + n_tok).to(DEV))
    if n_exp == 1:
        ids = None
    else:
        ids = torch.stack([torch.randperm(n_exp, generator=torch.Generator().manual_seed(800 + t))
                           [:n_used] for t in range(n_tok)]).to(torch.int32).to(DEV)
    r = q8.moe_up_gate_swiglu(P, xq, xd, ids, want_hq=True, want_gu=True)
    h_ref = _check_up_gate(P, xq, xd, ids, r)
    gq, gd = oracle.quantize_rows(wg.numpy().reshape(-1, n_embd))
    uq, ud = oracle.quantize_rows(wu.numpy().reshape(-1, n_embd))
    sh_q, sh_d = (n_exp, n_ff, n_embd), (n_exp, n_ff, n_embd // 32)
    h_split = oracle.up_gate_swiglu_split(gq.reshape(sh_q), gd.reshape(sh_d), uq.reshape(sh_q),
                                          ud.reshape(sh_d), host(xq), bits(xd),
                                          None if ids is None else host(ids))
    assert np.array_equal(h_split, h_ref)


@pytest.mark.parametrize("n_ff,n_embd,n_tok", [(64, 128, 1), (96, 256, 8), (32, 64, 11)])
def test_up_gate_dense(n_ff, n_embd, n_tok):
    t, UG, DN, ids, p = _layer(1, n_ff, n_embd, n_tok, 1, seed=40 + n_tok)
    xq, xd = q8.quantize_row(t["x"].to(DEV))
    r = q8.moe_up_gate_swiglu(UG, xq, xd, None, want_hq=True, want_gu=True)
    _check_up_gate(UG, xq, xd, None, r)
    # dense == one expert with every id 0 (bitwise)
    ids0 = torch.zeros((n_tok, 1), dtype=torch.int32, device=DEV)
    r0 = q8.moe_up_gate_swiglu(UG, xq, xd, ids0, want_hq=True)
    assert torch.equal(r["h"], r0["h"]) and torch.equal(r["hq"], r0["hq"])


def test_halves_split_exactly():
    """g and u equal mul_mat_id / GEMV on the gate and up row views, bitwise."""
    t, UG, DN, ids, p = _layer(6, 64, 128, 4, 3, seed=7)
    xq, xd = q8.quantize_row(t["x"].to(DEV))
    r = q8.moe_up_gate_swiglu(UG, xq, xd, ids, want_gu=True)
    g2 = q8.mul_mat_id(UG.gate(), xq, xd, ids, a_per_slot=False)
    u2 = q8.mul_mat_id(UG.up(), xq, xd, ids, a_per_slot=False)
    assert torch.equal(r["g"], g2) and torch.equal(r["u"], u2)
    idh = host(ids)
    e = int(idh[1, 2])
    one = UG.row_view(e * UG.mat_stride, UG.rows // 2)
    one.n_mat = 1
    gv = q8.gemv(one, xq[1:2], xd[1:2])
    assert torch.equal(gv[0], r["g"][1, 2])
    # silu(g) * u recomputed from the views gives h within P4
    hh = host(g2).astype(np.float64)
    sw = hh / (1 + np.exp(-hh)) * host(u2)
    assert np.all(np.abs(host(r["h"]) - sw) <= TOL * (np.abs(sw) + 1e-30))


def test_routing_selects_named_experts():
    n_exp, n_ff, n_embd, n_tok, n_used = 12, 32, 64, 6, 3
    t, UG, DN, ids, p = _layer(n_exp, n_ff, n_embd, n_tok, n_used, seed=13)
    xq, xd = q8.quantize_row(t["x"].to(DEV))
    idh = host(ids)
    marker = int(idh[2, 1])
    w = t["up_gate"].clone()
    keep = w[marker].clone()
    w.zero_()
    w[marker] = keep
    Z = q8.pack(w.to(DEV))
    h = host(q8.moe_up_gate_swiglu(Z, xq, xd, ids)["h"])
    assert np.array_equal(np.any(h != 0, axis=2), idh == marker)
    # perturbing an expert that no token names leaves the output bitwise unchanged
    unused = sorted(set(range(n_exp)) - set(idh.ravel().tolist()))
    assert unused
    ref = q8.moe_up_gate_swiglu(UG, xq, xd, ids)["h"].clone()
    w2 = t["up_gate"].clone()
    w2[unused[0]] = -w2[unused[0]] * 3
    P2 = q8.pack(w2.to(DEV))
    assert torch.equal(q8.moe_up_gate_swiglu(P2, xq, xd, ids)["h"], ref)


def test_token_permutation_and_determinism():
    t, UG, DN, ids, p = _layer(16, 64, 128, 10, 4, seed=17)
    x = t["x"].to(DEV)
    out1 = q8.moe_ffn(UG, DN, x, ids, p)
    out2 = q8.moe_ffn(UG, DN, x, ids, p)
    assert torch.equal(out1.view(torch.int32), out2.view(torch.int32))
    perm = torch.randperm(10, generator=torch.Generator().manual_seed(3)).to(DEV)
    outp = q8.moe_ffn(UG, DN, x[perm].contiguous(), ids[perm].contiguous(), p[perm].contiguous())
    assert torch.equal(outp, out1[perm])


@pytest.mark.parametrize("a_per_slot", [True, False])
def test_mul_mat_id_p3(a_per_slot):
    n_mat, rows, k, n_tok, n_used = 9, 70, 704, 5, 4
    w = synth.normal((n_mat, rows, k), seed=901, std=0.02)
    W = q8.pack(w.to(DEV))
    na = n_tok * n_used if a_per_slot else n_tok
    a = synth.normal((na, k), seed=902)
    aq, ad = q8.quantize_row(a.to(DEV))
    ids = synth.routing_ids(n_tok, n_mat, n_used, seed=903).to(DEV)
    y = torch.full((n_tok, n_used, rows), float("nan"), device=DEV)
    q8.mul_mat_id(W, aq, ad, ids, a_per_slot=a_per_slot, y=y)
    wq, wd = _w_host(W)
    aqh, adh = host(aq), bits(ad)
    if a_per_slot:
        aqh, adh = aqh.reshape(n_tok, n_used, k), adh.reshape(n_tok, n_used, k // 32)
    ref = oracle.mul_mat_id(wq, wd, aqh, adh, host(ids), a_per_slot)
    yh = host(y)
    idh = host(ids)
    for t_ in range(n_tok):
        for s in range(n_used):
            e = idh[t_, s]
            arow = (aqh[t_, s], adh[t_, s]) if a_per_slot else (aqh[t_], adh[t_])
            S = S_norm(wq[e], wd[e], arow[0][None], arow[1][None])[0]
            assert_p3(yh[t_, s], ref[t_, s], S, "mul_mat_id")


def test_combine():
    y = synth.normal((7, 8, 2816), seed=950).to(DEV)
    pw = synth.routing_weights(7, 8, seed=951).to(DEV)
    out = host(q8.moe_combine(y, pw))
    ref = oracle.combine(host(y).astype(np.float64), host(pw))
    S = np.einsum("tk,tkr->tr", np.abs(host(pw)).astype(np.float64), np.abs(host(y)))
    assert np.all(np.abs(out - ref) <= 1e-6 * S)


@pytest.mark.parametrize("n_exp,n_ff,n_embd,n_tok,n_used", [(8, 64, 128, 3, 2),
                                                            (128, 704, 2816, 1, 8)])
def test_moe_ffn_staged(n_exp, n_ff, n_embd, n_tok, n_used):
    """The whole step equals the chain of separate calls bitwise; the chain is
    checked stage by stage (P1, P3-P5); the end-to-end difference from the
    oracle's own chain is reported (P6, not gated: a one-step int8 flip in h
    is allowed)."""
    t, UG, DN, ids, p = _layer(n_exp, n_ff, n_embd, n_tok, n_used, seed=60 + n_exp,
                               x_std=1.0)
    x = t["x"].to(DEV)
    out = q8.moe_ffn(UG, DN, x, ids, p)
    xq, xd = q8.quantize_row(x)
    rq, rd = oracle.quantize_rows(t["x"].numpy())
    assert np.array_equal(host(xq), rq) and np.array_equal(bits(xd), rd)
    r = q8.moe_up_gate_swiglu(UG, xq, xd, ids, want_hq=True, want_gu=True)
    _check_up_gate(UG, xq, xd, ids, r)
    hq2 = r["hq"].reshape(n_tok * n_used, n_ff)
    hd2 = r["hd"].reshape(n_tok * n_used, n_ff // 32)
    y = q8.mul_mat_id(DN, hq2, hd2, ids, a_per_slot=True)
    out2 = q8.moe_combine(y, p)
    assert torch.equal(out, out2)
    wq, wd = _w_host(DN)
    yr = oracle.mul_mat_id(wq, wd, host(hq2).reshape(n_tok, n_used, n_ff),
                           bits(hd2).reshape(n_tok, n_used, n_ff // 32), host(ids), True)
    idh = host(ids)
    for t_ in range(n_tok):
        for s in range(n_used):
            e = idh[t_, s]
            S = S_norm(wq[e], wd[e], host(hq2)[t_ * n_used + s][None],
                       bits(hd2)[t_ * n_used + s][None])[0]
            assert_p3(host(y)[t_, s], yr[t_, s], S, "down")
    # P6 (reported): the oracle's chain from x alone
    full = oracle.moe_ffn(*_w_host(UG), wq, wd, t["x"].numpy(), host(ids), host(p))
    rel = np.abs(host(out) - full["out"]).max() / (np.abs(full["out"]).max() + 1e-30)
    print(f"P6 end-to-end max |diff| / max |out| = {rel:.3e}")


def test_dense_ffn():
    t, UG, DN, ids, p = _layer(1, 64, 256, 2, 1, seed=81)
    x = t["x"].to(DEV)
    out = q8.moe_ffn(UG, DN, x)
    xq, xd = q8.quantize_row(x)
    r = q8.moe_up_gate_swiglu(UG, xq, xd, None, want_hq=True)
    y = q8.gemv(DN, r["hq"].reshape(2, 64), r["hd"].reshape(2, 2))
    assert torch.equal(out, y)


def test_poison_every_output_written():
    t, UG, DN, ids, p = _layer(32, 64, 128, 5, 4, seed=91)
    xq, xd = q8.quantize_row(t["x"].to(DEV))
    out = {"h": torch.full((5, 4, 64), float("nan"), device=DEV),
           "hq": torch.full((5, 4, 64), 0x7F, dtype=torch.int8, device=DEV),
           "hd": torch.full((5, 4, 2), float("nan"), dtype=torch.float16, device=DEV)}
    r = q8.moe_up_gate_swiglu(UG, xq, xd, ids, want_hq=True, out=out)
    assert not torch.isnan(r["h"]).any()
    assert not torch.isnan(r["hd"]).any()
    ref, _ = oracle.quantize_rows(host(r["h"]).reshape(-1, 64))
    assert np.array_equal(host(r["hq"]).reshape(-1, 64), ref)


def test_bad_ids_reported_without_fault():
    t, UG, DN, ids, p = _layer(8, 32, 64, 4, 2, seed=95)
    xq, xd = q8.quantize_row(t["x"].to(DEV))
    bad = ids.clone()
    bad[1, 0] = 8                      # out of range
    ws = q8.moe_workspace(4, 2, 8)
    q8.moe_up_gate_swiglu(UG, xq, xd, bad, ws=ws)
    with pytest.raises(q8.Q8Error) as ei:
        q8.check(ws)
    assert ei.value.name == "Q8_E_BAD_ID"
    rep = ids.clone()
    rep[2, 1] = rep[2, 0]              # repeated within a token
    q8.moe_up_gate_swiglu(UG, xq, xd, rep, ws=ws)
    with pytest.raises(q8.Q8Error):
        q8.check(ws)
    # the context is still usable, and a good call clears the report
    q8.moe_up_gate_swiglu(UG, xq, xd, ids, ws=ws)
    q8.check(ws)


TC_MIN_ROWS = 4  # the library's tensor-core threshold (routed rows per expert)


@pytest.mark.parametrize("n_exp,n_ff,n_embd,n_tok,n_used", [
    (128, 704, 2816, 1, 8), (128, 704, 2816, 16, 8), (16, 64, 128, 5, 4), (1, 64, 256, 3, 1),
    (32, 96, 2048, 33, 2)])
def test_fp32_entry_points_match_workspace_path(n_exp, n_ff, n_embd, n_tok, n_used):
    """The small-batch fp32 calls (quantize in the kernel, group in every CTA)
    give bitwise the results of quantize + grouping + the Q8_0 calls on the
    dp4a kernels: the up/gate reference asks for the g/u taps, which keep
    every expert on dp4a; in the down projection the experts with at least
    TC_MIN_ROWS rows take the tensor cores (P3 against the fp32 entry, whose
    dp4a sums differ only in the fp32 accumulation order), the rest bitwise."""
    t, UG, DN, ids, p = _layer(n_exp, n_ff, n_embd, n_tok, n_used, seed=300 + n_tok + n_exp)
    x = t["x"].to(DEV)
    xq, xd = q8.quantize_row(x)
    ref = q8.moe_up_gate_swiglu(UG, xq, xd, ids, want_hq=True, want_gu=True)
    h = q8.moe_up_gate_swiglu_fp32(UG, x, ids)
    assert torch.equal(h, ref["h"])
    if ids is not None:
        y = q8.mul_mat_id_fp32(DN, h.reshape(-1, n_ff), ids, True)
        hq, hd = ref["hq"].reshape(-1, n_ff), ref["hd"].reshape(-1, n_ff // 32)
        y2 = q8.mul_mat_id(DN, hq, hd, ids, True)
        counts = torch.bincount(ids.flatten().long(), minlength=n_exp)
        dp4a = counts[ids.long()] < TC_MIN_ROWS  # [n_tok, n_used]
        assert torch.equal(y[dp4a], y2[dp4a])
        wq, wd = _w_host(DN)
        hqh = host(hq).reshape(n_tok, n_used, n_ff)
        hdh = bits(hd).reshape(n_tok, n_used, n_ff // 32)
        idh, yh, y2h = host(ids), host(y), host(y2)
        for t_, s in zip(*np.nonzero(~host(dp4a))):
            e = idh[t_, s]
            S = S_norm(wq[e], wd[e], hqh[t_, s][None], hdh[t_, s][None])[0]
            assert np.all(np.abs(yh[t_, s] - y2h[t_, s]) <= 2 * TOL * S + 1e-30)
        # the whole step through q8_moe_ffn: up to 32 pairs one fused kernel
        # on dp4a (the fp32 chain's bits); above, the grouped Q8_0 calls
        # (tensor cores for the experts with at least TC_MIN_ROWS rows)
        out = q8.moe_ffn(UG, DN, x, ids, p)
        if n_tok * n_used <= 32:
            assert torch.equal(out, q8.moe_combine(y, p))
        else:
            r2 = q8.moe_up_gate_swiglu(UG, xq, xd, ids, want_hq=True)
            y3 = q8.mul_mat_id(DN, r2["hq"].reshape(-1, n_ff),
                               r2["hd"].reshape(-1, n_ff // 32), ids, True)
            assert torch.equal(out, q8.moe_combine(y3, p))


def test_fp32_entry_reports_bad_ids():
    t, UG, DN, ids, p = _layer(8, 32, 64, 4, 2, seed=97)
    x = t["x"].to(DEV)
    err = torch.zeros(1, dtype=torch.int32, device=DEV)
    q8.moe_up_gate_swiglu_fp32(UG, x, ids, err_word=err)
    assert int(err.item()) == 0
    bad = ids.clone()
    bad[3, 1] = -1
    q8.moe_up_gate_swiglu_fp32(UG, x, bad, err_word=err)
    assert int(err.item()) != 0
    rep = ids.clone()
    rep[0, 1] = rep[0, 0]
    q8.mul_mat_id_fp32(DN, torch.zeros((8, 32), device=DEV), rep, True, err_word=err)
    assert int(err.item()) != 0
