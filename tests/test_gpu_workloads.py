"""GPU parity of every benchmarked workload at its full size, in the launch
configuration bench.py times: the workloads are built by bench.py's own
classes (same seeds, same packed weights, same public calls, same kernels and
kernel instances), issued once, and their outputs compared with the oracle.

  config 1  the 768 x 768 GEMV (q8_gemv_batched, one problem, batch 1)
  config 2  the 85 matvecs of a Llama-2-110M-shaped decode step, every
            output element, in one q8_gemv_batched launch (gemv_batched_kernel
            with one activation row per pass, the host's equal-cost tile
            split over 85 problems, the 32000 x 768 classifier in the batch)
  config 3  the dense 4096 / 14336 feed-forward step at 1 and 8 tokens (the
            fp32 up/gate kernel at n_ff 14336, then the fp32-staged down
            projection at K = 14336, which splits each row over 8 warps)
  config 4  the MoE layer at 1 token (the fused layer kernel) and 16 tokens
  config 5  the 30-layer sweep at 1 / 4 / 16 / 64 / 256 tokens (layers 0 and
            29 of the sweep, built with their own seeds)

The rule is the staged parity rule of the other GPU tests: P1 on the packed
weights, P3 on every matmul output given the same quantized inputs, the bound
P3 on g and u implies for h, P5 on h -> Q8_0, and the combine held to the
fp32 rounding of its fma chain.
"""
import os
import sys

import numpy as np
import pytest
import torch

import oracle
from helpers import S_norm, TOL, assert_p3, bits, canon_d, host
from moe_up_gate_b200 import q8, synth

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)
import bench  # noqa: E402

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _check_gemv_set(wl):
    """Every output of every problem of a LlamaDecode workload, on every
    rotating weight copy (the first against the oracle, the others bitwise)."""
    wl.oracle_setup()  # the oracle's own Q8_0 of the same fp32 weights
    for (wq, wd), W in zip(wl.ow, wl.W[0]):
        assert np.array_equal(host(W.qs), wq)  # P1
        assert np.array_equal(canon_d(W.d, W.k), wd)
    first = None
    for copy in range(wl.copies):
        for y in wl.y:
            y.fill_(float("nan"))
        wl.issue(copy, bench.NoMarks())
        torch.cuda.synchronize()
        got = [host(y).copy() for y in wl.y]
        if first is None:
            first = got
            for (name, rows, k), (wq, wd), x, yg in zip(wl.mats, wl.ow, wl.ox, got):
                xq, xd = oracle.quantize_rows(x)
                ref = oracle.gemv(wq, wd, xq, xd)
                assert not np.isnan(yg).any(), name
                assert_p3(yg, ref, S_norm(wq, wd, xq, xd), f"{wl.name} {name} {rows}x{k}")
        else:
            for a, b in zip(first, got):
                assert np.array_equal(a.view(np.int32), b.view(np.int32))


def test_config1_gemv_768():
    _check_gemv_set(bench.LlamaDecode(DEV, gemv768=True))


def test_config2_llama_decode_all_matvecs():
    wl = bench.LlamaDecode(DEV)
    assert len(wl.mats) == 85 and wl.mats[-1] == ("classifier", 32000, 768)
    _check_gemv_set(wl)


def _h_bound(g, u, h_ref, Sg, Su):
    sg = g / (1 + np.exp(-g))
    return TOL * (1.2 * np.abs(u) * Sg + np.abs(sg) * Su) + 1e-6 * np.abs(h_ref) + 1e-30


@pytest.mark.parametrize("T", [1, 8])
def test_config3_dense_ffn_full_size(T):
    wl = bench.MoeWorkload(DEV, "dense_ffn", T)
    D, F = synth.DENSE_FFN.n_embd, synth.DENSE_FFN.n_ff
    wl.h.fill_(float("nan"))
    wl.out.fill_(float("nan"))
    wl.issue(0, bench.NoMarks())
    torch.cuda.synchronize()
    UG, DN = wl.L[0]
    x = wl.x_host[0][0].numpy()
    xq, xd = oracle.quantize_rows(x)
    wq, wd = host(UG.qs), canon_d(UG.d, D)
    h_ref, g_ref, u_ref = oracle.up_gate_swiglu(wq, wd, xq, xd, None, want_gu=True)
    h = host(wl.h).reshape(T, F).astype(np.float64)
    Sg = S_norm(wq[:F], wd[:F], xq, xd)
    Su = S_norm(wq[F:], wd[F:], xq, xd)
    bound = _h_bound(g_ref[:, 0], u_ref[:, 0], h_ref[:, 0], Sg, Su)
    assert np.all(np.abs(h - h_ref[:, 0]) <= bound)
    # the down projection takes h quantized by the Q8_0 rule (P5: bitwise the
    # oracle's quantization of the GPU's h, checked where h is quantized once
    # before the GEMV) and P3 on its output
    hq, hd = oracle.quantize_rows(host(wl.h).reshape(T, F))
    if wl.h_once:
        assert np.array_equal(host(wl.hq).reshape(T, F), hq)
        assert np.array_equal(bits(wl.hd).reshape(T, F // 32), hd)
    dq, dd = host(DN.qs), canon_d(DN.d, F)
    y_ref = oracle.gemv(dq, dd, hq, hd)
    assert_p3(host(wl.out)[0], y_ref, S_norm(dq, dd, hq, hd), f"dense down T={T}")
    # the public whole-step call runs the same kernels: bitwise the same output
    out2 = q8.moe_ffn(UG, DN, wl.x[0][0])
    assert torch.equal(out2, wl.out[0])


def _check_moe_layer(UG, DN, x, ids, p, out, tokens):
    """out: the workload's output of one layer; checked bitwise against the
    chain of separate public calls, whose stages are held to the oracle on the
    sampled tokens."""
    n_exp, F, D = UG.n_mat, UG.rows // 2, UG.k
    xq, xd = q8.quantize_row(x)
    r = q8.moe_up_gate_swiglu(UG, xq, xd, ids, want_hq=True)
    y = q8.mul_mat_id(DN, r["hq"].reshape(-1, F), r["hd"].reshape(-1, F // 32), ids, True)
    ref_out = q8.moe_combine(y, p)
    assert torch.equal(out, ref_out)
    ugq = host(UG.qs).reshape(n_exp, 2 * F, D)
    ugd = canon_d(UG.d, D).reshape(n_exp, 2 * F, D // 32)
    dnq = host(DN.qs).reshape(n_exp, D, F)
    dnd = canon_d(DN.d, F).reshape(n_exp, D, F // 32)
    xqh, xdh, idh, ph = host(xq), bits(xd), host(ids), host(p).astype(np.float64)
    hh, hqh, hdh, yh = host(r["h"]), host(r["hq"]), bits(r["hd"]), host(y)
    oh = host(out).astype(np.float64)
    # P5 on every pair
    rq, rd = oracle.quantize_rows(hh.reshape(-1, F))
    assert np.array_equal(hqh.reshape(-1, F), rq) and np.array_equal(hdh.reshape(-1, F // 32), rd)
    for tok in tokens:
        sub = idh[tok:tok + 1]
        h_ref, g_ref, u_ref = oracle.up_gate_swiglu(ugq, ugd, xqh[tok:tok + 1], xdh[tok:tok + 1],
                                                    sub, want_gu=True)
        y_ref = oracle.mul_mat_id(dnq, dnd, hqh[tok][None], hdh[tok][None], sub, True)
        want = np.zeros(D)
        bound = np.zeros(D)
        for s in range(sub.shape[1]):
            e = sub[0, s]
            Sg = S_norm(ugq[e, :F], ugd[e, :F], xqh[tok:tok + 1], xdh[tok:tok + 1])[0]
            Su = S_norm(ugq[e, F:], ugd[e, F:], xqh[tok:tok + 1], xdh[tok:tok + 1])[0]
            hb = _h_bound(g_ref[0, s], u_ref[0, s], h_ref[0, s], Sg, Su)
            assert np.all(np.abs(hh[tok, s] - h_ref[0, s]) <= hb), (tok, s)
            S = S_norm(dnq[e], dnd[e], hqh[tok, s][None], hdh[tok, s][None])[0]
            assert_p3(yh[tok, s], y_ref[0, s], S, f"down t={tok} s={s}")
            want += ph[tok, s] * y_ref[0, s]
            bound += abs(ph[tok, s]) * (TOL * S + 1e-6 * np.abs(y_ref[0, s]) + 1e-30)
        assert np.all(np.abs(oh[tok] - want) <= bound), tok


def _issue_and_check(wl, tokens):
    wl.out.fill_(float("nan"))
    wl.issue(0, bench.NoMarks())
    torch.cuda.synchronize()
    for li, (UG, DN) in enumerate(wl.L):
        _check_moe_layer(UG, DN, wl.x[0][li], wl.ids[0][li], wl.p[0][li], wl.out[li], tokens)


@pytest.mark.parametrize("T", [1, 16])
def test_config4_moe_layer(T):
    wl = bench.MoeWorkload(DEV, "moe_layer", T)
    assert wl.fused == (T == 1)
    _issue_and_check(wl, sorted({0, T // 2, T - 1}))


_SWEEP_PACKED = {}


@pytest.mark.parametrize("T", list(synth.MOE_SWEEP_TOKENS))
def test_config5_sweep_layers(T):
    """Layers 0 and 29 of the 30-layer sweep (their own seeds) at every token
    count of the sweep, through the calls and kernels the sweep times."""
    wl = bench.MoeWorkload(DEV, "moe_30layer", T, layer_ids=[0, 29],
                           packed=_SWEEP_PACKED.get("L"))
    _SWEEP_PACKED["L"] = wl.L
    if T == 256:  # the seeded batch sends some experts to the tensor cores
        counts = torch.bincount(wl.ids[0][0].flatten().long(), minlength=128)
        assert int((counts >= 16).sum()) > 0
    _issue_and_check(wl, sorted({0, T // 2, T - 1}))
    if T == synth.MOE_SWEEP_TOKENS[-1]:
        _SWEEP_PACKED.clear()


def test_llama_ffn_separate_gate_up_fused():
    """The Llama-2-110M feed-forward layers with separate gate (w1) and up
    (w3) weights: packed once into the combined up/gate tensor, they run as
    one dense fused up/gate + SwiGLU per layer, then w2.  h is held to the
    oracle's separate-weights path (two GEMVs, then silu(g) * u), the down
    projection to P3 on the oracle's quantization of the GPU's h."""
    wl = bench.MoeWorkload(DEV, "llama2_110m_ffn", 1, layer_ids=[0, 11])
    D, F = synth.LLAMA_DIM, synth.LLAMA_HIDDEN
    wl.h.fill_(float("nan"))
    wl.out.fill_(float("nan"))
    hs = []
    # the workload shares one h buffer across layers: issue layer by layer
    for li, l in enumerate(wl.layer_ids):
        UG, DN = wl.L[li]
        t = synth.llama_ffn_tensors(l, 1, device=DEV)
        gq, gd = oracle.quantize_rows(t["w1"].cpu().numpy())
        uq, ud = oracle.quantize_rows(t["w3"].cpu().numpy())
        # P1: the combined tensor holds the gate rows, then the up rows
        assert np.array_equal(host(UG.qs)[:F], gq) and np.array_equal(host(UG.qs)[F:], uq)
        assert np.array_equal(canon_d(UG.d, D)[:F], gd) and np.array_equal(canon_d(UG.d, D)[F:], ud)
        x = wl.x[0][li]  # the workload's own input (drawn on the host)
        h = q8.moe_up_gate_swiglu_fp32(UG, x, None)
        out = torch.full((1, D), float("nan"), device=DEV)
        q8.gemv_batched([(DN, h.reshape(1, F), out)], n_tok=1)
        torch.cuda.synchronize()
        xq, xd = oracle.quantize_rows(x.cpu().numpy())
        h_ref, g_ref, u_ref = oracle.up_gate_swiglu_split(gq, gd, uq, ud, xq, xd, None,
                                                          want_gu=True)
        Sg = S_norm(gq, gd, xq, xd)
        Su = S_norm(uq, ud, xq, xd)
        bound = _h_bound(g_ref[:, 0], u_ref[:, 0], h_ref[:, 0], Sg, Su)
        assert np.all(np.abs(host(h).reshape(1, F) - h_ref[:, 0]) <= bound)
        hq, hd = oracle.quantize_rows(host(h).reshape(1, F))
        dq, dd = oracle.quantize_rows(t["w2"].cpu().numpy())
        assert np.array_equal(host(DN.qs), dq)
        y_ref = oracle.gemv(dq, dd, hq, hd)
        assert_p3(host(out), y_ref, S_norm(dq, dd, hq, hd), f"w2 layer {l}")
        hs.append(out)
    # the workload's own step gives the same outputs (the last layer's h is
    # the shared buffer's final content)
    wl.issue(0, bench.NoMarks())
    torch.cuda.synchronize()
    for li in range(len(wl.layer_ids)):
        assert torch.equal(wl.out[li], hs[li])
