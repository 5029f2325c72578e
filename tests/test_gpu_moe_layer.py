"""GPU parity of the fused MoE layer kernel: q8_moe_ffn runs small routed
batches (at most 32 pairs) as one cooperative kernel (grouping, up/gate +
SwiGLU, grid barrier, down projection + combine).  Its output must be bitwise
the chain of separate calls (same row sums, same h quantization, same combine
order), whose stages are pinned to the oracle elsewhere; here the down outputs
are also held to the oracle with P3 on sampled rows, the barrier words must be
left on a multiple of the grid size, repeated calls must agree, and bad ids must be reported."""
import numpy as np
import pytest
import torch

import oracle
from helpers import S_norm, TOL, bits, canon_d, host
from moe_up_gate_b200 import q8, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _layer(n_exp, n_ff, n_embd, n_tok, n_used, seed, x_std=1.0):
    shape = synth.MoeShape(n_embd=n_embd, n_ff=n_ff, n_exp=n_exp, n_used=n_used)
    t = synth.moe_layer_tensors(seed, 0, shape, n_tok, x_std)
    UG = q8.pack(t["up_gate"].to(DEV))
    DN = q8.pack(t["down"].to(DEV))
    return t, UG, DN, t["ids"].to(DEV), t["p"].to(DEV)


def _chain(UG, DN, x, ids, p):
    n_ff = UG.rows // 2
    xq, xd = q8.quantize_row(x)
    r = q8.moe_up_gate_swiglu(UG, xq, xd, ids, want_hq=True)
    y = q8.mul_mat_id(DN, r["hq"].reshape(-1, n_ff), r["hd"].reshape(-1, n_ff // 32), ids, True)
    return q8.moe_combine(y, p), r, y


@pytest.mark.parametrize("n_exp,n_ff,n_embd,n_tok,n_used", [
    (128, 704, 2816, 1, 8),     # one decode token of the MoE layer
    (128, 704, 2816, 2, 8),
    (128, 704, 2816, 4, 8),     # 32 pairs: the largest fused batch
    (16, 64, 128, 5, 4),        # whole-row tiles of 32 rows (k <= 1024)
    (8, 96, 4096, 3, 2),        # k at the whole-row limit
    (3, 32, 64, 7, 3),          # more pairs per expert than rows per pass
    (512, 64, 256, 1, 32),      # 32 experts of one token: four phase-B groups
])
def test_fused_layer_equals_chain(n_exp, n_ff, n_embd, n_tok, n_used):
    t, UG, DN, ids, p = _layer(n_exp, n_ff, n_embd, n_tok, n_used, seed=900 + n_tok + n_exp)
    x = t["x"].to(DEV)
    ws = q8.moe_ffn_workspace(n_tok, n_used, n_exp, n_embd, n_ff, DEV)
    out = torch.full((n_tok, n_embd), float("nan"), device=DEV)
    q8.moe_ffn(UG, DN, x, ids, p, ws=ws, out=out)
    q8.check(ws)
    ref, r, y = _chain(UG, DN, x, ids, p)
    assert torch.equal(out, ref)
    # again with the same workspace: the barrier counter was left on a multiple of the grid
    out2 = q8.moe_ffn(UG, DN, x, ids, p, ws=ws)
    assert torch.equal(out2, out)
    # P3 on the down outputs of sampled rows against the oracle (from the
    # chain's hq, bit-identical to the fused kernel's by the equality above)
    wq = host(DN.qs).reshape(n_exp, n_embd, n_ff)
    wd = canon_d(DN.d, n_ff).reshape(n_exp, n_embd, n_ff // 32)
    hq = host(r["hq"]).reshape(n_tok, n_used, n_ff)
    hd = bits(r["hd"]).reshape(n_tok, n_used, n_ff // 32)
    idh, ph = host(ids), host(p).astype(np.float64)
    rows = np.unique(np.linspace(0, n_embd - 1, 9).astype(int))
    for tok in range(n_tok):
        ref_out = np.zeros(len(rows))
        bound = np.zeros(len(rows))
        for s in range(n_used):
            e = idh[tok, s]
            yr = oracle.mul_mat_id(wq[e:e + 1, rows], wd[e:e + 1, rows], hq[tok:tok + 1, s:s + 1],
                                   hd[tok:tok + 1, s:s + 1], np.zeros((1, 1), np.int32), True)[0, 0]
            S = S_norm(wq[e, rows], wd[e, rows], hq[tok, s][None], hd[tok, s][None])[0]
            ref_out += ph[tok, s] * yr
            # P3 on y, plus the fp32 rounding of the combine's fma chain
            bound += abs(ph[tok, s]) * (TOL * S + 1e-6 * np.abs(yr) + 1e-30)
        got = host(out)[tok, rows].astype(np.float64)
        assert np.all(np.abs(got - ref_out) <= bound), tok


def test_fused_layer_many_calls_one_workspace():
    """Layers of a decode step reuse one workspace back to back (the grid
    barrier's arrival counter keeps counting, a multiple of the grid between
    calls)."""
    t, UG, DN, ids, p = _layer(128, 704, 2816, 1, 8, seed=931)
    x = t["x"].to(DEV)
    ws = q8.moe_ffn_workspace(1, 8, 128, 2816, 704, DEV)
    outs = [q8.moe_ffn(UG, DN, x, ids, p, ws=ws) for _ in range(20)]
    q8.check(ws)
    for o in outs[1:]:
        assert torch.equal(o, outs[0])


def test_fused_layer_reports_bad_ids():
    t, UG, DN, ids, p = _layer(16, 64, 128, 3, 4, seed=941)
    x = t["x"].to(DEV)
    ws = q8.moe_ffn_workspace(3, 4, 16, 128, 64, DEV)
    bad = ids.clone()
    bad[1, 2] = 16
    q8.moe_ffn(UG, DN, x, bad, p, ws=ws)
    with pytest.raises(q8.Q8Error) as ei:
        q8.check(ws)
    assert ei.value.name == "Q8_E_BAD_ID"
    rep = ids.clone()
    rep[0, 3] = rep[0, 1]
    q8.moe_ffn(UG, DN, x, rep, p, ws=ws)
    with pytest.raises(q8.Q8Error):
        q8.check(ws)
    # the device stays usable and a good call clears the report
    out = q8.moe_ffn(UG, DN, x, ids, p, ws=ws)
    q8.check(ws)
    assert torch.equal(out, _chain(UG, DN, x, ids, p)[0])


def test_workspace_serves_a_large_then_a_small_call():
    """One workspace sized for a 256-token call serves a 1-token call next
    (and back again): the large call's grouping tables cover much of the
    workspace, but the fused layer kernel's grid-barrier words have a fixed
    place in the header that no grouping writes, so the small call's barrier
    starts from zero.  The results equal those on fresh workspaces."""
    shape = synth.MOE_LAYER
    big = synth.moe_layer_tensors(951, 0, shape, 256, 1.0, device=DEV)
    UG = q8.pack(big["up_gate"])
    DN = q8.pack(big["down"])
    small = synth.moe_layer_tensors(952, 0, shape, 1, 1.0)
    xs, ids_s, p_s = small["x"].to(DEV), small["ids"].to(DEV), small["p"].to(DEV)
    xb, ids_b, p_b = big["x"], big["ids"].to(DEV), big["p"].to(DEV)
    ws = q8.moe_ffn_workspace(256, 8, 128, 2816, 704, DEV)
    ref_small = q8.moe_ffn(UG, DN, xs, ids_s, p_s)  # fresh workspaces
    ref_big = q8.moe_ffn(UG, DN, xb, ids_b, p_b)
    for _ in range(3):
        out_b = q8.moe_ffn(UG, DN, xb, ids_b, p_b, ws=ws)
        out_s = q8.moe_ffn(UG, DN, xs, ids_s, p_s, ws=ws)
        q8.check(ws)
        assert torch.equal(out_b, ref_big)
        assert torch.equal(out_s, ref_small)
