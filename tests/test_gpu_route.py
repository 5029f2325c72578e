"""GPU parity of the router (q8_route) against the oracle's router_logits and
route: the logits (fp64 sums) within 1e-12 of sum |w x|; the selected ids
equal where the oracle's margin at the cut (the n_used-th largest logit
minus the next) is wider than the logits' tolerance, and otherwise a valid
top-n_used by the tolerance; the routing weights within 1e-6 relative (both
sides softmax in fp64; the GPU stores fp32).  Special cases: exact ties
(duplicated router rows; all rows equal) go by ascending expert index,
n_used == 1 gives weight 1, n_used == n_exp selects every expert in order,
ragged token groups, and the ids feed q8_moe_ffn directly."""
import numpy as np
import pytest
import torch

import oracle
from helpers import host
from moe_up_gate_b200 import q8, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
LG_TOL = 1e-12


def _check(w, x, n_used, ids, rw, lg):
    wh, xh = host(w).astype(np.float64), host(x).astype(np.float64)
    ref_lg = oracle.router_logits(host(w), host(x))
    S = np.abs(xh) @ np.abs(wh).T
    assert np.all(np.abs(host(lg) - ref_lg) <= LG_TOL * S + 1e-300)
    ref_ids, ref_p = oracle.route(ref_lg, n_used)
    gi, gp = host(ids), host(rw).astype(np.float64)
    for t in range(ref_lg.shape[0]):
        srt = np.sort(ref_lg[t])[::-1]
        tol = 2 * LG_TOL * S[t].max()
        margin = srt[n_used - 1] - srt[n_used] if n_used < ref_lg.shape[1] else np.inf
        if margin > tol:
            assert list(gi[t]) == list(ref_ids[t]), t
            assert np.all(np.abs(gp[t] - ref_p[t]) <= 1e-6 * ref_p[t] + 1e-12), t
        else:  # a near tie at the cut: any valid top-n_used
            assert len(set(gi[t])) == n_used
            assert ref_lg[t, gi[t]].min() >= srt[n_used - 1] - tol
        assert abs(gp[t].sum() - 1.0) <= 1e-5


@pytest.mark.parametrize("n_tok,n_embd,n_exp,n_used", [
    (1, 2816, 128, 8),       # one decode token of the MoE layer's router
    (16, 2816, 128, 8),
    (256, 2816, 128, 8),     # the largest batch of the sweep
    (7, 64, 16, 4),          # ragged token groups (4 per cluster)
    (5, 4096, 1024, 32),     # the most experts and the most per token
    (3, 128, 9, 9),          # n_used == n_exp: every expert, in order
    (4, 96, 33, 1),          # n_used == 1: weight 1
    (7, 8192, 32, 4),        # rows long enough that 3 tokens share a cluster
    (2, 16384, 64, 8),       # the longest rows: one token per cluster
])
def test_route_matches_oracle(n_tok, n_embd, n_exp, n_used):
    w = synth.normal((n_exp, n_embd), seed=1300 + n_exp, std=synth.W_STD).to(DEV)
    x = synth.normal((n_tok, n_embd), seed=1301 + n_tok).to(DEV)
    ids, rw, lg = q8.route(w, x, n_used, want_logits=True)
    torch.cuda.synchronize()
    _check(w, x, n_used, ids, rw, lg)
    if n_used == 1:
        assert torch.all(rw == 1.0)
    if n_used == n_exp:
        ref_ids, _ = oracle.route(host(lg), n_used)
        assert np.array_equal(host(ids), ref_ids)
    # deterministic, and the logits output is optional
    ids2, rw2 = q8.route(w, x, n_used)
    assert torch.equal(ids, ids2) and torch.equal(rw, rw2)


def test_route_exact_ties_by_ascending_index():
    n_embd, n_exp, n_used = 256, 64, 8
    w = synth.normal((n_exp, n_embd), seed=1310, std=synth.W_STD)
    x = synth.normal((6, n_embd), seed=1311)
    # experts 9 and 41 get the same (largest) row: equal logits, 9 first
    big = w[0].abs() * 10 * torch.sign(x[0])
    w[9] = big
    w[41] = big
    w, x = w.to(DEV), x.to(DEV)
    ids, rw, lg = q8.route(w, x, n_used, want_logits=True)
    lgh = host(lg)
    assert np.array_equal(lgh[:, 9], lgh[:, 41])
    assert list(host(ids)[0][:2]) == [9, 41]
    assert host(rw)[0][0] == host(rw)[0][1]
    _check(w, x, n_used, ids, rw, lg)
    # every row equal: every logit ties, the first n_used experts are taken
    weq = w[3:4].expand(n_exp, n_embd).contiguous()
    ids, rw = q8.route(weq, x, n_used)
    assert np.array_equal(host(ids), np.tile(np.arange(n_used, dtype=np.int32), (6, 1)))
    assert np.allclose(host(rw), 1.0 / n_used, rtol=1e-7)


def test_route_feeds_the_ffn():
    """Router -> q8_moe_ffn: the fused layer consumes the router's ids and
    weights (the same as feeding them from the host)."""
    shape = synth.MOE_LAYER
    t = synth.moe_layer_tensors(1320, 0, shape, 2, 1.0)
    UG = q8.pack(t["up_gate"].to(DEV))
    DN = q8.pack(t["down"].to(DEV))
    w = synth.normal((shape.n_exp, shape.n_embd), seed=1321, std=synth.W_STD).to(DEV)
    x = t["x"].to(DEV)
    ids, rw = q8.route(w, x, shape.n_used)
    out = q8.moe_ffn(UG, DN, x, ids, rw)
    ids_h, rw_h = ids.cpu().to(DEV), rw.cpu().to(DEV)
    out2 = q8.moe_ffn(UG, DN, x, ids_h, rw_h)
    assert torch.equal(out, out2)
    ref_ids, _ = oracle.route(oracle.router_logits(host(w), host(x)), shape.n_used)
    assert np.array_equal(host(ids), ref_ids)
