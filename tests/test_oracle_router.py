"""Pins for the oracle's router (CPU only): top-n_used selection with its tie
rule and the softmax over the selected logits, plus the router logits.

What pins what:
  * selection: brute force by counting -- an expert is selected iff fewer than
    n_used experts beat it (a larger logit, or an equal logit and a lower
    index) -- and its rank is that count; all-equal logits pick 0..n_used-1.
  * softmax: closed form (logits 0 and ln 3 give 3/4 and 1/4), p sums to 1,
    ratios p_i / p_j = exp(l_i - l_j), a shift of every logit changes
    nothing, n_used == 1 gives 1.
  * logits: an explicit Python sum of products (math.fsum) on tiny shapes.
  * mutants: a higher-index tie rule, a softmax over all experts and an
    ascending order each fail one of these pins.
"""
import math

import numpy as np

import oracle


def _brute(lg, n_used):
    n_exp = lg.shape[0]
    rank = {}
    for e in range(n_exp):
        beaten_by = sum(1 for f in range(n_exp) if lg[f] > lg[e] or (lg[f] == lg[e] and f < e))
        if beaten_by < n_used:
            rank[beaten_by] = e
    return [rank[r] for r in range(n_used)]


def _selection_ok(route_fn, lg, n_used):
    ids, _ = route_fn(lg, n_used)
    return all(list(ids[t]) == _brute(lg[t], n_used) for t in range(lg.shape[0]))


def _softmax_ok(route_fn, lg, n_used):
    ids, p = route_fn(lg, n_used)
    for t in range(lg.shape[0]):
        if abs(p[t].sum() - 1.0) > 1e-14:
            return False
        sel = lg[t, ids[t]]
        if not np.allclose(p[t] / p[t][0], np.exp(sel - sel[0]), rtol=1e-13, atol=0):
            return False
    return True


def test_selection_brute_force():
    rng = np.random.default_rng(3)
    for n_exp, n_used in [(5, 2), (8, 8), (16, 4), (12, 1)]:
        lg = rng.standard_normal((20, n_exp))
        lg[:, 1] = lg[:, 3]                        # an exact tie in every row
        lg[::4, :] = np.round(lg[::4, :])          # many ties in some rows
        assert _selection_ok(oracle.route, lg, n_used)


def test_all_equal_logits_pick_lowest_indices():
    ids, p = oracle.route(np.zeros((3, 10)), 4)
    assert np.array_equal(ids, np.tile(np.arange(4, dtype=np.int32), (3, 1)))
    assert np.allclose(p, 0.25, rtol=0, atol=1e-16)


def test_softmax_closed_form_and_invariants():
    ids, p = oracle.route(np.array([[0.0, math.log(3.0), -5.0]]), 2)
    assert list(ids[0]) == [1, 0]
    assert abs(p[0, 0] - 0.75) < 1e-15 and abs(p[0, 1] - 0.25) < 1e-15
    rng = np.random.default_rng(9)
    lg = rng.standard_normal((12, 32)) * 3.0
    assert _softmax_ok(oracle.route, lg, 8)
    ids2, p2 = oracle.route(lg + 1000.0, 8)
    ids1, p1 = oracle.route(lg, 8)
    assert np.array_equal(ids1, ids2) and np.allclose(p1, p2, rtol=1e-12, atol=0)
    _, p_one = oracle.route(lg, 1)
    assert np.array_equal(p_one, np.ones((12, 1)))


def test_router_logits_explicit_sum():
    rng = np.random.default_rng(11)
    w = rng.standard_normal((5, 7)).astype(np.float32)
    x = rng.standard_normal((3, 7)).astype(np.float32)
    lg = oracle.router_logits(w, x)
    for t in range(3):
        for e in range(5):
            ref = math.fsum(float(w[e, i]) * float(x[t, i]) for i in range(7))
            assert abs(lg[t, e] - ref) <= 1e-14 * math.fsum(abs(float(w[e, i]) * float(x[t, i]))
                                                             for i in range(7))


def test_pins_catch_plausible_mistakes():
    def tie_high(lg, n_used):   # equal logits by descending index
        n_tok, n_exp = lg.shape
        ids = np.array([sorted(range(n_exp), key=lambda e: (-lg[t, e], -e))[:n_used]
                        for t in range(n_tok)], np.int32)
        return ids, oracle.route(lg, n_used)[1]

    def softmax_all(lg, n_used):   # normalised over every expert, not the selected
        ids, _ = oracle.route(lg, n_used)
        ex = np.exp(lg - lg.max(axis=1, keepdims=True))
        full = ex / ex.sum(axis=1, keepdims=True)
        return ids, np.take_along_axis(full, ids.astype(np.int64), axis=1)

    def ascending(lg, n_used):     # smallest logits first
        ids, p = oracle.route(-lg, n_used)
        return ids, p

    rng = np.random.default_rng(17)
    lg = np.round(rng.standard_normal((16, 10)), 1)
    assert _selection_ok(oracle.route, lg, 3) and _softmax_ok(oracle.route, lg, 3)
    assert not _selection_ok(tie_high, lg, 3)
    assert not _softmax_ok(softmax_all, lg, 3)
    assert not _selection_ok(ascending, lg, 3)
