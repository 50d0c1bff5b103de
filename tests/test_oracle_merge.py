"""Pins of the oracle's log-sum-exp merge of attention partials (the
exchange step of a context-parallel decode: each GPU attends over its own
slice of a sequence's resident tokens, then the partials are combined).

(1) Splitting the resident tokens into disjoint slices, decoding each slice
    (the other tokens marked dropped) and merging gives the decode over all
    tokens: softmax over a union factors into the slices' normalised sums
    weighted by their denominators exp(lse_r);
(2) one partial is returned unchanged;
(3) empty partials (lse = -inf) carry no weight, and all-empty gives 0 / -inf;
(4) a two-partial case computed by hand."""
import math

import numpy as np
import pytest

import oracle
from long_context_decode_ada_b200 import workloads as wl


def decode_on(w, tier):
    return oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, tier, w.q, w.q_dtype)


@pytest.mark.parametrize("R", [2, 3, 5])
def test_merge_of_slices_equals_full_decode(R):
    lens = [300, 170, 41]
    w = wl.custom(21, 3, 2, 4, 16, lens, wl.MODE_QUOTA,
                  quota=[[T // 4, T // 3, T // 4] for T in lens])
    tier = oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, None,
                           w.mode, w.budget, w.quota)
    out, lse = decode_on(w, tier)
    cuts = np.linspace(0, w.Tmax, R + 1).astype(int)
    outs, lses = [], []
    for r in range(R):
        tr = np.full_like(tier, 3)
        tr[:, :, cuts[r]:cuts[r + 1]] = tier[:, :, cuts[r]:cuts[r + 1]]
        o, l = decode_on(w, tr)
        outs.append(o)
        lses.append(l)
    mo, ml = oracle.merge_partials(outs, lses)
    np.testing.assert_allclose(mo, out, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(ml, lse, rtol=1e-13, atol=1e-13)


def test_single_partial_is_unchanged():
    rng = np.random.default_rng(1)
    o = rng.standard_normal((1, 3, 4, 8))
    l = rng.standard_normal((1, 3, 4)) * 5
    mo, ml = oracle.merge_partials(o, l)
    np.testing.assert_allclose(mo, o[0], rtol=1e-15, atol=1e-15)
    np.testing.assert_allclose(ml, l[0], rtol=1e-15, atol=1e-15)


def test_empty_partials_carry_no_weight():
    rng = np.random.default_rng(2)
    o = rng.standard_normal((3, 2, 8))
    l = rng.standard_normal((3, 2))
    l[1, 0] = -np.inf
    o[1, 0] = np.nan          # an empty partial's out is never read
    mo, ml = oracle.merge_partials(o, l)
    ref_o, ref_l = oracle.merge_partials(o[[0, 2], 0:1], l[[0, 2], 0:1])
    np.testing.assert_allclose(mo[0], ref_o[0], rtol=1e-15)
    assert ml[0] == pytest.approx(ref_l[0], rel=1e-15)
    l[:, 1] = -np.inf
    mo, ml = oracle.merge_partials(o, l)
    assert np.all(mo[1] == 0) and ml[1] == -np.inf


def test_two_partials_by_hand():
    # slice 1: logits (0, log 3) -> lse = log 4, out = (v_a + 3 v_b) / 4
    # slice 2: logit log 4 -> lse = log 4, out = v_c
    # union: weights 1, 3, 4 -> out = (v_a + 3 v_b + 4 v_c) / 8, lse = log 8
    va, vb, vc = np.array([1.0, 0.0]), np.array([0.0, 2.0]), np.array([-1.0, 1.0])
    o = np.array([(va + 3 * vb) / 4, vc])
    l = np.array([math.log(4), math.log(4)])
    mo, ml = oracle.merge_partials(o, l)
    np.testing.assert_allclose(mo, (va + 3 * vb + 4 * vc) / 8, rtol=1e-15, atol=1e-16)
    assert ml == pytest.approx(math.log(8), rel=1e-15)
