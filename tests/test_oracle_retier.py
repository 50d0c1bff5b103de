"""Pins of the oracle's re-tiering (oracle.retier): rows leaving the
protected recent window (T0, their exact fp16 keys still in the store) are
re-decided under the sequence's budget while every other resident token
keeps its tier (SPHERICAL KV, Technical Summary 2.2: keep/drop and tier per
token and head under a fixed budget; 2.3: the retention filter between the
codes and the store).

What fixes it independently of its own code: with nothing demoted it is the
identity; with every token demoted from an all-T0 store it is the budget
allocation itself (orc_allocate without protection); on tiny cases the
demoted tokens' assignment is optimal over all 4^n assignments at every
breakpoint of the budget left to them; kept tokens never change; the
budget holds; an over-budget store is reported."""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_ada_b200 import workloads as wl

TB = {0: 512, 1: 196, 2: 180, 3: 0}


def r2_of(K):
    return np.array([[[oracle.norm2(K[b, h, t].numpy().view(np.uint16)) * 2.0 ** -48
                       for t in range(K.shape[2])] for h in range(K.shape[1])]
                     for b in range(K.shape[0])])


def reserve(w):
    return w.Hkv * (w.P - 1) * (512 + 196 + 180)


def store_of(w, budget):
    return oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility,
                           w.protect, w.mode, budget, w.quota)


def test_nothing_demoted_is_the_identity():
    w = wl.custom(21, 2, 2, 1, 16, [300, 180], wl.MODE_BUDGET, protect_sink=4,
                  protect_recent=40, zipf_alpha=1.1)
    budget = [int(0.35 * 300 * 2 * 512)] * 2
    tier = store_of(w, budget)
    out = oracle.retier(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, tier,
                        np.zeros_like(tier), budget)
    assert np.array_equal(out, tier)


@pytest.mark.parametrize("frac", [0.05, 0.15, 0.3, 0.5, 0.9])
def test_demoting_an_all_t0_store_is_the_budget_allocation(frac):
    """An all-T0 store (every token protected) with every token demoted: no
    token is kept, so the walk is the allocation's over all tokens."""
    w = wl.custom(22, 2, 2, 1, 16, [260, 150], wl.MODE_BUDGET, zipf_alpha=1.2)
    budget = [int(frac * 260 * 2 * 512)] * 2
    all_t0 = np.zeros((w.B, w.Hkv, w.Tmax), np.uint8)
    for b in range(w.B):
        all_t0[b, :, w.seq_lens[b]:] = 3
    demote = (all_t0 == 0).astype(np.uint8)
    out, rc = oracle.retier(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, all_t0,
                            demote, budget, check=False)
    ref, rc_ref = oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility,
                                  None, w.mode, budget, w.quota, check=False)
    assert rc == rc_ref
    if rc == oracle.OK:   # (below the reserve both report the budget)
        assert np.array_equal(out, ref)


@pytest.mark.parametrize("seed", range(4))
def test_demoted_assignment_is_optimal_at_every_breakpoint(seed):
    """P = 1 (no reserve), three kept tokens of fixed tiers and n demoted
    T0 tokens: at every budget where the walk uses exactly the bytes left
    after the kept tokens, the demoted tokens' distortion sum u r^2 c(tier)
    is the minimum over all 4^n assignments of that cost or less."""
    n = 5 if seed % 2 else 4
    m = n + 3
    w = wl.custom(30 + seed, 1, 1, 1, 1, [m], wl.MODE_BUDGET, budget=[0])
    r = np.random.default_rng(seed)
    w.K = (w.K.to(torch.float32) * torch.tensor(
        r.uniform(0.2, 3.0, (1, 1, m, 1)), dtype=torch.float32)).to(torch.float16)
    w.utility = torch.tensor(r.uniform(0.01, 1.0, (1, 1, m)), dtype=torch.float32)
    tier_in = np.zeros((1, 1, m), np.uint8)
    tier_in[0, 0, n:] = [1, 2, 3]                 # kept: T1, T2, dropped
    demote = np.zeros_like(tier_in)
    demote[0, 0, :n] = 1
    kept = 196 + 180
    c = oracle.distortion()
    wr2 = w.utility.numpy()[0, 0].astype(np.float64) * r2_of(w.K)[0, 0]
    best = {}
    for assign in itertools.product(range(4), repeat=n):
        cost = sum(TB[a] for a in assign)
        dist = sum(wr2[t] * c[a] for t, a in enumerate(assign))
        best[cost] = min(best.get(cost, math.inf), dist)
    costs = sorted(best)
    nbreak = 0
    for left in range(0, 512 * n + 8, 4):
        out = oracle.retier(1, 1, m, w.d, 1, w.seq_lens, w.K, w.utility, tier_in, demote,
                            [kept + left])
        assert np.array_equal(out[0, 0, n:], tier_in[0, 0, n:]), "a kept token changed"
        used = sum(TB[int(t)] for t in out[0, 0, :n])
        assert used <= left
        if used == left:
            nbreak += 1
            dist = sum(wr2[t] * c[int(a)] for t, a in enumerate(out[0, 0, :n]))
            assert dist == pytest.approx(min(best[x] for x in costs if x <= left), rel=1e-12,
                                         abs=1e-300)
    assert nbreak >= 3 * n


@pytest.mark.parametrize("P", [16, 64])
def test_reserve_comes_off_the_budget_before_the_walk(P):
    """P > 1: the walk gets budget - kept bytes - Hkv (P - 1)(512 + 196 + 180).
    With the budget raised by exactly that reserve, the demoted tokens get
    the P = 1 assignment (no reserve) at every budget of a sweep; a budget
    one byte below the kept bytes plus the reserve is reported, with the
    demoted rows dropped and the kept rows unchanged."""
    n, m = 4, 7
    w = wl.custom(40 + P, 1, 1, 1, 1, [m], wl.MODE_BUDGET, budget=[0])
    r = np.random.default_rng(P)
    w.utility = torch.tensor(r.uniform(0.01, 1.0, (1, 1, m)), dtype=torch.float32)
    tier_in = np.zeros((1, 1, m), np.uint8)
    tier_in[0, 0, n:] = [1, 2, 3]
    demote = np.zeros_like(tier_in)
    demote[0, 0, :n] = 1
    reserve = (P - 1) * (512 + 196 + 180)
    kept = 196 + 180
    for left in range(0, 512 * n + 8, 20):
        ref = oracle.retier(1, 1, m, w.d, 1, w.seq_lens, w.K, w.utility, tier_in, demote,
                            [kept + left])
        got = oracle.retier(1, 1, m, w.d, P, w.seq_lens, w.K, w.utility, tier_in, demote,
                            [kept + left + reserve])
        assert np.array_equal(got, ref), left
    # below the reserve: reported, demoted rows dropped, kept rows unchanged
    out, rc = oracle.retier(1, 1, m, w.d, P, w.seq_lens, w.K, w.utility, tier_in, demote,
                            [kept + reserve - 1], check=False)
    assert rc == oracle.ERR_BUDGET
    assert np.all(out[0, 0, :n] == 3) and np.array_equal(out[0, 0, n:], tier_in[0, 0, n:])


def window_store(seed, T, A, recent, frac, B=2, Hkv=2):
    """A store allocated over the first T - A tokens (recent window of
    `recent` tokens protected, budget frac of dense at T - A) to which A
    tokens were then appended as T0: tiers for T tokens and the budget at
    T (frac of dense at T), which the appended bytes exceed."""
    w = wl.custom(seed, B, Hkv, 1, 16, [T] * B, wl.MODE_BUDGET, zipf_alpha=1.1)
    t0 = T - A
    budget = [int(frac * t0 * Hkv * 512)] * B
    prot = torch.zeros((B, Hkv, T), dtype=torch.uint8)
    prot[:, :, t0 - recent:t0] = 1
    tier = oracle.allocate(B, Hkv, T, w.d, w.P, [t0] * B, w.K, w.utility, prot, w.mode,
                           budget, w.quota)
    tier[:, :, t0:] = 0                      # the appended tokens
    return w, [int(frac * T * Hkv * 512)] * B, tier


def test_window_roll_keeps_the_rest_and_holds_the_budget():
    """After A appended T0 tokens the store is over budget; the oldest A
    rows of the recent window leave it: only those change (to T0, T1, T2 or
    dropped), and the resident bytes are back within the budget less the
    reserve."""
    T, A, recent = 400, 32, 64
    w, budget, tier = window_store(23, T, A, recent, 0.3)
    demote = np.zeros_like(tier)
    demote[:, :, T - A - recent:T - recent] = 1
    assert np.all(tier[demote == 1] == 0)
    for b in range(w.B):
        assert sum(TB[int(t)] for t in tier[b].ravel()) > budget[b] - reserve(w)
    out = oracle.retier(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, tier, demote,
                        budget)
    assert np.array_equal(out[demote == 0], tier[demote == 0])
    for b in range(w.B):
        used = sum(TB[int(t)] for t in out[b].ravel())
        assert used <= budget[b] - reserve(w)
    # at 30% of dense the demoted rows become codes or are dropped
    d = out[demote == 1]
    assert np.any(d == 3) and np.any((d == 1) | (d == 2))


def test_over_budget_store_is_reported_and_demoted_rows_dropped():
    T = 200
    w, budget, tier = window_store(24, T, 0, 40, 0.5, B=1)
    demote = np.zeros_like(tier)
    demote[:, :, T - 40:T - 20] = 1
    kept = sum(TB[int(t)] for t in tier[demote == 0].ravel())
    small = [kept + reserve(w) - 1]
    out, rc = oracle.retier(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, tier,
                            demote, small, check=False)
    assert rc == oracle.ERR_BUDGET
    assert np.all(out[demote == 1] == 3)
    assert np.array_equal(out[demote == 0], tier[demote == 0])
    out, rc = oracle.retier(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, tier,
                            demote, [kept + reserve(w)], check=False)
    assert rc == oracle.OK and np.all(out[demote == 1] == 3)   # nothing left to spend


def test_demoting_a_row_that_is_not_t0_is_an_error():
    w = wl.custom(25, 1, 1, 1, 16, [100], wl.MODE_BUDGET, zipf_alpha=1.1)
    budget = [int(0.3 * 100 * 512)]
    tier = store_of(w, budget)
    t = int(np.nonzero(tier[0, 0] != 0)[0][0])
    demote = np.zeros_like(tier)
    demote[0, 0, t] = 1
    _, rc = oracle.retier(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, tier,
                          demote, budget, check=False)
    assert rc == oracle.ERR_ARG
