"""skv_retier (re-tiering of the rows that leave the protected recent window,
on the store itself) against the oracle, after a cycle of appends: the
expected store is the oracle's re-tiering of the tiers (oracle.retier) and a
fresh pack of them (oracle.pack) -- tiers, row map and page table bit for
bit, every page's bytes equal page by page in list order -- and the decode
must match the oracle's attention over that store.  SPHERICAL KV technical
summary 2.2 (Rate-Distortion Retention) and 2.3 (System Integration).

The update is in place: pages wholly before the first changed row of their
(unit, tier) segment keep their slots, the others take fresh slots from the
free lists, and the old pages that are no longer referenced are listed."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_ada_b200 import skv
from long_context_decode_ada_b200 import workloads as wl
from _gpu import assert_close
from test_gpu_append import page_bytes, tier_indptr_of

pytestmark = pytest.mark.gpu


class Window:
    """A store of the first T - A tokens of every sequence (a sink and a
    recent window of `recent` tokens protected, budget frac of dense at
    T - A); append() makes the next tokens resident on the GPU as T0."""

    def __init__(self, seed, B, Hkv, P, T, A, recent, frac, sink=4, scatter=True):
        w = wl.custom(seed, B, Hkv, 4, P, [T] * B, wl.MODE_BUDGET, zipf_alpha=1.1)
        t0 = T - A
        prot = torch.zeros((B, Hkv, T), dtype=torch.uint8)
        prot[:, :, :sink] = 1
        prot[:, :, t0 - recent:t0] = 1
        slots = [B * Hkv * (T // P + 4)] * 3
        rng = np.random.default_rng(seed)
        free = [(rng.permutation(s) if scatter else np.arange(s)).astype(np.uint32)
                for s in slots]
        self.frac, self.recent = frac, recent
        self.w = dataclasses.replace(
            w, seq_lens=np.full(B, t0, np.int32), protect=prot,
            budget=np.full(B, int(frac * t0 * Hkv * 512), np.int64), pool_slots=slots,
            free_lists=free)
        self.ctx = skv.Context(P)
        self.dev = skv.workload_to_device(self.w)
        self.cache = skv.build_cache(self.ctx, self.w, self.dev)
        self.cache.check()
        self.seq = self.dev["seq_lens"].clone()
        self.T = t0
        self.tier = oracle.allocate(B, Hkv, T, w.d, P, self.w.seq_lens, w.K, w.utility, prot,
                                    w.mode, self.w.budget, w.quota)

    def append(self, n):
        w, dev = self.w, self.dev
        for _ in range(n):
            K_new = dev["K"][:, :, self.T].contiguous()
            V_new = dev["V"][:, :, self.T].contiguous()
            self.cache.append(K_new, V_new, self.seq)
            self.cache.check()
            self.tier[:, :, self.T] = 0
            self.T += 1
        assert np.all(self.seq.cpu().numpy() == self.T)
        assert np.array_equal(self.cache.tier.cpu().numpy(), self.tier), "tiers after appends"

    def snapshot(self):
        c = self.cache
        ip = c.page_indptr.cpu().numpy().copy()
        return dict(ip=ip, tip=c.page_tier_indptr.cpu().numpy().copy(),
                    ids=c.page_ids[:ip[-1]].cpu().numpy().view(np.uint32).copy(),
                    cursor=c.free_cursor().cpu().numpy().copy(),
                    tier=c.tier.cpu().numpy().copy(), row_of=c.row_of.cpu().numpy().copy())

    def retier(self, lo, hi, budget_frac=None, expect_err=None):
        """Demote positions [lo, hi) of every sequence and head under the
        budget frac of dense at the current length; returns the expected
        tiers, the status of the oracle and the released ids."""
        w = self.w
        B, Hkv = w.B, w.Hkv
        demote = np.zeros((B, Hkv, w.Tmax), np.uint8)
        demote[:, :, lo:hi] = 1
        frac = self.frac if budget_frac is None else budget_frac
        budget = np.full(B, int(frac * self.T * Hkv * 512), np.int64)
        exp, rc = oracle.retier(B, Hkv, w.Tmax, w.d, w.P, np.full(B, self.T, np.int32), w.K,
                                w.utility, self.tier, demote, budget, check=False)
        released, nrel = self.cache.retier(self.dev["utility"],
                                           torch.from_numpy(demote).cuda(),
                                           torch.from_numpy(budget).cuda(), self.seq)
        if expect_err is None:
            self.cache.check()
        else:
            with pytest.raises(skv.SkvError) as ei:
                self.cache.check()
            assert ei.value.code == expect_err
        self.tier = exp
        n = int(nrel.item())
        return rc, released[:n].cpu().numpy().view(np.uint32).copy()

    def check_store(self):
        """The store against a fresh oracle pack of the current tiers, and the
        decode against the oracle's attention."""
        w, c = self.w, self.cache
        seq = np.full(w.B, self.T, np.int32)
        ref = oracle.pack(w.B, w.Hkv, w.Tmax, w.d, w.P, seq, w.K, w.V, self.tier, w.free_lists,
                          w.pool_slots)
        assert np.array_equal(c.tier.cpu().numpy(), self.tier), "tiers"
        assert np.array_equal(c.row_of.cpu().numpy(), ref["row_of"]), "row map"
        ip = c.page_indptr.cpu().numpy()
        assert np.array_equal(ip, ref["page_indptr"]), "page_indptr"
        ids = c.page_ids[:ip[-1]].cpu().numpy().view(np.uint32)
        ref_ids = np.asarray(ref["page_ids"], np.uint32)
        assert np.array_equal(c.page_tier_indptr.cpu().numpy(), tier_indptr_of(ref_ids, ip)), \
            "page_tier_indptr"
        got = page_bytes(ids, ip, [p.cpu().numpy() for p in c.pools], w.P)
        exp = page_bytes(ref_ids, ip, ref["pools"], w.P)
        for u, (a, b) in enumerate(zip(got, exp)):
            assert len(a) == len(b), f"unit {u}: page count"
            for k, (pa, pb) in enumerate(zip(a, b)):
                assert pa[0] == pb[0], f"unit {u} page {k}: tier"
                assert pa[1] == pb[1], f"unit {u} page {k}: bytes"
        out, lse = c.decode(self.dev["q"], self.dev["q_dtype"], w.Hq)
        c.check()
        ro, rl = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, seq, w.K, w.V, self.tier, w.q,
                               w.q_dtype)
        assert_close(out.cpu().numpy(), ro, "out after re-tiering")
        assert_close(lse.cpu().numpy(), rl, "lse after re-tiering")


def check_pages_in_place(before, after, released, P):
    """Every old page is either still referenced or released (never both);
    new pages come from the free lists at the cursors; in each T1 / T2
    segment that only grew at its end, every full old page kept its slot."""
    old, new, rel = set(before["ids"].tolist()), set(after["ids"].tolist()), set(released.tolist())
    assert len(rel) == len(released), "a page released twice"
    assert rel.isdisjoint(new), "a released page is still referenced"
    assert old == (old & new) | rel, "an old page neither kept nor released"
    taken = after["cursor"] - before["cursor"]
    fresh = np.array(sorted(new - old), np.uint32)
    assert np.array_equal(np.bincount(fresh >> 30, minlength=3)[:3], taken), "free slots taken"
    U = len(before["ip"]) - 1
    kept_any = 0
    for u in range(U):
        for t in (1, 2):
            a0, a1 = before["tip"][3 * u + t], before["tip"][3 * u + t + 1]
            b0 = after["tip"][3 * u + t]
            n_old_rows = int(((before["tier"].reshape(U, -1)[u]) == t).sum())
            full = n_old_rows // P
            assert full <= a1 - a0
            assert np.array_equal(after["ids"][b0:b0 + full], before["ids"][a0:a0 + full]), \
                f"unit {u} tier {t}: full pages moved"
            kept_any += full
    return kept_any


@pytest.mark.parametrize("seed,B,Hkv,P,T,A,recent,frac", [
    (41, 2, 2, 16, 600, 40, 64, 0.3),
    (42, 1, 4, 64, 2100, 70, 256, 0.25),
    (43, 3, 1, 16, 500, 33, 48, 0.9),   # a generous budget: demoted rows stay T0 too
    (48, 2, 2, 32, 900, 50, 64, 0.2),  # P = 32 and a tight budget: T2 pages, dropped rows
])
def test_retier_after_appends_matches_the_oracle(seed, B, Hkv, P, T, A, recent, frac):
    win = Window(seed, B, Hkv, P, T, A, recent, frac)
    win.append(A)
    t0 = T - A
    before = win.snapshot()
    rc, released = win.retier(t0 - recent, t0 - recent + A)
    assert rc == oracle.OK
    win.check_store()
    after = win.snapshot()
    kept = check_pages_in_place(before, after, released, P)
    assert kept > 0
    d = win.tier[:, :, t0 - recent:t0 - recent + A]
    if frac < 0.5:
        assert np.any(d == 3) and np.any((d == 1) | (d == 2)), "demoted rows coded and dropped"
    if frac <= 0.2:
        assert np.any(win.tier == 2), "the store holds T2 pages"


def test_two_window_cycles():
    """Append, re-tier, append, re-tier: the window moves twice."""
    T, A, recent = 560, 24, 64
    win = Window(44, 2, 2, 16, T, 2 * A, recent, 0.35)
    lo = T - 2 * A - recent
    for cycle in range(2):
        win.append(A)
        before = win.snapshot()
        rc, released = win.retier(lo + cycle * A, lo + (cycle + 1) * A)
        assert rc == oracle.OK
        win.check_store()
        check_pages_in_place(before, win.snapshot(), released, 16)


def test_nothing_demoted_leaves_the_store_as_it_is():
    win = Window(46, 2, 2, 16, 300, 20, 32, 0.4)
    win.append(20)
    before = win.snapshot()
    pools = [p.cpu().numpy().copy() for p in win.cache.pools]
    rc, released = win.retier(0, 0, budget_frac=1.0)
    assert rc == oracle.OK
    after = win.snapshot()
    assert len(released) == 0
    for k in ("ip", "tip", "ids", "cursor", "tier", "row_of"):
        assert np.array_equal(before[k], after[k]), k
    for a, b in zip(pools, win.cache.pools):
        assert np.array_equal(a, b.cpu().numpy())
    win.check_store()


def test_over_budget_store_is_reported_and_demoted_rows_dropped():
    """A budget below the kept tokens plus the reserve: SKV_ERR_BUDGET, the
    demoted rows are dropped (as in the oracle) and the store stays
    consistent."""
    T, A, recent = 400, 30, 64
    win = Window(47, 2, 2, 16, T, A, recent, 0.3)
    win.append(A)
    lo = T - A - recent
    rc, released = win.retier(lo, lo + A, budget_frac=0.02, expect_err=skv.SKV_ERR_BUDGET)
    assert rc == oracle.ERR_BUDGET
    assert np.all(win.tier[:, :, lo:lo + A] == 3)
    win.check_store()
