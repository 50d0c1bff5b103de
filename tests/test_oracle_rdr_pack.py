"""Pins of the oracle's Rate-Distortion Retention and page packing.

SPHERICAL KV, Technical Summary section 2.2 (and the arXiv abstract): a keep
or drop decision and a precision tier per token and head under a fixed
budget, protected states always kept at the top tier, and tier-homogeneous
pages read in one header-guided pass.  These tests hold the oracle to
(4) brute-force optimality of its greedy allocation at every breakpoint,
(5) the budget, protection and tier-homogeneity invariants, plus the page
layout written out field by field."""
import itertools
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_ada_b200 import workloads as wl

TB = {0: 512, 1: 196, 2: 180, 3: 0}
LEVEL = {3: 0, 2: 1, 1: 2, 0: 3}         # tier code -> number of upgrade steps


def alloc(w, budget=None, quota=None, protect="w"):
    return oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility,
                           w.protect if protect == "w" else protect, w.mode,
                           w.budget if budget is None else budget,
                           w.quota if quota is None else quota)


def r2_of(K):
    return np.array([[[oracle.norm2(K[b, h, t].numpy().view(np.uint16)) * 2.0 ** -48
                       for t in range(K.shape[2])] for h in range(K.shape[1])]
                     for b in range(K.shape[0])])


@pytest.mark.parametrize("seed", range(6))
def test_greedy_is_optimal_at_every_breakpoint(seed):
    n = 5 if seed % 2 else 6
    w = wl.custom(seed, 1, 1, 1, 1, [n], wl.MODE_BUDGET, budget=[0],
                  k_scale=1.0)
    # vary key scales and utilities so that slopes spread out
    r = np.random.default_rng(seed)
    w.K = (w.K.to(torch.float32) * torch.tensor(
        r.uniform(0.2, 3.0, (1, 1, n, 1)), dtype=torch.float32)).to(torch.float16)
    w.utility = torch.tensor(r.uniform(0.01, 1.0, (1, 1, n)), dtype=torch.float32)
    c = oracle.distortion()
    wr2 = w.utility.numpy()[0, 0].astype(np.float64) * r2_of(w.K)[0, 0]
    best = {}
    for assign in itertools.product(range(4), repeat=n):
        cost = sum(TB[a] for a in assign)
        dist = sum(wr2[t] * c[a] for t, a in enumerate(assign))
        best[cost] = min(best.get(cost, math.inf), dist)
    costs = sorted(best)
    # prefix minimum: min distortion at cost <= x
    pm = {}
    run = math.inf
    for x in costs:
        run = min(run, best[x])
        pm[x] = run

    def min_at_most(x):
        ok = [cc for cc in costs if cc <= x]
        return pm[ok[-1]]

    nbreak = 0
    prev_level = None
    for budget in range(0, 512 * n + 8, 4):
        tier = alloc(w, budget=[budget])[0, 0, :n]
        used = sum(TB[int(t)] for t in tier)
        assert used <= budget
        lvl = np.array([LEVEL[int(t)] for t in tier])
        if prev_level is not None:
            assert np.all(lvl >= prev_level), "a larger budget lowered a tier"
        prev_level = lvl
        if used == budget:
            nbreak += 1
            dist = sum(wr2[t] * c[int(a)] for t, a in enumerate(tier))
            assert dist == pytest.approx(min_at_most(budget), rel=1e-12, abs=1e-300)
    assert nbreak >= 3 * n


def full_pools(w):
    """free lists able to hold every token in any one tier"""
    n = sum(w.Hkv * (-(-int(T) // w.P)) for T in w.seq_lens)
    w.pool_slots = [n, n, n]
    w.free_lists = [np.arange(n, dtype=np.uint32) for _ in range(3)]
    return w


def test_budget_respected_and_protection_kept():
    w = full_pools(wl.custom(11, 2, 2, 1, 16, [300, 257], wl.MODE_BUDGET, protect_sink=5,
                             protect_recent=20, zipf_alpha=1.1))
    dense = 300 * 2 * 512
    reserve = 2 * 15 * (512 + 196 + 180)
    for frac in [0.0, 0.05, 0.12, 0.2, 0.3, 0.4, 0.6, 0.9, 1.0, 1.3]:
        budget = [int(frac * dense)] * 2
        tier, rc = oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility,
                                   w.protect, w.mode, budget, w.quota, check=False)
        prot = w.protect.numpy()
        nprot = [int(prot[b, :, :w.seq_lens[b]].sum()) for b in range(2)]
        need = [nprot[b] * 512 + reserve for b in range(2)]
        if any(budget[b] < need[b] for b in range(2)):
            assert rc == oracle.ERR_BUDGET
            continue
        assert rc == oracle.OK
        assert np.all(tier[prot == 1] == 0)
        packed = oracle.pack(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.V, tier,
                             w.free_lists, w.pool_slots)
        ids = packed["page_ids"]
        ip = packed["page_indptr"]
        for b in range(2):
            units = range(b * 2, b * 2 + 2)
            pages = ids[ip[units[0]]:ip[units[-1] + 1]]
            payload = sum(w.P * TB[int(p >> 30)] for p in pages)
            assert payload <= budget[b]
        # above dense + reserve everything is T0
        if frac >= 1.3:
            for b in range(2):
                assert np.all(tier[b, :, :w.seq_lens[b]] == 0)


def test_budget_mode_prefers_high_utility_and_large_keys():
    w = wl.custom(12, 1, 1, 1, 16, [400], wl.MODE_BUDGET, zipf_alpha=1.1)
    tier = alloc(w, budget=[400 * 200])
    u = w.utility.numpy()[0, 0]
    r2 = r2_of(w.K)[0, 0]
    lvl = np.array([LEVEL[int(t)] for t in tier[0, 0]])
    wgt = u * r2
    order = np.argsort(-wgt)
    # levels are non-increasing in u * r^2 (up to equal weights)
    assert np.all(np.diff(lvl[order]) <= 0)
    assert len(set(lvl.tolist())) >= 2


def test_quota_mode_counts_and_ranking():
    lens = [100, 64, 7]
    quota = [[10, 50, 25], [0, 0, 64], [3, 3, 3]]
    w = wl.custom(13, 3, 2, 1, 16, lens, wl.MODE_QUOTA, quota=quota)
    tier = alloc(w)
    u = w.utility.numpy()
    for b in range(3):
        T = lens[b]
        for h in range(2):
            t = tier[b, h, :T]
            q0, q1, q2 = quota[b]
            n0 = min(q0, T)
            n1 = min(q1, T - n0)
            n2 = min(q2, T - n0 - n1)
            assert (t == 0).sum() == n0 and (t == 1).sum() == n1 and (t == 2).sum() == n2
            assert (t == 3).sum() == T - n0 - n1 - n2
            # ranked by utility, highest first
            lv = np.array([LEVEL[int(x)] for x in t])
            order = np.lexsort((np.arange(T), -u[b, h, :T]))
            assert np.all(np.diff(lv[order]) <= 0)
            assert np.all(tier[b, h, T:] == 3)


def test_quota_without_utility_uses_position_order():
    w = wl.custom(14, 1, 1, 1, 16, [20], wl.MODE_QUOTA, quota=[[2, 3, 4]], utility=False)
    tier = alloc(w)[0, 0]
    assert list(tier[:9]) == [0, 0, 1, 1, 1, 2, 2, 2, 2]
    assert np.all(tier[9:] == 3)


# ------------------------------------------------------------- packing ----

def read_header(page):
    return dict(count=int(page[0]) | int(page[1]) << 8, tier=int(page[2]), magic=int(page[3]),
                seq=int.from_bytes(bytes(page[4:8]), "little"),
                head=int.from_bytes(bytes(page[8:12]), "little"),
                tier_page=int.from_bytes(bytes(page[12:16]), "little"))


def v_frag_index(r, dd, elem):
    """Documented V fragment position of element (row r, dim dd)."""
    k, tr = divmod(r, 8)
    t4, lo = divmod(tr, 2)
    mt, rem = divmod(dd, 16)
    hi, g = divmod(rem, 8)
    L = 4 * g + t4
    e = 2 * hi + lo
    if elem == 1:
        return k * 1024 + 512 * (mt // 4) + 16 * L + 4 * (mt % 4) + e
    return k * 2048 + 512 * (mt // 2) + 16 * L + 8 * (mt % 2) + 2 * e


def read_row(page, tier, P, r):
    """Decode row r of a page back into (K or codes, V) per the documented layout."""
    if tier == 0:
        K = np.zeros(128, np.uint16)
        V = np.zeros(128, np.uint16)
        for dd in range(128):
            c, e = divmod(dd, 8)
            pos = c ^ (4 * (r & 1))
            o = 16 + r * 256 + pos * 16 + e * 2
            K[dd] = int(page[o]) | int(page[o + 1]) << 8
            o = 16 + 256 * P + v_frag_index(r, dd, 2)
            V[dd] = int(page[o]) | int(page[o + 1]) << 8
        return dict(K=K, V=V)
    cb = 64 if tier == 1 else 48
    rs = 16
    cs = rs + 2 * P
    ss = cs + cb * P
    vs = ss + 2 * P
    rt = int(page[rs + 2 * r]) | int(page[rs + 2 * r + 1]) << 8
    sc = int(page[ss + 2 * r]) | int(page[ss + 2 * r + 1]) << 8
    row = page[cs + cb * r: cs + cb * (r + 1)]
    th = np.zeros(64, np.int64)
    rho = np.zeros(64, np.int64)
    for p in range(64):
        g = (p // 4) % 4
        j = 4 * (p // 16) + p % 4
        if tier == 1:
            byte = int(row[16 * g + j])
            th[p], rho[p] = byte >> 2, byte & 3
        else:
            th[p] = (int(row[8 * g + j // 2]) >> (4 * (j % 2))) & 15
            rho[p] = (int(row[32 + 4 * g + j // 4]) >> (2 * (j % 4))) & 3
    v8 = np.array([np.int8(np.uint8(page[vs + v_frag_index(r, dd, 1)])) for dd in range(128)])
    return dict(rt=rt, scale=sc, theta=th, rho=rho, v8=v8)


@pytest.mark.parametrize("P,scatter", [(16, True), (32, False)])
def test_pack_layout_reads_back_to_the_primitives(P, scatter):
    lens = [45, 70]
    w = wl.custom(21, 2, 2, 2, P, lens, wl.MODE_QUOTA,
                  quota=[[7, 20, 11], [16, 33, 17]], scatter=scatter)
    tier = alloc(w)
    pk = oracle.pack(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.V, tier,
                     w.free_lists, w.pool_slots)
    ids, ip, row_of, pools = pk["page_ids"], pk["page_indptr"], pk["row_of"], pk["pools"]
    taken = [0, 0, 0]
    seen = 0
    for b in range(2):
        for h in range(2):
            u = b * 2 + h
            plist = ids[ip[u]:ip[u + 1]]
            tiers = [int(p >> 30) for p in plist]
            assert tiers == sorted(tiers)            # T0 pages, then T1, then T2
            for i, pid in enumerate(plist):
                tr, slot = int(pid >> 30), int(pid & ((1 << 30) - 1))
                assert slot == w.free_lists[tr][taken[tr]]   # canonical free-list order
                taken[tr] += 1
                stride = oracle.page_stride(tr, P)
                page = pools[tr][slot * stride: slot * stride + oracle.page_payload(tr, P)]
                hd = read_header(page)
                assert hd["tier"] == tr and hd["magic"] == 0x5A
                assert hd["seq"] == b and hd["head"] == h
                assert 1 <= hd["count"] <= P
                # rows beyond count are all zero: check their r~ / K bytes
                for r in range(hd["count"], P):
                    rr = read_row(page, tr, P, r)
                    if tr == 0:
                        assert not rr["K"].any() and not rr["V"].any()
                    else:
                        assert rr["rt"] == 0 and not rr["theta"].any() and not rr["v8"].any()
                seen += hd["count"]
            # every resident token is in exactly the row row_of says
            for t in range(lens[b]):
                tr = int(tier[b, h, t])
                if tr == 3:
                    assert row_of[b, h, t] == -1
                    continue
                pi, r = divmod(int(row_of[b, h, t]), P)
                pid = plist[pi]
                assert int(pid >> 30) == tr
                slot = int(pid & ((1 << 30) - 1))
                stride = oracle.page_stride(tr, P)
                page = pools[tr][slot * stride: slot * stride + oracle.page_payload(tr, P)]
                rr = read_row(page, tr, P, r)
                k = w.K[b, h, t].numpy().view(np.uint16)
                v = w.V[b, h, t].numpy().view(np.uint16)
                if tr == 0:
                    assert np.array_equal(rr["K"], k) and np.array_equal(rr["V"], v)
                    continue
                bits = 6 if tr == 1 else 4
                R2 = oracle.norm2(k)
                assert rr["rt"] == oracle.rtilde(k)
                for p in range(64):
                    assert rr["theta"][p] == oracle.angle_code(int(k[2 * p]), int(k[2 * p + 1]), bits)
                    assert rr["rho"][p] == oracle.rho_code(int(k[2 * p]), int(k[2 * p + 1]), R2, 128)
                v8, sc = oracle.vquant(v)
                assert rr["scale"] == sc and np.array_equal(rr["v8"], v8)
            # within a tier, rows follow ascending position
            for tr in range(3):
                pos = [t for t in range(lens[b]) if tier[b, h, t] == tr]
                rows = [int(row_of[b, h, t]) for t in pos]
                assert rows == sorted(rows)
    assert seen == int((tier != 3).sum())


def test_v_fragment_positions_are_a_bijection():
    for elem, block in ((1, 1024), (2, 2048)):
        pos = sorted(v_frag_index(r, dd, elem) for r in range(8) for dd in range(128))
        assert pos == list(range(0, block, elem))


def test_pack_reports_short_pool():
    w = wl.custom(22, 1, 1, 1, 16, [64], wl.MODE_QUOTA, quota=[[0, 64, 0]])
    tier = alloc(w)
    free = [w.free_lists[0], w.free_lists[1][:3], w.free_lists[2]]
    res = oracle.pack(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.V, tier, free,
                      w.pool_slots, check=False)
    assert res["status"] == oracle.ERR_POOL


def test_page_sizes():
    assert oracle.page_payload(0, 64) == 16 + 64 * 512
    assert oracle.page_payload(1, 64) == 16 + 64 * 196
    assert oracle.page_payload(2, 16) == 16 + 16 * 180
    for t in range(3):
        for P in (16, 32, 64):
            s = oracle.page_stride(t, P)
            assert s % 128 == 0 and 0 <= s - oracle.page_payload(t, P) < 128
