"""skv_append (decode-time ingest of the newest token as T0) against the
oracle: after n appends the store must be what the oracle's pack gives for
the initial tiers with the appended positions set to T0 -- tiers, row map
and page table bit for bit, every page's bytes equal page by page in list
order (slots are chosen differently: the oracle takes them in (seq, head,
page) order, the append in step order) -- and the decode must match the
oracle's attention over that store."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_ada_b200 import skv
from long_context_decode_ada_b200 import workloads as wl
from _gpu import assert_close

pytestmark = pytest.mark.gpu


def tier_indptr_of(ids: np.ndarray, indptr: np.ndarray) -> np.ndarray:
    U = len(indptr) - 1
    out = np.zeros(3 * U + 1, np.int32)
    for u in range(U):
        tr = ids[indptr[u]:indptr[u + 1]] >> 30
        for t in range(3):
            out[3 * u + t] = indptr[u] + int((tr < t).sum())
    out[3 * U] = indptr[U]
    return out


def page_bytes(ids, indptr, pools, P):
    """Per unit, the payload bytes of its pages in list order."""
    res = []
    for u in range(len(indptr) - 1):
        pages = []
        for g in range(int(indptr[u]), int(indptr[u + 1])):
            pid = int(ids[g])
            t, slot = pid >> 30, pid & ((1 << 30) - 1)
            st, pay = oracle.page_stride(t, P), oracle.page_payload(t, P)
            pages.append((t, pools[t][slot * st: slot * st + pay].tobytes()))
        res.append(pages)
    return res


def append_case(w_full, n_steps, extra_t0_pages):
    """Store of w_full with every sequence n_steps tokens short, then n_steps
    appends on the GPU; returns (cache, expected dict, final tiers)."""
    B, Hkv, P = w_full.B, w_full.Hkv, w_full.P
    seq0 = (w_full.seq_lens - n_steps).astype(np.int32)
    slots = list(w_full.pool_slots)
    slots[0] += extra_t0_pages
    free = [np.arange(s, dtype=np.uint32) for s in slots]
    w0 = dataclasses.replace(w_full, seq_lens=seq0, pool_slots=slots, free_lists=free)
    ctx = skv.Context(P)
    dev = skv.workload_to_device(w0)
    cache = skv.build_cache(ctx, w0, dev)
    cache.check()
    seq = dev["seq_lens"].clone()
    for step in range(n_steps):
        pos = [int(seq0[b]) + step for b in range(B)]
        K_new = torch.stack([dev["K"][b, :, pos[b]] for b in range(B)]).contiguous()
        V_new = torch.stack([dev["V"][b, :, pos[b]] for b in range(B)]).contiguous()
        cache.append(K_new, V_new, seq)
        cache.check()
    assert np.array_equal(seq.cpu().numpy(), w_full.seq_lens)
    # the oracle: the initial tiers, the appended positions as T0, a fresh pack
    tier = oracle.allocate(B, Hkv, w0.Tmax, w0.d, P, seq0, w0.K, w0.utility, w0.protect,
                           w0.mode, w0.budget, w0.quota)
    for b in range(B):
        tier[b, :, int(seq0[b]):int(w_full.seq_lens[b])] = 0
    ref = oracle.pack(B, Hkv, w0.Tmax, w0.d, P, w_full.seq_lens, w0.K, w0.V, tier, free, slots)
    return ctx, dev, cache, ref, tier


def check_against_oracle(w_full, cache, dev, ref, tier):
    P = w_full.P
    assert np.array_equal(cache.tier.cpu().numpy(), tier), "tiers"
    assert np.array_equal(cache.row_of.cpu().numpy(), ref["row_of"]), "row map"
    ip = cache.page_indptr.cpu().numpy()
    assert np.array_equal(ip, ref["page_indptr"]), "page_indptr"
    ids = cache.page_ids[: ip[-1]].cpu().numpy().view(np.uint32)
    ref_ids = np.asarray(ref["page_ids"], np.uint32)
    assert np.array_equal(cache.page_tier_indptr.cpu().numpy(), tier_indptr_of(ref_ids, ip)), \
        "page_tier_indptr"
    pools = [p.cpu().numpy() for p in cache.pools]
    got = page_bytes(ids, ip, pools, P)
    exp = page_bytes(ref_ids, ip, ref["pools"], P)
    for u, (a, b) in enumerate(zip(got, exp)):
        assert len(a) == len(b), f"unit {u}: page count"
        for k, (pa, pb) in enumerate(zip(a, b)):
            assert pa[0] == pb[0], f"unit {u} page {k}: tier"
            assert pa[1] == pb[1], f"unit {u} page {k}: bytes"
    out, lse = cache.decode(dev["q"], dev["q_dtype"], w_full.Hq)
    cache.check()
    ro, rl = oracle.decode(w_full.B, w_full.Hq, w_full.Hkv, w_full.Tmax, w_full.d,
                           w_full.seq_lens, w_full.K, w_full.V, tier, w_full.q, w_full.q_dtype)
    assert_close(out.cpu().numpy(), ro, "out after appends")
    assert_close(lse.cpu().numpy(), rl, "lse after appends")


def test_append_budget_mode_crosses_pages():
    # P = 16: 37 appends fill the partial last T0 page and open new ones
    lens = [300, 150]
    w = wl.custom(81, 2, 2, 4, 16, lens, wl.MODE_BUDGET, protect_sink=16, protect_recent=24,
                  zipf_alpha=1.1, budget=[int(0.35 * T * 2 * 512) for T in lens])
    ctx, dev, cache, ref, tier = append_case(w, 37, extra_t0_pages=16)
    check_against_oracle(w, cache, dev, ref, tier)


def test_append_first_t0_page_of_a_unit():
    # no T0 tokens at first (quota 0, nothing protected): the first append
    # opens each unit's T0 segment in front of its T1/T2 pages
    lens = [120, 97, 64]
    w = wl.custom(82, 3, 2, 2, 32, lens, wl.MODE_QUOTA,
                  quota=[[0, T // 3, T // 4] for T in lens], q_dtype="fp16")
    ctx, dev, cache, ref, tier = append_case(w, 40, extra_t0_pages=16)
    check_against_oracle(w, cache, dev, ref, tier)


def test_append_refuses_a_full_sequence():
    lens = [40]
    w = wl.custom(83, 1, 2, 4, 16, lens, wl.MODE_QUOTA, quota=[[8, 16, 8]])
    ctx = skv.Context(16)
    dev = skv.workload_to_device(w)
    cache = skv.build_cache(ctx, w, dev)
    cache.check()
    before = (cache.page_indptr.clone(), cache.page_ids.clone(), cache.tier.clone())
    seq = dev["seq_lens"].clone()   # == Tmax: no room for another token
    K_new = dev["K"][:, :, 0].contiguous()
    cache.append(K_new, K_new, seq)
    with pytest.raises(skv.SkvError):
        cache.check()
    cache.err.zero_()
    assert torch.equal(cache.page_indptr, before[0])
    assert torch.equal(cache.page_ids, before[1])
    assert torch.equal(cache.tier, before[2])
    assert int(seq[0]) == 40
