"""Helpers for the GPU parity tests: run a workload through libskv and through
the oracle, and compare.  Bit-exact for tiers, page tables, row maps and page
bytes; attention outputs within |gpu - ref| <= 1e-3 + 2e-3 |ref|."""
import numpy as np
import torch

import oracle
from long_context_decode_ada_b200 import skv

ATOL = 1e-3
RTOL = 2e-3


def run_gpu(w, num_splits=0, ctx=None, decode=True):
    ctx = ctx or skv.Context(w.P)
    dev = skv.workload_to_device(w)
    cache = skv.build_cache(ctx, w, dev)
    cache.check()
    res = dict(ctx=ctx, cache=cache, dev=dev)
    if decode:
        out, lse = cache.decode(dev["q"], dev["q_dtype"], w.Hq, num_splits=num_splits)
        cache.check()
        res.update(out=out.cpu().numpy(), lse=lse.cpu().numpy())
    return res


def tier_indptr_of(indptr, ids):
    """CSR offsets per (unit, tier) segment 3u + t of a page table whose
    units list their T0 pages, then T1, then T2 (checked here)."""
    U = len(indptr) - 1
    out = np.zeros(3 * U + 1, np.int32)
    for u in range(U):
        a, b = int(indptr[u]), int(indptr[u + 1])
        tiers = np.asarray(ids[a:b], np.uint32) >> 30
        assert np.all(np.diff(tiers.astype(np.int64)) >= 0), "unit pages not ordered by tier"
        for t in range(3):
            out[3 * u + t] = a + int((tiers < t).sum())
    out[3 * U] = int(indptr[-1])
    return out


def compare_store(w, g, ref):
    """Tiers, row map, page table and every used page's payload bytes."""
    cache = g["cache"]
    tier = cache.tier.cpu().numpy()
    assert np.array_equal(tier, ref["tier"]), "tier mismatch"
    row_of = cache.row_of.cpu().numpy()
    assert np.array_equal(row_of, ref["row_of"]), "row_of mismatch"
    ip = cache.page_indptr.cpu().numpy()
    assert np.array_equal(ip, ref["page_indptr"]), "page_indptr mismatch"
    n = int(ip[-1])
    ids = cache.page_ids[:n].cpu().numpy().view(np.uint32)
    assert np.array_equal(ids, ref["page_ids"][:n]), "page_ids mismatch"
    tip = cache.page_tier_indptr.cpu().numpy()
    assert np.array_equal(tip, tier_indptr_of(ref["page_indptr"], ref["page_ids"])), \
        "page_tier_indptr mismatch"
    pools_gpu = [p.cpu().numpy() for p in cache.pools]
    bad = 0
    for pid in ids:
        t, slot = int(pid) >> 30, int(pid) & ((1 << 30) - 1)
        st = oracle.page_stride(t, w.P)
        pay = oracle.page_payload(t, w.P)
        a = pools_gpu[t][slot * st: slot * st + pay]
        b = ref["pools"][t][slot * st: slot * st + pay]
        if not np.array_equal(a, b):
            bad += 1
            if bad == 1:
                diff = np.nonzero(a != b)[0]
                first = diff[:8]
                msg = f"page {pid:#x} (tier {t}) differs at {len(diff)} bytes, first {first}: " \
                      f"gpu {a[first]} ref {b[first]}"
    assert bad == 0, msg
    return n


def assert_close(got, ref, what):
    ref = np.asarray(ref, np.float64)
    got = np.asarray(got, np.float64)
    fin = np.isfinite(ref)
    assert np.array_equal(np.isfinite(got), fin), f"{what}: finiteness differs"
    assert np.array_equal(got[~fin], ref[~fin]), f"{what}: infinities differ"
    err = np.abs(got[fin] - ref[fin])
    lim = ATOL + RTOL * np.abs(ref[fin])
    worst = np.argmax(err - lim) if err.size else 0
    assert np.all(err <= lim), (f"{what}: {int((err > lim).sum())} elements out of tolerance; "
                                f"worst err {err.flat[worst]:.3g} at ref {ref[fin].flat[worst]:.4g}")


def upload_oracle_store(ctx, w, ref):
    """A PagedCache whose pools and page table are the oracle's bytes."""
    cache = skv.PagedCache(ctx, w.B, w.Hkv, w.Tmax, w.pool_slots)
    for t in range(3):
        src = torch.from_numpy(ref["pools"][t])
        cache.pools[t][: src.numel()].copy_(src.to(cache.device))
    cache.page_indptr.copy_(torch.from_numpy(ref["page_indptr"]).to(cache.device))
    cache.page_tier_indptr.copy_(torch.from_numpy(
        tier_indptr_of(ref["page_indptr"], ref["page_ids"])).to(cache.device))
    n = int(ref["page_indptr"][-1])
    if n:
        cache.page_ids[:n].copy_(torch.from_numpy(ref["page_ids"][:n].view(np.int32)).to(
            cache.device))
    return cache
