"""Outlier-aware protection (skv_config.outlier_protect) against the oracle:
the tiers are bit for bit the oracle's allocation with the caller's
protection mask joined by oracle.outlier_flags, and the decode over the
store matches the oracle's decode with those tiers."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_ada_b200 import skv
from long_context_decode_ada_b200 import workloads as wl
from _gpu import assert_close

pytestmark = pytest.mark.gpu


def with_outliers(w, head, channel, every, scale=20.0):
    """Scale one channel of one kv head on every `every`-th position, and
    size the T0 pool for every position (protected tokens come on top of a
    quota's T0 count)."""
    K = w.K.clone()
    K[:, head, ::every, channel] *= scale
    slots = list(w.pool_slots)
    slots[0] = w.B * w.Hkv * (-(-w.Tmax // w.P)) + 1
    free = list(w.free_lists)
    free[0] = np.arange(slots[0], dtype=np.uint32)
    return dataclasses.replace(w, K=K, pool_slots=slots, free_lists=free)


def check(w):
    ctx = skv.Context(w.P, outlier_protect=True)
    dev = skv.workload_to_device(w)
    cache = skv.build_cache(ctx, w, dev)
    cache.check()
    flags = oracle.outlier_flags(w.B, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K)
    prot = flags.copy()
    if w.protect is not None:
        prot |= w.protect.numpy().astype(np.uint8)
    tier = oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, prot,
                           w.mode, w.budget, w.quota)
    got = cache.tier.cpu().numpy()
    assert np.array_equal(got, tier), f"{int((got != tier).sum())} tiers differ"
    assert np.all(got[flags == 1] == 0)
    out, lse = cache.decode(dev["q"], dev["q_dtype"], w.Hq)
    cache.check()
    ro, rl = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, tier, w.q,
                           w.q_dtype)
    assert_close(out.cpu().numpy(), ro, "out")
    assert_close(lse.cpu().numpy(), rl, "lse")
    return flags


def test_outlier_protection_budget_mode():
    lens = [700, 240]
    w = wl.custom(61, 2, 2, 4, 16, lens, wl.MODE_BUDGET, protect_sink=4, protect_recent=8,
                  zipf_alpha=1.1,
                  budget=[int(0.35 * T * 2 * 512) + 2 * 15 * 888 + 12 * 2 * 512 for T in lens])
    w = with_outliers(w, head=1, channel=77, every=9)
    flags = check(w)
    assert flags.sum() > 20


def test_outlier_protection_quota_mode_g1():
    lens = [500, 33]
    w = wl.custom(62, 2, 2, 1, 32, lens, wl.MODE_QUOTA,
                  quota=[[T // 8, T // 3, T // 4] for T in lens], q_dtype="fp16")
    w = with_outliers(w, head=0, channel=3, every=5)
    flags = check(w)
    assert flags.sum() > 20


def test_without_the_option_nothing_changes():
    lens = [400]
    w = wl.custom(63, 1, 2, 4, 16, lens, wl.MODE_QUOTA, quota=[[40, 150, 100]])
    w = with_outliers(w, head=0, channel=10, every=3)
    ctx = skv.Context(w.P)
    dev = skv.workload_to_device(w)
    cache = skv.build_cache(ctx, w, dev)
    cache.check()
    tier = oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, None,
                           w.mode, w.budget, w.quota)
    assert np.array_equal(cache.tier.cpu().numpy(), tier)


def test_infeasible_protection_is_a_budget_error():
    # every key of both heads is an outlier: protecting them all needs the
    # whole dense size, above the budget; the oracle refuses the same input
    lens = [300]
    w = wl.custom(64, 1, 2, 4, 16, lens, wl.MODE_BUDGET, zipf_alpha=1.1,
                  budget=[int(0.3 * 300 * 2 * 512) + 2 * 15 * 888])
    K = w.K.clone()
    K[:, :, :, 5] = 40.0
    w = dataclasses.replace(w, K=K)
    flags = oracle.outlier_flags(w.B, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K)
    assert flags[0, :, :300].all()
    with pytest.raises(oracle.OracleError):
        oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, flags,
                        w.mode, w.budget, w.quota)
    ctx = skv.Context(w.P, outlier_protect=True)
    dev = skv.workload_to_device(w)
    cache = skv.PagedCache(ctx, w.B, w.Hkv, w.Tmax, w.pool_slots)
    cache.allocate(dev["K"], dev["seq_lens"], dev["utility"], dev["protect"], w.mode,
                   dev["budget"], dev["quota"], dev["free_lists"])
    with pytest.raises(skv.SkvError) as e:
        cache.check()
    assert e.value.code == skv.SKV_ERR_BUDGET
