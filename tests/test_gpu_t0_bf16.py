"""The fused T0 / bf16 path (skv_config.t0_bf16) against the oracle's bf16 T0
storage (oracle.t0_bf16): T0 rows hold K and V rounded to bf16, T1 / T2
rows are unchanged, and the decode takes the dense kernel's bf16 logit and
P.V steps on T0 pages (SPHERICAL KV technical summary 2.2, precision tiers).

Store: tiers, row map, page table and every page's bytes bit for bit.
Decode tolerance: the suite's |gpu - ref| <= 1e-3 + 2e-3 |ref| plus the
extra rounding of this path.  Its T0 weights enter the P.V product as bf16
(relative error <= 2^-9, against 2^-12 for the fp16 weights of the mixed
kernel), so an output element can move by up to 2^-9 sum_{t in T0} w_t |v_t|
more, w_t the token's softmax weight: that sum is computed per element from
the oracle's lse and the textbook bf16 logits of the T0 rows."""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_ada_b200 import skv
from long_context_decode_ada_b200 import workloads as wl
from _gpu import ATOL, RTOL, compare_store
from test_gpu_utility import assert_utility

pytestmark = pytest.mark.gpu


def t0_bound(w, tier, lse):
    """2^-9 sum_{t in T0} w_t |v_t| per (b, hq, dim), w_t = exp(l_t - lse)."""
    q = (w.q.view(torch.int16).view(torch.bfloat16).double() if w.q_dtype == "bf16"
         else w.q.view(torch.float16).double()).numpy()
    G = w.Hq // w.Hkv
    out = np.zeros((w.B, w.Hq, 128))
    for b in range(w.B):
        T = int(w.seq_lens[b])
        for h in range(w.Hkv):
            sel = torch.from_numpy(np.nonzero(tier[b, h, :T] == 0)[0])
            if sel.numel() == 0:
                continue
            Kb = w.K[b, h, sel].to(torch.bfloat16).double().numpy()
            Vb = np.abs(w.V[b, h, sel].to(torch.bfloat16).double().numpy())
            for hq in range(h * G, (h + 1) * G):
                if not np.isfinite(lse[b, hq]):
                    continue
                wt = np.exp(Kb @ q[b, hq] / np.sqrt(128) - lse[b, hq])
                out[b, hq] = 2.0 ** -9 * (wt[:, None] * Vb).sum(0)
    return out


def check_decode(out, lse, ro, rl, bound):
    err = np.abs(out - ro)
    lim = ATOL + RTOL * np.abs(ro) + bound
    assert np.all(err <= lim), f"out: worst excess {np.max(err - lim):.3g}"
    fin = np.isfinite(rl)
    assert np.array_equal(np.isfinite(lse), fin)
    assert np.all(np.abs(lse[fin] - rl[fin]) <= ATOL + RTOL * np.abs(rl[fin]))


def store_case(w):
    ctx = skv.Context(w.P, t0_bf16=True)
    dev = skv.workload_to_device(w)
    cache = skv.build_cache(ctx, w, dev)
    cache.check()
    with oracle.t0_bf16():
        ref = oracle.run_workload(w)
    compare_store(w, dict(cache=cache), ref)
    out, lse = cache.decode(dev["q"], dev["q_dtype"], w.Hq)
    cache.check()
    return ctx, dev, cache, ref, out.cpu().numpy(), lse.cpu().numpy()


@pytest.mark.parametrize("q_dtype", ["bf16", "fp16"])
def test_budget_store_and_decode(q_dtype):
    w = wl.custom(71, 2, 2, 4, 16, [700, 333], wl.MODE_BUDGET, protect_sink=4,
                  protect_recent=64, zipf_alpha=1.1, q_dtype=q_dtype,
                  budget=[int(0.3 * 700 * 2 * 512)] * 2, scatter=True)
    ctx, dev, cache, ref, out, lse = store_case(w)
    counts = np.bincount(ref["tier"].ravel(), minlength=4)
    assert counts[0] and counts[1] and counts[2] and counts[3]
    check_decode(out, lse, ref["out"], ref["lse"], t0_bound(w, ref["tier"], ref["lse"]))


def test_t0_heavy_quota_store_with_several_splits():
    w = wl.custom(72, 3, 2, 4, 64, [900, 130, 515], wl.MODE_QUOTA,
                  quota=[[300, 300, 200], [60, 40, 20], [200, 200, 100]], k_scale=2.0)
    ctx, dev, cache, ref, out, lse = store_case(w)
    bound = t0_bound(w, ref["tier"], ref["lse"])
    check_decode(out, lse, ref["out"], ref["lse"], bound)
    for splits in (7, 40):
        o, l = cache.decode(dev["q"], dev["q_dtype"], w.Hq, num_splits=splits)
        cache.check()
        check_decode(o.cpu().numpy(), l.cpu().numpy(), ref["out"], ref["lse"], bound)


def test_utility_decode_on_bf16_t0_pages():
    """The logit-capturing variant of the path: the same outputs, and the
    utility update against the oracle's attention mass over bf16 T0 rows
    (the T0 logits are the bf16 path's; the tolerance of test_gpu_utility
    covers them since the logits are as exact as the fp16 path's)."""
    w = wl.custom(73, 1, 2, 4, 16, [400], wl.MODE_QUOTA, quota=[[120, 180, 60]])
    ctx, dev, cache, ref, out, lse = store_case(w)
    u0 = np.random.default_rng(3).random((w.B, w.Hkv, w.Tmax)).astype(np.float32)
    ut = torch.from_numpy(u0).to(cache.device)
    o, l = cache.decode_utility(dev["q"], dev["q_dtype"], w.Hq, dev["seq_lens"], ut, gamma=0.5)
    cache.check()
    check_decode(o.cpu().numpy(), l.cpu().numpy(), ref["out"], ref["lse"],
                 t0_bound(w, ref["tier"], ref["lse"]))
    with oracle.t0_bf16():
        mass = oracle.attention_mass(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K,
                                     ref["tier"], w.q, w.q_dtype)
    want = 0.5 * u0.astype(np.float64) + mass
    assert_utility(ut.cpu().numpy(), want, "utility")


def test_appended_rows_are_bf16():
    """Appended tokens join the T0 pages as bf16: after the appends the store
    equals the oracle's bf16 pack of the tiers with the new positions T0."""
    n = 21
    w_full = wl.custom(74, 2, 2, 4, 16, [300, 260], wl.MODE_QUOTA,
                       quota=[[40, 100, 80], [30, 90, 70]])
    seq0 = (w_full.seq_lens - n).astype(np.int32)
    slots = list(w_full.pool_slots)
    slots[0] += 8
    free = [np.arange(s, dtype=np.uint32) for s in slots]
    w0 = dataclasses.replace(w_full, seq_lens=seq0, pool_slots=slots, free_lists=free)
    ctx = skv.Context(16, t0_bf16=True)
    dev = skv.workload_to_device(w0)
    cache = skv.build_cache(ctx, w0, dev)
    cache.check()
    seq = dev["seq_lens"].clone()
    for step in range(n):
        K_new = torch.stack([dev["K"][b, :, int(seq0[b]) + step] for b in range(w0.B)]).contiguous()
        V_new = torch.stack([dev["V"][b, :, int(seq0[b]) + step] for b in range(w0.B)]).contiguous()
        cache.append(K_new, V_new, seq)
        cache.check()
    tier = oracle.allocate(w0.B, w0.Hkv, w0.Tmax, w0.d, 16, seq0, w0.K, w0.utility, w0.protect,
                           w0.mode, w0.budget, w0.quota)
    for b in range(w0.B):
        tier[b, :, int(seq0[b]):int(w_full.seq_lens[b])] = 0
    with oracle.t0_bf16():
        ref = oracle.pack(w0.B, w0.Hkv, w0.Tmax, w0.d, 16, w_full.seq_lens, w0.K, w0.V, tier,
                          free, slots)
    from test_gpu_append import page_bytes
    ip = cache.page_indptr.cpu().numpy()
    assert np.array_equal(ip, ref["page_indptr"])
    ids = cache.page_ids[:ip[-1]].cpu().numpy().view(np.uint32)
    got = page_bytes(ids, ip, [p.cpu().numpy() for p in cache.pools], 16)
    exp = page_bytes(np.asarray(ref["page_ids"], np.uint32), ip, ref["pools"], 16)
    assert got == exp


def test_retier_and_variant_combinations_are_refused():
    with pytest.raises(skv.SkvError) as e:
        skv.Context(16, t0_bf16=True, t1_angle_bits=5)
    assert e.value.code == skv.SKV_ERR_ARG
    with pytest.raises(skv.SkvError) as e:
        skv.Context(16, t0_bf16=True, share_grid=1)
    assert e.value.code == skv.SKV_ERR_ARG
    w = wl.custom(75, 1, 1, 4, 16, [100], wl.MODE_BUDGET, protect_recent=20, zipf_alpha=1.1,
                  budget=[30000])
    ctx, dev, cache, ref, out, lse = store_case(w)
    demote = torch.zeros((1, 1, w.Tmax), dtype=torch.uint8, device=cache.device)
    with pytest.raises(skv.SkvError) as e:
        cache.retier(dev["utility"], demote, dev["budget"], dev["seq_lens"])
    assert e.value.code == skv.SKV_ERR_ARG


def test_long_context_store_full_size():
    """The 128K store with bf16 T0 pages (the bench's fused-path variant):
    tiers, row map, page tables and every page's bytes bit-exact against the
    oracle's bf16 T0 pack; sampled rows of the decode against the oracle
    within the bound above."""
    from test_gpu_fullsize import sample_rows
    w = wl.long_context()
    ctx = skv.Context(w.P, t0_bf16=True)
    dev = skv.workload_to_device(w)
    cache = skv.build_cache(ctx, w, dev)
    cache.check()
    with oracle.t0_bf16():
        ref = oracle.run_workload(w, do_decode=False)
        compare_store(w, dict(cache=cache), ref)
        rows = sample_rows(w, 16, 77)
        ro, rl = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, ref["tier"],
                               w.q, w.q_dtype, units=rows)
    out, lse = cache.decode(dev["q"], dev["q_dtype"], w.Hq)
    cache.check()
    b, h = rows[:, 0], rows[:, 1]
    bound = t0_bound(w, ref["tier"], rl)[b, h]
    check_decode(out.cpu().numpy()[b, h], lse.cpu().numpy()[b, h], ro[b, h], rl[b, h], bound)
