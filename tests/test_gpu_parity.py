"""GPU parity: the CUDA path through the C-ABI against the oracle.

Bit-exact: tiers, row map, page table, every used page's bytes.
Attention out and lse: |gpu - ref| <= 1e-3 + 2e-3 |ref| (the fp32-accumulated
output tolerance of the pinned scheme)."""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_ada_b200 import skv
from long_context_decode_ada_b200 import workloads as wl
from _gpu import assert_close, compare_store, run_gpu, upload_oracle_store

pytestmark = pytest.mark.gpu


def full_check(w, num_splits=0, decode_oracle_pages=True):
    ref = oracle.run_workload(w)
    g = run_gpu(w, num_splits=num_splits)
    compare_store(w, g, ref)
    assert_close(g["out"], ref["out"], "out")
    assert_close(g["lse"], ref["lse"], "lse")
    if decode_oracle_pages:
        cache = upload_oracle_store(g["ctx"], w, ref)
        out, lse = cache.decode(g["dev"]["q"], g["dev"]["q_dtype"], w.Hq, num_splits=num_splits)
        cache.check()
        assert_close(out.cpu().numpy(), ref["out"], "out (oracle pages)")
        assert_close(lse.cpu().numpy(), ref["lse"], "lse (oracle pages)")
    return g, ref


def test_tiny_all_t2_config():
    """B=1, one head, T=4096, P=16, every token T2, fp16 q."""
    w = wl.tiny(seed=0)
    g, ref = full_check(w)
    assert np.all(ref["tier"] == 2)


@pytest.mark.parametrize("P", [16, 32, 64])
@pytest.mark.parametrize("G", [1, 2, 4])
def test_quota_mixed_tiers_ragged(P, G):
    lens = [1000, 129, 517]
    quota = [[int(0.1 * T), int(0.5 * T), int(0.25 * T)] for T in lens]
    w = wl.custom(40 + P + G, 3, 2, G, P, lens, wl.MODE_QUOTA, quota=quota,
                  q_dtype="bf16" if G != 2 else "fp16", scatter=(P == 16))
    full_check(w)


def test_budget_mode_long_context_small():
    T = 3000
    w = wl.custom(50, 1, 2, 4, 64, [T], wl.MODE_BUDGET, protect_sink=64, protect_recent=256,
                  zipf_alpha=1.1, budget=[int(0.4 * T * 2 * 512)])
    w = wl._finish("budget_small", w.B, w.Hq, w.Hkv, w.P, w.Tmax, w.seq_lens, w.K, w.V, w.q,
                   w.q_dtype, w.mode, w.utility, w.protect, w.budget, w.quota, 50, False)
    g, ref = full_check(w)
    counts = np.bincount(ref["tier"].ravel(), minlength=4)
    assert counts[0] > 0 and counts[1] > 0 and counts[3] >= 0


def test_budget_mode_batch_with_outliers():
    lens = [700, 1300]
    B, Hkv = 2, 2
    w = wl.custom(51, B, Hkv, 4, 32, lens, wl.MODE_BUDGET, zipf_alpha=1.2,
                  budget=[int(0.3 * T * Hkv * 512) for T in lens], k_scale=1.0)
    K = w.K.float()
    K[:, 1, :, 5] *= 20
    K[:, 0, :, 77] *= 20
    w.K = K.to(torch.float16)
    w = wl._finish("outliers", w.B, w.Hq, w.Hkv, w.P, w.Tmax, w.seq_lens, w.K, w.V, w.q,
                   w.q_dtype, w.mode, w.utility, w.protect, w.budget, w.quota, 51, False)
    full_check(w)


@pytest.mark.parametrize("splits", [1, 2, 7, 64, 1000])
def test_split_counts_do_not_change_results(splits):
    lens = [600, 20, 333]
    w = wl.custom(60, 3, 2, 4, 16, lens, wl.MODE_QUOTA,
                  quota=[[T // 5, 2 * T // 5, T // 4] for T in lens], scatter=True)
    full_check(w, num_splits=splits, decode_oracle_pages=False)


@pytest.mark.parametrize("splits", [1, 3, 148, 5000])
def test_split_by_bytes_and_by_pages_agree_with_oracle(splits):
    """The decode cuts the page list into runs of equal bytes (per-tier
    offsets given) or of equal page counts (offsets withheld); both, at run
    counts from one up to far more runs than pages (empty runs, pages
    costlier than a run), match the oracle."""
    lens = [900, 64, 2500, 17]
    w = wl.custom(63, 4, 2, 4, 64, lens, wl.MODE_QUOTA,
                  quota=[[T // 3, T // 3, T // 6] for T in lens], scatter=True)
    ref = oracle.run_workload(w)
    g = run_gpu(w, num_splits=splits)
    cache = g["cache"]
    for by_bytes in (True, False):
        cache.split_by_bytes = by_bytes
        out, lse = cache.decode(g["dev"]["q"], g["dev"]["q_dtype"], w.Hq, num_splits=splits)
        cache.check()
        assert_close(out.cpu().numpy(), ref["out"], f"out (by_bytes={by_bytes})")
        assert_close(lse.cpu().numpy(), ref["lse"], f"lse (by_bytes={by_bytes})")


def test_edge_cases_empty_dropped_single():
    # seq 0 empty, seq 1 has every token dropped, seq 2 a single token, seq 3 ragged tail
    lens = [0, 40, 1, 77]
    quota = [[0, 0, 0], [0, 0, 0], [0, 1, 0], [3, 30, 40]]
    w = wl.custom(61, 4, 2, 4, 16, lens, wl.MODE_QUOTA, quota=quota)
    g, ref = full_check(w)
    assert np.all(g["out"][0] == 0) and np.all(np.isneginf(g["lse"][0]))
    assert np.all(g["out"][1] == 0) and np.all(np.isneginf(g["lse"][1]))


def test_large_and_small_magnitudes():
    lens = [300]
    w = wl.custom(62, 1, 1, 4, 64, lens, wl.MODE_QUOTA, quota=[[50, 150, 100]], k_scale=6.0)
    # queries with large and tiny entries
    q = w.q.view(torch.int16).view(torch.bfloat16).float()
    q[0, 0] *= 4.0
    q[0, 1] *= 1e-3
    w.q = wl.to_bf16_bits(q)
    full_check(w)


def test_dense_bf16_baseline_matches_textbook():
    lens = [500, 231]
    w = wl.custom(70, 2, 2, 4, 64, lens, wl.MODE_QUOTA, quota=[[0, 0, 0]] * 2)
    ctx = skv.Context(64)
    dev = skv.workload_to_device(w)
    n_pages = sum(2 * (-(-T // 64)) for T in lens)
    dc = skv.DenseCache(ctx, w.B, w.Hkv, w.Tmax, n_pages + 3)
    perm = torch.randperm(n_pages + 3, generator=torch.Generator().manual_seed(1)).to(torch.int32)
    dc.pack(dev["K"], dev["V"], dev["seq_lens"], perm)
    dc.check()
    out, lse = dc.decode(dev["q"], dev["q_dtype"], w.Hq)
    dc.check()
    Kb = w.K.to(torch.bfloat16).double().numpy()
    Vb = w.V.to(torch.bfloat16).double().numpy()
    qf = w.q.view(torch.int16).view(torch.bfloat16).double().numpy()
    ref = np.zeros((w.B, w.Hq, 128))
    rlse = np.zeros((w.B, w.Hq))
    for b in range(w.B):
        for hq in range(w.Hq):
            h = hq // 4
            T = lens[b]
            l = Kb[b, h, :T] @ qf[b, hq] / np.sqrt(128)
            m = l.max()
            e = np.exp(l - m)
            ref[b, hq] = (e[:, None] * Vb[b, h, :T]).sum(0) / e.sum()
            rlse[b, hq] = m + np.log(e.sum())
    # P is rounded to bf16 for the tensor-core P.V: relative error ~2^-9 per weight
    got = out.cpu().numpy()
    assert np.max(np.abs(got - ref)) < 5e-3
    assert_close(lse.cpu().numpy(), rlse, "dense lse")


def test_corrupt_page_id_is_reported_without_fault():
    w = wl.custom(80, 1, 1, 4, 16, [100], wl.MODE_QUOTA, quota=[[10, 50, 40]])
    g = run_gpu(w, decode=False)
    cache = g["cache"]
    cache.page_ids[2] = (1 << 30) | (cache.pool_slots[1] + 5)   # slot out of range
    out, lse = cache.decode(g["dev"]["q"], g["dev"]["q_dtype"], w.Hq)
    with pytest.raises(skv.SkvError) as e:
        cache.check()
    assert e.value.code == skv.SKV_ERR_CORRUPT
    cache.page_ids[2] = (3 << 30) - (1 << 32)   # tier 3 does not exist (as int32)
    cache.decode(g["dev"]["q"], g["dev"]["q_dtype"], w.Hq)
    with pytest.raises(skv.SkvError) as e:
        cache.check()
    assert e.value.code == skv.SKV_ERR_CORRUPT


def test_budget_and_pool_errors():
    w = wl.custom(81, 1, 2, 4, 16, [200], wl.MODE_BUDGET, protect_sink=150, zipf_alpha=1.1,
                  budget=[150 * 2 * 512])   # protected bytes alone exceed budget - reserve
    ctx = skv.Context(16)
    dev = skv.workload_to_device(w)
    cache = skv.PagedCache(ctx, w.B, w.Hkv, w.Tmax, [100, 100, 100])
    cache.allocate(dev["K"], dev["seq_lens"], dev["utility"], dev["protect"], w.mode,
                   dev["budget"], dev["quota"], dev["free_lists"])
    with pytest.raises(skv.SkvError) as e:
        cache.check()
    assert e.value.code == skv.SKV_ERR_BUDGET
    w2 = wl.custom(82, 1, 1, 4, 16, [200], wl.MODE_QUOTA, quota=[[0, 200, 0]])
    dev2 = skv.workload_to_device(w2)
    cache2 = skv.PagedCache(ctx, 1, 1, 200, [20, 5, 20])
    short = [torch.arange(20, dtype=torch.int32), torch.arange(5, dtype=torch.int32),
             torch.arange(20, dtype=torch.int32)]
    cache2.allocate(dev2["K"], dev2["seq_lens"], dev2["utility"], None, w2.mode, None,
                    dev2["quota"], short)
    with pytest.raises(skv.SkvError) as e:
        cache2.check()
    assert e.value.code == skv.SKV_ERR_POOL


def test_permuted_slots_give_identical_outputs():
    lens = [400, 250]
    quota = [[40, 160, 120], [25, 100, 75]]
    w1 = wl.custom(90, 2, 2, 4, 16, lens, wl.MODE_QUOTA, quota=quota, scatter=False)
    w2 = wl.custom(90, 2, 2, 4, 16, lens, wl.MODE_QUOTA, quota=quota, scatter=True)
    g1 = run_gpu(w1)
    g2 = run_gpu(w2)
    assert np.array_equal(g1["cache"].tier.cpu().numpy(), g2["cache"].tier.cpu().numpy())
    np.testing.assert_allclose(g1["out"], g2["out"], rtol=0, atol=2e-6)


def test_gqa_group_equals_single_head_runs():
    lens = [300]
    w = wl.custom(91, 1, 2, 4, 16, lens, wl.MODE_QUOTA, quota=[[30, 120, 90]])
    g = run_gpu(w)
    for hq in range(w.Hq):
        h = hq // 4
        w1 = wl.custom(91, 1, 2, 4, 16, lens, wl.MODE_QUOTA, quota=[[30, 120, 90]])
        w1.K = w.K[:, h:h + 1].contiguous()
        w1.V = w.V[:, h:h + 1].contiguous()
        w1.utility = w.utility[:, h:h + 1].contiguous()
        w1.q = w.q[:, hq:hq + 1].contiguous()
        w1.Hkv, w1.Hq = 1, 1
        w1 = wl._finish("one", 1, 1, 1, 16, w.Tmax, w.seq_lens, w1.K, w1.V, w1.q, w.q_dtype,
                        w.mode, w1.utility, None, w.budget, w.quota, 91, False)
        g1 = run_gpu(w1)
        np.testing.assert_allclose(g1["out"][0, 0], g["out"][0, hq], rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("splits", [0, 16, 40])
def test_dynamic_chunks_eager_and_graph_replays(splits):
    """Unit-aligned split (num_splits >= 8 units): the last eighth of each
    unit's pages is handed out at run time through a per-unit counter that
    every launch tags and resets.  Eager calls and every replay of a
    captured CUDA graph (several decodes per replay, one workspace) match
    the oracle.  The chunk assignment may differ between launches, and with
    it which rows share a warp's running maximum (the scale at which P is
    rounded to fp16 for the P.V MMA): replays agree with each other to
    1e-4, ten times inside the parity tolerance."""
    lens = [9000, 6100]
    quota = [[T // 10, 6 * T // 10, T // 5] for T in lens]
    w = wl.custom(64, 2, 2, 4, 64, lens, wl.MODE_QUOTA, quota=quota, scatter=True)
    ref = oracle.run_workload(w)
    g = run_gpu(w, num_splits=splits)
    assert_close(g["out"], ref["out"], "out (eager)")
    assert_close(g["lse"], ref["lse"], "lse (eager)")
    cache, dev = g["cache"], g["dev"]
    ws = cache.workspace(w.Hq, splits)
    out = torch.empty((w.B, w.Hq, 128), dtype=torch.float32, device="cuda")
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        for _ in range(3):
            cache.decode(dev["q"], dev["q_dtype"], w.Hq, out=out, lse=lse, workspace=ws,
                         num_splits=splits)
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr, stream=s):
            for _ in range(3):
                cache.decode(dev["q"], dev["q_dtype"], w.Hq, out=out, lse=lse, workspace=ws,
                             num_splits=splits)
    torch.cuda.synchronize()
    first = None
    for rep in range(5):
        out.zero_()
        gr.replay()
        torch.cuda.synchronize()
        cache.check()
        o = out.cpu().numpy()
        assert_close(o, ref["out"], f"out (replay {rep})")
        assert_close(lse.cpu().numpy(), ref["lse"], f"lse (replay {rep})")
        if first is None:
            first = o
        np.testing.assert_allclose(o, first, rtol=0, atol=1e-4)


def test_deterministic_context_gives_bit_identical_calls():
    """skv_config.deterministic: the unit-aligned split keeps every page in
    a static run (no run-time chunks), so repeated calls and graph replays
    return bit-identical results, which also match the oracle."""
    lens = [9000, 6100]
    quota = [[T // 10, 6 * T // 10, T // 5] for T in lens]
    w = wl.custom(64, 2, 2, 4, 64, lens, wl.MODE_QUOTA, quota=quota, scatter=True)
    ref = oracle.run_workload(w)
    ctx = skv.Context(w.P, deterministic=True)
    g = run_gpu(w, ctx=ctx)
    assert_close(g["out"], ref["out"], "out")
    cache, dev = g["cache"], g["dev"]
    outs = []
    for _ in range(4):
        o, l = cache.decode(dev["q"], dev["q_dtype"], w.Hq)
        cache.check()
        outs.append((o.cpu().numpy(), l.cpu().numpy()))
    for o, l in outs[1:]:
        assert np.array_equal(o, outs[0][0]) and np.array_equal(l, outs[0][1])
    assert np.array_equal(outs[0][0], g["out"])
