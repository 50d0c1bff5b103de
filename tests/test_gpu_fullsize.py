"""GPU parity at the full sizes of the configured workloads, in the launch
configuration bench.py times (default split count, runs cut by streamed
bytes): tiers, row map, both page tables and every used page's bytes are
compared with the oracle bit for bit; attention outputs are compared on
sampled (sequence, query head) rows, which the oracle computes one by one.

Workloads: the Llama-3-8B-shaped layer (8 x 32768, P = 64, quota tiers),
the 128K long-context store (budget mode, protected sink and recent
window), the ragged batch of 64 sequences (P = 16, scattered pages) and
eight layers of the 32-layer pipeline (budget mode, outlier channels)."""
import numpy as np
import pytest

import oracle
from long_context_decode_ada_b200 import workloads as wl
from _gpu import assert_close, compare_store, run_gpu

pytestmark = pytest.mark.gpu


def sample_rows(w, n, seed):
    """n (b, hq) rows: the first and last of the batch plus seeded picks,
    always including rows of the longest and the shortest sequence."""
    rng = np.random.default_rng(seed)
    lens = np.asarray(w.seq_lens)
    rows = {(0, 0), (w.B - 1, w.Hq - 1), (int(lens.argmax()), 1), (int(lens.argmin()), w.Hq - 2)}
    while len(rows) < n:
        rows.add((int(rng.integers(w.B)), int(rng.integers(w.Hq))))
    return np.array(sorted(rows), np.int32)


def full_size_check(w, nrows=24, seed=0):
    g = run_gpu(w)  # num_splits = 0: the bench's launch configuration
    ref = oracle.run_workload(w, do_decode=False)
    npages = compare_store(w, g, ref)
    rows = sample_rows(w, nrows, seed)
    out, lse = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, ref["tier"], w.q,
                             w.q_dtype, units=rows)
    b, h = rows[:, 0], rows[:, 1]
    assert_close(g["out"][b, h], out[b, h], "out (sampled rows)")
    assert_close(g["lse"][b, h], lse[b, h], "lse (sampled rows)")
    return g, ref, npages


def test_llama_layer_full_size():
    w = wl.llama_layer()
    g, ref, npages = full_size_check(w, seed=2)
    counts = np.bincount(ref["tier"].ravel(), minlength=4)
    assert counts[0] and counts[1] and counts[2] and counts[3]


def test_long_context_128k_full_size():
    w = wl.long_context()
    g, ref, npages = full_size_check(w, seed=3)
    # the budget holds, and the protected sink and recent window are T0
    tier = ref["tier"]
    assert np.all(tier[:, :, :64] == 0) and np.all(tier[:, :, -1024:] == 0)
    used = sum(int((tier == t).sum()) * oracle.tier_bytes(t) for t in range(3))
    assert used <= int(w.budget[0])


def test_ragged_batch_full_size():
    w = wl.ragged_batch()
    full_size_check(w, nrows=32, seed=4)


@pytest.mark.parametrize("layer", [0, 4, 9, 13, 18, 22, 27, 31])
def test_pipeline_layer_full_size(layer):
    """Eight layers spread over the 32 (each its own outlier channels and
    utilities): store bit-exact, sampled rows within tolerance; the stores
    hold T2 pages and dropped tokens."""
    w = wl.pipeline_layer(layer)
    g, ref, npages = full_size_check(w, nrows=16 if layer not in (0, 31) else 24, seed=5 + layer)
    counts = np.bincount(ref["tier"].ravel(), minlength=4)
    assert counts[1] and counts[2] and counts[3]


def test_long_context_window_roll_full_size():
    """The 128K store built 64 tokens short, 64 decode-time appends, then
    skv_retier of the protected window's oldest 63 rows under the budget
    grown with the appended tokens (the bench's window roll): tiers and row
    map bit-exact against the oracle's re-tiering, every unit's page bytes in
    list order against the oracle's pack of those tiers, and sampled rows of
    the decode against the oracle."""
    import dataclasses

    import torch

    from long_context_decode_ada_b200 import skv
    from test_gpu_append import page_bytes

    w = wl.long_context()
    T, n_app = int(w.seq_lens[0]), 64
    slots = [x + w.B * w.Hkv * (1024 // w.P + 4) for x in w.pool_slots]
    slots[0] += w.B * w.Hkv * (n_app // w.P + 2)
    free = [np.arange(x, dtype=np.uint32) for x in slots]
    wa = dataclasses.replace(w, seq_lens=(w.seq_lens - n_app).astype(np.int32), pool_slots=slots,
                             free_lists=free)
    ctx = skv.Context(w.P)
    da = skv.workload_to_device(wa)
    ca = skv.build_cache(ctx, wa, da)
    ca.check()
    seq = da["seq_lens"].clone()
    for i in range(n_app):
        ca.append(da["K"][:, :, T - n_app + i].contiguous(), da["V"][:, :, T - n_app + i].contiguous(),
                  seq)
    ca.check()
    tier = oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, wa.seq_lens, w.K, w.utility, w.protect,
                           w.mode, w.budget, w.quota)
    tier[:, :, T - n_app:T] = 0
    assert np.array_equal(ca.tier.cpu().numpy(), tier), "tiers after the appends"
    lo = T - 1024
    demote = np.zeros_like(tier)
    demote[:, :, lo:lo + n_app - 1] = 1
    budget = (w.budget + int(0.4 * n_app * w.Hkv * 512)).astype(np.int64)
    exp = oracle.retier(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, tier, demote,
                        budget)
    ca.retier(da["utility"], torch.from_numpy(demote).cuda(), torch.from_numpy(budget).cuda(), seq)
    ca.check()
    assert np.array_equal(ca.tier.cpu().numpy(), exp), "tiers after the re-tiering"
    assert np.any(exp[demote == 1] != 0), "some demoted rows leave T0"
    ref = oracle.pack(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.V, exp, free, slots)
    assert np.array_equal(ca.row_of.cpu().numpy(), ref["row_of"]), "row map"
    ip = ca.page_indptr.cpu().numpy()
    assert np.array_equal(ip, ref["page_indptr"]), "page_indptr"
    ids = ca.page_ids[:ip[-1]].cpu().numpy().view(np.uint32)
    got = page_bytes(ids, ip, [p.cpu().numpy() for p in ca.pools], w.P)
    want = page_bytes(np.asarray(ref["page_ids"], np.uint32), ip, ref["pools"], w.P)
    assert got == want, "page bytes"
    out, lse = ca.decode(da["q"], da["q_dtype"], w.Hq)
    ca.check()
    rows = sample_rows(w, 16, 41)
    ro, rl = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, exp, w.q,
                           w.q_dtype, units=rows)
    b, h = rows[:, 0], rows[:, 1]
    assert_close(out.cpu().numpy()[b, h], ro[b, h], "out (sampled rows)")
    assert_close(lse.cpu().numpy()[b, h], rl[b, h], "lse (sampled rows)")
