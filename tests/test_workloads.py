"""The synthetic input recipes: shapes, value structure and reproducibility
of the seeded workloads that stand in for the pages' evaluation inputs
(small sizes where the recipe takes a size argument; the bench's full
sizes for the recipes whose structure depends on them)."""
import math

import numpy as np
import pytest
import torch

from long_context_decode_ada_b200 import workloads as wl


def test_long_context_recipe():
    T = 8192
    w = wl.long_context(T=T)
    assert (w.B, w.Hq, w.Hkv, w.d, w.P, w.Tmax) == (1, 32, 8, 128, 64, T)
    assert w.mode == wl.MODE_BUDGET and w.q_dtype == "bf16"
    assert w.K.dtype == torch.float16 and w.q.dtype == torch.uint16
    prot = w.protect.numpy()
    assert prot[:, :, :64].all() and prot[:, :, T - 1024:].all()
    assert prot[:, :, 64:T - 1024].sum() == 0
    assert int(w.budget[0]) == math.floor(0.40 * T * 8 * 512)
    # Zipf(1.1) over a seeded permutation of positions, per head: the values
    # are (1 + rank)^-1.1, every rank once
    u = w.utility.numpy()[0]
    for h in range(w.Hkv):
        ranks = np.rint(u[h] ** (-1 / 1.1) - 1).astype(np.int64)
        assert sorted(ranks.tolist()) == list(range(T))
    K = w.K.to(torch.float64)
    assert abs(float(K.mean())) < 0.01 and abs(float(K.std()) - 1) < 0.01


def test_recipes_are_reproducible_and_seeded():
    a, b, c = wl.long_context(seed=0, T=2048), wl.long_context(seed=0, T=2048), \
        wl.long_context(seed=1, T=2048)
    assert torch.equal(a.K, b.K) and torch.equal(a.q, b.q) and torch.equal(a.utility, b.utility)
    assert not torch.equal(a.K, c.K)


def test_ragged_batch_recipe():
    w = wl.ragged_batch()
    lens = np.asarray(w.seq_lens)
    assert w.B == 64 and w.P == 16 and (w.Hq, w.Hkv) == (32, 8)
    assert lens.min() >= 1024 and lens.max() <= 8192 and len(set(lens.tolist())) > 40
    q = np.asarray(w.quota)
    np.testing.assert_array_equal(q.sum(1), lens)          # nothing dropped
    assert np.all(np.abs(q[:, 0] - 0.2 * lens) <= 1) and np.all(np.abs(q[:, 1] - 0.4 * lens) <= 1)
    # scattered pages: each free list is a permutation of its pool, not the identity
    for t in range(3):
        f = np.asarray(w.free_lists[t])
        assert sorted(f.tolist()) == list(range(w.pool_slots[t]))
        assert not np.array_equal(f, np.arange(len(f)))


def test_pipeline_layer_outlier_channels():
    w = wl.pipeline_layer(0, T=1024)
    K = w.K.to(torch.float64)
    # per (head, channel) standard deviation: ten channels scaled twentyfold
    sd = K.std(dim=(0, 2))                                  # [Hkv][d]
    big = (sd > 5).nonzero().tolist()
    assert len(big) == round(0.01 * w.Hkv * w.d) == 10
    for h, c in big:
        assert 15 < float(sd[h, c]) < 25
    assert float(sd[sd <= 5].mean()) == pytest.approx(1.0, abs=0.05)
    w31 = wl.pipeline_layer(31, T=1024)
    big31 = (w31.K.to(torch.float64).std(dim=(0, 2)) > 5).nonzero().tolist()
    assert big31 != big                                     # seeded per layer


def test_tiny_and_llama_recipes():
    t = wl.tiny(T=256)
    assert (t.B, t.Hq, t.Hkv, t.P) == (1, 1, 1, 16)
    assert np.asarray(t.quota)[0].tolist() == [0, 0, 256]    # all T2
    w = wl.llama_layer(T=1024, B=2)
    q = np.asarray(w.quota)
    for b in range(2):   # 10 / 50 / 25 % of the tokens to T0 / T1 / T2, the rest dropped
        assert abs(q[b, 0] - 0.10 * 1024) <= 1 and abs(q[b, 1] - 0.50 * 1024) <= 1
        assert abs(q[b, 2] - 0.25 * 1024) <= 1
    # per (head, channel) log-normal scales: the channel spread of K is wide
    sd = w.K.to(torch.float64).std(dim=(0, 2))
    assert float(sd.max() / sd.min()) > 3
