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
