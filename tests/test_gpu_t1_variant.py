"""The code variants against the oracle's matching schemes: the T1 variant
(skv_config.t1_angle_bits = 5: 5-bit angle + 3-bit share, the same code
byte) and the Lloyd-Max 2-bit share grid (skv_config.share_grid = 1), alone
and together: the page bytes bit for bit, and the decode within tolerance;
and, against exact fp16 attention, a lower output error than the pinned
6 + 2 scheme."""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_ada_b200 import skv
from long_context_decode_ada_b200 import workloads as wl
from _gpu import assert_close, compare_store

pytestmark = pytest.mark.gpu


def run(w, bits, num_splits=0, grid=0):
    ctx = skv.Context(w.P, t1_angle_bits=bits, share_grid=grid)
    dev = skv.workload_to_device(w)
    cache = skv.build_cache(ctx, w, dev)
    cache.check()
    out, lse = cache.decode(dev["q"], dev["q_dtype"], w.Hq, num_splits=num_splits)
    cache.check()
    return dict(ctx=ctx, cache=cache, dev=dev, out=out.cpu().numpy(), lse=lse.cpu().numpy())


@pytest.mark.parametrize("num_splits", [0, 3])
def test_variant_store_and_decode_against_oracle(num_splits):
    lens = [900, 301, 17]
    w = wl.custom(73, 3, 2, 4, 16, lens, wl.MODE_QUOTA,
                  quota=[[T // 8, T // 2, T // 4] for T in lens])
    g = run(w, 5, num_splits)
    with oracle.t1_scheme(1):
        ref = oracle.run_workload(w)
    compare_store(w, g, ref)
    assert_close(g["out"], ref["out"], "out")
    assert_close(g["lse"], ref["lse"], "lse")


def test_variant_budget_mode_g2_fp16():
    lens = [640, 200]
    w = wl.custom(74, 2, 4, 2, 32, lens, wl.MODE_BUDGET, protect_sink=4, protect_recent=8,
                  zipf_alpha=1.1, q_dtype="fp16",
                  budget=[int(0.35 * T * 4 * 512) + 4 * 31 * 888 + 12 * 4 * 512 for T in lens])
    g = run(w, 5)
    with oracle.t1_scheme(1):
        ref = oracle.run_workload(w)
    compare_store(w, g, ref)
    assert_close(g["out"], ref["out"], "out")
    assert_close(g["lse"], ref["lse"], "lse")


def test_variant_is_closer_to_exact_attention():
    # every token T1: the output error against attention over the fp16 keys
    lens = [2048]
    w = wl.custom(75, 1, 4, 4, 64, lens, wl.MODE_QUOTA, quota=[[0, 2048, 0]])
    exact = np.zeros((1, w.Hkv, w.Tmax), np.uint8)   # all T0: the uncompressed keys
    eo, el = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, exact, w.q,
                           w.q_dtype)
    # the output error is driven by the logit error (softmax weights move by
    # about the logit error; int8 V adds a floor two orders smaller here)
    errs = {}
    for bits in (6, 5):
        g = run(w, bits)
        errs[bits] = (float(np.sqrt(np.mean((g["out"] - eo) ** 2))),
                      float(np.sqrt(np.mean((g["lse"] - el) ** 2))))
    assert errs[5][0] < 0.8 * errs[6][0], errs


def test_variant_long_context_128k_full_size():
    """The 128K store with the T1 variant in the bench's launch
    configuration: tiers, row map and page table bit-exact (the variant
    changes only T1's code bytes), every T1 page's bytes on a sample of
    pages, and sampled rows of the decode against the oracle."""
    w = wl.long_context()
    g = run(w, 5)
    with oracle.t1_scheme(1):
        ref = oracle.run_workload(w, do_decode=False)
        rows = np.array([[0, 0], [0, 9], [0, 22], [0, 31]], np.int32)
        ro, rl = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, ref["tier"],
                               w.q, w.q_dtype, units=rows)
    compare_store(w, g, ref)
    b, h = rows[:, 0], rows[:, 1]
    assert_close(g["out"][b, h], ro[b, h], "out (sampled rows)")
    assert_close(g["lse"][b, h], rl[b, h], "lse (sampled rows)")


@pytest.mark.parametrize("bits", [6, 5])
def test_lloyd_max_share_grid_against_oracle(bits):
    lens = [700, 260]
    w = wl.custom(76, 2, 2, 4, 16, lens, wl.MODE_QUOTA,
                  quota=[[T // 8, T // 3, T // 3] for T in lens])
    g = run(w, bits, grid=1)
    with oracle.t1_scheme(1 if bits == 5 else 0), oracle.share_grid(1):
        ref = oracle.run_workload(w)
    compare_store(w, g, ref)
    assert_close(g["out"], ref["out"], "out")
    assert_close(g["lse"], ref["lse"], "lse")


def test_lloyd_max_grid_lowers_the_t2_error():
    lens = [2048]
    w = wl.custom(77, 1, 4, 4, 64, lens, wl.MODE_QUOTA, quota=[[0, 0, 2048]])
    exact = np.zeros((1, w.Hkv, w.Tmax), np.uint8)
    eo, el = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, exact, w.q,
                           w.q_dtype)
    errs = {}
    for grid in (0, 1):
        g = run(w, 6, grid=grid)
        errs[grid] = float(np.sqrt(np.mean((g["out"] - eo) ** 2)))
    assert errs[1] < errs[0], errs
