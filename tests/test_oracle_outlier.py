"""Pins of the oracle's outlier flag (outlier-aware protection: a key with a
pair whose share lies far beyond the 2-bit share grid is kept at the top
tier, SPHERICAL KV Technical Summary section 2.2, protection constraints).

The flag is: some pair i has u_i = (rho_i / r) sqrt(d/2) > 4.  Pinned by
exact rational arithmetic on the fp16 values (Python fractions), by keys
whose u sits exactly on the threshold, and by the outlier-channel recipe."""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_ada_b200 import workloads as wl


def exact_flag(k: np.ndarray) -> bool:
    v = [Fraction(float(x)) for x in k.astype(np.float16)]
    d = len(v)
    r2 = sum(x * x for x in v)
    if r2 == 0:
        return False
    for i in range(d // 2):
        rho2 = v[2 * i] ** 2 + v[2 * i + 1] ** 2
        if rho2 * Fraction(d, 2) > 16 * r2:      # u^2 > 16
            return True
    return False


def test_one_hot_and_uniform_keys():
    for d in (128, 64, 36):
        k = np.zeros(d, np.float16)
        k[5] = 3.0
        assert oracle.outlier(k.view(np.uint16))          # u = sqrt(d/2) > 4
    k = np.zeros(32, np.float16)
    k[5] = 3.0
    assert not oracle.outlier(k.view(np.uint16))          # u = 4 exactly: a tie
    assert not oracle.outlier(np.full(128, 0.5, np.float16).view(np.uint16))   # u = 1
    assert not oracle.outlier(np.zeros(128, np.float16).view(np.uint16))       # r = 0


def test_threshold_is_exact():
    # d = 128: u^2 = 64 rho^2 / r^2 > 16  <=>  rho^2 / r^2 > 1/4
    # pair 0 = (8, 0): rho^2 = 64; the rest sums to 192: r^2 = 256, u = 4
    k = np.zeros(128, np.float16)
    k[0] = 8.0
    k[2:14] = 4.0                 # 12 * 16 = 192
    assert not oracle.outlier(k.view(np.uint16))
    k2 = k.copy()
    k2[1] = 0.0625                # rho^2 = 64 + 2^-8: just above a quarter
    assert oracle.outlier(k2.view(np.uint16))
    k3 = k.copy()
    k3[14] = 0.0625               # r^2 grows instead: just below
    assert not oracle.outlier(k3.view(np.uint16))


def test_random_keys_against_fractions():
    rng = np.random.default_rng(7)
    n_true = 0
    for i in range(400):
        d = int(rng.choice([16, 32, 128]))
        k = rng.standard_normal(d)
        if i % 2:
            j = int(rng.integers(d))
            k[j] *= float(rng.choice([4.0, 20.0, 50.0]))
        k = k.astype(np.float16)
        want = exact_flag(k)
        n_true += want
        assert oracle.outlier(k.view(np.uint16)) == want, (i, d)
    assert 20 < n_true < 380     # both outcomes are exercised


def test_flags_follow_the_outlier_channels():
    w = wl.custom(51, 2, 2, 1, 16, [200, 77], wl.MODE_QUOTA, quota=[[0, 0, 0]] * 2)
    K = w.K.clone()
    K[:, 1, :, 17] *= 20          # kv head 1: one channel twentyfold (the outlier recipe)
    flags = oracle.outlier_flags(w.B, w.Hkv, w.Tmax, w.d, w.seq_lens, K)
    for b, T in enumerate([200, 77]):
        assert flags[b, 1, :T].mean() > 0.5    # unless the channel's own draw is small
        assert flags[b, 0, :T].sum() == 0          # Gaussian keys: about 1 in 10^5
        assert np.all(flags[b, :, T:] == 0)
    for b, h, t in [(0, 0, 3), (0, 1, 150), (1, 1, 76)]:
        assert flags[b, h, t] == exact_flag(K[b, h, t].numpy())


def test_protecting_flagged_keys_keeps_them_t0():
    lens = [300]
    w = wl.custom(52, 1, 2, 4, 16, lens, wl.MODE_BUDGET, zipf_alpha=1.1,
                  budget=[int(0.3 * 300 * 2 * 512) + 2 * 15 * 888])
    K = w.K.clone()
    K[0, 0, ::7, 40] *= 20
    flags = oracle.outlier_flags(w.B, w.Hkv, w.Tmax, w.d, w.seq_lens, K)
    assert flags.sum() > 30
    tier = oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, K, w.utility, flags,
                           w.mode, w.budget, w.quota)
    assert np.all(tier[flags == 1] == 0)
