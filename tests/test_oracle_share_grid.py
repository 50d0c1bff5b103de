"""Pins of the oracle's non-uniform (Lloyd-Max) 2-bit share grid: its exact
levels and thresholds against the numerical Lloyd-Max optimum of the
Rayleigh density, the code against exact rationals and an exact tie, and the
compressed-domain logit against the tier study's measure."""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from oracle import tier_study as ts

LEVELS = np.array([383, 807, 1249, 1831]) / 1024
THRESH = np.sqrt(np.array([22, 64, 145]) / 64)


def test_exact_grid_is_next_to_the_optimum():
    lv, th = ts.lloyd_max_grid(4)
    np.testing.assert_allclose(LEVELS, lv, atol=5e-4)
    np.testing.assert_allclose(THRESH, th, atol=6e-3)
    assert np.all(LEVELS[:-1] < THRESH) and np.all(THRESH < LEVELS[1:])
    with oracle.share_grid(1):
        for c in range(4):
            assert oracle.rho_level(c, 128) == pytest.approx(LEVELS[c] / 8, rel=1e-15)
    assert oracle.rho_level(2, 128) == pytest.approx(1.5 / 8, rel=1e-15)   # default restored


def exact_code(x, y, k):
    v = [Fraction(float(t)) for t in k.astype(np.float16)]
    r2 = sum(t * t for t in v)
    u2 = (Fraction(float(np.float16(x))) ** 2 + Fraction(float(np.float16(y))) ** 2) * 64 / r2
    return sum(1 for n in (22, 64, 145) if u2 > Fraction(n, 64))


def test_code_against_fractions_and_a_tie():
    rng = np.random.default_rng(21)
    with oracle.share_grid(1):
        for i in range(200):
            k = (rng.standard_normal(128) * (4.0 if i % 4 == 0 else 1.0)).astype(np.float16)
            R2 = oracle.norm2(k.view(np.uint16))
            for p in rng.integers(0, 64, 4):
                p = int(p)
                x, y = int(k[2 * p].view(np.uint16)), int(k[2 * p + 1].view(np.uint16))
                assert oracle.rho_code(x, y, R2, 128) == exact_code(k[2 * p], k[2 * p + 1], k)
        # u = 1 exactly: pair (2, 0), the rest 15^2 + 5^2 + 1 + 1 = 252, r^2 = 256
        k = np.zeros(128, np.float16)
        k[0] = 2.0
        k[2:6] = [15.0, 5.0, 1.0, 1.0]
        R2 = oracle.norm2(k.view(np.uint16))
        x, y = int(k[0].view(np.uint16)), int(k[1].view(np.uint16))
        assert oracle.rho_code(x, y, R2, 128) == 1          # a tie goes to the lower code
        k2 = k.copy()
        k2[1] = 0.0625
        R2b = oracle.norm2(k2.view(np.uint16))
        assert oracle.rho_code(x, int(k2[1].view(np.uint16)), R2b, 128) == 2


def test_logit_matches_the_study_and_improves_on_uniform():
    K, Q = ts.samples(300, 5, False)
    with oracle.share_grid(1):
        e2 = r2 = 0.0
        for k, q in zip(K, Q):
            exact = float(np.dot(q, k.astype(np.float64))) / math.sqrt(128)
            e2 += (oracle.logit_codes(q, k.view(np.uint16), 4) - exact) ** 2
            r2 += exact ** 2
    got = math.sqrt(e2 / r2)
    assert got == pytest.approx(ts.rel_logit_error(4, (LEVELS, THRESH), K, Q), rel=1e-9)
    assert got < ts.rel_logit_error(4, ts.uniform_grid(4), K, Q)
