"""Pins of the tier-variant study (oracle/tier_study.py): its grids, its
error measure, and the scaling laws the study must reproduce."""
import math

import numpy as np
import pytest

import oracle
from oracle import tier_study as ts


def test_uniform_two_bit_grid_is_the_kernels_scheme():
    lv, th = ts.uniform_grid(4)
    np.testing.assert_array_equal(lv, [0.5, 1.0, 1.5, 2.0])
    np.testing.assert_array_equal(th, [0.75, 1.25, 1.75])
    d = 128
    for c in range(4):
        assert oracle.rho_level(c, d) == pytest.approx(lv[c] / math.sqrt(d / 2), rel=1e-15)


def test_lloyd_max_is_a_fixed_point_of_lloyds_conditions():
    # one level: the mean of the Rayleigh density, sqrt(pi) / 2
    lv, th = ts.lloyd_max_grid(1)
    assert lv[0] == pytest.approx(math.sqrt(math.pi) / 2, rel=1e-12)
    for L in (2, 4, 8):
        lv, th = ts.lloyd_max_grid(L)
        np.testing.assert_allclose(th, (lv[:-1] + lv[1:]) / 2, rtol=1e-12)
        # each level is the centroid of its cell, by numerical integration
        edges = [0.0] + list(th) + [12.0]
        for j in range(L):
            u = np.linspace(edges[j], edges[j + 1], 200001)
            f = 2 * u * np.exp(-u * u)
            cen = np.trapezoid(u * f, u) / np.trapezoid(f, u)
            assert lv[j] == pytest.approx(cen, rel=1e-6)


def test_error_measure_matches_the_code_domain_logit():
    K, Q = ts.samples(200, 3, False)
    got = ts.rel_logit_error(6, ts.uniform_grid(4), K, Q)
    e2 = r2 = 0.0
    for k, q in zip(K, Q):
        exact = float(np.dot(q, k.astype(np.float64))) / math.sqrt(128)
        e2 += (oracle.logit_codes(q, k.view(np.uint16), 6) - exact) ** 2
        r2 += exact ** 2
    assert got == pytest.approx(math.sqrt(e2 / r2), rel=1e-9)


def test_angle_error_halves_per_bit_and_grids_order_as_expected():
    K, Q = ts.samples(400, 4, False)
    e = {b: ts.rel_logit_error(b, None, K, Q) for b in (4, 5, 6, 7)}
    for b in (4, 5, 6):
        assert 1.7 < e[b] / e[b + 1] < 2.3          # uniform angle quantiser: error ~ 2^-b
    # at equal share bits the MSE-optimal grid is no worse than the uniform one
    for s in (1, 2, 3):
        lm = ts.rel_logit_error(6, ts.lloyd_max_grid(2 ** s), K, Q)
        un = ts.rel_logit_error(6, ts.uniform_grid(2 ** s), K, Q)
        assert lm <= un * 1.01


def test_bytes_per_token_of_the_kernels_tiers():
    assert ts.bytes_per_token(6, 2) == oracle.tier_bytes(1)
    assert ts.bytes_per_token(4, 2) == oracle.tier_bytes(2)
