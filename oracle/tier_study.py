"""Bytes per token versus logit error of tier variants, computed with the
oracle (test infrastructure: it runs only the oracle's CPU arithmetic).

A compressed tier stores, per (token, kv head): the fp16 radius r~ (2 B),
per pair a b-bit angle code and an s-bit share code (64 pairs at d = 128),
and int8 V with an fp16 scale (130 B).  The variants differ in b, in s and
in the share grid: the levels of u = (rho_i / r) sqrt(d/2), the pair's
share scaled so that u^2 is about Exp(1) for Gaussian keys (u is then
Rayleigh distributed, density 2u exp(-u^2)).

Grids:
- "uniform": L = 2^s levels (j + 1) * 2 / L, j < L, thresholds at the
  midpoints (s = 2 is the scheme the kernels use: levels 0.5 .. 2.0);
- "lloyd-max": the L levels and thresholds that minimise E[(u^ - u)^2]
  under the Rayleigh density (Lloyd's iteration: thresholds at midpoints,
  levels at the centroids of their cells, closed-form integrals);
- "exact": the share unquantised (the limit s -> infinity).

Error: sqrt(E[(l^ - l)^2] / E[l^2]) over seeded (key, query) pairs, l the
logit q . k / sqrt(d) of the fp16 key in fp64, l^ the variant's
compressed-domain logit (oracle.logit_grid).  Two key sets: N(0,1) keys,
and keys with one channel scaled twentyfold (an outlier channel).

Run: python -m oracle.tier_study [--n 2000]   (prints a markdown table)
"""
from __future__ import annotations

import argparse
import math

import numpy as np

import oracle

D = 128


def uniform_grid(L: int, umax: float = 2.0):
    levels = np.array([(j + 1) * umax / L for j in range(L)])
    return levels, (levels[:-1] + levels[1:]) / 2


def _rayleigh_mass(a: float, b: float) -> float:
    return math.exp(-a * a) - (math.exp(-b * b) if math.isfinite(b) else 0.0)


def _rayleigh_first_moment(a: float, b: float) -> float:
    """integral over [a, b] of u * 2u exp(-u^2) du."""
    eb = b * math.exp(-b * b) if math.isfinite(b) else 0.0
    erf_b = math.erf(b) if math.isfinite(b) else 1.0
    return (a * math.exp(-a * a) - eb) + math.sqrt(math.pi) / 2 * (erf_b - math.erf(a))


def lloyd_max_grid(L: int, iters: int = 500):
    """Levels and thresholds of the MSE-optimal L-level quantiser of a
    Rayleigh variable (density 2u exp(-u^2) on u >= 0)."""
    levels = np.array([(j + 0.5) * 2.0 / L for j in range(L)])
    for _ in range(iters):
        th = (levels[:-1] + levels[1:]) / 2
        edges = [0.0] + list(th) + [math.inf]
        levels = np.array([_rayleigh_first_moment(edges[j], edges[j + 1]) /
                           _rayleigh_mass(edges[j], edges[j + 1]) for j in range(L)])
    return levels, (levels[:-1] + levels[1:]) / 2


def bytes_per_token(b: int, s_bits: int) -> float:
    return 2 + D // 2 * (b + s_bits) / 8 + 128 + 2


def samples(n: int, seed: int, outlier: bool):
    rng = np.random.default_rng(seed)
    K = rng.standard_normal((n, D))
    if outlier:
        K[:, 17] *= 20.0
    Q = rng.standard_normal((n, D))
    return K.astype(np.float16), Q


def rel_logit_error(b: int, grid, K: np.ndarray, Q: np.ndarray) -> float:
    levels, th = grid if grid is not None else (None, None)
    err2 = ref2 = 0.0
    for k, q in zip(K, Q):
        exact = float(np.dot(q, k.astype(np.float64))) / math.sqrt(D)
        got = oracle.logit_grid(q, k.view(np.uint16), b, levels, th)
        err2 += (got - exact) ** 2
        ref2 += exact ** 2
    return math.sqrt(err2 / ref2)


def variants():
    for b in (3, 4, 5, 6, 7, 8):
        yield b, "exact", 0, None
        for s in (1, 2, 3):
            yield b, "uniform", s, uniform_grid(2 ** s)
            yield b, "lloyd-max", s, lloyd_max_grid(2 ** s)


def table(n: int = 2000, seed: int = 0) -> str:
    Kg, Qg = samples(n, seed, False)
    Ko, Qo = samples(n, seed + 1, True)
    rows = ["| angle bits b | share grid | share bits | bytes / token | rel. logit error "
            "(Gaussian keys) | rel. logit error (outlier channel) |",
            "|---|---|---|---|---|---|"]
    for b, name, s, grid in variants():
        eg = rel_logit_error(b, grid, Kg, Qg)
        eo = rel_logit_error(b, grid, Ko, Qo)
        by = f"{bytes_per_token(b, s):.0f}" if name != "exact" else "-"
        rows.append(f"| {b} | {name} | {s if name != 'exact' else '-'} | {by} | {eg:.4f} | "
                    f"{eo:.4f} |")
    return "\n".join(rows)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--n", type=int, default=2000)
    ap.add_argument("--seed", type=int, default=0)
    a = ap.parse_args()
    for L in (2, 4, 8):
        lv, th = lloyd_max_grid(L)
        print(f"lloyd-max L={L}: levels {np.round(lv, 4).tolist()} thresholds "
              f"{np.round(th, 4).tolist()}")
    print(table(a.n, a.seed))


if __name__ == "__main__":
    main()
