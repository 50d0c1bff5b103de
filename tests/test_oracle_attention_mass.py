"""Pins of the oracle's attention mass (the per-token utility signal).

The mass of a resident token is the softmax weight it receives in the decode
(SPHERICAL KV, Technical Summary section 2.1: the attention over the
compressed-domain logits), summed over the query heads that share its kv
head.  Pinned here by:
(1) all tokens T0: textbook softmax weights of q K^T / sqrt(d) in numpy;
(2) mixed tiers: the same softmax over the keys rebuilt by the separately
    pinned reconstruction primitive (dropped tokens left out);
(3) invariants: sum_t mass = G for every unit with a resident token, 0 for
    dropped tokens, positions >= seq_lens[b] and units with nothing resident;
(4) a d = 2 case whose logits are derived by hand;
(5) the decode's output is the mass-weighted value sum: for a group of
    one query head, out = sum_t mass_t v^_t."""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_ada_b200 import workloads as wl


def q_f64(w):
    if w.q_dtype == "bf16":
        return w.q.view(torch.int16).view(torch.bfloat16).to(torch.float64).numpy()
    return w.q.to(torch.float64).numpy()


def tiers_of(w):
    return oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, w.protect,
                           w.mode, w.budget, w.quota)


def mass_of(w, tier):
    return oracle.attention_mass(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, tier, w.q,
                                 w.q_dtype)


@pytest.mark.parametrize("G,q_dtype", [(1, "fp16"), (4, "bf16"), (2, "fp16")])
def test_all_t0_mass_is_textbook_softmax(G, q_dtype):
    lens = [45, 19]
    w = wl.custom(11, 2, 2, G, 16, lens, wl.MODE_QUOTA, quota=[[T, 0, 0] for T in lens],
                  q_dtype=q_dtype)
    tier = tiers_of(w)
    mass = mass_of(w, tier)
    K = w.K.to(torch.float64).numpy()
    q = q_f64(w)
    for b, T in enumerate(lens):
        for h in range(w.Hkv):
            want = np.zeros(w.Tmax)
            for g in range(G):
                l = K[b, h, :T] @ q[b, h * G + g] / math.sqrt(w.d)
                e = np.exp(l - l.max())
                want[:T] += e / e.sum()
            np.testing.assert_allclose(mass[b, h], want, rtol=1e-12, atol=1e-15)


def test_mixed_tier_mass_uses_reconstructed_keys():
    lens = [70, 41]
    w = wl.custom(12, 2, 2, 4, 16, lens, wl.MODE_QUOTA,
                  quota=[[T // 4, T // 3, T // 4] for T in lens])
    tier = tiers_of(w)
    assert set(np.unique(tier[0, :, :70])) == {0, 1, 2, 3}
    mass = mass_of(w, tier)
    K = w.K.numpy()
    q = q_f64(w)
    for b, T in enumerate(lens):
        for h in range(w.Hkv):
            keep = [t for t in range(T) if tier[b, h, t] != 3]
            kh = np.stack([K[b, h, t].astype(np.float64) if tier[b, h, t] == 0 else
                           oracle.reconstruct(K[b, h, t].view(np.uint16),
                                              6 if tier[b, h, t] == 1 else 4) for t in keep])
            want = np.zeros(w.Tmax)
            for g in range(w.Hq // w.Hkv):
                l = kh @ q[b, h * 4 + g] / math.sqrt(w.d)
                e = np.exp(l - l.max())
                want[keep] += e / e.sum()
            np.testing.assert_allclose(mass[b, h], want, rtol=1e-12, atol=1e-15)


def test_mass_invariants_in_budget_mode():
    lens = [200, 130, 0]
    w = wl.custom(13, 3, 2, 4, 16, lens, wl.MODE_BUDGET, protect_sink=4, protect_recent=8,
                  zipf_alpha=1.2, budget=[int(0.3 * T * 2 * 512) + 2 * 15 * 888 for T in lens])
    tier = tiers_of(w)
    mass = mass_of(w, tier)
    G = w.Hq // w.Hkv
    for b, T in enumerate(lens):
        for h in range(w.Hkv):
            resident = tier[b, h, :T] != 3
            if resident.any():
                assert mass[b, h].sum() == pytest.approx(G, rel=1e-13)
            else:
                assert np.all(mass[b, h] == 0)
            assert np.all(mass[b, h, :T][~resident] == 0)
            assert np.all(mass[b, h, T:] == 0)
            assert np.all(mass[b, h, :T][resident] > 0)
            assert np.all(mass[b, h] <= G)


def test_units_with_nothing_resident_have_zero_mass():
    K = torch.ones((2, 1, 4, 128), dtype=torch.float16)
    q = torch.ones((2, 3, 128), dtype=torch.float16)
    tier = np.full((2, 1, 4), 3, np.uint8)
    tier[1, 0, :2] = 0
    mass = oracle.attention_mass(2, 3, 1, 4, 128, np.array([4, 0], np.int32), K, tier, q, "fp16")
    assert np.all(mass == 0)


def test_tiny_d2_hand_derived_mass():
    """d = 2, one kv head, two query heads (G = 2), three T1 tokens.  With
    d = 2 the single pair holds the whole key (share code 1, rho^ = 1), so
    k^ = r~ (cos, sin)(2 pi c / 64):
      k=(1,0) -> (1,0);  k=(0,1) -> (cos pi/2, 1);  k=(-2,0) -> (-2, 2 sin pi).
    Query heads q0 = (1, 0.5), q1 = (-1, 2)."""
    keys = np.array([[1, 0], [0, 1], [-2, 0]], np.float16).reshape(1, 1, 3, 2)
    qs = np.array([[1.0, 0.5], [-1.0, 2.0]], np.float16).reshape(1, 2, 2)
    tier = np.ones((1, 1, 3), np.uint8)
    mass = oracle.attention_mass(1, 2, 1, 3, 2, np.array([3], np.int32), torch.tensor(keys), tier,
                                 torch.tensor(qs), "fp16")
    kh = np.array([[1.0, 0.0], [math.cos(math.pi / 2), 1.0], [-2.0, 2.0 * math.sin(math.pi)]])
    want = np.zeros(3)
    for qv in ([1.0, 0.5], [-1.0, 2.0]):
        l = kh @ np.array(qv) / math.sqrt(2)
        e = np.exp(l - l.max())
        want += e / e.sum()
    np.testing.assert_allclose(mass[0, 0], want, rtol=1e-14, atol=1e-16)
    # by hand: q0 logits (1, 0.5, -2)/sqrt2, q1 logits (-1, 2, 2)/sqrt2
    s = math.sqrt(2)
    z0 = math.exp(1 / s) + math.exp(0.5 / s) + math.exp(-2 / s)
    z1 = math.exp(-1 / s) + 2 * math.exp(2 / s)
    assert mass[0, 0, 0] == pytest.approx(math.exp(1 / s) / z0 + math.exp(-1 / s) / z1, rel=1e-6)
    assert mass[0, 0, 2] == pytest.approx(math.exp(-2 / s) / z0 + math.exp(2 / s) / z1, rel=1e-6)


def test_decode_output_is_mass_weighted_values():
    """G = 1: the decode's output is sum_t mass_t v^_t with v^ the fp16 V
    (T0) or the int8 code times its fp16 scale (T1/T2)."""
    lens = [60]
    w = wl.custom(14, 1, 2, 1, 16, lens, wl.MODE_QUOTA, quota=[[12, 20, 16]])
    tier = tiers_of(w)
    mass = mass_of(w, tier)
    out, _ = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, tier, w.q,
                           w.q_dtype)
    V = w.V.numpy()
    for h in range(w.Hkv):
        acc = np.zeros(w.d)
        for t in range(lens[0]):
            tr = tier[0, h, t]
            if tr == 3:
                continue
            if tr == 0:
                vh = V[0, h, t].astype(np.float64)
            else:
                codes, sc = oracle.vquant(V[0, h, t].view(np.uint16))
                vh = codes.astype(np.float64) * oracle.h2d(sc)
            acc += mass[0, h, t] * vh
        np.testing.assert_allclose(out[0, h], acc, rtol=1e-12, atol=1e-14)


def test_utility_accumulation_rule():
    u = np.array([[[1.0, 2.0, 3.0, 4.0]]])
    m = np.array([[[0.5, 0.25, 0.0, 0.7]]])
    got = oracle.accumulate_utility(u, m, np.array([3], np.int32), 0.5)
    np.testing.assert_array_equal(got, [[[1.0, 1.25, 1.5, 4.0]]])
