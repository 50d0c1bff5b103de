"""Pins of the oracle's logits and attention.

(1) with every token dense (T0) the oracle is textbook softmax attention on
    the fp16 K/V, recomputed here independently in numpy;
(2) the compressed-domain logit (r~/sqrt d) sum_i rho^_i LUT_i[c_i]
    (SPHERICAL KV, Technical Summary section 2.1, compressed-domain
    similarity) equals q . k^ / sqrt(d) of the reconstructed key;
(3) as the angle bits b grow, the logit converges to q . k / sqrt(d) within
    the Cauchy-Schwarz bound of the angle and radius quantisation;
(4) tiny cases whose codes and softmax are derived by hand."""
import math

import numpy as np
import pytest
import torch

import oracle
from long_context_decode_ada_b200 import workloads as wl


def rng(seed=0):
    return np.random.default_rng(seed)


def f16(x):
    return np.asarray(x, np.float16)


def textbook(q, K, V, d):
    """softmax(q K^T / sqrt d) V in float64, with log-sum-exp."""
    l = K @ q / math.sqrt(d)
    m = l.max()
    w = np.exp(l - m)
    return (w[:, None] * V).sum(0) / w.sum(), m + math.log(w.sum())


@pytest.mark.parametrize("G,q_dtype", [(1, "fp16"), (4, "bf16")])
def test_all_t0_is_textbook_attention(G, q_dtype):
    B, Hkv, P = 2, 2, 16
    lens = [37, 50]
    w = wl.custom(3, B, Hkv, G, P, lens, wl.MODE_QUOTA, quota=[[l, 0, 0] for l in lens],
                  q_dtype=q_dtype)
    tier = oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, None,
                           w.mode, w.budget, w.quota)
    assert np.all(tier[0, :, :37] == 0) and np.all(tier[0, :, 37:] == 3)
    out, lse = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, tier, w.q,
                             w.q_dtype)
    Kf = w.K.to(torch.float64).numpy()
    Vf = w.V.to(torch.float64).numpy()
    if q_dtype == "bf16":
        qf = w.q.view(torch.int16).view(torch.bfloat16).to(torch.float64).numpy()
    else:
        qf = w.q.to(torch.float64).numpy()
    for b in range(B):
        for hq in range(w.Hq):
            h = hq // G
            T = lens[b]
            o, s = textbook(qf[b, hq], Kf[b, h, :T], Vf[b, h, :T], w.d)
            np.testing.assert_allclose(out[b, hq], o, rtol=1e-12, atol=1e-13)
            assert lse[b, hq] == pytest.approx(s, rel=1e-12, abs=1e-12)


@pytest.mark.parametrize("b", [4, 6])
def test_code_domain_logit_equals_reconstructed_dot(b):
    r = rng(b)
    for i in range(300):
        k = (r.standard_normal(128) * 10.0 ** r.integers(-2, 2)).astype(np.float16)
        q = r.standard_normal(128) * 10.0 ** r.integers(-1, 2)
        a = oracle.logit_codes(q, k.view(np.uint16), b)
        c = oracle.logit_recon(q, k.view(np.uint16), b)
        assert a == pytest.approx(c, rel=1e-12, abs=1e-12 * np.linalg.norm(q) *
                                  np.linalg.norm(k.astype(np.float64)))
        assert oracle.logit_variant(q, k.view(np.uint16), b, 1) == pytest.approx(a, rel=1e-13,
                                                                                abs=1e-13)


def cs_bound(q, k, b):
    r = float(np.linalg.norm(k.astype(np.float64)))
    d = k.size
    return (np.linalg.norm(q) * r / math.sqrt(d)) * (
        2 * math.sin(math.pi / 2 ** (b + 1)) * (1 + 2 ** -11) + 2 ** -11)


def test_exact_share_logit_converges_to_true_logit():
    r = rng(21)
    bits = [4, 6, 8, 10, 12, 16]
    worst = {b: 0.0 for b in bits}
    for i in range(150):
        k = r.standard_normal(128).astype(np.float16)
        q = r.standard_normal(128)
        true = float(q @ k.astype(np.float64)) / math.sqrt(128)
        for b in bits:
            got = oracle.logit_variant(q, k.view(np.uint16), b, 0)
            err = abs(got - true)
            assert err <= cs_bound(q, k, b)
            worst[b] = max(worst[b], err / (np.linalg.norm(q) * np.linalg.norm(
                k.astype(np.float64)) / math.sqrt(128)))
    for a, b in zip(bits, bits[1:]):
        if b <= 10:
            assert worst[b] < worst[a] / 2
    assert worst[16] < 1e-3


def test_two_bit_share_logit_converges_to_quantised_share_limit():
    r = rng(22)
    for i in range(100):
        k = r.standard_normal(128).astype(np.float16)
        q = r.standard_normal(128)
        limit = oracle.logit_variant(q, k.view(np.uint16), 0, 2)
        prev = None
        for b in [4, 6, 8, 12, 16]:
            got = oracle.logit_variant(q, k.view(np.uint16), b, 1)
            err = abs(got - limit)
            assert err <= cs_bound(q, k, b)
            prev = err
        assert prev <= 1e-3 * np.linalg.norm(q) * np.linalg.norm(k.astype(np.float64))


def test_uniform_share_on_axis_key_reconstructs_exactly():
    # every pair (a, 0): shares are all 1/8, u = 1 -> level 1, angle code 0
    for a in (1.0, 0.5, 3.0, 2.0 ** -10):
        k = np.zeros(128, np.float16)
        k[0::2] = a
        for b in (4, 6):
            kh = oracle.reconstruct(k.view(np.uint16), b)
            np.testing.assert_array_equal(kh, k.astype(np.float64))
    # pairs (0, a): angle code 2^(b-2), i.e. a quarter turn
    k = np.zeros(128, np.float16)
    k[1::2] = 2.0
    for b in (4, 6):
        kh = oracle.reconstruct(k.view(np.uint16), b)
        np.testing.assert_allclose(kh[1::2], 2.0, rtol=0, atol=1e-15)
        np.testing.assert_allclose(kh[0::2], 0.0, rtol=0, atol=1e-15)


def test_one_hot_key_uses_top_and_bottom_share_levels():
    k = np.zeros(128, np.float16)
    k[10] = 4.0     # pair 5 holds all the energy: share 1 -> u = 8 -> level 2 (1/4)
    kh = oracle.reconstruct(k.view(np.uint16), 6)
    assert kh[10] == pytest.approx(4.0 * 0.25, abs=1e-15)
    # every empty pair decodes to the lowest level 1/16 at angle 0
    others = [i for i in range(64) if i != 5]
    for i in others:
        assert kh[2 * i] == pytest.approx(4.0 / 16, abs=1e-15)
        assert kh[2 * i + 1] == pytest.approx(0.0, abs=1e-15)


def _tiny_case(d, keys, vals, q, tiers):
    T = len(keys)
    K = torch.tensor(np.asarray(keys, np.float16).reshape(1, 1, T, d))
    V = torch.tensor(np.asarray(vals, np.float16).reshape(1, 1, T, d))
    qq = torch.tensor(np.asarray(q, np.float16).reshape(1, 1, d))
    tier = np.asarray(tiers, np.uint8).reshape(1, 1, T)
    return oracle.decode(1, 1, 1, T, d, np.array([T], np.int32), K, V, tier, qq, "fp16")


def test_tiny_d2_hand_checked_softmax():
    """d = 2, three T1 tokens.  With d = 2 the single pair holds the whole key,
    so its share code is 1 and rho^ = 1: k^ = r~ (cos, sin)(2 pi c / 64).
      k=(1,0): r~=1, c=0   -> k^=(1,0)
      k=(0,1): r~=1, c=16  -> k^=(cos pi/2, sin pi/2)
      k=(-2,0): r~=2, c=32 -> k^=(-2, 2 sin pi)
    V = multiples of 2^-7 with absmax 127 * 2^-7, so the int8 step is exactly
    2^-7 and v^ = v."""
    keys = [[1, 0], [0, 1], [-2, 0]]
    a = 127 / 128
    vals = [[a, -0.5], [0.25, a], [-a, 0.0]]
    q = [1.0, 0.5]
    out, lse = _tiny_case(2, keys, vals, q, [1, 1, 1])
    l = np.array([1.0, math.cos(math.pi / 2) + 0.5, -2.0 + 0.5 * 2 * math.sin(math.pi)])
    l /= math.sqrt(2)
    w = np.exp(l - l.max())
    want = (w[:, None] * np.array(vals, np.float64)).sum(0) / w.sum()
    np.testing.assert_allclose(out[0, 0], want, rtol=1e-14, atol=1e-15)
    assert lse[0, 0] == pytest.approx(l.max() + math.log(w.sum()), rel=1e-14)


def test_tiny_d4_mixed_tiers_and_drop():
    """d = 4 (two pairs, u = share * sqrt 2).  Token 0 is T0 (exact), token 1
    is T2 with pairs (1,1),(0,0): share of pair 0 is 1 -> u = 1.41, above the
    thresholds 0.75 and 1.25 -> level 1.5 (rho^ = 1.5/sqrt2); its angle code
    (b=4) is 2; pair 1 is empty -> level 0.5 (rho^ = 0.5/sqrt2) at angle 0.
    r~ = fp16(sqrt 2).  Token 2 is dropped."""
    keys = [[0.5, -1.0, 2.0, 0.25], [1.0, 1.0, 0.0, 0.0], [3.0, 3.0, 3.0, 3.0]]
    a = 127 / 128
    vals = [[0.5, 0.25, -0.125, 1.0], [a, -0.5, 0.0, 0.5], [9.0, 9.0, 9.0, 9.0]]
    q = [1.0, -0.5, 0.25, 2.0]
    out, lse = _tiny_case(4, keys, vals, q, [0, 2, 3])
    r_t = float(np.float16(math.sqrt(2.0)))        # r~ is fp16
    k1 = np.array([r_t * (1.5 / math.sqrt(2)) * math.cos(2 * math.pi * 2 / 16),
                   r_t * (1.5 / math.sqrt(2)) * math.sin(2 * math.pi * 2 / 16),
                   r_t * (0.5 / math.sqrt(2)),
                   0.0])
    l = np.array([np.dot(q, keys[0]), np.dot(q, k1)]) / 2.0
    w = np.exp(l - l.max())
    v1 = np.array(vals[1], np.float64)   # int8 step 2^-7 (absmax 127/128): exact
    want = (w[0] * np.array(vals[0], np.float64) + w[1] * v1) / w.sum()
    np.testing.assert_allclose(out[0, 0], want, rtol=1e-14, atol=1e-15)


def test_empty_unit_gives_zero_and_minus_inf():
    K = torch.zeros((1, 1, 4, 128), dtype=torch.float16)
    V = torch.ones((1, 1, 4, 128), dtype=torch.float16)
    q = torch.ones((1, 2, 128), dtype=torch.float16)
    tier = np.full((1, 1, 4), 3, np.uint8)
    out, lse = oracle.decode(1, 2, 1, 4, 128, np.array([4], np.int32), K, V, tier, q, "fp16")
    assert np.all(out == 0) and np.all(lse == -np.inf)
    out, lse = oracle.decode(1, 2, 1, 4, 128, np.array([0], np.int32), K, V,
                             np.zeros((1, 1, 4), np.uint8), q, "fp16")
    assert np.all(out == 0) and np.all(lse == -np.inf)


def test_gqa_group_equals_separate_single_head_runs():
    w = wl.custom(5, 1, 2, 4, 16, [70], wl.MODE_QUOTA, quota=[[10, 30, 20]])
    tier = oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, None,
                           w.mode, w.budget, w.quota)
    out, lse = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, tier, w.q,
                             w.q_dtype)
    for hq in range(w.Hq):
        h = hq // 4
        o1, l1 = oracle.decode(1, 1, 1, w.Tmax, w.d, w.seq_lens, w.K[:, h:h + 1].contiguous(),
                               w.V[:, h:h + 1].contiguous(), np.ascontiguousarray(tier[:, h:h + 1]),
                               w.q[:, hq:hq + 1].contiguous(), w.q_dtype)
        np.testing.assert_array_equal(out[0, hq], o1[0, 0])
        assert lse[0, hq] == l1[0, 0]


def test_subset_units_match_full_decode():
    w = wl.custom(6, 2, 2, 2, 16, [40, 33], wl.MODE_QUOTA, quota=[[5, 10, 10], [3, 10, 10]])
    tier = oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, None,
                           w.mode, w.budget, w.quota)
    out, lse = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, tier, w.q,
                             w.q_dtype)
    units = np.array([[1, 3], [0, 0]], np.int32)
    o2, l2 = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, tier, w.q,
                           w.q_dtype, units=units)
    np.testing.assert_array_equal(o2[1, 3], out[1, 3])
    np.testing.assert_array_equal(o2[0, 0], out[0, 0])
    assert np.isnan(o2[1, 0]).all()
