"""Pins of the oracle's T1 variant (5-bit angle + 3-bit share on the uniform
8-level grid, one code byte (angle << 3) | share per pair): the share code
against exact rational arithmetic and exact ties, the reconstruction against
the tier study's logit, the packed bytes read back field by field, and the
attention over such a store against a numpy softmax of the rebuilt keys."""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from oracle import tier_study as ts
from long_context_decode_ada_b200 import workloads as wl


def exact_code3(x, y, k):
    v = [Fraction(float(t)) for t in k.astype(np.float16)]
    r2 = sum(t * t for t in v)
    u2 = (Fraction(float(np.float16(x))) ** 2 + Fraction(float(np.float16(y))) ** 2) * 64 / r2
    return sum(1 for j in range(7) if u2 > Fraction(2 * j + 3, 8) ** 2)


def test_share_code3_against_fractions():
    rng = np.random.default_rng(11)
    for i in range(300):
        k = (rng.standard_normal(128) * (3.0 if i % 3 == 0 else 1.0)).astype(np.float16)
        if i % 2:
            k[int(rng.integers(128))] *= 6
        R2 = oracle.norm2(k.view(np.uint16))
        for p in rng.integers(0, 64, 4):
            p = int(p)
            got = oracle.rho_code3(int(k[2 * p].view(np.uint16)), int(k[2 * p + 1].view(np.uint16)),
                                   R2, 128)
            assert got == exact_code3(k[2 * p], k[2 * p + 1], k), (i, p)


def test_share_code3_ties_go_to_the_lower_code():
    # pair 0 = (3, 0), the rest sums to 4087: r^2 = 4096, u = 8 * 3 / 64 = 3/8 exactly
    k = np.zeros(128, np.float16)
    k[0] = 3.0
    k[2:6] = [63.0, 10.0, 4.0, 1.0]
    k[6] = 1.0
    R2 = oracle.norm2(k.view(np.uint16))
    x, y = int(k[0].view(np.uint16)), int(k[1].view(np.uint16))
    assert oracle.rho_code3(x, y, R2, 128) == 0
    k2 = k.copy()
    k2[1] = 0.0625
    R2b = oracle.norm2(k2.view(np.uint16))
    assert oracle.rho_code3(x, int(k2[1].view(np.uint16)), R2b, 128) == 1
    for c in range(8):
        assert oracle.rho_level3(c, 128) == pytest.approx(0.25 * (c + 1) / 8, rel=1e-15)


def test_reconstruction_matches_the_study_logit():
    rng = np.random.default_rng(12)
    grid = ts.uniform_grid(8)
    with oracle.t1_scheme(1):
        for _ in range(200):
            k = rng.standard_normal(128).astype(np.float16)
            q = rng.standard_normal(128)
            kh = oracle.reconstruct_tier(k.view(np.uint16), 1)
            want = oracle.logit_grid(q, k.view(np.uint16), 5, *grid)
            assert float(q @ kh) / math.sqrt(128) == pytest.approx(want, rel=1e-12, abs=1e-12)
    # scheme 0 is the pinned reconstruction
    k = rng.standard_normal(128).astype(np.float16)
    np.testing.assert_array_equal(oracle.reconstruct_tier(k.view(np.uint16), 1),
                                  oracle.reconstruct(k.view(np.uint16), 6))


def test_packed_t1_bytes_read_back():
    w = wl.custom(71, 1, 2, 1, 16, [90], wl.MODE_QUOTA, quota=[[10, 60, 20]])
    tier = oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, None,
                           w.mode, w.budget, w.quota)
    with oracle.t1_scheme(1):
        ref = oracle.pack(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.V, tier,
                          w.free_lists, w.pool_slots)
    P = w.P
    K = w.K.numpy()
    checked = 0
    for h in range(w.Hkv):
        for t in range(90):
            if tier[0, h, t] != 1:
                continue
            loc = int(ref["row_of"][0, h, t])
            pid = int(ref["page_ids"][int(ref["page_indptr"][h]) + loc // P])
            assert pid >> 30 == 1
            slot, row = pid & ((1 << 30) - 1), loc % P
            base = slot * oracle.page_stride(1, P)
            codes = ref["pools"][1][base + 16 + 2 * P + 64 * row: base + 16 + 2 * P + 64 * row + 64]
            k = K[0, h, t]
            R2 = oracle.norm2(k.view(np.uint16))
            for byte in range(64):
                g, j = byte // 16, byte % 16
                p = 16 * (j >> 2) + 4 * g + (j & 3)
                x, y = int(k[2 * p].view(np.uint16)), int(k[2 * p + 1].view(np.uint16))
                want = (oracle.angle_code(x, y, 5) << 3) | oracle.rho_code3(x, y, R2, 128)
                assert codes[byte] == want, (h, t, byte)
            checked += 1
    assert checked == 120


def test_attention_over_the_variant_store_is_softmax_of_rebuilt_keys():
    lens = [80, 41]
    w = wl.custom(72, 2, 2, 4, 16, lens, wl.MODE_QUOTA,
                  quota=[[T // 4, T // 2, T // 8] for T in lens])
    tier = oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, None,
                           w.mode, w.budget, w.quota)
    with oracle.t1_scheme(1):
        out, lse = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, tier, w.q,
                                 w.q_dtype)
        K = w.K.numpy()
        V = w.V.numpy()
        q = w.q.view(torch.int16).view(torch.bfloat16).to(torch.float64).numpy()
        for b, T in enumerate(lens):
            for h in range(w.Hkv):
                keep = [t for t in range(T) if tier[b, h, t] != 3]
                kh, vh = [], []
                for t in keep:
                    tr = int(tier[b, h, t])
                    if tr == 0:
                        kh.append(K[b, h, t].astype(np.float64))
                        vh.append(V[b, h, t].astype(np.float64))
                    else:
                        kh.append(oracle.reconstruct_tier(K[b, h, t].view(np.uint16), tr))
                        c, sc = oracle.vquant(V[b, h, t].view(np.uint16))
                        vh.append(c.astype(np.float64) * oracle.h2d(sc))
                kh, vh = np.stack(kh), np.stack(vh)
                for g in range(4):
                    l = kh @ q[b, 4 * h + g] / math.sqrt(128)
                    e = np.exp(l - l.max())
                    np.testing.assert_allclose(out[b, 4 * h + g], (e @ vh) / e.sum(), rtol=1e-11,
                                               atol=1e-13)
                    assert lse[b, 4 * h + g] == pytest.approx(l.max() + math.log(e.sum()),
                                                              rel=1e-12)
