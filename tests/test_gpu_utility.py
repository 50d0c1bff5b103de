"""skv_decode_utility against the oracle: the decode's out / lse as for
skv_decode_attention, and utility <- gamma utility + attention mass, the
mass of a token being its softmax weight summed over the query heads of its
kv head (oracle.attention_mass, oracle.accumulate_utility).

Tolerance of the utility: |gpu - ref| <= 1e-6 + 2e-3 |ref|.  A token's mass
is 2^(l - lse log2 e) with the kernel's fp32 logit l; an absolute logit
error e (log2 units) moves the weight by the factor 2^e, so the relative
error is about ln 2 |e| -- the 2e-3 relative bound of the attention
outputs, applied per weight (most weights of a long context are far below
the outputs' 1e-3 absolute floor, so that floor would test nothing)."""
import numpy as np
import pytest
import torch

import oracle
from long_context_decode_ada_b200 import skv
from long_context_decode_ada_b200 import workloads as wl
from _gpu import assert_close

pytestmark = pytest.mark.gpu

U_ATOL = 1e-6
U_RTOL = 2e-3


def assert_utility(got, ref, what):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert np.all(np.isfinite(got)), f"{what}: non-finite values"
    err = np.abs(got - ref)
    lim = U_ATOL + U_RTOL * np.abs(ref)
    bad = err > lim
    worst = int(np.argmax(err - lim))
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} out of tolerance; worst err "
                           f"{err.flat[worst]:.3g} at ref {ref.flat[worst]:.4g}")


def oracle_tiers(w):
    return oracle.allocate(w.B, w.Hkv, w.Tmax, w.d, w.P, w.seq_lens, w.K, w.utility, w.protect,
                           w.mode, w.budget, w.quota)


def utility_case(w, gammas, num_splits=0, seed=0):
    """Run len(gammas) utility decodes on one store and compare every step."""
    ctx = skv.Context(w.P)
    dev = skv.workload_to_device(w)
    cache = skv.build_cache(ctx, w, dev)
    cache.check()
    tier = oracle_tiers(w)
    assert np.array_equal(cache.tier.cpu().numpy(), tier), "tiers"
    u0 = np.random.default_rng(seed).random((w.B, w.Hkv, w.Tmax)).astype(np.float32)
    ut = torch.from_numpy(u0).to(cache.device)
    mass = oracle.attention_mass(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, tier, w.q,
                                 w.q_dtype)
    ro, rl = oracle.decode(w.B, w.Hq, w.Hkv, w.Tmax, w.d, w.seq_lens, w.K, w.V, tier, w.q,
                           w.q_dtype)
    want = u0.astype(np.float64)
    ws = cache.utility_workspace(w.Hq, num_splits)
    for k, gamma in enumerate(gammas):
        out, lse = cache.decode_utility(dev["q"], dev["q_dtype"], w.Hq, dev["seq_lens"], ut,
                                        gamma, workspace=ws, num_splits=num_splits)
        cache.check()
        want = oracle.accumulate_utility(want, mass, w.seq_lens, gamma)
        got = ut.cpu().numpy()
        assert_utility(got, want, f"utility after step {k}")
        assert_close(out.cpu().numpy(), ro, f"out, step {k}")
        assert_close(lse.cpu().numpy(), rl, f"lse, step {k}")
    # positions past each sequence are never touched
    for b in range(w.B):
        T = int(w.seq_lens[b])
        assert np.array_equal(got[b, :, T:], u0[b, :, T:])
    return got, mass, tier


@pytest.mark.parametrize("num_splits", [1, 0, 400])
def test_utility_quota_mixed_tiers_ragged(num_splits):
    # P = 16, several pages per tier and a ragged last page; one sequence of
    # one token, one with nothing resident beyond its T2 share
    lens = [700, 129, 1, 333]
    quota = [[100, 250, 200], [10, 40, 60], [1, 0, 0], [0, 0, 150]]
    w = wl.custom(91, 4, 2, 4, 16, lens, wl.MODE_QUOTA, quota=quota)
    utility_case(w, [0.5, 1.0], num_splits=num_splits, seed=1)


def test_utility_budget_mode_fp16_g2():
    lens = [900, 64, 517]
    w = wl.custom(92, 3, 4, 2, 32, lens, wl.MODE_BUDGET, protect_sink=8, protect_recent=32,
                  zipf_alpha=1.1, q_dtype="fp16",
                  budget=[int(0.3 * T * 4 * 512) + 4 * 31 * 888 + 40 * 4 * 512 for T in lens])
    utility_case(w, [0.875], seed=2)


def test_utility_g1_and_empty_units():
    # sequence 0 is empty, sequence 1 keeps nothing in kv head 0's quota
    # beyond one T1 token; G = 1
    lens = [0, 40, 1, 77]
    quota = [[0, 0, 0], [0, 1, 0], [0, 1, 0], [3, 30, 40]]
    w = wl.custom(93, 4, 2, 1, 16, lens, wl.MODE_QUOTA, quota=quota, q_dtype="fp16")
    got, mass, tier = utility_case(w, [1.0], seed=3)
    dropped = tier == 3
    for b, T in enumerate(lens):
        d = dropped[b, :, :T]
        # a dropped token's utility only decays (gamma = 1: unchanged)
        u0 = np.random.default_rng(3).random((w.B, w.Hkv, w.Tmax)).astype(np.float32)
        assert np.array_equal(got[b, :, :T][d], u0[b, :, :T][d])


def test_utility_long_context_128k_full_size():
    """The 128K store in the bench's launch configuration: the mass of every
    unit sums to G, and two sampled units match the oracle token by token
    (the oracle's mass of one unit needs only that unit's keys and heads)."""
    w = wl.long_context()
    ctx = skv.Context(w.P)
    dev = skv.workload_to_device(w)
    cache = skv.build_cache(ctx, w, dev)
    cache.check()
    ut = torch.zeros((w.B, w.Hkv, w.Tmax), dtype=torch.float32, device=cache.device)
    out, lse = cache.decode_utility(dev["q"], dev["q_dtype"], w.Hq, dev["seq_lens"], ut, 1.0)
    cache.check()
    got = ut.cpu().numpy()
    G = w.Hq // w.Hkv
    sums = got.astype(np.float64).sum(axis=2)
    np.testing.assert_allclose(sums, G, rtol=2e-3)
    tier = cache.tier.cpu().numpy()
    assert np.all(got[tier == 3] == 0)
    for b, h in [(0, 0), (0, w.Hkv - 1)]:
        K1 = w.K[b:b + 1, h:h + 1].contiguous()
        q1 = w.q[b:b + 1, h * G:(h + 1) * G].contiguous()
        t1 = np.ascontiguousarray(tier[b:b + 1, h:h + 1])
        m = oracle.attention_mass(1, G, 1, w.Tmax, w.d, w.seq_lens[b:b + 1], K1, t1, q1, w.q_dtype)
        assert_utility(got[b, h], m[0, 0], f"mass of unit ({b}, {h})")


def test_utility_workspace_too_small_is_refused():
    w = wl.custom(94, 1, 2, 4, 16, [100], wl.MODE_QUOTA, quota=[[20, 30, 30]])
    ctx = skv.Context(w.P)
    dev = skv.workload_to_device(w)
    cache = skv.build_cache(ctx, w, dev)
    ut = torch.zeros((w.B, w.Hkv, w.Tmax), dtype=torch.float32, device=cache.device)
    small = cache.workspace(w.Hq)  # the plain decode's size: no room for the logits
    with pytest.raises(skv.SkvError):
        cache.decode_utility(dev["q"], dev["q_dtype"], w.Hq, dev["seq_lens"], ut, 1.0,
                             workspace=small)
    assert torch.count_nonzero(ut) == 0
