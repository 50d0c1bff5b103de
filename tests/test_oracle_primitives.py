"""Pins of the oracle's encode primitives against mathematics that the oracle
does not itself use: exact rational arithmetic, numpy/Python library
conversions, closed forms and brute force.

The pages (SPHERICAL KV, Technical Summary section 2.1) only say that a key
is stored as a quantised radius plus packed angle codes; the concrete scheme
(fp16 radius, per-pair b-bit angle code, 2-bit share code, int8 V) is the
pinned reading these tests hold the oracle to."""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle

pytestmark = []


def rng(seed=0):
    return np.random.default_rng(seed)


def f16_bits(x):
    return np.asarray(x, np.float16).view(np.uint16)


# ---------------------------------------------------------------- fp16 ----

def test_d2h_matches_numpy_double_to_half():
    r = rng(1)
    xs = np.concatenate([
        r.standard_normal(20000) * 10.0 ** r.integers(-9, 5, 20000),
        [0.0, 65504.0, 65519.99, 2 ** -24, 2 ** -25, 3 * 2 ** -26, 2 ** -14, 1 + 2 ** -11,
         1 + 3 * 2 ** -11, 2048 + 1, 2048 + 3, 6.1e-5],
    ])
    for x in xs:
        want = int(np.float16(np.float64(x)).view(np.uint16))
        assert oracle.d2h(float(x)) == want, x


def test_h2d_exact_for_every_finite_half():
    bits = np.arange(0, 1 << 16, dtype=np.uint16)
    vals = bits.view(np.float16).astype(np.float64)
    for b in range(0, 1 << 16, 97):
        if not np.isfinite(vals[b]):
            continue
        assert oracle.h2d(int(b)) == vals[b]


# ---------------------------------------------------------------- norm ----

def exact_r2(k16):
    """sum over c of (k_c * 2^24)^2 from the numpy decode of the halves."""
    s = 0
    for x in np.asarray(k16, np.uint16).view(np.float16).astype(np.float64):
        m = Fraction(float(x)) * (1 << 24)
        assert m.denominator == 1
        s += int(m) ** 2
    return s


@pytest.mark.parametrize("seed", range(5))
def test_norm2_exact(seed):
    r = rng(seed)
    k = (r.standard_normal(128) * 10.0 ** r.integers(-6, 4, 128)).astype(np.float16)
    k = np.where(np.isfinite(k), k, np.float16(0))
    assert oracle.norm2(k.view(np.uint16)) == exact_r2(k.view(np.uint16))


def test_norm2_extremes_and_one_hot():
    k = np.zeros(128, np.float16)
    assert oracle.norm2(k.view(np.uint16)) == 0
    k[:] = np.float16(65504)
    assert oracle.norm2(k.view(np.uint16)) == 128 * (65504 * 2 ** 24) ** 2
    k[:] = np.float16(-65504)
    assert oracle.norm2(k.view(np.uint16)) == 128 * (65504 * 2 ** 24) ** 2
    k[:] = np.float16(2 ** -24)          # smallest subnormal: m = 1
    assert oracle.norm2(k.view(np.uint16)) == 128
    for c, x in [(0, 3.0), (77, -0.5), (127, 1e-6)]:
        k = np.zeros(128, np.float16)
        k[c] = x
        m = Fraction(float(np.float16(x))) * (1 << 24)
        assert oracle.norm2(k.view(np.uint16)) == int(m) ** 2


def rtilde_ref(R2):
    """fp16(min(sqrt(double(R2)) * 2^-24, 65504)) via Python's correctly
    rounded int->float, math.sqrt and numpy's double->half."""
    r = math.sqrt(float(R2)) * 2.0 ** -24
    return int(np.float16(min(r, 65504.0)).view(np.uint16))


def test_rtilde_matches_library_route_and_exact_value():
    r = rng(7)
    for i in range(3000):
        k = (r.standard_normal(128) * 10.0 ** r.integers(-7, 3)).astype(np.float16)
        R2 = exact_r2(k.view(np.uint16))
        got = oracle.rtilde(k.view(np.uint16))
        assert got == rtilde_ref(R2)
        # against the exact radius: within half an fp16 ulp (plus the double rounding)
        exact = math.isqrt(R2 << 80) / 2.0 ** 40 * 2.0 ** -24   # sqrt(R2) * 2^-24, to 2^-40 abs in sqrt(R2)
        v = float(np.uint16(got).view(np.float16))
        if exact >= 2 ** -14:
            ulp = 2.0 ** (math.floor(math.log2(exact)) - 10)
        else:
            ulp = 2.0 ** -24
        assert abs(v - exact) <= 0.5 * ulp * (1 + 1e-9)


def test_rtilde_closed_forms():
    k = np.zeros(128, np.float16)
    k[5] = np.float16(3.0)
    assert oracle.rtilde(k.view(np.uint16)) == f16_bits(3.0)
    k = np.full(128, np.float16(1.0))        # |k| = sqrt(128)
    assert oracle.rtilde(k.view(np.uint16)) == f16_bits(math.sqrt(128.0))
    k = np.full(128, np.float16(65504))      # saturates
    assert oracle.rtilde(k.view(np.uint16)) == f16_bits(65504.0)
    assert oracle.rtilde(np.zeros(128, np.uint16)) == 0


# --------------------------------------------------------------- angles ----

def atan2_code(x, y, b):
    n = 1 << b
    a = math.atan2(y, x)
    if a < 0:
        a += 2 * math.pi
    return int(math.floor(a / (2 * math.pi / n) + 0.5)) % n


def dist_to_boundary(x, y, b):
    n = 1 << b
    a = math.atan2(y, x) % (2 * math.pi)
    delta = 2 * math.pi / n
    f = a / delta - 0.5
    return abs(f - round(f)) * delta


@pytest.mark.parametrize("b", [2, 3, 4, 6, 8, 12, 16])
def test_angle_code_matches_atan2_rounding(b):
    r = rng(b)
    xs = f16_bits(r.standard_normal(4000) * 10.0 ** r.integers(-4, 3, 4000))
    ys = f16_bits(r.standard_normal(4000) * 10.0 ** r.integers(-4, 3, 4000))
    near = 0
    for xh, yh in zip(xs, ys):
        x = float(np.uint16(xh).view(np.float16))
        y = float(np.uint16(yh).view(np.float16))
        if x == 0 and y == 0:
            continue
        got = oracle.angle_code(int(xh), int(yh), b)
        want = atan2_code(x, y, b)
        if got != want:
            # only allowed within a hair of a sector boundary
            assert dist_to_boundary(x, y, b) < 1e-6 * (2 * math.pi / (1 << b)), (x, y, got, want)
            near += 1
    assert near <= 2


@pytest.mark.parametrize("b", [2, 4, 6, 8, 16])
def test_angle_code_axes_and_origin(b):
    n = 1 << b
    one, m1, z = f16_bits(1.0), f16_bits(-1.0), f16_bits(0.0)
    assert oracle.angle_code(int(one), int(z), b) == 0
    assert oracle.angle_code(int(z), int(one), b) == n // 4
    assert oracle.angle_code(int(m1), int(z), b) == n // 2
    assert oracle.angle_code(int(z), int(m1), b) == 3 * n // 4
    assert oracle.angle_code(int(z), int(z), b) == 0
    neg0 = f16_bits(-0.0)
    assert oracle.angle_code(int(neg0), int(neg0), b) == 0
    assert oracle.angle_code(int(one), int(neg0), b) == 0


def test_angle_code_b2_diagonal_ties_go_counter_clockwise():
    for xs, ys, want in [(1, 1, 1), (-1, 1, 2), (-1, -1, 3), (1, -1, 0)]:
        x, y = f16_bits(float(xs)), f16_bits(float(ys))
        assert oracle.angle_code(int(x), int(y), 2) == want


def test_angle_code_sector_is_exact_against_fp32_boundaries():
    """Every point's code c satisfies: it lies on-or-CCW of boundary c-1 and
    strictly clockwise of boundary c, with the cross products evaluated in
    exact rationals from the fp32 boundary table."""
    b = 6
    n = 1 << b
    bx, by = oracle.boundaries(b)
    r = rng(11)
    xs = f16_bits(r.standard_normal(1500))
    ys = f16_bits(r.standard_normal(1500))
    for xh, yh in zip(xs, ys):
        x = Fraction(float(np.uint16(xh).view(np.float16)))
        y = Fraction(float(np.uint16(yh).view(np.float16)))
        c = oracle.angle_code(int(xh), int(yh), b)
        lo, hi = (c - 1) % n, c
        side_lo = Fraction(float(bx[lo])) * y - Fraction(float(by[lo])) * x
        side_hi = Fraction(float(bx[hi])) * y - Fraction(float(by[hi])) * x
        assert side_lo >= 0 and side_hi < 0


def test_boundary_table_is_cos_sin_of_half_offsets():
    for b in (4, 6):
        bx, by = oracle.boundaries(b)
        n = 1 << b
        j = np.arange(n)
        beta = (j + 0.5) * 2 * np.pi / n
        assert np.array_equal(bx, np.cos(beta).astype(np.float32))
        assert np.array_equal(by, np.sin(beta).astype(np.float32))


# ----------------------------------------------------------------- rho ----

def rho_code_exact(xh, yh, R2, d):
    x = Fraction(float(np.uint16(xh).view(np.float16)))
    y = Fraction(float(np.uint16(yh).view(np.float16)))
    rho2 = x * x + y * y
    r2 = Fraction(R2, 1 << 48)
    code = 0
    for t in (Fraction(3, 4), Fraction(5, 4), Fraction(7, 4)):
        # (rho / r) * sqrt(d/2) > t
        if rho2 * Fraction(d, 2) > t * t * r2:
            code += 1
    return code


def test_rho_code_d2_share_one_is_level_one():
    r = rng(3)
    for _ in range(500):
        k = f16_bits(r.standard_normal(2) * 10.0 ** r.integers(-3, 3))
        R2 = exact_r2(k)
        if R2 == 0:
            continue
        assert oracle.rho_code(int(k[0]), int(k[1]), R2, 2) == 1
        assert oracle.rho_level(1, 2) == 1.0


def test_rho_code_matches_exact_rationals_near_thresholds():
    r = rng(5)
    d = 128
    checked = 0
    for _ in range(400):
        k = f16_bits(r.standard_normal(d))
        R2 = exact_r2(k)
        rr = math.sqrt(R2) * 2.0 ** -24
        for t in (0.75, 1.25, 1.75):
            # put pair 0 right at the threshold share and step it by ulps
            target = t * rr / math.sqrt(d / 2)
            base = np.float16(target)
            for step in range(-2, 3):
                xh = int(base.view(np.uint16)) + step
                if xh < 0:
                    continue
                kk = k.copy()
                kk[0] = xh
                kk[1] = 0
                R2k = exact_r2(kk)
                got = oracle.rho_code(int(kk[0]), int(kk[1]), R2k, d)
                assert got == rho_code_exact(kk[0], kk[1], R2k, d)
                checked += 1
    assert checked > 1000


def test_rho_code_brute_force_random():
    r = rng(9)
    for d in (2, 4, 16, 128):
        for _ in range(300):
            k = f16_bits(r.standard_normal(d) * 10.0 ** r.integers(-3, 3))
            R2 = exact_r2(k)
            i = int(r.integers(0, d // 2))
            got = oracle.rho_code(int(k[2 * i]), int(k[2 * i + 1]), R2, d)
            assert got == rho_code_exact(k[2 * i], k[2 * i + 1], R2, d)


def test_rho_levels():
    assert [oracle.rho_level(c, 128) for c in range(4)] == [1 / 16, 1 / 8, 3 / 16, 1 / 4]
    assert [oracle.rho_level(c, 2) for c in range(4)] == [0.5, 1.0, 1.5, 2.0]


# ------------------------------------------------------------------- V ----

@pytest.mark.parametrize("seed", range(4))
def test_vquant_roundtrip_within_half_step(seed):
    r = rng(seed)
    for _ in range(200):
        v = (r.standard_normal(128) * 10.0 ** r.integers(-5, 3)).astype(np.float16)
        codes, sh = oracle.vquant(v.view(np.uint16))
        s = float(np.uint16(sh).view(np.float16))
        vf = v.astype(np.float64)
        assert np.all(np.abs(codes.astype(np.int32)) <= 127)
        amax = np.max(np.abs(vf))
        # scale = fp16 of absmax / 127
        assert sh == int(np.float16(np.float32(amax) / np.float32(127)).view(np.uint16)) or \
            abs(s - amax / 127) <= 2 ** -24
        if s == 0:
            assert np.all(codes == 0)
            continue
        recon = s * codes.astype(np.float64)
        unclamped = np.abs(vf / s) < 126.5
        assert np.all(np.abs(recon - vf)[unclamped] <= s / 2 * (1 + 2e-7))
        if amax / 127 >= 2 ** -14:         # scale is a normal half: absmax maps to +-127
            j = int(np.argmax(np.abs(vf)))
            assert abs(int(codes[j])) == 127


def test_vquant_special_vectors():
    codes, sh = oracle.vquant(np.zeros(128, np.uint16))
    assert sh == 0 and np.all(codes == 0)
    v = np.full(128, np.float16(2.5))
    codes, sh = oracle.vquant(v.view(np.uint16))
    assert np.all(codes == 127)
    v = np.full(128, np.float16(-0.75))
    codes, sh = oracle.vquant(v.view(np.uint16))
    assert np.all(codes == -127)
    assert sh == int(np.float16(np.float32(0.75) / np.float32(127)).view(np.uint16))


# ------------------------------------------------------------ distortion ----

def test_distortion_constants_closed_form():
    c = oracle.distortion()
    assert c[0] == 0.0 and c[3] == 1.0
    for tier, b in ((1, 6), (2, 4)):
        x = math.pi / 2 ** b
        assert c[tier] == pytest.approx(2 * (1 - math.sin(x) / x), rel=1e-15)
        # small-angle form delta^2 / 12
        assert c[tier] == pytest.approx((2 * math.pi / 2 ** b) ** 2 / 12, rel=2e-2)
    k = oracle.kappa(128)
    assert k[0] > k[1] > k[2] > 0
    assert oracle.tier_bytes(0) == 512 and oracle.tier_bytes(1) == 196 and oracle.tier_bytes(2) == 180


@pytest.mark.parametrize("tier,b", [(1, 6), (2, 4)])
def test_distortion_matches_monte_carlo_of_the_angle_quantiser(tier, b):
    """c(b) is the mean squared logit error of the oracle's own angle coder,
    relative to the mean squared logit, for random directions (shares exact)."""
    r = rng(100 + b)
    n = 40000
    ang_k = r.uniform(0, 2 * np.pi, n)
    ang_q = r.uniform(0, 2 * np.pi, n)
    err2 = 0.0
    ref2 = 0.0
    xs = f16_bits(np.cos(ang_k) * 4)
    ys = f16_bits(np.sin(ang_k) * 4)
    delta = 2 * np.pi / 2 ** b
    for i in range(n):
        c = oracle.angle_code(int(xs[i]), int(ys[i]), b)
        x = float(np.uint16(xs[i]).view(np.float16))
        y = float(np.uint16(ys[i]).view(np.float16))
        a = math.atan2(y, x)
        lq = math.cos(ang_q[i] - a)
        lhat = math.cos(ang_q[i] - c * delta)
        err2 += (lhat - lq) ** 2
        ref2 += lq ** 2
    est = err2 / ref2
    assert est == pytest.approx(oracle.distortion()[tier], rel=0.04)
