"""The oracle against the hand-worked examples in tests/golden/.  The pages
print no worked example, so each fixture is derived by hand from the
passage it cites.  Each expected number is also recomputed here from the
closed form the fixture states, so that a typo in a fixture fails as
well."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_tier_bytes():
    g = load("tier_bytes.json")
    d = g["d"]
    assert g["bytes"]["T0"] == 2 * d + 2 * d
    assert g["bytes"]["T1"] == 2 + (d // 2) * (6 + 2) // 8 + d + 2
    assert g["bytes"]["T2"] == 2 + (d // 2) * (4 + 2) // 8 + d + 2
    for t, name in enumerate(("T0", "T1", "T2")):
        assert oracle.tier_bytes(t, d) == g["bytes"][name]


def test_codes():
    g = load("codes_d2.json")
    for c in g["cases"]:
        k = np.array(c["key"], np.float16)
        p = c.get("pair", 0)
        x, y = k[2 * p], k[2 * p + 1]
        # closed form: nearest sector of the angle, share thresholds on u
        ang = math.atan2(float(y), float(x)) % (2 * math.pi)
        n = 1 << c["b"]
        want_angle = int(math.floor(ang / (2 * math.pi / n) + 0.5)) % n if (x or y) else 0
        r = float(np.linalg.norm(k.astype(np.float64)))
        u = math.hypot(float(x), float(y)) / r * math.sqrt(len(k) / 2)
        want_share = sum(u > t for t in (0.75, 1.25, 1.75))
        assert (want_angle, want_share) == (c["angle_code"], c["share_code"]), c["why"]
        xh, yh = int(k[2 * p].view(np.uint16)), int(k[2 * p + 1].view(np.uint16))
        assert oracle.angle_code(xh, yh, c["b"]) == c["angle_code"], c["why"]
        R2 = oracle.norm2(k.view(np.uint16))
        assert oracle.rho_code(xh, yh, R2, len(k)) == c["share_code"], c["why"]


def test_attention_d2_t1():
    g = load("attention_d2_t1.json")
    keys, vals, q = np.array(g["keys"]), np.array(g["values"]), np.array(g["q"])
    # closed form: the rebuilt keys of the fixture's note
    kh = np.array([[1.0, 0.0], [math.cos(math.pi / 2), 1.0], [-2.0, 2.0 * math.sin(math.pi)]])
    l = kh @ q / math.sqrt(2)
    np.testing.assert_allclose(l, g["logits"], rtol=1e-15)
    w = np.exp(l - l.max())
    np.testing.assert_allclose((w[:, None] * vals).sum(0) / w.sum(), g["out"], rtol=1e-14)
    T = len(keys)
    K = torch.tensor(keys.astype(np.float16).reshape(1, 1, T, 2))
    V = torch.tensor(vals.astype(np.float16).reshape(1, 1, T, 2))
    qq = torch.tensor(q.astype(np.float16).reshape(1, 1, 2))
    tier = np.ones((1, 1, T), np.uint8)
    out, lse = oracle.decode(1, 1, 1, T, 2, np.array([T], np.int32), K, V, tier, qq, "fp16")
    np.testing.assert_allclose(out[0, 0], g["out"], rtol=0, atol=g["out_tolerance"])
    assert lse[0, 0] == pytest.approx(l.max() + math.log(w.sum()), rel=1e-14)
