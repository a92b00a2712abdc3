"""Pins of the oracle's Normalize-Shift-Normalize: a hand-derived worked
example (tests/golden/nsn_worked_example_d4.json), the invariants the method
states (token norm sqrt(d), zero channel mean after the shift, exact
reconstruction from s1, o, s2), commutation with the Hadamard rotation, the
degenerate cases, and the near-N(0,1) output distribution on inputs with
outlier channels."""
import json
import os

import numpy as np
import pytest

from oracle import nsn_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "nsn_worked_example_d4.json")


def outlier_tokens(rng, n, d=128, n_out=5):
    x = rng.standard_normal((n, d))
    ch = rng.choice(d, n_out, replace=False)
    x[:, ch] = 3.0 * (x[:, ch] + rng.normal(0.0, 4.0, size=n_out))
    return x


def test_worked_example():
    with open(GOLDEN) as f:
        g = json.load(f)
    for case in g["cases"]:
        x = np.array(case["x"], dtype=np.float64)
        y = orc.rotate(x)
        assert np.allclose(y, case["y"], atol=1e-15, rtol=0)
        u, s1, o, s2 = orc.nsn(y)
        assert np.allclose(s1, case["s1"], atol=1e-15, rtol=0)
        assert np.allclose(o, case["o"], atol=1e-15, rtol=0)
        assert np.allclose(s2, case["s2"], atol=1e-15, rtol=0)
        assert np.allclose(u, case["u"], atol=1e-15, rtol=0)


def test_invariants():
    rng = np.random.default_rng(1)
    x = outlier_tokens(rng, 128)
    y = orc.rotate(x)
    u, s1, o, s2 = orc.nsn(y)
    d = 128
    assert np.allclose(np.linalg.norm(u, axis=1), np.sqrt(d), rtol=1e-13)
    z = u * s2[:, None]
    assert np.abs(z.sum(axis=0)).max() < 1e-12           # zero channel mean after shift
    n1 = y / s1[:, None]
    assert np.allclose(np.linalg.norm(n1, axis=1), np.sqrt(d), rtol=1e-13)
    assert np.allclose(n1.mean(axis=0), o, atol=1e-14)
    rec = (u * s2[:, None] + o[None, :]) * s1[:, None]
    assert np.abs(rec - y).max() < 1e-12                 # reconstruction


def test_commutes_with_rotation():
    # Token norms and the channel mean commute with a per-token orthogonal map:
    # NSN(H x) has the same s1, s2 as NSN(x), and o, u rotate with H.
    rng = np.random.default_rng(2)
    x = outlier_tokens(rng, 96)
    ux, s1x, ox, s2x = orc.nsn(x)
    uy, s1y, oy, s2y = orc.nsn(orc.rotate(x))
    assert np.allclose(s1x, s1y, rtol=1e-13)
    assert np.allclose(s2x, s2y, rtol=1e-12)
    assert np.allclose(orc.rotate(ox[None, :])[0], oy, atol=1e-13)
    assert np.allclose(orc.rotate(ux), uy, atol=1e-12)


def test_degenerate_cases():
    rng = np.random.default_rng(3)
    x = rng.standard_normal((8, 128))
    x[3] = 0.0                                            # zero token: s1 = 0
    u, s1, o, s2 = orc.nsn(orc.rotate(x))
    assert s1[3] == 0.0
    rec = (u * s2[:, None] + o) * s1[:, None]
    assert np.abs(rec - orc.rotate(x)).max() < 1e-12
    same = np.tile(rng.standard_normal(128), (5, 1))     # identical tokens: s2 = 0
    u, s1, o, s2 = orc.nsn(orc.rotate(same))
    assert np.all(s2 < 1e-7) or np.all(s2 == 0)
    one = rng.standard_normal((1, 128))                   # one-token block
    u, s1, o, s2 = orc.nsn(orc.rotate(one))
    assert s2[0] == 0.0 and np.all(u == 0)
    with pytest.raises(ValueError):
        orc.nsn(np.zeros((0, 128)))


def test_output_close_to_standard_normal():
    # Claim of the method: Hadamard + NSN turn outlier-laden KV into roughly
    # N(0,1) channels.  Sanity check, not a parity pin.
    rng = np.random.default_rng(4)
    blocks = []
    for _ in range(32):
        x = outlier_tokens(rng, 128)
        blocks.append(orc.nsn(orc.rotate(x))[0])
    u = np.concatenate(blocks)
    assert np.abs(u.mean(axis=0)).max() < 0.05
    assert np.abs(u.var(axis=0) - 1).max() < 0.15
    kurt = ((u - u.mean(0)) ** 4).mean(0) / u.var(0) ** 2
    assert np.abs(np.median(kurt) - 3.0) < 0.3


# ---- double quantization of the stored scalars ----------------------------------

def test_dq4_hand_cases():
    r = orc.dq4(np.arange(16.0))
    assert (r["lo"], r["hi"]) == (0.0, 15.0)
    assert np.array_equal(r["levels"], np.arange(16)) and np.array_equal(r["values"], np.arange(16.0))
    # round half to even on the level grid: 0.5 -> 0, 1.5 -> 2, 2.5 -> 2
    r = orc.dq4(np.array([0.0, 0.5, 1.5, 2.5, 15.0]))
    assert list(r["levels"]) == [0, 0, 2, 2, 15]
    # a constant group has one level and reproduces its (fp16) value
    r = orc.dq4(np.full(7, 0.3))
    assert np.all(r["levels"] == 0) and np.all(r["values"] == np.float16(0.3))


def test_dq4_error_bound_and_range():
    rng = np.random.default_rng(4)
    for _ in range(20):
        x = rng.normal(size=128) * rng.uniform(0.01, 5)
        r = orc.dq4(x)
        step = (r["hi"] - r["lo"]) / 15
        assert r["levels"].min() >= 0 and r["levels"].max() <= 15
        # half a level plus the fp16 rounding of the end points
        slack = max(abs(r["lo"] - x.min()), abs(r["hi"] - x.max()))
        assert np.max(np.abs(r["values"] - x)) <= step / 2 + slack + 1e-15
        # every value is exactly on the grid
        assert np.allclose((r["values"] - r["lo"]) / step, r["levels"], atol=1e-9)


def test_double_quant_changes_only_the_stored_scalars():
    x = np.random.default_rng(5).normal(size=(128, 128))
    cb = np.random.default_rng(6).normal(size=(256, 8))
    a = orc.quantize_block(x, cb, 1)
    b = orc.quantize_block(x, cb, 1, double_quant=True)
    assert np.array_equal(a["codes"], b["codes"]) and np.array_equal(a["s2"], b["s2"])
    assert np.allclose(b["s1"], orc.dq4(b["s1_dq"]["values"])["values"])
    assert np.max(np.abs(b["o"] - a["o"])) <= (b["o_dq"]["hi"] - b["o_dq"]["lo"]) / 30 + 1e-3
