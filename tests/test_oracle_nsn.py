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
