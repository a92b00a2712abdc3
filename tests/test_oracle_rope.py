"""Pins of the oracle's rotary position embedding (pre-RoPE keys).

Source: "NSNQuant: A Double Normalization Approach for Calibration-Free Low-Bit
Vector Quantization of KV Cache", technical summary, Metodologia 4 -- NSN is
applied to the keys before RoPE, so attention rotates each dequantized key at its
position.  Every check here comes from the mathematics of the rotation, not from
the oracle's own formula: the complex-number form, relative-position invariance,
an exact quarter turn, orthogonality, and the reduction to plain attention.
"""
import numpy as np
import pytest

from oracle import nsn_oracle as O
from oracle import codebook_oracle as CB

D = 128


def _rope_complex(x, positions, theta):
    """The same rotation as a complex product: (x_i + i x_{i+d/2}) e^{i pos theta_i}."""
    half = x.shape[1] // 2
    z = x[:, :half] + 1j * x[:, half:]
    z = z * np.exp(1j * np.asarray(positions, np.float64)[:, None] * theta[None, :])
    return np.concatenate([z.real, z.imag], axis=1)


def test_inv_freq_closed_form():
    th = O.rope_inv_freq(D, 500000.0)
    assert th.shape == (64,)
    assert th[0] == 1.0
    assert th[63] == pytest.approx(500000.0 ** (-126.0 / 128.0), rel=1e-14)
    ratio = th[1:] / th[:-1]
    np.testing.assert_allclose(ratio, 500000.0 ** (-2.0 / 128.0), rtol=1e-13)


def test_matches_complex_form():
    rng = np.random.default_rng(7)
    x = rng.standard_normal((9, D))
    pos = rng.integers(0, 131072, size=9)
    th = O.rope_inv_freq(D, 500000.0)
    np.testing.assert_allclose(O.apply_rope(x, pos, th), _rope_complex(x, pos, th), rtol=1e-12, atol=1e-12)


def test_quarter_turn_and_identity():
    x = np.arange(1.0, D + 1.0)[None, :]
    th = np.zeros(64)
    th[0] = np.pi / 2
    y = O.apply_rope(x, [1], th)[0]
    assert y[0] == pytest.approx(-x[0, 64], abs=1e-12)   # x_0 -> -x_64
    assert y[64] == pytest.approx(x[0, 0], abs=1e-12)    # x_64 -> x_0
    keep = np.ones(D, bool)
    keep[[0, 64]] = False
    np.testing.assert_array_equal(y[keep], x[0, keep])  # zero frequencies: unchanged
    np.testing.assert_array_equal(O.apply_rope(x, [0], O.rope_inv_freq(D, 1e4)), x)  # position 0


def test_orthogonal_and_relative_position():
    rng = np.random.default_rng(3)
    th = O.rope_inv_freq(D, 500000.0)
    q = rng.standard_normal((1, D))
    k = rng.standard_normal((1, D))
    np.testing.assert_allclose(np.linalg.norm(O.apply_rope(k, [777], th)), np.linalg.norm(k), rtol=1e-13)
    for m, n, c in [(5, 2, 9), (40000, 31, 1234), (0, 130000, 17)]:
        a = O.apply_rope(q, [m], th) @ O.apply_rope(k, [n], th).T
        b = O.apply_rope(q, [m + c], th) @ O.apply_rope(k, [n + c], th).T
        np.testing.assert_allclose(a, b, rtol=1e-9, atol=1e-9)
        # only the offset matters: q . R_{n-m} k
        np.testing.assert_allclose(a, q @ O.apply_rope(k, [n - m], th).T, rtol=1e-9, atol=1e-9)


def _tiny_cache(rng, n_quant, n_win, mode):
    cb = CB.build_codebook(seed=1, n_samples=4096, n_codes=256, dim=8, abs_mode=(mode == 2), iters=3)
    x = rng.standard_normal((n_quant + n_win, D))
    x[:, 5] += 6.0
    q = O.quantize_sequence(x[:n_quant], cb, mode, window=0)
    kq = {k: q[k] for k in ("codes", "signs", "s1", "s2", "o")}
    return cb, kq, x[n_quant:].astype(np.float16).astype(np.float64)


@pytest.mark.parametrize("mode", [1, 2])
def test_decode_rope_reduces_and_rotates(mode):
    rng = np.random.default_rng(11 + mode)
    cb, kq, kw = _tiny_cache(rng, 256, 5, mode)
    _, vq, vw = _tiny_cache(rng, 256, 5, mode)
    qg = rng.standard_normal((4, D))
    scale = 1.0 / np.sqrt(D)
    plain = O.decode_attention(qg, kq, vq, kw, vw, cb, cb, mode, mode, scale)
    zero = O.decode_attention_rope(qg, kq, vq, kw, vw, cb, cb, mode, mode, scale, np.zeros(64))
    np.testing.assert_allclose(zero, plain, rtol=1e-13, atol=1e-13)
    # explicit: rotate the dequantized keys by the complex form, then attend
    th = O.rope_inv_freq(D, 500000.0)
    keys = np.concatenate([O.dequantize(kq["codes"], kq["signs"], kq["s1"], kq["s2"], kq["o"], cb, mode), kw])
    vals = np.concatenate([O.dequantize(vq["codes"], vq["signs"], vq["s1"], vq["s2"], vq["o"], cb, mode), vw])
    rk = _rope_complex(keys, np.arange(keys.shape[0]), th)
    s = qg @ rk.T * scale
    p = np.exp(s - s.max(axis=1, keepdims=True))
    ref = (p / p.sum(axis=1, keepdims=True)) @ vals
    got = O.decode_attention_rope(qg, kq, vq, kw, vw, cb, cb, mode, mode, scale, th)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-11)
    assert not np.allclose(got, plain, atol=1e-3)  # the rotation changes the result
