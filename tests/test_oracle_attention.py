"""Pins of the oracle's dequantization and attention: torch's
scaled_dot_product_attention (fp64, CPU) as a library reference, closed-form
special cases, an identity "codebook" that must reproduce exact attention on
the raw keys/values, and the folded score form s1 (s2 q~.u_hat + q~.o)."""
import numpy as np
import pytest
import torch

from oracle import nsn_oracle as orc


def test_attention_matches_torch_sdpa():
    rng = np.random.default_rng(8)
    q = rng.standard_normal((4, 128))
    k = rng.standard_normal((300, 128)) * 2
    v = rng.standard_normal((300, 128))
    scale = 1 / np.sqrt(128)
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None], torch.tensor(k)[None], torch.tensor(v)[None], scale=scale)[0].numpy()
    assert np.abs(orc.attention(q, k, v, scale) - ref).max() < 1e-13


def test_attention_special_cases():
    rng = np.random.default_rng(9)
    k = rng.standard_normal((10, 16))
    v = rng.standard_normal((10, 16))
    assert np.allclose(orc.attention(rng.standard_normal((1, 16)), k[:1], v[:1], 0.3), v[:1], atol=1e-15)
    assert np.allclose(orc.attention(np.zeros((1, 16)), k, v, 0.3), v.mean(0, keepdims=True), atol=1e-15)
    k2 = k.copy()
    k2[4] = 50.0 * np.ones(16)
    out = orc.attention(np.ones((1, 16)), k2, v, 1.0)
    assert np.allclose(out, v[4:5], atol=1e-12)


def test_identity_codebook_reproduces_exact_attention():
    # Use the exact u sub-vectors of every token as the "codebook" and the
    # unrounded s1, s2, o: dequantize must return the raw tokens, and decode
    # attention must equal plain attention on raw K/V.
    rng = np.random.default_rng(10)
    d, n = 128, 64
    xk = rng.standard_normal((n, d)) * 1.5 + 2.0
    xv = rng.standard_normal((n, d))

    def identity_cache(x):
        u, s1, o, s2 = orc.nsn(orc.rotate(x))
        cb = u.reshape(-1, 8)
        codes = np.arange(n * 16).reshape(n, 16)
        return {"codes": codes, "signs": None, "s1": s1, "s2": s2, "o": o[None, :]}, cb

    kq, cbk = identity_cache(xk)
    vq, cbv = identity_cache(xv)
    khat = orc.dequantize(kq["codes"], None, kq["s1"], kq["s2"], kq["o"], cbk, orc.MODE_1BIT)
    assert np.abs(khat - xk).max() < 1e-12
    q = rng.standard_normal((4, d))
    out = orc.decode_attention(q, kq, vq, np.zeros((0, d)), np.zeros((0, d)), cbk, cbv,
                               orc.MODE_1BIT, orc.MODE_1BIT, 1 / np.sqrt(d))
    assert np.abs(out - orc.attention(q, xk, xv, 1 / np.sqrt(d))).max() < 1e-10


def test_folded_score_form():
    rng = np.random.default_rng(11)
    d, n = 128, 32
    uh = rng.standard_normal((n, d))
    s1 = rng.uniform(0.5, 3, n)
    s2 = rng.uniform(0.5, 1.5, n)
    o = rng.standard_normal(d) * 0.3
    q = rng.standard_normal((3, d))
    xhat = ((uh * s2[:, None] + o) * s1[:, None]) @ orc.hadamard_matrix(d)
    assert np.allclose(orc.nsn_score_terms(q, uh, s1, s2, o), q @ xhat.T, atol=1e-11)


def test_window_only_attention():
    rng = np.random.default_rng(12)
    d = 128
    kw = orc.to_f16(rng.standard_normal((7, d)))
    vw = orc.to_f16(rng.standard_normal((7, d)))
    empty = {"codes": np.zeros((0, 16), np.int64), "signs": None, "s1": np.zeros(0),
             "s2": np.zeros(0), "o": np.zeros((0, d))}
    q = rng.standard_normal((2, d))
    cb = np.zeros((256, 8))
    out = orc.decode_attention(q, empty, empty, kw, vw, cb, cb, 1, 1, 0.1)
    assert np.allclose(out, orc.attention(q, kw, vw, 0.1), atol=1e-15)


def test_prefill_split():
    assert orc.prefill_split(4096, 128, 128) == 3968
    assert orc.prefill_split(128, 128, 128) == 0
    assert orc.prefill_split(129, 128, 128) == 128
    assert orc.prefill_split(256, 128, 0) == 256
    assert orc.prefill_split(200, 128, 0) == 200
    assert orc.prefill_split(0, 128, 128) == 0


def test_quantize_sequence_layout():
    rng = np.random.default_rng(13)
    x = rng.standard_normal((300, 128))
    a = np.abs(rng.standard_normal((256, 8)))
    qs = orc.quantize_sequence(x, a, orc.MODE_2BIT, block=128, window=128)
    assert qs["n_quant"] == 256
    assert qs["codes"].shape == (256, 16) and qs["signs"].shape == (256, 16)
    assert qs["o"].shape == (2, 128) and qs["window"].shape == (44, 128)
    b1 = orc.quantize_block(x[128:256], a, orc.MODE_2BIT)
    assert np.array_equal(qs["codes"][128:], b1["codes"])
    assert np.array_equal(qs["o"][1], b1["o"])
