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


def test_identity_codebook_over_several_blocks():
    # Three quantization blocks (128, 128 and a partial 44 tokens), each NSN'd on
    # its own, so every block has its own channel mean o_b.  With the exact u
    # sub-vectors as the "codebook" and unrounded scalars, dequantize must give
    # back every raw token, which only holds if token t reads the mean of its own
    # block t // 128 ([TS] Metodologia 1: the byproducts s1, o, s2 reconstruct
    # the tensor).  A per-block offset makes the blocks' means differ.
    rng = np.random.default_rng(21)
    d, n, blk = 128, 300, 128
    xk = rng.standard_normal((n, d)) * 1.5
    xv = rng.standard_normal((n, d))
    for a in range(0, n, blk):
        xk[a:a + blk] += rng.standard_normal(d) * 4.0
        xv[a:a + blk] += rng.standard_normal(d) * 2.0

    def identity_cache(x):
        s1s, s2s, os_, us = [], [], [], []
        for a in range(0, n, blk):
            u, s1, o, s2 = orc.nsn(orc.rotate(x[a:a + blk]))
            us.append(u)
            s1s.append(s1)
            s2s.append(s2)
            os_.append(o)
        cb = np.concatenate(us).reshape(-1, 8)
        codes = np.arange(n * 16).reshape(n, 16)
        return {"codes": codes, "signs": None, "s1": np.concatenate(s1s), "s2": np.concatenate(s2s),
                "o": np.stack(os_)}, cb

    kq, cbk = identity_cache(xk)
    vq, cbv = identity_cache(xv)
    assert kq["o"].shape == (3, d) and np.abs(kq["o"][0] - kq["o"][2]).max() > 0.1
    for cache, cb, x in ((kq, cbk, xk), (vq, cbv, xv)):
        xhat = orc.dequantize(cache["codes"], None, cache["s1"], cache["s2"], cache["o"], cb, orc.MODE_1BIT)
        assert np.abs(xhat - x).max() < 1e-11
    q = rng.standard_normal((4, d))
    out = orc.decode_attention(q, kq, vq, np.zeros((0, d)), np.zeros((0, d)), cbk, cbv,
                               orc.MODE_1BIT, orc.MODE_1BIT, 1 / np.sqrt(d))
    assert np.abs(out - orc.attention(q, xk, xv, 1 / np.sqrt(d))).max() < 1e-10


@pytest.mark.parametrize("mode", [orc.MODE_1BIT, orc.MODE_2BIT])
def test_stored_s2_preserves_the_component_along_u(mode):
    # [TS] Metodologia 3 (scale adjustment): the quantized vector is rescaled so
    # that its component along the original vector is the original one.  In the
    # original domain, with v_t = x_t - s1_t H o (the token without its block
    # mean part, = s1 s2 H u), the reconstruction x_hat from the stored scalars
    # must have no error along v_t: (x_hat_t - x_t) . v_t = 0 up to the fp16
    # rounding of the stored s1, s2' and o.  Without the factor alpha the error
    # along v_t is the full (u . u_hat - |u|^2) s2 s1^2, several percent of
    # |v_t|^2 at these bit widths.
    from scipy.linalg import hadamard

    rng = np.random.default_rng(22)
    d, n = 128, 128
    x = rng.standard_normal((n, d))
    ch = rng.choice(d, 5, replace=False)
    x[:, ch] = 3.0 * (x[:, ch] + rng.standard_normal(5) * 4.0)
    if mode == orc.MODE_2BIT:
        cb = np.abs(rng.standard_normal((256, 8)))
    else:
        cb = rng.standard_normal((256, 8))
    qb = orc.quantize_block(x, cb, mode)
    xhat = orc.dequantize(qb["codes"], qb["signs"], qb["s1"], qb["s2"], qb["o"][None, :], cb, mode)
    h = hadamard(d) / np.sqrt(d)
    v = x - qb["s1"][:, None] * (qb["o"] @ h)[None, :]
    along = np.einsum("td,td->t", xhat - x, v) / np.einsum("td,td->t", v, v)
    assert np.abs(along).max() < 3e-3
    # the same reconstruction with alpha left out errs along v_t by far more
    raw = orc.quantize_block(x, cb, mode, scale_adjust=False)
    xraw = orc.dequantize(raw["codes"], raw["signs"], raw["s1"], raw["s2"], raw["o"][None, :], cb, mode)
    along_raw = np.einsum("td,td->t", xraw - x, v) / np.einsum("td,td->t", v, v)
    assert np.median(np.abs(along_raw)) > 10 * np.abs(along).max()


def test_extend_attention_is_causal_attention_over_the_cache():
    # chunked prefill: C queries, the chunk's tokens at the end of the window.  The
    # same result as plain softmax attention over [dequantized keys, window keys]
    # with a causal mask on the window part; the last query is the decode of the
    # full cache; changing window tokens after query i leaves query i unchanged.
    rng = np.random.default_rng(23)
    d, g, C, nw = 128, 3, 5, 9
    cb = np.abs(rng.standard_normal((256, 8)))
    x = rng.standard_normal((256, d))
    kq = orc.quantize_sequence(x, cb, orc.MODE_2BIT, 128, 0)
    vq = orc.quantize_sequence(x[::-1].copy(), cb, orc.MODE_2BIT, 128, 0)
    kw, vw = rng.standard_normal((nw, d)), rng.standard_normal((nw, d))
    q = rng.standard_normal((C, g, d))
    got = orc.extend_attention(q, kq, vq, kw, vw, cb, cb, 2, 2, 0.1)
    khat = orc.dequantize(kq["codes"], kq["signs"], kq["s1"], kq["s2"], kq["o"], cb, 2)
    vhat = orc.dequantize(vq["codes"], vq["signs"], vq["s1"], vq["s2"], vq["o"], cb, 2)
    keys, vals = np.concatenate([khat, kw]), np.concatenate([vhat, vw])
    for i in range(C):
        s = q[i] @ keys.T * 0.1
        s[:, 256 + nw - C + 1 + i:] = -np.inf    # window slots after query i
        p = np.exp(s - s.max(axis=1, keepdims=True))
        p /= p.sum(axis=1, keepdims=True)
        assert np.abs(got[i] - p @ vals).max() < 1e-12
    full = orc.decode_attention(q[-1], kq, vq, kw, vw, cb, cb, 2, 2, 0.1)
    assert np.abs(got[-1] - full).max() < 1e-15
    kw2 = kw.copy()
    kw2[nw - C + 2:] += 5.0                      # tokens after query 0
    again = orc.extend_attention(q, kq, vq, kw2, vw, cb, cb, 2, 2, 0.1)
    assert np.array_equal(again[0], got[0]) and not np.allclose(again[-1], got[-1])
