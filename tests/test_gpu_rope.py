"""GPU parity of the pre-RoPE key decode (nsn_decode_attention_rope) against the
CPU oracle's decode_attention_rope.

"NSNQuant ..." technical summary, Metodologia 4: NSN is applied to the keys before
the rotary position embedding, so the cache holds pre-RoPE keys and each key is
rotated at its position when attended.  Checked: random compressed caches (every
mode pair and GQA group size, several splits, window only, empty), large
positions with fast frequencies (the fp64 angle reduction), prefill -> appends
across a flush end to end, double quantization, and the zero-frequency reduction
to the plain decode."""
import math

import numpy as np
import pytest
import torch

from calibration_free_vector_b200 import nsn, synthetic
from oracle import nsn_oracle as orc
import nsn_testlib as tl
from nsn_testlib import fill_cache, oracle_seq, oracle_pipeline

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)


def inv_freq(base: float) -> np.ndarray:
    """theta_i = base^(-2i/128) as the fp32 table both sides receive."""
    return (float(base) ** (-2.0 * np.arange(64) / 128.0)).astype(np.float32)


def run_rope(kc, vc, q, cbk, cbv, theta):
    out = torch.empty((q.shape[0], q.shape[1], 128), dtype=torch.float32, device="cuda")
    ws = nsn.decode_rope_workspace(kc, q.shape[1])
    nsn.nsn_decode_attention_rope(kc, vc, q.cuda(), SCALE, torch.from_numpy(theta).cuda(),
                                  torch.from_numpy(cbk).cuda(), torch.from_numpy(cbv).cuda(), out, ws)
    torch.cuda.synchronize()
    return out.cpu().numpy()


@pytest.mark.parametrize("g", [1, 2, 4, 8])
@pytest.mark.parametrize("mk,mv", [(1, 1), (1, 2), (2, 1), (2, 2)])
def test_rope_random_cache(mk, mv, g):
    B, H, cap = 3, 2, 2304
    shape = {(0, 0): (2304, 128), (0, 1): (128, 5), (1, 0): (896, 0), (1, 1): (0, 77),
             (2, 0): (1152, 1), (2, 1): (0, 0)}
    kc, vc = nsn.Cache(B, H, cap, 128, mk), nsn.Cache(B, H, cap, 128, mv)
    kcont, vcont = {}, {}
    for (b, h), (nq, nw) in shape.items():
        seed = 2000 * b + 10 * h + 100 * mk + mv
        kcont[(b, h)] = synthetic.random_cache_contents(seed, nq, nw, mk)
        vcont[(b, h)] = synthetic.random_cache_contents(seed + 5, nq, nw, mv)
    fill_cache(kc, kcont)
    fill_cache(vc, vcont)
    cbk, cbv = tl.codebook(mk), tl.codebook(mv)
    theta = inv_freq(500000.0)
    q = synthetic.queries(17, B, H * g, torch.bfloat16, "cpu")
    out = run_rope(kc, vc, q, cbk, cbv, theta)
    qf = q.float().numpy().astype(np.float64)
    for (b, h), (nq, nw) in shape.items():
        got = out[b, h * g:(h + 1) * g]
        if nq + nw == 0:
            assert np.all(got == 0.0)
            continue
        ref = orc.decode_attention_rope(qf[b, h * g:(h + 1) * g], oracle_seq(kcont[(b, h)]),
                                        oracle_seq(vcont[(b, h)]), kcont[(b, h)]["window"].astype(np.float64),
                                        vcont[(b, h)]["window"].astype(np.float64), cbk.astype(np.float64),
                                        cbv.astype(np.float64), mk, mv, SCALE, theta.astype(np.float64))
        err = tl.attn_error(got, ref)
        assert err <= tl.ATTN_TOL, f"(b={b}, h={h}) nq={nq} nw={nw}: error {err:.3g}"


def test_rope_long_positions_fast_frequencies():
    # positions up to 33k with theta_0 = 1 rad/token: angles of 3e4 rad need the fp64 reduction
    B, H, g, cap = 1, 2, 4, 32768
    shape = {(0, 0): (32768, 100), (0, 1): (16384, 128)}
    kc, vc = nsn.Cache(B, H, cap, 128, 2), nsn.Cache(B, H, cap, 128, 2)
    kcont = {k: synthetic.random_cache_contents(31 + k[1], nq, nw, 2) for k, (nq, nw) in shape.items()}
    vcont = {k: synthetic.random_cache_contents(41 + k[1], nq, nw, 2) for k, (nq, nw) in shape.items()}
    fill_cache(kc, kcont)
    fill_cache(vc, vcont)
    cb = tl.codebook(2)
    theta = inv_freq(100.0)
    q = synthetic.queries(19, B, H * g, torch.bfloat16, "cpu")
    # sharpen the scores so that the late (large-angle) keys carry weight
    q = (q.float() * 4.0).to(torch.bfloat16)
    out = run_rope(kc, vc, q, cb, cb, theta)
    qf = q.float().numpy().astype(np.float64)
    for (b, h) in shape:
        ref = orc.decode_attention_rope(qf[b, h * g:(h + 1) * g], oracle_seq(kcont[(b, h)]),
                                        oracle_seq(vcont[(b, h)]), kcont[(b, h)]["window"].astype(np.float64),
                                        vcont[(b, h)]["window"].astype(np.float64), cb.astype(np.float64),
                                        cb.astype(np.float64), 2, 2, SCALE, theta.astype(np.float64))
        err = tl.attn_error(out[b, h * g:(h + 1) * g], ref)
        assert err <= tl.ATTN_TOL, f"h={h}: error {err:.3g}"


@pytest.mark.parametrize("mk,mv,g", [(2, 2, 4), (1, 1, 8), (2, 1, 1)])
def test_rope_end_to_end(mk, mv, g):
    # Llama-shaped keys with channel outliers, prefill of 1000 tokens, 140 appends across a flush
    B, H, T, steps = 2, 2, 1000, 140
    rk, rv = synthetic.KVRecipe(61 + mk, H, "llama"), synthetic.KVRecipe(71 + mv, H, "llama")
    xk = rk.tokens(B, T + steps, torch.bfloat16, "cpu")
    xv = rv.tokens(B, T + steps, torch.bfloat16, "cpu")
    cbk, cbv = tl.codebook(mk), tl.codebook(mv)
    dk, dv = torch.from_numpy(cbk).cuda(), torch.from_numpy(cbv).cuda()
    kc, vc = nsn.Cache(B, H, 1152, 128, mk), nsn.Cache(B, H, 1152, 128, mv)
    nsn.nsn_quantize_kv(kc, xk[:, :T].cuda(), dk)
    nsn.nsn_quantize_kv(vc, xv[:, :T].cuda(), dv)
    for s in range(T, T + steps):
        nsn.nsn_append_residual(kc, vc, xk[:, s].cuda(), xv[:, s].cuda(), dk, dv)
    theta = inv_freq(500000.0)
    q = synthetic.queries(67, B, H * g, torch.bfloat16, "cpu")
    out = run_rope(kc, vc, q, cbk, cbv, theta)
    qf = q.float().numpy().astype(np.float64)
    xkf, xvf = xk.float().numpy().astype(np.float64), xv.float().numpy().astype(np.float64)
    th = theta.astype(np.float64)
    for b in range(B):
        for h in range(H):
            # over what the GPU stored ...
            gk, gv = tl.read_cache(kc, b, h), tl.read_cache(vc, b, h)
            ref = orc.decode_attention_rope(qf[b, h * g:(h + 1) * g], gk, gv, gk["window"], gv["window"],
                                            cbk.astype(np.float64), cbv.astype(np.float64), mk, mv, SCALE, th)
            assert tl.attn_error(out[b, h * g:(h + 1) * g], ref) <= tl.ATTN_TOL, (b, h)
            # ... and over the oracle's own quantization of the same tokens
            (kq, kw), (vq, vw) = oracle_pipeline(xkf[b, :, h], xvf[b, :, h], T, T + steps,
                                                 cbk.astype(np.float64), cbv.astype(np.float64), mk, mv, 128)
            ref2 = orc.decode_attention_rope(qf[b, h * g:(h + 1) * g], kq, vq, kw, vw, cbk.astype(np.float64),
                                             cbv.astype(np.float64), mk, mv, SCALE, th)
            assert tl.attn_error(out[b, h * g:(h + 1) * g], ref2) <= tl.ATTN_TOL, (b, h)


def test_rope_double_quant_random_levels():
    B, H, g, cap = 2, 2, 4, 640
    rng = np.random.default_rng(19)
    caches = []
    for mode in (2, 1):
        c = nsn.Cache(B, H, cap, 128, mode, double_quant=True)
        c.codes.copy_(torch.from_numpy(rng.integers(0, 256, c.codes.shape, dtype=np.uint8)))
        if mode == 2:
            c.signs.copy_(torch.from_numpy(rng.integers(0, 256, c.signs.shape, dtype=np.uint8)))
        c.norms.copy_(torch.from_numpy(rng.uniform(0.5, 1.5, c.norms.shape).astype(np.float16)))
        c.s1_levels.copy_(torch.from_numpy(rng.integers(0, 256, c.s1_levels.shape, dtype=np.uint8)))
        c.means.copy_(torch.from_numpy(rng.integers(0, 256, c.means.shape, dtype=np.uint8)))
        par = np.zeros(c.dq_params.shape, dtype=np.float16)
        lo1 = rng.uniform(0.5, 1.0, par.shape[:-1])
        par[..., 0], par[..., 1] = lo1, lo1 + rng.uniform(0.1, 2.0, lo1.shape)
        lo2 = rng.uniform(-0.6, -0.1, par.shape[:-1])
        par[..., 2], par[..., 3] = lo2, lo2 + rng.uniform(0.2, 1.2, lo2.shape)
        c.dq_params.copy_(torch.from_numpy(par))
        c.window_buf.copy_(torch.from_numpy(rng.normal(size=c.window_buf.shape).astype(np.float16)))
        c.n_quant.copy_(torch.tensor([[640, 256], [384, 0]], dtype=torch.int32))
        c.n_window.copy_(torch.tensor([[128, 3], [0, 40]], dtype=torch.int32))
        caches.append(c)
    kc, vc = caches
    cbk, cbv = tl.codebook(2), tl.codebook(1)
    theta = inv_freq(10000.0)
    q = synthetic.queries(93, B, H * g, torch.bfloat16, "cpu")
    out = run_rope(kc, vc, q, cbk, cbv, theta)
    qf = q.float().numpy().astype(np.float64)
    for b in range(B):
        for h in range(H):
            gk, gv = tl.read_cache(kc, b, h), tl.read_cache(vc, b, h)
            ref = orc.decode_attention_rope(qf[b, h * g:(h + 1) * g], gk, gv, gk["window"], gv["window"],
                                            cbk.astype(np.float64), cbv.astype(np.float64), 2, 1, SCALE,
                                            theta.astype(np.float64))
            assert tl.attn_error(out[b, h * g:(h + 1) * g], ref) <= tl.ATTN_TOL, (b, h)


def test_rope_zero_frequencies_equal_plain_decode():
    # theta = 0: no rotation, the same attention as nsn_decode_attention (both within tolerance of the oracle)
    B, H, g, cap = 2, 2, 4, 1024
    kc, vc = nsn.Cache(B, H, cap, 128, 2), nsn.Cache(B, H, cap, 128, 2)
    shape = {(0, 0): (1024, 60), (0, 1): (512, 128), (1, 0): (256, 0), (1, 1): (0, 9)}
    fill_cache(kc, {k: synthetic.random_cache_contents(51 + 3 * k[0] + k[1], *v, 2) for k, v in shape.items()})
    fill_cache(vc, {k: synthetic.random_cache_contents(57 + 3 * k[0] + k[1], *v, 2) for k, v in shape.items()})
    cb = tl.codebook(2)
    q = synthetic.queries(29, B, H * g, torch.bfloat16, "cpu")
    got = run_rope(kc, vc, q, cb, cb, np.zeros(64, np.float32))
    plain = torch.empty((B, H * g, 128), dtype=torch.float32, device="cuda")
    dcb = torch.from_numpy(cb).cuda()
    nsn.nsn_decode_attention(kc, vc, q.cuda(), SCALE, dcb, dcb, plain, nsn.decode_workspace(kc, H * g))
    torch.cuda.synchronize()
    assert tl.attn_error(got, plain.cpu().numpy()) <= tl.ATTN_TOL
