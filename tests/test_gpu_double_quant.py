"""GPU parity of double quantization (cache flag double_quant: s1 and o stored as
4-bit levels of 16 uniform steps between the fp16-rounded group min and max).

The quantizer must store the oracle's levels and (lo, hi) pairs bit for bit
(outside exact rounding ties of the level grid, which are counted), the same
codes and alpha*s2 as without double quantization, and the decode must match the
oracle's attention over the values read back from the levels."""
import math

import numpy as np
import pytest
import torch

from calibration_free_vector_b200 import nsn, synthetic
from oracle import nsn_oracle as orc
import nsn_testlib as tl

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)


def check_dq_sequence(got, ref):
    assert got["n_quant"] == ref["n_quant"]
    if not ref["n_quant"]:
        return 0
    tl.compare_codes(got, ref, ref["u"])
    mism = (got["codes"] != ref["codes"]).any(axis=1)
    rel = np.abs(got["s2"] - ref["s2"]) / np.maximum(np.abs(ref["s2"]), 1e-30)
    assert ((rel <= tl.NORM_RTOL) | mism | ((ref["s2"] == 0) & (got["s2"] == 0))).all()
    ties = 0
    for k, (q1, qo) in enumerate(zip(ref["s1_dq"], ref["o_dq"])):
        assert np.array_equal(got["params"][k], [q1["lo"], q1["hi"], qo["lo"], qo["hi"]]), k
        g1 = got["s1_levels"][k * 128: k * 128 + len(q1["levels"])]
        for g, r, xs, lo, hi in ((g1, q1["levels"], None, q1["lo"], q1["hi"]),
                                 (got["o_levels"][k], qo["levels"], None, qo["lo"], qo["hi"])):
            diff = g != r
            ties += int(diff.sum())
            # a level may differ only by one step (an exact-half rounding tie in fp64)
            assert (np.abs(g - r) <= 1).all() and diff.sum() <= 2, (k, np.argwhere(diff)[:4])
    return ties


@pytest.mark.parametrize("mode,window,dtype", [(2, 128, torch.bfloat16), (1, 0, torch.float32)])
def test_double_quant_prefill_matches_the_oracle(mode, window, dtype):
    B, H, T = 2, 2, 700
    x = synthetic.KVRecipe(71 + mode, H, "llama").tokens(B, T, dtype, "cpu")
    cb = tl.codebook(mode)
    cache = nsn.Cache(B, H, 768, window, mode, double_quant=True)
    nsn.nsn_quantize_kv(cache, x.cuda(), torch.from_numpy(cb).cuda())
    torch.cuda.synchronize()
    xf = x.float().numpy().astype(np.float64)
    ties = 0
    for b in range(B):
        for h in range(H):
            ref = orc.quantize_sequence(xf[b, :, h], cb.astype(np.float64), mode, 128, window, double_quant=True)
            ties += check_dq_sequence(tl.read_cache(cache, b, h), ref)
    assert ties <= 2


def test_double_quant_end_to_end_decode_matches_the_oracle():
    # 2-bit K / 1-bit V, prefill of 1000 tokens, 130 appends across a flush, G = 4
    B, H, g, mk, mv, T, steps = 2, 2, 4, 2, 1, 1000, 130
    rk, rv = synthetic.KVRecipe(81, H, "llama"), synthetic.KVRecipe(82, H, "llama")
    xk = rk.tokens(B, T + steps, torch.bfloat16, "cpu")
    xv = rv.tokens(B, T + steps, torch.bfloat16, "cpu")
    cbk, cbv = tl.codebook(mk), tl.codebook(mv)
    dk, dv = torch.from_numpy(cbk).cuda(), torch.from_numpy(cbv).cuda()
    kc = nsn.Cache(B, H, 1152, 128, mk, double_quant=True)
    vc = nsn.Cache(B, H, 1152, 128, mv, double_quant=True)
    nsn.nsn_quantize_kv(kc, xk[:, :T].cuda(), dk)
    nsn.nsn_quantize_kv(vc, xv[:, :T].cuda(), dv)
    for s in range(T, T + steps):
        nsn.nsn_append_residual(kc, vc, xk[:, s].cuda(), xv[:, s].cuda(), dk, dv)
    q = synthetic.queries(83, B, H * g, torch.bfloat16, "cpu")
    out = torch.empty((B, H * g, 128), dtype=torch.float32, device="cuda")
    nsn.nsn_decode_attention(kc, vc, q.cuda(), SCALE, dk, dv, out, nsn.decode_workspace(kc, H * g))
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    qf = q.float().numpy().astype(np.float64)
    for b in range(B):
        for h in range(H):
            # the decode over what the GPU stored (levels read back in fp64) ...
            gk, gv = tl.read_cache(kc, b, h), tl.read_cache(vc, b, h)
            ref = orc.decode_attention(qf[b, h * g:(h + 1) * g], gk, gv, gk["window"], gv["window"],
                                       cbk.astype(np.float64), cbv.astype(np.float64), mk, mv, SCALE)
            assert tl.attn_error(out[b, h * g:(h + 1) * g], ref) <= tl.ATTN_TOL, (b, h)
            # ... and what was stored equals the oracle's double quantization of the same tokens
            xkf = xk[b, :, h].float().numpy().astype(np.float64)
            seq = orc.quantize_sequence(xkf[:T], cbk.astype(np.float64), mk, 128, 128, double_quant=True)
            nq0 = seq["n_quant"]
            assert np.array_equal(gk["params"][: nq0 // 128],
                                  [[a["lo"], a["hi"], c["lo"], c["hi"]] for a, c in zip(seq["s1_dq"], seq["o_dq"])])


def test_double_quant_decode_random_levels():
    # random stored contents (levels, (lo, hi), alpha*s2) against the oracle over the values read back
    B, H, g, cap = 2, 2, 8, 640
    rng = np.random.default_rng(9)
    caches = []
    for mode in (2, 2):
        c = nsn.Cache(B, H, cap, 128, mode, double_quant=True)
        c.codes.copy_(torch.from_numpy(rng.integers(0, 256, c.codes.shape, dtype=np.uint8)))
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
    cb = tl.codebook(2)
    dcb = torch.from_numpy(cb).cuda()
    q = synthetic.queries(91, B, H * g, torch.bfloat16, "cpu")
    out = torch.empty((B, H * g, 128), dtype=torch.float32, device="cuda")
    nsn.nsn_decode_attention(kc, vc, q.cuda(), SCALE, dcb, dcb, out, nsn.decode_workspace(kc, H * g))
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    qf = q.float().numpy().astype(np.float64)
    for b in range(B):
        for h in range(H):
            gk, gv = tl.read_cache(kc, b, h), tl.read_cache(vc, b, h)
            ref = orc.decode_attention(qf[b, h * g:(h + 1) * g], gk, gv, gk["window"], gv["window"],
                                       cb.astype(np.float64), cb.astype(np.float64), 2, 2, SCALE)
            assert tl.attn_error(out[b, h * g:(h + 1) * g], ref) <= tl.ATTN_TOL, (b, h)
