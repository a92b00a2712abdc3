"""GPU parity with a cosine-tuned codebook ([TS] Metodologia 3: the k-means
codebook fine-tuned for the cosine distance; [GH] Codebook tuning, "--method
learned"), built by nsn_build_codebook_cosine_host, in both assignment rules the
quantizer offers: the nearest codeword and the codeword of largest cosine
similarity (nsn_cache.assign = 1).  A prefill with a full residual window, appends
whose first one flushes the window through the quantizer, and a decode; every
stored code, sign bit, norm, mean and window row, and the attention output, are
compared with the CPU oracle's pipeline under the same rule."""
import math

import numpy as np
import pytest
import torch

from calibration_free_vector_b200 import nsn, synthetic
from oracle import nsn_oracle as orc
import nsn_testlib as tl

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)


def cosine_codebook(abs_mode: bool) -> np.ndarray:
    return nsn.nsn_build_codebook_cosine_host(0x4E534E77 + int(abs_mode), n_samples=16384, kmeans_iters=6,
                                              cosine_iters=4, abs_mode=abs_mode)


@pytest.mark.parametrize("cosine", [False, True])
@pytest.mark.parametrize("mk,mv", [(2, 1), (1, 2)])
def test_cosine_tuned_codebook_prefill_flush_decode(cosine, mk, mv):
    B, H, g, T, steps = 2, 2, 4, 384, 3
    cbk, cbv = cosine_codebook(mk == 2), cosine_codebook(mv == 2)
    rk, rv = synthetic.KVRecipe(61 + mk, H), synthetic.KVRecipe(71 + mv, H)
    xk = rk.tokens(B, T + steps, torch.bfloat16, "cpu")
    xv = rv.tokens(B, T + steps, torch.bfloat16, "cpu")
    dk, dv = torch.from_numpy(cbk).cuda(), torch.from_numpy(cbv).cuda()
    kc = nsn.Cache(B, H, 512, 128, mk, cosine=cosine)
    vc = nsn.Cache(B, H, 512, 128, mv, cosine=cosine)
    nsn.nsn_quantize_kv(kc, xk[:, :T].cuda(), dk)
    nsn.nsn_quantize_kv(vc, xv[:, :T].cuda(), dv)
    for s in range(T, T + steps):  # the first append flushes the full window as block 2
        nsn.nsn_append_residual(kc, vc, xk[:, s].cuda(), xv[:, s].cuda(), dk, dv)
    q = synthetic.queries(81, B, H * g, torch.bfloat16, "cpu")
    out = torch.empty((B, H * g, 128), dtype=torch.float32, device="cuda")
    nsn.nsn_decode_attention(kc, vc, q.cuda(), SCALE, dk, dv, out, nsn.decode_workspace(kc, H * g))
    torch.cuda.synchronize()
    assert int(kc.status.item()) == 0 and int(vc.status.item()) == 0
    out = out.cpu().numpy()
    xkf = xk.float().numpy().astype(np.float64)
    xvf = xv.float().numpy().astype(np.float64)
    qf = q.float().numpy().astype(np.float64)
    for b in range(B):
        for h in range(H):
            (kq, kw), (vq, vw) = tl.oracle_pipeline(xkf[b, :, h], xvf[b, :, h], T, T + steps,
                                                    cbk.astype(np.float64), cbv.astype(np.float64), mk, mv, 128,
                                                    cosine=cosine)
            for cache, ref_q, ref_w, x, cb, mode in ((kc, kq, kw, xkf, cbk, mk), (vc, vq, vw, xvf, cbv, mv)):
                got = tl.read_cache(cache, b, h)
                assert got["n_quant"] == ref_q["codes"].shape[0] == 384 and got["n_window"] == ref_w.shape[0]
                # codes need the oracle's gaps and u: re-run its blocks (prefill blocks 0, 1 and the flush)
                xs = x[b, :, h]
                blocks = [orc.quantize_block(xs[128 * i:128 * (i + 1)], cb.astype(np.float64), mode,
                                             cosine=cosine) for i in range(2)]
                blocks.append(orc.quantize_block(orc.to_f16(xs[256:384]), cb.astype(np.float64), mode,
                                                 cosine=cosine))
                ref = {"codes": np.concatenate([r["codes"] for r in blocks]),
                       "signs": None if mode == 1 else np.concatenate([r["signs"] for r in blocks]),
                       "gap": np.concatenate([r["gap"] for r in blocks]),
                       "s1": np.concatenate([r["s1"] for r in blocks]),
                       "s2": np.concatenate([r["s2"] for r in blocks]),
                       "o": np.stack([r["o"] for r in blocks])}
                assert np.array_equal(ref["codes"], ref_q["codes"])
                tl.compare_codes(got, ref, np.concatenate([r["u"] for r in blocks]))
                tl.compare_norms_means(got, ref, (got["codes"] != ref["codes"]).any(axis=1))
                assert np.array_equal(got["window"], ref_w)
            want = orc.decode_attention(qf[b, h * g:(h + 1) * g], kq, vq, kw, vw, cbk.astype(np.float64),
                                        cbv.astype(np.float64), mk, mv, SCALE)
            err = tl.attn_error(out[b, h * g:(h + 1) * g], want)
            assert err <= tl.ATTN_TOL, f"(b={b}, h={h}) attention error {err:.3g}"


def test_cosine_rule_changes_codes():
    # the two rules choose differently on the same data (otherwise the test above
    # could not tell them apart)
    rng = np.random.default_rng(5)
    cb = cosine_codebook(True).astype(np.float64)
    u = np.abs(rng.standard_normal((2000, 8)))
    assert (orc.cosine_codeword(u, cb)[0] != orc.nearest_codeword(u, cb)[0]).mean() > 0.01
