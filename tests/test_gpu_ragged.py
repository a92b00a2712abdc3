"""GPU parity of the ragged prefill (nsn_quantize_kv_ragged): every batch row has
its own prompt length, read from device memory.  Each sequence must match the
oracle's quantize_sequence of its own length (codes, signs, norms, means, window,
counters), equal-length rows must reproduce nsn_quantize_kv byte for byte, a
decode over the ragged caches must match the oracle's attention, and an
out-of-range length must leave its row empty and set status bit 4."""
import math

import numpy as np
import pytest
import torch

from calibration_free_vector_b200 import nsn, synthetic
from oracle import nsn_oracle as orc
import nsn_testlib as tl

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)


def cache_bytes(cache):
    parts = [cache.codes, cache.norms, cache.means, cache.n_quant, cache.n_window]
    if cache.signs is not None:
        parts.append(cache.signs)
    if cache.window_buf is not None:
        parts.append(cache.window_buf)
    return [p.cpu().clone() for p in parts]


def check_rows(x, lengths, cb, cache, mode, window):
    xf = x.float().numpy().astype(np.float64)
    for b, L in enumerate(lengths):
        for h in range(x.shape[2]):
            ref = orc.quantize_sequence(xf[b, :L, h, :], cb.astype(np.float64), mode, 128, window)
            got = tl.read_cache(cache, b, h)
            assert got["n_quant"] == ref["n_quant"], (b, L)
            assert got["n_window"] == ref["window"].shape[0], (b, L)
            if ref["n_quant"]:
                tl.compare_codes(got, ref, ref["u"])
                tl.compare_norms_means(got, ref, (got["codes"] != ref["codes"]).any(axis=1))
            assert np.array_equal(got["window"], ref["window"])


@pytest.mark.parametrize("mode,window", [(2, 128), (1, 128), (2, 0)])
def test_ragged_rows_match_the_oracle_per_sequence(mode, window):
    lengths = [0, 1, 127, 128, 129, 300, 641]
    B, H, T = len(lengths), 2, max(lengths)
    x = synthetic.KVRecipe(404 + mode, H, "llama").tokens(B, T, torch.bfloat16, "cpu")
    cb = tl.codebook(mode)
    cap = ((T + 127) // 128) * 128
    cache = nsn.Cache(B, H, cap, window, mode)
    lens = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    nsn.nsn_quantize_kv_ragged(cache, x.cuda(), lens, torch.from_numpy(cb).cuda())
    torch.cuda.synchronize()
    assert int(cache.status.item()) == 0
    check_rows(x, lengths, cb, cache, mode, window)


def test_equal_lengths_reproduce_the_common_length_prefill():
    B, H, T, mode = 3, 4, 1061, 2
    x = synthetic.KVRecipe(9, H, "llama").tokens(B, T, torch.bfloat16, "cuda")
    cb = torch.from_numpy(tl.codebook(mode)).cuda()
    a, r = nsn.Cache(B, H, 1024, 128, mode), nsn.Cache(B, H, 1024, 128, mode)
    nsn.nsn_quantize_kv(a, x, cb)
    nsn.nsn_quantize_kv_ragged(r, x, torch.full((B,), T, dtype=torch.int32, device="cuda"), cb)
    torch.cuda.synchronize()
    for p, q in zip(cache_bytes(a), cache_bytes(r)):
        assert torch.equal(p, q)


def test_out_of_range_length_sets_status_and_leaves_row_empty():
    B, H, T, mode = 3, 1, 300, 1
    x = synthetic.KVRecipe(3, H, "llama").tokens(B, T, torch.bfloat16, "cuda")
    cb = torch.from_numpy(tl.codebook(mode)).cuda()
    cache = nsn.Cache(B, H, 384, 128, mode)
    nsn.nsn_quantize_kv_ragged(cache, x, torch.tensor([200, -5, 301], dtype=torch.int32, device="cuda"), cb,
                               max_tokens=300)
    torch.cuda.synchronize()
    assert int(cache.status.item()) & 4
    nq, nw = cache.n_quant.cpu().numpy()[:, 0], cache.n_window.cpu().numpy()[:, 0]
    assert (nq[0], nw[0]) == (128, 72)
    assert (nq[1], nw[1]) == (0, 0) and (nq[2], nw[2]) == (0, 0)


def test_decode_over_ragged_caches_matches_the_oracle():
    lengths = [1, 129, 500, 1200]
    B, H, g, mk, mv = len(lengths), 2, 4, 2, 1
    T = max(lengths)
    xk = synthetic.KVRecipe(11, H, "llama").tokens(B, T, torch.bfloat16, "cpu")
    xv = synthetic.KVRecipe(12, H, "llama").tokens(B, T, torch.bfloat16, "cpu")
    cbk, cbv = tl.codebook(mk), tl.codebook(mv)
    cap = ((T + 127) // 128) * 128
    kc, vc = nsn.Cache(B, H, cap, 128, mk), nsn.Cache(B, H, cap, 128, mv)
    lens = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    dk, dv = torch.from_numpy(cbk).cuda(), torch.from_numpy(cbv).cuda()
    nsn.nsn_quantize_kv_ragged(kc, xk.cuda(), lens, dk)
    nsn.nsn_quantize_kv_ragged(vc, xv.cuda(), lens, dv)
    q = synthetic.queries(13, B, H * g, torch.bfloat16, "cpu")
    out = torch.empty((B, H * g, 128), dtype=torch.float32, device="cuda")
    nsn.nsn_decode_attention(kc, vc, q.cuda(), SCALE, dk, dv, out, nsn.decode_workspace(kc, H * g))
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    xkf, xvf = xk.float().numpy().astype(np.float64), xv.float().numpy().astype(np.float64)
    qf = q.float().numpy().astype(np.float64)
    for b, L in enumerate(lengths):
        for h in range(H):
            ks = orc.quantize_sequence(xkf[b, :L, h], cbk.astype(np.float64), mk, 128, 128)
            vs = orc.quantize_sequence(xvf[b, :L, h], cbv.astype(np.float64), mv, 128, 128)
            ref = orc.decode_attention(qf[b, h * g:(h + 1) * g], ks, vs, ks["window"], vs["window"],
                                       cbk.astype(np.float64), cbv.astype(np.float64), mk, mv, SCALE)
            assert tl.attn_error(out[b, h * g:(h + 1) * g], ref) <= tl.ATTN_TOL, (b, h, L)
