"""Parity at the full workload sizes, in the launch configuration the bench uses.

For each of the decode-throughput layer (batch 16 x 32k, 2-bit K/V, after 1 and
after 64 decode steps; also with
pre-RoPE keys), the extreme
compression layer (batch 64 x 8k, 1-bit K/V) and the long-context layer (batch 4 x
128k, 2-bit K / 1-bit V; also with pre-RoPE keys): prefill on the GPU, append the workload's decode tokens
(the first append flushes the full window), decode, then check
  * sampled prefill blocks of many (batch, kv-head) sequences element by element
    against the oracle's quantizer (blocks are independent), and
  * one sampled sequence end to end: the oracle quantizes it whole (blocks in a
    spawn process pool), replays the appends, and its decode attention must match
    the GPU output of that kv-head's query heads within the attention tolerance.
The codes compared are counted: sub-vectors, the oracle's near-ties (top-2
distance gap <= 1e-6 relative, excluded from the bit-exact check), how many of
those differ, and differing sign bits; each workload prints its counts and
asserts that near-ties stay below 0.1 % of the sub-vectors compared.
"""
import concurrent.futures as cf
import math
import multiprocessing as mp

import numpy as np
import pytest
import torch

from calibration_free_vector_b200 import nsn, synthetic
from oracle import nsn_oracle as orc
import nsn_testlib as tl

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)


@pytest.fixture(scope="module")
def pool():
    with cf.ProcessPoolExecutor(max_workers=min(16, mp.cpu_count()), mp_context=mp.get_context("spawn")) as ex:
        yield ex


def rope_theta():
    """RoPE frequencies of the Llama-3-8B shape, theta_i = 500000^(-2i/128), as fp32."""
    return (500000.0 ** (-2.0 * np.arange(64) / 128.0)).astype(np.float32)


def run_workload(cfg_id, steps, pool, sample_blocks=12, seed_off=0, double_quant=False, rope=False):
    W = synthetic.WORKLOADS[cfg_id]
    B, H, HQ, T, mk, mv = W["batch"], W["n_kv_heads"], W["n_q_heads"], W["seq"], W["mode_k"], W["mode_v"]
    g = HQ // H
    dev = torch.device("cuda")
    rk = synthetic.KVRecipe(synthetic.config_seed(cfg_id, "k") + seed_off, H)
    rv = synthetic.KVRecipe(synthetic.config_seed(cfg_id, "v") + seed_off, H)
    xk = rk.tokens(B, T + steps, torch.bfloat16, dev)
    xv = rv.tokens(B, T + steps, torch.bfloat16, dev)
    cbk, cbv = tl.codebook(mk), tl.codebook(mv)
    dk, dv = torch.from_numpy(cbk).to(dev), torch.from_numpy(cbv).to(dev)
    cap = ((T + steps + 255) // 128) * 128
    kc = nsn.Cache(B, H, cap, 128, mk, device=dev, double_quant=double_quant)
    vc = nsn.Cache(B, H, cap, 128, mv, device=dev, double_quant=double_quant)
    nsn.nsn_quantize_kv(kc, xk[:, :T], dk)
    nsn.nsn_quantize_kv(vc, xv[:, :T], dv)
    for s in range(T, T + steps):
        nsn.nsn_append_residual(kc, vc, xk[:, s], xv[:, s], dk, dv)
    q = synthetic.queries(synthetic.config_seed(cfg_id, "q") + seed_off, B, HQ, torch.bfloat16, dev)
    out = torch.empty((B, HQ, 128), dtype=torch.float32, device=dev)
    if rope:  # the cache holds pre-RoPE keys; every key is rotated at its position
        nsn.nsn_decode_attention_rope(kc, vc, q, SCALE, torch.from_numpy(rope_theta()).to(dev), dk, dv, out,
                                      nsn.decode_rope_workspace(kc, HQ, dev))
    else:
        nsn.nsn_decode_attention(kc, vc, q, SCALE, dk, dv, out, nsn.decode_workspace(kc, HQ, dev))
    torch.cuda.synchronize()
    assert int(kc.status.item()) == 0 and int(vc.status.item()) == 0

    rng = np.random.default_rng(cfg_id)
    n_quant0 = 128 * ((T - 1) // 128)
    counts = {"n": 0, "near_ties": 0, "tie_mismatch": 0, "sign_bits_differing": 0}

    def count(r):
        for k in counts:
            counts[k] += r.get(k, 0)

    # ---- sampled prefill blocks ----
    jobs, where = [], []
    for _ in range(sample_blocks):
        b, h, blk = int(rng.integers(B)), int(rng.integers(H)), int(rng.integers(n_quant0 // 128))
        for cache, x, cb, mode in ((kc, xk, cbk, mk), (vc, xv, cbv, mv)):
            xb = x[b, 128 * blk:128 * (blk + 1), h].float().cpu().numpy().astype(np.float64)
            jobs.append((xb, cb.astype(np.float64), mode, double_quant))
            where.append((cache, b, h, blk))
    refs = list(pool.map(tl._oracle_block, jobs))
    for (cache, b, h, blk), ref in zip(where, refs):
        sl = slice(128 * blk, 128 * (blk + 1))
        got = {"codes": tl.codes_to_natural(cache.codes[b, h, sl].cpu().numpy()).astype(np.int64),
               "signs": None if cache.signs is None else tl.signs_to_natural(cache.signs[b, h, sl].cpu().numpy())}
        s2 = cache.norms[b, h, sl] if double_quant else cache.norms[b, h, sl, 1]
        count(tl.compare_codes(dict(got, s2=s2.float().cpu().numpy().astype(np.float64)), ref, ref["u"]))
        if double_quant:
            par = cache.dq_params[b, h, blk, :4].float().cpu().numpy().astype(np.float64)
            q1, qo = ref["s1_dq"], ref["o_dq"]
            assert np.array_equal(par, [q1["lo"], q1["hi"], qo["lo"], qo["hi"]])
            s1_lev = tl.unpack_levels(cache.s1_levels[b, h, 64 * blk:64 * (blk + 1)].cpu().numpy())
            o_lev = tl.unpack_levels(cache.means[b, h, blk].cpu().numpy())
            for g_, r_ in ((s1_lev, q1["levels"]), (o_lev, qo["levels"])):
                assert (np.abs(g_ - r_) <= 1).all() and (g_ != r_).sum() <= 2
        else:
            got.update(s1=cache.norms[b, h, sl, 0].float().cpu().numpy().astype(np.float64),
                       s2=cache.norms[b, h, sl, 1].float().cpu().numpy().astype(np.float64),
                       o=cache.means[b, h, blk:blk + 1].float().cpu().numpy().astype(np.float64))
            ref = dict(ref, o=ref["o"][None])
            tl.compare_norms_means(got, ref, (got["codes"] != ref["codes"]).any(axis=1))

    # ---- one sequence end to end ----
    b, h = int(rng.integers(B)), int(rng.integers(H))
    seqs = []
    for x, cb, mode in ((xk, cbk, mk), (xv, cbv, mv)):
        xs = x[b, :, h].float().cpu().numpy().astype(np.float64)
        seqs.append(tl.oracle_cache_sequence(pool, xs, T, T + steps, cb.astype(np.float64), mode,
                                             double_quant=double_quant))
    (kq, kw), (vq, vw) = seqs
    got_k = tl.read_cache(kc, b, h)
    assert got_k["n_quant"] == kq["codes"].shape[0] and got_k["n_window"] == kw.shape[0]
    count(tl.compare_codes(got_k, kq, kq["u"]))
    print(f"workload {cfg_id}{' dq' if double_quant else ''}{' pre-RoPE' if rope else ''}: codes compared {counts}")
    assert counts["near_ties"] <= 1e-3 * counts["n"], counts
    assert counts["tie_mismatch"] <= counts["near_ties"]
    qf = q[b, h * g:(h + 1) * g].float().cpu().numpy().astype(np.float64)
    if rope:
        ref = orc.decode_attention_rope(qf, kq, vq, kw, vw, cbk.astype(np.float64), cbv.astype(np.float64), mk, mv,
                                        SCALE, rope_theta().astype(np.float64))
    else:
        ref = orc.decode_attention(qf, kq, vq, kw, vw, cbk.astype(np.float64), cbv.astype(np.float64), mk, mv,
                                   SCALE)
    err = tl.attn_error(out[b, h * g:(h + 1) * g].cpu().numpy(), ref)
    assert err <= tl.ATTN_TOL, f"workload {cfg_id}: (b={b}, h={h}) attention error {err:.3g}"
    return err


def test_fullsize_decode_throughput_layer(pool):
    # batch 16, 32k context, 2-bit K/V, window 128; one decode step (the append flushes)
    run_workload(3, 1, pool)


def test_fullsize_extreme_compression_layer(pool):
    # batch 64, 8k context, 1-bit K/V (one of the 32 identical layers)
    run_workload(4, 1, pool)


def test_fullsize_long_context(pool):
    # batch 4, 128k-token prefill, 2-bit K / 1-bit V, 16 decode steps
    run_workload(5, 16, pool)


def test_fullsize_decode_throughput_layer_double_quant(pool):
    # the same layer with s1 and o stored in 4 bits (bench.py --double-quant)
    run_workload(3, 1, pool, double_quant=True)


def test_fullsize_decode_throughput_layer_pre_rope(pool):
    # the same layer with pre-RoPE keys (bench.py --rope): positions up to 32k
    run_workload(3, 1, pool, sample_blocks=2, rope=True)


def test_fullsize_long_context_pre_rope(pool):
    # batch 4, 128k context, pre-RoPE keys: angles up to about 1.3e5 rad at theta_0 = 1
    run_workload(5, 16, pool, sample_blocks=2, rope=True)


def test_fullsize_decode_throughput_layer_64_steps(pool):
    # the state the bench times: 64 decode steps, the first append flushes the full
    # window into the quantized part and the window then grows back to 64 tokens
    run_workload(3, 64, pool, sample_blocks=2, seed_off=1)
