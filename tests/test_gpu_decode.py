"""GPU parity of decode attention (nsn_decode_attention) against the CPU oracle:
first on random compressed caches written directly into the buffers (isolates
decode from the quantizer), then end to end (prefill -> append/flush -> decode)
on the tiny fp32 workload, the Llama-3-8B layer shape and a mixed-mode cache."""
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


@pytest.mark.parametrize("g", [1, 2, 4, 8])
@pytest.mark.parametrize("mk,mv", [(1, 1), (1, 2), (2, 1), (2, 2)])
def test_decode_random_cache(mk, mv, g):
    B, H, cap = 3, 2, 2304
    # (n_quant, n_window) per (b, h): several splits, one block, window only, nothing
    shape = {(0, 0): (2304, 128), (0, 1): (128, 5), (1, 0): (896, 0), (1, 1): (0, 77),
             (2, 0): (1152, 1), (2, 1): (0, 0)}
    kc, vc = nsn.Cache(B, H, cap, 128, mk), nsn.Cache(B, H, cap, 128, mv)
    kcont, vcont = {}, {}
    for (b, h), (nq, nw) in shape.items():
        seed = 1000 * b + 10 * h + 100 * mk + mv
        kcont[(b, h)] = synthetic.random_cache_contents(seed, nq, nw, mk)
        vcont[(b, h)] = synthetic.random_cache_contents(seed + 5, nq, nw, mv)
    fill_cache(kc, kcont)
    fill_cache(vc, vcont)
    cbk, cbv = tl.codebook(mk), tl.codebook(mv)
    q = synthetic.queries(7, B, H * g, torch.bfloat16, "cpu")
    out = torch.empty((B, H * g, 128), dtype=torch.float32, device="cuda")
    ws = nsn.decode_workspace(kc, H * g)
    nsn.nsn_decode_attention(kc, vc, q.cuda(), SCALE, torch.from_numpy(cbk).cuda(), torch.from_numpy(cbv).cuda(),
                             out, ws)
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    qf = q.float().numpy().astype(np.float64)
    for (b, h), (nq, nw) in shape.items():
        got = out[b, h * g:(h + 1) * g]
        if nq + nw == 0:
            assert np.all(got == 0.0)
            continue
        ref = orc.decode_attention(qf[b, h * g:(h + 1) * g], oracle_seq(kcont[(b, h)]), oracle_seq(vcont[(b, h)]),
                                   kcont[(b, h)]["window"].astype(np.float64),
                                   vcont[(b, h)]["window"].astype(np.float64),
                                   cbk.astype(np.float64), cbv.astype(np.float64), mk, mv, SCALE)
        err = tl.attn_error(got, ref)
        assert err <= tl.ATTN_TOL, f"(b={b}, h={h}) nq={nq} nw={nw}: error {err:.3g}"


def run_e2e(B, H, g, T, steps, mk, mv, dtype, kind, seeds, window=128):
    rk, rv = synthetic.KVRecipe(seeds[0], H, kind), synthetic.KVRecipe(seeds[1], H, kind)
    xk = rk.tokens(B, T + steps, dtype, "cpu")
    xv = rv.tokens(B, T + steps, dtype, "cpu")
    cbk, cbv = tl.codebook(mk), tl.codebook(mv)
    dk, dv = torch.from_numpy(cbk).cuda(), torch.from_numpy(cbv).cuda()
    cap = max(128, ((T + steps + 127) // 128) * 128)
    kc, vc = nsn.Cache(B, H, cap, window, mk), nsn.Cache(B, H, cap, window, mv)
    nsn.nsn_quantize_kv(kc, xk[:, :T].cuda(), dk)
    nsn.nsn_quantize_kv(vc, xv[:, :T].cuda(), dv)
    for s in range(T, T + steps):
        nsn.nsn_append_residual(kc, vc, xk[:, s].cuda(), xv[:, s].cuda(), dk, dv)
    q = synthetic.queries(seeds[2], B, H * g, dtype, "cpu")
    out = torch.empty((B, H * g, 128), dtype=torch.float32, device="cuda")
    nsn.nsn_decode_attention(kc, vc, q.cuda(), SCALE, dk, dv, out, nsn.decode_workspace(kc, H * g))
    torch.cuda.synchronize()
    out = out.cpu().numpy()
    xkf, xvf = xk.float().numpy().astype(np.float64), xv.float().numpy().astype(np.float64)
    qf = q.float().numpy().astype(np.float64)
    worst = 0.0
    for b in range(B):
        for h in range(H):
            (kq, kw), (vq, vw) = oracle_pipeline(xkf[b, :, h], xvf[b, :, h], T, T + steps,
                                                 cbk.astype(np.float64), cbv.astype(np.float64), mk, mv, window)
            got_k = tl.read_cache(kc, b, h)
            assert got_k["n_quant"] == kq["codes"].shape[0] and got_k["n_window"] == kw.shape[0]
            ref = orc.decode_attention(qf[b, h * g:(h + 1) * g], kq, vq, kw, vw, cbk.astype(np.float64),
                                       cbv.astype(np.float64), mk, mv, SCALE)
            worst = max(worst, tl.attn_error(out[b, h * g:(h + 1) * g], ref))
    assert worst <= tl.ATTN_TOL, f"worst attention error {worst:.3g}"
    return worst


def test_e2e_config1_tiny():
    # 1 kv-head, 256 fp32 tokens, 1-bit, quantize all (no window), one fp32 query.
    run_e2e(1, 1, 1, 256, 0, 1, 1, torch.float32, "tiny",
            (synthetic.config_seed(1, "k"), synthetic.config_seed(1, "v"), synthetic.config_seed(1, "q")), window=0)


def test_e2e_config2_llama_layer():
    # Llama-3-8B layer: 32 q / 8 kv heads, 4096 bf16 tokens, 2-bit K/V, window 128,
    # one decode step (the append flushes the full window first).
    run_e2e(1, 8, 4, 4096, 1, 2, 2, torch.bfloat16, "llama",
            (synthetic.config_seed(2, "k"), synthetic.config_seed(2, "v"), synthetic.config_seed(2, "q")))


def test_e2e_mixed_modes_across_flushes():
    # 2-bit K / 1-bit V (the long-context mix), 130 appends crossing a flush.
    run_e2e(2, 2, 4, 1000, 130, 2, 1, torch.bfloat16, "llama", (31, 32, 33))


def test_workspace_counters_return_to_zero_and_calls_repeat():
    # The decode merges its split partials through one counter per (sequence,
    # head group) at the start of the workspace; every completed call leaves the
    # counters at zero, so back-to-back calls on one workspace agree exactly.
    B, H, g, mk, mv = 2, 2, 8, 2, 1
    shape = {(0, 0): (2304, 128), (0, 1): (640, 7), (1, 0): (128, 0), (1, 1): (0, 33)}
    kc, vc = nsn.Cache(B, H, 2304, 128, mk), nsn.Cache(B, H, 2304, 128, mv)
    kcont, vcont = {}, {}
    for (b, h), (nq, nw) in shape.items():
        kcont[(b, h)] = synthetic.random_cache_contents(50 + 10 * b + h, nq, nw, mk)
        vcont[(b, h)] = synthetic.random_cache_contents(70 + 10 * b + h, nq, nw, mv)
    fill_cache(kc, kcont)
    fill_cache(vc, vcont)
    cbk = torch.from_numpy(tl.codebook(mk)).cuda()
    cbv = torch.from_numpy(tl.codebook(mv)).cuda()
    q = synthetic.queries(9, B, H * g, torch.bfloat16, "cuda")
    ws = nsn.decode_workspace(kc, H * g)
    outs = []
    for _ in range(3):
        out = torch.full((B, H * g, 128), float("nan"), dtype=torch.float32, device="cuda")
        nsn.nsn_decode_attention(kc, vc, q, SCALE, cbk, cbv, out, ws)
        torch.cuda.synchronize()
        outs.append(out.cpu())
        counters = ws[: 4 * 2 * B * H].view(torch.int32).cpu()
        assert int(counters.abs().sum()) == 0, "merge counters not back to zero"
    assert torch.isfinite(outs[0]).all()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[1], outs[2])
    qf = q.float().cpu().numpy().astype(np.float64)
    cbk64, cbv64 = tl.codebook(mk).astype(np.float64), tl.codebook(mv).astype(np.float64)
    for (b, h) in shape:
        ref = orc.decode_attention(qf[b, h * g:(h + 1) * g], oracle_seq(kcont[(b, h)]), oracle_seq(vcont[(b, h)]),
                                   kcont[(b, h)]["window"].astype(np.float64),
                                   vcont[(b, h)]["window"].astype(np.float64), cbk64, cbv64, mk, mv, SCALE)
        assert tl.attn_error(outs[0][b, h * g:(h + 1) * g].numpy(), ref) <= tl.ATTN_TOL
