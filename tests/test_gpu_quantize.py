"""GPU parity of the quantizer (nsn_quantize_kv, nsn_append_residual) against
the CPU oracle, element by element, on seeded synthetic inputs: several
blocks, ragged tails, both modes, all input dtypes, degenerate tokens."""
import numpy as np
import pytest
import torch

from calibration_free_vector_b200 import nsn, synthetic
from oracle import nsn_oracle as orc
import nsn_testlib as tl

pytestmark = pytest.mark.gpu

DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def run_prefill(batch, heads, seq, mode, dtype, window, kind="llama", seed=1, capacity=None, x=None, cb=None):
    if x is None:
        x = synthetic.KVRecipe(seed, heads, kind).tokens(batch, seq, DT[dtype], "cpu")
    cb = tl.codebook(mode) if cb is None else cb
    cap = capacity or max(128, ((seq + 127) // 128) * 128)
    cache = nsn.Cache(batch, heads, cap, window, mode)
    nsn.nsn_quantize_kv(cache, x.cuda(), torch.from_numpy(cb).cuda())
    torch.cuda.synchronize()
    return x, cb, cache


def check_prefill(x, cb, cache, mode, window):
    stats = {"n": 0, "near_ties": 0, "tie_mismatch": 0}
    batch, seq, heads, _ = x.shape
    xf = x.float().numpy().astype(np.float64)
    for b in range(batch):
        for h in range(heads):
            ref = orc.quantize_sequence(xf[b, :, h, :], cb.astype(np.float64), mode, 128, window)
            got = tl.read_cache(cache, b, h)
            assert got["n_quant"] == ref["n_quant"]
            assert got["n_window"] == ref["window"].shape[0]
            r = tl.compare_codes(got, ref, ref["u"])
            for k in stats:
                stats[k] += r[k]
            mism_rows = (got["codes"] != ref["codes"]).any(axis=1)
            tl.compare_norms_means(got, ref, mism_rows)
            assert np.array_equal(got["window"], ref["window"])
    # near-ties are counted, not failed; they must stay rare
    assert stats["near_ties"] <= max(2, 1e-3 * stats["n"]), stats
    return stats


@pytest.mark.parametrize("mode", [1, 2])
def test_config1_tiny_fp32(mode):
    # 1 kv-head, 256 fp32 tokens with 5 offset channels, no window: 2 full blocks.
    x, cb, cache = run_prefill(1, 1, 256, mode, "f32", 0, kind="tiny",
                               seed=synthetic.config_seed(1, "k"))
    st = check_prefill(x, cb, cache, mode, 0)
    assert st["n"] == 256 * 16


@pytest.mark.parametrize("mode,dtype", [(2, "bf16"), (1, "bf16"), (2, "f16"), (1, "f32")])
def test_llama_shape_ragged(mode, dtype):
    # 8 kv-heads, 1061 tokens -> 1024 quantized in 8 blocks + 37 in the window.
    x, cb, cache = run_prefill(1, 8, 1061, mode, dtype, 128, seed=synthetic.config_seed(2, "k"))
    check_prefill(x, cb, cache, mode, 128)


@pytest.mark.parametrize("mode", [1, 2])
def test_codebook_not_fp16_representable(mode):
    # The quantizer takes any fp32 codebook: its tensor-core scores use the fp16
    # rounding of it, and the decision bound then widens by ||a|| ||c - fp16(c)||.
    # The codes must still be the exact nearest of the fp32 codebook.
    rng = np.random.default_rng(5 + mode)
    cb = (tl.codebook(mode).astype(np.float64) * (1.0 + 3e-4 * rng.standard_normal((256, 8)))).astype(np.float32)
    assert np.any(cb != cb.astype(np.float16).astype(np.float32))
    x, cb, cache = run_prefill(1, 4, 700, mode, "bf16", 128, seed=91, cb=cb)
    check_prefill(x, cb, cache, mode, 128)


def test_duplicate_codeword_ties_go_to_the_lower_index():
    # Codeword 200 repeats codeword 17 exactly: every sub-vector nearest to it is an
    # exact tie, which the exact path resolves to the lower index, as the oracle does.
    cb = tl.codebook(2).copy()
    cb[200] = cb[17]
    x, cb, cache = run_prefill(1, 2, 1000, 2, "bf16", 128, seed=93, cb=cb)
    xf = x.float().numpy().astype(np.float64)
    hits = 0
    for h in range(2):
        ref = orc.quantize_sequence(xf[0, :, h, :], cb.astype(np.float64), 2, 128, 128)
        got = tl.read_cache(cache, 0, h)
        assert not np.any(got["codes"] == 200) and not np.any(ref["codes"] == 200)
        assert np.array_equal(got["codes"] == 17, ref["codes"] == 17)
        hits += int(np.sum(ref["codes"] == 17))
    assert hits > 0  # the tie is actually exercised


def test_partial_last_block_no_window():
    x, cb, cache = run_prefill(2, 2, 200, 2, "bf16", 0, seed=77)
    check_prefill(x, cb, cache, 2, 0)


def test_strided_input_view():
    # x as a view with a non-compact token stride (every other token of a bigger buffer).
    big = synthetic.KVRecipe(5, 4, "llama").tokens(1, 700, torch.bfloat16, "cpu")
    x = big[:, ::2]
    assert not x.is_contiguous()
    cb = tl.codebook(1)
    cache = nsn.Cache(1, 4, 384, 128, 1)
    nsn.nsn_quantize_kv(cache, big.cuda()[:, ::2], torch.from_numpy(cb).cuda())
    torch.cuda.synchronize()
    check_prefill(x.contiguous(), cb, cache, 1, 128)


@pytest.mark.parametrize("mode", [1, 2])
def test_degenerate_tokens(mode):
    # zero token (s1 = 0), a block of identical tokens (s2 = 0 everywhere),
    # a one-token block, and a huge-offset token.
    rec = synthetic.KVRecipe(9, 1, "llama")
    x = rec.tokens(1, 257, torch.float32, "cpu")
    x[0, 5, 0, :] = 0.0
    x[0, 128:256, 0, :] = x[0, 128, 0, :]
    x[0, 7, 0, 3] = 3000.0
    x_, cb, cache = run_prefill(1, 1, 257, mode, "f32", 0, x=x)
    got = tl.read_cache(cache, 0, 0)
    assert got["s1"][5] == 0.0
    assert np.all(got["s2"][128:256] == 0.0)
    check_prefill(x, cb, cache, mode, 0)


def test_empty_and_short_prefill():
    x, cb, cache = run_prefill(1, 2, 0, 2, "bf16", 128)
    assert cache.n_quant.sum().item() == 0 and cache.n_window.sum().item() == 0
    x, cb, cache = run_prefill(1, 2, 128, 2, "bf16", 128)
    assert cache.n_quant.sum().item() == 0 and (cache.n_window == 128).all()
    check_prefill(x, cb, cache, 2, 128)


@pytest.mark.parametrize("mk,mv", [(2, 2), (2, 1), (1, 1)])
def test_append_flush(mk, mv):
    # Prefill 384 tokens (256 quantized + full window of 128), then append 3
    # tokens: the first append flushes the window as block 2.
    heads, batch = 4, 2
    rk, rv = synthetic.KVRecipe(21, heads), synthetic.KVRecipe(22, heads)
    xk = rk.tokens(batch, 387, torch.bfloat16, "cpu")
    xv = rv.tokens(batch, 387, torch.bfloat16, "cpu")
    cbk, cbv = tl.codebook(mk), tl.codebook(mv)
    kc = nsn.Cache(batch, heads, 512, 128, mk)
    vc = nsn.Cache(batch, heads, 512, 128, mv)
    dk, dv = torch.from_numpy(cbk).cuda(), torch.from_numpy(cbv).cuda()
    nsn.nsn_quantize_kv(kc, xk[:, :384].cuda(), dk)
    nsn.nsn_quantize_kv(vc, xv[:, :384].cuda(), dv)
    for s in range(384, 387):
        nsn.nsn_append_residual(kc, vc, xk[:, s].cuda(), xv[:, s].cuda(), dk, dv)
    torch.cuda.synchronize()
    assert (kc.n_quant == 384).all() and (kc.n_window == 3).all()
    assert (vc.n_quant == 384).all() and (vc.n_window == 3).all()
    assert kc.status.item() == 0
    for cache, x, cb, mode in ((kc, xk, cbk, mk), (vc, xv, cbv, mv)):
        xf = x.float().numpy().astype(np.float64)
        for b in range(batch):
            for h in range(heads):
                got = tl.read_cache(cache, b, h)
                pre = orc.quantize_sequence(xf[b, :384, h], cb.astype(np.float64), mode, 128, 128)
                flushed = orc.quantize_block(orc.to_f16(xf[b, 256:384, h]), cb.astype(np.float64), mode)
                ref = {
                    "codes": np.concatenate([pre["codes"], flushed["codes"]]),
                    "signs": None if mode == 1 else np.concatenate([pre["signs"], flushed["signs"]]),
                    "s1": np.concatenate([pre["s1"], flushed["s1"]]),
                    "s2": np.concatenate([pre["s2"], flushed["s2"]]),
                    "o": np.concatenate([pre["o"], flushed["o"][None]]),
                    "gap": np.concatenate([pre["gap"], flushed["gap"]]),
                }
                u = np.concatenate([pre["u"], flushed["u"]])
                tl.compare_codes(got, ref, u)
                tl.compare_norms_means(got, ref, (got["codes"] != ref["codes"]).any(axis=1))
                assert np.array_equal(got["window"], orc.to_f16(xf[b, 384:387, h]))


def test_append_capacity_overflow_sets_status():
    kc = nsn.Cache(1, 1, 128, 128, 2)
    vc = nsn.Cache(1, 1, 128, 128, 2)
    cb = torch.from_numpy(tl.codebook(2)).cuda()
    x = synthetic.KVRecipe(3, 1).tokens(1, 257, torch.bfloat16, "cuda")
    nsn.nsn_quantize_kv(kc, x[:, :256], cb)     # 128 quantized (capacity full) + 128 window
    nsn.nsn_quantize_kv(vc, x[:, :256], cb)
    nsn.nsn_append_residual(kc, vc, x[:, 256], x[:, 256], cb, cb)
    torch.cuda.synchronize()
    assert kc.status.item() & 1 and vc.status.item() & 1
    assert kc.n_quant.item() == 128 and kc.n_window.item() == 128   # unchanged


def test_invalid_arguments_launch_nothing():
    cache = nsn.Cache(1, 1, 128, 128, 2)
    cb = torch.from_numpy(tl.codebook(2)).cuda()
    x = torch.zeros((1, 300, 1, 128), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(nsn.NsnError) as e:
        nsn.nsn_quantize_kv(cache, x, cb)        # 256 quantized tokens > capacity 128
    assert e.value.status == 1
    torch.cuda.synchronize()
    assert cache.n_quant.item() == 0
    with pytest.raises(nsn.NsnError):
        nsn.nsn_quantize_kv(cache, x[:, :10], cb.view(-1)[1:])  # misaligned codebook pointer
