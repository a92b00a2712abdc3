"""CPU checks of bench.py's host logic: the pre-RoPE leg's frequency table is the
oracle's closed form in fp32 and its CPU baseline runs the oracle's pre-RoPE
decode; the code and sign unpacking of the sampled parity check equal the test
library's; both arms print the same config object; the parity check counts a
planted code mismatch."""
import os
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from oracle import nsn_oracle as orc  # noqa: E402


def test_rope_theta_is_the_llama3_table_in_fp32():
    th = bench.rope_theta()
    assert th.dtype == np.float32 and th.shape == (64,)
    np.testing.assert_array_equal(th, orc.rope_inv_freq(128, 500000.0).astype(np.float32))


def test_cpu_baseline_sample_runs_the_pre_rope_oracle():
    t, n, threads = bench.oracle_decode_sample(0.0, seed=3, rope=True)
    assert n == 1 and t > 0.0 and threads >= 1


def test_code_records_store_even_sub_vectors_first():
    from tests import nsn_testlib as tl
    x = np.arange(48, dtype=np.uint8).reshape(3, 16)
    st = tl.natural_to_codes(x)
    assert st[0].tolist() == list(range(0, 16, 2)) + list(range(1, 16, 2))
    np.testing.assert_array_equal(tl.codes_to_natural(st), x)
    np.testing.assert_array_equal(bench.codes_natural(st), x)


def test_bench_sign_unpacking_matches_the_test_library():
    from tests import nsn_testlib as tl
    rs = np.random.RandomState(5)
    stored = rs.randint(0, 256, size=(37, 16)).astype(np.uint8)
    np.testing.assert_array_equal(bench.signs_natural(stored), tl.signs_to_natural(stored))


def test_both_arms_print_the_same_config(capsys, monkeypatch):
    # the reference arm's config object is the shared one the GPU arm prints
    monkeypatch.setenv("RANK", "0")
    monkeypatch.setenv("WORLD_SIZE", "1")
    monkeypatch.setattr(bench, "oracle_decode_sample", lambda budget, seed=0, rope=False, W=None: (0.01, 1, 1))

    class A:
        steps, warmup, workload, batch, rope, double_quant = 2, 3, 4, 0, False, False
    assert bench.run_reference(A()) == 0
    import json
    line = json.loads(capsys.readouterr().out.strip().splitlines()[-1])
    W = bench.WORKLOADS[4]
    assert line["config"] == bench.config_dict(W, A(), 1, W["batch"])
    assert line["config"]["layers"] == 32 and line["config"]["mode_k"] == 1
    # 64 sequences x 8 kv-heads x 32 layers of 10 ms each per step
    assert line["ms_per_step"] == pytest.approx(0.01 * 64 * 8 * 32 * 1e3)


def test_oracle_quantize_check_counts_mismatches():
    # the bench's sampled parity check: identical codes give no mismatch, a
    # planted wrong code (outside the near-ties) gives one
    from oracle import nsn_oracle as orc
    rs = np.random.RandomState(6)
    x = rs.normal(size=(1, 128, 128)).astype(np.float32)
    cb = np.abs(rs.normal(size=(256, 8)))
    ref = orc.quantize_block(x[0].astype(np.float64), cb, 2)
    from tests import nsn_testlib as tl
    signs = tl.natural_to_signs(ref["signs"].astype(np.uint8))[None]
    codes = ref["codes"][None].copy()
    _, n, nsub, ntie, nbad, nsbad = bench.oracle_quantize_check(x, cb, 2, codes, signs, 60.0)
    assert (n, nsub, nbad, nsbad) == (1, 128 * 16, 0, 0)
    i = int(np.argmax(ref["gap"].reshape(-1)))
    codes.reshape(-1)[i] = (codes.reshape(-1)[i] + 1) % 256
    assert bench.oracle_quantize_check(x, cb, 2, codes, signs, 60.0)[4] == 1
