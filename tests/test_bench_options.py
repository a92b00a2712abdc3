"""CPU checks of the bench's pre-RoPE leg: the frequency table it passes to the
library is the oracle's closed form in fp32, and its CPU baseline sample runs
the oracle's pre-RoPE decode."""
import os
import sys

import numpy as np

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
