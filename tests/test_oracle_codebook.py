"""Pins of the oracle's codebook construction: Philox4x64-10 against numpy's
own Philox bit generator, Box-Muller output statistics, and k-means against
scipy's Lloyd iteration from the same initial centroids plus the fixed-point
property."""
import math

import numpy as np
import pytest
from scipy import stats
from scipy.cluster.vq import kmeans2

from oracle import codebook_oracle as cbo


def test_philox_matches_numpy_bit_generator():
    for key in ([0, 0], [123, cbo.STREAM_KEY1], [2**64 - 1, 2**63 + 5]):
        bg = np.random.Philox(key=np.array(key, dtype=np.uint64), counter=0)
        raw = [int(x) for x in bg.random_raw(4 * 6)]
        # numpy advances the counter before its first block: its block j is ours j+1.
        ours = []
        for j in range(1, 7):
            ours.extend(cbo.philox4x64_10((j, 0, 0, 0), key))
        assert raw == ours


def test_philox_counter_carry():
    bg = np.random.Philox(key=np.array([7, 9], dtype=np.uint64), counter=2**64 - 1)
    raw = [int(x) for x in bg.random_raw(4)]
    assert raw == list(cbo.philox4x64_10((0, 1, 0, 0), (7, 9)))


def test_uniform_in_open_interval():
    assert cbo.uniform_open(0) == 2.0 ** -53
    assert cbo.uniform_open(2**64 - 1) == 1.0 - 2.0 ** -53


def test_normal_stream_statistics():
    z = cbo.normal_stream(2024, 40000)
    assert abs(z.mean()) < 0.02 and abs(z.var() - 1) < 0.03
    assert stats.kstest(z, "norm").pvalue > 1e-3
    assert np.array_equal(cbo.normal_stream(2024, 10), z[:10])
    s = cbo.normal_samples(5, 100, 8, abs_mode=True)
    assert s.shape == (100, 8) and np.all(s >= 0)


def test_kmeans_matches_scipy_lloyd():
    rng = np.random.default_rng(14)
    x = rng.standard_normal((3000, 8))
    ours = cbo.kmeans(x, 32, iters=6)
    ref, _ = kmeans2(x, x[:32].copy(), iter=6, minit="matrix", missing="warn")
    assert np.allclose(ours, ref, atol=1e-12)


def test_kmeans_fixed_point_and_monotone():
    x = cbo.normal_samples(11, 4000, 8, abs_mode=False)
    prev = np.inf
    for it in (1, 3, 8, 20):
        c = cbo.kmeans(x, 16, iters=it)
        d = ((x[:, None, :] - c[None]) ** 2).sum(-1)
        obj = d.min(1).sum()
        assert obj <= prev + 1e-9
        prev = obj
    lab = d.argmin(1)
    c_next = np.stack([x[lab == k].mean(0) for k in range(16)])
    assert np.abs(c_next - c).max() < 0.05


def test_build_codebook_is_fp16_representable():
    cb = cbo.build_codebook(3, 1024, 16, 8, abs_mode=True, iters=3)
    assert np.array_equal(cb, cb.astype(np.float16).astype(np.float64))
    assert np.all(cb >= 0)


# ---- cosine fine-tuning -------------------------------------------------------

def test_cosine_step_2d_closed_form():
    # One codeword, members on the plane: the summed cosine is maximised by the
    # direction of the summed unit vectors, atan2(sum sin, sum cos), and the
    # least-squares length is the mean projection on it.
    rng = np.random.default_rng(3)
    theta = rng.uniform(-0.7, 0.9, 50)
    r = rng.uniform(0.5, 2.0, 50)
    x = np.stack([r * np.cos(theta), r * np.sin(theta)], axis=1)
    new = cbo.cosine_step(x, np.array([[1.0, 0.0]]), np.zeros(50, dtype=np.int64))
    phi = math.atan2(np.sin(theta).sum(), np.cos(theta).sum())
    length = np.mean(r * np.cos(theta - phi))
    assert np.allclose(new[0], length * np.array([math.cos(phi), math.sin(phi)]), rtol=0, atol=1e-12)


def test_cosine_step_is_locally_optimal_and_least_squares():
    x = cbo.normal_samples(11, 2000, 8, False)
    cent = cbo.kmeans(x, 16, 4)
    label = cbo.nearest(x, cent)
    new = cbo.cosine_step(x, cent, label)
    rng = np.random.default_rng(0)
    for k in range(16):
        m = x[label == k]
        u = new[k] / np.linalg.norm(new[k])
        base = np.sum(m @ u / np.linalg.norm(m, axis=1))
        for _ in range(20):   # no small turn of the direction raises the summed cosine
            v = u + 1e-3 * rng.standard_normal(8)
            v /= np.linalg.norm(v)
            assert np.sum(m @ v / np.linalg.norm(m, axis=1)) <= base + 1e-12
        s = np.linalg.norm(new[k])   # d/ds sum ||x - s u||^2 = 2 sum (s - x.u) = 0
        assert abs(np.sum(s - m @ u)) <= 1e-9 * len(m)


def test_cosine_step_keeps_codewords_without_members():
    x = np.array([[1.0, 0.0], [0.9, 0.1]])
    cent = np.array([[1.0, 0.0], [-5.0, 3.0]])
    new = cbo.cosine_step(x, cent, np.array([0, 0]))
    assert np.array_equal(new[1], cent[1])


@pytest.mark.parametrize("abs_mode", [False, True])
def test_cosine_finetune_lowers_the_cosine_distance(abs_mode):
    x = cbo.normal_samples(21, 8192, 8, abs_mode)
    km = cbo.kmeans(x, 32, 6)
    ft = cbo.cosine_finetune(x, km, 5)
    assert cbo.cosine_distance(x, ft) < cbo.cosine_distance(x, km)


def test_cosine_zero_iterations_is_the_kmeans_codebook():
    a = cbo.build_codebook_cosine(9, 4096, 32, 8, True, 5, 0)
    b = cbo.build_codebook(9, 4096, 32, 8, True, 5)
    assert np.array_equal(a, b)


def test_codebook_4bit_hand_cases():
    # entries 0..15 are already the 16 levels; 0.5 and 2.5 round to the even level
    cb = np.arange(16.0).reshape(2, 8)
    assert np.array_equal(cbo.codebook_4bit(cb), cb)
    cb2 = np.array([[0.0, 0.5, 2.5, 15.0, 1.0, 3.0, 7.0, 9.0]])
    assert list(cbo.codebook_4bit(cb2)[0]) == [0.0, 0.0, 2.0, 15.0, 1.0, 3.0, 7.0, 9.0]
