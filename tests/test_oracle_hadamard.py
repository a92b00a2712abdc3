"""Pins of the oracle's Hadamard transform (plain Sylvester matrix, natural
order) against closed forms and scipy's Sylvester construction."""
import numpy as np
import pytest
import scipy.linalg

from oracle import nsn_oracle as orc



@pytest.mark.parametrize("d", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_matches_scipy_sylvester(d):
    ref = scipy.linalg.hadamard(d) / np.sqrt(d)
    assert np.array_equal(orc.hadamard_matrix(d), ref)


def test_recursive_definition():
    # H_{2n} = [[H_n, H_n], [H_n, -H_n]] / sqrt(2), built independently.
    h = np.array([[1.0]])
    for _ in range(7):
        h = np.block([[h, h], [h, -h]]) / np.sqrt(2.0)
    assert np.allclose(orc.hadamard_matrix(128), h, atol=1e-15, rtol=0)


def test_orthonormal_symmetric_involution():
    h = orc.hadamard_matrix(128)
    assert np.array_equal(h, h.T)
    assert np.abs(h @ h.T - np.eye(128)).max() < 1e-14
    assert np.abs(h @ h - np.eye(128)).max() < 1e-14


def test_norm_preserved_and_columns():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((64, 128)) * 5
    y = orc.rotate(x)
    assert np.allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-13)
    assert np.allclose(orc.rotate(y), x, atol=1e-12)
    eye = np.eye(128)
    assert np.array_equal(orc.rotate(eye), orc.hadamard_matrix(128).T)


def test_rejects_non_power_of_two():
    with pytest.raises(ValueError):
        orc.hadamard_matrix(96)
