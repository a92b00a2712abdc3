"""Pins of the oracle's nearest-codeword assignment, 2-bit sign/abs split and
adaptive scale: hand-computed cases, scipy's cdist, exhaustive search over all
signed codewords, and the defining property of the scale factor."""
import itertools
import math

import numpy as np
import pytest
from scipy.spatial.distance import cdist

from oracle import nsn_oracle as orc


def test_hand_cases_1bit_and_ties():
    cb = np.array([[1.0, 0.0], [0.0, 1.0], [-1.0, 0.0], [0.0, -1.0]])
    codes, signs, gap = orc.assign(np.array([[0.9, 0.2], [0.5, 0.5], [-0.2, -0.9]]), cb, orc.MODE_1BIT)
    # (0.9,0.2): d = 0.05, 1.45, 3.65, 2.25 -> 0
    # (0.5,0.5): d0 = d1 = 0.5 -> tie -> lowest index 0, gap 0
    # (-0.2,-0.9): d = 2.25, 3.65, 1.45, 0.05 -> 3
    assert codes.tolist() == [0, 0, 3]
    assert signs is None
    assert gap[1] == 0.0
    # second nearest of (0.9,0.2) is code 1 at 1.45: gap = (1.45 - 0.05) / 1.45
    assert abs(gap[0] - (1.45 - 0.05) / 1.45) < 1e-14


def test_hand_case_2bit():
    a = np.array([[1.0, 0.0], [0.0, 1.0], [0.5, 0.5]])
    codes, signs, _ = orc.assign(np.array([[-0.9, 0.2], [0.1, -0.8], [-0.0, 0.0]]), a, orc.MODE_2BIT)
    # |(-0.9,0.2)| = (0.9,0.2): d = 0.05, 1.45, 0.25 -> 0; sign bit0 set
    # |(0.1,-0.8)| = (0.1,0.8): d = 1.45, 0.05, 0.25 -> 1; sign bit1 set
    # |(-0.0,0.0)| = (0,0): d = 1, 1, 0.5 -> 2; -0.0 is not < 0 -> no sign bit
    assert codes.tolist() == [0, 1, 2]
    assert signs.tolist() == [1, 2, 0]
    uh = orc.reconstruct_sub(codes, signs, a, orc.MODE_2BIT)
    assert np.array_equal(uh[0], [-1.0, 0.0])
    assert np.array_equal(uh[1], [0.0, -1.0])


def test_gap_zero_codeword_distances():
    cb = np.array([[0.0, 0.0], [1.0, 1.0]])
    codes, _, gap = orc.assign(np.array([[0.0, 0.0]]), cb, orc.MODE_1BIT)
    assert codes[0] == 0 and gap[0] == 1.0


def test_matches_scipy_cdist():
    rng = np.random.default_rng(5)
    cb = rng.standard_normal((256, 8))
    pts = rng.standard_normal((3000, 8)) * 1.3
    codes, _, gap = orc.assign(pts, cb, orc.MODE_1BIT)
    ref = cdist(pts, cb, "sqeuclidean")
    assert np.array_equal(codes, ref.argmin(axis=1))
    srt = np.sort(ref, axis=1)
    assert np.allclose(gap, (srt[:, 1] - srt[:, 0]) / srt[:, 1], rtol=1e-9, atol=1e-12)


def test_two_bit_equals_exhaustive_signed_search():
    # For an abs codebook (A >= 0) the best signed codeword s*A_k has s = sign(u)
    # and k = argmin || |u| - A_k ||.  Compare against all 256*256 signed codewords.
    rng = np.random.default_rng(6)
    a = np.abs(rng.standard_normal((256, 8)))
    u = rng.standard_normal((120, 8))
    codes, signs, _ = orc.assign(u, a, orc.MODE_2BIT)
    sign_patterns = np.array(list(itertools.product([1.0, -1.0], repeat=8)))[:, ::-1]
    # pattern index p has bit i set iff component i is negated
    pidx = np.array([sum((1 << i) for i in range(8) if pat[i] < 0) for pat in sign_patterns])
    signed = (sign_patterns[:, None, :] * a[None, :, :]).reshape(-1, 8)   # [256 patterns * 256 codes, 8]
    d = cdist(u, signed, "sqeuclidean")
    best = d.argmin(axis=1)
    best_pat = pidx[best // 256]
    best_code = best % 256
    assert np.array_equal(best_code, codes)
    assert np.array_equal(best_pat, signs.astype(np.int64))
    uh = orc.reconstruct_sub(codes, signs, a, orc.MODE_2BIT)
    assert np.allclose(((u - uh) ** 2).sum(1), d.min(axis=1), rtol=1e-12)


def test_scale_factor_property():
    rng = np.random.default_rng(7)
    u = rng.standard_normal((50, 128))
    uh = u + 0.4 * rng.standard_normal((50, 128))
    alpha = orc.scale_factor(u, uh)
    # The component of alpha*u_hat along u equals u:  (alpha u_hat . u) / ||u||^2 = 1.
    proj = alpha * np.sum(uh * u, axis=1) / np.sum(u * u, axis=1)
    assert np.allclose(proj, 1.0, rtol=1e-13)
    assert np.array_equal(orc.scale_factor(np.zeros((1, 4)), np.ones((1, 4))), [1.0])
    assert np.array_equal(orc.scale_factor(np.ones((1, 4)), -np.ones((1, 4))), [1.0])


def test_scale_hand_case():
    cb = np.array([[1.0, 0.0], [0.0, 1.0], [-1.0, 0.0], [0.0, -1.0]])
    u = np.array([[0.9, 0.2, -0.9, 0.2]])
    codes, _, _ = orc.assign(u.reshape(2, 2), cb, orc.MODE_1BIT)
    assert codes.tolist() == [0, 2]
    uh = orc.reconstruct_sub(codes, None, cb, orc.MODE_1BIT).reshape(1, 4)
    assert np.allclose(orc.scale_factor(u, uh), [1.7 / 1.8], rtol=1e-15)


def test_f16_rounding_is_round_to_nearest_even():
    # 1 + 2^-11 lies halfway between 1 and 1 + 2^-10: ties to even -> 1.
    assert orc.to_f16(1.0 + 2.0 ** -11)[()] == 1.0
    assert orc.to_f16(1.0 + 3 * 2.0 ** -11)[()] == 1.0 + 2.0 ** -9
    with np.errstate(over="ignore"):
        assert orc.to_f16(65520.0)[()] == np.inf


def test_sign_layout_conversion_roundtrip():
    import nsn_testlib as tl
    rng = np.random.default_rng(15)
    nat = rng.integers(0, 256, size=(50, 16)).astype(np.uint8)
    stored = tl.natural_to_signs(nat)
    assert np.array_equal(tl.signs_to_natural(stored), nat)
    # single bit: dim 8*3 + 5 (sub 3, i 5) -> field 5 (bytes 10, 11), bit 15 - 3 = 12 -> byte 11 bit 4
    one = np.zeros((1, 16), np.uint8)
    one[0, 3] = 1 << 5
    st = tl.natural_to_signs(one)
    assert st[0, 11] == 1 << 4 and st.sum() == 16


# ---------------------------------------------------------------------------
# Cosine-assignment variant ([TS] Metodologia 3: codebook tuned for the cosine
# distance between a vector and its quantized version)
# ---------------------------------------------------------------------------
def test_cosine_assignment_by_brute_force_angles():
    # the chosen codeword has the smallest angle to the point, computed with arccos
    rng = np.random.default_rng(31)
    pts = rng.standard_normal((300, 8))
    cb = rng.standard_normal((64, 8)) * rng.uniform(0.2, 3.0, (64, 1))
    idx, _ = orc.cosine_codeword(pts, cb)
    for i in range(pts.shape[0]):
        ang = [math.acos(np.clip(pts[i] @ c / (np.linalg.norm(pts[i]) * np.linalg.norm(c)), -1, 1)) for c in cb]
        assert idx[i] == int(np.argmin(ang))


def test_cosine_assignment_ignores_codeword_lengths():
    # rescaling codewords by positive factors changes the nearest codeword but not
    # the cosine choice
    rng = np.random.default_rng(32)
    pts = np.abs(rng.standard_normal((500, 8)))
    cb = np.abs(rng.standard_normal((256, 8)))
    a, _ = orc.cosine_codeword(pts, cb)
    b, _ = orc.cosine_codeword(pts, cb * rng.uniform(0.1, 10.0, (256, 1)))
    assert np.array_equal(a, b)
    near, _ = orc.nearest_codeword(pts, cb * rng.uniform(0.1, 10.0, (256, 1)))
    assert (near != a).any()


def test_cosine_equals_nearest_for_unit_vectors():
    # for unit points and unit codewords ||p - c||^2 = 2 - 2 cos: the same choice
    rng = np.random.default_rng(33)
    pts = rng.standard_normal((400, 8))
    pts /= np.linalg.norm(pts, axis=1, keepdims=True)
    cb = rng.standard_normal((256, 8))
    cb /= np.linalg.norm(cb, axis=1, keepdims=True)
    assert np.array_equal(orc.cosine_codeword(pts, cb)[0], orc.nearest_codeword(pts, cb)[0])


def test_cosine_hand_case_and_ties():
    cb = np.array([[1.0, 0.0], [10.0, 1.0], [0.0, 0.0], [2.0, 0.0]])
    # (3, 0.2) is nearest to (2, 0) but closest in angle to (10, 1)
    idx, _ = orc.cosine_codeword(np.array([[3.0, 0.2]]), cb)
    assert idx[0] == 1
    assert orc.nearest_codeword(np.array([[3.0, 0.2]]), cb)[0][0] == 3
    # (1, 0): codewords 0 and 3 have the same direction -> the lower index, gap 0
    idx, gap = orc.cosine_codeword(np.array([[1.0, 0.0]]), cb)
    assert idx[0] == 0 and gap[0] == 0.0


def test_cosine_assign_2bit_uses_abs_and_signs():
    rng = np.random.default_rng(34)
    u = rng.standard_normal((50, 8))
    A = np.abs(rng.standard_normal((256, 8)))
    codes, signs, _ = orc.assign(u, A, orc.MODE_2BIT, cosine=True)
    assert np.array_equal(codes, orc.cosine_codeword(np.abs(u), A)[0])
    c1, s1, _ = orc.assign(u, A, orc.MODE_2BIT)
    assert np.array_equal(signs, s1)
