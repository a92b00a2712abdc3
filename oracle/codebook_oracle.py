"""Plain CPU oracle of the codebook construction.  TEST INFRASTRUCTURE ONLY.

The pages build the single global codebook by k-means on synthetic standard
normal samples (torch.randn) -- "NSNQuant ... technical summary", Metodologia 3
"Codebook: construccion" -- and the 2-bit variant on absolute values
("NSNQuant" README, "Codebook tuning": ``--abs``).  The same passage then
fine-tunes the codebook to minimise the cosine distance between vectors and
their quantized versions (README: ``--method learned``); `cosine_finetune`
restates the reading of that step given below.

The seeded standard-normal samples come from a counter-based generator that
each side implements from its published definition:
  * Philox4x64-10: J. Salmon, M. Moraes, R. Dror, D. Shaw, "Parallel Random
    Numbers: As Easy as 1, 2, 3", SC'11 (round function, multipliers and Weyl
    key increments as defined there).
  * Box-Muller: G. Box, M. Muller, "A Note on the Generation of Random Normal
    Deviates", Ann. Math. Statist. 29 (1958).
Stream layout (a reading; documented in the C header as well): key =
(seed, 0x4E534E51), counter = (j, 0, 0, 0) for block j; the block's four
64-bit words w0..w3 become uniforms u = ((w >> 12) + 0.5) * 2^-52 and the pairs
(u0, u1), (u2, u3) give normals (r cos(2 pi u_b), r sin(2 pi u_b)) with
r = sqrt(-2 ln u_a).  Normal number i*dim + c is component c of sample i.

k-means (a reading of "K-Means on randn"): Lloyd iterations, initial centroids =
the first K samples, nearest centroid by squared Euclidean distance with ties to
the lowest index, empty clusters keep their centroid, a fixed iteration count;
the result is rounded to fp16-representable values so that the fp32 quantizer
and the fp16 decode read identical codewords.

Cosine fine-tuning (a reading; the pages give no procedure): alternate
(1) nearest-codeword assignment as above and (2) for every codeword with
members, the direction maximising the summed cosine with its members (the
normalised sum of their unit vectors) with the least-squares length along it
(the members' mean projection); a codeword with no members, a zero direction
sum or a non-positive mean projection is kept.

Pinned by tests/test_oracle_codebook.py against numpy's own Philox bit
generator, the moments and a Kolmogorov-Smirnov test of the normal stream, scipy's
Lloyd iteration (kmeans2 from the same initial centroids) and k-means fixed-point
properties.
"""
from __future__ import annotations

import math

import numpy as np

_MASK64 = (1 << 64) - 1
PHILOX_M0 = 0xD2E7470EE14C6C93
PHILOX_M1 = 0xCA5A826395121157
PHILOX_W0 = 0x9E3779B97F4A7C15
PHILOX_W1 = 0xBB67AE8584CAA73B
STREAM_KEY1 = 0x4E534E51


def philox4x64_10(counter, key):
    """One Philox4x64 block with 10 rounds (python ints, exact)."""
    x0, x1, x2, x3 = (int(c) & _MASK64 for c in counter)
    k0, k1 = (int(k) & _MASK64 for k in key)
    for _ in range(10):
        p0 = PHILOX_M0 * x0
        p1 = PHILOX_M1 * x2
        hi0, lo0 = p0 >> 64, p0 & _MASK64
        hi1, lo1 = p1 >> 64, p1 & _MASK64
        x0, x1, x2, x3 = (hi1 ^ x1 ^ k0), lo1, (hi0 ^ x3 ^ k1), lo0
        k0 = (k0 + PHILOX_W0) & _MASK64
        k1 = (k1 + PHILOX_W1) & _MASK64
    return x0, x1, x2, x3


def uniform_open(word: int) -> float:
    """Map a 64-bit word to a double in the open interval (0, 1).

    The top 52 bits plus one half, times 2^-52: exact, in [2^-53, 1 - 2^-53].
    """
    return ((word >> 12) + 0.5) * (2.0 ** -52)


def normal_stream(seed: int, count: int) -> np.ndarray:
    """The first `count` standard normals of the stream for `seed`."""
    out = np.empty(count)
    key = (seed & _MASK64, STREAM_KEY1)
    nblocks = (count + 3) // 4
    for j in range(nblocks):
        w = philox4x64_10((j, 0, 0, 0), key)
        u = [uniform_open(x) for x in w]
        zs = []
        for a, b in ((u[0], u[1]), (u[2], u[3])):
            r = math.sqrt(-2.0 * math.log(a))
            zs.append(r * math.cos(2.0 * math.pi * b))
            zs.append(r * math.sin(2.0 * math.pi * b))
        for t in range(4):
            i = 4 * j + t
            if i < count:
                out[i] = zs[t]
    return out


def normal_samples(seed: int, n_samples: int, dim: int, abs_mode: bool) -> np.ndarray:
    """[n_samples, dim] standard normals (absolute values in abs mode)."""
    z = normal_stream(seed, n_samples * dim).reshape(n_samples, dim)
    return np.abs(z) if abs_mode else z


def kmeans(samples: np.ndarray, n_codes: int, iters: int) -> np.ndarray:
    """Lloyd's k-means in fp64 (see module docstring for the readings)."""
    x = np.asarray(samples, dtype=np.float64)
    if x.shape[0] < n_codes:
        raise ValueError("need at least n_codes samples")
    cent = x[:n_codes].copy()
    for _ in range(iters):
        diff_sq = np.empty((x.shape[0], n_codes))
        for a in range(0, x.shape[0], 4096):
            diff = x[a:a + 4096, None, :] - cent[None, :, :]
            diff_sq[a:a + 4096] = np.sum(diff * diff, axis=2)
        label = np.argmin(diff_sq, axis=1)
        for k in range(n_codes):
            members = x[label == k]
            if members.shape[0] > 0:
                cent[k] = members.sum(axis=0) / members.shape[0]
    return cent


def nearest(x: np.ndarray, cent: np.ndarray) -> np.ndarray:
    """Index of the nearest centroid (squared Euclidean, lowest index on ties)."""
    diff_sq = np.empty((x.shape[0], cent.shape[0]))
    for a in range(0, x.shape[0], 4096):
        diff = x[a:a + 4096, None, :] - cent[None, :, :]
        diff_sq[a:a + 4096] = np.sum(diff * diff, axis=2)
    return np.argmin(diff_sq, axis=1)


def cosine_step(x: np.ndarray, cent: np.ndarray, label: np.ndarray) -> np.ndarray:
    """One cosine update of the centroids for fixed assignments `label`."""
    x = np.asarray(x, dtype=np.float64)
    new = np.array(cent, dtype=np.float64, copy=True)
    norms = np.sqrt(np.sum(x * x, axis=1))
    unit = np.divide(x, norms[:, None], out=np.zeros_like(x), where=norms[:, None] > 0)
    for k in range(cent.shape[0]):
        members = label == k
        if not members.any():
            continue
        direction = unit[members].sum(axis=0)
        length = math.sqrt(float(np.sum(direction * direction)))
        if length == 0.0:
            continue
        direction = direction / length
        proj = float(np.mean(x[members] @ direction))
        if proj > 0.0:
            new[k] = direction * proj
    return new


def cosine_finetune(samples: np.ndarray, cent: np.ndarray, iters: int) -> np.ndarray:
    """Alternating nearest assignment and cosine update, `iters` times."""
    x = np.asarray(samples, dtype=np.float64)
    c = np.array(cent, dtype=np.float64, copy=True)
    for _ in range(iters):
        c = cosine_step(x, c, nearest(x, c))
    return c


def cosine_distance(x: np.ndarray, cent: np.ndarray) -> float:
    """Mean 1 - cos(x, nearest codeword) over the samples (zero rows count 1)."""
    x = np.asarray(x, dtype=np.float64)
    q = cent[nearest(x, cent)]
    num = np.sum(x * q, axis=1)
    den = np.sqrt(np.sum(x * x, axis=1) * np.sum(q * q, axis=1))
    cos = np.divide(num, den, out=np.zeros_like(num), where=den > 0)
    return float(np.mean(1.0 - cos))


def build_codebook_cosine(seed: int, n_samples: int, n_codes: int, dim: int, abs_mode: bool,
                          kmeans_iters: int, cosine_iters: int) -> np.ndarray:
    """k-means codebook fine-tuned for cosine distance, as fp16-representable values (fp64)."""
    x = normal_samples(seed, n_samples, dim, abs_mode)
    cent = cosine_finetune(x, kmeans(x, n_codes, kmeans_iters), cosine_iters)
    return cent.astype(np.float16).astype(np.float64)


def build_codebook(seed: int, n_samples: int, n_codes: int, dim: int,
                   abs_mode: bool, iters: int) -> np.ndarray:
    """Codebook [n_codes, dim] as fp16-representable values (returned fp64)."""
    cent = kmeans(normal_samples(seed, n_samples, dim, abs_mode), n_codes, iters)
    return cent.astype(np.float16).astype(np.float64)


def codebook_4bit(codebook: np.ndarray) -> np.ndarray:
    """Codebook entries on 16 uniform levels between the fp16-rounded min and max
    of all entries (double quantization of the codebook, [TS] Metodologia 3), each
    rounded to fp16.  Same level rule as the stored scalars: round half to even,
    clamped to 0..15."""
    cb = np.asarray(codebook, dtype=np.float64)
    flat = cb.reshape(-1)
    lo = float(np.float16(flat.min()))
    hi = float(np.float16(flat.max()))
    step = (hi - lo) / 15.0
    levels = np.clip(np.rint((flat - lo) / step), 0, 15) if step > 0 else np.zeros_like(flat)
    return (lo + levels * step).astype(np.float16).astype(np.float64).reshape(cb.shape)
