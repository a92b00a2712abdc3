"""Plain fp64 CPU oracle of the NSNQuant KV-cache hot path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product (the CUDA library and its
Python binding) imports, links or executes this module; only the tests, the
smoke check and the bench's CPU-baseline leg call it.  It shares no code with
the CUDA path.  It is written to be read against the method's description, not
to be fast: explicit Hadamard matrix, NSN in fp64, exhaustive nearest-codeword
search, fp64 softmax attention.

Sources (titles and sections of the pages that describe the method):
  [TS]  "NSNQuant: A Double Normalization Approach for Calibration-Free Low-Bit
        Vector Quantization of KV Cache", technical summary (gist.science, es/de):
          - Metodologia 1 "Normalizar-Desplazar-Normalizar (NSN)"
          - Metodologia 2 "Transformada de Hadamard"
          - Metodologia 3 "Cuantizacion Vectorial y Codebook" (codebook,
            adaptive scale adjustment)
          - Metodologia 4 "Detalles de Implementacion" (KIVI-style residual,
            attention scores that fold in s1, s2, o)
  [GH]  "NSNQuant" repository README (DHdroid/NSNQuant): Overview;
        "Codebook tuning" (--abs 2-bit codebook, 1-bit codebook).
  [NW]  "New Quantization Technique Cuts LLM Memory Use Without Training Data",
        section "How NSNQuant Works" (the three NSN steps).

Readings where the pages are silent:
  * Hadamard is applied to every token before NSN (plain Sylvester matrix in
    natural order, no random signs).  NSN commutes with any per-token
    orthogonal map, so the order only moves o into the rotated domain.
  * The channel mean of the shift step is taken over the tokens of one
    quantization block (128 tokens) of one (batch, kv-head).
  * Nearest codeword = smallest squared Euclidean distance; ties go to the
    lowest index.  2-bit mode: sign bit i = (u_i < 0), code over |u|.
  * Cosine assignment (optional variant): the codeword of largest cosine
    similarity p . c / ||c||, ties to the lowest index.
  * Adaptive scale: alpha = ||u||^2 / (u . u_hat) per token (alpha = 1 when
    u . u_hat <= 0), folded into the stored s2.
  * Stored s1, s2*alpha and o are rounded to fp16 (round-to-nearest-even).
  * Degenerate norms: s1 = 0 gives n1 = 0; s2 = 0 gives u = 0.
  * Double quantization (optional): s1 and o stored in 4 bits, 16 uniform
    levels between the fp16-rounded group min and max (`dq4`).
  * Pre-RoPE keys (optional): rotate-half pairing (i, i + d/2), angle
    pos * theta_i, key position = index in the sequence (`apply_rope`).

Parity pins: every function here is pinned in tests/test_oracle_*.py against
closed forms, a hand-derived worked example (tests/golden/), library routines
(scipy's Sylvester Hadamard, scipy cdist) or brute force on tiny inputs.
"""
from __future__ import annotations

import numpy as np

# 1-bit and 2-bit storage modes (an 8-bit code per 8-dim sub-vector; 2-bit adds
# 8 sign bits per sub-vector) -- [GH] "Codebook tuning".
MODE_1BIT = 1
MODE_2BIT = 2


# ---------------------------------------------------------------------------
# Hadamard transform -- [TS] Metodologia 2
# ---------------------------------------------------------------------------
def hadamard_matrix(d: int) -> np.ndarray:
    """Orthonormal Sylvester Hadamard matrix, natural order.

    H[i, j] = (-1)^popcount(i & j) / sqrt(d).  Symmetric, H @ H = I.
    """
    if d <= 0 or d & (d - 1):
        raise ValueError("d must be a power of two")
    i = np.arange(d)[:, None]
    j = np.arange(d)[None, :]
    bits = i & j
    parity = np.zeros_like(bits)
    while np.any(bits):
        parity ^= bits & 1
        bits = bits >> 1
    return np.where(parity == 1, -1.0, 1.0) / np.sqrt(d)


def rotate(x: np.ndarray) -> np.ndarray:
    """y = H x for every row x (one row per token)."""
    x = np.asarray(x, dtype=np.float64)
    return x @ hadamard_matrix(x.shape[-1]).T


# ---------------------------------------------------------------------------
# Normalize-Shift-Normalize -- [TS] Metodologia 1, [NW] "How NSNQuant Works"
# ---------------------------------------------------------------------------
def nsn(y: np.ndarray):
    """NSN of one block of rotated tokens y [n, d] (fp64).

    Step 1 (token-wise normalize): s1 = ||y_t|| / sqrt(d), n1_t = y_t / s1.
    Step 2 (channel-wise shift):   o = mean_t n1_t, z_t = n1_t - o.
    Step 3 (token-wise normalize): s2 = ||z_t|| / sqrt(d), u_t = z_t / s2.
    Returns (u [n, d], s1 [n], o [d], s2 [n]); y_t = (u_t s2 + o) s1.
    """
    y = np.asarray(y, dtype=np.float64)
    n, d = y.shape
    if n == 0:
        raise ValueError("empty block")
    root_d = np.sqrt(d)
    s1 = np.sqrt(np.sum(y * y, axis=1)) / root_d
    n1 = np.zeros_like(y)
    nz = s1 > 0
    n1[nz] = y[nz] / s1[nz, None]
    o = np.sum(n1, axis=0) / n
    z = n1 - o[None, :]
    s2 = np.sqrt(np.sum(z * z, axis=1)) / root_d
    u = np.zeros_like(z)
    nz2 = s2 > 0
    u[nz2] = z[nz2] / s2[nz2, None]
    return u, s1, o, s2


# ---------------------------------------------------------------------------
# Vector quantization -- [TS] Metodologia 3, [GH] "Codebook tuning"
# ---------------------------------------------------------------------------
def squared_distances(points: np.ndarray, codebook: np.ndarray) -> np.ndarray:
    """D[m, k] = sum_i (points[m, i] - codebook[k, i])^2, fp64, written out."""
    points = np.asarray(points, dtype=np.float64)
    codebook = np.asarray(codebook, dtype=np.float64)
    out = np.empty((points.shape[0], codebook.shape[0]))
    step = 4096
    for a in range(0, points.shape[0], step):
        diff = points[a:a + step, None, :] - codebook[None, :, :]
        out[a:a + step] = np.sum(diff * diff, axis=2)
    return out


def nearest_codeword(points: np.ndarray, codebook: np.ndarray):
    """Exhaustive nearest codeword, ties to the lowest index.

    Returns (index [m], relative top-2 gap [m]) where the gap is
    (d_second - d_best) / d_second (0 when d_second is 0).  Callers use the
    gap to recognise near-ties.
    """
    dist = squared_distances(points, codebook)
    idx = np.argmin(dist, axis=1)  # first occurrence = lowest index
    srt = np.sort(dist, axis=1)
    d1, d2 = srt[:, 0], srt[:, 1]
    gap = np.where(d2 > 0, (d2 - d1) / np.where(d2 > 0, d2, 1.0), 0.0)
    return idx, gap


def cosine_codeword(points: np.ndarray, codebook: np.ndarray):
    """Codeword of largest cosine similarity, ties to the lowest index.

    The cosine-assignment variant of the codebook tuning ([TS] Metodologia 3: the
    codebook is fine-tuned for the cosine distance between a vector and its
    quantized version): code = argmax_k p . c_k / ||c_k|| (the factor 1/||p|| is the
    same for every k; a zero codeword scores 0).  The gap is defined as for the
    nearest codeword on the distances d_k = ||p|| - p . c_k / ||c_k||
    (= ||p|| (1 - cos)).  Returns (index [m], relative top-2 gap [m]).
    """
    points = np.asarray(points, dtype=np.float64)
    codebook = np.asarray(codebook, dtype=np.float64)
    norms = np.sqrt(np.sum(codebook * codebook, axis=1))
    inv = np.where(norms > 0, 1.0 / np.where(norms > 0, norms, 1.0), 0.0)
    score = (points @ codebook.T) * inv[None, :]
    dist = np.sqrt(np.sum(points * points, axis=1))[:, None] - score
    idx = np.argmin(dist, axis=1)
    srt = np.sort(dist, axis=1)
    d1, d2 = srt[:, 0], srt[:, 1]
    gap = np.where(d2 > 0, (d2 - d1) / np.where(d2 > 0, d2, 1.0), 0.0)
    return idx, gap


def assign(u_sub: np.ndarray, codebook: np.ndarray, mode: int, cosine: bool = False):
    """Code (and sign bits) of every sub-vector u_sub [m, m_dim].

    1-bit: code = argmin_k ||u_s - C_k||^2.
    2-bit: sign bit i = 1 iff u_i < 0; code = argmin_k || |u_s| - A_k ||^2
           over the absolute-value codebook A (entries >= 0).
    cosine: the same with the codeword of largest cosine similarity instead of
           the nearest one (`cosine_codeword`).
    Returns (codes [m] int, signs [m] uint8 bit-packed or None, gap [m]).
    """
    u_sub = np.asarray(u_sub, dtype=np.float64)
    pick = cosine_codeword if cosine else nearest_codeword
    if mode == MODE_1BIT:
        codes, gap = pick(u_sub, codebook)
        return codes, None, gap
    if mode == MODE_2BIT:
        neg = u_sub < 0
        codes, gap = pick(np.abs(u_sub), codebook)
        weights = (1 << np.arange(u_sub.shape[1])).astype(np.int64)
        signs = (neg.astype(np.int64) * weights[None, :]).sum(axis=1)
        return codes, signs.astype(np.uint8), gap
    raise ValueError("mode must be 1 or 2")


def reconstruct_sub(codes, signs, codebook, mode):
    """u_hat sub-vectors [m, m_dim]: C_code (1-bit) or (+-1) * A_code (2-bit)."""
    cb = np.asarray(codebook, dtype=np.float64)
    v = cb[np.asarray(codes)]
    if mode == MODE_2BIT:
        bits = (np.asarray(signs, dtype=np.int64)[:, None] >> np.arange(cb.shape[1])[None, :]) & 1
        v = np.where(bits == 1, -v, v)
    return v


def scale_factor(u: np.ndarray, u_hat: np.ndarray) -> np.ndarray:
    """Adaptive scale per token: alpha = ||u||^2 / (u . u_hat).

    Makes the component of alpha*u_hat along u equal to u ([TS] Metodologia 3,
    scale adjustment).  alpha = 1 where u . u_hat <= 0 (reading; includes u = 0).
    """
    dot = np.sum(u * u_hat, axis=1)
    uu = np.sum(u * u, axis=1)
    return np.where(dot > 0, uu / np.where(dot > 0, dot, 1.0), 1.0)


def to_f16(x) -> np.ndarray:
    """Round to fp16 (round-to-nearest-even) and return as fp64."""
    return np.asarray(x, dtype=np.float64).astype(np.float16).astype(np.float64)


def dq4(x) -> dict:
    """4-bit quantization of one group of stored scalars (double quantization,
    [TS] Metodologia 3: the NSN byproducts o and s1 are stored in 4 bits).

    Reading (the pages give only the bit width): 16 uniform levels between
    lo = fp16(min x) and hi = fp16(max x); step = (hi - lo) / 15;
    level = clip(round-half-even((x - lo) / step), 0, 15) (step = 0 gives level 0);
    value = lo + level * step.  Returns levels (int), lo, hi (fp64 holding fp16
    values) and the dequantized values.
    """
    x = np.asarray(x, dtype=np.float64)
    lo = float(to_f16(x.min()))
    hi = float(to_f16(x.max()))
    step = (hi - lo) / 15.0
    if step > 0.0:
        levels = np.clip(np.rint((x - lo) / step), 0, 15).astype(np.int64)
    else:
        levels = np.zeros(x.shape, dtype=np.int64)
    return {"levels": levels, "lo": lo, "hi": hi, "values": lo + levels * step}


def quantize_block(x: np.ndarray, codebook: np.ndarray, mode: int,
                   sub_dim: int = 8, scale_adjust: bool = True, double_quant: bool = False,
                   cosine: bool = False) -> dict:
    """Quantize one block of raw tokens x [n, d] (one batch row, one kv-head).

    Hadamard -> NSN -> per-sub-vector nearest codeword -> adaptive scale ->
    fp16 rounding of the stored scalars.  Returns a dict with
      codes [n, d/sub_dim] int, signs [n, d/sub_dim] uint8 (2-bit) or None,
      s1 [n], s2 [n] (= alpha * s2, fp16-rounded), o [d] (fp16-rounded),
      gap [n, d/sub_dim] (relative top-2 distance gap of each assignment),
      u [n, d] (fp64 NSN output, for diagnostics).
    With double_quant, s1 and o are stored in 4 bits instead (`dq4` over the
    block's tokens and over its 128 channels); "s1" and "o" then hold the
    dequantized values and "s1_dq" / "o_dq" the levels and (lo, hi).  The NSN,
    the assignment and alpha use the exact values either way.  With cosine the
    codes are the codewords of largest cosine similarity (`cosine_codeword`).
    """
    x = np.asarray(x, dtype=np.float64)
    n, d = x.shape
    nsub = d // sub_dim
    y = rotate(x)
    u, s1, o, s2 = nsn(y)
    codes, signs, gap = assign(u.reshape(n * nsub, sub_dim), codebook, mode, cosine=cosine)
    u_hat = reconstruct_sub(codes, signs, codebook, mode).reshape(n, d)
    alpha = scale_factor(u, u_hat) if scale_adjust else np.ones(n)
    out = {
        "codes": codes.reshape(n, nsub),
        "signs": None if signs is None else signs.reshape(n, nsub),
        "s1": to_f16(s1),
        "s2": to_f16(alpha * s2),
        "o": to_f16(o),
        "gap": gap.reshape(n, nsub),
        "u": u,
    }
    if double_quant:
        q1, qo = dq4(s1), dq4(o)
        out.update(s1=q1["values"], o=qo["values"], s1_dq=q1, o_dq=qo)
    return out


def prefill_split(n_tokens: int, block: int, window: int) -> int:
    """Number of tokens that go to the quantized part on prefill.

    KIVI-style residual ([TS] Metodologia 4): with a residual window the
    quantized part holds whole blocks and the window keeps the 1..window most
    recent tokens, Q = block * floor((L - 1) / block).  Without a window every
    token is quantized (the last block may be partial).
    """
    if n_tokens <= 0:
        return 0
    if window == 0:
        return n_tokens
    return block * ((n_tokens - 1) // block)


def quantize_sequence(x: np.ndarray, codebook: np.ndarray, mode: int,
                      block: int = 128, window: int = 128,
                      scale_adjust: bool = True, double_quant: bool = False, cosine: bool = False) -> dict:
    """Prefill of one (batch, kv-head) sequence x [L, d].

    Returns codes/signs/s1/s2 per quantized token, o per block, the fp16
    residual window, and the gaps.  Blocks are independent (the mean of the
    shift step is per block).
    """
    x = np.asarray(x, dtype=np.float64)
    L, d = x.shape
    q = prefill_split(L, block, window)
    parts = [quantize_block(x[a:min(a + block, q)], codebook, mode,
                            scale_adjust=scale_adjust, double_quant=double_quant, cosine=cosine)
             for a in range(0, q, block)]
    nsub = d // 8

    def cat(key, shape):
        if not parts:
            return np.zeros(shape)
        return np.concatenate([p[key] for p in parts], axis=0)

    return {
        "n_quant": q,
        "codes": cat("codes", (0, nsub)).astype(np.int64),
        "signs": None if mode == MODE_1BIT else cat("signs", (0, nsub)).astype(np.uint8),
        "s1": cat("s1", (0,)),
        "s2": cat("s2", (0,)),
        "o": np.stack([p["o"] for p in parts]) if parts else np.zeros((0, d)),
        "gap": cat("gap", (0, nsub)),
        "u": cat("u", (0, d)),
        "window": to_f16(x[q:]),
        "s1_dq": [p["s1_dq"] for p in parts] if double_quant else None,
        "o_dq": [p["o_dq"] for p in parts] if double_quant else None,
    }


# ---------------------------------------------------------------------------
# Dequantization and attention -- [TS] Metodologia 4 (scores with s1, s2, o)
# ---------------------------------------------------------------------------
def dequantize(codes, signs, s1, s2, o_blocks, codebook, mode, block=128):
    """Reconstructed tokens in the ORIGINAL domain.

    x_hat_t = H^T ((u_hat_t s2_t + o_b) s1_t), b = t // block, from the stored
    (fp16) scalars and the codebook as given.
    """
    codes = np.asarray(codes)
    n, nsub = codes.shape
    if n == 0:
        return np.zeros((0, np.asarray(o_blocks).shape[-1]))
    cb = np.asarray(codebook, dtype=np.float64)
    sub = cb.shape[1]
    flat_signs = None if signs is None else np.asarray(signs).reshape(-1)
    u_hat = reconstruct_sub(codes.reshape(-1), flat_signs, cb, mode).reshape(n, nsub * sub)
    o = np.asarray(o_blocks, dtype=np.float64)[np.arange(n) // block]
    rot = (u_hat * np.asarray(s2, dtype=np.float64)[:, None] + o) * np.asarray(s1, dtype=np.float64)[:, None]
    return rot @ hadamard_matrix(nsub * sub)  # H^T = H


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """softmax(q k^T * scale) v for q [g, d], k [n, d], v [n, d]; fp64."""
    s = (np.asarray(q, np.float64) @ np.asarray(k, np.float64).T) * scale
    s = s - s.max(axis=1, keepdims=True)
    p = np.exp(s)
    p /= p.sum(axis=1, keepdims=True)
    return p @ np.asarray(v, np.float64)


def decode_attention(q_group: np.ndarray, kq: dict, vq: dict, k_window: np.ndarray,
                     v_window: np.ndarray, codebook_k, codebook_v, mode_k: int,
                     mode_v: int, scale: float, block: int = 128) -> np.ndarray:
    """Decode attention for the g query heads that share one kv-head.

    Keys/values = dequantized tokens followed by the fp16 residual window.
    kq / vq hold codes, signs, s1, s2, o of the quantized part.
    """
    k_hat = dequantize(kq["codes"], kq["signs"], kq["s1"], kq["s2"], kq["o"],
                       codebook_k, mode_k, block)
    v_hat = dequantize(vq["codes"], vq["signs"], vq["s1"], vq["s2"], vq["o"],
                       codebook_v, mode_v, block)
    keys = np.concatenate([k_hat, np.asarray(k_window, np.float64)], axis=0)
    vals = np.concatenate([v_hat, np.asarray(v_window, np.float64)], axis=0)
    if keys.shape[0] == 0:
        raise ValueError("attention over zero tokens")
    return attention(q_group, keys, vals, scale)


def extend_attention(q_chunk: np.ndarray, kq: dict, vq: dict, k_window: np.ndarray,
                     v_window: np.ndarray, codebook_k, codebook_v, mode_k: int,
                     mode_v: int, scale: float, block: int = 128) -> np.ndarray:
    """Chunked-prefill attention of the last C tokens of one sequence, which all
    sit in the residual window ([TS] Metodologia 4: quantized part + residual).

    q_chunk [C, g, d]: query i (the token at window slot n_window - C + i) attends
    every dequantized token and the window slots 0 .. n_window - C + i.  Returns
    [C, g, d]: for each query the decode attention over that causal prefix.
    """
    q_chunk = np.asarray(q_chunk, dtype=np.float64)
    C, nw = q_chunk.shape[0], np.asarray(k_window).shape[0]
    if C > nw:
        raise ValueError("every query of the chunk must be a window token")
    return np.stack([decode_attention(q_chunk[i], kq, vq, k_window[:nw - C + 1 + i], v_window[:nw - C + 1 + i],
                                      codebook_k, codebook_v, mode_k, mode_v, scale, block) for i in range(C)])


# ---------------------------------------------------------------------------
# Rotary position embedding of the keys -- [TS] Metodologia 4: NSN is applied to
# the keys BEFORE the rotary position embedding, so the cache holds pre-RoPE keys
# and attention rotates each dequantized key at its own position.
# Readings (the pages name RoPE only): the Llama "rotate-half" pairing, dim i with
# dim i + d/2 at angle pos * theta_i; theta_i = base^(-2i/d) for the standard
# table; the position of a cached key is its index in the sequence (quantized
# tokens first, then the window); the query arrives already rotated.
# ---------------------------------------------------------------------------
def rope_inv_freq(d: int, base: float) -> np.ndarray:
    """theta_i = base^(-2i/d), i < d/2 (fp64)."""
    i = np.arange(d // 2, dtype=np.float64)
    return np.power(float(base), -2.0 * i / d)


def apply_rope(x: np.ndarray, positions, inv_freq) -> np.ndarray:
    """Rows x [n, d] rotated at their positions [n] (rotate-half pairing).

    For i < d/2, angle a = pos * theta_i:
      out[i]       = x[i] cos a - x[i + d/2] sin a
      out[i + d/2] = x[i + d/2] cos a + x[i] sin a
    """
    x = np.asarray(x, dtype=np.float64)
    n, d = x.shape
    half = d // 2
    theta = np.asarray(inv_freq, dtype=np.float64)
    if theta.shape != (half,):
        raise ValueError("inv_freq must hold d/2 frequencies")
    ang = np.asarray(positions, dtype=np.float64)[:, None] * theta[None, :]
    c, s = np.cos(ang), np.sin(ang)
    lo, hi = x[:, :half], x[:, half:]
    return np.concatenate([lo * c - hi * s, hi * c + lo * s], axis=1)


def decode_attention_rope(q_group: np.ndarray, kq: dict, vq: dict, k_window: np.ndarray,
                          v_window: np.ndarray, codebook_k, codebook_v, mode_k: int,
                          mode_v: int, scale: float, inv_freq, block: int = 128) -> np.ndarray:
    """Decode attention over pre-RoPE keys ([TS] Metodologia 4).

    Every key -- dequantized tokens at positions 0 .. n_quant-1, then the window
    at n_quant .. -- is rotated at its position before the scores; q_group is
    the already-rotated query.  Values are not rotated.
    """
    k_hat = dequantize(kq["codes"], kq["signs"], kq["s1"], kq["s2"], kq["o"],
                       codebook_k, mode_k, block)
    v_hat = dequantize(vq["codes"], vq["signs"], vq["s1"], vq["s2"], vq["o"],
                       codebook_v, mode_v, block)
    keys = np.concatenate([k_hat, np.asarray(k_window, np.float64)], axis=0)
    vals = np.concatenate([v_hat, np.asarray(v_window, np.float64)], axis=0)
    if keys.shape[0] == 0:
        raise ValueError("attention over zero tokens")
    keys = apply_rope(keys, np.arange(keys.shape[0]), inv_freq)
    return attention(q_group, keys, vals, scale)


def nsn_score_terms(q: np.ndarray, u_hat: np.ndarray, s1, s2, o: np.ndarray) -> np.ndarray:
    """Scores q . x_hat_t written with the NSN byproducts folded in.

    q . H^T((u_hat s2 + o) s1) = s1 (s2 (Hq) . u_hat + (Hq) . o), the form the
    attention kernels use ([TS] Metodologia 4).  Returned for one block
    (one o).  Used only to pin the decomposition against explicit attention.
    """
    qt = rotate(np.atleast_2d(q))
    return np.asarray(s1)[None, :] * (np.asarray(s2)[None, :] * (qt @ u_hat.T) + (qt @ o)[:, None])
