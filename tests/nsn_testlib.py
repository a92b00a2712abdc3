"""Glue for the parity tests: codebook fixtures, reading a compressed cache back
into the oracle's dict layout, and the comparison rules with their tolerances.

Tolerances (the method's parity contract):
  * codes and sign bits bit-exact, except assignments whose oracle top-2 distance
    gap is <= 1e-6 relative (near-ties), which are counted and reported, and
    tokens whose stored s2 is 0 on both sides (codes unused); a sign
    bit may differ only where the oracle's |u_i| <= 1e-6 * ||u_sub|| (its fp64
    sign is then decided below fp32 resolution), also counted.
  * stored norms s1, s2 within 1e-3 relative; block means within
    1e-3 * max|o| of the block.
  * attention outputs: max|diff| / max|ref| <= 2e-3 per (batch, q-head).
"""
from __future__ import annotations

import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
NEAR_TIE = 1e-6
NORM_RTOL = 1e-3
MEAN_RTOL = 1e-3
ATTN_TOL = 2e-3


def codebook(mode: int) -> np.ndarray:
    """Oracle-built fixture codebook [256, 8] (fp16-representable values)."""
    name = "codebook_1bit.txt" if mode == 1 else "codebook_2bit.txt"
    return np.loadtxt(os.path.join(GOLDEN, name)).astype(np.float32)


def codes_to_natural(stored: np.ndarray) -> np.ndarray:
    """Stored code records [..., 16] (the even sub-vectors' codes, then the odd
    ones') -> the oracle's layout [..., 16] (byte s = code of sub-vector s)."""
    stored = np.asarray(stored)
    out = np.empty_like(stored)
    out[..., 0::2] = stored[..., :8]
    out[..., 1::2] = stored[..., 8:]
    return out


def natural_to_codes(natural: np.ndarray) -> np.ndarray:
    """Inverse of codes_to_natural."""
    natural = np.asarray(natural)
    return np.concatenate([natural[..., 0::2], natural[..., 1::2]], axis=-1)


def signs_to_natural(stored: np.ndarray) -> np.ndarray:
    """Stored sign bytes [..., 16] (eight 16-bit fields; field i bit 15-s = sign of
    dim 8s+i) -> the oracle's layout [..., 16] (byte s bit i = sign of dim 8s+i)."""
    stored = np.asarray(stored, dtype=np.uint8)
    fields = stored.reshape(stored.shape[:-1] + (8, 2)).astype(np.uint32)
    fields = fields[..., 0] | (fields[..., 1] << 8)                     # [..., 8] field i
    out = np.zeros(stored.shape, dtype=np.uint8)
    for s in range(16):
        for i in range(8):
            bit = (fields[..., i] >> (15 - s)) & 1
            out[..., s] |= (bit << i).astype(np.uint8)
    return out


def natural_to_signs(natural: np.ndarray) -> np.ndarray:
    """Inverse of signs_to_natural."""
    natural = np.asarray(natural, dtype=np.uint8)
    fields = np.zeros(natural.shape[:-1] + (8,), dtype=np.uint32)
    for s in range(16):
        for i in range(8):
            bit = (natural[..., s].astype(np.uint32) >> i) & 1
            fields[..., i] |= bit << (15 - s)
    out = np.zeros(natural.shape, dtype=np.uint8)
    out[..., 0::2] = (fields & 0xFF).astype(np.uint8)
    out[..., 1::2] = (fields >> 8).astype(np.uint8)
    return out


def unpack_levels(packed: np.ndarray) -> np.ndarray:
    """Two 4-bit levels per byte (even index in the low nibble) -> one per element."""
    p = np.asarray(packed, dtype=np.uint8)
    return np.stack([p & 15, p >> 4], axis=-1).reshape(*p.shape[:-1], 2 * p.shape[-1]).astype(np.int64)


def read_cache(cache, b: int, h: int) -> dict:
    """Stored contents of one (b, h) sequence of an nsn.Cache as numpy (oracle layout).
    For a double-quantized cache s1 and o are the values read back from the 4-bit
    levels (lo + level * (hi - lo) / 15 in fp64), and the raw levels and (lo, hi)
    pairs are returned as well."""
    nq = int(cache.n_quant[b, h].item())
    nw = int(cache.n_window[b, h].item())
    nblk = (nq + 127) // 128
    out = {
        "n_quant": nq,
        "n_window": nw,
        "codes": codes_to_natural(cache.codes[b, h, :nq].cpu().numpy()).astype(np.int64),
        "signs": None if cache.signs is None else signs_to_natural(cache.signs[b, h, :nq].cpu().numpy()),
        "window": (cache.window_buf[b, h, :nw].float().cpu().numpy().astype(np.float64)
                   if cache.window_buf is not None else np.zeros((0, 128))),
    }
    if getattr(cache, "double_quant", False):
        par = cache.dq_params[b, h, :nblk].float().cpu().numpy().astype(np.float64)      # [nblk, 8]
        s1_lev = unpack_levels(cache.s1_levels[b, h].cpu().numpy())[: nblk * 128].reshape(nblk, 128)
        o_lev = unpack_levels(cache.means[b, h, :nblk].cpu().numpy())                   # [nblk, 128]
        s1_step = (par[:, 1] - par[:, 0]) / 15.0
        o_step = (par[:, 3] - par[:, 2]) / 15.0
        out["s1"] = (par[:, 0:1] + s1_lev * s1_step[:, None]).reshape(-1)[:nq]
        out["o"] = par[:, 2:3] + o_lev * o_step[:, None]
        out["s2"] = cache.norms[b, h, :nq].float().cpu().numpy().astype(np.float64)
        out["s1_levels"] = s1_lev.reshape(-1)[:nq]
        out["o_levels"] = o_lev
        out["params"] = par[:, :4]
    else:
        out["s1"] = cache.norms[b, h, :nq, 0].float().cpu().numpy().astype(np.float64)
        out["s2"] = cache.norms[b, h, :nq, 1].float().cpu().numpy().astype(np.float64)
        out["o"] = cache.means[b, h, :nblk].float().cpu().numpy().astype(np.float64)
    return out


def compare_codes(gpu: dict, ref: dict, u_ref: np.ndarray | None = None) -> dict:
    """Codes / signs parity with near-tie accounting.  Raises AssertionError on a
    mismatch that is not a near-tie."""
    gap = ref["gap"]
    mism = gpu["codes"] != ref["codes"]
    near = gap <= NEAR_TIE
    # A token whose stored s2 is 0 on both sides reconstructs to H^T(o s1) whatever
    # its codes are (its u is 0 by definition, but rounding noise of either side can
    # give it any direction): its codes are not compared.
    degenerate = ((np.asarray(gpu["s2"]) == 0) & (np.asarray(ref["s2"]) == 0))[:, None]
    mism = mism & ~degenerate
    bad = mism & ~near
    assert not bad.any(), (
        f"{int(bad.sum())} code mismatches outside the near-tie band; first at "
        f"{np.argwhere(bad)[:5].tolist()} gaps {gap[bad][:5]}")
    res = {"n": int(mism.size), "near_ties": int(near.sum()), "tie_mismatch": int(mism.sum())}
    if ref.get("signs") is not None:
        diff = np.bitwise_xor(gpu["signs"].astype(np.int64), ref["signs"].astype(np.int64))
        diff = np.where(degenerate, 0, diff)
        res["sign_bits_differing"] = int(np.unpackbits(diff.astype(np.uint8)).sum())
        if res["sign_bits_differing"]:
            assert u_ref is not None, "sign bits differ"
            n, nsub = diff.shape
            u = u_ref.reshape(n, nsub, 8)
            bits = (diff[:, :, None] >> np.arange(8)[None, None, :]) & 1
            tiny = np.abs(u) <= 1e-6 * np.linalg.norm(u, axis=2, keepdims=True)
            assert not (bits.astype(bool) & ~tiny).any(), "sign bit differs where the oracle's sign is clear"
    return res


def compare_norms_means(gpu: dict, ref: dict, mismatch_rows=None) -> None:
    for key in ("s1", "s2"):
        g, r = gpu[key], ref[key]
        rel = np.abs(g - r) / np.maximum(np.abs(r), 1e-30)
        ok = (rel <= NORM_RTOL) | ((r == 0) & (g == 0))
        if key == "s2" and mismatch_rows is not None:
            ok |= mismatch_rows   # alpha depends on the (near-tie) code choice
        assert ok.all(), f"{key}: {int((~ok).sum())} tokens beyond {NORM_RTOL} rel, worst {rel.max():.3g}"
    go, ro = gpu["o"], ref["o"]
    scale = np.maximum(np.abs(ro).max(axis=1, keepdims=True), 1e-30)
    err = np.abs(go - ro) / scale
    assert (err <= MEAN_RTOL).all(), f"means: worst {err.max():.3g} of block max"


def attn_error(out: np.ndarray, ref: np.ndarray) -> float:
    """max over rows of max|out - ref| / max|ref| (rows = last axis vectors)."""
    out = out.reshape(-1, out.shape[-1])
    ref = ref.reshape(-1, ref.shape[-1])
    num = np.abs(out - ref).max(axis=1)
    den = np.maximum(np.abs(ref).max(axis=1), 1e-30)
    return float((num / den).max())


# ---------------------------------------------------------------------------
# Oracle pipeline of one (batch, kv-head) sequence, block quantization spread over
# a process pool (the oracle itself is unchanged; blocks are independent).
# ---------------------------------------------------------------------------
def _oracle_block(args):
    from oracle import nsn_oracle as orc
    x, cb, mode = args[:3]
    dq = len(args) > 3 and args[3]
    r = orc.quantize_block(x, cb, mode, double_quant=dq)
    keys = ("codes", "signs", "s1", "s2", "o", "gap", "u") + (("s1_dq", "o_dq") if dq else ())
    return {k: r[k] for k in keys}


def oracle_cache_sequence(pool, x, n_prefill, n_total, cb, mode, window=128, double_quant=False):
    """Oracle cache of one sequence x [T, 128] (fp64) after a prefill of n_prefill
    tokens and appends up to n_total: (quantized dict, fp16 window rows)."""
    from oracle import nsn_oracle as orc
    q = orc.prefill_split(n_prefill, 128, window)
    blocks = [(x[a:min(a + 128, q)], cb, mode, double_quant) for a in range(0, q, 128)]
    parts = list(pool.map(_oracle_block, blocks, chunksize=4)) if blocks else []
    win = list(orc.to_f16(x[q:n_prefill]))
    for t in range(n_prefill, n_total):
        if len(win) == window:
            parts.append(_oracle_block((np.array(win), cb, mode, double_quant)))
            win = []
        win.append(orc.to_f16(x[t]))
    cat = lambda k: np.concatenate([p[k] for p in parts])  # noqa: E731
    seq = {"codes": cat("codes"), "signs": None if mode == 1 else cat("signs"), "s1": cat("s1"),
           "s2": cat("s2"), "o": np.stack([p["o"] for p in parts]), "gap": cat("gap"), "u": cat("u")}
    return seq, np.array(win).reshape(-1, 128)


# ---------------------------------------------------------------------------
# Shared set-up of the decode parity tests (plain and pre-RoPE keys)
# ---------------------------------------------------------------------------
def fill_cache(cache, contents):
    """Writes per-(b, h) random contents into a Cache (test set-up, no math)."""
    import torch
    for (b, h), c in contents.items():
        nq, nw = c["codes"].shape[0], c["window"].shape[0]
        cache.codes[b, h, :nq] = torch.from_numpy(natural_to_codes(c["codes"]))
        if c["signs"] is not None:
            cache.signs[b, h, :nq] = torch.from_numpy(c["signs"])
        cache.norms[b, h, :nq, 0] = torch.from_numpy(c["s1"])
        cache.norms[b, h, :nq, 1] = torch.from_numpy(c["s2"])
        cache.means[b, h, :c["o"].shape[0]] = torch.from_numpy(c["o"])
        if nw:
            cache.window_buf[b, h, :nw] = torch.from_numpy(c["window"])
        cache.n_quant[b, h] = nq
        cache.n_window[b, h] = nw


def oracle_seq(c):
    """The same random contents in the oracle's layout (sign bits reordered)."""
    f = lambda a: None if a is None else np.asarray(a, dtype=np.float64)  # noqa: E731
    signs = None if c["signs"] is None else signs_to_natural(c["signs"])
    return {"codes": c["codes"].astype(np.int64), "signs": signs, "s1": f(c["s1"]), "s2": f(c["s2"]),
            "o": f(c["o"])}


def oracle_pipeline(xk, xv, n_prefill, n_total, cbk, cbv, mk, mv, window, cosine=False):
    """Oracle cache of one (b, h) after a prefill of n_prefill tokens and
    appends up to n_total (flushes of the full window as fp16 blocks); with cosine
    the codes are the codewords of largest cosine similarity."""
    from oracle import nsn_oracle as orc
    out = []
    for x, cb, mode in ((xk, cbk, mk), (xv, cbv, mv)):
        seq = orc.quantize_sequence(x[:n_prefill], cb, mode, 128, window, cosine=cosine)
        codes, signs, s1, s2, o = [seq["codes"]], [seq["signs"]], [seq["s1"]], [seq["s2"]], [seq["o"]]
        nq = seq["n_quant"]
        win = list(orc.to_f16(x[nq:n_prefill]))
        for t in range(n_prefill, n_total):
            if len(win) == window:
                blk = orc.quantize_block(np.array(win), cb, mode, cosine=cosine)
                codes.append(blk["codes"]); signs.append(blk["signs"]); s1.append(blk["s1"])
                s2.append(blk["s2"]); o.append(blk["o"][None])
                win = []
            win.append(orc.to_f16(x[t]))
        out.append(({"codes": np.concatenate(codes), "signs": None if mode == 1 else np.concatenate(signs),
                     "s1": np.concatenate(s1), "s2": np.concatenate(s2), "o": np.concatenate(o)},
                    np.array(win).reshape(-1, 128)))
    return out
