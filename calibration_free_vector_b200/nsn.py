"""Thin Python binding of the C ABI in include/nsn.h (ctypes, argument
marshalling only).  Every step of the path runs in libnsn.so; there is no CPU
fallback.  torch is used for device memory and streams only.

Functions keep the C names: nsn_build_codebook_host, nsn_quantize_kv,
nsn_append_residual, nsn_decode_workspace_bytes, nsn_decode_attention,
nsn_decode_rope_workspace_bytes, nsn_decode_attention_rope,
nsn_cache_buffer_sizes.  `Cache` allocates the buffers of one nsn_cache with
torch and fills the C struct.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int, c_int32, c_int64, c_size_t, c_uint64, c_void_p

import numpy as np

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libnsn.so")

HEAD_DIM = 128
SUB_DIM = 8
N_SUB = 16
N_CODES = 256
BLOCK = 128
MODE_1BIT = 1
MODE_2BIT = 2
DTYPE_F32, DTYPE_BF16, DTYPE_F16 = 0, 1, 2


class NsnError(RuntimeError):
    def __init__(self, status: int, where: str):
        lib = load()
        msg = lib.nsn_status_string(status).decode()
        if status == 4:
            msg += ": " + lib.nsn_last_cuda_error().decode()
        super().__init__(f"{where}: {msg} (status {status})")
        self.status = status


class nsn_cache(ctypes.Structure):
    _fields_ = [
        ("batch", c_int32), ("n_kv_heads", c_int32), ("capacity", c_int32), ("window", c_int32),
        ("mode", c_int32), ("scale_adjust", c_int32),
        ("codes", c_void_p), ("signs", c_void_p), ("norms", c_void_p), ("means", c_void_p),
        ("window_buf", c_void_p), ("n_quant", c_void_p), ("n_window", c_void_p), ("status", c_void_p),
        ("double_quant", c_int32), ("s1_levels", c_void_p), ("dq_params", c_void_p),
        ("assign", c_int32),
    ]


class nsn_cache_sizes(ctypes.Structure):
    _fields_ = [(n, c_size_t) for n in ("codes", "signs", "norms", "means", "window_buf", "n_quant", "n_window",
                                        "s1_levels", "dq_params")]


_lib = None


def load():
    """Loads libnsn.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m calibration_free_vector_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    lib.nsn_version.restype = c_int
    lib.nsn_status_string.restype = c_char_p
    lib.nsn_status_string.argtypes = [c_int]
    lib.nsn_last_cuda_error.restype = c_char_p
    lib.nsn_cache_buffer_sizes.restype = c_int
    lib.nsn_cache_buffer_sizes.argtypes = [c_int, c_int, c_int, c_int, c_int, c_int, POINTER(nsn_cache_sizes)]
    lib.nsn_build_codebook_host.restype = c_int
    lib.nsn_build_codebook_host.argtypes = [c_uint64, c_int, c_int, c_int, c_int, c_int, POINTER(c_float)]
    lib.nsn_build_codebook_cosine_host.restype = c_int
    lib.nsn_build_codebook_cosine_host.argtypes = [c_uint64, c_int, c_int, c_int, c_int, c_int, c_int,
                                                   POINTER(c_float)]
    lib.nsn_codebook_4bit_host.restype = c_int
    lib.nsn_codebook_4bit_host.argtypes = [POINTER(c_float), c_int]
    lib.nsn_quantize_kv.restype = c_int
    lib.nsn_quantize_kv.argtypes = [POINTER(nsn_cache), c_void_p, c_int, c_int64, c_int64, c_int64, c_int,
                                    c_void_p, c_void_p]
    lib.nsn_selftest_bounded_wait.restype = c_int
    lib.nsn_selftest_bounded_wait.argtypes = [c_void_p, c_int, c_void_p]
    lib.nsn_selftest_tensor_scores.restype = c_int
    lib.nsn_selftest_tensor_scores.argtypes = [c_void_p, c_int, c_void_p, c_int, c_void_p, c_void_p, c_void_p]
    lib.nsn_quantize_kv_ragged.restype = c_int
    lib.nsn_quantize_kv_ragged.argtypes = [POINTER(nsn_cache), c_void_p, c_int, c_int64, c_int64, c_int64, c_void_p,
                                           c_int, c_void_p, c_void_p]
    lib.nsn_append_residual.restype = c_int
    lib.nsn_append_residual.argtypes = [POINTER(nsn_cache), POINTER(nsn_cache), c_void_p, c_void_p, c_int,
                                        c_int64, c_int64, c_void_p, c_void_p, c_void_p]
    lib.nsn_decode_workspace_bytes.restype = c_size_t
    lib.nsn_decode_workspace_bytes.argtypes = [POINTER(nsn_cache), c_int]
    lib.nsn_decode_attention.restype = c_int
    lib.nsn_decode_attention.argtypes = [POINTER(nsn_cache), POINTER(nsn_cache), c_void_p, c_int, c_int, c_int64,
                                         c_int64, c_float, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                         c_void_p]
    lib.nsn_extend_attention.restype = c_int
    lib.nsn_extend_attention.argtypes = [POINTER(nsn_cache), POINTER(nsn_cache), c_void_p, c_int, c_int, c_int,
                                         c_int64, c_int64, c_int64, c_float, c_void_p, c_void_p, c_void_p, c_void_p,
                                         c_size_t, c_void_p]
    lib.nsn_decode_rope_workspace_bytes.restype = c_size_t
    lib.nsn_decode_rope_workspace_bytes.argtypes = [POINTER(nsn_cache), c_int]
    lib.nsn_decode_attention_rope.restype = c_int
    lib.nsn_decode_attention_rope.argtypes = [POINTER(nsn_cache), POINTER(nsn_cache), c_void_p, c_int, c_int,
                                              c_int64, c_int64, c_float, c_void_p, c_void_p, c_void_p, c_void_p,
                                              c_void_p, c_size_t, c_void_p]
    lib.nsn_decode_attention_static.restype = c_int
    lib.nsn_decode_attention_static.argtypes = [POINTER(nsn_cache), POINTER(nsn_cache), c_void_p, c_int, c_int,
                                                c_int64, c_int64, c_float, c_void_p, c_void_p, c_void_p, c_void_p]
    _lib = lib
    return lib


def _check(status: int, where: str) -> None:
    if status != 0:
        raise NsnError(status, where)


def _dtype_code(t) -> int:
    import torch
    m = {torch.float32: DTYPE_F32, torch.bfloat16: DTYPE_BF16, torch.float16: DTYPE_F16}
    if t.dtype not in m:
        raise TypeError(f"unsupported dtype {t.dtype}")
    return m[t.dtype]


def _stream_ptr(stream) -> int:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


# ---------------------------------------------------------------------------
# Host codebook
# ---------------------------------------------------------------------------
def nsn_build_codebook_host(seed: int, n_samples: int = 65536, n_codes: int = N_CODES, dim: int = SUB_DIM,
                            abs_mode: bool = False, iters: int = 50) -> np.ndarray:
    """k-means codebook [n_codes, dim] float32 (see include/nsn.h)."""
    out = np.empty((n_codes, dim), dtype=np.float32)
    st = load().nsn_build_codebook_host(c_uint64(seed & (2**64 - 1)), n_samples, n_codes, dim,
                                        1 if abs_mode else 0, iters,
                                        out.ctypes.data_as(POINTER(c_float)))
    _check(st, "nsn_build_codebook_host")
    return out


def nsn_build_codebook_cosine_host(seed: int, n_samples: int = 65536, n_codes: int = N_CODES, dim: int = SUB_DIM,
                                   abs_mode: bool = False, kmeans_iters: int = 50,
                                   cosine_iters: int = 10) -> np.ndarray:
    """k-means codebook fine-tuned for cosine distance [n_codes, dim] float32 (see include/nsn.h)."""
    out = np.empty((n_codes, dim), dtype=np.float32)
    st = load().nsn_build_codebook_cosine_host(c_uint64(seed & (2**64 - 1)), n_samples, n_codes, dim,
                                               1 if abs_mode else 0, kmeans_iters, cosine_iters,
                                               out.ctypes.data_as(POINTER(c_float)))
    _check(st, "nsn_build_codebook_cosine_host")
    return out


def nsn_codebook_4bit_host(codebook: np.ndarray) -> np.ndarray:
    """Copy of a float32 codebook with its entries on 16 uniform levels (see include/nsn.h)."""
    out = np.ascontiguousarray(codebook, dtype=np.float32).copy()
    _check(load().nsn_codebook_4bit_host(out.ctypes.data_as(POINTER(c_float)), int(out.size)),
           "nsn_codebook_4bit_host")
    return out


def nsn_cache_buffer_sizes(batch: int, n_kv_heads: int, capacity: int, window: int, mode: int,
                           double_quant: bool = False) -> dict:
    s = nsn_cache_sizes()
    _check(load().nsn_cache_buffer_sizes(batch, n_kv_heads, capacity, window, mode, 1 if double_quant else 0,
                                         ctypes.byref(s)),
           "nsn_cache_buffer_sizes")
    return {n: getattr(s, n) for n, _ in nsn_cache_sizes._fields_}


# ---------------------------------------------------------------------------
# Cache buffers (torch-allocated, caller-owned)
# ---------------------------------------------------------------------------
class Cache:
    """Device buffers of one compressed K or V cache and the matching C struct."""

    def __init__(self, batch: int, n_kv_heads: int, capacity: int, window: int, mode: int,
                 scale_adjust: bool = True, device="cuda", double_quant: bool = False, cosine: bool = False):
        import torch
        sizes = nsn_cache_buffer_sizes(batch, n_kv_heads, capacity, window, mode, double_quant)
        self.batch, self.n_kv_heads, self.capacity, self.window, self.mode = batch, n_kv_heads, capacity, window, mode
        self.scale_adjust = bool(scale_adjust)
        self.double_quant = bool(double_quant)
        self.cosine = bool(cosine)  # codeword of largest cosine similarity instead of the nearest one
        u8 = dict(dtype=torch.uint8, device=device)
        f16 = dict(dtype=torch.float16, device=device)
        nblk = capacity // BLOCK
        self.codes = torch.zeros((batch, n_kv_heads, capacity, N_SUB), **u8)
        self.signs = torch.zeros((batch, n_kv_heads, capacity, N_SUB), **u8) if mode == MODE_2BIT else None
        if double_quant:
            # norms: alpha*s2; means: 4-bit o levels; s1_levels: 4-bit s1 levels; dq_params: (lo, hi) pairs
            self.norms = torch.zeros((batch, n_kv_heads, capacity), **f16)
            self.means = torch.zeros((batch, n_kv_heads, nblk, HEAD_DIM // 2), **u8)
            self.s1_levels = torch.zeros((batch, n_kv_heads, capacity // 2), **u8)
            self.dq_params = torch.zeros((batch, n_kv_heads, nblk, 8), **f16)
        else:
            self.norms = torch.zeros((batch, n_kv_heads, capacity, 2), **f16)
            self.means = torch.zeros((batch, n_kv_heads, nblk, HEAD_DIM), **f16)
            self.s1_levels = None
            self.dq_params = None
        self.window_buf = torch.zeros((batch, n_kv_heads, window, HEAD_DIM), **f16) if window > 0 else None
        self.n_quant = torch.zeros((batch, n_kv_heads), dtype=torch.int32, device=device)
        self.n_window = torch.zeros((batch, n_kv_heads), dtype=torch.int32, device=device)
        self.status = torch.zeros((1,), dtype=torch.int32, device=device)
        for name in ("codes", "norms", "means", "s1_levels", "dq_params"):
            t = getattr(self, name)
            assert (0 if t is None else t.numel() * t.element_size()) == sizes[name], name
        self.c = nsn_cache(
            batch, n_kv_heads, capacity, window, mode, 1 if scale_adjust else 0,
            self.codes.data_ptr(), self.signs.data_ptr() if self.signs is not None else None,
            self.norms.data_ptr(), self.means.data_ptr(),
            self.window_buf.data_ptr() if self.window_buf is not None else None,
            self.n_quant.data_ptr(), self.n_window.data_ptr(), self.status.data_ptr(),
            1 if double_quant else 0,
            self.s1_levels.data_ptr() if self.s1_levels is not None else None,
            self.dq_params.data_ptr() if self.dq_params is not None else None,
            1 if cosine else 0)

    def nbytes_allocated(self) -> int:
        bufs = [self.codes, self.signs, self.norms, self.means, self.window_buf, self.n_quant, self.n_window,
                self.s1_levels, self.dq_params]
        return sum(b.numel() * b.element_size() for b in bufs if b is not None)


# ---------------------------------------------------------------------------
# Device entry points
# ---------------------------------------------------------------------------
def nsn_quantize_kv(cache: Cache, x, codebook, stream=None) -> None:
    """Prefill quantization of x [B, T, H_kv, 128] (any strides with unit last dim)."""
    if x.dim() != 4 or x.shape[-1] != HEAD_DIM or x.stride(-1) != 1:
        raise ValueError("x must be [B, T, H_kv, 128] with a contiguous last dimension")
    if x.shape[0] != cache.batch or x.shape[2] != cache.n_kv_heads:
        raise ValueError("x batch / kv-head count does not match the cache")
    st = load().nsn_quantize_kv(ctypes.byref(cache.c), x.data_ptr(), _dtype_code(x), x.stride(0), x.stride(1),
                                x.stride(2), x.shape[1], codebook.data_ptr(), _stream_ptr(stream))
    _check(st, "nsn_quantize_kv")


def nsn_quantize_kv_ragged(cache: Cache, x, lengths, codebook, max_tokens=None, stream=None) -> None:
    """Ragged prefill of x [B, T, H_kv, 128]: sequence b takes lengths[b] tokens
    (lengths: device int32 [B]); max_tokens defaults to T."""
    if x.dim() != 4 or x.shape[-1] != HEAD_DIM or x.stride(-1) != 1:
        raise ValueError("x must be [B, T, H_kv, 128] with a contiguous last dimension")
    if x.shape[0] != cache.batch or x.shape[2] != cache.n_kv_heads:
        raise ValueError("x batch / kv-head count does not match the cache")
    import torch
    if lengths.dtype != torch.int32 or lengths.dim() != 1 or lengths.shape[0] != cache.batch:
        raise ValueError("lengths must be int32 [B]")
    if lengths.stride(0) != 1 or lengths.device != x.device:
        raise ValueError("lengths must be contiguous and on the device of x")
    mt = x.shape[1] if max_tokens is None else int(max_tokens)
    if mt > x.shape[1]:
        raise ValueError("max_tokens exceeds the rows of x")
    st = load().nsn_quantize_kv_ragged(ctypes.byref(cache.c), x.data_ptr(), _dtype_code(x), x.stride(0),
                                       x.stride(1), x.stride(2), lengths.data_ptr(), mt, codebook.data_ptr(),
                                       _stream_ptr(stream))
    _check(st, "nsn_quantize_kv_ragged")


def nsn_append_residual(k_cache: Cache, v_cache: Cache, k_new, v_new, cb_k, cb_v, stream=None) -> None:
    """Appends one token per (b, h): k_new / v_new [B, H_kv, 128] (same strides)."""
    if k_new.shape != v_new.shape or k_new.stride() != v_new.stride() or k_new.dtype != v_new.dtype:
        raise ValueError("k_new and v_new must share shape, strides and dtype")
    if k_new.dim() != 3 or k_new.shape[-1] != HEAD_DIM or k_new.stride(-1) != 1:
        raise ValueError("k_new must be [B, H_kv, 128] with a contiguous last dimension")
    st = load().nsn_append_residual(ctypes.byref(k_cache.c), ctypes.byref(v_cache.c), k_new.data_ptr(),
                                    v_new.data_ptr(), _dtype_code(k_new), k_new.stride(0), k_new.stride(1),
                                    cb_k.data_ptr(), cb_v.data_ptr(), _stream_ptr(stream))
    _check(st, "nsn_append_residual")


def nsn_selftest_bounded_wait(status, max_attempts: int = 8, stream=None) -> None:
    """Runs the bounded-wait diagnostic; `status` is a device int32 tensor of one element."""
    _check(load().nsn_selftest_bounded_wait(status.data_ptr(), max_attempts, _stream_ptr(stream)),
           "nsn_selftest_bounded_wait")


def nsn_selftest_tensor_scores(rows, codebook, assign: int, scores, status, stream=None) -> None:
    """Raw tensor-core scores of rows [n, 8] (n <= 128, device fp32) against the codebook
    [256, 8] into scores [n, 256] (device fp32); status: device int32 [1]."""
    if rows.dim() != 2 or rows.shape[1] != 8 or scores.shape != (rows.shape[0], 256):
        raise ValueError("rows must be [n, 8] and scores [n, 256]")
    _check(load().nsn_selftest_tensor_scores(rows.data_ptr(), rows.shape[0], codebook.data_ptr(), int(assign),
                                             scores.data_ptr(), status.data_ptr(), _stream_ptr(stream)),
           "nsn_selftest_tensor_scores")


def nsn_decode_workspace_bytes(k_cache: Cache, n_q_heads: int) -> int:
    return int(load().nsn_decode_workspace_bytes(ctypes.byref(k_cache.c), n_q_heads))


def decode_workspace(k_cache: Cache, n_q_heads: int, device="cuda"):
    import torch
    n = nsn_decode_workspace_bytes(k_cache, n_q_heads)
    if n == 0:
        raise ValueError("invalid cache or head count for decode")
    # zero-filled: the leading merge counters must start at zero
    return torch.zeros((n,), dtype=torch.uint8, device=device)


def nsn_decode_attention(k_cache: Cache, v_cache: Cache, q, softmax_scale: float, cb_k, cb_v, out, workspace,
                         stream=None) -> None:
    """Decode attention: q [B, H_q, 128] -> out [B, H_q, 128] float32."""
    if q.dim() != 3 or q.shape[-1] != HEAD_DIM or q.stride(-1) != 1:
        raise ValueError("q must be [B, H_q, 128] with a contiguous last dimension")
    import torch
    if out.dtype != torch.float32 or not out.is_contiguous() or tuple(out.shape) != tuple(q.shape):
        raise ValueError("out must be a contiguous float32 tensor shaped like q")
    st = load().nsn_decode_attention(ctypes.byref(k_cache.c), ctypes.byref(v_cache.c), q.data_ptr(),
                                     _dtype_code(q), q.shape[1], q.stride(0), q.stride(1), float(softmax_scale),
                                     cb_k.data_ptr(), cb_v.data_ptr(), out.data_ptr(), workspace.data_ptr(),
                                     workspace.numel(), _stream_ptr(stream))
    _check(st, "nsn_decode_attention")


def nsn_extend_attention(k_cache: Cache, v_cache: Cache, q, softmax_scale: float, cb_k, cb_v, out, workspace,
                         stream=None) -> None:
    """Chunked-prefill attention: q [B, C, H_q, 128] (the last C tokens of every
    sequence, all in the residual window) -> out [B, C, H_q, 128] float32; query i
    attends the quantized part and the window up to its own token."""
    if q.dim() != 4 or q.shape[-1] != HEAD_DIM or q.stride(-1) != 1:
        raise ValueError("q must be [B, C, H_q, 128] with a contiguous last dimension")
    import torch
    if out.dtype != torch.float32 or not out.is_contiguous() or tuple(out.shape) != tuple(q.shape):
        raise ValueError("out must be a contiguous float32 tensor shaped like q")
    st = load().nsn_extend_attention(ctypes.byref(k_cache.c), ctypes.byref(v_cache.c), q.data_ptr(),
                                     _dtype_code(q), q.shape[2], q.shape[1], q.stride(0), q.stride(1), q.stride(2),
                                     float(softmax_scale), cb_k.data_ptr(), cb_v.data_ptr(), out.data_ptr(),
                                     workspace.data_ptr(), workspace.numel(), _stream_ptr(stream))
    _check(st, "nsn_extend_attention")


def nsn_decode_rope_workspace_bytes(k_cache: Cache, n_q_heads: int) -> int:
    return int(load().nsn_decode_rope_workspace_bytes(ctypes.byref(k_cache.c), n_q_heads))


def decode_rope_workspace(k_cache: Cache, n_q_heads: int, device="cuda"):
    import torch
    n = nsn_decode_rope_workspace_bytes(k_cache, n_q_heads)
    if n == 0:
        raise ValueError("invalid cache or head count for decode")
    return torch.zeros((n,), dtype=torch.uint8, device=device)


def nsn_decode_attention_rope(k_cache: Cache, v_cache: Cache, q, softmax_scale: float, inv_freq, cb_k, cb_v, out,
                              workspace, stream=None) -> None:
    """Decode attention over pre-RoPE keys: every cached key is rotated at its
    position (quantized token t at t, window slot w at n_quant + w) with the
    rotate-half pairing (i, i + 64) and angle pos * inv_freq[i]; q [B, H_q, 128]
    is the already-rotated query; inv_freq a device float32 tensor of 64."""
    if q.dim() != 3 or q.shape[-1] != HEAD_DIM or q.stride(-1) != 1:
        raise ValueError("q must be [B, H_q, 128] with a contiguous last dimension")
    import torch
    if out.dtype != torch.float32 or not out.is_contiguous() or tuple(out.shape) != tuple(q.shape):
        raise ValueError("out must be a contiguous float32 tensor shaped like q")
    if inv_freq.dtype != torch.float32 or inv_freq.numel() != HEAD_DIM // 2 or not inv_freq.is_contiguous():
        raise ValueError("inv_freq must be a contiguous float32 tensor of 64")
    st = load().nsn_decode_attention_rope(ctypes.byref(k_cache.c), ctypes.byref(v_cache.c), q.data_ptr(),
                                          _dtype_code(q), q.shape[1], q.stride(0), q.stride(1),
                                          float(softmax_scale), inv_freq.data_ptr(), cb_k.data_ptr(),
                                          cb_v.data_ptr(), out.data_ptr(), workspace.data_ptr(), workspace.numel(),
                                          _stream_ptr(stream))
    _check(st, "nsn_decode_attention_rope")


def nsn_decode_attention_static(k_cache: Cache, v_cache: Cache, q, softmax_scale: float, cb_k, cb_v, out,
                                stream=None) -> None:
    """Decode attention without a workspace argument.

    For callers that cannot allocate device memory when they decode (for example
    code running inside an allocator callback, or a framework that reserved all
    device memory up front).  The partial results go to a fixed device array
    inside the library instead (include/nsn.h: NSN_DECODE_SCRATCH_BYTES); calls
    that overlap on the GPU race on it.  Same result as nsn_decode_attention.
    """
    if q.dim() != 3 or q.shape[-1] != HEAD_DIM or q.stride(-1) != 1:
        raise ValueError("q must be [B, H_q, 128] with a contiguous last dimension")
    import torch
    if out.dtype != torch.float32 or not out.is_contiguous() or tuple(out.shape) != tuple(q.shape):
        raise ValueError("out must be a contiguous float32 tensor shaped like q")
    st = load().nsn_decode_attention_static(ctypes.byref(k_cache.c), ctypes.byref(v_cache.c), q.data_ptr(),
                                            _dtype_code(q), q.shape[1], q.stride(0), q.stride(1),
                                            float(softmax_scale), cb_k.data_ptr(), cb_v.data_ptr(),
                                            out.data_ptr(), _stream_ptr(stream))
    _check(st, "nsn_decode_attention_static")
