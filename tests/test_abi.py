"""CPU checks of the C ABI: the library builds/loads, exports every symbol that
include/nsn.h declares, validates arguments without a GPU, and its host-side
codebook builder matches the oracle's k-means bit for bit."""
import ctypes
import os
import re

import numpy as np
import pytest

from calibration_free_vector_b200 import nsn
from calibration_free_vector_b200.build import build
from oracle import codebook_oracle as cbo

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "nsn.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return nsn.load()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nsn_[a-z_0-9]+)\s*\(", text)))


def test_exports_every_declared_symbol(lib):
    names = declared_functions()
    assert len(names) >= 9
    for n in names:
        assert hasattr(lib, n), n


def test_version_and_status_strings(lib):
    assert lib.nsn_version() >= 100
    assert lib.nsn_status_string(0) == b"ok"
    assert lib.nsn_status_string(3) == b"workspace too small"


def test_buffer_sizes(lib):
    s = nsn.nsn_cache_buffer_sizes(16, 8, 32896, 128, 2)
    assert s["codes"] == 16 * 8 * 32896 * 16 == s["signs"]
    assert s["norms"] == 16 * 8 * 32896 * 4
    assert s["means"] == 16 * 8 * (32896 // 128) * 128 * 2
    assert s["window_buf"] == 16 * 8 * 128 * 128 * 2
    s1 = nsn.nsn_cache_buffer_sizes(1, 1, 256, 0, 1)
    assert s1["signs"] == 0 and s1["window_buf"] == 0
    d = nsn.nsn_cache_buffer_sizes(16, 8, 32896, 128, 2, double_quant=True)
    assert d["codes"] == s["codes"] and d["signs"] == s["signs"]
    assert d["norms"] == 16 * 8 * 32896 * 2                       # alpha*s2 only
    assert d["means"] == 16 * 8 * (32896 // 128) * 64              # 4-bit o levels
    assert d["s1_levels"] == 16 * 8 * 32896 // 2
    assert d["dq_params"] == 16 * 8 * (32896 // 128) * 16
    assert s["s1_levels"] == 0 and s["dq_params"] == 0
    with pytest.raises(nsn.NsnError):
        nsn.nsn_cache_buffer_sizes(1, 1, 100, 128, 2)   # capacity not a multiple of 128
    with pytest.raises(nsn.NsnError):
        nsn.nsn_cache_buffer_sizes(1, 1, 128, 64, 2)    # window must be 0 or 128


def test_host_validation_without_gpu(lib):
    # Every device entry point rejects bad arguments before touching the GPU.
    c = nsn.nsn_cache(1, 1, 128, 128, 2, 1, 16, 16, 16, 16, 16, 16, 16, None)
    assert lib.nsn_quantize_kv(ctypes.byref(c), None, 1, 0, 0, 0, 10, 16, None) == 1
    bad = nsn.nsn_cache(1, 1, 100, 128, 2, 1, 16, 16, 16, 16, 16, 16, 16, None)
    assert lib.nsn_quantize_kv(ctypes.byref(bad), 16, 1, 0, 0, 0, 10, 16, None) == 1
    odd = nsn.nsn_cache(1, 1, 128, 64, 2, 1, 16, 16, 16, 16, 16, 16, 16, None)
    assert lib.nsn_quantize_kv(ctypes.byref(odd), 16, 1, 0, 0, 0, 10, 16, None) == 2
    # misaligned x, unaligned token stride, too many tokens
    assert lib.nsn_quantize_kv(ctypes.byref(c), 18, 1, 0, 1024, 128, 10, 16, None) == 1
    assert lib.nsn_quantize_kv(ctypes.byref(c), 16, 1, 0, 1020, 128, 10, 16, None) == 1
    assert lib.nsn_quantize_kv(ctypes.byref(c), 16, 1, 0, 1024, 128, 300, 16, None) == 1
    # double quantization: its buffers are required, the flag is 0 or 1, and K / V must agree
    dq_missing = nsn.nsn_cache(1, 1, 128, 128, 2, 1, 16, 16, 16, 16, 16, 16, 16, None, 1, None, None)
    assert lib.nsn_quantize_kv(ctypes.byref(dq_missing), 16, 1, 0, 1024, 128, 10, 16, None) == 1
    dq_flag = nsn.nsn_cache(1, 1, 128, 128, 2, 1, 16, 16, 16, 16, 16, 16, 16, None, 2, 16, 16)
    assert lib.nsn_quantize_kv(ctypes.byref(dq_flag), 16, 1, 0, 1024, 128, 10, 16, None) == 1
    dq_ok = nsn.nsn_cache(1, 2, 128, 128, 2, 1, 16, 16, 16, 16, 16, 16, 16, None, 1, 16, 16)
    c2b = nsn.nsn_cache(1, 2, 128, 128, 2, 1, 16, 16, 16, 16, 16, 16, 16, None)
    assert lib.nsn_append_residual(ctypes.byref(dq_ok), ctypes.byref(c2b), 16, 16, 1, 0, 128, 16, 16, None) == 1
    # ragged prefill: lengths missing or misaligned, bound over capacity, negative bound
    assert lib.nsn_quantize_kv_ragged(ctypes.byref(c), 16, 1, 0, 1024, 128, None, 10, 16, None) == 1
    assert lib.nsn_quantize_kv_ragged(ctypes.byref(c), 16, 1, 0, 1024, 128, 18, 10, 16, None) == 1
    assert lib.nsn_quantize_kv_ragged(ctypes.byref(c), 16, 1, 0, 1024, 128, 16, 300, 16, None) == 1
    assert lib.nsn_quantize_kv_ragged(ctypes.byref(c), 16, 1, 0, 1024, 128, 16, -1, 16, None) == 1
    assert lib.nsn_quantize_kv_ragged(ctypes.byref(odd), 16, 1, 0, 1024, 128, 16, 10, 16, None) == 2
    # decode: head count not a multiple, GQA group > 8, workspace too small
    c2 = nsn.nsn_cache(1, 2, 128, 128, 2, 1, 16, 16, 16, 16, 16, 16, 16, None)
    assert lib.nsn_decode_attention(ctypes.byref(c2), ctypes.byref(c2), 16, 1, 3, 0, 128, 0.1, 16, 16, 16, 16,
                                    1 << 20, None) == 1
    assert lib.nsn_decode_attention(ctypes.byref(c2), ctypes.byref(c2), 16, 1, 32, 0, 128, 0.1, 16, 16, 16, 16,
                                    1 << 20, None) == 2
    assert lib.nsn_decode_attention(ctypes.byref(c2), ctypes.byref(c2), 16, 1, 8, 0, 128, 0.1, 16, 16, 16, 16,
                                    16, None) == 3
    need = lib.nsn_decode_workspace_bytes(ctypes.byref(c2), 8)
    assert need > 0
    # pre-RoPE decode: frequency table required, the same head rules, the larger workspace
    need_r = lib.nsn_decode_rope_workspace_bytes(ctypes.byref(c2), 8)
    assert need_r >= need + 1 * 8 * (128 + 128) * 4
    assert lib.nsn_decode_attention_rope(ctypes.byref(c2), ctypes.byref(c2), 16, 1, 8, 0, 128, 0.1, None, 16, 16,
                                         16, 16, need_r, None) == 1
    assert lib.nsn_decode_attention_rope(ctypes.byref(c2), ctypes.byref(c2), 16, 1, 8, 0, 128, 0.1, 8, 16, 16,
                                         16, 16, need_r, None) == 1   # inv_freq not 16-byte aligned
    assert lib.nsn_decode_attention_rope(ctypes.byref(c2), ctypes.byref(c2), 16, 1, 3, 0, 128, 0.1, 16, 16, 16,
                                         16, 16, need_r, None) == 1
    assert lib.nsn_decode_attention_rope(ctypes.byref(c2), ctypes.byref(c2), 16, 1, 32, 0, 128, 0.1, 16, 16, 16,
                                         16, 16, need_r, None) == 2
    assert lib.nsn_decode_attention_rope(ctypes.byref(c2), ctypes.byref(c2), 16, 1, 8, 0, 128, 0.1, 16, 16, 16,
                                         16, 16, need, None) == 3
    # append: window 0 caches cannot append; shapes must agree
    c0 = nsn.nsn_cache(1, 2, 128, 0, 2, 1, 16, 16, 16, 16, None, 16, 16, None)
    assert lib.nsn_append_residual(ctypes.byref(c0), ctypes.byref(c0), 16, 16, 1, 0, 128, 16, 16, None) == 2
    assert lib.nsn_append_residual(ctypes.byref(c), ctypes.byref(c2), 16, 16, 1, 0, 128, 16, 16, None) == 1


@pytest.mark.parametrize("batch,heads,cap,window,hq", [(1, 2, 128, 128, 8), (4, 8, 4096, 128, 32),
                                                        (3, 2, 1152, 0, 2), (16, 8, 32896, 128, 64)])
def test_rope_workspace_is_decode_workspace_plus_logits(lib, batch, heads, cap, window, hq):
    # layout (include/nsn.h): the decode workspace, then from a 256-byte boundary the
    # K logits, batch * n_q_heads * rs_cap fp32 with rs_cap = capacity + window
    # rounded up to 64 tokens
    c = nsn.nsn_cache(batch, heads, cap, window, 2, 1, 16, 16, 16, 16, 16 if window else None, 16, 16, None)
    ws = lib.nsn_decode_workspace_bytes(ctypes.byref(c), hq)
    rope = lib.nsn_decode_rope_workspace_bytes(ctypes.byref(c), hq)
    rs_cap = ((cap + window + 63) // 64) * 64
    assert ws > 0
    assert rope == ((ws + 255) // 256) * 256 + batch * hq * rs_cap * 4


def test_host_codebook_matches_oracle(lib):
    for abs_mode in (False, True):
        ours = nsn.nsn_build_codebook_host(0x1234, 8192, 64, 8, abs_mode, 12)
        ref = cbo.build_codebook(0x1234, 8192, 64, 8, abs_mode, 12)
        assert np.array_equal(ours.astype(np.float64), ref)


def test_host_cosine_codebook_matches_oracle(lib):
    for abs_mode in (False, True):
        ours = nsn.nsn_build_codebook_cosine_host(0x77, 8192, 64, 8, abs_mode, 8, 4)
        ref = cbo.build_codebook_cosine(0x77, 8192, 64, 8, abs_mode, 8, 4)
        assert np.array_equal(ours.astype(np.float64), ref)
    with pytest.raises(nsn.NsnError):
        nsn.nsn_build_codebook_cosine_host(1, 100, 256, 8, False, 3, -1)


def test_codebook_4bit_matches_oracle(lib):
    for abs_mode in (False, True):
        cb = nsn.nsn_build_codebook_host(0x99, 8192, 256, 8, abs_mode, 4)
        ours = nsn.nsn_codebook_4bit_host(cb)
        ref = cbo.codebook_4bit(cb)
        assert np.array_equal(ours.astype(np.float64), ref)
        assert len(np.unique(ours)) <= 16
        assert np.array_equal(nsn.nsn_codebook_4bit_host(ours), ours)   # already on the grid


def test_host_codebook_full_size_properties(lib):
    cb = nsn.nsn_build_codebook_host(7, 65536, 256, 8, True, 3)
    assert cb.shape == (256, 8) and np.all(cb >= 0)
    assert np.array_equal(cb, cb.astype(np.float16).astype(np.float32))
    with pytest.raises(nsn.NsnError):
        nsn.nsn_build_codebook_host(7, 100, 256, 8, False, 3)
