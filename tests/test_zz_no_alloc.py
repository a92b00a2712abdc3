"""GPU test of the allocation-free decode entry point (nsn_decode_attention_static).

That entry point serves callers that cannot allocate device memory when they
decode (for example code running inside an allocator callback, or a framework
that reserved all device memory up front): it keeps its decode partials in a
fixed device array inside the library instead of a caller-provided workspace.
Here it must give the same output as nsn_decode_attention (within the attention
tolerance of the other decode tests) on two calls in a row, and refuse, before
any launch, a shape whose partials would not fit the array.

The file name makes pytest collect it last, so a run that stops at the first
failure has already run every other test; it also passes on its own in a fresh
process.
"""
import math

import numpy as np
import pytest
import torch

from calibration_free_vector_b200 import nsn, synthetic
import nsn_testlib as tl

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)


def random_caches(B, H, cap, mk, mv, shape, seed):
    kc, vc = nsn.Cache(B, H, cap, 128, mk), nsn.Cache(B, H, cap, 128, mv)
    for cache, mode, off in ((kc, mk, 0), (vc, mv, 5)):
        for (b, h), (nq, nw) in shape.items():
            c = synthetic.random_cache_contents(seed + 97 * b + 13 * h + off, nq, nw, mode)
            cache.codes[b, h, :nq] = torch.from_numpy(c["codes"])
            if c["signs"] is not None:
                cache.signs[b, h, :nq] = torch.from_numpy(c["signs"])
            cache.norms[b, h, :nq, 0] = torch.from_numpy(c["s1"])
            cache.norms[b, h, :nq, 1] = torch.from_numpy(c["s2"])
            cache.means[b, h, :c["o"].shape[0]] = torch.from_numpy(c["o"])
            if nw:
                cache.window_buf[b, h, :nw] = torch.from_numpy(c["window"])
            cache.n_quant[b, h] = nq
            cache.n_window[b, h] = nw
    return kc, vc


@pytest.mark.parametrize("mk,mv,g", [(2, 2, 4), (1, 1, 1), (2, 1, 8)])
def test_static_scratch_matches_workspace_entry_point(mk, mv, g):
    B, H, cap = 2, 2, 2304
    shape = {(0, 0): (2304, 128), (0, 1): (640, 7), (1, 0): (128, 0), (1, 1): (0, 33)}
    kc, vc = random_caches(B, H, cap, mk, mv, shape, seed=11 + 10 * mk + mv)
    cbk = torch.from_numpy(tl.codebook(mk)).cuda()
    cbv = torch.from_numpy(tl.codebook(mv)).cuda()
    q = synthetic.queries(5, B, H * g, torch.bfloat16, "cuda")
    ref = torch.empty((B, H * g, 128), dtype=torch.float32, device="cuda")
    nsn.nsn_decode_attention(kc, vc, q, SCALE, cbk, cbv, ref, nsn.decode_workspace(kc, H * g))
    torch.cuda.synchronize()
    for _ in range(2):   # two calls in a row share (and reuse) the same scratch array
        out = torch.full((B, H * g, 128), float("nan"), dtype=torch.float32, device="cuda")
        nsn.nsn_decode_attention_static(kc, vc, q, SCALE, cbk, cbv, out)
        torch.cuda.synchronize()
        err = tl.attn_error(out.cpu().numpy(), ref.cpu().numpy())
        assert np.isfinite(out.cpu().numpy()).all()
        assert err <= tl.ATTN_TOL, f"static-scratch decode differs from the workspace decode: {err:.3g}"


def test_static_scratch_rejects_shapes_that_do_not_fit():
    # 64 x 32 sequences of 4 query heads need more partial storage than the array holds.
    B, H = 64, 32
    kc, vc = nsn.Cache(B, H, 128, 128, 1), nsn.Cache(B, H, 128, 128, 1)
    need = nsn.nsn_decode_workspace_bytes(kc, 4 * H)
    assert need > (8 << 20)
    cb = torch.from_numpy(tl.codebook(1)).cuda()
    q = torch.zeros((B, 4 * H, 128), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((B, 4 * H, 128), dtype=torch.float32, device="cuda")
    with pytest.raises(nsn.NsnError) as e:
        nsn.nsn_decode_attention_static(kc, vc, q, SCALE, cb, cb, out)
    assert e.value.status == 3   # NSN_ERR_WORKSPACE
