"""GPU test of the allocation-free decode entry point (nsn_decode_attention_static).

That entry point serves callers that cannot allocate device memory when they
decode (for example code running inside an allocator callback, or a framework
that reserved all device memory up front): it keeps its decode partials in a
fixed device array inside the library instead of a caller-provided workspace.
Here it must give the same output as nsn_decode_attention (within the attention
tolerance of the other decode tests) on two calls in a row, match the CPU oracle
directly, leave the free device memory unchanged on the second call, and refuse,
before any launch, a shape whose partials would not fit the array.

The file name makes pytest collect it last, so a run that stops at the first
failure has already run every other test; it also passes on its own in a fresh
process.
"""
import math

import numpy as np
import pytest
import torch

from calibration_free_vector_b200 import nsn, synthetic
from oracle import nsn_oracle as orc
import nsn_testlib as tl

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)


def random_caches(B, H, cap, mk, mv, shape, seed):
    kc, vc = nsn.Cache(B, H, cap, 128, mk), nsn.Cache(B, H, cap, 128, mv)
    contents = []
    for cache, mode, off in ((kc, mk, 0), (vc, mv, 5)):
        cont = {(b, h): synthetic.random_cache_contents(seed + 97 * b + 13 * h + off, nq, nw, mode)
                for (b, h), (nq, nw) in shape.items()}
        tl.fill_cache(cache, cont)
        contents.append(cont)
    return kc, vc, contents


@pytest.mark.parametrize("mk,mv,g", [(2, 2, 4), (1, 1, 1), (2, 1, 8)])
def test_static_scratch_matches_workspace_entry_point(mk, mv, g):
    B, H, cap = 2, 2, 2304
    shape = {(0, 0): (2304, 128), (0, 1): (640, 7), (1, 0): (128, 0), (1, 1): (0, 33)}
    kc, vc, (kcont, vcont) = random_caches(B, H, cap, mk, mv, shape, seed=11 + 10 * mk + mv)
    cbk_np, cbv_np = tl.codebook(mk), tl.codebook(mv)
    cbk, cbv = torch.from_numpy(cbk_np).cuda(), torch.from_numpy(cbv_np).cuda()
    q = synthetic.queries(5, B, H * g, torch.bfloat16, "cuda")
    ref = torch.empty((B, H * g, 128), dtype=torch.float32, device="cuda")
    nsn.nsn_decode_attention(kc, vc, q, SCALE, cbk, cbv, ref, nsn.decode_workspace(kc, H * g))
    torch.cuda.synchronize()
    outs = []
    for call in range(2):   # two calls in a row share (and reuse) the same scratch array
        out = torch.full((B, H * g, 128), float("nan"), dtype=torch.float32, device="cuda")
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        nsn.nsn_decode_attention_static(kc, vc, q, SCALE, cbk, cbv, out)
        torch.cuda.synchronize()
        if call == 1:   # after the first call nothing more is allocated
            assert torch.cuda.mem_get_info()[0] == free_before
        err = tl.attn_error(out.cpu().numpy(), ref.cpu().numpy())
        assert np.isfinite(out.cpu().numpy()).all()
        assert err <= tl.ATTN_TOL, f"static-scratch decode differs from the workspace decode: {err:.3g}"
        outs.append(out.cpu().numpy())
    # and the oracle itself, for every sequence that holds tokens
    qf = q.float().cpu().numpy().astype(np.float64)
    for (b, h), (nq, nw) in shape.items():
        if nq + nw == 0:
            continue
        want = orc.decode_attention(qf[b, h * g:(h + 1) * g], tl.oracle_seq(kcont[(b, h)]),
                                    tl.oracle_seq(vcont[(b, h)]), kcont[(b, h)]["window"].astype(np.float64),
                                    vcont[(b, h)]["window"].astype(np.float64), cbk_np.astype(np.float64),
                                    cbv_np.astype(np.float64), mk, mv, SCALE)
        for o in outs:
            assert tl.attn_error(o[b, h * g:(h + 1) * g], want) <= tl.ATTN_TOL


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
