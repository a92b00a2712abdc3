"""GPU parity of the chunked-prefill ("extend") attention (nsn_extend_attention):
the last C tokens of every sequence sit in the residual window and query i of
the chunk attends the quantized part plus the window up to its own token
([TS] Metodologia 4).  Random compressed contents of several shapes (many
splits, one block, window only) against the oracle's extend_attention, every
query of the chunk; a sequence whose window is shorter than the chunk sets
status bit 8."""
import math

import numpy as np
import pytest
import torch

from calibration_free_vector_b200 import nsn, synthetic
from oracle import nsn_oracle as orc
import nsn_testlib as tl

pytestmark = pytest.mark.gpu
SCALE = 1.0 / math.sqrt(128)


@pytest.mark.parametrize("mk,mv,g,C", [(2, 2, 4, 1), (2, 1, 4, 9), (1, 1, 2, 33), (1, 2, 8, 128)])
def test_extend_matches_oracle(mk, mv, g, C):
    B, H, cap = 2, 2, 2304
    nwin = max(C, 40)
    shape = {(0, 0): (2304, 128), (0, 1): (640, nwin), (1, 0): (128, max(C, 77)), (1, 1): (0, 128)}
    kc, vc = nsn.Cache(B, H, cap, 128, mk), nsn.Cache(B, H, cap, 128, mv)
    kcont, vcont = {}, {}
    for (b, h), (nq, nw) in shape.items():
        seed = 500 * b + 10 * h + 100 * mk + mv + C
        kcont[(b, h)] = synthetic.random_cache_contents(seed, nq, nw, mk)
        vcont[(b, h)] = synthetic.random_cache_contents(seed + 5, nq, nw, mv)
    tl.fill_cache(kc, kcont)
    tl.fill_cache(vc, vcont)
    cbk, cbv = tl.codebook(mk), tl.codebook(mv)
    q = torch.stack([synthetic.queries(31 + i, B, H * g, torch.bfloat16, "cpu") for i in range(C)], dim=1)
    out = torch.empty((B, C, H * g, 128), dtype=torch.float32, device="cuda")
    ws = nsn.decode_workspace(kc, H * g)
    nsn.nsn_extend_attention(kc, vc, q.cuda(), SCALE, torch.from_numpy(cbk).cuda(), torch.from_numpy(cbv).cuda(),
                             out, ws)
    torch.cuda.synchronize()
    assert int(kc.status.item()) == 0
    out = out.cpu().numpy()
    qf = q.float().numpy().astype(np.float64)
    for (b, h), (nq, nw) in shape.items():
        want = orc.extend_attention(qf[b, :, h * g:(h + 1) * g], tl.oracle_seq(kcont[(b, h)]),
                                    tl.oracle_seq(vcont[(b, h)]), kcont[(b, h)]["window"].astype(np.float64),
                                    vcont[(b, h)]["window"].astype(np.float64), cbk.astype(np.float64),
                                    cbv.astype(np.float64), mk, mv, SCALE)
        for i in range(C):
            err = tl.attn_error(out[b, i, h * g:(h + 1) * g], want[i])
            assert err <= tl.ATTN_TOL, f"(b={b}, h={h}) query {i} of {C}: error {err:.3g}"


def test_extend_flags_a_window_shorter_than_the_chunk():
    B, H, g, C = 1, 2, 4, 8
    kc, vc = nsn.Cache(B, H, 256, 128, 1), nsn.Cache(B, H, 256, 128, 1)
    cont = {(0, 0): synthetic.random_cache_contents(1, 128, 20, 1), (0, 1): synthetic.random_cache_contents(2, 128, 5, 1)}
    tl.fill_cache(kc, cont)
    tl.fill_cache(vc, cont)
    cb = torch.from_numpy(tl.codebook(1)).cuda()
    q = torch.randn((B, C, H * g, 128), device="cuda").bfloat16()
    out = torch.empty((B, C, H * g, 128), dtype=torch.float32, device="cuda")
    nsn.nsn_extend_attention(kc, vc, q, SCALE, cb, cb, out, nsn.decode_workspace(kc, H * g))
    torch.cuda.synchronize()
    assert int(kc.status.item()) & 8
    assert np.isfinite(out.cpu().numpy()).all()
