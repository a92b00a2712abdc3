"""GPU test of the error path for a shared-memory copy that never lands.

nsn_selftest_bounded_wait arms an mbarrier for 16 bytes that are never sent and
waits on it with the decode's bounded wait.  The wait must give up after the
given number of attempts, set status bit 2 and return; the CUDA context must
stay usable (a decode afterwards still matches the workspace path).  Nothing
faults, traps or hangs."""
import math
import time

import pytest
import torch

from calibration_free_vector_b200 import nsn, synthetic
import nsn_testlib as tl

pytestmark = pytest.mark.gpu


def test_bounded_wait_gives_up_sets_status_and_returns():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    t0 = time.perf_counter()
    nsn.nsn_selftest_bounded_wait(status, 8)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert int(status.item()) == 2

    # the context is still usable
    B, H, g, mode = 1, 1, 4, 2
    kc, vc = nsn.Cache(B, H, 256, 128, mode), nsn.Cache(B, H, 256, 128, mode)
    x = synthetic.KVRecipe(5, H, "llama").tokens(B, 300, torch.bfloat16, "cuda")
    cb = torch.from_numpy(tl.codebook(mode)).cuda()
    nsn.nsn_quantize_kv(kc, x, cb)
    nsn.nsn_quantize_kv(vc, x, cb)
    q = synthetic.queries(6, B, H * g, torch.bfloat16, "cuda")
    out = torch.empty((B, H * g, 128), dtype=torch.float32, device="cuda")
    nsn.nsn_decode_attention(kc, vc, q, 1 / math.sqrt(128), cb, cb, out, nsn.decode_workspace(kc, H * g))
    torch.cuda.synchronize()
    assert torch.isfinite(out).all() and int(kc.status.item()) == 0


def test_bounded_wait_rejects_bad_arguments():
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    for n in (0, -1, 5000):
        with pytest.raises(nsn.NsnError):
            nsn.nsn_selftest_bounded_wait(status, n)
