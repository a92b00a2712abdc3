"""Seeded synthetic inputs (Llama-shaped KV with channel outliers).

Only input generation lives here -- none of the method's arithmetic -- so that
tests and the bench can hand identical bytes to the CUDA path and to the CPU
oracle.  Recipes (the pages describe KV caches whose early layers keep a few
high-variance outlier channels; the workloads below reproduce that shape):

  * "tiny" (one kv-head, fp32): x ~ N(0,1); on 5 random channels a constant
    offset delta_c ~ N(0, sd=3) is added.
  * "llama" (bf16): x ~ N(0,1); on round(0.04*128) = 5 random channels per
    kv-head x_c <- 3 * (x_c + delta_c), delta_c ~ N(0, sd=4).  Channels and
    offsets are fixed per (recipe seed, kv-head) and shared by every batch row
    and by tokens appended later.
  * queries: q ~ N(0,1).

The random draws use torch's seeded generator on the requested device, so a
given (seed, shape, device) always gives the same tensor.
"""
from __future__ import annotations

import numpy as np
import torch

HEAD_DIM = 128


class KVRecipe:
    """Outlier-channel pattern of one K or V tensor (per kv-head)."""

    def __init__(self, seed: int, n_kv_heads: int, kind: str = "llama"):
        if kind not in ("llama", "tiny"):
            raise ValueError(kind)
        self.seed, self.n_kv_heads, self.kind = int(seed), int(n_kv_heads), kind
        rs = np.random.RandomState(self.seed % (2**32))
        n_out = 5
        self.channels = np.stack([rs.choice(HEAD_DIM, n_out, replace=False) for _ in range(n_kv_heads)])
        sd = 3.0 if kind == "tiny" else 4.0
        self.deltas = rs.normal(0.0, sd, size=(n_kv_heads, n_out))

    def tokens(self, batch: int, n_tokens: int, dtype=torch.bfloat16, device="cpu", stream_id: int = 0):
        """[batch, n_tokens, n_kv_heads, 128] tensor; stream_id selects the draw."""
        g = torch.Generator(device=device)
        g.manual_seed((self.seed * 1000003 + 7919 * stream_id) % (2**63))
        x = torch.randn((batch, n_tokens, self.n_kv_heads, HEAD_DIM), generator=g, device=device,
                        dtype=torch.float32)
        for h in range(self.n_kv_heads):
            ch = torch.as_tensor(self.channels[h], device=device)
            dl = torch.as_tensor(self.deltas[h], device=device, dtype=torch.float32)
            if self.kind == "tiny":
                x[:, :, h, ch] += dl
            else:
                x[:, :, h, ch] = 3.0 * (x[:, :, h, ch] + dl)
        return x.to(dtype)


def queries(seed: int, batch: int, n_q_heads: int, dtype=torch.bfloat16, device="cpu"):
    """q ~ N(0,1) of shape [batch, n_q_heads, 128]."""
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) % (2**63))
    return torch.randn((batch, n_q_heads, HEAD_DIM), generator=g, device=device).to(dtype)


def config_seed(config: int, tensor: str, layer: int = 0) -> int:
    """Seed of one tensor of one workload: 0x4E534E00 + 16*config + {K:0, V:1, q:2} + 1000*layer."""
    return 0x4E534E00 + 16 * config + {"k": 0, "v": 1, "q": 2}[tensor] + 1000 * layer


def random_cache_contents(seed: int, n_tokens: int, n_window: int, mode: int) -> dict:
    """Random contents of one (b, h) compressed sequence, for decode-only tests.

    codes uniform in [0, 256); sign bytes uniform; s1 ~ U(0.5, 3), s2 ~ U(0.5, 1.5),
    block means ~ N(0, 0.3^2), window tokens ~ N(0, 1) -- all rounded to fp16.
    """
    rs = np.random.RandomState(int(seed) % (2**32))
    nblk = (n_tokens + 127) // 128
    f16 = lambda a: a.astype(np.float16)  # noqa: E731
    return {
        "codes": rs.randint(0, 256, size=(n_tokens, 16)).astype(np.uint8),
        "signs": rs.randint(0, 256, size=(n_tokens, 16)).astype(np.uint8) if mode == 2 else None,
        "s1": f16(rs.uniform(0.5, 3.0, n_tokens)),
        "s2": f16(rs.uniform(0.5, 1.5, n_tokens)),
        "o": f16(rs.normal(0.0, 0.3, (nblk, HEAD_DIM))),
        "window": f16(rs.normal(0.0, 1.0, (n_window, HEAD_DIM))),
    }


# The five workloads (sizes of each config; modes: 1 = 1-bit, 2 = 2-bit).
WORKLOADS = {
    1: dict(name="tiny-1bit", batch=1, n_kv_heads=1, n_q_heads=1, seq=256, mode_k=1, mode_v=1, window=0,
            steps=0, layers=1, dtype="f32", kind="tiny"),
    2: dict(name="llama8b-layer-2bit", batch=1, n_kv_heads=8, n_q_heads=32, seq=4096, mode_k=2, mode_v=2,
            window=128, steps=1, layers=1, dtype="bf16", kind="llama"),
    3: dict(name="decode-b16-32k-2bit", batch=16, n_kv_heads=8, n_q_heads=32, seq=32768, mode_k=2, mode_v=2,
            window=128, steps=64, layers=1, dtype="bf16", kind="llama"),
    4: dict(name="extreme-b64-8k-1bit-32layers", batch=64, n_kv_heads=8, n_q_heads=32, seq=8192, mode_k=1,
            mode_v=1, window=128, steps=1, layers=32, dtype="bf16", kind="llama"),
    5: dict(name="longctx-b4-128k-2bitK-1bitV", batch=4, n_kv_heads=8, n_q_heads=32, seq=131072, mode_k=2,
            mode_v=1, window=128, steps=16, layers=1, dtype="bf16", kind="llama"),
}
