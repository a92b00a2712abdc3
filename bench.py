"""Benchmark of the NSNQuant KV hot path on B200.

Workloads (one GPU each; `--workload`, default 3):
  3  decode-throughput layer: batch 16, 32 query / 8 KV heads, head_dim 128, a
     32768-token context per sequence quantized to 2-bit K and V, 128-token fp16
     residual window.
  4  extreme compression: batch 64, 8192 tokens, 1-bit K and V, 32 layers of the
     same shape (each with its own seeded K/V); one step decodes all 32 layers.
  5  long context: batch 4, a 131072-token prefill per sequence, 2-bit K / 1-bit V.
One timed step = one decode step of the whole batch: per layer, append one new
K/V token per (sequence, kv-head) (flushing the full window through the
quantizer on the first step) + decode attention of all 32 query heads.
`value` = generated tokens/s = batch * steps / time.

The same JSON line also carries the compressed-KV GB/s, the roofline of the
decode call, the prefill quantizer's throughput (tokens/s) with its HBM and
tensor rooflines, an end-to-end number through the public API with host
buffers, the SM clocks seen during the timed region, and the CPU oracle
baseline together with a sampled parity check of the timed prefill (codes of
the first blocks against the oracle, near-ties counted).

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload 3|4|5]
For N > 1 launch one process per GPU with torchrun; each rank runs an
independent replica (the path shards by sequence; no collective is needed).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn tokens/s & compressed-KV GB/s vs HBM peak; quantize tokens/s"
WORKLOADS = {
    3: dict(config=3, name="decode-b16-32k-2bit", batch=16, n_kv_heads=8, n_q_heads=32, seq=32768,
            mode_k=2, mode_v=2, window=128, layers=1),
    4: dict(config=4, name="extreme-b64-8k-1bit-32layers", batch=64, n_kv_heads=8, n_q_heads=32, seq=8192,
            mode_k=1, mode_v=1, window=128, layers=32),
    5: dict(config=5, name="longctx-b4-128k-2bitK-1bitV", batch=4, n_kv_heads=8, n_q_heads=32, seq=131072,
            mode_k=2, mode_v=1, window=128, layers=1),
}
WORKLOAD = WORKLOADS[3]
BYTES_PER_TOKEN = {1: 16 + 4, 2: 16 + 16 + 4}   # codes (+ signs) + (s1, s2) per token-head
MEAN_BYTES_PER_BLOCK = 128 * 2
# With double quantization s1 is a 4-bit level (0.5 B) next to fp16 alpha*s2, and a
# block's o is 64 B of levels plus 16 B of (lo, hi) parameters.
BYTES_PER_TOKEN_DQ = {1: 16 + 2.5, 2: 16 + 16 + 2.5}
MEAN_BYTES_PER_BLOCK_DQ = 64 + 16
# Kernels one decode step launches per layer: append_kernel (K and V, flush
# included) and decode_kernel (splits, residual window and merge).
LAUNCHES_PER_STEP = 2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


# DRAM bytes (read + write) per decode_kernel launch on this workload, from one
# ncu capture (dram__bytes_read.sum + dram__bytes_write.sum of the launch list of
# this workload, taken with --metrics and --clock-control none), valid only for the sources the
# decode kernel is compiled from with this SHA-256 (decode.cu, nsn_common.cuh,
# comments and whitespace removed).
# Any later change to those files makes the figure stale; the bench then reports null.
DECODE_TRAFFIC = {"sha256": "cd324c724a8ffcb74d40f3f35a5dbc92c074525abbfb0fa5db97801f25f3152f",
                  "bytes_per_launch": (320936192 + 320983040) // 2 + (3968000 + 882432) // 2}


def decode_sources_sha256() -> str:
    """SHA-256 of the decode kernel's sources with comments and whitespace removed
    (a comment edit does not change the kernel the traffic figure belongs to)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for name in ("decode.cu", "nsn_common.cuh"):
        with open(os.path.join(ROOT, "calibration_free_vector_b200", "csrc", name)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()


def decode_traffic():
    return DECODE_TRAFFIC["bytes_per_launch"] if decode_sources_sha256() == DECODE_TRAFFIC["sha256"] else None


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")), int(os.environ.get("WORLD_SIZE", "1"))


def max_over_ranks(ms: float, world: int, device) -> float:
    """The largest of the ranks' times (every rank gets it); ms itself when alone."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, max_ms: float) -> float:
    """Whole-job units/s: what all ranks processed over the slowest rank's time."""
    return world * units_per_rank / (max_ms * 1e-3)


def rank_seed_offset(rank: int) -> int:
    """Each replica draws its own synthetic batch."""
    return 7 * rank


def workload_name(W: dict, args) -> str:
    return W["name"] + ("-dq" if args.double_quant else "") + ("-prerope" if args.rope else "")


def config_dict(W: dict, args, world: int, batch: int) -> dict:
    """The `config` object of the JSON line; both arms print the same one."""
    return {"workload": workload_name(W, args), "batch": batch, "seq_len": W["seq"], "n_q_heads": W["n_q_heads"],
            "n_kv_heads": W["n_kv_heads"], "head_dim": 128, "layers": W["layers"], "mode_k": W["mode_k"],
            "mode_v": W["mode_v"], "window": W["window"], "double_quant": bool(args.double_quant),
            "pre_rope_keys": bool(args.rope), **({"rope_theta_base": 500000.0} if args.rope else {}),
            "parallelism": "replicas" if world > 1 else "single"}


# ---------------------------------------------------------------------------
# clocks sampler (nvidia-smi during the timed region)
# ---------------------------------------------------------------------------
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.gpu_id, self.proc, self.lines = gpu_id, None, []

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu_id), f"--query-gpu={self.FIELDS}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# CPU oracle baseline (test infrastructure; the only other place bench runs oracle/)
# ---------------------------------------------------------------------------
def rope_theta() -> np.ndarray:
    """RoPE frequencies of the Llama-3-8B shape: theta_i = 500000^(-2i/128), fp32."""
    return (500000.0 ** (-2.0 * np.arange(64) / 128.0)).astype(np.float32)


def oracle_decode_sample(budget_s: float, seed: int = 0, rope: bool = False, W: dict | None = None):
    """Times the oracle's decode attention (pre-RoPE keys with `rope`) for sampled
    (b, kv-head) sequences of the workload shape (random compressed contents in
    the workload's K and V modes, full window).  Returns (seconds per
    (b, kv-head), sequences timed, threads)."""
    from calibration_free_vector_b200 import synthetic
    from oracle import nsn_oracle as orc
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        threads = 1
    W = W or WORKLOAD
    nq = W["seq"] - 128
    g = W["n_q_heads"] // W["n_kv_heads"]
    cbk = np.abs(np.random.RandomState(seed).normal(size=(256, 8)))
    cbv = cbk if W["mode_v"] == 2 else np.random.RandomState(seed + 7).normal(size=(256, 8))
    if W["mode_k"] == 1:
        cbk = np.random.RandomState(seed + 7).normal(size=(256, 8))
    rs = np.random.RandomState(seed + 1)
    times, n = [], 0
    t_start = time.perf_counter()
    while True:
        kc = synthetic.random_cache_contents(seed + 10 * n, nq, 128, W["mode_k"])
        vc = synthetic.random_cache_contents(seed + 10 * n + 5, nq, 128, W["mode_v"])
        f = lambda c: {"codes": c["codes"].astype(np.int64), "signs": c["signs"],  # noqa: E731
                       "s1": c["s1"].astype(np.float64), "s2": c["s2"].astype(np.float64),
                       "o": c["o"].astype(np.float64)}
        q = rs.normal(size=(g, 128))
        t0 = time.perf_counter()
        if rope:
            orc.decode_attention_rope(q, f(kc), f(vc), kc["window"].astype(np.float64),
                                      vc["window"].astype(np.float64), cbk, cbv, W["mode_k"], W["mode_v"],
                                      1 / math.sqrt(128), rope_theta().astype(np.float64))
        else:
            orc.decode_attention(q, f(kc), f(vc), kc["window"].astype(np.float64), vc["window"].astype(np.float64),
                                 cbk, cbv, W["mode_k"], W["mode_v"], 1 / math.sqrt(128))
        times.append(time.perf_counter() - t0)
        n += 1
        if time.perf_counter() - t_start > budget_s or n >= 64:
            break
    return float(np.mean(times)), n, threads


def oracle_quantize_check(x_blocks: np.ndarray, codebook: np.ndarray, mode: int, got_codes: np.ndarray,
                          got_signs, budget_s: float):
    """Times the oracle quantizing the first 128-token blocks of the prefill the
    bench timed (same bf16 tokens, same codebook) and compares the GPU's codes and
    sign bytes with it.  Returns (seconds per block, blocks, sub-vectors compared,
    oracle near-ties (top-2 gap <= 1e-6 relative), code mismatches outside the
    near-ties, sign-byte mismatches)."""
    from oracle import nsn_oracle as orc
    times, n_sub, n_tie, n_bad, n_sbad = [], 0, 0, 0, 0
    t_start = time.perf_counter()
    for i in range(x_blocks.shape[0]):
        t0 = time.perf_counter()
        ref = orc.quantize_block(x_blocks[i].astype(np.float64), codebook.astype(np.float64), mode)
        times.append(time.perf_counter() - t0)
        tie = ref["gap"] <= 1e-6
        n_sub += tie.size
        n_tie += int(tie.sum())
        n_bad += int(((got_codes[i] != ref["codes"]) & ~tie).sum())
        if mode == 2:
            n_sbad += int((signs_natural(got_signs[i]) != ref["signs"]).sum())
        if time.perf_counter() - t_start > budget_s:
            break
    return float(np.mean(times)), len(times), n_sub, n_tie, n_bad, n_sbad


def codes_natural(code_bytes: np.ndarray) -> np.ndarray:
    """The cache's code records [n, 16] (the even sub-vectors' codes, then the odd
    ones') in natural sub-vector order."""
    out = np.empty_like(code_bytes)
    out[:, 0::2] = code_bytes[:, :8]
    out[:, 1::2] = code_bytes[:, 8:]
    return out


def signs_natural(sign_bytes: np.ndarray) -> np.ndarray:
    """The cache's sign records [n, 16] (field i = dim i of the 16 sub-vectors,
    sub-vector s at bit 15 - s) as the natural layout [n, 16] (byte s, bit i)."""
    fields = sign_bytes.astype(np.uint32).reshape(-1, 8, 2)
    fields = fields[:, :, 0] | (fields[:, :, 1] << 8)          # [n, 8] 16-bit fields
    s_idx = np.arange(16)
    bits = (fields[:, None, :] >> (15 - s_idx)[None, :, None]) & 1  # [n, 16 s, 8 i]
    return (bits * (1 << np.arange(8))[None, None, :]).sum(axis=2).astype(np.uint8)


def run_reference(args):
    """--impl reference: the CPU oracle on the host cores, same metric/unit/config."""
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    W = WORKLOADS[getattr(args, "workload", 3)]
    B = getattr(args, "batch", 0) or W["batch"]
    rope = bool(getattr(args, "rope", False))
    args.rope, args.double_quant = rope, bool(getattr(args, "double_quant", False))
    per_seq = []
    for _ in range(args.warmup):
        oracle_decode_sample(0.0, seed=99, rope=rope, W=W)
    threads = 1
    per_step_budget = min(5.0, 100.0 / max(1, args.steps))
    for s in range(args.steps):
        t, n, threads = oracle_decode_sample(per_step_budget, seed=s, rope=rope, W=W)
        per_seq.append(t)
    step_s = float(np.mean(per_seq)) * B * W["n_kv_heads"] * W["layers"]
    value = B / step_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_dict(W, args, world, B),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"each step: oracle decode attention{' (pre-RoPE keys)' if rope else ''} "
                                   f"of >=1 sampled (batch, kv-head) sequence ({W['seq'] - 128} quantized + 128 "
                                   f"window tokens, {W['n_q_heads'] // W['n_kv_heads']} q-heads), timed and "
                                   f"scaled to {B}x{W['n_kv_heads']} sequences x {W['layers']} layer(s) per step; "
                                   f"ms_per_step is that extrapolation, not a full step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def run_ours(args):
    import torch
    import torch.distributed as dist

    from calibration_free_vector_b200 import nsn, synthetic
    from calibration_free_vector_b200.build import build

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    if rank == 0:
        build()
    if world > 1:
        dist.barrier()
    nsn.load()

    W = WORKLOADS[args.workload]
    B, H, HQ, T, NL = args.batch or W["batch"], W["n_kv_heads"], W["n_q_heads"], W["seq"], W["layers"]
    g = HQ // H
    K, WU = args.steps, args.warmup
    e2e_steps = 0 if args.lite else K
    total_steps = WU + K + e2e_steps
    cap = ((T + K + e2e_steps + 255) // 128) * 128
    cfg = W["config"]

    # codebooks from the host builder (k-means on seeded randn; abs values for 2-bit)
    iters = 3 if args.lite else 20
    cb_np = {m: nsn.nsn_build_codebook_host(0x4E534E00 + m, 65536, 256, 8, m == 2, iters) for m in (1, 2)}
    cbk, cbv = (torch.from_numpy(cb_np[W["mode_k"]]).to(dev), torch.from_numpy(cb_np[W["mode_v"]]).to(dev))

    rk = [synthetic.KVRecipe(synthetic.config_seed(cfg, "k", l) + rank_seed_offset(rank), H) for l in range(NL)]
    rv = [synthetic.KVRecipe(synthetic.config_seed(cfg, "v", l) + rank_seed_offset(rank), H) for l in range(NL)]
    kcs = [nsn.Cache(B, H, cap, W["window"], W["mode_k"], device=dev, double_quant=args.double_quant)
           for _ in range(NL)]
    vcs = [nsn.Cache(B, H, cap, W["window"], W["mode_v"], device=dev, double_quant=args.double_quant)
           for _ in range(NL)]
    per_token_bytes = BYTES_PER_TOKEN_DQ if args.double_quant else BYTES_PER_TOKEN
    mean_block_bytes = MEAN_BYTES_PER_BLOCK_DQ if args.double_quant else MEAN_BYTES_PER_BLOCK
    stream = torch.cuda.current_stream()

    # ---- prefill (quantizer throughput is measured on layer 0) ----
    q_tokens = 128 * ((T - 1) // 128)
    quant_ms = []
    xk = rk[0].tokens(B, T, torch.bfloat16, dev, stream_id=0)
    xv = rv[0].tokens(B, T, torch.bfloat16, dev, stream_id=0)
    for rep in range(2 if args.lite else 3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        nsn.nsn_quantize_kv(kcs[0], xk, cbk)
        nsn.nsn_quantize_kv(vcs[0], xv, cbv)
        e1.record(stream)
        torch.cuda.synchronize()
        quant_ms.append(e0.elapsed_time(e1))
    quant_ms_best = min(quant_ms[1:])
    # the first blocks of layer 0's K prefill, for the sampled parity check against the oracle
    nchk = 0 if args.lite else 8
    chk_x = xk[0, :128 * nchk, 0].float().cpu().numpy().reshape(nchk, 128, 128)
    chk_codes = codes_natural(kcs[0].codes[0, 0, :128 * nchk].cpu().numpy()).reshape(nchk, 128, 16)
    chk_signs = (kcs[0].signs[0, 0, :128 * nchk].cpu().numpy().reshape(nchk, 128, 16)
                 if W["mode_k"] == 2 else None)
    del xk, xv

    def prefill_all():
        for l in range(NL):
            nsn.nsn_quantize_kv(kcs[l], rk[l].tokens(B, T, torch.bfloat16, dev, stream_id=0), cbk)
            nsn.nsn_quantize_kv(vcs[l], rv[l].tokens(B, T, torch.bfloat16, dev, stream_id=0), cbv)

    # per-step new tokens, [layers][steps, B, H_kv, 128], and queries [layers][steps, B, H_q, 128]
    new_k = [rk[l].tokens(B, total_steps, torch.bfloat16, dev, stream_id=1).transpose(0, 1).contiguous()
             for l in range(NL)]
    new_v = [rv[l].tokens(B, total_steps, torch.bfloat16, dev, stream_id=1).transpose(0, 1).contiguous()
             for l in range(NL)]
    qs = [torch.stack([synthetic.queries(synthetic.config_seed(cfg, "q", l) + s, B, HQ, torch.bfloat16, dev)
                       for s in range(total_steps)]) for l in range(NL)]
    outs = [torch.empty((B, HQ, 128), dtype=torch.float32, device=dev) for _ in range(NL)]
    ws = nsn.decode_rope_workspace(kcs[0], HQ, dev) if args.rope else nsn.decode_workspace(kcs[0], HQ, dev)
    scale = 1.0 / math.sqrt(128)
    theta = torch.from_numpy(rope_theta()).to(dev)

    def decode_call(l, q_, out_):
        if args.rope:  # pre-RoPE keys: every key rotated at its position (two launches)
            nsn.nsn_decode_attention_rope(kcs[l], vcs[l], q_, scale, theta, cbk, cbv, out_, ws)
        else:
            nsn.nsn_decode_attention(kcs[l], vcs[l], q_, scale, cbk, cbv, out_, ws)

    for s in range(WU):
        for l in range(NL):
            nsn.nsn_append_residual(kcs[l], vcs[l], new_k[l][s], new_v[l][s], cbk, cbv)
            decode_call(l, qs[l][s], outs[l])
    # Re-prefill every layer so that the timed steps start from the workload's state:
    # a full residual window, which the first timed append flushes.
    prefill_all()
    torch.cuda.synchronize()
    nq_start, nw_start = int(kcs[0].n_quant[0, 0].item()), int(kcs[0].n_window[0, 0].item())

    # ---- timed region ----
    props = torch.cuda.get_device_properties(dev)
    try:
        gpu_id = f"{int(props.pci_domain_id):08X}:{int(props.pci_bus_id):02X}:{int(props.pci_device_id):02X}.0"
    except (AttributeError, TypeError, ValueError):
        gpu_id = str(local_rank)
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.3)
    ev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(NL)]
          for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(K):
        s = WU + i
        for l in range(NL):
            nsn.nsn_append_residual(kcs[l], vcs[l], new_k[l][s], new_v[l][s], cbk, cbv)
            ev[i][l][0].record(stream)
            decode_call(l, qs[l][s], outs[l])
            ev[i][l][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    # keep the same load for ~1 s more so that the clock sampler sees it
    soak_end = time.perf_counter() + (0.0 if args.lite else 1.0)
    while time.perf_counter() < soak_end:
        for _ in range(20):
            decode_call(0, qs[0][WU + K - 1], outs[0])
        torch.cuda.synchronize()
    clocks = sampler.stop()
    clocks["window"] = "timed region + 1 s of the same decode call right after it"

    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    decode_ms = [a.elapsed_time(b) for row in ev for a, b in row]
    ms_per_step = ms / K

    # ---- algorithmic bytes of one decode call, averaged over the timed steps ----
    # The (n_quant, n_window) of every step follow from the state before the timed
    # region: each append first flushes a full window into one quantized block.
    seqs = B * H
    per_tok = per_token_bytes[W["mode_k"]] + per_token_bytes[W["mode_v"]]

    def call_bytes(nq_s, nw_s):
        compressed_s = seqs * (nq_s * per_tok + 2 * (nq_s // 128) * mean_block_bytes)
        return compressed_s + seqs * 2 * nw_s * 128 * 2 + B * HQ * 128 * (2 + 4)

    nq_s, nw_s, step_bytes = nq_start, nw_start, []
    for _ in range(K):
        if nw_s >= W["window"]:
            nq_s, nw_s = nq_s + 128, 0
        nw_s += 1
        step_bytes.append(call_bytes(nq_s, nw_s))
    nq, nw = int(kcs[0].n_quant[0, 0].item()), int(kcs[0].n_window[0, 0].item())
    assert (nq, nw) == (nq_s, nw_s), "counter schedule differs from the cache state"
    compressed = NL * seqs * (nq * per_tok + 2 * (nq // 128) * mean_block_bytes)
    decode_bytes = float(np.mean(step_bytes))          # per decode call (one layer)
    dec_avg_ms = float(np.mean(decode_ms))
    peaks, peak_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    achieved = decode_bytes / (dec_avg_ms * 1e-3) / 1e9

    # ---- end to end through the public API with host buffers, over the same K steps ----
    e2e_ms, h2d, d2h = 0.0, 0, 0
    if not args.lite:
        pin_k = [t.cpu().pin_memory() for t in new_k]
        pin_v = [t.cpu().pin_memory() for t in new_v]
        pin_q = [t.cpu().pin_memory() for t in qs]
        # Pipelined like a serving loop: step s+1's inputs go up on one copy
        # stream and step s-1's outputs come down on another while step s runs;
        # device inputs and outputs are double-buffered and ordered by events.
        host_out = [[torch.empty((B, HQ, 128), dtype=torch.float32).pin_memory() for _ in range(NL)]
                    for _ in range(2)]
        d_in = [[(torch.empty_like(new_k[0][0]), torch.empty_like(new_v[0][0]), torch.empty_like(qs[0][0]))
                 for _ in range(NL)] for _ in range(2)]
        d_out = [[torch.empty((B, HQ, 128), dtype=torch.float32, device=dev) for _ in range(NL)] for _ in range(2)]
        up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of a buffer are on the device
        ev_done = [torch.cuda.Event() for _ in range(2)]   # the step using a buffer has finished
        ev_out = [torch.cuda.Event() for _ in range(2)]    # the outputs of a buffer are on the host
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        up.wait_event(e0)
        down.wait_event(e0)
        for i in range(e2e_steps):
            s, j = WU + K + i, i % 2
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(ev_done[j])
                for l in range(NL):
                    for dst, src in zip(d_in[j][l], (pin_k[l][s], pin_v[l][s], pin_q[l][s])):
                        dst.copy_(src, non_blocking=True)
                ev_in[j].record(up)
            stream.wait_event(ev_in[j])
            if i >= 2:
                stream.wait_event(ev_out[j])
            for l in range(NL):
                dk, dv, dq = d_in[j][l]
                nsn.nsn_append_residual(kcs[l], vcs[l], dk, dv, cbk, cbv)
                decode_call(l, dq, d_out[j][l])
            ev_done[j].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev_done[j])
                for l in range(NL):
                    host_out[j][l].copy_(d_out[j][l], non_blocking=True)
                ev_out[j].record(down)
        for j in range(2):
            stream.wait_event(ev_out[j])
        e1.record(stream)
        torch.cuda.synchronize()
        h2d = int(NL * sum(t.numel() * t.element_size() for t in d_in[0][0]))
        d2h = int(NL * d_out[0][0].numel() * d_out[0][0].element_size())
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)

    status = 0
    for c in kcs + vcs:
        status |= int(c.status.item())

    # ---- quantizer rooflines (prefill of one layer, K + V) ----
    # HBM: bf16 tokens in (256 B per token-head) plus the compressed cache out.
    # Tensor: the exhaustive search is a dense contraction (16 sub-vectors x 256
    # codewords x 8 dims per token-head) run on the tensor cores with fp16
    # operands; its algorithmic FLOPs against the measured dense 16-bit peak.
    qtoken_heads = 2 * B * H * q_tokens
    q_bytes = B * H * q_tokens * (2 * 256 + (per_token_bytes[W["mode_k"]] + per_token_bytes[W["mode_v"]])) \
        + 2 * B * H * (q_tokens // 128) * mean_block_bytes
    mac_per_th = 16 * 256 * 8
    tc_peak = float(peaks["bf16_tflops"])
    q_ach = qtoken_heads * 2 * mac_per_th / (quant_ms_best * 1e-3) / 1e12

    if rank == 0 and args.lite:
        print(json.dumps({"lite": True, "workload": W["name"], "batch": B, "steps": K, "ms_per_step": ms_per_step,
                          "decode_call_ms": dec_avg_ms, "decode_gbs": achieved, "quantize_ms": quant_ms_best,
                          "cache_status": status}), flush=True)
    elif rank == 0:
        cpu_t, cpu_n, cpu_threads = oracle_decode_sample(float(os.environ.get("NSN_CPU_BUDGET_S", "15")),
                                                         rope=args.rope, W=W)
        cpu_step = cpu_t * B * H * NL
        cq_t, cq_n, ck_sub, ck_tie, ck_bad, ck_sbad = oracle_quantize_check(
            chk_x, cb_np[W["mode_k"]], W["mode_k"], chk_codes, chk_signs, 8.0)
        modes = f"K {W['mode_k']}-bit + V {W['mode_v']}-bit"
        line = {
            "metric": METRIC,
            "value": job_throughput(B * K, world, ms),
            "unit": "tokens/s",
            "n_gpus": world, "steps": K, "warmup": WU, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {**config_dict(W, args, world, B),
                       "l2": f"inputs larger than L2 (compressed cache {compressed / 1e6:.0f} MB per step)"},
            "compressed_kv_gbs": NL * decode_bytes / (ms_per_step * 1e-3) / 1e9,
            "decode_call_ms": dec_avg_ms,
            "roofline": {"kernel": ("rope_scores_kernel + decode_kernel (two launches per decode call; "
                                    "the logits kernel is issue-bound)") if args.rope
                         else "decode_kernel (one launch per decode call)", "bound": "hbm",
                         "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                         "peak_kind": peak_kind,
                         "traffic": None if (args.double_quant or args.rope or args.workload != 3)
                         else decode_traffic(),
                         "algorithmic_bytes_per_launch": decode_bytes,
                         "frac_of_8tbs_spec": achieved / 8000.0},
            "quantize": {"workload": f"prefill {B}x{q_tokens} tokens x {H} kv-heads, {modes}, bf16 in"
                                     + (" (one of the 32 layers)" if NL > 1 else ""),
                         "tokens_per_s": B * q_tokens / (quant_ms_best * 1e-3),
                         "token_heads_per_s": qtoken_heads / (quant_ms_best * 1e-3),
                         "ms": quant_ms_best, "gbs": q_bytes / (quant_ms_best * 1e-3) / 1e9,
                         "hbm_frac": q_bytes / (quant_ms_best * 1e-3) / 1e9 / hbm,
                         "hbm_frac_of_8tbs_spec": q_bytes / (quant_ms_best * 1e-3) / 1e9 / 8000.0,
                         "roofline": {"kernel": "quantize_prefill_ws_kernel", "bound": "tensor", "achieved": q_ach,
                                      "peak": tc_peak, "unit": "TFLOP/s", "frac": q_ach / tc_peak,
                                      "peak_kind": peak_kind,
                                      "algorithmic_flop_per_token_head": 2 * mac_per_th,
                                      "note": "scores on the tensor cores (tcgen05, fp16 hi+lo operand plus a "
                                              "bias MMA, so the MMAs do four times the algorithmic FLOPs); the "
                                              "kernel is bound by issue and latency, not by the tensor pipe"},
                         "parity_sample": {"blocks": cq_n, "sub_vectors": ck_sub, "oracle_near_ties": ck_tie,
                                           "code_mismatches_outside_near_ties": ck_bad,
                                           "sign_byte_mismatches": ck_sbad,
                                           "what": "the first 128-token blocks of layer 0's K prefill "
                                                   "(sequence 0, kv-head 0) re-quantized by the oracle from "
                                                   "the same bf16 tokens and codebook"}},
            "e2e": {"value": job_throughput(B * e2e_steps, world, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "copies": "every step: its new K/V tokens and q (every layer) from pinned host memory, its "
                              "outputs back; uploads of step s+1 and the download of step s-1 overlap step s"},
            "gpu_launches": K * NL * (LAUNCHES_PER_STEP + (1 if args.rope else 0)),
            "clocks": clocks,
            "cache_status": status,
            "cpu_baseline": {"value": B / cpu_step, "unit": "tokens/s", "cores": cpu_threads, "kind": "oracle",
                             "sample": f"oracle decode attention of {cpu_n} sampled (batch, kv-head) sequences "
                                       f"({nq} quantized + 128 window tokens, {g} q-heads) scaled to "
                                       f"{B}x{H} sequences x {NL} layer(s) per step",
                             "quantize_token_heads_per_s": 128 / cq_t,
                             "quantize_sample": f"{cq_n} oracle 128-token blocks of the timed prefill"},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=64)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--batch", type=int, default=0, help="override the batch (profiling runs)")
    ap.add_argument("--double-quant", action="store_true",
                    help="the same workload with double quantization (4-bit s1 and o)")
    ap.add_argument("--rope", action="store_true",
                    help="the same workload with pre-RoPE keys (every key rotated at its position at decode)")
    ap.add_argument("--lite", action="store_true",
                    help="profiling run: no e2e leg, no clock soak, no CPU baseline; short summary line")
    ap.add_argument("--workload", type=int, default=3, choices=sorted(WORKLOADS),
                    help="3: decode-throughput layer (default); 4: extreme compression, 32 layers; "
                         "5: long context")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
