"""Benchmark of the NSNQuant KV hot path on B200.

Default workload (one GPU): the decode-throughput layer -- batch 16, 32 query /
8 KV heads, head_dim 128, 32768-token context per sequence quantized to 2-bit K
and V with a 128-token fp16 residual window.  One timed step = one decode step
of the whole batch: append one new K/V token per (sequence, kv-head) (flushing
the full window through the quantizer on the first step) + decode attention of
all 32 query heads.  `value` = generated tokens/s = batch * steps / time.

The same JSON line also carries the compressed-KV GB/s, the roofline of the
decode call, the prefill quantizer's throughput (tokens/s) with its own ALU
roofline, an end-to-end number through the public API with host buffers, the
SM clocks seen during the timed region, and the CPU oracle baseline.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
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
WORKLOAD = dict(config=3, name="decode-b16-32k-2bit", batch=16, n_kv_heads=8, n_q_heads=32, seq=32768,
                mode_k=2, mode_v=2, window=128)
BYTES_PER_TOKEN = {1: 16 + 4, 2: 16 + 16 + 4}   # codes (+ signs) + (s1, s2) per token-head
MEAN_BYTES_PER_BLOCK = 128 * 2
# With double quantization s1 is a 4-bit level (0.5 B) next to fp16 alpha*s2, and a
# block's o is 64 B of levels plus 16 B of (lo, hi) parameters.
BYTES_PER_TOKEN_DQ = {1: 16 + 2.5, 2: 16 + 16 + 2.5}
MEAN_BYTES_PER_BLOCK_DQ = 64 + 16
# Kernels one decode step launches: append_kernel (K and V, flush included) and
# decode_kernel (splits, residual window and merge).
LAUNCHES_PER_STEP = 2
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0}


# DRAM bytes (read + write) per decode_kernel launch on this workload, from one
# ncu capture (dram__bytes_read.sum + dram__bytes_write.sum of the launch list of
# this workload, taken with --metrics and --clock-control none), valid only for the sources the
# decode kernel is compiled from with this SHA-256 (decode.cu, nsn_common.cuh,
# comments and whitespace removed).
# Any later change to those files makes the figure stale; the bench then reports null.
DECODE_TRAFFIC = {"sha256": "ea241b89a8f2a1e6dad9d25fdcf849fe9ecc0b2c00ca6d3ef9d8527751ea33b8",
                  "bytes_per_launch": (321008128 + 321048320) // 2 + (4360704 + 441856) // 2}


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


def oracle_decode_sample(budget_s: float, seed: int = 0, rope: bool = False):
    """Times the oracle's decode attention (pre-RoPE keys with `rope`) for sampled
    (b, kv-head) sequences of the workload shape (random compressed contents,
    2-bit K/V, full window).  Returns (seconds per (b, kv-head), sequences timed,
    threads)."""
    from calibration_free_vector_b200 import synthetic
    from oracle import nsn_oracle as orc
    try:
        from threadpoolctl import threadpool_info
        threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    except Exception:  # pragma: no cover
        threads = 1
    W = WORKLOAD
    nq = W["seq"] - 128
    g = W["n_q_heads"] // W["n_kv_heads"]
    cbk = np.abs(np.random.RandomState(seed).normal(size=(256, 8)))
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
                                      vc["window"].astype(np.float64), cbk, cbk, W["mode_k"], W["mode_v"],
                                      1 / math.sqrt(128), rope_theta().astype(np.float64))
        else:
            orc.decode_attention(q, f(kc), f(vc), kc["window"].astype(np.float64), vc["window"].astype(np.float64),
                                 cbk, cbk, W["mode_k"], W["mode_v"], 1 / math.sqrt(128))
        times.append(time.perf_counter() - t0)
        n += 1
        if time.perf_counter() - t_start > budget_s or n >= 64:
            break
    return float(np.mean(times)), n, threads


def oracle_quantize_sample(budget_s: float, seed: int = 0):
    """Times the oracle quantizing sampled 128-token blocks of the workload's K
    (2-bit).  Returns (seconds per block, blocks timed)."""
    import torch
    from calibration_free_vector_b200 import synthetic
    from oracle import nsn_oracle as orc
    cb = np.abs(np.random.RandomState(seed).normal(size=(256, 8)))
    x = synthetic.KVRecipe(seed, 1).tokens(1, 128 * 8, torch.bfloat16, "cpu").float().numpy()[0, :, 0]
    times = []
    t_start = time.perf_counter()
    for i in range(8):
        t0 = time.perf_counter()
        orc.quantize_block(x[128 * i:128 * (i + 1)].astype(np.float64), cb, 2)
        times.append(time.perf_counter() - t0)
        if time.perf_counter() - t_start > budget_s:
            break
    return float(np.mean(times)), len(times)


def run_reference(args):
    """--impl reference: the CPU oracle on the host cores, same metric/unit."""
    rank, _, world = dist_env()
    if rank != 0:
        return 0
    W = WORKLOAD
    per_seq = []
    for _ in range(args.warmup):
        oracle_decode_sample(0.0, seed=99, rope=args.rope)
    threads = 1
    per_step_budget = min(5.0, 100.0 / max(1, args.steps))
    for s in range(args.steps):
        t, n, threads = oracle_decode_sample(per_step_budget, seed=s, rope=args.rope)
        per_seq.append(t)
    step_s = float(np.mean(per_seq)) * W["batch"] * W["n_kv_heads"]
    value = W["batch"] / step_s
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": W["name"] + ("-dq" if args.double_quant else "") + ("-prerope" if args.rope else ""),
                   "batch": W["batch"], "seq_len": W["seq"], "n_q_heads": W["n_q_heads"],
                   "n_kv_heads": W["n_kv_heads"], "mode_k": W["mode_k"], "mode_v": W["mode_v"],
                   "window": W["window"], "double_quant": bool(args.double_quant), "pre_rope_keys": bool(args.rope),
                   "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
                         "sample": f"each step: oracle decode attention{' (pre-RoPE keys)' if args.rope else ''} "
                                   f"of >=1 sampled (batch, kv-head) "
                                   f"sequence ({W['seq'] - 128} quantized + 128 window tokens, 4 q-heads), "
                                   f"scaled to {W['batch']}x{W['n_kv_heads']} sequences"},
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

    W = WORKLOAD
    B, H, HQ, T = args.batch or W["batch"], W["n_kv_heads"], W["n_q_heads"], W["seq"]
    g = HQ // H
    K, WU = args.steps, args.warmup
    e2e_steps = 0 if args.lite else max(4, K // 2)
    total_steps = WU + K + e2e_steps
    cap = ((T + K + e2e_steps + 255) // 128) * 128

    # codebooks from the host builder (k-means on seeded randn)
    iters = 3 if args.lite else 20
    cbk_np = nsn.nsn_build_codebook_host(0x4E534E02, 65536, 256, 8, W["mode_k"] == 2, iters)
    cbv_np = nsn.nsn_build_codebook_host(0x4E534E02 if W["mode_v"] == 2 else 0x4E534E01, 65536, 256, 8,
                                         W["mode_v"] == 2, iters)
    cbk, cbv = torch.from_numpy(cbk_np).to(dev), torch.from_numpy(cbv_np).to(dev)

    rk = synthetic.KVRecipe(synthetic.config_seed(3, "k") + rank_seed_offset(rank), H)
    rv = synthetic.KVRecipe(synthetic.config_seed(3, "v") + rank_seed_offset(rank), H)
    kc = nsn.Cache(B, H, cap, W["window"], W["mode_k"], device=dev, double_quant=args.double_quant)
    vc = nsn.Cache(B, H, cap, W["window"], W["mode_v"], device=dev, double_quant=args.double_quant)
    per_token_bytes = BYTES_PER_TOKEN_DQ if args.double_quant else BYTES_PER_TOKEN
    mean_block_bytes = MEAN_BYTES_PER_BLOCK_DQ if args.double_quant else MEAN_BYTES_PER_BLOCK
    stream = torch.cuda.current_stream()

    # ---- prefill (quantizer throughput is measured here) ----
    xk = rk.tokens(B, T, torch.bfloat16, dev, stream_id=0)
    xv = rv.tokens(B, T, torch.bfloat16, dev, stream_id=0)
    q_tokens = 128 * ((T - 1) // 128)
    quant_ms = []
    for rep in range(2 if args.lite else 3):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        e0.record(stream)
        nsn.nsn_quantize_kv(kc, xk, cbk)
        nsn.nsn_quantize_kv(vc, xv, cbv)
        e1.record(stream)
        torch.cuda.synchronize()
        quant_ms.append(e0.elapsed_time(e1))
    quant_ms_best = min(quant_ms[1:])
    # per-step new tokens, [steps, B, H_kv, 128]
    new_k = rk.tokens(B, total_steps, torch.bfloat16, dev, stream_id=1).transpose(0, 1).contiguous()
    new_v = rv.tokens(B, total_steps, torch.bfloat16, dev, stream_id=1).transpose(0, 1).contiguous()
    qs = torch.stack([synthetic.queries(synthetic.config_seed(3, "q") + s, B, HQ, torch.bfloat16, dev)
                      for s in range(total_steps)])
    del xk, xv
    out = torch.empty((B, HQ, 128), dtype=torch.float32, device=dev)
    ws = nsn.decode_rope_workspace(kc, HQ, dev) if args.rope else nsn.decode_workspace(kc, HQ, dev)
    scale = 1.0 / math.sqrt(128)
    theta = torch.from_numpy(rope_theta()).to(dev)

    def decode_call(q_, out_):
        if args.rope:  # pre-RoPE keys: every key rotated at its position (two launches)
            nsn.nsn_decode_attention_rope(kc, vc, q_, scale, theta, cbk, cbv, out_, ws)
        else:
            nsn.nsn_decode_attention(kc, vc, q_, scale, cbk, cbv, out_, ws)

    def step(s):
        nsn.nsn_append_residual(kc, vc, new_k[s], new_v[s], cbk, cbv)
        decode_call(qs[s], out)

    for s in range(WU):
        step(s)
    # Re-prefill so that the timed steps start from the workload's state: a full
    # residual window, which the first timed append flushes (then one flush per
    # 128 steps, as in the 64-step decode-throughput run).
    nsn.nsn_quantize_kv(kc, rk.tokens(B, T, torch.bfloat16, dev, stream_id=0), cbk)
    nsn.nsn_quantize_kv(vc, rv.tokens(B, T, torch.bfloat16, dev, stream_id=0), cbv)
    torch.cuda.synchronize()
    nq_start, nw_start = int(kc.n_quant[0, 0].item()), int(kc.n_window[0, 0].item())

    # ---- timed region ----
    props = torch.cuda.get_device_properties(dev)
    try:
        gpu_id = f"{int(props.pci_domain_id):08X}:{int(props.pci_bus_id):02X}:{int(props.pci_device_id):02X}.0"
    except (AttributeError, TypeError, ValueError):
        gpu_id = str(local_rank)
    sampler = ClockSampler(gpu_id)
    sampler.start()
    time.sleep(0.3)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    t0.record(stream)
    for i in range(K):
        s = WU + i
        nsn.nsn_append_residual(kc, vc, new_k[s], new_v[s], cbk, cbv)
        ev[i][0].record(stream)
        decode_call(qs[s], out)
        ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    # keep the same load for ~1 s more so that the clock sampler sees it
    soak_end = time.perf_counter() + (0.0 if args.lite else 1.0)
    while time.perf_counter() < soak_end:
        for _ in range(20):
            decode_call(qs[WU + K - 1], out)
        torch.cuda.synchronize()
    clocks = sampler.stop()
    clocks["window"] = "timed region + 1 s of the same decode call right after it"

    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    decode_ms = [a.elapsed_time(b) for a, b in ev]
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
    nq, nw = int(kc.n_quant[0, 0].item()), int(kc.n_window[0, 0].item())
    assert (nq, nw) == (nq_s, nw_s), "counter schedule differs from the cache state"
    compressed = seqs * (nq * per_tok + 2 * (nq // 128) * mean_block_bytes)
    decode_bytes = float(np.mean(step_bytes))
    dec_avg_ms = float(np.mean(decode_ms))
    peaks, peak_kind = load_peaks()
    hbm = float(peaks["hbm_gbs"])
    achieved = decode_bytes / (dec_avg_ms * 1e-3) / 1e9

    # ---- end to end through the public API with host buffers ----
    e2e_ms, h2d, d2h = 0.0, 0, 0
    if not args.lite:
        pin_k = new_k.cpu().pin_memory()
        pin_v = new_v.cpu().pin_memory()
        pin_q = qs.cpu().pin_memory()
        # Pipelined like a serving loop: step s+1's inputs go up on one copy
        # stream and step s-1's output comes down on another while step s runs;
        # device inputs and outputs are double-buffered and ordered by events.
        host_out = [torch.empty((B, HQ, 128), dtype=torch.float32).pin_memory() for _ in range(2)]
        d_in = [(torch.empty_like(new_k[0]), torch.empty_like(new_v[0]), torch.empty_like(qs[0])) for _ in range(2)]
        d_out = [torch.empty((B, HQ, 128), dtype=torch.float32, device=dev) for _ in range(2)]
        up, down = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]     # inputs of a buffer are on the device
        ev_done = [torch.cuda.Event() for _ in range(2)]   # the step using a buffer has finished
        ev_out = [torch.cuda.Event() for _ in range(2)]    # the output of a buffer is on the host
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
                for dst, src in zip(d_in[j], (pin_k[s], pin_v[s], pin_q[s])):
                    dst.copy_(src, non_blocking=True)
                ev_in[j].record(up)
            stream.wait_event(ev_in[j])
            if i >= 2:
                stream.wait_event(ev_out[j])
            dk, dv, dq = d_in[j]
            nsn.nsn_append_residual(kc, vc, dk, dv, cbk, cbv)
            decode_call(dq, d_out[j])
            ev_done[j].record(stream)
            with torch.cuda.stream(down):
                down.wait_event(ev_done[j])
                host_out[j].copy_(d_out[j], non_blocking=True)
                ev_out[j].record(down)
        for j in range(2):
            stream.wait_event(ev_out[j])
        e1.record(stream)
        torch.cuda.synchronize()
        h2d = int(sum(t.numel() * t.element_size() for t in d_in[0]))
        d2h = int(d_out[0].numel() * d_out[0].element_size())
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world, dev)

    status = int(kc.status.item()) | int(vc.status.item())

    # ---- quantizer roofline: the exhaustive search is a dense contraction
    # (16 sub-vectors x 256 codewords x 8 dims per token-head) run on the tensor
    # cores with fp16 operands; its algorithmic FLOPs against the measured dense
    # 16-bit tensor peak (fp16 and bf16 run at the same rate) ----
    qtoken_heads = 2 * B * H * q_tokens
    q_bytes = B * H * q_tokens * (2 * 256 + (per_token_bytes[W["mode_k"]] + per_token_bytes[W["mode_v"]])) \
        + 2 * B * H * (q_tokens // 128) * mean_block_bytes
    mac_per_th = 16 * 256 * 8
    tc_peak = float(peaks["bf16_tflops"])
    q_ach = qtoken_heads * 2 * mac_per_th / (quant_ms_best * 1e-3) / 1e12

    if rank == 0 and args.lite:
        print(json.dumps({"lite": True, "batch": B, "steps": K, "ms_per_step": ms_per_step,
                          "decode_call_ms": dec_avg_ms, "decode_gbs": achieved, "quantize_ms": quant_ms_best,
                          "cache_status": int(kc.status.item()) | int(vc.status.item())}), flush=True)
    elif rank == 0:
        cpu_t, cpu_n, cpu_threads = oracle_decode_sample(float(os.environ.get("NSN_CPU_BUDGET_S", "15")),
                                                         rope=args.rope)
        cpu_step = cpu_t * B * H
        cq_t, cq_n = oracle_quantize_sample(8.0)
        line = {
            "metric": METRIC,
            "value": job_throughput(B * K, world, ms),
            "unit": "tokens/s",
            "n_gpus": world, "steps": K, "warmup": WU, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": W["name"] + ("-dq" if args.double_quant else "") + ("-prerope" if args.rope else ""),
                       "batch": B, "seq_len": T, "n_q_heads": HQ, "n_kv_heads": H,
                       "double_quant": bool(args.double_quant),
                       "pre_rope_keys": bool(args.rope), **({"rope_theta_base": 500000.0} if args.rope else {}),
                       "head_dim": 128, "mode_k": W["mode_k"], "mode_v": W["mode_v"], "window": W["window"],
                       "parallelism": "replicas" if world > 1 else "single",
                       "l2": f"inputs larger than L2 (compressed cache {compressed / 1e6:.0f} MB per step)"},
            "compressed_kv_gbs": decode_bytes / (ms_per_step * 1e-3) / 1e9,
            "decode_call_ms": dec_avg_ms,
            "roofline": {"kernel": ("rope_scores_kernel + decode_kernel (two launches per decode call; "
                                    "the logits kernel is issue-bound)") if args.rope
                         else "decode_kernel (one launch per decode call)", "bound": "hbm",
                         "achieved": achieved, "peak": hbm, "unit": "GB/s", "frac": achieved / hbm,
                         "peak_kind": peak_kind,
                         "traffic": None if (args.double_quant or args.rope) else decode_traffic(),
                         "algorithmic_bytes_per_launch": decode_bytes,
                         "frac_of_8tbs_spec": achieved / 8000.0},
            "quantize": {"workload": f"prefill {B}x{q_tokens} tokens x {H} kv-heads, K 2-bit + V 2-bit, bf16 in",
                         "tokens_per_s": B * q_tokens / (quant_ms_best * 1e-3),
                         "token_heads_per_s": qtoken_heads / (quant_ms_best * 1e-3),
                         "ms": quant_ms_best, "gbs": q_bytes / (quant_ms_best * 1e-3) / 1e9,
                         "hbm_frac": q_bytes / (quant_ms_best * 1e-3) / 1e9 / hbm,
                         "hbm_frac_of_8tbs_spec": q_bytes / (quant_ms_best * 1e-3) / 1e9 / 8000.0,
                         "roofline": {"kernel": "quantize_prefill_kernel", "bound": "tensor", "achieved": q_ach,
                                      "peak": tc_peak, "unit": "TFLOP/s", "frac": q_ach / tc_peak,
                                      "peak_kind": peak_kind,
                                      "algorithmic_flop_per_token_head": 2 * mac_per_th,
                                      "note": "scores on the tensor cores (fp16 hi+lo operand, so the MMAs do "
                                              "twice the algorithmic FLOPs); the kernel is bound by issue and "
                                              "latency, not by the tensor pipe"}},
            "e2e": {"value": job_throughput(B * e2e_steps, world, e2e_ms), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "copies": "every step: its new K/V token and q from pinned host memory, its output back; "
                              "uploads of step s+1 and the download of step s-1 overlap step s"},
            "gpu_launches": K * (LAUNCHES_PER_STEP + (1 if args.rope else 0)),
            "clocks": clocks,
            "cache_status": status,
            "cpu_baseline": {"value": B / cpu_step, "unit": "tokens/s", "cores": cpu_threads, "kind": "oracle",
                             "sample": f"oracle decode attention of {cpu_n} sampled (batch, kv-head) sequences "
                                       f"({nq} quantized + 128 window tokens, {g} q-heads) scaled to "
                                       f"{B}x{H} sequences per step",
                             "quantize_token_heads_per_s": 128 / cq_t,
                             "quantize_sample": f"{cq_n} oracle 128-token 2-bit blocks"},
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
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
