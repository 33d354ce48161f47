#!/usr/bin/env python
"""Benchmark of the attention hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
  1. prefill attention forward on the GQA causal 2K workload
     (B=4, Hq=32, Hkv=8, Nq=Nk=2048, d=128, bf16, causal), then
  2. one paged-KV decode step on the 64-sequence workload
     (Hq=64, Hkv=8, d=128, 16-token pages, lengths uniform in [512, 32768]).
The decode streams about 4.6 GB of cached K/V, far more than the 126 MB L2, so every
prefill launch starts with a cold L2 for its own inputs.

Printed (rank 0, one JSON line): prefill TFLOP/s as `value` (causal FLOPs counted as
half of 4*B*Hq*Nq*Nk*d), the decode KV-read GB/s in `decode`, roofline fractions
against MEASURED_PEAKS.json, the end-to-end figures through the public API with host
buffers (`e2e` for the prefill, `decode.e2e` for the decode; two buffer slots overlap
the copies of neighbouring steps with the kernel, and the back-to-back figure is kept
beside it as `sequential`), the fp64 CPU oracle timed
on a bounded sample (`cpu_baseline`), and the SM clocks sampled during the run.  After
the timed step, the other prefill configurations (the tiny d=64 case, the 16K
long-context case and the peaked d=256 case) are each timed on their own, L2 flushed
before every launch, and reported under `workloads` with their own roofline, clocks
and CPU baseline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload serving_step|gqa_causal_16k|peaked_mha_d256|tiny_mha_d64]

With N > 1 (launched by torchrun, one process per GPU) every rank runs its own
independent copy of the workload (weak scaling: the path shards into independent
problems and has no exchange step); times are the maximum over ranks.
"""

from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from attn_fwd_05_b200 import counts, synth  # noqa: E402

METRIC = "attn fwd TFLOPS & % of BF16 tensor peak; paged decode KV-read GB/s & % HBM"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=200)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="serving_step",
                   choices=["serving_step", "gqa_causal_16k", "peaked_mha_d256", "tiny_mha_d64", "gqa_causal_2k",
                            "gqa_causal_2k_bwd", "gqa_causal_16k_bwd", "gqa_causal_2k_fp8", "gqa_causal_16k_fp8"])
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--cpu-seconds", type=float, default=10.0, help="bounded CPU-baseline sample length")
    p.add_argument("--decode-seqs", type=int, default=64,
                   help="sequences in the decode batch (64 is the workload; fewer only for small profiles)")
    p.add_argument("--no-other-workloads", action="store_true",
                   help="serving step only: skip the per-workload records of the other prefill configs")
    return p.parse_args()


CSRC = ("attn_api.cu", "backward_sm100.cuh", "decode_sm100.cuh", "fwd_fp8_sm100.cuh", "prefill_d256_sm100.cuh",
        "prefill_sm100.cuh", "sm100_common.cuh")


# the sources each committed ncu summary's kernel is built from (kernel header, shared
# device helpers, host launch code)
PROFILE_SOURCES = {
    "attn_fwd_pingpong_gqa_causal_2k.md": ("attn_api.cu", "prefill_sm100.cuh", "sm100_common.cuh"),
    "attn_fwd_pingpong_gqa_causal_16k.md": ("attn_api.cu", "prefill_sm100.cuh", "sm100_common.cuh"),
    "attn_fwd_single_peaked_mha_d256.md": ("attn_api.cu", "prefill_d256_sm100.cuh", "prefill_sm100.cuh",
                                           "sm100_common.cuh"),
    "attn_decode_split_paged_decode.md": ("attn_api.cu", "decode_sm100.cuh", "sm100_common.cuh"),
    "attn_bwd_gqa_causal_2k.md": ("attn_api.cu", "backward_sm100.cuh", "sm100_common.cuh"),
    "attn_fwd_fp8_gqa_causal_2k.md": ("attn_api.cu", "fwd_fp8_sm100.cuh", "sm100_common.cuh"),
    "attn_fwd_fp8_gqa_causal_16k.md": ("attn_api.cu", "fwd_fp8_sm100.cuh", "sm100_common.cuh"),
    "attn_bwd_gqa_causal_16k.md": ("attn_api.cu", "backward_sm100.cuh", "sm100_common.cuh"),
}


def csrc_digest(files=CSRC) -> str:
    """sha256 prefix of kernel sources without their comments and blank space, to match
    against the committed ncu summaries (a comment edit does not change the kernels)."""
    import hashlib
    import re
    h = hashlib.sha256()
    for name in files:
        with open(os.path.join(ROOT, "attn_fwd_05_b200", "csrc", name)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


# committed ncu summary of the prefill kernel, per workload
PREFILL_PROFILES = {
    "serving_step": "attn_fwd_pingpong_gqa_causal_2k.md",
    "gqa_causal_2k": "attn_fwd_pingpong_gqa_causal_2k.md",
    "gqa_causal_16k": "attn_fwd_pingpong_gqa_causal_16k.md",
    "peaked_mha_d256": "attn_fwd_single_peaked_mha_d256.md",
}


def profiled_traffic(profile: str, scale: float = 1.0):
    """DRAM bytes per launch from a committed ncu summary, or None when the kernel sources
    changed since it was captured (its counters no longer describe the current kernels)."""
    path = os.path.join(ROOT, "profiles", profile)
    try:
        text = open(path).read()
    except OSError:
        return None
    import re
    m_sha = re.search(r"csrc sha256 prefix `([0-9a-f]+)`", text)
    m_b = re.search(r"traffic_bytes_per_launch: (\d+)", text)
    if not (m_sha and m_b) or m_sha.group(1) != csrc_digest(PROFILE_SOURCES.get(profile, CSRC)):
        return None
    return int(m_b.group(1)) * scale


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS if k in d}, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


# ----------------------------------------------------------------------------- distributed

class Dist:
    def __init__(self):
        self.world = int(os.environ.get("WORLD_SIZE", "1"))
        self.rank = int(os.environ.get("RANK", "0"))
        self.local = int(os.environ.get("LOCAL_RANK", "0"))
        self.on = self.world > 1

    def init(self, backend="nccl"):
        self.backend = backend
        if self.on:
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=300),
                                    device_id=torch.device("cuda", self.local) if backend == "nccl" else None)

    def barrier(self):
        if self.on:
            import torch.distributed as dist
            dist.barrier()

    def max(self, x: float) -> float:
        """The maximum of x over all ranks (timings are reported as the slowest rank's)."""
        if not self.on:
            return x
        import torch.distributed as dist
        dev = torch.device("cuda", self.local) if getattr(self, "backend", "nccl") == "nccl" else torch.device("cpu")
        t = torch.tensor([x], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.on:
            import torch.distributed as dist
            dist.destroy_process_group()


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock/throttle sampling in the background while the GPU works."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,utilization.gpu,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.proc = None
        self.path = None
        try:
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
        except Exception:
            uuid = str(device_index)
        self.uuid = uuid

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.uuid, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        # nvidia-smi takes a while to start: wait (up to 3 s) for its first sample, so that a
        # short timed region is still sampled
        t0 = time.perf_counter()
        while time.perf_counter() - t0 < 3.0 and self.proc.poll() is None:
            if os.path.getsize(self.path) > 0:
                break
            time.sleep(0.01)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.12)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 10:
                    rows.append(parts)
        os.unlink(self.path)
        busy = [r for r in rows if _num(r[4]) and _num(r[4]) > 0] or rows
        sm = [_num(r[1]) for r in busy if _num(r[1])]
        mx = [_num(r[2]) for r in busy if _num(r[2])]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in busy for i in range(4) if r[6 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(busy),
                "power_w_max": max((_num(r[3]) or 0.0) for r in busy) if busy else None}


def _num(s):
    try:
        return float(s)
    except Exception:
        return None


# ----------------------------------------------------------------------------- workloads

def rank_seed(base: int, rank: int) -> int:
    """Each rank draws an independent problem of the same shape (weak scaling)."""
    return base + 7919 * rank


def prefill_shape(name: str):
    return synth.WORKLOADS["gqa_causal_2k" if name == "serving_step" else name]


def make_prefill(shape, seed, dev):
    q, k, v = synth.prefill_inputs(shape, seed)
    o = torch.empty((shape.B, shape.Hq, shape.Nq, shape.d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((shape.B, shape.Hq, shape.Nq), dtype=torch.float32, device=dev)
    return {"host": (q, k, v), "dev": (q.to(dev), k.to(dev), v.to(dev)), "o": o, "lse": lse}


def make_decode(seed, dev, nseqs=64):
    import dataclasses

    import attn_fwd_05_b200 as ab
    s = dataclasses.replace(synth.WORKLOADS["paged_decode_gqa"], S=nseqs)
    kv = synth.decode_inputs(s, seed)
    S = s.S
    ws_bytes = ab.attn_decode_paged_workspace_size(S, s.Hq, s.Hkv, s.d, kv.max_pages_per_seq, s.page_size)
    return {
        "kv": kv, "shape": s,
        "q": kv.q.to(dev), "k_pool": kv.k_pool.to(dev), "v_pool": kv.v_pool.to(dev),
        "table": kv.block_table.to(dev), "lens": kv.seq_lens.to(dev),
        "o": torch.empty((S, s.Hq, s.d), dtype=torch.bfloat16, device=dev),
        "lse": torch.empty((S, s.Hq), dtype=torch.float32, device=dev),
        "ws": torch.empty(ws_bytes, dtype=torch.uint8, device=dev),
        "kv_bytes": counts.decode_kv_bytes(kv.seq_lens.tolist(), s.Hkv, s.d),
    }


# ----------------------------------------------------------------------------- CPU oracle (baseline / reference arm)

def oracle_prefill_sample(shape, q, k, v, seconds: float, max_heads=None):
    """Time the fp64 oracle on whole heads of the workload until `seconds` have passed."""
    from oracle import attention
    threads = os.cpu_count() or 1
    scale = synth.default_scale(shape.d)
    G = shape.Hq // shape.Hkv
    heads = [(b, h) for b in range(shape.B) for h in range(shape.Hq)]
    if max_heads:
        heads = heads[:max_heads]
    done = 0
    t0 = time.perf_counter()
    i = 0
    while i < len(heads):
        batch = heads[i:i + threads]
        qs = torch.stack([q[b, h] for b, h in batch])[None]
        ks = torch.stack([k[b, h // G] for b, h in batch])[None]
        vs = torch.stack([v[b, h // G] for b, h in batch])[None]
        attention(qs, ks, vs, scale, shape.causal, threads=threads)
        done += len(batch)
        i += len(batch)
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    flops = counts.prefill_flops(1, done, shape.Nq, shape.Nk, shape.d, shape.causal)
    full = counts.prefill_flops(shape.B, shape.Hq, shape.Nq, shape.Nk, shape.d, shape.causal)
    rate = flops / dt
    rec = {"value": rate / 1e12, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
           "sample": f"{done} of {len(heads)} (batch, head) pairs of the workload, {dt:.1f} s, fp64 numpy"}
    if done < len(heads):
        rec["workload_s_extrapolated"] = full / rate
        rec["sample"] += "; the whole workload's time is extrapolated linearly from the sample's rate"
    else:
        rec["workload_s"] = dt
    return rec


def oracle_decode_sample(dec, seconds: float):
    from oracle import decode_paged
    kv = dec["kv"]
    s = dec["shape"]
    scale = synth.default_scale(s.d)
    t0 = time.perf_counter()
    seqs = []
    for n in range(s.S):
        decode_paged(kv.q, kv.k_pool, kv.v_pool, kv.block_table, kv.seq_lens, s.page_size, scale, seqs=[n])
        seqs.append(n)
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    nbytes = counts.decode_kv_bytes([int(kv.seq_lens[i]) for i in seqs], s.Hkv, s.d)
    return {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"{len(seqs)} of {s.S} sequences, {dt:.1f} s, fp64 numpy"}


# ----------------------------------------------------------------------------- arms

def run_reference_variant(args, dist):
    """Reference arm of the backward and FP8 workloads: the fp64 backward oracle, or the
    fp64 attention of the dequantized e4m3 inputs, on bounded samples of whole heads."""
    import oracle
    bwd = args.workload.endswith("_bwd")
    name = args.workload[:-4]
    shape = synth.WORKLOADS[name]
    seed = synth.workload_seed(name)
    q, k, v = synth.prefill_inputs(shape, seed)
    scale = synth.default_scale(shape.d)
    fwd_flops = counts.prefill_flops(shape.B, shape.Hq, shape.Nq, shape.Nk, shape.d, shape.causal)
    per_step = max(0.5, min(5.0, 120.0 / max(1, args.steps + args.warmup)))
    if bwd:
        do = synth.upstream_grad(shape, seed)
        run = lambda: oracle_backward_sample(shape, (q, k, v), do, scale, 2.5 * fwd_flops, per_step)  # noqa: E731
        metric, dtype = "attn bwd TFLOPS & % of BF16 tensor peak", "f64"
    else:
        q8, qs = oracle.block_quantize(q, 128)
        k8, ks = oracle.block_quantize(k, 128)
        v8, vs = oracle.block_quantize(v, shape.Nk)
        qd, kd = torch.from_numpy(oracle.dequantize(q8, qs)), torch.from_numpy(oracle.dequantize(k8, ks))
        vd = torch.from_numpy(oracle.dequantize(v8, vs, block=shape.Nk))
        run = lambda: oracle_prefill_sample(shape, qd, kd, vd, per_step, max_heads=os.cpu_count())  # noqa: E731
        metric, dtype = "attn fwd TFLOPS (e4m3 inputs) & % of FP8 tensor peak", "f64"
    for _ in range(args.warmup):
        run()
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        vals.append(run()["value"])
    total = time.perf_counter() - t0
    value = statistics.mean(vals) if vals else 0.0
    sample = ("per step: whole (batch, head) pairs of the fp64 backward oracle, one thread" if bwd else
              f"per step: {os.cpu_count()} (batch, head) pairs of the fp64 oracle on the dequantized inputs")
    line = {
        "impl": "reference", "metric": metric, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * total / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype, "data": "synthetic",
        "config": {"workload": args.workload,
                   "prefill": {"B": shape.B, "Hq": shape.Hq, "Hkv": shape.Hkv, "Nq": shape.Nq, "Nk": shape.Nk,
                               "d": shape.d, "causal": shape.causal},
                   "parallelism": f"independent replicas x{args.gpus} (no data-path collective)"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1 if bwd else os.cpu_count(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_reference(args, dist):
    """The oracle, as it stands, on the host cores, on the same config and metric."""
    if dist.rank != 0:
        return 0
    if args.workload.endswith(("_bwd", "_fp8")):
        return run_reference_variant(args, dist)
    shape = prefill_shape(args.workload)
    q, k, v = synth.prefill_inputs(shape, synth.workload_seed(
        "gqa_causal_2k" if args.workload == "serving_step" else args.workload))
    per_step = max(0.5, min(5.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_prefill_sample(shape, q, k, v, per_step, max_heads=os.cpu_count())
    vals, secs = [], []
    r = {"sample": "no step run"}
    t0 = time.perf_counter()
    for _ in range(args.steps):
        r = oracle_prefill_sample(shape, q, k, v, per_step, max_heads=os.cpu_count())
        vals.append(r["value"])
    total = time.perf_counter() - t0
    value = statistics.mean(vals) if vals else 0.0
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * total / max(1, args.steps),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_block(args, shape),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                         "sample": "per step: " + r["sample"]},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def config_block(args, shape):
    cfg = {"workload": "gqa_causal_2k prefill + paged_decode_gqa decode" if args.workload == "serving_step"
           else args.workload,
           "prefill": {"B": shape.B, "Hq": shape.Hq, "Hkv": shape.Hkv, "Nq": shape.Nq, "Nk": shape.Nk, "d": shape.d,
                       "causal": shape.causal, "qk_std": shape.qk_std}}
    if args.workload == "serving_step":
        s = synth.WORKLOADS["paged_decode_gqa"]
        cfg["decode"] = {"seqs": args.decode_seqs, "Hq": s.Hq, "Hkv": s.Hkv, "d": s.d, "page_size": s.page_size,
                         "len_range": [s.len_lo, s.len_hi]}
        cfg["l2"] = "inputs larger than L2: each step's 4.6 GB decode KV stream evicts the prefill inputs"
    else:
        cfg["l2"] = "L2 flushed between steps by writing a 256 MB buffer"
    cfg["parallelism"] = f"independent replicas x{args.gpus} (no data-path collective)"
    return cfg


def timed_launches(step, K, W, flush, stream, dist, dev):
    """W untimed calls, then K calls each after an L2 flush, each bracketed by CUDA events on
    the launching stream (barrier and synchronize on both sides); the clocks are sampled
    throughout.  Returns the per-call milliseconds and the clock record."""
    clocks = ClockSampler(dist.local)
    clocks.start()
    for _ in range(W):
        step()
        flush.zero_()
    torch.cuda.synchronize(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * K)]
    dist.barrier()
    torch.cuda.synchronize(dev)
    for i in range(K):
        flush.zero_()
        ev[2 * i].record(stream)
        step()
        ev[2 * i + 1].record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    clk = clocks.stop()
    return [ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(K)], clk


def bwd_record(args, ab, name, dev, stream, dist, peaks, peak_src, K, W, cpu=True):
    """Backward pass (attn_bwd: the delta kernel, then one pass that computes the five
    products per block) of a prefill workload.  FLOPs are the method's five products, 2.5x
    the forward's (causal halved), as the pages' FA figures count them."""
    shape = synth.WORKLOADS[name]
    seed = rank_seed(synth.workload_seed(name), dist.rank)
    pre = make_prefill(shape, seed, dev)
    qd, kd, vd = pre["dev"]
    do = synth.upstream_grad(shape, seed).to(dev)
    scale = synth.default_scale(shape.d)
    ab.attn_fwd(qd, kd, vd, pre["o"], pre["lse"], shape.causal, scale, stream)
    dq = torch.empty((shape.B, shape.Hq, shape.Nq, shape.d), dtype=torch.float32, device=dev)
    dk = torch.empty((shape.B, shape.Hkv, shape.Nk, shape.d), dtype=torch.float32, device=dev)
    dv = torch.empty_like(dk)
    ws = torch.empty(ab.attn_bwd_workspace_size(shape.B, shape.Hq, shape.Nq), dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flops = 2.5 * counts.prefill_flops(shape.B, shape.Hq, shape.Nq, shape.Nk, shape.d, shape.causal)

    def step():
        ab.attn_bwd(qd, kd, vd, pre["o"], do, pre["lse"], dq, dk, dv, shape.causal, scale, ws, stream)

    ms, clk = timed_launches(step, K, W, flush, stream, dist, dev)
    st = ab.attn_get_device_status(stream)
    if st != 0:
        raise RuntimeError(f"kernel fault in the timed region: {ab.attn_status_string(st)}")
    tot = dist.max(sum(ms))
    achieved = flops / (sum(ms) / K * 1e-3) / 1e12
    rec = {
        "metric": "attn bwd TFLOPS & % of BF16 tensor peak", "unit": "TFLOP/s",
        "value": dist.world * flops * K / (tot * 1e-3) / 1e12, "steps": K, "ms_per_launch": tot / K,
        "median_ms": statistics.median(ms),
        "shape": {"B": shape.B, "Hq": shape.Hq, "Hkv": shape.Hkv, "Nq": shape.Nq, "Nk": shape.Nk, "d": shape.d,
                  "causal": shape.causal},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"],
                     "traffic": profiled_traffic(f"attn_bwd_{name}.md") if name in ("gqa_causal_2k", "gqa_causal_16k")
                     else None,
                     "peak_source": f"{peak_src} bf16_tflops (burst cuBLAS)",
                     "kernel": "attn_bwd_kernel + attn_bwd_delta_kernel (one call)",
                     "flops_per_launch": flops},
        "l2": "L2 flushed before every call by writing a 256 MB buffer",
        "clocks": clk, "gpu_launches": 2 * K,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline and cpu:
        rec["cpu_baseline"] = oracle_backward_sample(shape, pre["host"], do.cpu(), scale, flops, args.cpu_seconds / 2)
    return rec


def fp8_record(args, ab, name, dev, stream, dist, peaks, peak_src, K, W, cpu=True):
    """FP8 forward (attn_fwd_fp8) of a d = 128 prefill workload: inputs quantized on the GPU
    once (Q, K per 128 rows, V per head), outside the timed region.  The tensor peak for
    e4m3 is the measured bf16 figure times the nominal dense ratio 4.5 / 2.25 = 2."""
    shape = synth.WORKLOADS[name]
    seed = rank_seed(synth.workload_seed(name), dist.rank)
    pre = make_prefill(shape, seed, dev)
    qd, kd, vd = pre["dev"]
    q8, qs = ab.attn_quantize_fp8(qd, 128)
    k8, ks = ab.attn_quantize_fp8(kd, 128)
    v8, vs = ab.attn_quantize_fp8(vd, shape.Nk)
    vs = vs[..., 0].contiguous()
    scale = synth.default_scale(shape.d)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    flops = counts.prefill_flops(shape.B, shape.Hq, shape.Nq, shape.Nk, shape.d, shape.causal)

    def step():
        ab.attn_fwd_fp8(q8, qs, k8, ks, v8, vs, pre["o"], pre["lse"], shape.causal, scale, stream)

    ms, clk = timed_launches(step, K, W, flush, stream, dist, dev)
    st = ab.attn_get_device_status(stream)
    if st != 0:
        raise RuntimeError(f"kernel fault in the timed region: {ab.attn_status_string(st)}")
    tot = dist.max(sum(ms))
    achieved = flops / (sum(ms) / K * 1e-3) / 1e12
    peak = 2.0 * peaks["bf16_tflops"]
    rec = {
        "metric": "attn fwd TFLOPS (e4m3 inputs) & % of FP8 tensor peak", "unit": "TFLOP/s",
        "value": dist.world * flops * K / (tot * 1e-3) / 1e12, "steps": K, "ms_per_launch": tot / K,
        "median_ms": statistics.median(ms), "dtype": "e4m3 (fp32 accumulate)",
        "shape": {"B": shape.B, "Hq": shape.Hq, "Hkv": shape.Hkv, "Nq": shape.Nq, "Nk": shape.Nk, "d": shape.d,
                  "causal": shape.causal},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak,
                     "traffic": profiled_traffic(f"attn_fwd_fp8_{name}.md")
                     if name in ("gqa_causal_2k", "gqa_causal_16k") else None,
                     "peak_source": f"2 x {peak_src} bf16_tflops (nominal e4m3 : bf16 dense ratio)",
                     "kernel": "attn_fwd_fp8_kernel", "flops_per_launch": flops},
        "l2": "L2 flushed before every launch by writing a 256 MB buffer",
        "clocks": clk, "gpu_launches": K,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline and cpu:
        import oracle
        q, k, v = pre["host"]
        q8h, qsh = oracle.block_quantize(q, 128)
        k8h, ksh = oracle.block_quantize(k, 128)
        v8h, vsh = oracle.block_quantize(v, shape.Nk)
        qdq = torch.from_numpy(oracle.dequantize(q8h, qsh))
        kdq = torch.from_numpy(oracle.dequantize(k8h, ksh))
        vdq = torch.from_numpy(oracle.dequantize(v8h, vsh, block=shape.Nk))
        rec["cpu_baseline"] = oracle_prefill_sample(shape, qdq, kdq, vdq, args.cpu_seconds / 2)
        rec["cpu_baseline"]["sample"] += " (exact attention of the dequantized e4m3 inputs)"
    return rec


def variant_line(args, dist, rec, workload):
    """The JSON line of a --workload *_bwd / *_fp8 run, built from its record."""
    shape = rec["shape"]
    line = {
        "metric": rec["metric"], "value": rec["value"], "unit": rec["unit"], "n_gpus": dist.world,
        "steps": rec["steps"], "warmup": args.warmup, "ms_per_step": rec["ms_per_launch"],
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": rec.get("dtype", "bf16"),
        "data": "synthetic",
        "config": {"workload": workload, "prefill": shape, "l2": rec["l2"],
                   "parallelism": f"independent replicas x{dist.world} (no data-path collective)"},
        "roofline": dict(rec["roofline"], median_ms=rec["median_ms"]),
        "gpu_launches": rec["gpu_launches"], "clocks": rec["clocks"],
    }
    if "cpu_baseline" in rec:
        line["cpu_baseline"] = rec["cpu_baseline"]
    return line


def run_backward(args, dist):
    import attn_fwd_05_b200 as ab
    ab.load_library()
    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream(dev)
    rec = bwd_record(args, ab, args.workload[: -len("_bwd")], dev, stream, dist, peaks, peak_src, args.steps,
                     args.warmup)
    if dist.rank == 0:
        print(json.dumps(variant_line(args, dist, rec, args.workload)), flush=True)
    return 0


def oracle_backward_sample(shape, host, do, scale, flops, seconds):
    """The fp64 backward oracle on whole (batch, query head) pairs until about `seconds`
    have passed, scaled to the workload's FLOPs by the share of heads done."""
    import oracle
    try:
        from threadpoolctl import threadpool_limits
        limit = threadpool_limits(1)  # the matrix products of numpy's BLAS on one thread
    except Exception:
        limit = None
    q, k, v = host
    G = shape.Hq // shape.Hkv
    t0 = time.perf_counter()
    heads = 0
    done = False
    for b in range(shape.B):
        for h in range(shape.Hq):
            kv = h // G
            oracle.attention_head_backward(oracle.as_f64(q[b, h]), oracle.as_f64(k[b, kv]), oracle.as_f64(v[b, kv]),
                                           oracle.as_f64(do[b, h]), scale, shape.causal)
            heads += 1
            if time.perf_counter() - t0 > seconds:
                done = True
                break
        if done:
            break
    dt = time.perf_counter() - t0
    if limit is not None:
        limit.unregister()
    share = heads / (shape.B * shape.Hq)
    return {"value": flops * share / dt / 1e12, "unit": "TFLOP/s", "cores": 1 if limit is not None else os.cpu_count(),
            "kind": "oracle",
            "sample": f"{heads} of {shape.B * shape.Hq} (batch, head) pairs, fp64 backward, one thread, {dt:.1f} s"}


def run_fp8(args, dist):
    import attn_fwd_05_b200 as ab
    ab.load_library()
    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream(dev)
    rec = fp8_record(args, ab, args.workload[: -len("_fp8")], dev, stream, dist, peaks, peak_src, args.steps,
                     args.warmup)
    if dist.rank == 0:
        print(json.dumps(variant_line(args, dist, rec, args.workload)), flush=True)
    return 0


def run_ours(args, dist):
    import attn_fwd_05_b200 as ab
    ab.load_library()
    dev = torch.device("cuda", dist.local)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    shape = prefill_shape(args.workload)
    seed = synth.workload_seed("gqa_causal_2k" if args.workload == "serving_step" else args.workload)
    pre = make_prefill(shape, rank_seed(seed, dist.rank), dev)
    dec = make_decode(rank_seed(synth.workload_seed("paged_decode_gqa"), dist.rank), dev, args.decode_seqs) \
        if args.workload == "serving_step" else None
    flush = None if dec is not None else torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    scale = synth.default_scale(shape.d)
    flops = counts.prefill_flops(shape.B, shape.Hq, shape.Nq, shape.Nk, shape.d, shape.causal)
    stream = torch.cuda.current_stream(dev)

    qd, kd, vd = pre["dev"]

    def prefill():
        ab.attn_fwd(qd, kd, vd, pre["o"], pre["lse"], shape.causal, scale, stream)

    def decode():
        ab.attn_decode_paged(dec["q"], dec["k_pool"], dec["v_pool"], dec["table"], dec["lens"],
                             dec["shape"].page_size, dec["o"], dec["lse"], scale, dec["ws"], stream)

    clocks = ClockSampler(dist.local)
    clocks.start()
    for _ in range(args.warmup):
        prefill()
        if dec is not None:
            decode()
        else:
            flush.zero_()
    torch.cuda.synchronize(dev)
    st = ab.attn_get_device_status(stream)
    if st != 0:
        raise RuntimeError(f"kernel fault during warm-up: {ab.attn_status_string(st)}")

    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3 * K)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize(dev)
    t_start.record(stream)
    for i in range(K):
        if dec is None:
            flush.zero_()
        ev[3 * i].record(stream)
        prefill()
        ev[3 * i + 1].record(stream)
        if dec is not None:
            decode()
        ev[3 * i + 2].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    clk = clocks.stop()
    st = ab.attn_get_device_status(stream)
    if st != 0:
        raise RuntimeError(f"kernel fault in the timed region: {ab.attn_status_string(st)}")

    pre_ms = [ev[3 * i].elapsed_time(ev[3 * i + 1]) for i in range(K)]
    dec_ms = [ev[3 * i + 1].elapsed_time(ev[3 * i + 2]) for i in range(K)] if dec is not None else []
    total_ms = t_start.elapsed_time(t_end)
    pre_sum = dist.max(sum(pre_ms))
    dec_sum = dist.max(sum(dec_ms)) if dec is not None else 0.0
    total_ms = dist.max(total_ms)
    N = dist.world

    prefill_tflops = N * flops * K / (pre_sum * 1e-3) / 1e12
    avg_pre_ms = sum(pre_ms) / K
    achieved = flops / (avg_pre_ms * 1e-3) / 1e12
    kname = "attn_fwd_pingpong_kernel<128>" if shape.d <= 128 else "attn_fwd_single_kernel<256>"
    prefill_roofline = {
        "bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
        "frac": achieved / peaks["bf16_tflops"],
        "traffic": profiled_traffic(PREFILL_PROFILES[args.workload]) if args.workload in PREFILL_PROFILES else None,
        "peak_source": f"{peak_src} bf16_tflops (burst cuBLAS); frac of the sustained figure "
                       f"{achieved / peaks['bf16_tflops_sustained']:.3f}",
        "kernel": kname, "flops_per_launch": flops, "median_ms": statistics.median(pre_ms)}
    line = {
        "metric": METRIC,
        "value": prefill_tflops,
        "unit": "TFLOP/s",
        "n_gpus": N,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": total_ms / K,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": config_block(args, shape),
        "roofline": prefill_roofline,
        "gpu_launches": K * (1 + (3 if dec is not None else 0)),
        "clocks": clk,
    }
    if dec is not None:
        kvb = dec["kv_bytes"]
        avg_dec_ms = sum(dec_ms) / K
        gbs = kvb / (avg_dec_ms * 1e-3) / 1e9
        full = args.decode_seqs == 64
        decode_roofline = {
            "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": gbs / peaks["hbm_gbs"],
            "traffic": profiled_traffic("attn_decode_split_paged_decode.md") if full else None,
            "peak_source": f"{peak_src} hbm_gbs (copy)",
            "kernel": "attn_decode_split_kernel<128> (timed with its plan and merge kernels: one decode call)",
            "bytes_per_launch": kvb, "median_ms": statistics.median(dec_ms)}
        line["decode"] = {
            "metric": "paged decode KV-read GB/s", "value": N * kvb * K / (dec_sum * 1e-3) / 1e9, "unit": "GB/s",
            "kv_bytes_per_step": kvb, "roofline": decode_roofline,
        }
        # the decode call takes about 4/5 of the step: it is the step's dominant kernel
        if avg_dec_ms > avg_pre_ms:
            line["roofline"] = decode_roofline
            line["prefill_roofline"] = prefill_roofline

    if not args.no_e2e:
        line["e2e"] = e2e_prefill(args, ab, pre, shape, scale, flops, dev, stream, dist)
        if dec is not None:
            line["decode"]["e2e"] = e2e_decode(args, ab, dec, scale, dev, stream, dist)
    if dist.rank == 0 and N == 1 and not args.no_cpu_baseline:
        q, k, v = pre["host"]
        line["cpu_baseline"] = oracle_prefill_sample(shape, q, k, v, args.cpu_seconds)
        if dec is not None:
            line["decode"]["cpu_baseline"] = oracle_decode_sample(dec, max(2.0, args.cpu_seconds / 3))
    if args.workload == "serving_step" and not args.no_other_workloads:
        # the other prefill configurations, each timed on its own (not part of the step)
        del pre, dec
        torch.cuda.empty_cache()
        line["workloads"] = {name: prefill_record(args, ab, name, dev, stream, dist, peaks, peak_src)
                             for name in OTHER_PREFILL}
        # the backward pass and the FP8 forward of the two GQA causal workloads
        # (CPU baselines for the 2K variants only: one 16K head of the fp64 backward oracle
        # takes minutes on one thread, and the 16K forward's oracle rate is in its own record)
        for name in ("gqa_causal_2k", "gqa_causal_16k"):
            small = name == "gqa_causal_2k"
            K = max(3, min(args.steps, 20 if small else 8))
            line["workloads"][name + "_fp8"] = fp8_record(args, ab, name, dev, stream, dist, peaks, peak_src, K,
                                                          max(3, args.warmup), cpu=small)
            line["workloads"][name + "_bwd"] = bwd_record(args, ab, name, dev, stream, dist, peaks, peak_src, K,
                                                          max(3, args.warmup), cpu=small)
    if dist.rank == 0:
        print(json.dumps(line), flush=True)
    return 0


OTHER_PREFILL = ("tiny_mha_d64", "gqa_causal_16k", "peaked_mha_d256")


def prefill_record(args, ab, name, dev, stream, dist, peaks, peak_src):
    """One prefill workload timed on its own: W warm-up launches, then K launches, each
    after a 256 MB write that flushes L2, timed by CUDA events on the launching stream.
    Returns the workload's record (median and mean launch time, TFLOP/s, roofline against
    the measured peak, DRAM traffic from the committed ncu summary, clocks, and on rank 0
    at N = 1 the oracle's rate on a bounded sample)."""
    shape = synth.WORKLOADS[name]
    seed = rank_seed(synth.workload_seed(name), dist.rank)
    pre = make_prefill(shape, seed, dev)
    qd, kd, vd = pre["dev"]
    scale = synth.default_scale(shape.d)
    flops = counts.prefill_flops(shape.B, shape.Hq, shape.Nq, shape.Nk, shape.d, shape.causal)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    K = max(3, min(args.steps, 100 if flops < 1e12 else 30))

    def launch():
        ab.attn_fwd(qd, kd, vd, pre["o"], pre["lse"], shape.causal, scale, stream)

    clocks = ClockSampler(dist.local)
    clocks.start()
    for _ in range(max(3, args.warmup)):
        flush.zero_()
        launch()
    torch.cuda.synchronize(dev)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(2 * K)]
    dist.barrier()
    torch.cuda.synchronize(dev)
    for i in range(K):
        flush.zero_()
        ev[2 * i].record(stream)
        launch()
        ev[2 * i + 1].record(stream)
    torch.cuda.synchronize(dev)
    dist.barrier()
    clk = clocks.stop()
    st = ab.attn_get_device_status(stream)
    if st != 0:
        raise RuntimeError(f"kernel fault in the timed region of {name}: {ab.attn_status_string(st)}")
    ms = [ev[2 * i].elapsed_time(ev[2 * i + 1]) for i in range(K)]
    tot = dist.max(sum(ms))
    achieved = flops / (sum(ms) / K * 1e-3) / 1e12
    kname = "attn_fwd_pingpong_kernel<%d>" % shape.d if shape.d <= 128 else "attn_fwd_single_kernel<256>"
    rec = {
        "metric": "attn fwd TFLOPS & % of BF16 tensor peak", "unit": "TFLOP/s",
        "value": dist.world * flops * K / (tot * 1e-3) / 1e12, "steps": K, "ms_per_launch": tot / K,
        "median_ms": statistics.median(ms),
        "shape": {"B": shape.B, "Hq": shape.Hq, "Hkv": shape.Hkv, "Nq": shape.Nq, "Nk": shape.Nk, "d": shape.d,
                  "causal": shape.causal, "qk_std": shape.qk_std},
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": achieved / peaks["bf16_tflops"],
                     "traffic": profiled_traffic(PREFILL_PROFILES[name]) if name in PREFILL_PROFILES else None,
                     "peak_source": f"{peak_src} bf16_tflops (burst cuBLAS); frac of the sustained figure "
                                    f"{achieved / peaks['bf16_tflops_sustained']:.3f}",
                     "kernel": kname, "flops_per_launch": flops},
        "l2": "L2 flushed before every launch by writing a 256 MB buffer",
        "clocks": clk, "gpu_launches": K,
    }
    if dist.rank == 0 and dist.world == 1 and not args.no_cpu_baseline:
        q, k, v = pre["host"]
        rec["cpu_baseline"] = oracle_prefill_sample(shape, q, k, v, args.cpu_seconds)
    return rec


def _pipelined_e2e(K, h2d, launch, d2h, stream, dev, dist, slots=2):
    """Time K steps of (copy in, launch, copy out) as a serving loop runs them: two slots of
    device buffers, the host-to-device copies on one stream, the kernels on the caller's
    stream and the device-to-host copies on a third, so step i+1's inputs go up and step
    i-1's outputs come down while step i computes (PCIe is full duplex).  Events order each
    slot's reuse: a copy into slot j waits for the kernel that last read it, a kernel
    writing slot j waits for the copy that last read its outputs.  The timed region starts
    before the first copy in and ends after the last copy out.  Returns the max over ranks
    of the region's milliseconds."""
    s_in = torch.cuda.Stream(dev)
    s_out = torch.cuda.Stream(dev)
    in_done = [torch.cuda.Event() for _ in range(slots)]
    comp_done = [torch.cuda.Event() for _ in range(slots)]
    out_done = [torch.cuda.Event() for _ in range(slots)]

    def step(i):
        j = i % slots
        s_in.wait_event(comp_done[j])  # no-op until the event is first recorded
        with torch.cuda.stream(s_in):
            h2d(j)
        in_done[j].record(s_in)
        stream.wait_event(in_done[j])
        stream.wait_event(out_done[j])
        launch(j)
        comp_done[j].record(stream)
        s_out.wait_event(comp_done[j])
        with torch.cuda.stream(s_out):
            d2h(j)
        out_done[j].record(s_out)

    for i in range(3):
        step(i)
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    dist.barrier()
    a.record(stream)
    s_in.wait_event(a)
    for i in range(K):
        step(i)
    for e in out_done:
        stream.wait_event(e)
    b.record(stream)
    torch.cuda.synchronize(dev)
    return dist.max(a.elapsed_time(b))


def _sequential_e2e(K, h2d, launch, d2h, stream, dev, dist):
    """K steps of (copy in, launch, copy out), all on the caller's stream, one after the
    other.  Returns the max over ranks of the timed region's milliseconds."""
    def step():
        with torch.cuda.stream(stream):
            h2d(0)
            launch(0)
            d2h(0)

    for _ in range(3):
        step()
    torch.cuda.synchronize(dev)
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    dist.barrier()
    a.record(stream)
    for _ in range(K):
        step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    return dist.max(a.elapsed_time(b))


def e2e_decode(args, ab, dec, scale, dev, stream, dist):
    """The decode metric through the public API with host buffers: every step copies the
    step's inputs (the query tokens, the block table and the sequence lengths) from
    pinned host memory, runs attn_decode_paged, and copies O and LSE back, all inside the
    timed region.  The paged K/V pools are the cache: they stay resident in HBM across
    steps, as a serving engine keeps them.  The headline value overlaps the copies of
    neighbouring steps with the kernel (two buffer slots); the sequential figure runs
    copy, kernel and copy back to back."""
    hin = [t.pin_memory() for t in (dec["kv"].q, dec["kv"].block_table, dec["kv"].seq_lens)]
    din = [[torch.empty_like(t, device=dev) for t in hin] for _ in range(2)]
    dout = [(torch.empty_like(dec["o"]), torch.empty_like(dec["lse"])) for _ in range(2)]
    hout = [(torch.empty(dec["o"].shape, dtype=torch.bfloat16).pin_memory(),
             torch.empty(dec["lse"].shape, dtype=torch.float32).pin_memory()) for _ in range(2)]

    def h2d(j):
        for d, h in zip(din[j], hin):
            d.copy_(h, non_blocking=True)

    def launch(j):
        qd, td, ld = din[j]
        ab.attn_decode_paged(qd, dec["k_pool"], dec["v_pool"], td, ld, dec["shape"].page_size, dout[j][0],
                             dout[j][1], scale, dec["ws"], stream)

    def d2h(j):
        for h, d in zip(hout[j], dout[j]):
            h.copy_(d, non_blocking=True)

    K = max(3, min(args.steps, 20))
    ms = _pipelined_e2e(K, h2d, launch, d2h, stream, dev, dist)
    seq_ms = _sequential_e2e(K, h2d, launch, d2h, stream, dev, dist)
    h2d_b = sum(t.numel() * t.element_size() for t in hin)
    d2h_b = sum(t.numel() * t.element_size() for t in hout[0])
    rate = dist.world * dec["kv_bytes"] * K / 1e9
    return {"value": rate / (ms * 1e-3), "unit": "GB/s", "h2d_bytes_per_step": h2d_b,
            "d2h_bytes_per_step": d2h_b, "steps": K, "ms_per_step": ms / K,
            "sequential": {"value": rate / (seq_ms * 1e-3), "ms_per_step": seq_ms / K},
            "note": "paged K/V pools resident in HBM (the cache); query, block table and lengths copied in, "
                    "O and LSE copied out every step; two buffer slots, copies of neighbouring steps "
                    "overlap the kernel (sequential: copy, kernel, copy back to back)"}


def e2e_prefill(args, ab, pre, shape, scale, flops, dev, stream, dist):
    """Same metric through the public API with host buffers: every step copies q, k, v in
    from pinned memory, runs attn_fwd and copies o and lse out, all inside the timed
    region.  The headline value overlaps the copies of neighbouring steps with the kernel
    (two buffer slots); the sequential figure runs copy, kernel and copy back to back."""
    hin = [t.pin_memory() for t in pre["host"]]
    din = [[torch.empty_like(t, device=dev) for t in hin] for _ in range(2)]
    dout = [(torch.empty_like(pre["o"]), torch.empty_like(pre["lse"])) for _ in range(2)]
    hout = [(torch.empty(pre["o"].shape, dtype=torch.bfloat16).pin_memory(),
             torch.empty(pre["lse"].shape, dtype=torch.float32).pin_memory()) for _ in range(2)]

    def h2d(j):
        for d, h in zip(din[j], hin):
            d.copy_(h, non_blocking=True)

    def launch(j):
        ab.attn_fwd(*din[j], dout[j][0], dout[j][1], shape.causal, scale, stream)

    def d2h(j):
        for h, d in zip(hout[j], dout[j]):
            h.copy_(d, non_blocking=True)

    K = max(3, min(args.steps, 20))
    ms = _pipelined_e2e(K, h2d, launch, d2h, stream, dev, dist)
    seq_ms = _sequential_e2e(K, h2d, launch, d2h, stream, dev, dist)
    h2d_b = sum(t.numel() * t.element_size() for t in hin)
    d2h_b = sum(t.numel() * t.element_size() for t in hout[0])
    rate = dist.world * flops * K / 1e12
    return {"value": rate / (ms * 1e-3), "unit": "TFLOP/s", "h2d_bytes_per_step": h2d_b,
            "d2h_bytes_per_step": d2h_b, "steps": K, "ms_per_step": ms / K,
            "sequential": {"value": rate / (seq_ms * 1e-3), "ms_per_step": seq_ms / K},
            "note": "two buffer slots: step i+1's copy in and step i-1's copy out overlap step i's kernel "
                    "(sequential: copy, kernel, copy back to back)"}


def main():
    args = parse()
    dist = Dist()
    if args.impl == "reference":
        return run_reference(args, dist)
    dist.init("nccl")
    try:
        if args.workload.endswith("_bwd"):
            return run_backward(args, dist)
        if args.workload.endswith("_fp8"):
            return run_fp8(args, dist)
        return run_ours(args, dist)
    finally:
        dist.close()


if __name__ == "__main__":
    sys.exit(main())
