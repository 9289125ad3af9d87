"""Benchmark of the exact tiled attention kernels on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--quick] [--config 1-5]

Headline (one JSON line on rank 0): causal bf16 prefill forward on
B=4, Hq=Hkv=16, L=2048, D=128 (Q x4 on heads 0-7, seed 1), in TFLOP/s with the
causal (query, key) pairs counted once.  A step is one fa_fwd call over the
whole batch, inputs resident in HBM, L2 flushed before every timed step.  The
same line carries, under "sections", the other workloads measured in the same
run (long-context GQA prefill, training forward+backward, split-KV decode).

Multi-GPU: replicas only (every rank runs the same workload on its own copy;
no collective on the data path); value = all ranks' FLOPs / max-over-ranks time.

--impl reference times the CPU fp64 oracle on a bounded sample of the same
workload (rank 0 only), as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from exact_tiled_attention_46_b200 import inputs as synth  # noqa: E402

METRIC = "attn fwd/bwd TFLOP/s & % BF16 tensor peak; decode KV-read GB/s & % of HBM"
HEADLINE = "causal_prefill"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# Nominal per-GPU figures, reported beside the measured ones for context:
# dense BF16 2.25 PFLOP/s (NVIDIA's DGX B200 figure of 36 PFLOP/s BF16 for 8 GPUs
# is quoted with 2:4 sparsity; dense is half, per GPU 36 / 8 / 2) and HBM3e
# ~8 TB/s (the same datasheet's 64 TB/s for 8 GPUs; the "~8 TB/s" the decode
# target is stated against).
NOMINAL_PEAKS = {"bf16_tflops": 2250.0, "hbm_gbs": 8000.0,
                 "source": "NVIDIA DGX B200 datasheet per GPU: 36 PF BF16 sparse / 8 / 2; 64 TB/s HBM3e / 8"}

# DRAM bytes (read + write) per launch from ncu captures, valid only while the
# kernel's sources hash to the recorded value (otherwise the roofline's traffic
# is reported as null).  "per_unit" records are scaled to the bench's launch by
# its units of work (see the profiles/ summaries for the captured case).
PROFILED_TRAFFIC = {
    "fwd_kernel causal_prefill": {"sources": ("csrc/fa_fwd.cuh", "csrc/sm100.cuh"),
                                  "sha256_16": "644cd20e74d80560", "bytes": 126125824 + 9488384},
    "fwd_kernel long_gqa_prefill": {"sources": ("csrc/fa_fwd.cuh", "csrc/sm100.cuh"),
                                    "sha256_16": "644cd20e74d80560", "bytes": 352846080 + 97611776},
    "fwd_kernel<fp8> causal_prefill": {"sources": ("csrc/fa_fwd.cuh", "csrc/sm100.cuh"),
                                       "sha256_16": "644cd20e74d80560", "bytes": 50400256 + 3337728},
    "bwd_main_kernel train_fwd_bwd": {"sources": ("csrc/fa_bwd.cuh", "csrc/sm100.cuh"),
                                      "sha256_16": "2ce9742435305e4b", "bytes": 406921728 + 223515392},
    # captured on the first 16 sequences of the decode workload (1.35888 GB of KV
    # rows), scaled to a launch by the KV bytes it reads
    "decode_split_kernel splitkv_decode": {"sources": ("csrc/fa_decode.cuh", "csrc/sm100.cuh"),
                                           "sha256_16": "cc6efd0dad8ce196",
                                           "bytes_per_kv_byte": (1362351360 + 12924672) / 1358876672},
    "decode_split_kernel<append> splitkv_decode": {"sources": ("csrc/fa_decode.cuh", "csrc/sm100.cuh"),
                                                   "sha256_16": "cc6efd0dad8ce196",
                                                   "bytes_per_kv_byte": (1366708480 + 19545344) / 1358876672},
    "decode_split_kernel<paged16> splitkv_decode": {"sources": ("csrc/fa_decode.cuh", "csrc/sm100.cuh"),
                                                    "sha256_16": "cc6efd0dad8ce196",
                                                    "bytes_per_kv_byte": (1362181376 + 13036544) / 1358876672},
}


def sources_hash(rels):
    import hashlib
    h = hashlib.sha256()
    for rel in rels:
        with open(os.path.join(ROOT, "exact_tiled_attention_46_b200", rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def profiled_traffic(key, kv_bytes=None):
    rec = PROFILED_TRAFFIC.get(key)
    if rec is None or sources_hash(rec["sources"]) != rec["sha256_16"]:
        return None
    if rec.get("bytes") is not None:
        return rec["bytes"]
    if rec.get("bytes_per_kv_byte") is not None and kv_bytes is not None:
        return rec["bytes_per_kv_byte"] * kv_bytes
    return None


def roofline(bound, achieved, peaks, peak_src, unit, traffic=None, algorithmic_bytes=None, sustained=False):
    """Roofline block: achieved against the measured peak (burst for a kernel
    timed alone, sustained inside a long step) and against the nominal one."""
    if bound == "tensor":
        key = "bf16_tflops_sustained" if sustained and "bf16_tflops_sustained" in peaks else "bf16_tflops"
        peak, nominal = peaks[key], NOMINAL_PEAKS["bf16_tflops"]
        src = f"{peak_src} {'bf16 sustained' if key.endswith('sustained') else 'bf16 burst'}"
    else:
        peak, nominal = peaks["hbm_gbs"], NOMINAL_PEAKS["hbm_gbs"]
        src = f"{peak_src} HBM copy"
    r = {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit, "frac": achieved / peak,
         "traffic": traffic, "peak_source": src, "peak_nominal": nominal, "frac_nominal": achieved / nominal}
    if algorithmic_bytes is not None:
        r["algorithmic_bytes"] = algorithmic_bytes
    return r


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def allowed_pairs(Lq, Lk, causal):
    if not causal:
        return Lq * Lk
    off = Lk - Lq
    i = np.arange(Lq, dtype=np.int64)
    return int(np.clip(i + off + 1, 0, Lk).sum())


def fwd_flops(w):
    return 4.0 * w.B * w.Hq * w.D * allowed_pairs(w.Lq, w.Lk, w.causal)


def fwd_bytes(w):
    # Q, K, V read once, O written once (bf16), LSE written (fp32)
    return 2.0 * (2 * w.B * w.Lq * w.Hq * w.D + 2 * w.B * w.Lk * w.Hkv * w.D) + 4.0 * w.B * w.Hq * w.Lq


# ----------------------------------------------------------------- clocks --
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.t0 = self.t1 = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), "--query-gpu=" + self.FIELDS, "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def mark(self, which):
        setattr(self, which, time.time())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [r.split(", ") for r in out.strip().splitlines() if r.count(",") >= 8]
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        busy = [s for s in sm if s > 0.5 * max(sm)] if sm else []
        reasons = set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for r in rows:
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(busy) if busy else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# ------------------------------------------------------- rank helpers ------
def max_over_ranks(ms, dist=None, device="cpu"):
    """Device time of the slowest rank (the whole job ends when it does)."""
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    if dist is not None and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(flops_per_step, world, steps, max_ms):
    """Replicas: every rank runs the same workload, so the job did world x steps of it."""
    return flops_per_step * world * steps / (max_ms * 1e-3) / 1e12


# ------------------------------------------------------------- our arm -----
def l2_flusher(dev):
    buf = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=dev)

    def flush():
        buf.fill_(1.0)
    return flush


class nvtx:
    """NVTX range around a bench section (visible to ncu / nsys)."""

    def __init__(self, name):
        self.name = name

    def __enter__(self):
        torch.cuda.nvtx.range_push(self.name)

    def __exit__(self, *exc):
        torch.cuda.nvtx.range_pop()


def time_steps(fn, steps, warmup, flush, stream):
    for _ in range(warmup):
        flush()
        fn()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for s, e in evs:
        flush()
        s.record(stream)
        fn()
        e.record(stream)
    torch.cuda.synchronize()
    return [s.elapsed_time(e) for s, e in evs]


def section_fwd(fa, name, steps, warmup, flush, stream, peaks, peak_src, dev):
    w = synth.WORKLOADS[name]
    x = synth.workload_inputs(w)
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Lq), dtype=torch.float32, device=dev)
    with nvtx(f"section {name}"):
        ms = time_steps(lambda: fa.fwd(q, k, v, scale=w.scale, causal=w.causal, out=o, lse=lse), steps, warmup,
                        flush, stream)
    t = statistics.mean(ms) * 1e-3
    tf = fwd_flops(w) / t / 1e12
    return {"workload": name, "kernel": "fwd_kernel", "ms": t * 1e3, "ms_median": statistics.median(ms),
            "tflops": tf, "frac_bf16_peak": tf / peaks["bf16_tflops"], "launches": steps,
            "roofline": roofline("tensor", tf, peaks, peak_src, "TFLOP/s",
                                 traffic=profiled_traffic(f"fwd_kernel {name}"), algorithmic_bytes=fwd_bytes(w))}


def section_fwd_fp8(fa, name, steps, warmup, flush, stream, peaks, peak_src, dev):
    """The forward on the same draws quantized to e4m3 (per-tensor scales);
    its peak is the measured bf16 one times the nominal fp8:bf16 ratio (2)."""
    w = synth.WORKLOADS[name]
    x = synth.prefill_inputs_fp8(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.D, w.seed, q_boost_heads=w.q_boost_heads)
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty((w.B, w.Lq, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.Hq, w.Lq), dtype=torch.float32, device=dev)
    with nvtx(f"section {name}_fp8"):
        ms = time_steps(lambda: fa.fwd_fp8(q, k, v, x["q_scale"], x["k_scale"], x["v_scale"], scale=w.scale,
                                           causal=w.causal, out=o, lse=lse), steps, warmup, flush, stream)
    t = statistics.mean(ms) * 1e-3
    tf = fwd_flops(w) / t / 1e12
    fp8_peaks = dict(peaks)
    fp8_peaks["bf16_tflops"] = 2.0 * peaks["bf16_tflops"]
    r = roofline("tensor", tf, fp8_peaks, peak_src, "TFLOP/s", traffic=profiled_traffic(f"fwd_kernel<fp8> {name}"),
                 algorithmic_bytes=fwd_bytes(w) - (w.B * w.Lq * w.Hq * w.D + 2 * w.B * w.Lk * w.Hkv * w.D))
    r["peak_source"] = f"{peak_src} bf16 burst x 2 (nominal fp8:bf16 ratio)"
    r["peak_nominal"] = 2.0 * NOMINAL_PEAKS["bf16_tflops"]
    r["frac_nominal"] = tf / r["peak_nominal"]
    return {"workload": f"{name}_fp8", "kernel": "fwd_kernel<fp8>", "dtype": "e4m3 in, fp32 accumulate",
            "ms": t * 1e3, "ms_median": statistics.median(ms), "tflops": tf, "launches": steps, "roofline": r}


def section_train(fa, steps, warmup, flush, stream, peaks, peak_src, dev):
    w = synth.WORKLOADS["train_fwd_bwd"]
    x = synth.workload_inputs(w)
    q, k, v, do = (x[n].to(dev) for n in ("q", "k", "v", "do"))
    o, lse = fa.fwd(q, k, v, scale=w.scale, causal=w.causal)
    ws = torch.empty(fa.bwd_workspace_size(w.B, w.Hq, w.Lq, w.D), dtype=torch.uint8, device=dev)
    try:
        fa.bwd(q, k, v, o, do, lse, scale=w.scale, causal=w.causal, workspace=ws)
    except fa.FaError as e:
        return {"workload": "train_fwd_bwd", "unavailable": str(e)}

    def step():
        fa.fwd(q, k, v, scale=w.scale, causal=w.causal, out=o, lse=lse)
        fa.bwd(q, k, v, o, do, lse, scale=w.scale, causal=w.causal, workspace=ws)
    with nvtx("section train_fwd_bwd"):
        ms = time_steps(step, steps, warmup, flush, stream)
        t = statistics.mean(ms) * 1e-3
        ms_b = time_steps(lambda: fa.bwd(q, k, v, o, do, lse, scale=w.scale, causal=w.causal, workspace=ws),
                          steps, warmup, flush, stream)
    tb = statistics.mean(ms_b) * 1e-3
    ff = fwd_flops(w)
    # algorithmic bytes of the backward: q, k, v, o, dO read, dq, dk, dv written (bf16), lse + Delta rows
    nq, nk = w.B * w.Lq * w.Hq * w.D, w.B * w.Lk * w.Hkv * w.D
    bwd_bytes = 2.0 * (3 * nq + 2 * nk) + 2.0 * (nq + 2 * nk) + 8.0 * w.B * w.Hq * w.Lq
    tfb = 2.5 * ff / tb / 1e12
    return {"workload": "train_fwd_bwd", "ms_fwd_bwd": t * 1e3, "ms_fwd_bwd_median": statistics.median(ms),
            "tflops_fwd_bwd": 3.5 * ff / t / 1e12,
            "ms_bwd": tb * 1e3, "ms_bwd_median": statistics.median(ms_b), "tflops_bwd": tfb,
            "frac_bf16_peak_fwd_bwd": 3.5 * ff / t / 1e12 / peaks["bf16_tflops"],
            "roofline": roofline("tensor", tfb, peaks, peak_src, "TFLOP/s",
                                 traffic=profiled_traffic("bwd_main_kernel train_fwd_bwd"),
                                 algorithmic_bytes=bwd_bytes),
            "roofline_note": "backward call (input maxima, pre-pass, main kernel, dQ post-pass); traffic is the "
                             "main kernel's; its products run on fp16 (same tensor rate as bf16)",
            "dtype": "bf16 in and out; fp16 products (power-of-two scaled inputs), fp32 accumulate"}


def section_decode(fa, steps, warmup, flush, stream, peaks, peak_src, dev):
    """Split-KV decode on the contiguous cache, then the same step with the new
    token's K/V appended (fused KV append + decode)."""
    w = synth.WORKLOADS["splitkv_decode"]
    x = synth.decode_inputs(w.B, w.Hq, w.Hkv, w.Lk, w.D, w.seed, w.len_lo, w.len_hi, device=dev)
    q, kc, vc, sl = x["q"].to(dev), x["k_cache"], x["v_cache"], x["seqlens"].to(dev)
    ws = torch.empty(fa.decode_workspace_size(w.B, w.Hq, w.Lk + 1, w.D), dtype=torch.uint8, device=dev)
    o = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
    with nvtx("section splitkv_decode"):
        ms = time_steps(lambda: fa.decode(q, kc, vc, sl, scale=w.scale, workspace=ws, out=o, lse=lse), steps,
                        warmup, flush, stream)
    t = statistics.mean(ms) * 1e-3
    kv_bytes = float(x["seqlens"].to(torch.int64).sum()) * w.Hkv * w.D * 2 * 2
    gbs = kv_bytes / t / 1e9
    res = {"workload": "splitkv_decode", "kernel": "decode_split_kernel+decode_combine_kernel", "ms": t * 1e3,
           "ms_median": statistics.median(ms), "kv_bytes": kv_bytes, "gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
           "launches": 2 * steps,
           "roofline": roofline("hbm", gbs, peaks, peak_src, "GB/s",
                                traffic=profiled_traffic("decode_split_kernel splitkv_decode", kv_bytes),
                                algorithmic_bytes=kv_bytes)}
    # the same step with the new token's rows attended and written at row seqlens[b]
    # (seqlens is not advanced, so every step does the same work)
    kn, vn = (t_.to(dev) for t_ in synth.decode_new_rows(w.B, w.Hkv, w.D, w.seed))
    with nvtx("section splitkv_decode_append"):
        ms_a = time_steps(lambda: fa.decode_append(q, kn, vn, kc, vc, sl, scale=w.scale, workspace=ws, out=o,
                                                   lse=lse), steps, warmup, flush, stream)
    ta = statistics.mean(ms_a) * 1e-3
    new_bytes = 2.0 * (2 * w.B * w.Hkv * w.D * 2)          # new K/V rows read once and written once
    gbs_a = (kv_bytes + new_bytes) / ta / 1e9
    app = {"workload": "splitkv_decode_append", "kernel": "decode_split_kernel<append>+decode_combine_kernel",
           "ms": ta * 1e3, "ms_median": statistics.median(ms_a), "bytes": kv_bytes + new_bytes, "gbs": gbs_a,
           "frac_hbm": gbs_a / peaks["hbm_gbs"], "launches": 2 * steps,
           "roofline": roofline("hbm", gbs_a, peaks, peak_src, "GB/s",
                                traffic=profiled_traffic("decode_split_kernel<append> splitkv_decode", kv_bytes),
                                algorithmic_bytes=kv_bytes + new_bytes)}
    return res, app


def section_decode_paged(fa, steps, warmup, flush, stream, peaks, peak_src, dev, page_size=16):
    """Split-KV decode from a paged cache (pool of page_size-row pages in a
    seeded random order) holding the decode workload's rows."""
    w = synth.WORKLOADS["splitkv_decode"]
    x = synth.paged_decode_inputs(w.B, w.Hq, w.Hkv, w.D, page_size, w.seed, w.len_lo, w.len_hi, device=dev)
    q, kp, vp = x["q"].to(dev), x["k_pages"], x["v_pages"]
    tab, sl = x["page_table"].to(dev), x["seqlens"].to(dev)
    cap = tab.shape[1] * page_size
    ws = torch.empty(fa.decode_workspace_size(w.B, w.Hq, cap, w.D), dtype=torch.uint8, device=dev)
    o = torch.empty((w.B, w.Hq, w.D), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.B, w.Hq), dtype=torch.float32, device=dev)
    with nvtx("section splitkv_decode_paged"):
        ms = time_steps(lambda: fa.decode_paged(q, kp, vp, tab, sl, scale=w.scale, workspace=ws, out=o, lse=lse),
                        steps, warmup, flush, stream)
    t = statistics.mean(ms) * 1e-3
    kv_bytes = float(x["seqlens"].to(torch.int64).sum()) * w.Hkv * w.D * 2 * 2
    gbs = kv_bytes / t / 1e9
    return {"workload": f"splitkv_decode_paged{page_size}",
            "kernel": "decode_split_kernel<paged>+decode_combine_kernel", "page_size": page_size,
            "pool_pages": int(kp.shape[0]), "ms": t * 1e3, "ms_median": statistics.median(ms), "kv_bytes": kv_bytes,
            "gbs": gbs, "frac_hbm": gbs / peaks["hbm_gbs"], "launches": 2 * steps,
            "roofline": roofline("hbm", gbs, peaks, peak_src, "GB/s",
                                 traffic=profiled_traffic(f"decode_split_kernel<paged{page_size}> splitkv_decode",
                                                          kv_bytes),
                                 algorithmic_bytes=kv_bytes)}


def run_ours(args):
    import exact_tiled_attention_46_b200 as fa
    from exact_tiled_attention_46_b200 import build
    build.build()
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    dist = None
    if world > 1:
        import torch.distributed as dist
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream(dev)
    flush = l2_flusher(dev)
    w = synth.WORKLOADS[HEADLINE]
    x = synth.workload_inputs(w)
    q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
    o = torch.empty_like(q)
    lse = torch.empty((w.B, w.Hq, w.Lq), dtype=torch.float32, device=dev)

    def step():
        fa.fwd(q, k, v, scale=w.scale, causal=w.causal, out=o, lse=lse)

    for _ in range(args.warmup):
        flush()
        step()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    if rank == 0:
        clocks.start()
    # timed region: barrier + sync on both sides, per-step CUDA events on the launching stream
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    region0 = torch.cuda.Event(enable_timing=True)
    region1 = torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("headline causal_prefill")
    region0.record(stream)
    for s, e in evs:
        flush()
        s.record(stream)
        step()
        e.record(stream)
    region1.record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize()
    if dist:
        dist.barrier()
    ck = clocks.stop() if rank == 0 else None
    kernel_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in evs), dist, dev)
    ms_step = kernel_ms / args.steps
    flops = fwd_flops(w)
    value = whole_job_tflops(flops, world, args.steps, kernel_ms)
    tf_rank = flops / (ms_step * 1e-3) / 1e12

    # end to end through the public API: every step copies its inputs from
    # pinned host memory to the device, runs the forward and reads O and the LSE
    # back.  Steps are pipelined over two buffer sets: step i's inputs go in on
    # one copy stream while step i - 1's result comes back on another (PCIe is
    # full duplex) and the forward runs on a third.
    hq, hk, hv = (x[n].pin_memory() for n in ("q", "k", "v"))
    ho = [torch.empty(o.shape, dtype=o.dtype).pin_memory() for _ in range(2)]
    hl = [torch.empty(lse.shape, dtype=lse.dtype).pin_memory() for _ in range(2)]
    din = [(torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)) for _ in range(2)]
    dout = [(torch.empty_like(o), torch.empty_like(lse)) for _ in range(2)]
    s_in, s_run, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def e2e_run(n):
        ran, back = [None, None], [None, None]     # per buffer set: its forward done / its result read back
        t0 = torch.cuda.Event(enable_timing=True)
        t0.record(s_in)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if ran[b] is not None:
                    s_in.wait_event(ran[b])           # the inputs of step i - 2 are no longer read
                for d, h in zip(din[b], (hq, hk, hv)):
                    d.copy_(h, non_blocking=True)
                e_in = torch.cuda.Event()
                e_in.record(s_in)
            with torch.cuda.stream(s_run):
                s_run.wait_event(e_in)
                if back[b] is not None:
                    s_run.wait_event(back[b])         # the result of step i - 2 has been read back
                fa.fwd(*din[b], scale=w.scale, causal=w.causal, out=dout[b][0], lse=dout[b][1])
                ran[b] = torch.cuda.Event()
                ran[b].record(s_run)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ran[b])
                ho[b].copy_(dout[b][0], non_blocking=True)
                hl[b].copy_(dout[b][1], non_blocking=True)
                back[b] = torch.cuda.Event()
                back[b].record(s_out)
        t1 = torch.cuda.Event(enable_timing=True)
        t1.record(s_out)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)
    e2e_run(3)
    n_e2e = max(3, args.steps // 4)
    e2e_ms = max_over_ranks(e2e_run(n_e2e), dist, dev) / n_e2e

    # kernel-only cross-check: the same call captured once in a CUDA graph and
    # replayed (no host work between the events but the replay itself)
    graph_ms = None
    try:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step()
        torch.cuda.synchronize()
        graph_ms = time_steps(g.replay, max(3, min(args.steps, 50)), 3, flush, stream)
        del g
    except Exception as e:  # reported, never fatal: the headline does not depend on it
        graph_ms = str(e)[:200]
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = ho[0].numel() * ho[0].element_size() + hl[0].numel() * hl[0].element_size()
    e2e_val = flops * world / (e2e_ms * 1e-3) / 1e12

    sections = {}
    if not args.quick:
        sec_steps = max(3, min(args.steps, 20))
        sections["long_gqa_prefill"] = section_fwd(fa, "long_gqa_prefill", sec_steps, 3, flush, stream, peaks,
                                                   peak_src, dev)
        sections["causal_prefill_fp8"] = section_fwd_fp8(fa, "causal_prefill", sec_steps, 3, flush, stream, peaks,
                                                         peak_src, dev)
        sections["train_fwd_bwd"] = section_train(fa, sec_steps, 3, flush, stream, peaks, peak_src, dev)
        sections["splitkv_decode"], sections["splitkv_decode_append"] = section_decode(
            fa, sec_steps, 3, flush, stream, peaks, peak_src, dev)
        torch.cuda.empty_cache()
        sections["splitkv_decode_paged16"] = section_decode_paged(fa, sec_steps, 3, flush, stream, peaks, peak_src,
                                                                  dev, 16)
        torch.cuda.empty_cache()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu:
        # the headline's GPU output, for the parity columns of the CPU-baseline leg
        fa.fwd(q, k, v, scale=w.scale, causal=w.causal, out=o, lse=lse)
        torch.cuda.synchronize()
        cpu = cpu_baseline(budget_s=args.cpu_budget, gpu_out=(o.cpu(), lse.cpu()))

    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1), bf16 RNE)",
        "config": {"workload": "causal_prefill B4 Hq16 Hkv16 L2048 D128 causal, Q x4 on heads 0-7",
                   "global_batch": w.B * world, "seq_len": w.Lq, "heads": w.Hq, "head_dim": w.D,
                   "parallelism": f"replicas{world}", "l2": "flushed (256 MiB write) before every timed step",
                   "flops_per_step": flops, "flop_count": "4*B*H*D*allowed_pairs, causal pairs counted once"},
        "ms_median": statistics.median(s.elapsed_time(e) for s, e in evs),
        "graph_replay_ms": (statistics.mean(graph_ms) if isinstance(graph_ms, list) else graph_ms),
        "roofline": roofline("tensor", tf_rank, peaks, peak_src, "TFLOP/s",
                             traffic=profiled_traffic("fwd_kernel causal_prefill"), algorithmic_bytes=fwd_bytes(w)),
        "e2e": {"value": e2e_val, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "schedule": "pinned host buffers; consecutive steps' H2D, forward and D2H overlapped on three "
                            "streams over two device buffer sets"},
        "gpu_launches": args.steps,
        "clocks": ck,
        "sections": sections,
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


# --------------------------------------------------------- oracle timing ---
def oracle_sample(w, n_heads, gpu_out=None):
    """The oracle on the first n_heads (batch, head) slices of the workload.

    With ``gpu_out`` = (O, LSE) of the CUDA path on the same inputs, also
    returns the parity errors of those slices (max / mean |O - oracle|, max
    |LSE - oracle|)."""
    sys.path.insert(0, ROOT)
    import oracle
    x = synth.workload_inputs(w)
    xf = {n: synth.as_f64(x[n]) for n in ("q", "k", "v")}
    G = w.Hq // w.Hkv
    pairs = [(b, h) for b in range(w.B) for h in range(w.Hq)][:n_heads]
    outs = []
    t0 = time.perf_counter()
    for b, h in pairs:
        outs.append(oracle.attn_fwd(xf["q"][b:b + 1, :, h:h + 1], xf["k"][b:b + 1, :, h // G:h // G + 1],
                                    xf["v"][b:b + 1, :, h // G:h // G + 1], w.scale, w.causal))
    dt = time.perf_counter() - t0
    flops = 4.0 * w.D * allowed_pairs(w.Lq, w.Lk, w.causal) * len(pairs)
    if gpu_out is None:
        return flops, dt
    go, gl = (t.to(torch.float64).numpy() for t in gpu_out)
    emax = emean = lmax = 0.0
    for (b, h), (ro, rl) in zip(pairs, outs):
        err = np.abs(go[b:b + 1, :, h:h + 1] - ro)
        emax, emean = max(emax, float(err.max())), emean + float(err.mean()) / len(pairs)
        fin = np.isfinite(rl)
        lmax = max(lmax, float(np.abs(gl[b:b + 1, h:h + 1][fin] - rl[fin]).max(initial=0.0)))
    return flops, dt, {"slices": len(pairs), "o_max_abs": emax, "o_mean_abs": emean, "lse_max_abs": lmax,
                       "o_dtype": "bf16 (errors include the output's own rounding)"}


def cpu_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


def cpu_baseline(budget_s=15.0, gpu_out=None):
    w = synth.WORKLOADS[HEADLINE]
    f1, t1 = oracle_sample(w, 1)
    n = max(1, min(w.B * w.Hq, int(budget_s / max(t1, 1e-3))))
    res = oracle_sample(w, n, gpu_out)
    f, t = res[0], res[1]
    out = {"value": f / t / 1e12, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
           "sample": f"{n} of {w.B * w.Hq} (batch, head) slices of causal_prefill, NumPy fp64, {t:.1f} s"}
    if gpu_out is not None:
        out["parity_vs_gpu"] = res[2]
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    w = synth.WORKLOADS[HEADLINE]
    oracle_sample(w, 1)   # warm imports / BLAS threads
    for _ in range(max(0, args.warmup - 1)):
        oracle_sample(w, 1)
    per = []
    flops_total, t_total = 0.0, 0.0
    for _ in range(args.steps):
        f, t = oracle_sample(w, 2)
        per.append(t)
        flops_total += f
        t_total += t
    value = flops_total / t_total / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t_total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded N(0,1), bf16 RNE)",
        "config": {"workload": "causal_prefill B4 Hq16 Hkv16 L2048 D128 causal, Q x4 on heads 0-7",
                   "sample_per_step": "2 (batch, head) slices"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
                         "sample": "2 (batch, head) slices of causal_prefill per step, NumPy fp64"},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def run_profile_case(args):
    """A few launches of one kernel on one workload, for ncu captures (no timing).

    causal_prefill / long_gqa_prefill / train_fwd_bwd: fa_fwd (and fa_bwd);
    splitkv_decode_small / _append_small / _paged16_small: split-KV decode
    (plain, with the new token appended, from 16-row pages) on the first 16
    sequences of the decode workload (KV rows 1.36 GB, larger than L2);
    causal_prefill_fp8: the causal prefill draws quantized to e4m3.
    """
    import exact_tiled_attention_46_b200 as fa
    from exact_tiled_attention_46_b200 import build
    build.build()
    dev = torch.device("cuda", 0)
    name = args.profile_case
    if name in ("splitkv_decode_small", "splitkv_decode_append_small"):
        w = synth.WORKLOADS["splitkv_decode"]
        B = 16
        x = synth.decode_inputs(B, w.Hq, w.Hkv, w.Lk, w.D, w.seed, w.len_lo, w.len_hi, device=dev)
        q, sl = x["q"].to(dev), x["seqlens"].to(dev)
        kn, vn = (t.to(dev) for t in synth.decode_new_rows(B, w.Hkv, w.D, w.seed))
        for _ in range(args.warmup + args.steps):
            if name == "splitkv_decode_small":
                fa.decode(q, x["k_cache"], x["v_cache"], sl, scale=w.scale)
            else:
                fa.decode_append(q, kn, vn, x["k_cache"], x["v_cache"], sl, scale=w.scale)
    elif name == "splitkv_decode_paged16_small":
        w = synth.WORKLOADS["splitkv_decode"]
        B = 16
        x = synth.paged_decode_inputs(B, w.Hq, w.Hkv, w.D, 16, w.seed, w.len_lo, w.len_hi, device=dev)
        q, tab, sl = x["q"].to(dev), x["page_table"].to(dev), x["seqlens"].to(dev)
        for _ in range(args.warmup + args.steps):
            fa.decode_paged(q, x["k_pages"], x["v_pages"], tab, sl, scale=w.scale)
    elif name == "causal_prefill_fp8":
        w = synth.WORKLOADS["causal_prefill"]
        x = synth.prefill_inputs_fp8(w.B, w.Hq, w.Hkv, w.Lq, w.Lk, w.D, w.seed, q_boost_heads=w.q_boost_heads)
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        for _ in range(args.warmup + args.steps):
            fa.fwd_fp8(q, k, v, x["q_scale"], x["k_scale"], x["v_scale"], scale=w.scale, causal=True)
    else:
        w = synth.WORKLOADS[name]
        x = synth.workload_inputs(w)
        q, k, v = (x[n].to(dev) for n in ("q", "k", "v"))
        o, lse = fa.fwd(q, k, v, scale=w.scale, causal=w.causal)
        if w.kind == "train":
            do = x["do"].to(dev)
            for _ in range(args.warmup + args.steps):
                fa.bwd(q, k, v, o, do, lse, scale=w.scale, causal=w.causal)
        else:
            for _ in range(args.warmup + args.steps):
                fa.fwd(q, k, v, scale=w.scale, causal=w.causal, out=o, lse=lse)
    torch.cuda.synchronize()
    print(f"profile case {name}: {args.warmup + args.steps} launches done")


CONFIGS = {1: "tiny_fwd", 2: "causal_prefill", 3: "long_gqa_prefill", 4: "train_fwd_bwd", 5: "splitkv_decode"}


def run_config(args):
    """One workload alone (configs 1-5 in the order the workloads are listed);
    prints one JSON line with that workload's own metric as the value."""
    import exact_tiled_attention_46_b200 as fa
    from exact_tiled_attention_46_b200 import build
    build.build()
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peaks, peak_src = load_peaks()
    stream = torch.cuda.current_stream(dev)
    flush = l2_flusher(dev)
    name = CONFIGS[args.config]
    clocks = ClockSampler(0)
    clocks.start()
    if name == "train_fwd_bwd":
        sec = section_train(fa, args.steps, args.warmup, flush, stream, peaks, peak_src, dev)
        value, unit, ms = sec.get("tflops_bwd"), "TFLOP/s", sec.get("ms_bwd")
    elif name == "splitkv_decode":
        sec, _ = section_decode(fa, args.steps, args.warmup, flush, stream, peaks, peak_src, dev)
        value, unit, ms = sec["gbs"], "GB/s", sec["ms"]
    else:
        sec = section_fwd(fa, name, args.steps, args.warmup, flush, stream, peaks, peak_src, dev)
        value, unit, ms = sec["tflops"], "TFLOP/s", sec["ms"]
    ck = clocks.stop()
    w = synth.WORKLOADS[name]
    print(json.dumps({"metric": METRIC, "value": value, "unit": unit, "n_gpus": 1, "steps": args.steps,
                      "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
                      "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1), bf16 RNE)",
                      "config": {"workload": name, "config_index": args.config, "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv,
                                 "L": w.Lk, "D": w.D, "causal": w.causal,
                                 "l2": "flushed (256 MiB write) before every timed step"},
                      "roofline": sec.get("roofline"), "clocks": ck, "section": sec}), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--profile-case", default=None,
                    choices=["causal_prefill", "long_gqa_prefill", "train_fwd_bwd", "splitkv_decode_small",
                             "splitkv_decode_append_small", "splitkv_decode_paged16_small", "causal_prefill_fp8"])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--quick", action="store_true", help="headline only, no extra sections")
    ap.add_argument("--no-cpu", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--cpu-budget", type=float, default=15.0)
    ap.add_argument("--config", type=int, choices=sorted(CONFIGS), default=None,
                    help="time one workload alone (1 tiny, 2 causal prefill = the default headline run, "
                         "3 long GQA, 4 training backward, 5 decode)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.profile_case:
        run_profile_case(args)
    elif args.config is not None and args.config != 2 and args.impl == "ours":
        run_config(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
