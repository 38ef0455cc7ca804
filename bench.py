#!/usr/bin/env python
"""Benchmark of the Elastic Attention prefill hot path on B200.

One step = one attention layer's prefill: the Attention Router
(ea_router_decide) on the key states, then the fused hybrid FA/SA attention
(ea_hybrid_attn_prefill), on seeded synthetic inputs already resident in HBM.
The headline workload is the largest single-GPU configuration, a 256K-token
layer (B1 N262144, 32 query / 8 kv heads, d128, sink 128, window 4096,
router-chosen ~75% sparse heads); the other configurations follow under
"workloads", each with its own roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Prints ONE JSON line on rank 0.  Multi-GPU runs (torchrun, one rank per GPU)
shard one layer over the ranks by (batch, kv group), balanced by the mask's
per-group cost; the router's pooled key vector is the one exchange (an NCCL
all-gather of the ranks' pooled slices).  The work is fixed as N grows
(strong scaling); the time is the max over ranks.

--impl reference times the CPU oracle (float64 numpy, the plain definition of
the method) on a bounded sample of the same workload, on the host cores.
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads  # noqa: E402

METRIC = "effective prefill attention TFLOPS and tokens/s at 1 B200; % of bf16 tensor peak"
UNIT = "TFLOP/s"
NOMINAL_BF16_TFLOPS = 2250.0   # dense bf16 per B200 (the 2:4-sparse figure halved)
L2_BYTES = 126 * 10 ** 6       # B200 L2
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "hbm_gbs": 6650.0}


# ---------------------------------------------------------------- helpers
def parse_args():
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="ext256k", choices=sorted(workloads.WORKLOADS),
                    help="headline workload (default: the largest single-GPU configuration)")
    ap.add_argument("--side-workload", default="llama8b", choices=sorted(workloads.WORKLOADS),
                    help="layer shape of the secondary measurements (packed batch, decode, "
                         "FP8, training) when the headline workload is ext256k")
    ap.add_argument("--no-extra-workloads", action="store_true",
                    help="skip the attention measurements of the other configurations")
    ap.add_argument("--e2e-steps", type=int, default=None,
                    help="steps of the host-buffer end-to-end measurement (default: --steps)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--seq", type=int, default=None,
                    help="override the workload's sequence length (profiling cases)")
    ap.add_argument("--decode-batch", type=int, default=16,
                    help="sequences in the decode measurement (0 skips it)")
    ap.add_argument("--decode-only", action="store_true",
                    help="run only the decode measurement and print its JSON object")
    ap.add_argument("--packed-seqs", type=int, default=8,
                    help="sequences in the packed-batch measurement (0 skips it)")
    ap.add_argument("--training-only", "--backward-only", dest="training_only",
                    action="store_true",
                    help="run only the training-step measurement (router, both-mode "
                         "forward, backward, router gradients)")
    ap.add_argument("--no-fp8", action="store_true",
                    help="skip the FP8-variant measurement of the default line")
    ap.add_argument("--fp8-only", action="store_true",
                    help="run only the FP8-variant measurement and print its JSON object")
    ap.add_argument("--no-training", action="store_true",
                    help="skip the training-step measurement of the default line")
    ap.add_argument("--packed-only", action="store_true",
                    help="run only the packed-batch measurement and print its JSON object")
    ap.add_argument("--ab-reps", type=int, default=20,
                    help="calls of each arm in the interleaved comparator timings")
    ap.add_argument("--quick", action="store_true",
                    help="timed region only: no comparators, e2e or CPU baseline")
    ap.add_argument("--unit-trace", action="store_true",
                    help="one fused-attention launch with the per-unit trace: the CTAs' "
                         "finish spread, busy fraction and FA/SA interleave (JSON)")
    ap.add_argument("--host-timeline", action="store_true",
                    help="one host-buffer call under the torch profiler: device busy and "
                         "overlap times of the uploads, downloads and kernels (JSON)")
    return ap.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(w: workloads.Workload, mask_frac: float) -> str:
    s = (f"{w.name}: B{w.batch} N{w.seq} Hq{w.hq} Hkv{w.hkv} d{w.d} sink{w.sink} "
         f"window{w.window}")
    if w.use_router:
        s += f" router {w.hkv * w.d}-{w.router_hidden}-{w.hq}"
    s += f" sparse-head fraction {mask_frac:.3f}"
    if w.layers > 1:
        s += f" x{w.layers} layers"
    return s


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 200 ms while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.idx = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.idx), "-lms", "200"], stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None, "reasons": reasons,
                "samples": len(rows)}


def visible_gpu_index(local_rank: int) -> int:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x for x in vis.split(",") if x.strip()]
        if local_rank < len(ids) and ids[local_rank].strip().isdigit():
            return int(ids[local_rank])
    return local_rank


ATTN_KERNEL_SOURCES = ("ea_attn.cu", "ea_sched.h", "ea_internal.h", "ea_ptx.cuh", "ea_tmem.cuh",
                       "ea_math.cuh")


def attn_kernel_source_hash() -> str:
    """sha256 (16 hex digits) over the fused attention kernel's source files,
    in the order of ATTN_KERNEL_SOURCES."""
    h = hashlib.sha256()
    for name in ATTN_KERNEL_SOURCES:
        with open(os.path.join(ROOT, "sparse_attention_head_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def traffic_for_current_kernel(workload: str, seq: int):
    """Per-launch DRAM bytes of the attention kernel on this workload, from the
    committed ncu summary: only if a capture exists for this workload at this
    sequence length and was taken on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "attn_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    if d.get("kernel_sha256_16") != attn_kernel_source_hash():
        return None
    e = d.get("workloads", {}).get(workload)
    if not e or int(e.get("seq", -1)) != int(seq):
        return None
    return e.get("dram_bytes_per_launch")


def roofline_peak(timed_region_ms: float):
    """The bf16 peak a kernel is held against: the burst figure for a kernel
    timed alone, the sustained one (seconds back to back under the power cap)
    when the timed region keeps the kernel busy for a second or more.
    Returns (peak, kind, burst peak, source)."""
    peaks, src = load_peaks()
    burst = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    sustained = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    if timed_region_ms >= 1000.0:
        return sustained, "sustained", burst, src
    return burst, "burst", burst, src


def bench_config(w: workloads.Workload, sparse_frac: float, world: int) -> dict:
    """The `config` of the JSON line; both arms print the same dict."""
    in_bytes = w.layers * w.batch * (w.hq + 2 * w.hkv) * w.seq * w.d * 2
    l2 = (("inputs %.1f MiB fit in L2: 256 MiB flush between timed steps, each step timed on "
           "its own" % (in_bytes / 2 ** 20)) if in_bytes < 2 * L2_BYTES else
          ("inputs exceed L2 (Q+K+V %.0f MiB > 126 MB), no flush" % (in_bytes / 2 ** 20)))
    return {"workload": workload_desc(w, sparse_frac), "global_batch": w.batch,
            "seq_len": w.seq,
            "parallelism": ("single GPU" if world == 1 else
                            f"(batch, kv group) shards x{world}, a group over a rank's share split "
                            "by query head: LPT on the mask's tile cost, "
                            "all-gather of the router's pooled slices"),
            "l2": l2}


def serial_dispatch_pass(q, k, v, mask, w: workloads.Workload, dev):
    """The serial dispatch that EA blog §3 sets the fused kernel against: the
    (b, h) heads are split by route into an FA group and an SA group, each
    group's q rows and K/V (repeated per query head, as a PyTorch-level split
    without a head map must) are gathered into a tensor of their own, each
    group runs in a launch of its own, and the two outputs are concatenated
    back into out's head order.  Returns (the pass, its output tensor); the
    gather and scatter buffers and the workspaces are allocated here, outside
    any timed region."""
    from sparse_attention_head_b200.api import attn_workspace, ea_hybrid_attn_prefill, make_params
    B, Hq, N, d = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    m = mask.reshape(-1).to(torch.int64)
    heads = torch.arange(B * Hq, device=dev)
    kv_of = (heads // Hq) * Hkv + (heads % Hq) // G
    q2, k2, v2 = q.reshape(B * Hq, N, d), k.reshape(B * Hkv, N, d), v.reshape(B * Hkv, N, d)
    out = torch.empty_like(q)
    out2 = out.view(B * Hq, N, d)
    groups = []
    for mode in (0, 1):
        idx = heads[m == mode] if mode == 0 else heads[m != 0]
        n = int(idx.numel())
        if n == 0:
            continue
        kv_idx = kv_of[idx]
        bufs = [torch.empty((1, n, N, d), dtype=q.dtype, device=dev) for _ in range(4)]
        gmask = torch.full((1, n), mode, dtype=torch.uint8, device=dev)
        ws = attn_workspace(make_params(1, n, n, N, d, w.sink, w.window), dev)
        groups.append((idx, kv_idx, bufs, gmask, ws))

    def serial():
        for idx, kv_idx, (qg, kg, vg, og), gmask, ws in groups:
            torch.index_select(q2, 0, idx, out=qg[0])
            torch.index_select(k2, 0, kv_idx, out=kg[0])
            torch.index_select(v2, 0, kv_idx, out=vg[0])
            ea_hybrid_attn_prefill(qg, kg, vg, gmask, w.sink, w.window, out=og, workspace=ws)
            out2.index_copy_(0, idx, og[0])
    return serial, out


def ab_medians(fns, reps: int, stream):
    """Median device time (ms) of each function, called in interleaved order
    (a, b, ..., a, b, ...) after one warm call each, every call timed with its
    own CUDA events on `stream`."""
    for fn in fns:
        fn()
    torch.cuda.synchronize()
    times = [[] for _ in fns]
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(reps)] for _ in fns]
    for r in range(reps):
        for i, fn in enumerate(fns):
            evs[i][r][0].record(stream)
            fn()
            evs[i][r][1].record(stream)
    torch.cuda.synchronize()
    for i in range(len(fns)):
        times[i] = [a.elapsed_time(b) for a, b in evs[i]]
    return [statistics.median(t) for t in times], times


# ---------------------------------------------------------------- ranks
def rank_seed(w: workloads.Workload, layer: int, rank: int) -> int:
    """Each rank runs its own replica of the workload with its own inputs."""
    return workloads.layer_seed(w, layer) + 7919 * rank


def max_over_ranks(value: float, world: int, device) -> float:
    """The slowest rank's time (every rank takes part; no-op on one rank)."""
    if world <= 1:
        return float(value)
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ---------------------------------------------------------------- inputs
def make_layer(w: workloads.Workload, layer: int, rank: int, device):
    seed = rank_seed(w, layer, rank)
    q, k, v = workloads.make_qkv(w, seed, device=device)
    if w.use_router:
        frac = workloads.layer_sparse_frac(w, layer)
        heads = workloads.sparse_head_set(w.hq, frac, seed)
        w1, b1, w2, b2 = workloads.make_router_weights(w.hkv * w.d, w.router_hidden, w.hq,
                                                       heads, seed)
        router = tuple(t.to(device) for t in (w1, b1, w2, b2))
        mask = None
    else:
        router = None
        mask = workloads.make_fixed_mask(w, seed).to(device)
    return {"q": q, "k": k, "v": v, "router": router, "mask": mask, "seed": seed}


# ---------------------------------------------------------------- our arm
def run_ours(args, rank, world, local_rank):
    from sparse_attention_head_b200 import flops
    from sparse_attention_head_b200.api import (EA_SELECT_FA, EA_SELECT_SA, HostPrefill,
                                                attn_workspace, ea_get_device_status,
                                                ea_hybrid_attn_prefill, ea_router_decide,
                                                ea_router_workspace_size, make_params)
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = workloads.get(args.workload)
    if args.seq:
        w = dataclasses.replace(w, seq=args.seq)
    B, Hq, Hkv, N, d = w.batch, w.hq, w.hkv, w.seq, w.d
    nlayers = w.layers
    # every layer's inputs stay resident in HBM (36 x 768 MiB for qwen8b36)
    layers = [make_layer(w, l, rank, dev) for l in range(nlayers)]
    p = make_params(B, Hq, Hkv, N, d, w.sink, w.window)
    aws = attn_workspace(p, dev)
    rws = torch.empty(max(ea_router_workspace_size(B, Hkv, N, d), 16), dtype=torch.uint8,
                      device=dev)
    outs = [torch.empty_like(L["q"]) for L in layers]
    masks = [torch.empty((B, Hq), dtype=torch.uint8, device=dev) if L["router"] is not None
             else L["mask"] for L in layers]
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        for li, L in enumerate(layers):
            if ev is not None:
                ev[li][0].record(stream)
            if L["router"] is not None:
                ea_router_decide(L["k"], *L["router"], workspace=rws, route_mask=masks[li],
                                 want_logits=False)
            if ev is not None:
                ev[li][1].record(stream)
            ea_hybrid_attn_prefill(L["q"], L["k"], L["v"], masks[li], w.sink, w.window,
                                   out=outs[li], workspace=aws)
            if ev is not None:
                ev[li][2].record(stream)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    if ea_get_device_status(aws) != 0:
        raise RuntimeError("device status word reports an error after warm-up")

    mask_host = [m.cpu().numpy() for m in masks]
    eff = sum(flops.effective_flops(m, N, d, w.sink, w.window) for m in mask_host)
    tile = sum(flops.tile_flops(m, N, d, w.sink, w.window) for m in mask_host)
    sparse_frac = float(np.mean([m.mean() for m in mask_host]))

    K = args.steps
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(nlayers)]
           for _ in range(K)]
    # Inputs that fit in L2 get it flushed between timed steps (a 256 MiB
    # write, outside the steps' events); larger inputs stream from HBM anyway.
    in_bytes = nlayers * B * (Hq + 2 * Hkv) * N * d * 2
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if in_bytes < 2 * L2_BYTES \
        else None
    step_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(visible_gpu_index(local_rank)) if rank == 0 else None
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    t0.record(stream)
    for i in range(K):
        if flush is not None:
            flush.fill_(i & 0xff)
        step_ev[i][0].record(stream)
        step(evs[i])
        step_ev[i][1].record(stream)
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = sampler.stop() if sampler else None
    # with flushes, the steps' own intervals; without, the whole region
    total_ms = (sum(a.elapsed_time(b) for a, b in step_ev) if flush is not None
                else t0.elapsed_time(t1))
    attn_ms = [evs[i][l][1].elapsed_time(evs[i][l][2]) for i in range(K) for l in range(nlayers)]
    router_ms = [evs[i][l][0].elapsed_time(evs[i][l][1]) for i in range(K)
                 for l in range(nlayers)]
    total_ms = max_over_ranks(total_ms, world, dev)
    if ea_get_device_status(aws) != 0:
        raise RuntimeError("device status word reports an error after the timed region")

    ms_per_step = total_ms / K
    value = eff * world / (ms_per_step * 1e-3) / 1e12
    tokens_per_s = B * N * world / (ms_per_step * 1e-3)
    peak, peak_kind, burst, peak_src = roofline_peak(total_ms)
    attn_avg_ms = statistics.mean(attn_ms)
    achieved = (eff / nlayers) / (attn_avg_ms * 1e-3) / 1e12

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": bench_config(w, sparse_frac, world),
        "tokens_per_s": round(tokens_per_s, 1),
        "pct_of_bf16_peak": round(100.0 * value / world / peak, 2),
        "pct_of_burst_bf16_peak": round(100.0 * value / world / burst, 2),
        # the same against the nominal dense bf16 figure (2.25 PFLOP/s per GPU)
        "pct_of_nominal_bf16_dense": round(100.0 * value / world / NOMINAL_BF16_TFLOPS, 2),
        "tile_granular_tflops": round(tile * world / (ms_per_step * 1e-3) / 1e12, 2),
        "attn_ms": round(attn_avg_ms, 4),
        "router_ms": round(statistics.mean(router_ms), 4),
        # router: pool, reduce and the two MLP layers; then the attention launch
        "gpu_launches": K * nlayers * (5 if layers[0]["router"] is not None else 1),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "peak_source": (f"{peak_src} bf16_tflops_{peak_kind}" if peak_kind ==
                                     "sustained" else f"{peak_src} bf16_tflops (burst)"),
                     "peak_rule": ("sustained: the timed region keeps the kernel busy back to "
                                   "back for %.1f s (>= 1 s, under the power cap)"
                                   % (total_ms / 1e3)) if peak_kind == "sustained" else
                                  ("burst: the timed region is %.0f ms (< 1 s)" % total_ms),
                     "frac_of_burst_peak": round(achieved / burst, 4),
                     "traffic": traffic_for_current_kernel(w.name, N),
                     "kernel": "ea_hybrid_attn_kernel<128>"},
        "clocks": clocks,
    }

    if not args.quick and world == 1:
        # comparators on the same inputs (outside the timed region), each pair
        # timed call by call in interleaved order, medians reported
        L = layers[0]
        m0 = masks[0]
        out_tmp = torch.empty_like(L["q"])
        reps = args.ab_reps

        def split_pass():
            ea_hybrid_attn_prefill(L["q"], L["k"], L["v"], m0, w.sink, w.window,
                                   select=EA_SELECT_FA, out=out_tmp, workspace=aws)
            ea_hybrid_attn_prefill(L["q"], L["k"], L["v"], m0, w.sink, w.window,
                                   select=EA_SELECT_SA, out=out_tmp, workspace=aws)

        def fused():
            ea_hybrid_attn_prefill(L["q"], L["k"], L["v"], m0, w.sink, w.window,
                                   out=out_tmp, workspace=aws)
        all_fa = torch.zeros_like(m0)

        def full_causal():
            ea_hybrid_attn_prefill(L["q"], L["k"], L["v"], all_fa, w.sink, w.window,
                                   out=out_tmp, workspace=aws)
        serial_pass, serial_out = serial_dispatch_pass(L["q"], L["k"], L["v"], m0, w, aws.device)
        (fused_ms, split_ms, serial_ms), (fused_t, split_t, serial_t) = ab_medians(
            [fused, split_pass, serial_pass], reps, stream)
        fused()
        serial_pass()
        torch.cuda.synchronize()
        serial_identical = bool(torch.equal(out_tmp, serial_out))
        del serial_pass, serial_out
        (full_ms,), _ = ab_medians([full_causal], max(3, min(reps, 5)), stream)
        full_eff = flops.effective_flops(all_fa.cpu().numpy(), N, d, w.sink, w.window)
        wins = sum(1 for a, b in zip(fused_t, split_t) if a < b)
        result["comparators"] = {
            "timing": f"interleaved A/B, {reps} calls each after one warm call, medians",
            "fused_attn_ms": round(fused_ms, 4),
            "split_fa_then_sa_ms": round(split_ms, 4),
            "fused_speedup_vs_split": round(split_ms / fused_ms, 4),
            "fused_faster_in_pairs": f"{wins}/{reps}",
            "fused_ms_range": [round(min(fused_t), 4), round(max(fused_t), 4)],
            "split_ms_range": [round(min(split_t), 4), round(max(split_t), 4)],
            "serial_dispatch_ms": round(serial_ms, 4),
            "fused_speedup_vs_serial_dispatch": round(serial_ms / fused_ms, 4),
            "fused_faster_than_serial_in_pairs":
                f"{sum(1 for a, b in zip(fused_t, serial_t) if a < b)}/{reps}",
            "serial_dispatch": "heads grouped by route as the pages' PyTorch-level pass does it: "
                               "q rows and each head's K/V gathered into one tensor per mode "
                               "(index_select), one launch per mode, outputs concatenated back "
                               "(index_copy_); the same kernel does the attention; output "
                               "bit-identical to the fused launch: %s" % serial_identical,
            "full_causal_ms": round(full_ms, 4),
            "full_causal_tflops": round(full_eff / (full_ms * 1e-3) / 1e12, 2),
            "elastic_speedup_vs_full_causal": round(full_ms / fused_ms, 3),
        }
        if L["router"] is not None:
            # router + attention: the two-launch pass against the one routed
            # (cooperative) launch that runs the router in its prologue
            from sparse_attention_head_b200.api import ea_hybrid_attn_prefill_routed
            m_tmp = torch.empty_like(masks[0])
            ws_routed = torch.zeros(
                max(1 << 24, ea_router_workspace_size(B, Hkv, N, d) + (1 << 20)),
                dtype=torch.uint8, device=dev)

            def two_launch():
                ea_router_decide(L["k"], *L["router"], workspace=rws, route_mask=m_tmp,
                                 want_logits=False)
                ea_hybrid_attn_prefill(L["q"], L["k"], L["v"], m_tmp, w.sink, w.window,
                                       out=out_tmp, workspace=aws)

            def routed():
                ea_hybrid_attn_prefill_routed(L["q"], L["k"], L["v"], *L["router"], w.sink,
                                              w.window, route_mask=m_tmp, out=out_tmp,
                                              workspace=ws_routed)
            (two_ms, routed_ms), (two_t, routed_t) = ab_medians([two_launch, routed], reps,
                                                                stream)
            if ea_get_device_status(ws_routed) != 0:
                raise RuntimeError("routed launch status word reports an error")
            result["comparators"].update({
                "router_then_attn_ms": round(two_ms, 4),
                "routed_one_launch_ms": round(routed_ms, 4),
                "routed_speedup_vs_two_launches": round(two_ms / routed_ms, 4),
                "routed_faster_in_pairs":
                    f"{sum(1 for a, b in zip(routed_t, two_t) if a < b)}/{reps}",
            })
        if rank == 0:
            result["cpu_baseline"] = cpu_baseline(w, L, m0.cpu().numpy(), args.cpu_seconds)
    if not args.quick:
        # end to end through the public API with host buffers, on every rank
        # (layer 0; for a multi-layer workload the metric uses that layer's
        # work only); the timed region is the slowest rank's
        L = layers[0]
        ek = args.e2e_steps or K
        router = L["router"] if L["router"] is not None else (None, None, None, None)
        hp = HostPrefill(B, Hq, Hkv, N, d, *router, w.sink, w.window, device=dev)
        qh = L["q"].cpu().pin_memory()
        kh = L["k"].cpu().pin_memory()
        vh = L["v"].cpu().pin_memory()
        mh = None if L["router"] is not None else L["mask"].cpu().pin_memory()
        for _ in range(2):
            hp(qh, kh, vh, mh)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(ek):
            hp(qh, kh, vh, mh)
        b.record(stream)
        torch.cuda.synchronize()
        if world > 1:
            torch.distributed.barrier()
        e2e_ms = max_over_ranks(a.elapsed_time(b) / ek, world, dev)
        if ea_get_device_status(hp.workspace) != 0:
            raise RuntimeError("host-buffer path status word reports an error")
        eff0 = flops.effective_flops(mask_host[0], N, d, w.sink, w.window)
        result["e2e"] = {"value": round(eff0 * world / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                         "h2d_bytes_per_step": hp.h2d_bytes() * world,
                         "d2h_bytes_per_step": hp.d2h_bytes() * world,
                         "ms_per_step": round(e2e_ms, 4),
                         "path": "ea_hybrid_attn_prefill_host: pinned host q,k,v -> " +
                                 ("ea_router_decide" if L["router"] is not None
                                  else "route mask copy") +
                                 f" -> {hp.chunks} kv-head chunks (upload, fused attention, "
                                 "download overlapped) -> pinned host out"
                                 + (" (layer 0)" if nlayers > 1 else "")
                                 + (f", one replica per rank x{world}" if world > 1 else "")}
    # The secondary measurements run on layers of their own: the headline's
    # tensors are released first.  With the 256K headline they take the
    # side workload's layer shape (each names its workload).
    layers.clear()
    outs.clear()
    masks.clear()
    L = hp = qh = kh = vh = mh = out_tmp = None
    torch.cuda.empty_cache()
    side = workloads.get(args.side_workload) if w.name == "ext256k" else w
    if not args.quick and world == 1 and not args.no_extra_workloads and args.seq is None:
        result["workloads"] = {}
        for name in ("llama8b", "qwen4b", "qwen8b36", "ext256k"):
            if name != w.name:
                result["workloads"][name] = measure_workload(workloads.get(name), dev, stream)
                torch.cuda.empty_cache()
    if not args.quick and world == 1 and args.packed_seqs > 0:
        result["packed"] = measure_packed(side, args.packed_seqs, max(args.steps, 5),
                                          max(args.warmup, 3), dev, stream)
    if not args.quick and world == 1 and args.decode_batch > 0:
        dec_sampler = ClockSampler(visible_gpu_index(local_rank))
        dec_sampler.start()
        result["decode"] = measure_decode(side, args.decode_batch, max(args.steps, 10),
                                          max(args.warmup, 3), dev, stream)
        # sampled over the whole measurement (setup and both arms): the decode
        # step is partly issue-bound, so its time follows the SM clock, which
        # the prefill workloads before it leave under the power cap
        result["decode"]["clocks_during_measurement"] = dec_sampler.stop()
    if not args.quick and world == 1 and not args.no_fp8 and side.d == 128:
        result["fp8"] = measure_fp8(side, max(args.steps, 5), max(args.warmup, 3), dev, stream)
    # the backward kernels are built for d = 128 (as the FP8 kernel)
    if not args.quick and world == 1 and not args.no_training and side.d == 128:
        result["training"] = measure_training(side, max(args.steps, 5), max(args.warmup, 3),
                                              dev, stream)
    return result


def run_sharded(args, rank, world, local_rank):
    """N > 1: ONE layer's prefill (per layer of the workload) head-sharded over
    the ranks: each rank pools its share of the (b, kv head) rows, one NCCL
    all-gather of the pooled slices feeds the router on every rank, the
    (b, kv group) groups are assigned by LPT on their cost under the mask (a
    group costlier than a rank's share split by query head),
    and each rank runs the fused attention on its groups.  Total work is
    fixed (strong scaling); the time is the slowest rank's."""
    from sparse_attention_head_b200 import flops
    from sparse_attention_head_b200.api import ea_get_device_status
    from sparse_attention_head_b200.shard import ShardedPrefill, head_costs, rank_loads
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    w = workloads.get(args.workload)
    if args.seq:
        w = dataclasses.replace(w, seq=args.seq)
    B, Hq, Hkv, N, d = w.batch, w.hq, w.hkv, w.seq, w.d
    stream = torch.cuda.current_stream(dev)
    # every rank holds the same layer (rank 0's seed): the shards split it
    layers = [make_layer(w, l, 0, dev) for l in range(w.layers)]
    sps = []
    for L in layers:
        r = L["router"] if L["router"] is not None else (None, None, None, None)
        sps.append(ShardedPrefill(B, Hq, Hkv, N, d, *r, w.sink, w.window, rank, world, dev,
                                  mask=L["mask"]))
    outs = [torch.empty_like(L["q"]) for L in layers]

    def step(ev=None):
        for li, (L, sp) in enumerate(zip(layers, sps)):
            if ev is not None:
                ev[li][0].record(stream)
            sp.route(L["k"], stream)
            sp.assign(stream)
            if ev is not None:
                ev[li][1].record(stream)
            sp.attend(L["q"], L["k"], L["v"], outs[li], stream)
            if ev is not None:
                ev[li][2].record(stream)

    for _ in range(max(args.warmup, 0)):
        step()
    torch.cuda.synchronize()
    K = args.steps
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in layers]
           for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(visible_gpu_index(local_rank)) if rank == 0 else None
    torch.distributed.barrier()
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
        time.sleep(0.3)
    t0.record(stream)
    for i in range(K):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize()
    torch.distributed.barrier()
    clocks = sampler.stop() if sampler else None
    total_ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    for sp in sps:
        if ea_get_device_status(sp.attn_ws) != 0:
            raise RuntimeError("device status word reports an error")
    masks = [sp.mask.cpu().numpy() for sp in sps]
    eff = sum(flops.effective_flops(m, N, d, w.sink, w.window) for m in masks)
    sparse_frac = float(np.mean([m.mean() for m in masks]))
    # this rank's share of the work, and its attention launches' time
    mine = 0.0
    for m, sp in zip(masks, sps):
        sel = sp.owner == rank          # [B, Hq]
        for b in range(B):
            for h in range(Hq):
                if sel[b, h]:
                    mine += flops.effective_flops(m[b, h:h + 1], N, d, w.sink, w.window)
    attn_ms = statistics.mean(evs[i][l][1].elapsed_time(evs[i][l][2]) for i in range(K)
                              for l in range(w.layers))
    route_ms = statistics.mean(evs[i][l][0].elapsed_time(evs[i][l][1]) for i in range(K)
                               for l in range(w.layers))
    ms_per_step = total_ms / K
    value = eff / (ms_per_step * 1e-3) / 1e12
    peak, peak_kind, burst, peak_src = roofline_peak(total_ms)
    achieved = (mine / w.layers) / (attn_ms * 1e-3) / 1e12
    loads = rank_loads(head_costs(masks[0], N, w.sink, w.window), sps[0].owner, world)
    result = {
        "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
        "steps": K, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": bench_config(w, sparse_frac, world),
        "tokens_per_s": round(B * N / (ms_per_step * 1e-3), 1),
        "pct_of_bf16_peak": round(100.0 * value / world / peak, 2),
        "route_ms_rank0": round(route_ms, 4),
        "attn_ms_rank0": round(attn_ms, 4),
        "lpt_tile_loads_layer0": loads,
        # per layer: pool rows + reduce (2), MLP (2), attention (1)
        "gpu_launches": K * w.layers * (5 if layers[0]["router"] is not None else 1),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "peak_source": f"{peak_src} bf16_tflops ({peak_kind})",
                     "frac_of_burst_peak": round(achieved / burst, 4),
                     "scope": "rank 0's fused attention launch on its groups",
                     "traffic": None, "kernel": "ea_hybrid_attn_kernel<128>"},
        "clocks": clocks,
    }
    if not args.quick:
        # end to end from pinned host buffers: each rank uploads the keys of
        # its pooling rows and the q, k, v of its groups, downloads its heads
        L, sp = layers[0], sps[0]
        qh, kh, vh = (L[n].cpu().pin_memory() for n in ("q", "k", "v"))
        oh = torch.empty_like(qh).pin_memory()
        for _ in range(2):
            sp.host_step(qh, kh, vh, oh, L["q"], L["k"], L["v"], outs[0], stream)
        torch.cuda.synchronize()
        torch.distributed.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ek = args.e2e_steps or K
        up = down = 0
        a.record(stream)
        for _ in range(ek):
            up, down = sp.host_step(qh, kh, vh, oh, L["q"], L["k"], L["v"], outs[0], stream)
        b.record(stream)
        torch.cuda.synchronize()
        torch.distributed.barrier()
        e2e_ms = max_over_ranks(a.elapsed_time(b) / ek, world, dev)
        tot = torch.tensor([up, down], dtype=torch.float64, device=dev)
        torch.distributed.all_reduce(tot)
        eff0 = flops.effective_flops(masks[0], N, d, w.sink, w.window)
        result["e2e"] = {"value": round(eff0 / (e2e_ms * 1e-3) / 1e12, 2), "unit": UNIT,
                         "h2d_bytes_per_step": int(tot[0].item()),
                         "d2h_bytes_per_step": int(tot[1].item()),
                         "ms_per_step": round(e2e_ms, 4),
                         "path": "ShardedPrefill.host_step: pooling rows' keys up, router "
                                 "all-gather, LPT groups' q/k/v up, fused attention, own heads "
                                 "down (layer 0)"}
    return result


def measure_workload(w: workloads.Workload, dev, stream, steps: int = 5, warmup: int = 3):
    """One more configuration's step (router, when it has one, then the fused
    attention, every layer), timed as the headline is (CUDA events per launch;
    inputs under 2x L2 get a 256 MiB flush between steps), with the attention
    kernel's own roofline."""
    from sparse_attention_head_b200 import flops
    from sparse_attention_head_b200.api import (attn_workspace, ea_get_device_status,
                                                ea_hybrid_attn_prefill, ea_router_decide,
                                                ea_router_workspace_size, make_params)
    B, Hq, Hkv, N, d = w.batch, w.hq, w.hkv, w.seq, w.d
    layers = [make_layer(w, l, 0, dev) for l in range(w.layers)]
    aws = attn_workspace(make_params(B, Hq, Hkv, N, d, w.sink, w.window), dev)
    rws = torch.empty(max(ea_router_workspace_size(B, Hkv, N, d), 16), dtype=torch.uint8,
                      device=dev)
    outs = [torch.empty_like(L["q"]) for L in layers]
    masks = [torch.empty((B, Hq), dtype=torch.uint8, device=dev) if L["router"] is not None
             else L["mask"] for L in layers]
    in_bytes = w.layers * B * (Hq + 2 * Hkv) * N * d * 2
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if in_bytes < 2 * L2_BYTES \
        else None
    ev = [[[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in layers]
          for _ in range(steps)]

    def step(e=None):
        for li, L in enumerate(layers):
            if e is not None:
                e[li][0].record(stream)
            if L["router"] is not None:
                ea_router_decide(L["k"], *L["router"], workspace=rws, route_mask=masks[li],
                                 want_logits=False)
            if e is not None:
                e[li][1].record(stream)
            ea_hybrid_attn_prefill(L["q"], L["k"], L["v"], masks[li], w.sink, w.window,
                                   out=outs[li], workspace=aws)
            if e is not None:
                e[li][2].record(stream)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    for i in range(steps):
        if flush is not None:
            flush.fill_(i & 0xff)
        step(ev[i])
    torch.cuda.synchronize()
    if ea_get_device_status(aws) != 0:
        raise RuntimeError(f"{w.name}: device status word reports an error")
    step_ms = [ev[i][0][0].elapsed_time(ev[i][-1][2]) for i in range(steps)]
    attn_ms = [ev[i][l][1].elapsed_time(ev[i][l][2]) for i in range(steps)
               for l in range(w.layers)]
    router_ms = [ev[i][l][0].elapsed_time(ev[i][l][1]) for i in range(steps)
                 for l in range(w.layers)]
    mask_host = [m.cpu().numpy() for m in masks]
    eff = sum(flops.effective_flops(m, N, d, w.sink, w.window) for m in mask_host)
    sparse_frac = float(np.mean([m.mean() for m in mask_host]))
    ms = statistics.mean(step_ms)
    attn_avg = statistics.mean(attn_ms)
    achieved = (eff / w.layers) / (attn_avg * 1e-3) / 1e12
    peak, kind, burst, src = roofline_peak(sum(step_ms))
    return {
        "config": bench_config(w, sparse_frac, 1),
        "steps": steps, "warmup": warmup,
        "ms_per_step": round(ms, 4),
        "effective_tflops": round(eff / (ms * 1e-3) / 1e12, 2),
        "tokens_per_s": round(B * N / (ms * 1e-3), 1),
        "attn_ms_per_layer": round(attn_avg, 4),
        "router_ms_per_layer": round(statistics.mean(router_ms), 4),
        "gpu_launches_per_step": w.layers * (5 if layers[0]["router"] is not None else 1),
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "peak_source": f"{src} bf16_tflops ({kind})",
                     "frac_of_burst_peak": round(achieved / burst, 4),
                     "traffic": traffic_for_current_kernel(w.name, N),
                     "kernel": "ea_hybrid_attn_kernel<128>"},
    }


# ---------------------------------------------------------------- FP8 variant
def measure_fp8(w: workloads.Workload, steps: int, warmup: int, dev, stream):
    """The FP8 (e4m3) variant of the fused attention on the same layer: Q, K, V
    quantized per head once (the quantization timed on its own), then the
    attention timed with CUDA events on resident e4m3 inputs; the bf16 kernel
    on the same layer and mask beside it."""
    from sparse_attention_head_b200 import flops
    from sparse_attention_head_b200.api import (ea_get_device_status, ea_hybrid_attn_prefill,
                                                ea_hybrid_attn_prefill_fp8, ea_quantize_fp8)
    B, Hq, Hkv, N, d, S, W = w.batch, w.hq, w.hkv, w.seq, w.d, w.sink, w.window
    seed = workloads.layer_seed(w, 0)
    q, k, v = workloads.make_qkv(w, seed, device=dev)
    heads = workloads.sparse_head_set(Hq, workloads.layer_sparse_frac(w, 0), seed)
    mask_h = np.zeros((B, Hq), np.uint8)
    mask_h[:, heads] = 1
    mask = torch.as_tensor(mask_h, device=dev)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    out = torch.empty_like(q)
    qw = torch.empty(1 << 16, dtype=torch.uint8, device=dev)

    def quant():
        a = ea_quantize_fp8(q, workspace=qw, stream=stream)
        b = ea_quantize_fp8(k, workspace=qw, stream=stream)
        c = ea_quantize_fp8(v, transpose=True, workspace=qw, stream=stream)
        return a, b, c

    def timed(fn, n):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    with torch.cuda.stream(stream):
        (q8, qs), (k8, ks), (vt8, vs) = quant()

        def fp8():
            ea_hybrid_attn_prefill_fp8(q8, k8, vt8, qs, ks, vs, mask, S, W, out=out,
                                       workspace=ws, stream=stream)

        def bf16():
            ea_hybrid_attn_prefill(q, k, v, mask, S, W, out=out, workspace=ws, stream=stream)

        for _ in range(warmup):
            quant()
            fp8()
            bf16()
        torch.cuda.synchronize()
        q_ms = timed(quant, steps)
        f_ms = timed(fp8, steps)
        b_ms = timed(bf16, steps)
    if ea_get_device_status(ws) != 0:
        raise RuntimeError("attention status word reports an error")
    eff = flops.effective_flops(mask_h, N, d, S, W)
    peaks, src = load_peaks()
    peak8 = 2.0 * float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    tf = eff / (f_ms * 1e-3) / 1e12
    # quantization bytes: bf16 read twice (amax, then convert), e4m3 written once
    nval = (B * Hq + 2 * B * Hkv) * N * d
    qbytes = nval * (2 + 2 + 1)
    return {
        "workload": f"{w.name} FP8 (e4m3 Q/K/V, per-head scales) prefill: B={B} Hq={Hq} "
                    f"Hkv={Hkv} N={N} d={d} S={S} W={W}, SA heads {mask_h.mean():.2f}",
        "steps": steps, "warmup": warmup,
        "ms_per_step": round(f_ms, 4),
        "effective_tflops": round(tf, 2),
        "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": round(peak8, 1),
                     "unit": "TFLOP/s", "frac": round(tf / peak8, 4),
                     "peak_source": f"{src} bf16_tflops (burst) x 2, the nominal e4m3/bf16 "
                                    "dense ratio",
                     "scope": "fused FP8 attention kernel, effective flops"},
        "bf16_ms_per_step": round(b_ms, 4),
        "speedup_vs_bf16": round(b_ms / f_ms, 3),
        "quantize_ms": round(q_ms, 4),
        "quantize_gbs": round(qbytes / (q_ms * 1e-3) / 1e9, 1),
        "quantize_hbm_frac": round(qbytes / (q_ms * 1e-3) / 1e9 / hbm, 4),
        "gpu_launches_per_step": 1,
        "l2": (f"e4m3 inputs {(B * Hq + 2 * B * Hkv) * N * d / 1e6:.0f} MB "
               + ("exceed L2 (126 MB), no flush" if (B * Hq + 2 * B * Hkv) * N * d > 126e6
                  else "fit in L2 (126 MB): timed warm")),
    }


# ---------------------------------------------------------------- packed batches
def measure_packed(w: workloads.Workload, nseq: int, steps: int, warmup: int, dev, stream):
    """A ragged prefill batch (lengths uniform in [seq/8, seq]) packed token-
    major: router over each sequence's keys, then the fused attention, timed
    with CUDA events; then the same batch padded to its longest sequence
    through the padded entry points (the work a padded layout executes)."""
    from sparse_attention_head_b200 import flops
    from sparse_attention_head_b200.api import (ea_get_device_status, ea_hybrid_attn_prefill,
                                                ea_hybrid_attn_prefill_varlen, ea_router_decide,
                                                ea_router_decide_varlen)
    Hq, Hkv, d, S, W = w.hq, w.hkv, w.d, w.sink, w.window
    seed = workloads.layer_seed(w, 0) + 7000
    lens = workloads.packed_lengths(w, nseq, seed)
    cu_host = np.cumsum([0] + lens).astype(np.int32)
    T, Lmax = int(cu_host[-1]), int(max(lens))
    g = torch.Generator(device=dev)
    g.manual_seed(seed)

    def rand(*shape):
        return torch.randn(shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)

    q, k, v = rand(T, Hq, d), rand(T, Hkv, d), rand(T, Hkv, d)
    cu = torch.as_tensor(cu_host, device=dev)
    frac = workloads.layer_sparse_frac(w, 0)
    heads = workloads.sparse_head_set(Hq, frac, seed)
    w1, b1, w2, b2 = (t.to(dev) for t in workloads.make_router_weights(Hkv * d, w.router_hidden,
                                                                         Hq, heads, seed))
    out = torch.empty_like(q)
    ws = torch.zeros(256, dtype=torch.uint8, device=dev)
    mask = torch.empty((nseq, Hq), dtype=torch.uint8, device=dev)
    rws = torch.empty(1 << 24, dtype=torch.uint8, device=dev)

    def step():
        ea_router_decide_varlen(k, cu, Lmax, w1, b1, w2, b2, workspace=rws, route_mask=mask,
                                want_logits=False, stream=stream)
        ea_hybrid_attn_prefill_varlen(q, k, v, cu, mask, Lmax, S, W, out=out, workspace=ws,
                                      stream=stream)

    def timed(fn, n):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    ms = timed(step, steps)
    if ea_get_device_status(ws) != 0:
        raise RuntimeError("packed prefill status word reports an error")
    m = mask.cpu().numpy()
    eff = sum(flops.effective_flops(m[b:b + 1], lens[b], d, S, W) for b in range(nseq))
    # padded comparator: [nseq, H, Lmax, d] with zero rows past every length
    qp = torch.zeros((nseq, Hq, Lmax, d), dtype=torch.bfloat16, device=dev)
    kp = torch.zeros((nseq, Hkv, Lmax, d), dtype=torch.bfloat16, device=dev)
    vp = torch.zeros_like(kp)
    for b in range(nseq):
        t0, t1 = int(cu_host[b]), int(cu_host[b + 1])
        qp[b, :, :t1 - t0] = q[t0:t1].transpose(0, 1)
        kp[b, :, :t1 - t0] = k[t0:t1].transpose(0, 1)
        vp[b, :, :t1 - t0] = v[t0:t1].transpose(0, 1)
    outp = torch.empty_like(qp)
    maskp = torch.empty_like(mask)

    def padded_step():
        # the padded router pools zero rows too (its mask is only timed); the
        # attention runs the packed batch's routing, so both arms do the same
        # heads in the same modes
        ea_router_decide(kp, w1, b1, w2, b2, workspace=rws, route_mask=maskp, want_logits=False,
                         stream=stream)
        ea_hybrid_attn_prefill(qp, kp, vp, mask, S, W, out=outp, workspace=ws, stream=stream)

    for _ in range(2):
        padded_step()
    torch.cuda.synchronize()
    ms_pad = timed(padded_step, max(3, steps // 2))
    peaks, src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    tf = eff / (ms * 1e-3) / 1e12
    return {
        "workload": f"{w.name} packed prefill: {nseq} sequences, lengths {lens} "
                    f"(T={T}), Hq={Hq} Hkv={Hkv} d={d} S={S} W={W}, router-chosen mask "
                    f"(SA heads {m.mean():.2f})",
        "steps": steps, "warmup": warmup,
        "ms_per_step": round(ms, 4),
        "effective_tflops": round(tf, 2),
        "tokens_per_s": round(T / (ms * 1e-3), 1),
        "roofline": {"bound": "tensor", "achieved": round(tf, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(tf / peak, 4),
                     "peak_source": f"{src} bf16_tflops (burst)",
                     "scope": "router + fused attention on the packed batch, effective flops"},
        "gpu_launches_per_step": 5,
        "padded_ms_per_step": round(ms_pad, 4),
        "speedup_vs_padded": round(ms_pad / ms, 3),
    }


# ---------------------------------------------------------------- backward


def unit_trace(w: workloads.Workload, dev):
    """Layer 0's fused attention launch with the per-unit trace (after two
    untraced warm-up launches): how evenly the persistent CTAs finish, how
    busy they are, how much of the launch runs FA and SA units at the same
    time, and the time per KV tile of each mode."""
    from sparse_attention_head_b200.api import (attn_workspace, ea_hybrid_attn_prefill,
                                                ea_hybrid_attn_prefill_traced,
                                                ea_router_decide, make_params)
    L = make_layer(w, 0, 0, dev)
    B, Hq, Hkv, N, d = w.batch, w.hq, w.hkv, w.seq, w.d
    if L["router"] is not None:
        mask, _ = ea_router_decide(L["k"], *L["router"], want_logits=False)
    else:
        mask = L["mask"]
    ws = attn_workspace(make_params(B, Hq, Hkv, N, d, w.sink, w.window), dev)
    out = torch.empty_like(L["q"])
    for _ in range(2):
        ea_hybrid_attn_prefill(L["q"], L["k"], L["v"], mask, w.sink, w.window, out=out,
                               workspace=ws)
    torch.cuda.synchronize()
    _, rec, total = ea_hybrid_attn_prefill_traced(L["q"], L["k"], L["v"], mask, w.sink,
                                                  w.window, out=out, workspace=ws,
                                                  max_records=1 << 17)
    return {"workload": w.name, **summarize_unit_trace(rec, total)}


def summarize_unit_trace(rec: np.ndarray, total: int) -> dict:
    """Balance figures of one traced launch.  rec: int64 [n, 8] rows of
    (start, first S ready, last P handed over, end) in ns, CTA, rank, sparse,
    KV tiles, as ea_hybrid_attn_prefill_traced returns them; total: units
    the launch ran."""
    start, first_s, last_p, end = rec[:, 0], rec[:, 1], rec[:, 2], rec[:, 3]
    cta, sparse, tiles = rec[:, 4], rec[:, 6], rec[:, 7]
    t0 = start.min()
    span = float(end.max() - t0) / 1e3
    ctas = np.unique(cta)
    last_end = np.array([end[cta == c].max() for c in ctas], dtype=np.float64)
    busy = np.array([(end[cta == c] - start[cta == c]).sum() for c in ctas], dtype=np.float64)
    # time during which an FA unit and an SA unit are both in progress (an end
    # sorts before a start at the same instant: touching units do not overlap)
    ev = sorted([(int(a), 1, int(sp)) for a, sp in zip(start, sparse)] +
                [(int(b), -1, int(sp)) for b, sp in zip(end, sparse)])
    live = [0, 0]
    both, prev = 0, None
    for t, delta, sp in ev:
        if prev is not None and live[0] > 0 and live[1] > 0:
            both += t - prev
        live[sp] += delta
        prev = t
    per_tile = {}
    for sp, name in ((0, "fa"), (1, "sa")):
        sel = sparse == sp
        if sel.any():
            per_tile[name + "_us_per_tile"] = round(
                float((end[sel] - start[sel]).sum()) / 1e3 / float(tiles[sel].sum()), 3)
    return {
        "units": int(total), "ctas": int(len(ctas)),
        "fa_units": int((sparse == 0).sum()), "sa_units": int((sparse == 1).sum()),
        "span_us": round(span, 1),
        "cta_finish_us": {"min": round(float(last_end.min() - t0) / 1e3, 1),
                          "median": round(float(np.median(last_end) - t0) / 1e3, 1),
                          "max": round(float(last_end.max() - t0) / 1e3, 1)},
        "tail_us": round(float(last_end.max() - np.median(last_end)) / 1e3, 1),
        "busy_fraction": round(float(busy.sum()) / (len(ctas) * span * 1e3), 4),
        "fa_sa_concurrent_fraction": round(both / (span * 1e3), 4),
        **per_tile,
        # a unit's phases, as its first query slot sees them (mean, us): from
        # its start to its first score tile, from there to its last P, and
        # from its last P to its rows stored
        "unit_ramp_us": round(float((first_s - start).mean()) / 1e3, 3),
        "unit_body_us": round(float((last_p - first_s).mean()) / 1e3, 3),
        "unit_drain_us": round(float((end - last_p).mean()) / 1e3, 3),
        "unit_tiles_mean": round(float(tiles.mean()), 2),
    }


def _union_ms(intervals):
    """Total length of a union of (start, end) intervals (microseconds in,
    milliseconds out)."""
    total, cur_s, cur_e = 0.0, None, None
    for a, b in sorted(intervals):
        if cur_e is None or a > cur_e:
            if cur_e is not None:
                total += cur_e - cur_s
            cur_s, cur_e = a, b
        else:
            cur_e = max(cur_e, b)
    if cur_e is not None:
        total += cur_e - cur_s
    return total / 1000.0


def host_timeline(w: workloads.Workload, dev):
    """One call of the host-buffer path (after two warm-up calls) under the
    torch profiler, whose CUDA activity records give every copy and kernel
    its device start and end: the span of the call, the busy time of the
    uploads, the downloads and our kernels, and how much of the kernels' and
    the downloads' time overlaps the uploads."""
    from torch.profiler import ProfilerActivity, profile
    from sparse_attention_head_b200.api import HostPrefill
    L = make_layer(w, 0, 0, dev)
    B, Hq, Hkv, N, d = w.batch, w.hq, w.hkv, w.seq, w.d
    router = L["router"] if L["router"] is not None else (None, None, None, None)
    hp = HostPrefill(B, Hq, Hkv, N, d, *router, w.sink, w.window, device=dev)
    qh, kh, vh = (L[x].cpu().pin_memory() for x in ("q", "k", "v"))
    mh = None if L["router"] is not None else L["mask"].cpu().pin_memory()
    for _ in range(2):
        hp(qh, kh, vh, mh)
    torch.cuda.synchronize()
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        hp(qh, kh, vh, mh)
        torch.cuda.synchronize()
    h2d, d2h, kern = [], [], []
    for e in prof.events():
        if e.device_type.name != "CUDA":
            continue
        iv = (e.time_range.start, e.time_range.end)
        name = e.name.lower()
        if "memcpy" in name and "htod" in name:
            h2d.append(iv)
        elif "memcpy" in name and "dtoh" in name:
            d2h.append(iv)
        elif name.startswith("ea::") or "ea::" in name:
            kern.append(iv)
    every = h2d + d2h + kern
    span = (max(b for _, b in every) - min(a for a, _ in every)) / 1000.0 if every else 0.0
    up = _union_ms(h2d)
    return {
        "workload": w.name, "chunks": hp.chunks,
        "span_ms": round(span, 3),
        "h2d_busy_ms": round(up, 3), "d2h_busy_ms": round(_union_ms(d2h), 3),
        "kernel_busy_ms": round(_union_ms(kern), 3),
        "kernel_overlapping_h2d_ms": round(_union_ms(kern) + up - _union_ms(kern + h2d), 3),
        "d2h_overlapping_h2d_ms": round(_union_ms(d2h) + up - _union_ms(d2h + h2d), 3),
        "copies": {"h2d": len(h2d), "d2h": len(d2h)}, "kernels": len(kern),
        "h2d_bytes": hp.h2d_bytes(), "d2h_bytes": hp.d2h_bytes(),
    }


def measure_training(w: workloads.Workload, steps: int, warmup: int, dev, stream):
    """One layer's attention training step, every phase timed with CUDA events:
    the Gumbel-Softmax router decision, the forward of both modes in one
    launch (the straight-through router gradient needs both outputs), the
    attention backward of each head's chosen mode (D, dK/dV, dQ), and the
    router's straight-through gradients (added into dK).  Work: the forward's
    effective flops of both modes, 2.5x the chosen mode's for the backward
    (five products of the forward's size against its two)."""
    from sparse_attention_head_b200 import flops
    from sparse_attention_head_b200.api import (ea_get_device_status, ea_hybrid_attn_backward,
                                                ea_hybrid_attn_prefill_lse,
                                                ea_hybrid_attn_prefill_train,
                                                ea_router_decide_gumbel, ea_router_ste_backward)
    B, Hq, Hkv, N, d, S, W = w.batch, w.hq, w.hkv, w.seq, w.d, w.sink, w.window
    seed = workloads.layer_seed(w, 0) + 9000
    q, k, v = workloads.make_qkv(w, seed, device=dev)
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    dout = torch.randn(q.shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    frac = workloads.layer_sparse_frac(w, 0)
    heads = workloads.sparse_head_set(Hq, frac, seed)
    w1, b1, w2, b2 = (t.to(dev) for t in workloads.make_router_weights(
        Hkv * d, w.router_hidden, Hq, heads, seed))
    g0, g1 = workloads.gumbel_noise(B, Hq, seed, device=dev)
    tau = 1.0
    ws = torch.zeros(1 << 26, dtype=torch.uint8, device=dev)
    rws = torch.empty(1 << 26, dtype=torch.uint8, device=dev)
    out, other = torch.empty_like(q), torch.empty_like(q)
    lse = torch.empty((B, Hq, N), dtype=torch.float32, device=dev)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    mask = torch.empty((B, Hq), dtype=torch.uint8, device=dev)

    r_soft = torch.empty((B, Hq), dtype=torch.float32, device=dev)
    logits = torch.empty((B, Hq), dtype=torch.float32, device=dev)

    def router():
        ea_router_decide_gumbel(k, w1, b1, w2, b2, g0, g1, tau, route_mask=mask, r_soft=r_soft,
                                logits=logits, workspace=rws, stream=stream)

    def fwd():
        ea_hybrid_attn_prefill_train(q, k, v, mask, S, W, out=out, lse=lse, out_other=other,
                                     workspace=ws[:256], stream=stream)

    def fwd_chosen_only():
        ea_hybrid_attn_prefill_lse(q, k, v, mask, S, W, out=out, lse=lse, workspace=ws[:256],
                                   stream=stream)

    def bwd():
        ea_hybrid_attn_backward(q, k, v, out, dout, lse, mask, S, W, dq=dq, dk=dk, dv=dv,
                                workspace=ws, stream=stream)

    def ste():
        ea_router_ste_backward(k, w1, b1, w2, b2, g0, g1, tau, dout, out, other, mask,
                               dk_accum=dk, workspace=rws, stream=stream)

    def step():
        router()
        fwd()
        bwd()
        ste()

    def timed(fn, n):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(n):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / n

    with torch.cuda.stream(stream):
        for _ in range(warmup):
            step()
        torch.cuda.synchronize()
        r_ms = timed(router, steps)
        f_ms = timed(fwd, steps)
        f1_ms = timed(fwd_chosen_only, steps)
        fwd()
        b_ms = timed(bwd, steps)
        s_ms = timed(ste, steps)
        t_ms = timed(step, steps)
    if ea_get_device_status(ws) != 0 or ea_get_device_status(ws[:256]) != 0:
        raise RuntimeError("a training kernel's status word reports an error")
    hm = mask.cpu().numpy()
    eff = flops.effective_flops(hm, N, d, S, W)
    eff_both = (flops.effective_flops(np.zeros_like(hm), N, d, S, W) +
                flops.effective_flops(np.ones_like(hm), N, d, S, W))
    peaks, src = load_peaks()
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    btf = 2.5 * eff / (b_ms * 1e-3) / 1e12
    # router STE bytes: dO, out, out_other once (the dr reduction), K once
    # (the forward recompute), dK read and written (the in-place add)
    ste_bytes = 2 * (3 * B * Hq * N * d + B * Hkv * N * d + 2 * B * Hkv * N * d)
    return {
        "workload": f"{w.name} training step of one layer: B={B} Hq={Hq} Hkv={Hkv} N={N} d={d} "
                    f"S={S} W={W}, Gumbel routes with tau={tau}: SA heads {hm.mean():.2f}",
        "steps": steps, "warmup": warmup,
        "step_ms": round(t_ms, 4),
        "router_gumbel_ms": round(r_ms, 4),
        "forward_both_modes_ms": round(f_ms, 4),
        "forward_both_modes_tflops": round(eff_both / (f_ms * 1e-3) / 1e12, 2),
        "forward_chosen_mode_only_ms": round(f1_ms, 4),
        "backward_ms": round(b_ms, 4),
        "backward_tflops": round(btf, 2),
        "router_ste_ms": round(s_ms, 4),
        "router_ste_gbs": round(ste_bytes / (s_ms * 1e-3) / 1e9, 1),
        "router_ste_hbm_frac": round(ste_bytes / (s_ms * 1e-3) / 1e9 / hbm, 4),
        "roofline": {"bound": "tensor", "achieved": round(btf, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(btf / peak, 4),
                     "peak_source": f"{src} bf16_tflops (burst)",
                     "scope": "attention backward (rowdot + schedule + dK/dV + dQ kernels), 2.5x the "
                              "chosen mode's effective forward flops"},
        # router 4 + Gumbel 1; forward 1; backward 4 (rowdot, schedule, dK/dV, dQ); STE: recompute 4 + 7
        "gpu_launches_per_step": 5 + 1 + 4 + 11,
    }


# ---------------------------------------------------------------- decode
DECODE_WARMUP_S = 0.5


def measure_decode(w: workloads.Workload, batch: int, steps: int, warmup: int, dev, stream):
    """One decode step per sequence of a ragged serving batch (positions in
    [seq/2, seq)), caches under the per-head policy, timed with CUDA events;
    then the same step with every head FA (every kv head on a full cache)."""
    from sparse_attention_head_b200 import flops
    from sparse_attention_head_b200.api import (decode_workspace, ea_decode_kv_policy,
                                                ea_get_device_status, ea_hybrid_attn_decode,
                                                make_decode_params)
    B, Hq, Hkv, d, S, W = batch, w.hq, w.hkv, w.d, w.sink, w.window
    seed = workloads.layer_seed(w, 0) + 5000
    frac = workloads.layer_sparse_frac(w, 0)
    mask = workloads.make_fixed_mask(dataclasses.replace(w, batch=B, sparse_frac=frac,
                                                         layers=1), seed)
    pos0 = workloads.decode_positions(w, B, seed)
    max_len = int(pos0.max()) + steps + warmup + 1
    g = torch.Generator(device=dev)
    g.manual_seed(seed)

    def rand(*shape):
        return torch.randn(shape, generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)

    def setup(m):
        slots, n_full, n_sa = ea_decode_kv_policy(m, Hkv)
        kf = rand(n_full, max_len, d) if n_full else None
        vf = rand(n_full, max_len, d) if n_full else None
        ks = rand(n_sa, S + W, d) if n_sa else None
        vs = rand(n_sa, S + W, d) if n_sa else None
        return slots, n_full, n_sa, (kf, vf, ks, vs)

    q = rand(B, Hq, d)
    kn = rand(B, Hkv, d)
    vn = rand(B, Hkv, d)
    # positions of step i: pos0 + i (each step appends one token per sequence)
    pos_steps = [(pos0 + i).to(dev) for i in range(warmup + steps)]
    out = torch.empty_like(q)

    def run(m):
        slots_np, n_full, n_sa, caches = setup(m)
        slots = torch.as_tensor(slots_np, device=dev)
        m_dev = m.to(dev)
        ws = decode_workspace(make_decode_params(B, Hq, Hkv, d, S, W, max_len, n_full, n_sa),
                              dev)
        cache_bytes = sum(c.numel() * 2 for c in caches if c is not None)

        def step(i):
            ea_hybrid_attn_decode(q, kn, vn, pos_steps[i], m_dev, slots, *caches, S, W,
                                  max_len, out=out, workspace=ws, stream=stream)
        # warm-up: the W steps, then the last of them again (it rewrites the
        # same cache rows) until DECODE_WARMUP_S of steps have run, so the
        # timed steps start from steady clocks: right after a prefill
        # measurement the GPU is still coming out of its power cap, and a
        # step took 286 us there against 235 us half a second later
        t_end = time.perf_counter() + DECODE_WARMUP_S
        n = 0
        while n < warmup or time.perf_counter() < t_end:
            step(min(n, warmup - 1))
            n += 1
            if n % 32 == 0:
                torch.cuda.synchronize()
        torch.cuda.synchronize()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for i in range(steps):
            step(warmup + i)
        b.record(stream)
        torch.cuda.synchronize()
        if ea_get_device_status(ws) != 0:
            raise RuntimeError("decode status word reports an error")
        ms = a.elapsed_time(b) / steps
        mid = (pos0 + warmup + (steps - 1) // 2).numpy()
        byts = flops.decode_bytes(m.numpy(), mid, Hkv, d, S, W)
        del caches
        return ms, byts, cache_bytes

    ms, byts, cache_bytes = run(mask)
    full_mask = torch.zeros_like(mask)
    ms_full, byts_full, cache_full = run(full_mask)
    peaks, src = load_peaks()
    peak = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    gbs = byts["total"] / (ms * 1e-3) / 1e9
    return {
        "workload": f"{w.name} decode: B={B} Hq={Hq} Hkv={Hkv} d={d} S={S} W={W}, positions "
                    f"ragged in [{w.seq // 2}, {w.seq}) + step, SA heads {mask.float().mean():.2f},"
                    f" all-SA kv groups {byts['n_sa_groups']}/{byts['n_groups']}",
        "steps": steps, "warmup": warmup,
        "warmup_rule": f"{warmup} steps, then the last one repeated until {DECODE_WARMUP_S} s "
                       "of steps have run",
        "us_per_step": round(ms * 1e3, 2),
        "tokens_per_s": round(B / (ms * 1e-3), 1),
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs / peak, 4), "peak_source": f"{src} hbm_gbs",
                     "bytes_per_step": byts["total"],
                     "scope": "whole step (append kernel + split-K attention kernel with fused combine) over its "
                              "algorithmic bytes"},
        "gpu_launches_per_step": 2,
        "all_fa_us_per_step": round(ms_full * 1e3, 2),
        "all_fa_gbs": round(byts_full["total"] / (ms_full * 1e-3) / 1e9, 1),
        "speedup_vs_all_fa": round(ms_full / ms, 3),
        "cache_bytes": cache_bytes,
        "all_fa_cache_bytes": cache_full,
        "cache_saved_frac": round(1.0 - cache_bytes / cache_full, 4),
        "l2": "per-step bytes exceed L2" if byts["total"] > 126e6 else "per-step bytes fit L2",
    }


# ---------------------------------------------------------------- oracle arm
def oracle_sample(w, L_cpu, mask_np, target_s, rng):
    """Time the oracle on a bounded sample: the full router (when the workload
    has one) and sampled query rows of every head.  Returns (flops, seconds,
    description)."""
    import oracle
    q, k, v = L_cpu["q"], L_cpu["k"], L_cpu["v"]
    N, d = w.seq, w.d
    t_start = time.perf_counter()
    if L_cpu.get("router") is not None:
        w1, b1, w2, b2 = L_cpu["router"]
        oracle.router_decide(k, w1, b1, w2, b2)
    t_router = time.perf_counter() - t_start
    fl = 0.0
    rows_done = 0
    heads = [(b, h) for b in range(w.batch) for h in range(w.hq)]
    t_att = 0.0
    while t_att < max(0.5, target_s - t_router):
        b, h = heads[rows_done % len(heads)]
        rows = rng.integers(0, N, size=4)
        t0 = time.perf_counter()
        oracle.attention_rows(q, k, v, mask_np, b, h, rows, w.sink, w.window)
        t_att += time.perf_counter() - t0
        sparse = bool(mask_np[b, h])
        for i in rows:
            fl += 4.0 * d * len(oracle.visible_keys(int(i), sparse, w.sink, w.window))
        rows_done += 1
    desc = (f"oracle router on the full key tensor plus {4 * rows_done} sampled query rows "
            f"over all heads")
    return fl, t_router + t_att, desc


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count()


def host_layer(L):
    """float64 host copies of one layer's inputs for the oracle."""
    out = {"q": L["q"].float().cpu().double().numpy(), "k": L["k"].float().cpu().double().numpy(),
           "v": L["v"].float().cpu().double().numpy(), "router": None}
    if L["router"] is not None:
        out["router"] = tuple(t.cpu().double().numpy() for t in L["router"])
    return out


def cpu_baseline(w, L, mask_np, target_s):
    Lc = host_layer(L)
    fl, secs, desc = oracle_sample(w, Lc, mask_np, target_s, np.random.default_rng(5))
    return {"value": round(fl / secs / 1e12, 6), "unit": UNIT, "cores": blas_threads(),
            "kind": "oracle", "sample": desc + f"; {secs:.1f} s of CPU time"}


def run_reference(args):
    w = workloads.get(args.workload)
    if args.seq:
        w = dataclasses.replace(w, seq=args.seq)
    L = make_layer(w, 0, 0, "cpu")
    if L["router"] is not None:
        import oracle
        Lc = host_layer(L)
        mask_np, _ = oracle.router_decide(Lc["k"], *Lc["router"])
    else:
        Lc = host_layer(L)
        mask_np = L["mask"].numpy()
    rng = np.random.default_rng(11)
    # each step is a bounded sample; the whole run stays within about two minutes
    per_step = max(0.5, min(args.cpu_seconds, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, Lc, mask_np, per_step * 0.25, rng)
    tot_fl, tot_s = 0.0, 0.0
    desc = ""
    for _ in range(args.steps):
        fl, s, desc = oracle_sample(w, Lc, mask_np, per_step, rng)
        tot_fl += fl
        tot_s += s
    value = tot_fl / tot_s / 1e12
    sparse_frac = float(mask_np.mean())
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * tot_s / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        # the same config dict as our arm's line (the oracle's host cores are
        # described in cpu_baseline)
        "config": bench_config(w, sparse_frac, args.gpus),
        "cpu_baseline": {"value": round(value, 6), "unit": UNIT, "cores": blas_threads(),
                         "kind": "oracle", "sample": desc + " per step"},
        "e2e": {"value": round(value, 6), "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank != 0:
            return 0
        print(json.dumps(run_reference(args)), flush=True)
        return 0
    if args.fp8_only:
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        w = workloads.get(args.workload)
        if args.seq:
            w = dataclasses.replace(w, seq=args.seq)
        res = measure_fp8(w, args.steps, max(args.warmup, 3), dev, torch.cuda.current_stream(dev))
        if rank == 0:
            print(json.dumps(res), flush=True)
        return 0
    if args.training_only:
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        w = workloads.get(args.workload)
        if args.seq:
            w = dataclasses.replace(w, seq=args.seq)
        res = measure_training(w, args.steps, max(args.warmup, 3), dev,
                               torch.cuda.current_stream(dev))
        if rank == 0:
            print(json.dumps(res), flush=True)
        return 0
    if args.unit_trace:
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        w = workloads.get(args.workload)
        if args.seq:
            w = dataclasses.replace(w, seq=args.seq)
        res = unit_trace(w, dev)
        if rank == 0:
            print(json.dumps(res), flush=True)
        return 0
    if args.host_timeline:
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        w = workloads.get(args.workload)
        if args.seq:
            w = dataclasses.replace(w, seq=args.seq)
        res = host_timeline(w, dev)
        if rank == 0:
            print(json.dumps(res), flush=True)
        return 0
    if args.packed_only:
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        w = workloads.get(args.workload)
        if args.seq:
            w = dataclasses.replace(w, seq=args.seq)
        res = measure_packed(w, max(args.packed_seqs, 1), args.steps, max(args.warmup, 3), dev,
                             torch.cuda.current_stream(dev))
        if rank == 0:
            print(json.dumps(res), flush=True)
        return 0
    if args.decode_only:
        dev = torch.device("cuda", local_rank)
        torch.cuda.set_device(dev)
        w = workloads.get(args.workload)
        if args.seq:
            w = dataclasses.replace(w, seq=args.seq)
        sampler = ClockSampler(visible_gpu_index(local_rank))
        sampler.start()
        res = measure_decode(w, max(args.decode_batch, 1), args.steps, max(args.warmup, 3), dev,
                             torch.cuda.current_stream(dev))
        res["clocks_during_measurement"] = sampler.stop()
        if rank == 0:
            print(json.dumps(res), flush=True)
        return 0
    if world > 1:
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group(
            "nccl", timeout=datetime.timedelta(seconds=180),
            device_id=torch.device("cuda", local_rank))
    try:
        res = run_sharded(args, rank, world, local_rank) if world > 1 else \
            run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
