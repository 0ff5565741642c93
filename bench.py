#!/usr/bin/env python
"""Benchmark of the MoE expert-MLP hot path on B200.

One step = one forward pass of the whole path on one batch of the Mixtral-8x7B-shaped
BF16 layer (T=8192 tokens, H=4096, F=14336, 8 experts, top-2): moe_route ->
moe_permute -> grouped_mlp_fwd (fc1 + ScaledSwiGLU, fc2) -> moe_unpermute.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-cpu-baseline]

Prints one JSON line (rank 0). With N > 1 (torchrun) every rank runs its own replica of
the workload on its own GPU with its own seed (data-parallel, no collective on the data
path); the step time is the max over ranks and `value` counts all ranks' work.
`--impl reference` times the fp64 CPU oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

DEFAULT_WORKLOAD = "mixtral_bf16_fwd"
METRIC = "grouped-MLP TFLOP/s & tokens/s (fwd, fwd+bwd) on 1 B200; % of tensor-core peak"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# --------------------------------------------------------------------- distributed
def dist_setup(want_gpus: int):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def max_over_ranks(x: float, world: int) -> float:
    """Maximum of a per-rank float over all ranks (identity with one rank)."""
    if world <= 1:
        return float(x)
    import torch.distributed as dist
    dev = torch.device("cuda") if dist.get_backend() == "nccl" else torch.device("cpu")
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def rank_seed(base: int, rank: int) -> int:
    """Each replica draws its own batch (and weights) from seed base + rank."""
    return base + rank


# --------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int, out_path: str | None = None):
        self.dev = device_index
        self.proc = None
        self.path = out_path or f"/tmp/moe_bench_clocks_{os.getpid()}.csv"

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.dev)], stdout=self.f, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None:
            return None
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), parts[5:9], parts[4]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[2]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in rows), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
KERNEL_SOURCES = ["ptx_sm100.cuh", "token_kernels.cuh", "grouped_gemm_sm100.cuh", "grouped_gemm_mxf8_sm100.cuh",
                  "grouped_gemm_pair_sm100.cuh", "grouped_gemm_mxf8_pair_sm100.cuh",
                  "grouped_gemm_kgroup_pair_sm100.cuh", "moe_api.cu"]


def kernel_sources_sha256() -> str:
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "mixture_experts_grouped_top_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(workload: str):
    """DRAM bytes (read + write) of one grouped_mlp_fwd launch pair from the committed ncu
    summary, or None when the kernels changed since it was captured."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    if t.get("kernel_sources_sha256") != kernel_sources_sha256():
        return None
    entry = t.get("workloads", {}).get(workload)
    return None if entry is None else entry.get("grouped_mlp_fwd_dram_bytes")


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------- our GPU arm
def run_ours(args, world, rank, local):
    import mixture_experts_grouped_top_b200 as mb

    cfg = workloads.CONFIGS[args.workload]
    if args.tokens:
        cfg = dataclasses.replace(cfg, name=f"{cfg.name}_T{args.tokens}", T=args.tokens)
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    d = workloads.make_layer_inputs(cfg, seed=rank_seed(cfg.seed, rank), with_grad=cfg.passes == "fwd+bwd")
    layer = mb.MoEExpertLayer(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k, cfg.precision,
                              training=cfg.passes == "fwd+bwd", device=dev)
    w1, w2 = d["w1"].to(dev), d["w2"].to(dev)
    layer.set_weights(w1, w2)
    x, logits = d["x"].to(dev), d["logits"].to(dev)
    if cfg.passes == "fwd+bwd" and cfg.precision == "mxfp8":
        layer.xp_bf16 = torch.empty((cfg.R, cfg.H), dtype=torch.bfloat16, device=dev)
    grad = d["grad_out"].to(dev) if "grad_out" in d else None
    stream = torch.cuda.current_stream(dev)
    prec = cfg.precision

    training = cfg.passes == "fwd+bwd"

    def step(ev=None):
        """One pass of the path; `ev` = 4 events bracketing the grouped-GEMM calls."""
        if training and prec == "mxfp8":
            layer.set_weights(w1, w2)   # a training step re-quantises the bf16 masters
        mb.moe_route(logits, cfg.k, True, idx=layer.idx, prob=layer.prob)
        mb.moe_permute(x, layer.idx, layer.prob, cfg.E, prec, out=layer.perm, workspace=layer.perm_ws)
        if ev is not None:
            ev[0].record(stream)
        mb.grouped_mlp_fwd(layer.perm["xp"], layer.perm["split_sizes"], layer.w1, layer.w2,
                           layer.perm["probs_perm"], prec, xp_scale=layer.perm.get("xp_scale"),
                           w1_scale=layer.w1_scale, w2_scale=layer.w2_scale, yp=layer.yp, saved=layer.saved,
                           workspace=layer.mlp_ws, F=cfg.F)
        if ev is not None:
            ev[1].record(stream)
        mb.moe_unpermute(layer.yp, layer.perm["row_map"], cfg.T, cfg.k, out=layer.out)
        if training:
            if layer._bwd is None:
                layer._alloc_bwd()
            b = layer._bwd
            mb.moe_permute_rows(grad, layer.perm["row_map"], cfg.k, out=b["dy_perm"])
            if ev is not None:
                ev[2].record(stream)
            if prec == "mxfp8":
                mb.moe_permute_rows(x, layer.perm["row_map"], cfg.k, out=layer.xp_bf16)
            xp_b = layer.perm["xp"] if prec == "bf16" else layer.xp_bf16
            mb.grouped_mlp_bwd(b["dy_perm"], layer.perm["split_sizes"], xp_b, w1, w2,
                               layer.perm["probs_perm"], layer.saved, prec, dxp=b["dxp"], dw1=b["dw1"], dw2=b["dw2"],
                               dprobs_perm=b["dprobs_perm"], workspace=b["ws"])
            if ev is not None:
                ev[3].record(stream)
            mb.moe_unpermute(b["dxp"], layer.perm["row_map"], cfg.T, cfg.k, out=b["dx"])
            mb.moe_gather_slots(b["dprobs_perm"], layer.perm["row_map"], out=b["dprob"].view(-1))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if mb.moe_device_status() != 0:
        raise RuntimeError("device error during warm-up")

    K = args.steps
    mlp_events = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world)
    torch.cuda.synchronize(dev)
    launches0 = mb.moe_launch_count()
    with ClockSampler(local, args.clocks_csv) as clocks:
        wall0 = time.perf_counter()
        t0.record(stream)
        for i in range(K):
            step(mlp_events[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
        wall = time.perf_counter() - wall0
    launches = mb.moe_launch_count() - launches0
    barrier(world)
    ms = t0.elapsed_time(t1) / K
    ms_max = max_over_ranks(ms, world)
    mlp_ms = statistics.mean(ev[0].elapsed_time(ev[1]) + (ev[2].elapsed_time(ev[3]) if training else 0.0)
                             for ev in mlp_events)
    if mb.moe_device_status() != 0:
        raise RuntimeError("device error during the timed region")

    flops = cfg.gemm_flops()
    value = world * flops / (ms_max * 1e-3) / 1e12
    tokens_s = world * cfg.T / (ms_max * 1e-3)

    # ------------------------------------------------ end to end through host buffers
    # every step: pinned host -> device copies of the step's inputs, the path, and a
    # device -> host read of its result (the layer output; with backward also dx), through
    # the package's HostPipeline (transfers overlapped with the neighbouring steps' compute)
    x_h = d["x"].pin_memory()
    lg_h = d["logits"].pin_memory()
    g_h = d["grad_out"].pin_memory() if training else None
    out_h = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16).pin_memory()
    dx_h = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16).pin_memory() if training else None
    pipe = mb.HostPipeline(layer)

    def e2e_step():
        if training and prec == "mxfp8":
            layer.set_weights(w1, w2)
        pipe.step(x_h, lg_h, out_h, g_h, dx_h)

    for _ in range(2):
        e2e_step()
    pipe.flush()
    torch.cuda.synchronize(dev)
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(K):
        e2e_step()
    pipe.flush()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(e0.elapsed_time(e1) / K, world)
    e2e_val = world * flops / (e2e_ms * 1e-3) / 1e12
    h2d = x.numel() * 2 + logits.numel() * 4 + (grad.numel() * 2 if training else 0)
    d2h = cfg.T * cfg.H * 2 * (2 if training else 1)

    peaks, peak_src = load_peaks()
    # a timed region of a second or more runs under the power cap: compare with the
    # sustained GEMM peak; a shorter one with the burst peak
    regime = "sustained" if wall >= 1.0 else "burst"
    key = "bf16_tflops_sustained" if regime == "sustained" else "bf16_tflops"
    peak = peaks.get(key, FALLBACK_PEAKS[key])
    peak_note = f"{peak_src} bf16 {regime}"
    if prec == "mxfp8":
        # no measured MXFP8 figure: the measured bf16 one times the nominal dense ratio 4.5/2.25
        peak = 2.0 * peak
        peak_note = f"{peak_src} bf16 {regime} x 2 (nominal MXFP8/BF16 dense ratio)"
    achieved = flops / (mlp_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": round(ms_max, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if prec == "bf16" else "mxfp8(e4m3+e8m0)",
        "data": "synthetic (seeded N(0,1) tokens and router logits, N(0,0.02) weights)",
        "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "F": cfg.F, "E": cfg.E, "k": cfg.k,
                   "precision": prec, "pass": cfg.passes, "tokens_per_step_per_gpu": cfg.T,
                   "gemm_flop_per_step_per_gpu": flops,
                   "l2": "inputs larger than L2: the expert weights (%.2f GB) are re-read every step"
                         % ((d["w1"].numel() + d["w2"].numel()) * 2 / 1e9),
                   "parallelism": f"dp{world} replicas" if world > 1 else "single GPU"},
        "tokens_per_s": round(tokens_s, 1),
        "e2e": {"value": round(e2e_val, 3), "unit": "TFLOP/s", "ms_per_step": round(e2e_ms, 4),
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": int(launches),
        "roofline": {"kernel": ("grouped_mlp_fwd + grouped_mlp_bwd (the six tcgen05 grouped GEMMs)" if training
                               else "grouped_mlp_fwd (fc1 gate|up + ScaledSwiGLU, fc2: two tcgen05 grouped GEMMs)"),
                     "bound": "tensor", "achieved": round(achieved, 2),
                     "peak": peak, "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
                     "peak_source": f"{peak_note} (timed region {wall:.2f} s)",
                     "traffic": None if training else measured_traffic(cfg.name),
                     "avg_launch_ms": round(mlp_ms, 4)},
    }
    cl = clocks.summary()
    line["clocks"] = cl
    return line, cfg, d


# ------------------------------------------------------------------ oracle (CPU) arm
def oracle_sample(cfg, d, n_tokens: int, seed: int = 1):
    """Time the oracle (as it stands) on n_tokens sampled tokens of the workload.
    Returns (seconds, tokens, gemm flops done, threads used)."""
    from oracle import moe as om
    toks = workloads.sample_tokens(cfg.T, n_tokens, seed=seed)
    t = time.perf_counter()
    idx, prob = om.route(d["logits"][toks], cfg.k)
    om.moe_forward_sampled(d["x"][toks], idx, prob, d["w1"], d["w2"], np.arange(toks.size), a_round="bf16")
    sec = time.perf_counter() - t
    flops = 6.0 * cfg.H * cfg.F * toks.size * cfg.k
    return sec, int(toks.size), flops, torch.get_num_threads()


def cpu_baseline_entry(cfg, d, n_tokens):
    sec, n, flops, threads = oracle_sample(cfg, d, n_tokens)
    return {"value": round(flops / sec / 1e12, 6), "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
            "sample": f"{n} of {cfg.T} tokens of {cfg.name} (fp64 numpy/BLAS, routing + per-expert MLP), "
                      f"{sec:.2f} s; host has {os.cpu_count()} cores",
            "tokens_per_s": round(n / sec, 3)}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    cfg = workloads.CONFIGS[args.workload]
    d = workloads.make_layer_inputs(cfg, with_grad=False)
    n_tok = args.reference_tokens
    for _ in range(args.warmup):
        oracle_sample(cfg, d, max(8, n_tok // 8))
    secs = []
    flops = 0.0
    for i in range(args.steps):
        sec, n, flops, threads = oracle_sample(cfg, d, n_tok, seed=100 + i)
        secs.append(sec)
    sec = sum(secs) / len(secs)
    value = flops / sec / 1e12
    step_ms = sec * 1e3 * cfg.T / n_tok
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(step_ms, 2), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "F": cfg.F, "E": cfg.E, "k": cfg.k,
                   "precision": cfg.precision, "pass": cfg.passes},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": torch.get_num_threads(),
                         "kind": "oracle",
                         "sample": f"{n_tok} of {cfg.T} tokens per step (fp64 oracle); ms_per_step "
                                   f"extrapolated to all {cfg.T} tokens"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads.CONFIGS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=0, help="override T (profiling runs on a smaller batch)")
    ap.add_argument("--cpu-baseline-tokens", type=int, default=256)
    ap.add_argument("--reference-tokens", type=int, default=64)
    ap.add_argument("--clocks-csv", default=None,
                    help="keep the raw nvidia-smi clock samples of the timed region in this file")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    if args.impl == "reference":
        # the oracle runs on rank 0's host cores only; no process group is needed
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if int(os.environ.get("RANK", "0")) == 0:
            print(json.dumps(run_reference(args, world, 0)), flush=True)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        line, cfg, d = run_ours(args, world, rank, local)
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            line["cpu_baseline"] = cpu_baseline_entry(cfg, d, args.cpu_baseline_tokens)
        elif rank == 0:
            line["cpu_baseline"] = None
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
