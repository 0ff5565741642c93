#!/usr/bin/env python
"""Benchmark of the MoE expert-MLP hot path on B200.

The headline step is one forward + backward pass of the whole path on one batch of the
genomic long-sequence Mixtral-shaped MXFP8 layer (T=32768 tokens, H=4096, F=14336,
8 experts, top-2, expert 0 favoured): weight quantisation of the bf16 masters ->
moe_route_permute (router + permutation) -> grouped_mlp_fwd (fc1 + ScaledSwiGLU, fc2) ->
moe_unpermute -> moe_permute_rows(grad) -> grouped_mlp_bwd -> moe_unpermute(dxp) +
moe_gather_slots -> moe_route_bwd (router logits' gradient).
The same line reports, under ``workloads``, the other single-GPU layers (Mixtral BF16
and MXFP8 forward, Qwen3-30B-A3B BF16 forward + backward) with their own roofline
fractions, and the bandwidth of the permute and combine kernels.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-workloads] [--no-cpu-baseline]
    python bench.py --measure-peaks     # library MXFP8 / BF16 GEMM peaks -> profiles/mxfp8_peak.json

Prints one JSON line (rank 0). With N > 1 (torchrun) every rank runs its own replica of
the workload on its own GPU with its own seed (data-parallel, no collective on the data
path); the step time is the max over ranks and `value` counts all ranks' work.
`--impl reference` times the fp64 CPU oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import dataclasses
import datetime
import gc
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

DEFAULT_WORKLOAD = "genomic_mixtral_mxfp8_fwdbwd"
SECONDARY_WORKLOADS = ["mixtral_bf16_fwd", "mixtral_mxfp8_fwd", "qwen3_30b_a3b_bf16_fwdbwd"]
FUSED_COMBINE_WORKLOADS = ["mixtral_bf16_fwd", "qwen3_30b_a3b_bf16_fwdbwd"]
CAPACITY_WORKLOADS = ["mixtral_bf16_fwd"]
METRIC = "grouped-MLP TFLOP/s & tokens/s (fwd, fwd+bwd) on 1 B200; % of tensor-core peak"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
MXFP8_PEAK_FILE = os.path.join(ROOT, "profiles", "mxfp8_peak.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SPEC_TFLOPS = {"bf16": 2250.0, "mxfp8": 4500.0}
SPEC_HBM_GBS = 8000.0


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
        self.path = out_path or f"/tmp/moe_bench_clocks_{os.getpid()}_{device_index}.csv"

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
                  "grouped_gemm_kgroup_pair_sm100.cuh", "grouped_gemm_mxf8_kgroup_pair_sm100.cuh", "moe_api.cu"]


def kernel_sources_sha256() -> str:
    """sha256 of the kernel sources without their comment-only and blank lines (a comment
    edit does not change what the counters measured; any code change does)."""
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "mixture_experts_grouped_top_b200", "csrc", name), "rb") as f:
            for line in f.read().decode().splitlines():
                t = line.strip()
                if t and not t.startswith("//"):
                    h.update(line.encode() + b"\n")
    return h.hexdigest()


def measured_traffic(workload: str):
    """DRAM bytes (read + write) per launch of the roofline's kernel set for this workload
    from the committed ncu summary, or None when the kernels changed since it was taken."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    if t.get("kernel_sources_sha256") != kernel_sources_sha256():
        return None
    entry = t.get("workloads", {}).get(workload)
    return None if entry is None else entry.get("dram_bytes_per_step")


def load_peaks():
    try:
        with open(PEAKS_FILE) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


def load_mxfp8_peak():
    try:
        with open(MXFP8_PEAK_FILE) as f:
            return json.load(f)
    except (OSError, ValueError):
        return None


def gemm_peak(prec: str, regime: str):
    """(peak TFLOP/s, source) of a dense GEMM of this precision in this regime ("burst"
    for a short timed region, "sustained" for one of a second or more under the cap)."""
    peaks, src = load_peaks()
    key = "bf16_tflops_sustained" if regime == "sustained" else "bf16_tflops"
    if prec == "bf16":
        return float(peaks.get(key, FALLBACK_PEAKS[key])), f"{src} bf16 {regime} (cuBLAS)"
    mx = load_mxfp8_peak()
    mkey = "mxfp8_tflops_sustained" if regime == "sustained" else "mxfp8_tflops"
    if mx is not None and mx.get(mkey):
        return float(mx[mkey]), (f"measured MXFP8 {regime}: library block-scaled GEMM "
                                 f"({mx.get('library', 'torch scaled_mm')}, {mx.get('shape', '')}) in "
                                 f"profiles/mxfp8_peak.json")
    # no measured MXFP8 figure: the bf16 one times the nominal dense ratio 4.5/2.25
    return 2.0 * float(peaks.get(key, FALLBACK_PEAKS[key])), f"nominal: {src} bf16 {regime} x 2"


# -------------------------------------------------------------- library GEMM peaks
def measure_gemm_peaks(dev, n: int = 8192, sustained_s: float = 4.0) -> dict:
    """Dense-GEMM peaks of the library (cuBLAS / cuBLASLt through torch) on this GPU:
    BF16 ``torch.mm`` and MXFP8 ``torch.nn.functional.scaled_mm`` with E8M0 scales per
    32 values along K (the block-scaled tcgen05 path), both n x n x n. Burst: 20
    back-to-back calls after warm-up; sustained: calls repeated for ``sustained_s``
    seconds (under the power cap). Clocks are sampled during the sustained loops."""
    import torch.nn.functional as Fn
    torch.manual_seed(0)
    a16 = torch.randn(n, n, device=dev, dtype=torch.bfloat16)
    b16 = torch.randn(n, n, device=dev, dtype=torch.bfloat16)
    a8 = a16.to(torch.float8_e4m3fn)
    b8 = b16.to(torch.float8_e4m3fn)
    # n rows (a multiple of 128) x n/32 scale columns (a multiple of 4): the swizzled
    # layout holds exactly n * n/32 scales; every scale is 2**0 (code 127)
    sa = torch.full((n * (n // 32),), 127, dtype=torch.uint8, device=dev).view(torch.float8_e8m0fnu)
    sb = torch.full((n * (n // 32),), 127, dtype=torch.uint8, device=dev).view(torch.float8_e8m0fnu)

    def mx():
        return Fn.scaled_mm(a8, b8.t(), sa, Fn.ScalingType.BlockWise1x32, sb, Fn.ScalingType.BlockWise1x32,
                            swizzle_a=Fn.SwizzleType.SWIZZLE_32_4_4, swizzle_b=Fn.SwizzleType.SWIZZLE_32_4_4,
                            output_dtype=torch.bfloat16)

    def bf():
        return a16 @ b16

    # the MXFP8 library result must be the plain product of the dequantised operands
    ref = (a8.float() @ b8.float().t())
    got = mx().float()
    rel = float((got - ref).abs().max() / ref.abs().max())
    if not rel < 1e-2:
        raise RuntimeError(f"library MXFP8 GEMM disagrees with the fp32 product (rel {rel:.3g})")
    del ref, got
    flop = 2.0 * n ** 3
    out = {"library": "torch.nn.functional.scaled_mm (BlockWise1x32 e8m0, SWIZZLE_32_4_4) / torch.mm bf16",
           "shape": f"{n}x{n}x{n}", "check_rel_err": rel, "device": torch.cuda.get_device_name(dev)}
    stream = torch.cuda.current_stream(dev)
    for name, fn in (("mxfp8", mx), ("bf16", bf)):
        for _ in range(5):
            fn()
        torch.cuda.synchronize(dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(20):
            fn()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        out[f"{name}_tflops"] = round(flop * 20 / (e0.elapsed_time(e1) * 1e-3) / 1e12, 1)
        # sustained: calls in batches of 50 until sustained_s of device time
        with ClockSampler(dev.index if dev.index is not None else 0) as cs:
            total_ms, calls = 0.0, 0
            while total_ms < sustained_s * 1e3:
                e0.record(stream)
                for _ in range(50):
                    fn()
                e1.record(stream)
                torch.cuda.synchronize(dev)
                total_ms += e0.elapsed_time(e1)
                calls += 50
        out[f"{name}_tflops_sustained"] = round(flop * calls / (total_ms * 1e-3) / 1e12, 1)
        out[f"{name}_sustained_clocks"] = cs.summary()
    return out


# ------------------------------------------------------------------- our GPU arm
def ev():
    return torch.cuda.Event(enable_timing=True)


def run_workload(cfg, args, world, rank, local, steps, warmup, with_e2e=True, fused_combine=False):
    """Time `steps` passes of the whole path on one workload. Returns the JSON fields.
    fused_combine: the combine runs inside fc2's epilogue (grouped_mlp_fwd_combine)."""
    import mixture_experts_grouped_top_b200 as mb

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    training = cfg.passes == "fwd+bwd"
    prec = cfg.precision
    d = workloads.make_layer_inputs(cfg, seed=rank_seed(cfg.seed, rank), with_grad=training)
    layer = mb.MoEExpertLayer(cfg.T, cfg.H, cfg.F, cfg.E, cfg.k, prec, training=training, device=dev,
                              fused_combine=fused_combine)
    w1, w2 = d["w1"].to(dev), d["w2"].to(dev)
    layer.set_weights(w1, w2)
    x, logits = d["x"].to(dev), d["logits"].to(dev)
    grad = d["grad_out"].to(dev) if training else None
    stream = torch.cuda.current_stream(dev)

    # event slots: 0 step start, 1 after weight quantisation, 2 after permute, 3 after
    # grouped_mlp_fwd, 4 after unpermute, 5 after grad permute, 6 after grouped_mlp_bwd
    def step(e=None):
        def mark(i):
            if e is not None:
                e[i].record(stream)
        mark(0)
        if training and prec == "mxfp8":
            layer.set_weights(w1, w2)   # a training step re-quantises the bf16 masters
        mark(1)
        layer.perm["idx"], layer.perm["prob"] = layer.idx, layer.prob
        mb.moe_route_permute(logits, x, cfg.k, True, prec, out=layer.perm, workspace=layer.perm_ws)
        mark(2)
        if fused_combine:
            mb.grouped_mlp_fwd_combine(layer.perm["xp"], layer.perm["split_sizes"], layer.w1, layer.w2,
                                       layer.perm["probs_perm"], layer.perm["row_map"], cfg.T, cfg.k, prec,
                                       xp_scale=layer.perm.get("xp_scale"), w1_scale=layer.w1_scale,
                                       w2_scale=layer.w2_scale, out=layer.out, saved=layer.saved,
                                       workspace=layer.mlp_ws, F=cfg.F)
            mark(3)
        else:
            mb.grouped_mlp_fwd(layer.perm["xp"], layer.perm["split_sizes"], layer.w1, layer.w2,
                               layer.perm["probs_perm"], prec, xp_scale=layer.perm.get("xp_scale"),
                               w1_scale=layer.w1_scale, w2_scale=layer.w2_scale, yp=layer.yp, saved=layer.saved,
                               workspace=layer.mlp_ws, F=cfg.F)
            mark(3)
            mb.moe_unpermute(layer.yp, layer.perm["row_map"], cfg.T, cfg.k, out=layer.out)
        mark(4)
        if training:
            if layer._bwd is None:
                layer._alloc_bwd()
            b = layer._bwd
            if prec == "mxfp8":
                # xp along the expert rows, dy both ways: permuted and quantised in one pass
                layer.permute_for_backward(x)
                layer.permute_grad(grad)
                mark(5)
                mb.grouped_mlp_bwd(None, layer.perm["split_sizes"], None, w1, w2, layer.perm["probs_perm"],
                                   layer.saved, prec, dxp=b["dxp"], dw1=b["dw1"], dw2=b["dw2"],
                                   dprobs_perm=b["dprobs_perm"], workspace=b["ws"], operands=layer.bwd_operands(),
                                   shape=(cfg.R, cfg.H, cfg.F))
            else:
                mb.moe_permute_rows(grad, layer.perm["row_map"], cfg.k, out=b["dy_perm"])
                mark(5)
                mb.grouped_mlp_bwd(b["dy_perm"], layer.perm["split_sizes"], layer.perm["xp"], w1, w2,
                                   layer.perm["probs_perm"], layer.saved, prec, dxp=b["dxp"], dw1=b["dw1"],
                                   dw2=b["dw2"], dprobs_perm=b["dprobs_perm"], workspace=b["ws"])
            mark(6)
            if world > 1:
                # data-parallel replicas: the weight gradients are summed over the ranks
                mb.allreduce_grads([b["dw1"], b["dw2"]])
            mb.moe_unpermute(b["dxp"], layer.perm["row_map"], cfg.T, cfg.k, out=b["dx"])
            mb.moe_gather_slots(b["dprobs_perm"], layer.perm["row_map"], out=b["dprob"].view(-1))
            mb.moe_route_bwd(None, layer.idx, layer.prob, b["dprob"], True, dlogits=b["dlogits"])

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    if mb.moe_device_status() != 0:
        raise RuntimeError("device error during warm-up")

    K = steps
    evs = [[ev() for _ in range(7)] for _ in range(K)]
    t0, t1 = ev(), ev()
    barrier(world)
    torch.cuda.synchronize(dev)
    launches0 = mb.moe_launch_count()
    with ClockSampler(local, args.clocks_csv if with_e2e else None) as clocks:
        wall0 = time.perf_counter()
        t0.record(stream)
        for i in range(K):
            step(evs[i])
        t1.record(stream)
        torch.cuda.synchronize(dev)
        wall = time.perf_counter() - wall0
    launches = mb.moe_launch_count() - launches0
    barrier(world)
    ms = t0.elapsed_time(t1) / K
    ms_max = max_over_ranks(ms, world)
    if mb.moe_device_status() != 0:
        raise RuntimeError("device error during the timed region")

    def mean_ms(a, b):
        return statistics.mean(e[a].elapsed_time(e[b]) for e in evs)

    mlp_ms = mean_ms(2, 3) + (mean_ms(5, 6) if training else 0.0)
    perm_ms, unperm_ms = mean_ms(1, 2), (mean_ms(3, 4) if not fused_combine else 0.0)
    quant_ms = mean_ms(0, 1) if training and prec == "mxfp8" else 0.0

    flops = cfg.gemm_flops()
    value = world * flops / (ms_max * 1e-3) / 1e12
    tokens_s = world * cfg.T / (ms_max * 1e-3)

    regime = "sustained" if wall >= 1.0 else "burst"
    peak, peak_note = gemm_peak(prec, regime)
    achieved = flops / (mlp_ms * 1e-3) / 1e12
    spec = SPEC_TFLOPS[prec]
    # algorithmic bytes of the permute (data kernel; the index kernels are inside the
    # timed call) and of the combine
    T, H, R = cfg.T, cfg.H, cfg.R
    perm_bytes = T * H * 2 + (R * H * 2 if prec == "bf16" else R * (H + H // 32))
    unperm_bytes = R * H * 2 + T * H * 2
    peaks, psrc = load_peaks()
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    res = {
        "workload": cfg.name,
        "value": round(value, 3), "unit": "TFLOP/s", "ms_per_step": round(ms_max, 4),
        "tokens_per_s": round(tokens_s, 1), "steps": K, "warmup": warmup, "wall_s": round(wall, 3),
        "gpu_launches": int(launches),
        "config": {"workload": cfg.name, "T": cfg.T, "H": cfg.H, "F": cfg.F, "E": cfg.E, "k": cfg.k,
                   "precision": prec, "pass": cfg.passes, "tokens_per_step_per_gpu": cfg.T,
                   "gemm_flop_per_step_per_gpu": flops,
                   "l2": "inputs larger than L2: the expert weights (%.2f GB bf16) are re-read every step"
                         % ((d["w1"].numel() + d["w2"].numel()) * 2 / 1e9),
                   "parallelism": (f"dp{world} replicas" + (", dw1/dw2 all-reduced (NCCL) every step" if training
                                                              else "")) if world > 1 else "single GPU"},
        "roofline": {"kernel": ("grouped_mlp_fwd + grouped_mlp_bwd (the six tcgen05 grouped GEMMs; MXFP8: the "
                                "backward's operands come quantised from their producers)" if training else
                                "grouped_mlp_fwd (fc1 gate|up + ScaledSwiGLU, fc2: two tcgen05 grouped GEMMs)"),
                     "bound": "tensor", "achieved": round(achieved, 2), "peak": peak, "unit": "TFLOP/s",
                     "frac": round(achieved / peak, 4), "peak_source": f"{peak_note} (timed region {wall:.2f} s)",
                     "frac_of_spec": round(achieved / spec, 4), "spec_peak": spec,
                     "traffic": measured_traffic(cfg.name), "avg_launch_ms": round(mlp_ms, 4)},
        "bandwidth": {
            "permute": {"GB/s": round(perm_bytes / (perm_ms * 1e-3) / 1e9, 1), "ms": round(perm_ms, 4),
                        "bytes": perm_bytes, "note": "moe_route_permute call (routing and index kernels included)"},
            "unpermute": ({"GB/s": round(unperm_bytes / (unperm_ms * 1e-3) / 1e9, 1), "ms": round(unperm_ms, 4),
                           "bytes": unperm_bytes} if not fused_combine else
                          {"note": "fused into fc2's epilogue (timed inside grouped_mlp_fwd_combine)"}),
            "hbm_peak_gbs": hbm, "hbm_peak_source": f"{psrc} copy", "spec_gbs": SPEC_HBM_GBS},
        "clocks": clocks.summary(),
    }
    if quant_ms:
        both = training and prec == "mxfp8"
        wq_bytes = (d["w1"].numel() + d["w2"].numel()) * (2 + (2 if both else 1) * (1 + 1 / 32))
        res["bandwidth"]["weight_quant"] = {
            "GB/s": round(wq_bytes / (quant_ms * 1e-3) / 1e9, 1), "ms": round(quant_ms, 4), "bytes": wq_bytes,
            "note": ("both orientations of w1 and w2 in one pass (mxfp8_quantize_weights: the forward's and the "
                     "backward's operands)" if both else "the forward orientation of w1 and w2")}

    if with_e2e:
        # every step: pinned host -> device copies of the step's inputs, the path, and a
        # device -> host read of its result (the layer output; with backward also dx),
        # through the package's HostPipeline (transfers overlapped with compute)
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
        e0, e1 = ev(), ev()
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
        res["e2e"] = {"value": round(e2e_val, 3), "unit": "TFLOP/s", "ms_per_step": round(e2e_ms, 4),
                      "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}
        del pipe
    del layer
    return res, d


def run_capacity(cfg, args, local, factor: float, steps: int, warmup: int):
    """The capacity-padded dispatch (the padded batched_mm back-end) on a forward
    workload, as a comparison point: route, moe_permute_capacity (C = ceil(factor T k /
    E) rows per expert, overflow dropped), the grouped GEMMs over E*C rows, unpermute."""
    import math
    import mixture_experts_grouped_top_b200 as mb
    dev = torch.device("cuda", local)
    d = workloads.make_layer_inputs(cfg, with_grad=False)
    C = int(math.ceil(factor * cfg.T * cfg.k / cfg.E))
    x, logits = d["x"].to(dev), d["logits"].to(dev)
    w1, w2 = d["w1"].to(dev), d["w2"].to(dev)
    idx = torch.empty((cfg.T, cfg.k), dtype=torch.int32, device=dev)
    prob = torch.empty((cfg.T, cfg.k), dtype=torch.float32, device=dev)
    o = mb.moe_permute_capacity(x, *mb.moe_route(logits, cfg.k, True, idx=idx, prob=prob), cfg.E, C)
    ws = torch.empty(mb.moe_permute_capacity_workspace_size(cfg.T, cfg.k, cfg.E), dtype=torch.uint8, device=dev)
    mlp_ws = torch.empty(mb.grouped_mlp_workspace_size(cfg.E, cfg.E * C, cfg.H, cfg.F), dtype=torch.uint8, device=dev)
    yp = torch.empty((cfg.E * C, cfg.H), dtype=torch.bfloat16, device=dev)
    out = torch.empty((cfg.T, cfg.H), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step():
        mb.moe_route(logits, cfg.k, True, idx=idx, prob=prob)
        mb.moe_permute_capacity(x, idx, prob, cfg.E, C, out=o, workspace=ws)
        mb.grouped_mlp_fwd(o["xp"], o["split_sizes"], w1, w2, o["probs_perm"], yp=yp, workspace=mlp_ws)
        mb.moe_unpermute(yp, o["row_map"], cfg.T, cfg.k, out=out)

    for _ in range(warmup):
        step()
    torch.cuda.synchronize(dev)
    t0, t1 = ev(), ev()
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize(dev)
    if mb.moe_device_status() != 0:
        raise RuntimeError("device error in the capacity-padded run")
    ms = t0.elapsed_time(t1) / steps
    kept = int(o["kept"].sum().item())
    return {"capacity_factor": factor, "C": C, "ms_per_step": round(ms, 4),
            "value": round(cfg.gemm_flops() / (ms * 1e-3) / 1e12, 3),
            "padded_gemm_tflop": round(6.0 * cfg.H * cfg.F * cfg.E * C / 1e12, 3),
            "dropped_slot_frac": round(1.0 - kept / cfg.R, 5),
            "note": "value = the dropless layer's algorithmic FLOPs / time (padding computed, overflow dropped)"}


# ------------------------------------------------------------------ oracle (CPU) arm
def blas_threads() -> int:
    try:
        import threadpoolctl
        n = [i["num_threads"] for i in threadpoolctl.threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # pragma: no cover
        return 1


def oracle_sample(cfg, d, n_tokens: int, seed: int = 1):
    """Time the oracle (as it stands) on n_tokens sampled tokens of the workload: routing
    and the per-expert layer, plus its analytic backward for a forward + backward
    workload (the BF16 reading of the arithmetic, in fp64). Returns (seconds, tokens,
    gemm flops done)."""
    from oracle import moe as om
    toks = workloads.sample_tokens(cfg.T, n_tokens, seed=seed)
    training = cfg.passes == "fwd+bwd"
    t = time.perf_counter()
    xs = om.f64(d["x"][toks])
    idx, prob = om.route(d["logits"][toks], cfg.k)
    if not training:
        om.moe_forward_sampled(xs, idx, prob, d["w1"], d["w2"], np.arange(toks.size), a_round="bf16")
    else:
        row_map, split, offs = om.permute_index(idx, cfg.E)
        xp = om.permute_rows(xs, row_map, cfg.k)
        pp = om.permute_probs(prob, row_map)
        dyp = om.permute_rows(om.f64(d["grad_out"][toks]), row_map, cfg.k)
        for e in range(cfg.E):               # one expert's weights in fp64 at a time
            r = slice(int(offs[e]), int(offs[e + 1]))
            if r.stop == r.start:
                continue
            w1e, w2e = d["w1"][e:e + 1], d["w2"][e:e + 1]
            n = [r.stop - r.start]
            om.grouped_mlp_fwd(xp[r], n, w1e, w2e, pp[r], a_round="bf16")
            om.grouped_mlp_bwd(dyp[r], xp[r], n, w1e, w2e, pp[r], a_round="bf16")
    sec = time.perf_counter() - t
    flops = (18.0 if training else 6.0) * cfg.H * cfg.F * toks.size * cfg.k
    return sec, int(toks.size), flops


def _oracle_sample_text(cfg, n):
    what = "routing + per-expert MLP" + (" + analytic backward" if cfg.passes == "fwd+bwd" else "")
    prec = "" if cfg.precision == "bf16" else " (the BF16 reading: the MXFP8 codecs are not timed)"
    return f"{n} of {cfg.T} tokens of {cfg.name}: fp64 numpy oracle, {what}{prec}"


def cpu_baseline_entry(cfg, d, n_tokens):
    sec, n, flops = oracle_sample(cfg, d, n_tokens)
    return {"value": round(flops / sec / 1e12, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
            "sample": f"{_oracle_sample_text(cfg, n)}, {sec:.2f} s; cores = numpy BLAS threads "
                      f"(host has {os.cpu_count()} cores)",
            "tokens_per_s": round(n / sec, 3)}


def run_reference(args, world, rank):
    if rank != 0:
        return None
    cfg = workloads.CONFIGS[args.workload]
    d = workloads.make_layer_inputs(cfg, with_grad=cfg.passes == "fwd+bwd")
    n_tok = args.reference_tokens
    # one untimed call warms the host caches; more warm-up says nothing about a CPU program
    oracle_sample(cfg, d, max(4, n_tok // 8))
    secs = []
    flops = 0.0
    for i in range(args.steps):
        sec, n, flops = oracle_sample(cfg, d, n_tok, seed=100 + i)
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
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": blas_threads(), "kind": "oracle",
                         "sample": f"{_oracle_sample_text(cfg, n_tok)} per step; ms_per_step extrapolated "
                                   f"to all {cfg.T} tokens"},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_ours(args, world, rank, local):
    cfg = workloads.CONFIGS[args.workload]
    if args.tokens:
        cfg = dataclasses.replace(cfg, name=f"{cfg.name}_T{args.tokens}", T=args.tokens)
    if args.ffn:
        cfg = dataclasses.replace(cfg, name=f"{cfg.name}_F{args.ffn}", F=args.ffn)
    head, d = run_workload(cfg, args, world, rank, local, args.steps, args.warmup, with_e2e=True)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline_entry(cfg, d, args.cpu_baseline_tokens)
    del d
    gc.collect()
    torch.cuda.empty_cache()
    line = {
        "metric": METRIC, "value": head["value"], "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if cfg.precision == "bf16" else "mxfp8(e4m3+e8m0)",
        "data": "synthetic (seeded N(0,1) tokens, router logits and output gradients, N(0,0.02) weights)",
        "config": head["config"], "tokens_per_s": head["tokens_per_s"], "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"], "roofline": head["roofline"], "bandwidth": head["bandwidth"],
        "clocks": head["clocks"], "cpu_baseline": cpu,
    }
    if not args.no_workloads and not args.tokens and not args.ffn:
        line["workloads"] = {}
        for name in SECONDARY_WORKLOADS:
            if name == cfg.name:
                continue
            res, d = run_workload(workloads.CONFIGS[name], args, world, rank, local, args.workload_steps,
                                  args.warmup, with_e2e=False)
            del d
            gc.collect()
            torch.cuda.empty_cache()
            res.pop("config", None)
            line["workloads"][name] = res
            if name in FUSED_COMBINE_WORKLOADS:
                # the same layer with the combine fused into fc2's epilogue
                fres, d = run_workload(workloads.CONFIGS[name], args, world, rank, local, args.workload_steps,
                                       args.warmup, with_e2e=False, fused_combine=True)
                del d
                gc.collect()
                torch.cuda.empty_cache()
                res["fused_combine"] = {k: fres[k] for k in ("value", "ms_per_step", "tokens_per_s", "clocks")}
                res["fused_combine"]["roofline_frac"] = fres["roofline"]["frac"]
            if name in CAPACITY_WORKLOADS:
                res["capacity_padded"] = [run_capacity(workloads.CONFIGS[name], args, local, f, args.workload_steps,
                                                       args.warmup) for f in (1.0, 1.25)]
                gc.collect()
                torch.cuda.empty_cache()
        line["gpu_launches"] = head["gpu_launches"]
    return line


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(workloads.CONFIGS))
    ap.add_argument("--no-workloads", action="store_true", help="time only the headline workload")
    ap.add_argument("--workload-steps", type=int, default=20)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--tokens", type=int, default=0, help="override T (profiling runs on a smaller batch)")
    ap.add_argument("--ffn", type=int, default=0, help="override F (profiling runs on smaller experts)")
    ap.add_argument("--cpu-baseline-tokens", type=int, default=48)
    ap.add_argument("--reference-tokens", type=int, default=32)
    ap.add_argument("--clocks-csv", default=None,
                    help="keep the raw nvidia-smi clock samples of the timed region in this file")
    ap.add_argument("--measure-peaks", action="store_true",
                    help="measure the library BF16 and MXFP8 GEMM peaks and write profiles/mxfp8_peak.json")
    args = ap.parse_args(argv)
    args.warmup = max(args.warmup, 3)
    if args.measure_peaks:
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        res = measure_gemm_peaks(dev)
        res["command"] = "python bench.py --measure-peaks"
        with open(MXFP8_PEAK_FILE, "w") as f:
            json.dump(res, f, indent=1)
        print(json.dumps(res), flush=True)
        return
    if args.impl == "reference":
        # the oracle runs on rank 0's host cores only; no process group is needed
        world = int(os.environ.get("WORLD_SIZE", "1"))
        if int(os.environ.get("RANK", "0")) == 0:
            print(json.dumps(run_reference(args, world, 0)), flush=True)
        return
    world, rank, local = dist_setup(args.gpus)
    try:
        line = run_ours(args, world, rank, local)
        if rank == 0 and line is not None:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
