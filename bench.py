#!/usr/bin/env python
"""GPTQ layer quantization throughput on B200: weights quantized per second.

One step = the whole GPTQ path for one workload.  For every calibration
input: zero H, accumulate H = 2 X X^T over all of its tokens, damp and
factor H into G.  For every linear layer fed by that input: quantize and
pack all of its columns with that G.  Inputs are resident in HBM when the
timed region starts; every X is larger than L2.  With N GPUs every rank runs
its own independent copy of the workload (weak scaling, no collective on
the data path).

Workloads (``--workload``; ``--bits`` overrides the code width):

    down_proj_65b  (default) LLaMA-65B-shaped down projection: W 8192 x 22016,
                   131072 tokens (H of 22016^2), 4-bit asymmetric, g = 128
    gate_proj_65b  the 65B gate projection with its own H: W 22016 x 8192,
                   131072 tokens (H of 8192^2), 4-bit g = 128
    mlp_65b        the 65B-shaped MLP: gate and up 22016 x 8192 sharing one
                   input (H of 8192^2) plus the down projection; 2 Hessians,
                   3 layers
    block_7b       all 7 layers of a LLaMA-7B-shaped decoder block, g = 128:
                   q/k/v share one input, gate/up another, o and down have
                   their own; 4 Hessians, 7 layers
    down_proj_7b   W 4096 x 11008, 262144 tokens, 4-bit g = 128
    q_proj         W 4096 x 4096, 262144 tokens, 4-bit, one scale per row
    small          W 256 x 256, 2048 tokens (a parity case)

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--bits B] [--sym]

Prints one JSON line (rank 0).  Other measurements of the same library, each
its own JSON line:

    --w4a16 BATCH    the dequant-fused 4-bit matmul over the three LLaMA-65B MLP
                     layers (bytes streamed/s against HBM)
    --awq            the AWQ scale search on the q_proj layer, 32768 tokens
    --shard-layer    one q_proj layer strong-scaled across the ranks
                     (token-sharded H + all-reduce, row-sharded quantize)
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time
from datetime import timedelta

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "GPTQ weights quantized/s per linear layer"
UNIT = "weights/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0,
                  "bf16_tflops_sustained": 1400.0}
WORKLOADS = ("down_proj_65b", "gate_proj_65b", "mlp_65b", "block_7b", "down_proj_7b", "q_proj",
             "small")
SM_COUNT = 148


def parse_args(argv=None):
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", choices=WORKLOADS, default="down_proj_65b")
    p.add_argument("--tokens", type=int, default=0,
                   help="calibration tokens (default: the workload's); a smaller "
                        "full-path configuration for profiling captures")
    p.add_argument("--bits", type=int, default=0,
                   help="code width (default: the workload's); same path, other clip/pack widths")
    p.add_argument("--sym", action="store_true", help="symmetric quantizer instead of the workload's")
    p.add_argument("--w4a16", type=int, default=0, metavar="BATCH",
                   help="instead of quantization, time the dequant-fused matmul of "
                        "4-bit LLaMA-65B MLP layers with BATCH activation rows (1..8)")
    p.add_argument("--w4a16-group", type=int, default=128, metavar="G",
                   help="group size of the --w4a16 layers (0: one scale per output channel)")
    p.add_argument("--shard-layer", action="store_true",
                   help="strong scaling: ONE q_proj layer across the ranks (token-sharded H "
                        "summed by an NCCL all-reduce, row-sharded quantize, rows gathered)")
    p.add_argument("--awq", action="store_true",
                   help="time the AWQ scale search (20-point alpha grid) on the q_proj layer "
                        "with 32768 calibration tokens, 4-bit g128")
    p.add_argument("--route", choices=["inverse", "factor"], default="factor",
                   help="factor (default): F, G's diagonal blocks and V_ab G_bb "
                        "(prepare_factor + quantize_layer_factor), half the fp64 work; "
                        "inverse: G = chol(H^-1) (prepare_hinv + quantize_layer)")
    p.add_argument("--no-other-route", action="store_true",
                   help="skip timing the inverse route beside the factor route")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    return p.parse_args(argv)


# ---------------------------------------------------------------- workloads
def workload_layers(name: str, rank: int = 0, bits: int = 0, sym: bool = False,
                    tokens: int = 0):
    """The workload's layers grouped by calibration input: a list of groups,
    each a list of layer specs that share one X (and so one H and one G).
    Rank r of a weak-scaling run gets its own seeds for every W and X."""
    from post_weight_quantization_26_b200 import synth
    b = bits or 4
    table = {
        "small": lambda: [(synth.SMALL_256, 0)],
        "q_proj": lambda: [(synth.Q_PROJ_7B, 0)],
        "down_proj_7b": lambda: [(synth.DOWN_PROJ_7B, 0)],
        "block_7b": lambda: synth.decoder_block_7b(b),
        "mlp_65b": lambda: synth.mlp_65b(b),
        "down_proj_65b": lambda: [synth.mlp_65b(b)[2]],
        "gate_proj_65b": lambda: [synth.mlp_65b(b)[0]],
    }
    groups: dict[int, list] = {}
    for spec, xin in table[name]():
        spec = spec.with_(w_seed=spec.w_seed + rank, x_seed=spec.x_seed + 100 * rank)
        if bits:
            spec = spec.with_(bits=bits)
        if sym:
            spec = spec.with_(sym=True)
        if tokens:
            spec = spec.with_(n_tokens=tokens)
        groups.setdefault(xin, []).append(spec)
    return list(groups.values())


def workload_spec(name: str, rank: int):
    """The first layer of a workload (the only one for single-layer workloads)."""
    return workload_layers(name, rank)[0][0]


def work_model(groups, route="inverse"):
    """Algorithmic work of one step (per stage), counted as the method needs
    it: the SYRK d(d+1)n flops per input; the factorization 2/3 d^3 fp64
    flops per input on the inverse route (Cholesky d^3/3, triangular inverse
    d^3/3), d^3/3 + 128 d^2 on the factor route (Cholesky, and the panels
    V_ab G_bb of F: 2 * 128^2 flops per element row of each panel); the
    column sweep d_row d_col (d_col - 1) fp32 flops per layer; and the packed
    output d_row d_col (1 + b/8) bytes per layer."""
    w = {"weights": 0, "syrk_flops": 0.0, "chol_flops": 0.0, "prop_flops": 0.0,
         "pack_bytes": 0.0}
    for layers in groups:
        d, n = layers[0].d_col, layers[0].n_tokens
        w["syrk_flops"] += float(d) * (d + 1) * n
        if route == "factor":
            w["chol_flops"] += float(d) ** 3 / 3.0 + 128.0 * float(d) ** 2
        else:
            w["chol_flops"] += 2.0 / 3.0 * float(d) ** 3
        for s in layers:
            w["weights"] += s.d_row * s.d_col
            w["prop_flops"] += float(s.d_row) * s.d_col * (s.d_col - 1)
            w["pack_bytes"] += float(s.d_row) * s.d_col * (1 + s.bits / 8)
    return w


def workload_config(name, groups, world):
    layers = [s for g in groups for s in g]
    first = layers[0]
    x_bytes = sum(g[0].n_tokens * g[0].d_col * 2 for g in groups)
    cfg = {"workload": name if len(layers) > 1 else first.name,
           "layers": [f"{s.name} {s.d_row}x{s.d_col}" for s in layers],
           "inputs": len(groups),
           "bits": first.bits, "group_size": first.group, "sym": first.sym,
           "block": first.block, "damp": first.damp,
           "w": f"{first.w_dist} sigma={first.w_sigma} {'bf16' if first.w_bf16 else 'fp32'}",
           "x": "; ".join(f"{g[0].x_dist} bf16 {g[0].n_tokens} tokens x {g[0].d_col}, "
                          f"{g[0].outlier_count} channels x{g[0].outlier_scale:g}" for g in groups),
           "l2": "inputs larger than L2 (X bf16 %.2f GB per step)" % (x_bytes / 1e9),
           "parallelism": f"{world} independent workload copy(ies), one per GPU"}
    if len(layers) == 1:
        cfg.update(d_row=first.d_row, d_col=first.d_col, n_tokens=first.n_tokens)
    return cfg


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during a region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.lines: list[str] = []
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200", "-i", str(self.dev)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}




# --------------------------------------------------------- oracle baseline
def oracle_sample(groups, x_hosts, w_hosts, tokens, fac_dim, rows):
    """Time the CPU oracle, as it stands, on a bounded sample of the workload
    and extrapolate to the whole step.  The sample is the leading
    sub-problem: the first fac input channels, a token prefix and a few rows.
    Per input: the Hessian of the prefix over those channels (time scaled by
    n / prefix x (d / fac)^2) and its factorization (scaled by (d / fac)^3).
    Per layer: GPTQ of `rows` rows over those fac columns with that factor
    (scaled by d_row / rows x d_col / fac: linear in the width, which
    under-counts the oracle's O(d_col^2) trailing updates, so the estimate
    favours the oracle).  Returns the extrapolated seconds per step, the
    seconds the sample itself took, per-stage estimates, and a description."""
    import numpy as np

    from oracle import gptq_oracle as O
    est = {"hessian": 0.0, "factor": 0.0, "quantize": 0.0}
    t_all = time.perf_counter()
    parts = []
    for gi, layers in enumerate(groups):
        d, n = layers[0].d_col, layers[0].n_tokens
        tk, fac = min(tokens, n), min(fac_dim, d)
        t0 = time.perf_counter()
        h = O.hessian(x_hosts[gi][:tk, :fac].float().numpy())
        est["hessian"] += (time.perf_counter() - t0) * (n / tk) * (d / fac) ** 2
        t0 = time.perf_counter()
        hd, dead = O.dampen(h, layers[0].damp)
        u = O.hinv_cholesky_upper(hd)
        est["factor"] += (time.perf_counter() - t0) * (d / fac) ** 3
        for li, s in enumerate(layers):
            r = min(rows, s.d_row)
            w = w_hosts[gi][li][:r, :fac].numpy().astype(np.float64)
            t0 = time.perf_counter()
            O.gptq_quantize(w, u, s.bits, s.group, s.sym, s.block, dead=dead)
            est["quantize"] += (time.perf_counter() - t0) * (s.d_row / r) * (d / fac)
        parts.append(f"H over the first {fac} of {d} channels on {tk} of {n} tokens, its "
                     f"factor, GPTQ of {min(rows, layers[0].d_row)} rows x {fac} columns "
                     f"per layer ({len(layers)} layer(s))")
    sample_s = time.perf_counter() - t_all
    return {"seconds_per_step": sum(est.values()), "sample_seconds": sample_s,
            "stage_s": est,
            "sample": "; ".join(parts) + "; extrapolated: H x n/prefix x (d/fac)^2, factor x "
                      "(d/fac)^3, GPTQ x rows x width (linear)"}


def cpu_cores():
    cores = len(os.sched_getaffinity(0))
    try:
        from threadpoolctl import threadpool_info
        th = max((i.get("num_threads", 1) for i in threadpool_info()), default=cores)
        return min(cores, th) if th else cores
    except Exception:
        return cores


def host_inputs(groups, pin=False):
    """Seeded host inputs: one token-major bf16 X per input group, one fp32 W
    per layer (pinned when asked, for the device copies)."""
    import torch

    from post_weight_quantization_26_b200 import synth
    xs, ws = [], []
    for layers in groups:
        s0 = layers[0]
        x = torch.empty((s0.n_tokens, s0.d_col), dtype=torch.bfloat16)
        if pin:
            x = x.pin_memory()
        synth.gen_tokens(s0, out=x)
        xs.append(x)
        ws.append([synth.gen_weight(s).pin_memory() if pin else synth.gen_weight(s)
                   for s in layers])
    return xs, ws


# --------------------------------------------------------------- reference
def run_reference(args, rank, world):
    """The oracle arm: the CPU oracle timed on the host cores on a bounded
    sample of every step (rank 0 only).  `ms_per_step` is the time the sample
    took; `value` is the whole-step rate extrapolated from it."""
    if rank != 0:
        return
    groups = workload_layers(args.workload, 0, args.bits, args.sym, args.tokens)
    tokens, fac, rows = 1024, 4096, 8
    from post_weight_quantization_26_b200 import synth
    xs = [synth.gen_tokens(g[0], 0, min(tokens, g[0].n_tokens)) for g in groups]
    ws = [[synth.gen_weight(s.with_(d_row=min(rows, s.d_row))) for s in g] for g in groups]
    est, sample_s = [], []
    res = None
    for i in range(args.warmup + args.steps):
        res = oracle_sample(groups, xs, ws, tokens, fac, rows)
        if i >= args.warmup:
            est.append(res["seconds_per_step"])
            sample_s.append(res["sample_seconds"])
    sec = statistics.mean(est)
    value = work_model(groups)["weights"] / sec
    cores = cpu_cores()
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": statistics.mean(sample_s) * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(args.workload, groups, 1),
        "extrapolated": True,
        "extrapolated_ms_per_step": sec * 1e3,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                         "sample": res["sample"], "extrapolated": True},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time: every rank joins one MAX all-reduce (NCCL on
    the GPUs; any backend whose tensors live on ``device``)."""
    if world <= 1:
        return ms
    import torch
    import torch.distributed as dist
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_value(world: int, weights: int, ms_max: float) -> float:
    """Whole-job weights/s: every rank quantizes its own copy of the
    workload's `weights` weights, and the job takes as long as its slowest
    rank."""
    return world * weights / (ms_max / 1e3)


# ------------------------------------------------------------------- ours
def kernel_traffic(name: str, src_rel: str):
    """DRAM bytes per launch from a committed ncu summary, if it was taken on
    the current source of the kernel (else None)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f)[name]
        with open(os.path.join(ROOT, src_rel), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
        if rec.get("source_sha256") != sha:
            return None
        return rec["bytes_per_launch"]
    except (OSError, KeyError, ValueError):
        return None


def stage_roofline(work, stage_ms, ms, peaks, peak_src, clk, groups, name, timed_ms,
                   route="factor"):
    """Each stage against its own bound, the combined roofline T*, and the
    roofline object of the stage that takes the most time.  The bf16 peak is
    the measured burst figure when the timed region is shorter than a second
    and the sustained (power-capped) one when it is longer."""
    sm_mhz = (clk or {}).get("sm_mhz") or peaks.get("sm_max_mhz", 1965.0)
    sustained = timed_ms >= 1000.0
    bf16_key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    bf16 = peaks.get(bf16_key, FALLBACK_PEAKS[bf16_key])
    fp64 = SM_COUNT * 64 * 2 * sm_mhz * 1e6 / 1e12
    fp32 = SM_COUNT * 128 * 2 * sm_mhz * 1e6 / 1e12
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    t_star = (work["syrk_flops"] / (bf16 * 1e12) + work["chol_flops"] / (fp64 * 1e12)
              + work["prop_flops"] / (fp32 * 1e12) + work["pack_bytes"] / (hbm * 1e9))
    ach = {
        "hessian": work["syrk_flops"] / (stage_ms["hessian"] / 1e3) / 1e12,
        "prepare": work["chol_flops"] / (stage_ms["prepare"] / 1e3) / 1e12,
        "quantize": work["prop_flops"] / (stage_ms["quantize"] / 1e3) / 1e12,
    }
    stages = {
        "hessian": {"ms": stage_ms["hessian"], "tflops": ach["hessian"],
                    "frac": ach["hessian"] / bf16,
                    "bound": f"tensor bf16 {bf16:.0f} TF/s ({bf16_key} of {peak_src})"},
        "prepare": {"ms": stage_ms["prepare"], "tflops": ach["prepare"],
                    "frac": ach["prepare"] / fp64,
                    "bound": f"fp64 {fp64:.1f} TF/s derived: {SM_COUNT} SMs x 64 FMA/clk x 2 "
                             f"at {sm_mhz:.0f} MHz"},
        "quantize": {"ms": stage_ms["quantize"], "tflops": ach["quantize"],
                     "frac": ach["quantize"] / fp32,
                     "bound": f"fp32 {fp32:.1f} TF/s derived: {SM_COUNT} SMs x 128 FMA/clk x 2 "
                              f"at {sm_mhz:.0f} MHz",
                     "note": "the trailing updates run on the tensor cores as three TF32 "
                             "products per fp32 product, so the stage can pass the FFMA "
                             "bound that T* charges it with"},
        "zero_h": {"ms": stage_ms["zero_h"]},
        "combined_t_star_ms": t_star * 1e3,
        "combined_frac": t_star * 1e3 / ms,
    }
    top = max(("hessian", "prepare", "quantize"), key=lambda k: stage_ms[k])
    if top == "hessian":
        single = len(groups) == 1
        roof = {"bound": "tensor", "kernel": "syrk_bf16_tcgen05_kernel (the accumulate call's "
                                             "only kernel)",
                "achieved": ach["hessian"], "peak": bf16, "unit": "TFLOP/s",
                "frac": ach["hessian"] / bf16,
                "traffic": kernel_traffic(f"syrk_bf16_tcgen05_kernel/{name}",
                                          "post_weight_quantization_26_b200/csrc/syrk_tcgen05.cuh")
                if single else None,
                "peak_source": f"{bf16_key} of {peak_src} (timed region "
                               f"{timed_ms / 1e3:.1f} s)"}
    elif top == "prepare":
        roof = {"bound": "tensor", "kernel": "dgemm_nt_kernel (fp64 MMA), over the whole "
                                             "prepare stage (with leaf_kernel and the damping)",
                "achieved": ach["prepare"], "peak": fp64, "unit": "TFLOP/s",
                "frac": ach["prepare"] / fp64,
                "traffic": kernel_traffic(f"dgemm_nt_kernel/{name}" +
                                          ("/factor" if route == "factor" else ""),
                                          "post_weight_quantization_26_b200/csrc/chol_fp64.cuh"),
                "peak_source": f"derived: {SM_COUNT} SMs x 64 fp64 FMA/clk x 2 at the sampled "
                               f"{sm_mhz:.0f} MHz (no measured fp64 peak)"}
    else:
        roof = {"bound": "alu", "kernel": "block_step_kernel + trailing_tf32x3_kernel, over the "
                                          "whole quantize stage",
                "achieved": ach["quantize"], "peak": fp32, "unit": "TFLOP/s",
                "frac": ach["quantize"] / fp32, "traffic": None,
                "peak_source": f"derived: {SM_COUNT} SMs x 128 fp32 FMA/clk x 2 at the sampled "
                               f"{sm_mhz:.0f} MHz"}
    return stages, roof


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from post_weight_quantization_26_b200 import build as _build
    from post_weight_quantization_26_b200 import gptq as G

    if rank == 0:
        _build.build()
    if world > 1:
        dist.barrier()
    G.load_library()
    dev = torch.device("cuda", local_rank)
    groups = workload_layers(args.workload, rank, args.bits, args.sym, args.tokens)
    work = work_model(groups, args.route)
    x_hosts, w_hosts = host_inputs(groups, pin=True)
    factor = args.route == "factor"
    if factor and any(s.block != 128 or (s.group and 128 % s.group) for g in groups for s in g):
        raise SystemExit("--route factor needs block 128 and group_size 0 or a divisor of 128")
    routes = {"factor": (G.gptq_prepare_factor, G.gptq_quantize_layer_factor),
              "inverse": (G.gptq_prepare_hinv, G.gptq_quantize_layer)}
    prepare, quantize = routes[args.route]

    cfgs = [[G.make_config(bits=s.bits, group_size=s.group, sym=s.sym, block=s.block,
                           damp_rel=s.damp) for s in layers] for layers in groups]
    ws_bytes = max(G.gptq_workspace_size(s.d_row, s.d_col, c)
                   for layers, cl in zip(groups, cfgs) for s, c in zip(layers, cl))
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    dev_in = []
    for gi, layers in enumerate(groups):
        d = layers[0].d_col
        H = torch.zeros((d, d), dtype=torch.float32, device=dev)
        dev_in.append({
            "x": x_hosts[gi].to(dev), "H": H, "G": torch.empty_like(H),
            "dead": torch.empty(d, dtype=torch.uint8, device=dev),
            "w": [wh.to(dev) for wh in w_hosts[gi]],
            "out": [G.alloc_outputs(s.d_row, s.d_col, c, device=dev)
                    for s, c in zip(layers, cfgs[gi])]})
    stream = torch.cuda.current_stream(dev)

    def step(marks=None, route=None):
        prep, quant = routes[route or args.route]

        def mark(stage):
            if marks is not None:
                e = torch.cuda.Event(enable_timing=True)
                e.record(stream)
                marks.append((stage, e))
        mark("start")
        for gi, layers in enumerate(groups):
            b = dev_in[gi]
            b["H"].zero_()
            mark("zero_h")
            G.gptq_hessian_accumulate(b["H"], b["x"])
            mark("hessian")
            prep(b["H"], layers[0].damp, b["G"], b["dead"], ws)
            mark("prepare")
            for li, s in enumerate(layers):
                qw, sc, ze = b["out"][li]
                quant(b["w"][li], b["G"], b["dead"], cfgs[gi][li], qw, sc, ze, ws)
                mark("quantize")

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if G.gptq_device_status() != 0:
        raise RuntimeError("device status set during warm-up")

    marks = [[] for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    launches0 = G.gptq_launch_count()
    t0.record(stream)
    for i in range(args.steps):
        step(marks[i])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    launches = G.gptq_launch_count() - launches0
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    ms = t0.elapsed_time(t1) / args.steps
    stage_ms = {k: 0.0 for k in ("zero_h", "hessian", "prepare", "quantize")}
    for m in marks:
        for (_, a), (stage, b) in zip(m[:-1], m[1:]):
            stage_ms[stage] += a.elapsed_time(b) / args.steps
    if G.gptq_device_status() != 0:
        raise RuntimeError("device status set during the timed region")

    ms_max = max_over_ranks(ms, world, dev)
    value = weak_value(world, work["weights"], ms_max)

    # ---- the inverse route (G = chol(H^-1) whole) on the same inputs, for
    # comparison: same warm-up, up to 5 timed steps, its own stage times
    other = None
    if factor and not args.no_other_route:
        for _ in range(args.warmup):
            step(route="inverse")
        omarks = [[] for _ in range(min(args.steps, 5))]
        o0, o1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(dev)
        o0.record(stream)
        for m in omarks:
            step(m, route="inverse")
        o1.record(stream)
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        oms = max_over_ranks(o0.elapsed_time(o1) / len(omarks), world, dev)
        ostage = {k: 0.0 for k in ("zero_h", "hessian", "prepare", "quantize")}
        for m in omarks:
            for (_, a), (stage, b) in zip(m[:-1], m[1:]):
                ostage[stage] += a.elapsed_time(b) / len(omarks)
        if G.gptq_device_status() != 0:
            raise RuntimeError("device status set while timing the inverse route")
        owork = work_model(groups, "inverse")
        other = {"route": "inverse", "steps": len(omarks), "ms_per_step": oms,
                 "value": weak_value(world, owork["weights"], oms), "unit": UNIT,
                 "stage_ms": ostage,
                 "prepare_tflops": owork["chol_flops"] / (ostage["prepare"] / 1e3) / 1e12}

    # ---- end to end: host buffers in, host buffers out, through the same API
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, G, groups, cfgs, x_hosts, w_hosts, dev_in, ws, dev, stream, world,
                      work["weights"], prepare, quantize)

    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    stages, roofline = stage_roofline(work, stage_ms, ms, peaks, peak_src, clk, groups,
                                      args.workload, ms * args.steps, args.route)
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        res = oracle_sample(groups, x_hosts, w_hosts, tokens=4096, fac_dim=8192, rows=32)
        cpu = {"value": work["weights"] / res["seconds_per_step"], "unit": UNIT,
               "cores": cpu_cores(), "kind": "oracle", "sample": res["sample"],
               "extrapolated": True, "sample_seconds": res["sample_seconds"],
               "stage_s_est": res["stage_s"]}
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 in / f32 acc (H); f64 (factor); f32 (sweep)",
        "data": "synthetic (seeded LLaMA-shaped layers and activations)",
        "config": dict(workload_config(args.workload, groups, world), route=args.route),
        "stage_ms": stage_ms, "stages": stages,
        "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
        "gpu_launches": launches, "clocks": clk,
    }
    if other is not None:
        line["inverse_route"] = other
    print(json.dumps(line), flush=True)


def run_e2e(args, G, groups, cfgs, x_hosts, w_hosts, dev_in, ws, dev, stream, world, weights,
            prepare, quantize):
    """Same metric through the public API with host buffers: every step copies
    each X and each W from pinned host memory and reads the packed results
    back to the host.  The inputs are double-buffered on the device, and a
    copy stream brings in the next step's X and W while the current step
    computes (its factorization leaves the host link idle); the first timed
    step's copy runs before any compute, so the timed region holds exactly one
    copy of every step's inputs."""
    import torch
    import torch.distributed as dist
    copy_stream = torch.cuda.Stream(dev)
    bufs = [[{"x": torch.empty_like(b["x"]), "w": [torch.empty_like(w) for w in b["w"]]}
             for b in dev_in] for _ in range(2)]
    host_out = [[tuple(torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in o)
                 for o in b["out"]] for b in dev_in]
    copied = [torch.cuda.Event() for _ in range(2)]
    consumed = [torch.cuda.Event() for _ in range(2)]
    used = [False, False]

    def fetch(k):
        """Copy every input group's X and W into buffer set k (copy stream)."""
        with torch.cuda.stream(copy_stream):
            if used[k]:
                copy_stream.wait_event(consumed[k])
            for gi in range(len(groups)):
                bufs[k][gi]["x"].copy_(x_hosts[gi], non_blocking=True)
                for li in range(len(groups[gi])):
                    bufs[k][gi]["w"][li].copy_(w_hosts[gi][li], non_blocking=True)
            copied[k].record(copy_stream)

    def compute(k):
        stream.wait_event(copied[k])
        for gi, layers in enumerate(groups):
            b, inp = dev_in[gi], bufs[k][gi]
            b["H"].zero_()
            G.gptq_hessian_accumulate(b["H"], inp["x"])
            prepare(b["H"], layers[0].damp, b["G"], b["dead"], ws)
            for li, s in enumerate(layers):
                qw, sc, ze = b["out"][li]
                quantize(inp["w"][li], b["G"], b["dead"], cfgs[gi][li], qw, sc, ze, ws)
                for h, t in zip(host_out[gi][li], b["out"][li]):
                    h.copy_(t, non_blocking=True)
        consumed[k].record(stream)
        used[k] = True

    def run(nsteps):
        fetch(0)
        for i in range(nsteps):
            if i + 1 < nsteps:
                fetch((i + 1) & 1)
            compute(i & 1)

    steps = max(1, args.steps)
    run(max(1, min(args.warmup, 3)))
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    run(steps)
    t1.record(stream)
    torch.cuda.synchronize(dev)
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world, dev)
    h2d = sum(g[0].n_tokens * g[0].d_col * 2 + sum(s.d_row * s.d_col * 4 for s in g)
              for g in groups)
    d2h = sum(t.numel() * t.element_size() for b in dev_in for o in b["out"] for t in o)
    return {"value": weak_value(world, weights, ms), "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

# ------------------------------------------------- dequant-fused matmul
W4_METRIC = "W4A16 dequant-fused matmul, bytes streamed/s"
W4_LAYERS = (("gate_proj", 22016, 8192), ("up_proj", 22016, 8192), ("down_proj", 8192, 22016))


def run_w4a16(args, rank, world, local_rank):
    """One step = the three 4-bit (g = 128 by default) LLaMA-65B MLP matmuls for one
    batch of activation rows.  The packed layers total 271 MB, more than L2,
    and run back to back, so every step streams them from HBM.  Each rank
    runs its own copy (weak scaling, no collective)."""
    import torch
    import torch.distributed as dist

    from post_weight_quantization_26_b200 import build as _build
    from post_weight_quantization_26_b200 import gptq as G
    from post_weight_quantization_26_b200 import synth

    batch = args.w4a16
    if rank == 0:
        _build.build()
    if world > 1:
        dist.barrier()
    G.load_library()
    dev = torch.device("cuda", local_rank)
    group = args.w4a16_group
    cfg = G.make_config(bits=4, group_size=group)
    layers, host = [], []
    for i, (name, dr, dc) in enumerate(W4_LAYERS):
        words, scales, zeros = synth.gen_packed_layer(dr, dc, group, seed=100 * rank + i)
        xh = synth.gen_activations(batch, dc, seed=100 * rank + i).pin_memory()
        layers.append((words.to(dev), scales.to(dev), zeros.to(dev), xh.to(dev),
                       torch.empty((batch, dr), dtype=torch.float32, device=dev)))
        host.append((xh, torch.empty((batch, dr), dtype=torch.float32).pin_memory()))
    # algorithmic bytes: packed words + scales + zeros + X + Y, once per layer
    layer_bytes = [dr * dc // 2 + dr * (dc // group if group else 1) * 5 + batch * dc * 2 + batch * dr * 4
                   for _, dr, dc in W4_LAYERS]
    step_bytes = sum(layer_bytes)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        for i, (wq, sc, ze, x, y) in enumerate(layers):
            if ev:
                ev[i][0].record(stream)
            G.gptq_w4a16_matmul(wq, sc, ze, cfg, x, Y=y)
            if ev:
                ev[i][1].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    steps = max(1, args.steps)
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in W4_LAYERS]
           for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    launches0 = G.gptq_launch_count()
    t0.record(stream)
    for i in range(steps):
        step(evs[i])
    t1.record(stream)
    torch.cuda.synchronize(dev)
    launches = G.gptq_launch_count() - launches0
    clk = clocks.stop()
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, world, dev)
    per_layer_us = [statistics.mean(e[i][0].elapsed_time(e[i][1]) for e in evs) * 1e3
                    for i in range(len(W4_LAYERS))]

    e2e = None
    if not args.no_e2e:
        def e2e_step():
            for (wq, sc, ze, x, y), (xh, yh) in zip(layers, host):
                x.copy_(xh, non_blocking=True)
                G.gptq_w4a16_matmul(wq, sc, ze, cfg, x, Y=y)
                yh.copy_(y, non_blocking=True)
        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        ems = max_over_ranks(a.elapsed_time(b) / steps, world, dev)
        e2e = {"value": world * step_bytes / (ems / 1e3) / 1e9, "unit": "GB/s", "ms_per_step": ems,
               "h2d_bytes_per_step": sum(batch * dc * 2 for _, _, dc in W4_LAYERS),
               "d2h_bytes_per_step": sum(batch * dr * 4 for _, dr, _ in W4_LAYERS)}
    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    peak = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    big = max(range(len(W4_LAYERS)), key=lambda i: per_layer_us[i])
    achieved = layer_bytes[big] / (per_layer_us[big] / 1e6) / 1e9
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        import numpy as np

        from oracle import gptq_oracle as O
        name, dr, dc = W4_LAYERS[1]
        rows = 512
        wq, sc, ze, _, _ = layers[1]
        wh, sch, zeh = (wq[:rows].cpu().numpy().view(np.uint32), sc[:rows].cpu().numpy(),
                        ze[:rows].cpu().numpy())
        xf = host[1][0].float().numpy()
        t = time.perf_counter()
        O.dequantized_matmul(wh, sch, zeh, xf, 4, group)
        sec = (time.perf_counter() - t) * dr / rows * len(W4_LAYERS)
        cpu = {"value": step_bytes / sec / 1e9, "unit": "GB/s", "cores": cpu_cores(),
               "kind": "oracle",
               "sample": f"{name} rows 0..{rows - 1} of {dr} (x{dr / rows:g}), x3 layers"}
    line = {
        "metric": W4_METRIC, "value": world * step_bytes / (ms / 1e3) / 1e9, "unit": "GB/s",
        "n_gpus": world, "steps": steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "u4 weights, bf16 activations, f32 accumulate", "data": "synthetic",
        "config": {"workload": f"LLaMA-65B MLP (gate, up 22016x8192; down 8192x22016), "
                               f"4-bit {f'g{group}' if group else 'per channel'}, batch {batch}",
                   "batch": batch, "l2": "inputs larger than L2 (271 MB of packed layers per step)",
                   "parallelism": f"{world} independent replica(s), one per GPU"},
        "per_layer_us": dict(zip([n for n, _, _ in W4_LAYERS], per_layer_us)),
        "roofline": {"bound": "hbm",
                     "kernel": ("w4a16_wide_kernel" if group == 0 or group % 128 == 0
                                else "w4a16_matmul_kernel") + f" ({W4_LAYERS[big][0]})",
                     "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "traffic": kernel_traffic(f"w4a16_matmul_kernel/{W4_LAYERS[big][0]}",
                                               "post_weight_quantization_26_b200/csrc/w4a16.cuh"),
                     "algorithmic_bytes": layer_bytes[big],
                     "peak_source": f"hbm_gbs of {peak_src}"},
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clk,
    }
    print(json.dumps(line), flush=True)

# ------------------------------------------------- one layer across ranks
def run_sharded(args, rank, world, local_rank):
    """Strong scaling of one q_proj layer: rank r accumulates H over its
    token shard, one NCCL all-reduce sums H, every rank factors it, and rank
    r quantizes its row shard; the packed rows are gathered in rank order.
    Value = the layer's weights / the slowest rank's step time."""
    import torch
    import torch.distributed as dist

    from post_weight_quantization_26_b200 import build as _build
    from post_weight_quantization_26_b200 import gptq as G
    from post_weight_quantization_26_b200 import sharded, synth

    if rank == 0:
        _build.build()
    if world > 1:
        dist.barrier()
    G.load_library()
    dev = torch.device("cuda", local_rank)
    spec = synth.Q_PROJ_7B  # the same layer on every rank
    if args.tokens:
        spec = spec.with_(n_tokens=args.tokens, name=f"{spec.name}_n{args.tokens}")
    d, dr = spec.d_col, spec.d_row
    t0, t1 = sharded.shard(spec.n_tokens, world, rank)
    r0, r1 = sharded.shard(dr, world, rank)
    cfg = G.make_config(bits=spec.bits, group_size=spec.group, sym=spec.sym,
                        block=spec.block, damp_rel=spec.damp)
    x = synth.gen_tokens(spec, t0, t1).to(dev)
    w = synth.gen_weight(spec)[r0:r1].contiguous().to(dev)
    stream = torch.cuda.current_stream(dev)
    base = sharded.cuda_steps(cfg, spec.damp, world, dev, route=args.route)
    marks = {}

    def timed(name, fn):
        def run(*a):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            out = fn(*a)
            e1.record(stream)
            marks.setdefault(name, []).append((e0, e1))
            return out
        return run

    steps = sharded.Steps(base.zeros_h, timed("hessian", base.accumulate),
                          timed("allreduce", base.allreduce_sum), timed("prepare", base.prepare),
                          timed("quantize", base.quantize), timed("gather", base.allgather_rows))

    def step():
        return sharded.quantize_layer_sharded(steps, x, w, d)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    if G.gptq_device_status() != 0:
        raise RuntimeError("device status set during warm-up")
    marks.clear()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    launches0 = G.gptq_launch_count()
    a.record(stream)
    for _ in range(args.steps):
        step()
    b.record(stream)
    torch.cuda.synchronize(dev)
    launches = G.gptq_launch_count() - launches0
    clk = clocks.stop()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(a.elapsed_time(b) / args.steps, world, dev)
    stage_ms = {k: statistics.mean(e0.elapsed_time(e1) for e0, e1 in v) for k, v in marks.items()}
    if G.gptq_device_status() != 0:
        raise RuntimeError("device status set during the timed region")
    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    achieved = d * (d + 1) * (t1 - t0) / (stage_ms["hessian"] / 1e3) / 1e12
    line = {
        "metric": METRIC, "value": dr * d / (ms / 1e3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
        "higher_is_better": True, "scaling": "strong", "vs_baseline": None,
        "dtype": "bf16 in / f32 acc (H); f64 (factor); f32 (sweep)",
        "data": "synthetic (seeded LLaMA-7B-shaped layer and activations)",
        "config": {"workload": f"{spec.name}, one layer across {world} GPU(s)",
                   "d_row": dr, "d_col": d, "n_tokens": spec.n_tokens,
                   "tokens_on_rank0": t1 - t0, "rows_on_rank0": r1 - r0,
                   "l2": "inputs larger than L2 (X bf16 %.2f GB over all ranks)"
                         % (spec.n_tokens * d * 2 / 1e9),
                   "parallelism": "token-sharded H + NCCL all-reduce, row-sharded quantize, "
                                  "rows all-gathered"},
        "stage_ms_rank0": stage_ms,
        "roofline": {"bound": "tensor", "kernel": "syrk_bf16_tcgen05_kernel (rank 0's tokens)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": None,
                     "peak_source": f"bf16_tflops_sustained of {peak_src}"},
        "cpu_baseline": None, "e2e": None, "gpu_launches": launches, "clocks": clk,
    }
    print(json.dumps(line), flush=True)

# ------------------------------------------------------ AWQ scale search
AWQ_METRIC = "AWQ scale search: weights quantized/s per linear layer"
AWQ_TOKENS = 32768  # the AWQ section's calibration size (~32K tokens)


def run_awq(args, rank, world, local_rank):
    """One step = the AWQ search for one q_proj layer: the channel scale and
    the Hessian over 32768 calibration tokens, the 20-point alpha grid (each
    point: quantize W diag(s), form dW, the output error through H) and the
    4-bit quantization at the best alpha.  Each rank searches its own layer
    (weak scaling, no collective)."""
    import numpy as np
    import torch
    import torch.distributed as dist

    from post_weight_quantization_26_b200 import build as _build
    from post_weight_quantization_26_b200 import gptq as G
    from post_weight_quantization_26_b200 import synth

    if rank == 0:
        _build.build()
    if world > 1:
        dist.barrier()
    G.load_library()
    dev = torch.device("cuda", local_rank)
    spec = workload_spec("q_proj", rank).with_(n_tokens=args.tokens or AWQ_TOKENS, group=128)
    d, n, dr = spec.d_col, spec.n_tokens, spec.d_row
    n_grid = 20
    cfg = G.make_config(bits=4, group_size=128)
    x_host = synth.gen_tokens(spec).pin_memory()
    w_host = synth.gen_weight(spec).pin_memory()
    x, w = x_host.to(dev), w_host.to(dev)
    H = torch.zeros((d, d), dtype=torch.float32, device=dev)
    sx = torch.empty(d, dtype=torch.float64, device=dev)
    ws = torch.empty(G.gptq_awq_workspace_size(dr, d, cfg), dtype=torch.uint8, device=dev)
    qw, sc, ze = G.alloc_outputs(dr, d, cfg, device=dev)
    out = (torch.empty(n_grid, dtype=torch.float64, device=dev),
           torch.empty(1, dtype=torch.int32, device=dev),
           torch.empty(d, dtype=torch.float32, device=dev), qw, sc, ze)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        if ev:
            ev[0].record(stream)
        G.gptq_awq_channel_scale(x, sx)
        H.zero_()
        G.gptq_hessian_accumulate(H, x)
        if ev:
            ev[1].record(stream)
        G.gptq_awq_search(w, H, sx, cfg, n_grid, ws=ws, out=out)
        if ev:
            ev[2].record(stream)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize(dev)
    if G.gptq_device_status() != 0:
        raise RuntimeError("device status set during warm-up")
    steps = max(1, args.steps)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(steps)]
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local_rank)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    launches0 = G.gptq_launch_count()
    a.record(stream)
    for i in range(steps):
        step(evs[i])
    b.record(stream)
    torch.cuda.synchronize(dev)
    launches = G.gptq_launch_count() - launches0
    clk = clocks.stop()
    ms = max_over_ranks(a.elapsed_time(b) / steps, world, dev)
    stats_ms = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    search_ms = statistics.mean(e[1].elapsed_time(e[2]) for e in evs)
    if G.gptq_device_status() != 0:
        raise RuntimeError("device status set during the timed region")
    best = int(out[1].item())

    e2e = None
    if not args.no_e2e:
        qh = torch.empty(qw.shape, dtype=qw.dtype).pin_memory()
        sh = torch.empty(sc.shape, dtype=sc.dtype).pin_memory()
        zh = torch.empty(ze.shape, dtype=ze.dtype).pin_memory()
        s_h = torch.empty(d, dtype=torch.float32).pin_memory()

        def e2e_step():
            x.copy_(x_host, non_blocking=True)
            w.copy_(w_host, non_blocking=True)
            step()
            qh.copy_(qw, non_blocking=True)
            sh.copy_(sc, non_blocking=True)
            zh.copy_(ze, non_blocking=True)
            s_h.copy_(out[2], non_blocking=True)
        e2e_step()
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        ems = max_over_ranks(e0.elapsed_time(e1) / steps, world, dev)
        e2e = {"value": world * dr * d / (ems / 1e3), "unit": UNIT, "ms_per_step": ems,
               "h2d_bytes_per_step": n * d * 2 + dr * d * 4,
               "d2h_bytes_per_step": qw.numel() * 4 + sc.numel() * 4 + ze.numel() + d * 4}
    if rank != 0:
        return
    peaks, peak_src = load_peaks()
    tf32_peak = peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]) * (1.1 / 2.25)
    tensor_flops = n_grid * 6.0 * dr * d * d  # three TF32 products of dW H per alpha
    achieved = tensor_flops / (search_ms / 1e3) / 1e12
    cpu = None
    if not args.no_cpu_baseline and world == 1:
        from oracle import awq_oracle as A
        from oracle import gptq_oracle as O
        rows, toks = 64, 8192
        t0 = time.perf_counter()
        xs = x_host[:toks].float().numpy()
        sx_c = A.channel_scale(xs)
        h_c = O.hessian(xs)
        t1 = time.perf_counter()
        A.search(w_host[:rows].numpy().astype(np.float64), h_c, sx_c, 4, 128, n_grid)
        t2 = time.perf_counter()
        sec = (t1 - t0) * n / toks + (t2 - t1) * dr / rows
        cpu = {"value": dr * d / sec, "unit": UNIT, "cores": cpu_cores(), "kind": "oracle",
               "sample": f"channel scale and H on {toks} of {n} tokens (x{n / toks:g}); the "
                         f"20-point search on {rows} of {dr} rows (x{dr / rows:g})"}
    line = {
        "metric": AWQ_METRIC, "value": world * dr * d / (ms / 1e3), "unit": UNIT, "n_gpus": world,
        "steps": steps, "warmup": max(3, args.warmup), "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16 in / f32 acc (H); split-TF32 (dW H); f64 (loss sums)",
        "data": "synthetic (seeded LLaMA-7B-shaped layer and activations)",
        "config": {"workload": f"AWQ {spec.name} 4096x4096, {n} tokens, 4-bit g128, "
                               f"{n_grid}-point alpha grid",
                   "d_row": dr, "d_col": d, "n_tokens": n, "group_size": 128, "n_grid": n_grid,
                   "l2": "inputs larger than L2 (X bf16 %.2f GB; dW splits and T 192 MB per "
                         "alpha)" % (n * d * 2 / 1e9),
                   "parallelism": f"{world} independent layer(s), one per GPU"},
        "stage_ms": {"channel_scale_and_hessian": stats_ms, "search": search_ms},
        "best_alpha": best / (n_grid - 1),
        "roofline": {"bound": "tensor", "kernel": "trailing_tf32x3_kernel (dW H), over the "
                                                  "whole search stage",
                     "achieved": achieved, "peak": tf32_peak, "unit": "TFLOP/s",
                     "frac": achieved / tf32_peak,
                     "traffic": kernel_traffic("trailing_tf32x3_kernel/awq_q_proj_4096",
                                               "post_weight_quantization_26_b200/csrc/trailing_tf32.cuh")
                     if (dr, d) == (4096, 4096) else None,
                     "peak_source": f"bf16_tflops_sustained of {peak_src} x 1.1/2.25 "
                                    "(nominal tf32/bf16)"},
        "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches, "clocks": clk,
    }
    print(json.dumps(line), flush=True)


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.w4a16:
            run_w4a16(args, rank, world, local_rank)
        elif args.shard_layer:
            run_sharded(args, rank, world, local_rank)
        elif args.awq:
            run_awq(args, rank, world, local_rank)
        else:
            run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
