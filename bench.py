"""Benchmark of the MX block-quantization hot path on one or more B200s.

Workload: a Llama-3-8B-shaped linear layer, A = 8192 x 4096 bf16 activations
(Laplace(0,1)), W = 14336 x 4096 bf16 weights (N(0, 0.02)), synthetic and
seeded.  One step = every memory-bound row of the path on A and W:
MXFP4 quantize+pack with fused fidelity stats, NVFP4 (tensor amax pre-pass +
UE4M3 quantize), 32-point Hadamard + MXFP4, MBS + OAS MXFP4, and dequantize
to bf16; launches alternate between A and W so that consecutive kernels read
different tensors (A + W = 176 MiB > the 126 MB L2).  ``value`` is the
step's algorithmic bytes (inputs read once, codes/scales/outputs written
once; the NVFP4 amax pre-pass is time, not bytes) over the step time, summed
over ranks.  The block-scaled FP4 GEMM (A^Q W^Q^T, FP32 accumulate) is timed
as its own leg in the same run and reported under ``gemm``.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
(N > 1: launched by torchrun, one process per GPU, weak scaling: every rank
quantizes its own copy of the layer, no data-path collective.)
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
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

M_TOK, K_DIM, N_OUT = 8192, 4096, 14336
R_PAIRS = 8          # repeats of a variant's A+W call per per-variant timing graph
WORKLOAD = ("Llama-3-8B-shaped linear layer: A 8192x4096 bf16 Laplace(0,1) seed 6, "
            "W 14336x4096 bf16 N(0,0.02) seed 7 (W stored out x in, product A W^T)")
METRIC = "MX quantize+pack GB/s (% of ~8 TB/s HBM); block-scaled FP4 GEMM TFLOPS"


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-gemm", action="store_true")
    ap.add_argument("--one-stream", action="store_true",
                    help="capture the step on one stream (default: two streams, see run_ours)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--kernel-case", default=None,
                    help="run one kernel alone (for ncu captures; a group_ prefix on a quant_ case runs it "
                         "as one grouped call over A- and W-shaped tensors): quant_mxfp4_row, quant_nvfp4_row, "
                         "quant_mxfp4_col, quant_mxfp4_2d, quant_had32_row, quant_mbs_oas_row, "
                         "dequant_mxfp4_row, gemm_mxfp4, gemm_nvfp4, gemm_qsnr_mxfp4, gemm_qsnr_nvfp4")
    ap.add_argument("--rows", type=int, default=16384)
    ap.add_argument("--cols", type=int, default=8192)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--no-stats", action="store_true", help="kernel cases: quantize without the fused stats")
    return ap.parse_args()


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return d, "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


# --------------------------------------------------------------- the step --
def step_plan(mx):
    """(name, tensor, config, kind) for every launch of one step."""
    mxfp4 = mx.MXFP4
    nvfp4 = mx.NVFP4
    had = mx.Config(hadamard=32)
    mbs = mx.Config(macro_block=128, rule=mx.RULE_OAS, oas_tau=7.0)
    return [
        ("mxfp4_row", "A", mxfp4, "q"), ("mxfp4_row", "W", mxfp4, "q"),
        ("nvfp4_row", "A", nvfp4, "q"), ("nvfp4_row", "W", nvfp4, "q"),
        ("had32_mxfp4", "A", had, "q"), ("had32_mxfp4", "W", had, "q"),
        ("mbs_oas_mxfp4", "A", mbs, "q"), ("mbs_oas_mxfp4", "W", mbs, "q"),
        ("dequant_mxfp4_bf16", "A", mxfp4, "d"), ("dequant_mxfp4_bf16", "W", mxfp4, "d"),
    ]


def step_calls(plan):
    """The step's calls: each quantizer variant as one grouped call over its
    tensors (A and W share the launch), each dequantizer one call per tensor.
    (name, tensors, config, kind), in plan order."""
    calls, seen = [], {}
    for name, t, cfg, kind in plan:
        if kind == "q":
            if name in seen:
                seen[name][1].append(t)
                continue
            seen[name] = (name, [t], cfg, kind)
            calls.append(seen[name])
        else:
            calls.append((name, [t], cfg, kind))
    return [(n, tuple(ts), c, k) for n, ts, c, k in calls]


def algo_bytes(cfg, rows, cols, kind, in_bytes=2):
    n = rows * cols
    code = n if cfg.elem in (2, 3) else n // 2
    nb = n // cfg.block if cfg.axis != 2 else n // 1024
    macro = n // 128 if cfg.macro_block else 0
    offs = 2 * nb if cfg.asymmetric else 0
    if kind == "q":
        return in_bytes * n + code + nb + macro + offs
    return code + nb + macro + offs + 2 * n       # dequantize to bf16


def launches_per_call(cfg, kind, ntensors=1):
    if kind == "d":
        return ntensors                    # one dequantizer launch per tensor
    groups = (ntensors + 3) // 4           # a grouped launch takes up to 4 tensors
    k = groups                             # quantize (the last CTA of each tensor sums its statistics)
    if cfg.tensor_scale == 1:
        k += groups                        # tensor-amax pre-pass
    return k


class ClockSampler:
    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={q}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = []
        try:
            with open(self.path) as f:
                for ln in f:
                    parts = [p.strip() for p in ln.split(",")]
                    if len(parts) >= 9:
                        rows.append(parts)
        except OSError:
            pass
        finally:
            if self.path:
                os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx_ = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx_) if mx_ else None, "reasons": reasons,
                "samples": len(rows)}


def traffic_record(kernel_key: str):
    """dram read+write bytes per launch from the committed ncu summary, or None
    when the kernel sources changed since it was taken."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel_key)
    except (OSError, ValueError):
        return None
    if not rec:
        return None
    h = hashlib.sha256()
    for rel in rec.get("sources", []):
        try:
            with open(os.path.join(ROOT, rel), "rb") as f:
                h.update(f.read())
        except OSError:
            return None
    if h.hexdigest()[:16] != rec.get("sources_sha256_16"):
        return None
    return rec.get("bytes_per_launch")


# ------------------------------------------------------------ our arm ------
def run_ours(args, rank, world, device):
    import microscaling_block_quantization_b200 as mx
    from microscaling_block_quantization_b200 import inputs

    A_cpu, W_cpu = inputs.llama_linear(M_TOK, K_DIM, N_OUT)
    A = A_cpu.to(device)
    W = W_cpu.to(device)
    T = {"A": A, "W": W}
    plan = step_plan(mx)
    stream = torch.cuda.current_stream(device)

    # pre-allocated outputs per launch (no allocation inside the timed region)
    outs = {}
    for name, t, cfg, kind in plan:
        key = (name, t)
        x = T[t]
        if kind == "q":
            outs[key] = mx.alloc_outputs(cfg, *x.shape, device, stats=True)
        else:
            src = outs[("mxfp4_row", t)]
            outs[key] = torch.empty(x.shape, dtype=torch.bfloat16, device=device)
            outs[(key, "src")] = src

    calls = step_calls(plan)
    # each stream owns a workspace per tensor: concurrent calls, and the
    # tensors of one grouped call, must not share control words
    wss = {(sd, t): mx.new_workspace(mx.MXFP4, *A.shape, device) for sd in ("main", "side") for t in T}

    def run_call(name, ts, cfg, kind, stream=None, wsk="main"):
        # stream=None: the current stream, i.e. the capture stream inside a graph
        if kind == "q":
            mx.quantize_group([T[t] for t in ts], cfg, outs=[outs[(name, t)] for t in ts], stream=stream,
                              workspaces=[wss[(wsk, t)] for t in ts])
        else:
            for t in ts:
                mx.dequantize(outs[((name, t), "src")], out=outs[(name, t)], stream=stream)

    # The step's launches are independent problems except that each
    # dequantizer reads the MXFP4 codes of its tensor.  They are captured on
    # two streams so that HBM-bound work (the NVFP4 tensor-amax passes, the
    # dequantizers) overlaps issue-bound quantizers: the MXFP4 / rotated / MBS
    # quantizers on the capture stream, NVFP4 and the dequantizers (after an
    # event on their codes) on a side stream, each stream with its own
    # workspace.
    side = torch.cuda.Stream(device)
    SIDE = {"nvfp4_row", "dequant_mxfp4_bf16"}

    def run_step():
        if args.one_stream:
            for call in calls:
                run_call(*call)
            return
        main = torch.cuda.current_stream(device)
        fork = torch.cuda.Event()
        fork.record(main)
        side.wait_event(fork)
        codes_ready = None
        for call in calls:
            name, ts, cfg, kind = call
            if name in SIDE:
                if kind == "d":
                    side.wait_event(codes_ready)
                with torch.cuda.stream(side):
                    run_call(*call, stream=side, wsk="side")
            else:
                run_call(*call)
                if name == "mxfp4_row":
                    codes_ready = torch.cuda.Event()
                    codes_ready.record(main)
        join = torch.cuda.Event()
        join.record(side)
        main.wait_event(join)

    step_bytes = sum(algo_bytes(cfg, *T[t].shape, kind) for _, t, cfg, kind in plan)
    launches = sum(launches_per_call(cfg, kind, len(ts)) for _, ts, cfg, kind in calls)

    # eager warm-up (caches kernel attributes)
    for _ in range(max(1, args.warmup)):
        run_step()
    torch.cuda.synchronize(device)

    # the step captured as a CUDA graph: the kernels run back to back with no
    # host work between them.  Per variant, a graph of R_PAIRS back-to-back
    # repeats of its call on A and W (one stream, the step's launch
    # configuration: one grouped quantizer launch over both tensors); the two
    # tensors together (176 MiB) are larger than L2, so no input comes from
    # L2, and the time over the repeats is the steady-state call duration
    # without graph-launch gaps
    step_graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(step_graph):
        run_step()
    variants = list(dict.fromkeys(name for name, _, _, _ in plan))
    pair_graphs = {}
    for name in variants:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(R_PAIRS):
                for call in calls:
                    if call[0] == name:
                        run_call(*call)
        pair_graphs[name] = g
    # NVFP4's quantizer launch alone (k_quant_fast without the tensor-amax
    # launch before it): the same grouped launch with each tensor's tensor
    # scale given (the values the step computes), into separate outputs
    nv_name, nv_ts, nv_cfg, _ = next(c for c in calls if c[0] == "nvfp4_row")
    nv_given = dataclasses.replace(nv_cfg, tensor_scale=mx.TS_GIVEN)
    nv_outs = [mx.alloc_outputs(nv_given, *T[t].shape, device, stats=True,
                                tensor_scale=outs[(nv_name, t)].tensor_scale.clone()) for t in nv_ts]
    nv_wss = [mx.new_workspace(nv_given, *T[t].shape, device) for t in nv_ts]

    def nv_quantizer_only():
        mx.quantize_group([T[t] for t in nv_ts], nv_given, outs=nv_outs, workspaces=nv_wss)
    nv_quantizer_only()
    torch.cuda.synchronize(device)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _ in range(R_PAIRS):
            nv_quantizer_only()
    pair_graphs["nvfp4_row_quantizer"] = g
    for _ in range(args.warmup):
        step_graph.replay()
    torch.cuda.synchronize(device)

    # timed region: exactly K steps between CUDA events on the replay stream
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(device.index) as clk:
        # the timed region is milliseconds long, shorter than the sampling
        # period: the GPU is held under the same load for about a second just
        # before it, so the clock samples describe the clocks it runs at
        t_soak = time.time()
        while time.time() - t_soak < 1.0:
            for _ in range(50):
                step_graph.replay()
            torch.cuda.synchronize(device)
        if world > 1:
            torch.distributed.barrier()
        torch.cuda.synchronize(device)
        start.record(stream)
        for s in range(args.steps):
            step_graph.replay()
        stop.record(stream)
        torch.cuda.synchronize(device)
    elapsed_ms = start.elapsed_time(stop)
    if world > 1:
        t = torch.tensor([elapsed_ms], device=device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        elapsed_ms = float(t.item())
        torch.distributed.barrier()
    ms_per_step = elapsed_ms / args.steps
    value = world * step_bytes / (ms_per_step * 1e-3) / 1e9

    # per-variant device time (A + W launches) from its pair graph
    rows = {}
    for name in variants + ["nvfp4_row_quantizer"]:
        g = pair_graphs[name]
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize(device)
        src = "nvfp4_row" if name == "nvfp4_row_quantizer" else name
        nb = sum(algo_bytes(cfg, *T[t].shape, kind) for n, t, cfg, kind in plan if n == src)
        ms = e0.elapsed_time(e1) / (args.steps * R_PAIRS)
        rows[name] = {"bytes": nb, "GB_per_s": round(nb / (ms * 1e-3) / 1e9, 1), "us": round(ms * 1e3, 2)}
    del pair_graphs

    pk, pk_src = peaks()
    # the dominant kernel of the step: k_quant_fast, the four grouped
    # quantizer launches over A and W, each timed alone (NVFP4's quantizer
    # launch without the tensor-amax launch, a separate kernel, before it);
    # the same with NVFP4's whole call (amax launch included) beside it
    qnames = ["mxfp4_row", "nvfp4_row_quantizer", "had32_mxfp4", "mbs_oas_mxfp4"]
    qnames_call = ["mxfp4_row", "nvfp4_row", "had32_mxfp4", "mbs_oas_mxfp4"]
    qbytes = sum(rows[n]["bytes"] for n in qnames)
    qus = sum(rows[n]["us"] for n in qnames)
    achieved = round(qbytes / (qus * 1e-6) / 1e9, 1)
    achieved_call = round(qbytes / (sum(rows[n]["us"] for n in qnames_call) * 1e-6) / 1e9, 1)
    traffic = traffic_record("mxfp4_row_AW")
    roofline = {"bound": "hbm",
                "kernel": "k_quant_fast (TMA-fed E2M1 quantizer, statistics summed by the last CTA of each "
                          "tensor): the step's 4 grouped launches, MXFP4 / NVFP4 / rotation-32 / MBS+OAS, "
                          "each over A and W, each launch timed alone (NVFP4's tensor-amax pre-pass is a "
                          "separate kernel, k_amax_vec: see achieved_with_amax_pass)",
                "achieved": achieved, "peak": pk["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / pk["hbm_gbs"], 4), "peak_source": pk_src,
                "achieved_with_amax_pass": achieved_call,
                "frac_with_amax_pass": round(achieved_call / pk["hbm_gbs"], 4),
                "traffic": traffic,
                "traffic_launch": "the grouped MXFP4 launch on A and W (dram read + write per launch, from the "
                                  "ncu capture of the 16384 x 8192 case scaled by elements)",
                "traffic_launch_algorithmic_bytes": algo_bytes(mx.MXFP4, M_TOK, K_DIM, "q")
                                                    + algo_bytes(mx.MXFP4, N_OUT, K_DIM, "q"),
                "algorithmic_bytes_per_step": qbytes,
                "by_variant_frac": {n: round(rows[n]["GB_per_s"] / pk["hbm_gbs"], 4) for n in qnames_call + ["nvfp4_row_quantizer"]}}

    extra = run_extra_rows(mx, A, W, device, args)
    try:
        extra["c2_block_size_sweep"] = run_c2_sweep(mx, device, args)
    except Exception as e:        # reported, not fatal: the headline step stands on its own
        extra["c2_block_size_sweep"] = {"unavailable": f"{type(e).__name__}: {e}"}

    # end to end through the public API with host buffers
    e2e = run_e2e(mx, A_cpu, W_cpu, plan, calls, wss, device, args, step_bytes, world)

    # fidelity of the step (sanity: the stats the kernels produced)
    fid = {f"{name}_{t}_qsnr_db": round(float(outs[(name, t)].stats[7].item()), 4)
           for name, t, cfg, kind in plan if kind == "q"}

    gemm = None if args.no_gemm else run_gemm(mx, A, W, device, args, world)
    return dict(value=value, ms_per_step=ms_per_step, step_bytes=step_bytes, launches=launches,
                rows=rows, roofline=roofline, e2e=e2e, fidelity=fid, gemm=gemm,
                clocks=dict(clk.summary(), window="1 s of step replays just before the timed region, "
                                                  "and the timed region"), extra=extra)


GRAD_ROWS, GRAD_COLS, GRAD_SEED = 4096, 14336, 5      # the fp32 gradient-like tensor of the extra rows


def extra_row_cases(mx):
    """(row name, tensors, config) of the extra rows: "A"/"W" the layer's
    operands (quantized together in one grouped call), "G" the fp32
    gradient-like tensor."""
    return [("mxfp4_col_AW", ("A", "W"), mx.Config(axis=1)), ("mxfp4_2d_AW", ("A", "W"), mx.Config(axis=2)),
            ("e2m1_sr_grad_fp32", ("G",), mx.Config(round=mx.ROUND_STOCHASTIC, seed=5)),
            ("e2m3_grad_fp32", ("G",), mx.Config(elem=mx.E2M3)),
            ("int4_asym_grad_fp32", ("G",), mx.Config(elem=mx.INT4, asymmetric=1, rule=mx.RULE_CEIL)),
            ("e3m0_ceil_grad_fp32", ("G",), mx.Config(elem=mx.E3M0, rule=mx.RULE_CEIL))]


def run_extra_rows(mx, A, W, device, args):
    """The other rows of the path, outside the headline step: column and 2D
    blocks on the layer's A and W (one grouped call over both), and on a
    gradient-like fp32 4096 x 14336 tensor stochastic rounding, FP6,
    asymmetric INT4 and E3M0 with the ceil scale.  Each row is a graph of
    R_PAIRS back-to-back calls (A and W together, and the 224 MiB gradient,
    are larger than L2, so no input is served from L2), replayed K times."""
    from microscaling_block_quantization_b200 import inputs
    G = inputs.gradient_like(GRAD_ROWS, GRAD_COLS, seed=GRAD_SEED).to(device)
    tens = {"A": A, "W": W, "G": G}
    cases = [(name, tuple(tens[t] for t in ts), cfg) for name, ts, cfg in extra_row_cases(mx)]
    out = {}
    stream = torch.cuda.current_stream(device)
    for name, xs, cfg in cases:
        qs = [mx.alloc_outputs(cfg, *x.shape, device, stats=True) for x in xs]
        wss = [mx.new_workspace(cfg, *x.shape, device) for x in xs]

        def call():
            # A and W in one grouped call (one launch), a single tensor alone
            if len(xs) > 1:
                mx.quantize_group(list(xs), cfg, outs=qs, workspaces=wss)
            else:
                mx.quantize(xs[0], cfg, out=qs[0], workspace=wss[0])
        call()
        torch.cuda.synchronize(device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for _ in range(R_PAIRS):
                call()
        g.replay()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            g.replay()
        e1.record(stream)
        torch.cuda.synchronize(device)
        ms = e0.elapsed_time(e1) / (args.steps * R_PAIRS)
        nb = sum(algo_bytes(cfg, *x.shape, "q", in_bytes=x.element_size()) for x in xs)
        out[name] = {"GB_per_s": round(nb / (ms * 1e-3) / 1e9, 1), "us": round(ms * 1e3, 2),
                     "qsnr_db": round(float(qs[0].stats[7].item()), 4), "bias": float(qs[0].stats[8].item())}
    del G
    return out


def run_c2_sweep(mx, device, args):
    """The block-size sweep of "Is Finer Better?": 4096 x 4096 weight-like
    N(0, sigma) tensors, sigma in {0.002, 0.02, 0.2} (seeds 1, 2, 3), E2M1
    with UE4M3 / UE5M3 nearest block scales, without and with the FP32 tensor
    scale, blocks 8 ... 256.  Per configuration: the per-tensor MSE at each
    sigma, and the quantize call's GB/s (tensor-amax pass included) with a
    cold L2: each timed call follows a read of a 256 MiB buffer, and is timed
    between event nodes of a graph on either side of it."""
    from microscaling_block_quantization_b200 import inputs
    sigmas = (0.002, 0.02, 0.2)
    xs = [inputs.normal(4096, 4096, sigma=sg, seed=i + 1).to(device) for i, sg in enumerate(sigmas)]
    evict = torch.ones(64 << 20, dtype=torch.float32, device=device)    # 256 MiB, read to evict L2
    stream = torch.cuda.current_stream(device)
    out = {}
    for fmt, fname in ((mx.SCALE_UE4M3, "UE4M3"), (mx.SCALE_UE5M3, "UE5M3")):
        for ts in (0, 1):
            for B in (8, 16, 32, 64, 128, 256):
                cfg = mx.Config(block=B, scale_fmt=fmt, rule=mx.RULE_NEAREST, tensor_scale=ts)
                ws = mx.new_workspace(cfg, 4096, 4096, device)
                qs = [mx.alloc_outputs(cfg, 4096, 4096, device, stats=True) for _ in xs]
                for x, q in zip(xs, qs):
                    mx.quantize(x, cfg, out=q, workspace=ws)
                torch.cuda.synchronize(device)
                rec = {"mse": {str(sg): float(q.stats[5].item()) for sg, q in zip(sigmas, qs)}}
                evs = [(torch.cuda.Event(enable_timing=True, external=True),
                        torch.cuda.Event(enable_timing=True, external=True)) for _ in xs]
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    for (ea, eb), x, q in zip(evs, xs, qs):
                        evict.sum()
                        ea.record()
                        mx.quantize(x, cfg, out=q, workspace=ws)
                        eb.record()
                ms = 0.0
                n = max(3, args.steps // 2)
                for _ in range(n + 1):
                    g.replay()
                    torch.cuda.synchronize(device)
                    if _ == 0:
                        continue
                    ms += sum(ea.elapsed_time(eb) for ea, eb in evs) / len(evs)
                ms /= n
                nb = algo_bytes(cfg, 4096, 4096, "q")
                rec["GB_per_s"] = round(nb / (ms * 1e-3) / 1e9, 1)
                rec["us"] = round(ms * 1e3, 2)
                out[f"{fname}_ts{ts}_B{B}"] = rec
                del g
    del evict
    return out


def run_e2e(mx, A_cpu, W_cpu, plan, calls, wss, device, args, step_bytes, world):
    """Same step through the public API, inputs copied from pinned host memory
    and the codes, scales and stats read back, inside the timed region.  The
    copies run on their own streams, and the device inputs and outputs are
    double-buffered: step i+1's inputs come in and its calls run while step
    i's results go out (PCIe is full duplex).  Events order every reuse of a
    device buffer."""
    compute = torch.cuda.current_stream(device)
    h2d, d2h = torch.cuda.Stream(device), torch.cuda.Stream(device)
    host = {"A": A_cpu.pin_memory(), "W": W_cpu.pin_memory()}
    bufs = []
    for _ in range(2):
        T = {t: torch.empty_like(h, device=device) for t, h in host.items()}
        o = {(name, t): mx.alloc_outputs(cfg, *T[t].shape, device, stats=True)
             for name, t, cfg, kind in plan if kind == "q"}
        back = [(d, torch.empty(d.shape, dtype=d.dtype).pin_memory())
                for q in o.values() for d in (q.codes, q.scales, q.stats)]
        deq = {(name, t): torch.empty(T[t].shape, dtype=torch.bfloat16, device=device)
               for name, t, cfg, kind in plan if kind == "d"}
        bufs.append({"T": T, "outs": o, "back": back, "deq": deq, "in": None, "done": None, "out": None})
    h2d_bytes = sum(h.numel() * h.element_size() for h in host.values())
    d2h_bytes = sum(d.numel() * d.element_size() for d, _ in bufs[0]["back"])
    it = [0]

    def one():
        b = bufs[it[0] % 2]
        it[0] += 1
        if b["done"] is not None:
            h2d.wait_event(b["done"])                    # this buffer's previous step has read its inputs
        with torch.cuda.stream(h2d):
            for t, h in host.items():
                b["T"][t].copy_(h, non_blocking=True)
        b["in"] = torch.cuda.Event()
        b["in"].record(h2d)
        compute.wait_event(b["in"])
        if b["out"] is not None:
            compute.wait_event(b["out"])                 # this buffer's previous results are on the host
        for name, ts, cfg, kind in calls:
            if kind == "q":
                mx.quantize_group([b["T"][t] for t in ts], cfg, outs=[b["outs"][(name, t)] for t in ts],
                                  stream=compute, workspaces=[wss[("main", t)] for t in ts])
            else:
                for t in ts:
                    mx.dequantize(b["outs"][("mxfp4_row", t)], out=b["deq"][(name, t)], stream=compute)
        b["done"] = torch.cuda.Event()
        b["done"].record(compute)
        d2h.wait_event(b["done"])
        with torch.cuda.stream(d2h):
            for d, h in b["back"]:
                h.copy_(d, non_blocking=True)
        b["out"] = torch.cuda.Event()
        b["out"].record(d2h)

    def drain():
        for b in bufs:
            if b["out"] is not None:
                compute.wait_event(b["out"])

    steps = max(3, args.steps // 4)
    for _ in range(2):
        one()
    drain()
    torch.cuda.synchronize(device)
    if world > 1:
        torch.distributed.barrier()
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(compute)
    h2d.wait_event(s)
    for _ in range(steps):
        one()
    drain()
    e.record(compute)
    torch.cuda.synchronize(device)
    ms = s.elapsed_time(e) / steps
    if world > 1:
        t = torch.tensor([ms], device=device)
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
        ms = float(t.item())
    return {"value": round(world * step_bytes / (ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "h2d_bytes_per_step": h2d_bytes, "d2h_bytes_per_step": d2h_bytes, "ms_per_step": round(ms, 3),
            "steps": steps,
            "overlap": "copy-in, compute and copy-out on three streams with double-buffered device inputs and "
                       "outputs (a step's results go out while the next step's inputs come in and its calls run)"}


def tensor_ceilings(mx, device, iters=100000):
    """Measured tensor-core ceiling of each block-scaled MMA kind on this GPU
    (mx_tensor_peak: every SM issues 128 x 256 MMAs on operands held in shared
    memory): MMAs alone, and with the per-stage scale copies into tensor
    memory rotating over four slots as the GEMM does.  Best of three launches."""
    stream = torch.cuda.current_stream(device)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    out = {}
    for kind, name in ((1, "mxf4"), (2, "mxf4nvf4"), (3, "mxf8f6f4")):
        rec = {}
        for sfc, key in ((0, "mma_only"), (2, "with_scale_copies")):
            mx.tensor_peak(kind, 2000, sfc, stream=stream)
            torch.cuda.synchronize(device)
            best = 0.0
            for _ in range(3):
                s.record(stream)
                f = mx.tensor_peak(kind, iters, sfc, stream=stream)
                e.record(stream)
                torch.cuda.synchronize(device)
                best = max(best, f / (s.elapsed_time(e) * 1e-3) / 1e12)
            rec[key] = round(best, 1)
        out[name] = rec
    out["unit"] = "TFLOP/s"
    return out


def run_gemm(mx, A, W, device, args, world):
    """Block-scaled GEMM C = A^Q W^Q^T (MXFP4, NVFP4, MBS operands on the NVFP4
    kind, MXFP6, MXFP6 activations with MXFP4 weights, Hadamard-rotated MXFP4,
    NVFP4 with MSE-optimised scales) and QSNR(AB)."""
    out = {}
    pk, pk_src = peaks()
    stream = torch.cuda.current_stream(device)
    flop = 2.0 * M_TOK * N_OUT * K_DIM
    ceil = tensor_ceilings(mx, device)
    out["tensor_ceiling"] = ceil
    mbs = mx.Config(macro_block=128)
    fp4 = mx.Config(sf_layout=1)
    nv = mx.Config(block=16, scale_fmt=1, rule=3, tensor_scale=1, sf_layout=1)
    nv_mse = mx.Config(block=16, scale_fmt=1, rule=mx.RULE_MSE, tensor_scale=1, sf_layout=1)
    for name, cfg, cfg_w in (("mxfp4", fp4, fp4),
                             ("nvfp4", nv, nv),
                             ("mbs_mxfp4_via_nvf4", mbs, mbs),
                             ("mxfp6_e2m3", mx.Config(elem=mx.E2M3, sf_layout=1), mx.Config(elem=mx.E2M3, sf_layout=1)),
                             ("mxfp6_e2m3_x_mxfp4", mx.Config(elem=mx.E2M3, sf_layout=1), fp4),
                             ("had32_mxfp4", mx.Config(hadamard=32, sf_layout=1), mx.Config(hadamard=32, sf_layout=1)),
                             ("nvfp4_mse_scales", nv_mse, nv_mse)):
        qa = mx.quantize(A, cfg, stats=False)
        if cfg_w.rule == mx.RULE_MSE:
            # the alternating global / group scale search on W: an offline
            # weight step, timed once here (not part of the GEMM time)
            torch.cuda.synchronize(device)
            s0, e0 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s0.record(stream)
            qw = mx.quantize(W, cfg_w, stats=False)
            e0.record(stream)
            torch.cuda.synchronize(device)
            mse_quant_ms = s0.elapsed_time(e0)
        else:
            qw = mx.quantize(W, cfg_w, stats=False)
        if cfg.macro_block:
            # Macro Block Scaling operands: S_M X folded into UE4M3 16-element
            # scales, the GEMM's NVFP4 kind (the fold is outside the timed GEMM)
            qa, qw = mx.mbs_gemm_operand(qa), mx.mbs_gemm_operand(qw)
        C = torch.empty((M_TOK, N_OUT), dtype=torch.bfloat16, device=device)
        try:
            mx.gemm(qa, qw, out=C)
        except mx.MXError as e:
            out[name] = {"unavailable": str(e)}
            continue
        for _ in range(args.warmup):
            mx.gemm(qa, qw, out=C)
        torch.cuda.synchronize(device)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            mx.gemm(qa, qw, out=C)
        g.replay()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        steps = max(5, args.steps)
        s.record(stream)
        for _ in range(steps):
            g.replay()
        e.record(stream)
        torch.cuda.synchronize(device)
        ms = s.elapsed_time(e) / steps
        tf = flop / (ms * 1e-3) / 1e12
        # the peak is the kind's measured tensor ceiling on this device (MMAs
        # on shared-memory operands, no global traffic); bf16 x the nominal
        # dense ratio (FP6 runs at the FP8 rate: 2x; FP4 4x) is kept as context
        fp6 = mx.E2M3 in (cfg.elem, cfg_w.elem) or mx.E3M2 in (cfg.elem, cfg_w.elem)
        ratio = 2.0 if fp6 else 4.0
        kind = "mxf8f6f4" if fp6 else ("mxf4nvf4" if (cfg.block == 16 or cfg.macro_block) else "mxf4")
        peak = ceil[kind]["mma_only"]
        rec = {"TFLOPS": round(tf, 1), "ms": round(ms, 4), "unit": "TFLOP/s", "kind": kind,
               "roofline": {"bound": "tensor", "achieved": round(tf, 1), "peak": round(peak, 1),
                            "unit": "TFLOP/s", "frac": round(tf / peak, 4),
                            "peak_source": f"measured kind::{kind} ceiling (mx_tensor_peak, this run)",
                            "frac_of_ceiling_with_scale_copies": round(tf / ceil[kind]["with_scale_copies"], 4),
                            "frac_of_bf16_x_nominal_ratio": round(tf / (pk["bf16_tflops"] * ratio), 4)}}
        try:
            st = mx.gemm_qsnr(A, W, qa, qw)
            torch.cuda.synchronize(device)
            s.record(stream)
            st = mx.gemm_qsnr(A, W, qa, qw)
            e.record(stream)
            torch.cuda.synchronize(device)
            rec["qsnr_ab_db"] = round(float(st[2].item()), 4)
            rec["qsnr_ab_ms"] = round(s.elapsed_time(e), 3)
            rec["device_status"] = mx.mx_device_status()
        except mx.MXError as e:
            rec["qsnr_ab"] = f"unavailable: {e}"
        if cfg_w.rule == mx.RULE_MSE:
            rec["w_quantize_ms"] = round(mse_quant_ms, 3)
            rec["w_quantize_note"] = "alternating global / group scale search on W (4 rounds + writing pass), once"
        out[name] = rec
    if "mxfp4" in out and "TFLOPS" in out.get("mbs_mxfp4_via_nvf4", {}):
        # the pages quote MBS's GEMM overhead against plain MXFP4
        out["mbs_mxfp4_via_nvf4"]["overhead_vs_mxfp4"] = round(
            out["mbs_mxfp4_via_nvf4"]["ms"] / out["mxfp4"]["ms"] - 1.0, 4)
    return out


# ------------------------------------------------------------ CPU oracle ---
_LAYER_CPU = {}


def oracle_sample(rows_a=512, rows_w=512, row0=0):
    """The oracle on a bounded sample of the step: rows row0.. of A and W
    through every launch of the step (same configs)."""
    import oracle as O
    import microscaling_block_quantization_b200 as mx
    from microscaling_block_quantization_b200 import inputs

    if not _LAYER_CPU:
        _LAYER_CPU["A"], _LAYER_CPU["W"] = inputs.llama_linear(M_TOK, K_DIM, N_OUT)
    A, W = _LAYER_CPU["A"], _LAYER_CPU["W"]
    T = {"A": A[row0:row0 + rows_a], "W": W[row0:row0 + rows_w]}
    plan = step_plan(mx)

    def ocfg(c):
        return O.Cfg(elem=c.elem, scale_fmt=c.scale_fmt, rule=c.rule, oas_tau=c.oas_tau,
                     block=c.block, axis=c.axis, round_mode=c.round, asymmetric=c.asymmetric,
                     tensor_scale=c.tensor_scale, macro_block=c.macro_block, hadamard=c.hadamard,
                     seed=c.seed)

    nbytes = sum(algo_bytes(cfg, *T[t].shape, kind) for _, t, cfg, kind in plan)

    def run():
        keep = {}
        for name, t, cfg, kind in plan:
            oc = ocfg(cfg)
            if kind == "q":
                r = O.quantize(oc, T[t])
                xh = O.dequantize(oc, r["packed"], r["scales"], r["tensor_scale"], r["macro"],
                                  r["offsets"], *T[t].shape)
                O.stats(r["y"], xh)
                keep[(name, t)] = r
            else:
                r = keep[("mxfp4_row", t)]
                O.dequantize(oc, r["packed"], r["scales"], None, None, None, *T[t].shape)
    return run, nbytes, f"first {rows_a} rows of A and {rows_w} rows of W through every launch of the step"


def host_cpu():
    """(logical cores, CPU model) of this host."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for ln in f:
                if ln.startswith("model name"):
                    model = ln.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return os.cpu_count() or 1, model


def _oracle_band(band):
    """One worker of the all-cores leg: the oracle, unchanged, on a band of
    rows of A and W through every launch of the step (a spawned process)."""
    from microscaling_block_quantization_b200 import inputs
    lo, hi = band
    if not _LAYER_CPU or _LAYER_CPU["A"].shape[0] < hi:
        # the first hi rows of the layer (numpy's streams are drawn in row order)
        _LAYER_CPU["A"], _LAYER_CPU["W"] = inputs.llama_linear(hi, K_DIM, hi)
    run, nbytes, _ = oracle_sample(rows_a=hi - lo, rows_w=hi - lo, row0=lo)
    run()
    return nbytes


def cpu_baseline(target_s=10.0):
    """The oracle as it stands on the host cores: one thread on the first 512
    rows of A and W, and all cores as independent processes, each running the
    unchanged oracle on its own band of rows (the oracle has no threading of
    its own; blocks are independent, so the bands need no exchange)."""
    import multiprocessing as mp
    cores, model = host_cpu()
    run, nbytes, sample = oracle_sample()
    t0 = time.perf_counter()
    run()
    one = time.perf_counter() - t0
    reps = max(1, int(target_s / max(one, 1e-3)))
    t0 = time.perf_counter()
    for _ in range(reps):
        run()
    dt = (time.perf_counter() - t0) / reps
    single = nbytes / dt / 1e9
    out = {"value": round(single, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
           "sample": f"{sample}; {reps} repetitions, {dt:.3f} s each, single-threaded scalar C",
           "host": {"logical_cores": cores, "cpu_model": model}}
    # all cores: one spawned process per core, 256 rows of A and W each
    rows = 256
    bands = [(i * rows, (i + 1) * rows) for i in range(cores)]
    try:
        ctx = mp.get_context("spawn")
        with ctx.Pool(cores) as pool:
            pool.map(_oracle_band, bands[:cores])          # import and build once per worker
            t0 = time.perf_counter()
            total = sum(pool.map(_oracle_band, bands))
            dt_all = time.perf_counter() - t0
        out["all_cores"] = {"value": round(total / dt_all / 1e9, 4), "unit": "GB/s", "cores": cores,
                            "sample": f"{cores} processes x (256 rows of A and of W through every launch of "
                                      f"the step), {dt_all:.3f} s"}
    except Exception as e:  # the single-thread figure stands on its own
        out["all_cores"] = {"unavailable": f"{type(e).__name__}: {e}"}
    return out


def run_reference(args, rank, world):
    """--impl reference: the CPU oracle, as it stands, on the host cores; each
    step a bounded sample of the workload."""
    if rank != 0:
        return None
    cores, model = host_cpu()
    run, nbytes, sample = oracle_sample(rows_a=256, rows_w=256)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    dt = (time.perf_counter() - t0) / args.steps
    value = nbytes / dt / 1e9
    return {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": sample},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": sample, "host": {"logical_cores": cores, "cpu_model": model}},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


def kernel_case(args):
    """One kernel on one synthetic tensor, `reps` times, each timed with CUDA
    events; the default 16384 x 8192 bf16 input (256 MiB) is larger than L2."""
    import microscaling_block_quantization_b200 as mx
    dev = torch.device("cuda", 0)
    g = torch.Generator(device=dev).manual_seed(0)
    case = args.kernel_case
    res = {"case": case, "stats": not args.no_stats}
    if case.startswith("gemm"):
        M, N, K = M_TOK, N_OUT, K_DIM
        qsnr = case.startswith("gemm_qsnr")
        case = case.replace("gemm_qsnr", "gemm")
        cfg = {"gemm_mxfp4": mx.Config(sf_layout=1),
               "gemm_nvfp4": mx.Config(block=16, scale_fmt=1, rule=3, tensor_scale=1, sf_layout=1),
               "gemm_mxfp6": mx.Config(elem=mx.E2M3, sf_layout=1),
               "gemm_mxfp6_x_mxfp4": mx.Config(elem=mx.E2M3, sf_layout=1)}[case]
        cfg_w = mx.Config(sf_layout=1) if case == "gemm_mxfp6_x_mxfp4" else cfg
        a = torch.randn(M, K, generator=g, device=dev).to(torch.bfloat16)
        w = (torch.randn(N, K, generator=g, device=dev) * 0.02).to(torch.bfloat16)
        qa, qw = mx.quantize(a, cfg, stats=False), mx.quantize(w, cfg_w, stats=False)
        c = torch.empty(M, N, dtype=torch.bfloat16, device=dev)
        if qsnr:
            # QSNR(AB): the block-scaled and the bf16 product, C not written
            a16, w16 = a.to(torch.bfloat16), w.to(torch.bfloat16)
            run = lambda: mx.gemm_qsnr(a16, w16, qa, qw)
            work, unit = 4.0 * M * N * K / 1e12, "TFLOP/s (both products)"
        else:
            run = lambda: mx.gemm(qa, qw, out=c)
            work, unit = 2.0 * M * N * K / 1e12, "TFLOP/s"
    else:
        # group_<case>: the quantizer case as one grouped call over the layer's
        # A-shaped and W-shaped tensors
        group = case.startswith("group_")
        if group:
            case = case[len("group_"):]
        R, Cc = args.rows, args.cols
        cfg = {"quant_mxfp4_row": mx.MXFP4, "quant_nvfp4_row": mx.NVFP4,
               "quant_mxfp4_col": mx.Config(axis=1), "quant_mxfp4_2d": mx.Config(axis=2),
               "quant_had32_row": mx.Config(hadamard=32), "dequant_mxfp4_row": mx.MXFP4,
               "quant_mbs_oas_row": mx.Config(macro_block=128, rule=mx.RULE_OAS, oas_tau=7.0),
               "quant_e2m1_sr_grad": mx.Config(round=mx.ROUND_STOCHASTIC, seed=5),
               "quant_e2m3_grad": mx.Config(elem=mx.E2M3),
               "quant_int4_asym_grad": mx.Config(elem=mx.INT4, asymmetric=1, rule=mx.RULE_CEIL),
               "quant_e3m0_ceil_grad": mx.Config(elem=mx.E3M0, rule=mx.RULE_CEIL),
               "quant_nvfp4_mse_row": mx.Config(block=16, scale_fmt=1, rule=mx.RULE_MSE, tensor_scale=1)}[case]
        if group:
            xs = [torch.randn(r, K_DIM, generator=g, device=dev).to(torch.bfloat16) for r in (M_TOK, N_OUT)]
            qs = mx.quantize_group(xs, cfg, stats=not args.no_stats)
            run = lambda: mx.quantize_group(xs, cfg, outs=qs)
            nbytes = sum(algo_bytes(cfg, *t.shape, "q") for t in xs)
        else:
            x = torch.randn(R, Cc, generator=g, device=dev)
            # gradient-like cases quantize binary32 input, the others bf16
            x = x * 1e-3 if case.endswith("_grad") else x.to(torch.bfloat16)
            q = mx.quantize(x, cfg, stats=not args.no_stats)
            if case.startswith("dequant"):
                out = torch.empty(R, Cc, dtype=torch.bfloat16, device=dev)
                run = lambda: mx.dequantize(q, out=out)
                kind = "d"
            else:
                run = lambda: mx.quantize(x, cfg, out=q)
                kind = "q"
            nbytes = algo_bytes(cfg, R, Cc, kind, in_bytes=x.element_size())
        work, unit = nbytes / 1e9, "GB/s"
        res["algorithmic_bytes"] = nbytes
    run()
    torch.cuda.synchronize()
    times = []
    for _ in range(args.reps):
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        run()
        e.record()
        torch.cuda.synchronize()
        times.append(s.elapsed_time(e))
    res["us"] = [round(t * 1e3, 2) for t in times]
    res[unit] = round(work / (min(times) * 1e-3), 1)
    print(json.dumps(res), flush=True)


def main():
    args = parse()
    if args.kernel_case:
        kernel_case(args)
        return
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    r = run_ours(args, rank, world, device)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline()
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank != 0:
        return
    pk, _ = peaks()
    line = {
        "metric": METRIC,
        "value": round(r["value"], 1),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(r["ms_per_step"], 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": WORKLOAD, "step": [f"{n}:{t}" for n, t, _, _ in step_plan(__import__("microscaling_block_quantization_b200"))],
                   "step_algorithmic_bytes": r["step_bytes"], "hbm_frac_of_8TBs": round(r["value"] / world / 8000, 4),
                   "quantize_only_GB_per_s": r["roofline"]["achieved_with_amax_pass"],
                   "quantize_only_note": "the step's 4 grouped quantizer calls on A and W (NVFP4's tensor-amax "
                                         "launch included, no dequantizer): their algorithmic bytes over their "
                                         "summed call durations, one stream",
                   "per_launch_timing": f"per variant a graph of {R_PAIRS} back-to-back calls over A and W "
                                        "(one grouped quantizer launch each), replayed K times (no graph-launch "
                                        "gap between launches)",
                   "l2": "inputs larger than L2 (A+W 176 MiB > 126 MB) read once per call",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
                   "streams": "one" if args.one_stream else
                              "two: MXFP4 / rotated / MBS quantizers on one stream, NVFP4 (tensor-amax pass + "
                              "quantizer) and the dequantizers (after their codes) on a second, each with its "
                              "own workspaces; per-variant figures come from one-stream graphs of back-to-back "
                              "A+W calls"},
        "roofline": r["roofline"],
        "cpu_baseline": cpu,
        "e2e": r["e2e"],
        "gpu_launches": r["launches"] * args.steps,
        "clocks": r["clocks"],
        "rows": r["rows"],
        "gemm": r["gemm"],
        "extra_rows": r["extra"],
        "fidelity": r["fidelity"],
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
