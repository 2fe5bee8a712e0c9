"""Benchmark: FP4 quantized linear layer fwd+bwd on a Llama-3.1-8B MLP shape.

One step = the whole hot path over one batch: six quantizations (X, W along K
for Fprop; dY along N and W along N for Dgrad; dY and X along the tokens for
Wgrad; NVFP4 tensor-amax passes included) and the three block-scaled FP4
GEMMs, through the library's C ABI. The headline `value` is 6 M N K / step
time (TFLOP/s) with inputs resident in HBM; `e2e` is the same metric through
qfp4_linear_fwd/bwd with host buffers (pinned H2D of X, W, dY and D2H of Y,
dX, dW inside the timed region). `quantize` reports the quantizer sweep
workload's GB/s. Synthetic inputs from fp4_precision_b200.inputs.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 runs N independent replicas (one per GPU, launched by torchrun); the
path has no exchange step, so there is no data-path collective.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FP4 linear fwd+bwd TFLOPS (8B MLP shapes) & quantize GB/s, as % of roofline"
WORKLOAD = "mlp_up"  # Llama-3.1-8B MLP up/gate: X [16384x4096], W [28672x4096], dY [16384x28672]
RECIPE = "QUARTET2_NVFP4"
NOMINAL_FP4_OVER_BF16 = 4.0  # dense FP4 9 PF / dense BF16 2.25 PF (nominal ratio)


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-sustained", action="store_true",
                    help="leave out the two-second sustained run of the step (its own key, not the headline)")
    ap.add_argument("--profile", choices=["gemm_fprop", "gemm_dgrad", "gemm_wgrad", "quant_row", "quant_col",
                                          "quant_sr_row", "quant_sr_col", "amax_row", "amax_col",
                                          "amax_rowcol"],
                    help="run only one kernel 3 times on a bounded case (for ncu captures), print nothing else")
    return ap.parse_args()


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def max_over_ranks(x: float, world: int, device) -> float:
    """The largest of the ranks' values, on every rank (a multi-GPU job's time
    is its slowest rank's): one all-reduce of a one-element tensor on `device`
    (the rank's GPU under NCCL, the CPU under gloo)."""
    if world <= 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measured_gemm_traffic():
    """DRAM bytes per GEMM launch (dram__bytes_read.sum + dram__bytes_write.sum)
    from the committed ncu record of this workload (profiles/gemm_traffic.json),
    or None when the GEMM kernel's sources have changed since those counters
    were taken (their SHA-256 is recorded beside the figures)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "gemm_traffic.json")) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    csrc = os.path.join(ROOT, "fp4_precision_b200", "csrc")
    for fname, digest in rec.get("source_sha256", {}).items():
        try:
            with open(os.path.join(csrc, fname), "rb") as f:
                if hashlib.sha256(f.read()).hexdigest() != digest:
                    return None
        except OSError:
            return None
    t = rec.get("traffic_bytes_per_launch")
    if not rec.get("source_sha256") or not isinstance(t, dict):
        return None
    return {k: int(t[k]) for k in ("fprop", "dgrad", "wgrad")}


# FP4 tensor-core work per SM and clock: one M128 x N256 x K64 block-scaled
# MMA (2 * 128 * 256 * 64 flops) per 128 cycles (9 PFLOP/s dense over 148 SMs
# at 1.855 GHz is the same figure).
FP4_FLOP_PER_SM_CYCLE = 2 * 128 * 256 * 64 / 128


def gemm_roofline(gemm_flops, gemm_ms, peaks, src, clocks, sms, timed_ms):
    """The dominant kernel's roofline object: the three GEMMs' algorithmic
    flops over their CUDA-event time against the dense FP4 peak derived from
    the measured bf16 cuBLAS peak (x 4, the nominal FP4/BF16 ratio): the burst
    figure when the timed region is short (under one second), else the
    sustained one; plus the clock-normalised fraction (flops per SM and cycle
    at the sampled median SM clock over the FP4 MMA's per-cycle work)."""
    achieved = sum(gemm_flops) / (sum(gemm_ms) * 1e-3) / 1e12
    sustained = timed_ms >= 1000.0
    key = "bf16_tflops_sustained" if sustained else "bf16_tflops"
    peak = peaks[key] * NOMINAL_FP4_OVER_BF16
    out = {"bound": "tensor", "kernel": "gemm_bs_fp4 (tcgen05 kind::mxf4nvf4)", "achieved": round(achieved, 1),
           "peak": round(peak, 1), "unit": "TFLOP/s", "frac": round(achieved / peak, 4),
           "peak_source": f"{src}: {key} {peaks[key]} x nominal FP4/BF16 ratio {NOMINAL_FP4_OVER_BF16} "
                          f"({'sustained: timed region >= 1 s' if sustained else 'burst: timed region < 1 s'})",
           "frac_of_nominal_9pf": round(achieved / 9000.0, 4)}
    mhz = clocks.get("sm_mhz")
    if mhz:
        per_cycle = achieved * 1e12 / (sms * mhz * 1e6)
        out["clock_normalised"] = {
            "sm_mhz_median": mhz, "flop_per_sm_cycle": round(per_cycle, 1),
            "fp4_mma_flop_per_sm_cycle": FP4_FLOP_PER_SM_CYCLE, "frac": round(per_cycle / FP4_FLOP_PER_SM_CYCLE, 4),
            "gemm_ms_x_mhz": round(sum(gemm_ms) * mhz, 1)}
    return out


# ---------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi clock / throttle-reason samples during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
         "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
         "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ---------------------------------------------------------------------------
def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from fp4_precision_b200 import inputs
    from fp4_precision_b200 import qfp4 as Q

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    wl = inputs.workload(WORKLOAD, device=dev)
    X, W, dY = wl["X"], wl["W"], wl["dY"]
    M, K = X.shape
    N = W.shape[0]
    rec = Q.recipe(RECIPE)
    seed = Q.make_seed(rot=0x0123_4567, sr=0x89AB_CDEF)
    stream = torch.cuda.current_stream()
    ws = torch.empty((Q.quantize_workspace_bytes(),), dtype=torch.uint8, device=dev)

    # quantized operands of the step, allocated once
    c = rec.fprop, rec.dgrad, rec.wgrad
    ops = [(X, c[0].fmt, c[0].rnd_a, c[0].had, Q.ROW, Q.make_seed(seed.rot, seed.sr, 0, 0)),
           (W, c[0].fmt, c[0].rnd_b, c[0].had, Q.ROW, Q.make_seed(seed.rot, seed.sr, 0, 1)),
           (dY, c[1].fmt, c[1].rnd_a, c[1].had, Q.ROW, Q.make_seed(seed.rot, seed.sr, 1, 2)),
           (W, c[1].fmt, c[1].rnd_b, c[1].had, Q.COL, Q.make_seed(seed.rot, seed.sr, 1, 3)),
           (dY, c[2].fmt, c[2].rnd_a, c[2].had, Q.COL, Q.make_seed(seed.rot, seed.sr, 2, 4)),
           (X, c[2].fmt, c[2].rnd_b, c[2].had, Q.COL, Q.make_seed(seed.rot, seed.sr, 2, 5))]
    qs = []
    for (t, fmt, rnd, had, axis, sd) in ops:
        rows, k = (t.shape[0], t.shape[1]) if axis == Q.ROW else (t.shape[1], t.shape[0])
        qs.append(Q.empty_qtensor(fmt, rows, k, dev))
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    dW = torch.empty((N, K), dtype=torch.float32, device=dev)
    gemm_flops = [2.0 * M * N * K] * 3
    quant_elems = [t.numel() for (t, *_rest) in ops]

    # dY is quantized along both axes, as qfp4_linear_bwd does it: with NVFP4 and
    # the same Hadamard for Dgrad and Wgrad one pass gives both tensor amaxes;
    # with round-to-nearest one pass gives both quantizations
    fused_dy_amax, dual_dy = dy_plan(Q, c, M)
    dy_amax = torch.empty((2,), dtype=torch.float32, device=dev)
    # X and W: the forward's amax read also gives the backward's tensor amaxes
    xw = xw_plan(Q, c)
    xw_amax = torch.empty((4,), dtype=torch.float32, device=dev)

    def step(ev=None, st=None):
        st = stream if st is None else st
        # ev: per kernel group (6 quantize calls, 3 GEMMs) a (start, end)
        # event pair or None; ev itself may be None
        def mark(j, k):
            if ev is not None and ev[j] is not None:
                ev[j][k].record(st)
        for i, (t, fmt, rnd, had, axis, sd) in enumerate(ops):
            mark(i, 0)
            if i in (2, 4):
                quantize_dy(Q, dY, c, ops, qs, i, fused_dy_amax, dual_dy, dy_amax, ws, st)
            else:
                quantize_xw(Q, ops, qs, i, xw, xw_amax, ws, st)
            mark(i, 1)
            if i == 1:
                mark(6, 0)
                Q.gemm(qs[0], qs[1], torch.bfloat16, out=Y, stream=st)
                mark(6, 1)
            if i == 3:
                mark(7, 0)
                Q.gemm(qs[2], qs[3], torch.bfloat16, out=dX, stream=st)
                mark(7, 1)
        mark(8, 0)
        Q.gemm(qs[4], qs[5], torch.float32, out=dW, stream=st)
        mark(8, 1)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    Q.status()
    barrier()

    # timed region: K steps, events on the launching stream
    evs = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in range(9)]
           for _ in range(args.steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    Q.launch_count(reset=True)
    with ClockSampler(local_rank) as clk:
        barrier()
        t0.record(stream)
        for s in range(args.steps):
            step(evs[s])
        t1.record(stream)
        barrier()
    launches = Q.launch_count(reset=True)
    Q.status()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev)
    ms_step = ms / args.steps
    per = [[evs[s][j][0].elapsed_time(evs[s][j][1]) for s in range(args.steps)] for j in range(9)]
    gemm_ms = [statistics.mean(per[6 + g]) for g in range(3)]
    quant_ms = [statistics.mean(per[i]) for i in range(6)]
    flops_step = 6.0 * M * N * K
    value = world * flops_step / (ms_step * 1e-3) / 1e12

    peaks, src = measured_peaks()
    clocks = clk.summary()
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    roofline = gemm_roofline(gemm_flops, gemm_ms, peaks, src, clocks, sms, ms)
    traffic = measured_gemm_traffic()
    roofline.update({
        "traffic": None if traffic is None else int(statistics.mean(traffic.values())),
        "traffic_unit": "DRAM bytes per GEMM launch (mean of Fprop, Dgrad, Wgrad; ncu dram__bytes_read.sum + "
                        "dram__bytes_write.sum, profiles/gemm_traffic.json; null when the GEMM sources changed since)",
        "traffic_per_gemm": traffic,
        "algorithmic_bytes_per_gemm": {
            "fprop": (M + N) * (K // 2 + K // 16) + M * N * 2,
            "dgrad": (M + K) * (N // 2 + N // 16) + M * K * 2,
            "wgrad": (N + K) * (M // 2 + M // 16) + N * K * 4},
        "per_gemm_ms": {"fprop": round(gemm_ms[0], 4), "dgrad": round(gemm_ms[1], 4), "wgrad": round(gemm_ms[2], 4)}})

    # the same step run for about two seconds (the GPU settles at its power cap):
    # step time and GEMM roofline against the sustained peak, with its clocks
    n_sus = 0 if args.no_sustained else max(20, int(2000.0 / max(ms_step, 0.05)))
    sevs = [[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in range(3 * n_sus)]
    with ClockSampler(local_rank) as sclk:
        barrier()
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s0.record(stream)
        for i in range(n_sus):
            step([None] * 6 + [sevs[3 * i], sevs[3 * i + 1], sevs[3 * i + 2]])
        s1.record(stream)
        barrier()
    Q.status()
    sus_ms = max_over_ranks(s0.elapsed_time(s1), world, dev)
    sustained = None
    if n_sus:
        sus_gemm = [statistics.mean(sevs[3 * i + g][0].elapsed_time(sevs[3 * i + g][1]) for i in range(n_sus))
                    for g in range(3)]
        sus_clocks = sclk.summary()
        sus_roof = gemm_roofline(gemm_flops, sus_gemm, peaks, src, sus_clocks, sms, sus_ms)
        sustained = {"steps": n_sus, "seconds": round(sus_ms / 1e3, 3), "ms_per_step": round(sus_ms / n_sus, 4),
                     "TFLOP/s": round(world * flops_step / (sus_ms / n_sus * 1e-3) / 1e12, 2),
                     "gemm_ms": {"fprop": round(sus_gemm[0], 4), "dgrad": round(sus_gemm[1], 4),
                                 "wgrad": round(sus_gemm[2], 4)},
                     "roofline": sus_roof, "clocks": sus_clocks}

    # Wgrad accumulating into an fp32 main gradient (dW += dY^T X) on the step's operands
    def wgrad(acc):
        if acc:
            Q.gemm_accumulate(qs[4], qs[5], dW, stream=stream)
        else:
            Q.gemm(qs[4], qs[5], torch.float32, out=dW, stream=stream)
    wg = {}
    for acc in (False, True, False, True):
        for _ in range(2):
            wgrad(acc)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(10):
            wgrad(acc)
        e1.record(stream)
        torch.cuda.synchronize()
        wg[acc] = e0.elapsed_time(e1) / 10
    Q.status()
    # Fprop whose epilogue also writes the MXFP4 operand of a next layer (Y along
    # N), or the NVFP4 tensor amax of Y that the next layer's quantization needs
    qy = Q.empty_qtensor(Q.MXFP4, M, N, dev)
    qyn = Q.empty_qtensor(Q.NVFP4, M, N, dev)
    y_amax = torch.empty((1,), dtype=torch.float32, device=dev)
    qseed = Q.make_seed(seed.rot, seed.sr, 3, 6)
    nh_next = rec.fprop.had  # the next layer's Fprop rotation of its input (Y)
    fq = {}
    for kind in ("gemm", "fused", "separate", "nv_fused", "nv_separate") * 2:
        def fprop_q():
            if kind == "gemm":
                Q.gemm(qs[0], qs[1], torch.bfloat16, out=Y, stream=stream)
            elif kind == "fused":
                Q.gemm_quantize(qs[0], qs[1], Q.HAD_NONE, qseed, out=Y, qout=qy, stream=stream)
            elif kind == "separate":
                Q.gemm(qs[0], qs[1], torch.bfloat16, out=Y, stream=stream)
                Q.quantize(Y, Q.MXFP4, Q.RTN, Q.HAD_NONE, Q.ROW, qseed, out=qy, stream=stream)
            elif kind == "nv_fused":
                Q.gemm_amax(qs[0], qs[1], nh_next, qseed, out=Y, amax=y_amax, workspace=ws, stream=stream)
                Q.quantize(Y, Q.NVFP4, Q.RTN, nh_next, Q.ROW, qseed, amax_in=y_amax, out=qyn, workspace=ws,
                           stream=stream)
            else:
                Q.gemm(qs[0], qs[1], torch.bfloat16, out=Y, stream=stream)
                Q.quantize(Y, Q.NVFP4, Q.RTN, nh_next, Q.ROW, qseed, out=qyn, workspace=ws, stream=stream)
        for _ in range(2):
            fprop_q()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(10):
            fprop_q()
        e1.record(stream)
        torch.cuda.synchronize()
        fq[kind] = min(fq.get(kind, 1e9), e0.elapsed_time(e1) / 10)
    Q.status()
    fprop_quant = {"gemm_ms": round(fq["gemm"], 4), "fused_ms": round(fq["fused"], 4),
                   "gemm_then_quantize_ms": round(fq["separate"], 4),
                   "nvfp4_gemm_amax_then_quantize_ms": round(fq["nv_fused"], 4),
                   "nvfp4_gemm_then_quantize_ms": round(fq["nv_separate"], 4),
                   "what": f"Fprop Y[{M}x{N}] bf16 alone; with its MXFP4 copy along N from the epilogue "
                           "(qfp4_gemm_quantize) vs followed by a separate row quantization of Y; and the next "
                           "layer's NVFP4 quantization of Y (round to nearest, its Fprop Hadamard) with the tensor "
                           "amax from the GEMM's epilogue (qfp4_gemm_amax, quantize with amax_in) vs quantize with "
                           "its own amax pass over Y; 10 launches each"}
    wgrad_acc = {"store_ms": round(wg[False], 4), "accumulate_ms": round(wg[True], 4),
                 "accumulate_TFLOP/s": round(gemm_flops[2] / (wg[True] * 1e-3) / 1e12, 1),
                 "what": "Wgrad of the step, dW = dY^T X vs dW += dY^T X (TMA reduce-add epilogue), fp32 dW "
                         f"[{N}x{K}]; 10 back-to-back launches each"}

    # the step captured once in a CUDA graph and replayed (the same launches, no
    # host-side launch work between them)
    graph = graph_time(step, args, stream, flops_step, world, dev)

    # quantizer sweep workload (GB/s of algorithmic bytes), L2 flushed between launches,
    # and the same kernels on dY [16384 x 28672] (940 MB, steady state)
    quant = quant_sweep(Q, inputs, dev, stream, peaks)
    quant["large"] = quant_large(Q, dY, stream, peaks)
    quant["startup_fit"] = quant_startup_fit(Q, dY, stream, peaks)

    # the other configurations of the MLP shapes (not part of the headline value)
    layers = more_layers(Q, inputs, X, W, dY, seed, stream, dev, roofline["peak"])

    # MXFP4 variants on the Wgrad product of this layer (quality, not speed)
    study = mxfp4_wgrad_study(Q, X, dY, stream)

    # linear API (device-resident) and end to end with host buffers
    api_ms = linear_api_time(Q, X, W, dY, rec, seed, args, stream, dev)
    e2e = None if args.no_e2e else e2e_time(Q, X, W, dY, rec, seed, args, stream, dev, world)

    out = {
        "metric": METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_step, 4), "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "e2m1", "data": "synthetic",
        "config": {"workload": "Llama-3.1-8B MLP up/gate linear fwd+bwd, X[16384x4096] W[28672x4096] "
                               "dY[16384x28672], NVFP4 Quartet II recipe",
                   "M": M, "N": N, "K": K, "recipe": RECIPE,
                   "l2": "inputs larger than L2 (dY 940 MB, W 235 MB, X 134 MB); no flush between steps",
                   "parallelism": f"replicas x{world}"},
        "roofline": roofline,
        "sustained": sustained,
        "graph": graph,
        "step_breakdown_ms": {"quantize": [round(v, 4) for v in quant_ms], "gemm": [round(v, 4) for v in gemm_ms]},
        "quantize": quant,
        "layers": layers,
        "study": study,
        "wgrad_accumulate": wgrad_acc,
        "fprop_quantized_output": fprop_quant,
        "linear_api_ms_per_step": round(api_ms, 4),
        "e2e": e2e,
        "gpu_launches": launches,
        "clocks": clocks,
    }
    return out


def graph_time(step, args, stream, flops_step, world, dev):
    """The step captured into one CUDA graph (on a side stream, as capture
    requires) and replayed K times, timed with CUDA events on that stream."""
    import torch
    s = torch.cuda.Stream(device=dev)
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    try:
        with torch.cuda.stream(s):
            step(None, s)  # outside the capture: lazy set-up, tensor maps, attributes
            torch.cuda.synchronize()
            with torch.cuda.graph(g, stream=s):
                step(None, s)
    except RuntimeError as e:  # capture refused: report why instead of a number
        return {"error": str(e).splitlines()[0][:200]}
    torch.cuda.synchronize()
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(3, args.steps)
    with torch.cuda.stream(s):
        e0.record(s)
        for _ in range(n):
            g.replay()
        e1.record(s)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / n, world, dev)
    del g
    return {"ms_per_step": round(ms, 4), "TFLOP/s": round(world * flops_step / (ms * 1e-3) / 1e12, 2), "steps": n,
            "what": "the headline step captured once in a CUDA graph and replayed"}


def quant_startup_fit(Q, dY, stream, peaks):
    """Why short quantizer launches read below the large-tensor figure: the
    NVFP4 RTN row quantizer (amax given) on the first 1024, 4096, 16384 (all)
    rows of dY — 58, 235, 940 MB — and on 256 rows (15 MB), L2 evicted before
    each launch by a 256 MiB read; a least-squares fit time = t0 + bytes / BW
    gives the fixed cost per launch t0 and the steady-state bandwidth BW."""
    import torch
    flush = torch.ones((64 << 20,), dtype=torch.float32, device=dY.device)
    ws = torch.empty((Q.quantize_workspace_bytes(),), dtype=torch.uint8, device=dY.device)
    seed = Q.make_seed(1, 2)
    pts = []
    for rows in (256, 1024, 4096, dY.shape[0]):
        x = dY[:rows]
        q = Q.empty_qtensor(Q.NVFP4, rows, x.shape[1], dY.device)
        am = Q.amax(x, Q.HAD_NONE, Q.ROW, seed, workspace=ws, stream=stream)
        times = []
        for it in range(7):
            flush.sum()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            Q.quantize(x, Q.NVFP4, Q.RTN, Q.HAD_NONE, Q.ROW, seed, amax_in=am, out=q, workspace=ws, stream=stream)
            e1.record(stream)
            torch.cuda.synchronize()
            if it >= 2:
                times.append(e0.elapsed_time(e1))
        pts.append((x.numel() * (2 + 0.5 + 1 / 16), statistics.median(times)))
        del q
    Q.status()
    n = len(pts)
    mx = sum(b for b, _ in pts) / n
    my = sum(t for _, t in pts) / n
    slope = sum((b - mx) * (t - my) for b, t in pts) / sum((b - mx) ** 2 for b, _ in pts)
    t0 = my - slope * mx
    bw = 1.0 / slope / 1e6  # bytes per ms -> GB/s
    return {"points": [{"MB": round(b / 1e6, 1), "ms": round(t, 4), "GB/s": round(b / (t * 1e-3) / 1e9, 1)}
                       for b, t in pts],
            "fixed_cost_us": round(t0 * 1e3, 2), "steady_GB/s": round(bw, 1),
            "steady_frac_of_measured_hbm": round(bw / peaks["hbm_gbs"], 3),
            "what": "NVFP4 RTN row quantizer on row slices of dY, L2 evicted before each launch; "
                    "time = fixed_cost + bytes / steady_GB/s"}


def dy_plan(Q, c, M):
    """How the layer quantizes dY, as qfp4_linear_bwd does: (fused row-and-column
    amax, dual row-and-column quantization from one read). The dual pass is
    taken for round-to-nearest only (memory-bound); stochastic and Quartet II
    rounding keep two passes."""
    had_n = {Q.HAD_NONE: 0, Q.HAD_DET16: 16, Q.HAD_DET32: 32, Q.HAD_RAND16: 16, Q.HAD_RAND32: 32}
    fused = (c[1].fmt == Q.NVFP4 and c[2].fmt == Q.NVFP4 and c[1].had == c[2].had
             and c[1].had in (Q.HAD_NONE, Q.HAD_DET16, Q.HAD_RAND16))
    dual = (c[1].fmt == c[2].fmt and c[1].rnd_a == Q.RTN and c[2].rnd_a == Q.RTN and M % 64 == 0
            and had_n[c[1].had] in (0, had_n[c[2].had]))
    return fused, dual


def quantize_dy(Q, dY, c, ops, qs, i, fused, dual, dy_amax, ws, stream):
    """Operand i (2: dY along N, 4: dY along the tokens) of the step."""
    t, fmt, rnd, had, axis, sd = ops[i]
    nv = c[1].fmt == Q.NVFP4
    if i == 2:
        if fused:
            Q.amax_rowcol(dY, had, ops[2][5], ops[4][5], out=dy_amax, workspace=ws, stream=stream)
        elif dual and nv:
            Q.amax(dY, c[1].had, Q.ROW, ops[2][5], out=dy_amax[0:1], workspace=ws, stream=stream)
            Q.amax(dY, c[2].had, Q.COL, ops[4][5], out=dy_amax[1:2], workspace=ws, stream=stream)
    am = dy_amax[0:1] if i == 2 else dy_amax[1:2]
    if dual:
        if i == 2:
            Q.quantize_dual(dY, fmt, rnd, c[1].had, c[2].had, ops[2][5], ops[4][5], dy_amax[0:1] if nv else None,
                            dy_amax[1:2] if nv else None, out_row=qs[2], out_col=qs[4], stream=stream)
        return
    Q.quantize(t, fmt, rnd, had, axis, sd, amax_in=am if fused else None, out=qs[i], workspace=ws, stream=stream)


def xw_plan(Q, c):
    """Whether the forward takes the backward's NVFP4 tensor amaxes of X and W
    in the read that gives its own (qfp4_amax_rowcol: the forward's Hadamard
    along K, the backward GEMM's along the other axis), so that the backward
    quantizes X and W without an amax pass of its own: (for X, for W). Both
    GEMMs that use the operand must quantize it to NVFP4. (The linear layer's
    entry points cannot do this: the forward and the backward are separate
    calls.)"""
    nv = lambda g: g.fmt == Q.NVFP4
    return (nv(c[0]) and nv(c[2]), nv(c[0]) and nv(c[1]))


def quantize_xw(Q, ops, qs, i, plan, xw_amax, ws, stream):
    """Operand i (0: X along K, 1: W along K, 3: W along N, 5: X along the
    tokens) of the step. With plan[X or W] the forward's call takes both
    tensor amaxes of the operand in one read and the backward's call uses the
    second (the same values the backward's own amax pass would give)."""
    t, fmt, rnd, had, axis, sd = ops[i]
    j = 0 if i in (0, 5) else 1
    if not plan[j]:
        Q.quantize(t, fmt, rnd, had, axis, sd, out=qs[i], workspace=ws, stream=stream)
        return
    am = xw_amax[2 * j:2 * j + 2]
    if i in (0, 1):
        b = 5 if i == 0 else 3
        Q.amax_rowcol(t, had, sd, ops[b][5], out=am, workspace=ws, stream=stream, had_col=ops[b][3])
        Q.quantize(t, fmt, rnd, had, axis, sd, amax_in=am[0:1], out=qs[i], workspace=ws, stream=stream)
    else:
        Q.quantize(t, fmt, rnd, had, axis, sd, amax_in=am[1:2], out=qs[i], workspace=ws, stream=stream)


def layer_step(Q, X, W, dY, rec, seed, steps, stream, dev):
    """One linear layer's fwd+bwd through the six quantize and three GEMM calls
    (the same sequence as the headline step), timed with CUDA events on the
    launching stream: ms per step and per GEMM."""
    import torch
    M, K = X.shape
    N = W.shape[0]
    ws = torch.empty((Q.quantize_workspace_bytes(),), dtype=torch.uint8, device=dev)
    c = rec.fprop, rec.dgrad, rec.wgrad
    ops = [(X, c[0].fmt, c[0].rnd_a, c[0].had, Q.ROW, Q.make_seed(seed.rot, seed.sr, 0, 0)),
           (W, c[0].fmt, c[0].rnd_b, c[0].had, Q.ROW, Q.make_seed(seed.rot, seed.sr, 0, 1)),
           (dY, c[1].fmt, c[1].rnd_a, c[1].had, Q.ROW, Q.make_seed(seed.rot, seed.sr, 1, 2)),
           (W, c[1].fmt, c[1].rnd_b, c[1].had, Q.COL, Q.make_seed(seed.rot, seed.sr, 1, 3)),
           (dY, c[2].fmt, c[2].rnd_a, c[2].had, Q.COL, Q.make_seed(seed.rot, seed.sr, 2, 4)),
           (X, c[2].fmt, c[2].rnd_b, c[2].had, Q.COL, Q.make_seed(seed.rot, seed.sr, 2, 5))]
    qs = []
    for (t, fmt, rnd, had, axis, sd) in ops:
        rows, k = (t.shape[0], t.shape[1]) if axis == Q.ROW else (t.shape[1], t.shape[0])
        qs.append(Q.empty_qtensor(fmt, rows, k, dev))
    dw_dtype = torch.float32 if rec.dw_dtype == Q.OUT_F32 else torch.bfloat16
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    dW = torch.empty((N, K), dtype=dw_dtype, device=dev)
    outs = [(0, 1, Y, torch.bfloat16), (2, 3, dX, torch.bfloat16), (4, 5, dW, dw_dtype)]

    fused_dy_amax, dual_dy = dy_plan(Q, c, M)
    dy_amax = torch.empty((2,), dtype=torch.float32, device=dev)
    xw = xw_plan(Q, c)
    xw_amax = torch.empty((4,), dtype=torch.float32, device=dev)

    def step(ev):
        for i, (t, fmt, rnd, had, axis, sd) in enumerate(ops):
            if i in (2, 4):
                quantize_dy(Q, dY, c, ops, qs, i, fused_dy_amax, dual_dy, dy_amax, ws, stream)
            else:
                quantize_xw(Q, ops, qs, i, xw, xw_amax, ws, stream)
            if i % 2 == 1:
                a, b, D, odt = outs[i // 2]
                if ev is not None:
                    ev[i // 2][0].record(stream)
                Q.gemm(qs[a], qs[b], odt, out=D, stream=stream)
                if ev is not None:
                    ev[i // 2][1].record(stream)

    for _ in range(3):
        step(None)
    torch.cuda.synchronize()
    evs = [[[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(3)] for _ in range(steps)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for st in range(steps):
        step(evs[st])
    t1.record(stream)
    torch.cuda.synchronize()
    Q.status()
    ms = t0.elapsed_time(t1) / steps
    gemm_ms = [statistics.mean(evs[st][g][0].elapsed_time(evs[st][g][1]) for st in range(steps)) for g in range(3)]
    flops = 2.0 * M * N * K
    return {"ms_per_step": round(ms, 4), "TFLOP/s": round(3 * flops / (ms * 1e-3) / 1e12, 1),
            "gemm_ms": {"fprop": round(gemm_ms[0], 4), "dgrad": round(gemm_ms[1], 4), "wgrad": round(gemm_ms[2], 4)},
            "gemm_TFLOP/s": round(3 * flops / (sum(gemm_ms) * 1e-3) / 1e12, 1)}


def more_layers(Q, inputs, X, W, dY, seed, stream, dev, fp4_peak):
    """The other configurations of the Llama-3.1-8B layer shapes (not part of
    the headline value): the MLP up/gate layer with the AMD MXFP4 recipe
    (deterministic 32x32 Hadamard on Wgrad), the attention QKV projection with
    the Quartet II NVFP4 recipe, and the MLP down layer with the Quartet II and
    the per-element SR NVFP4 recipes at 2048 ... 32768 tokens. Each entry: ms
    per fwd+bwd, TFLOP/s, per-GEMM ms and the GEMMs' fraction of the FP4 peak."""
    import torch

    def entry(r):
        r["gemm_frac_of_peak"] = round(r["gemm_TFLOP/s"] / fp4_peak, 4)
        return r
    out = {"mlp_up_AMD_MXFP4_H": entry(layer_step(Q, X, W, dY, Q.recipe("AMD_MXFP4_H"), seed, 10, stream, dev))}
    wl = inputs.workload("qkv", device=dev)
    out["qkv_QUARTET2_NVFP4"] = entry(layer_step(Q, wl["X"], wl["W"], wl["dY"], Q.recipe("QUARTET2_NVFP4"), seed, 10,
                                                 stream, dev))
    del wl
    for M in (2048, 4096, 8192, 16384, 32768):
        wl = inputs.workload("mlp_down", device=dev, M=M)
        for rec in ("QUARTET2_NVFP4", "NVIDIA_NVFP4"):
            out[f"mlp_down_M{M}_{rec}"] = entry(layer_step(Q, wl["X"], wl["W"], wl["dY"], Q.recipe(rec), seed, 10,
                                                           stream, dev))
        del wl
        torch.cuda.empty_cache()
    out["workloads"] = {"mlp_up": "X[16384x4096] W[28672x4096] dY[16384x28672]",
                        "qkv": "X[8192x4096] N(0,1)+0.1% x50 outliers, W[6144x4096] N(0,0.02), dY[8192x6144] N(0,1e-3)",
                        "mlp_down": "X[Mx14336] = SiLU(N(0,1))*N(0,1), W[4096x14336] N(0,0.02), dY[Mx4096] N(0,1e-3)"}
    out["peak_TFLOP/s"] = round(fp4_peak, 1)
    return out


SWEEP_FMTS = (("nvfp4", 0), ("mxfp4", 1), ("mxfp4ru", 2))          # Q.NVFP4, Q.MXFP4, Q.MXFP4_RU
SWEEP_HADS = (("none", 0), ("det16", 1), ("det32", 2), ("rand16", 3), ("rand32", 4))
SWEEP_RNDS = (("rtn", 0), ("sr", 1), ("q2", 2))
SWEEP_AXES = (("row", 0), ("col", 1))


def sweep_cases():
    """Every (format, Hadamard, rounding, axis) case of the quantizer sweep:
    NVFP4 and MXFP4 (60 cases) and the round-up MXFP4 variant (30 more)."""
    return [(f"{fn}_{rn}_{hn}_{an}", f, r, h, a) for fn, f in SWEEP_FMTS for hn, h in SWEEP_HADS
            for rn, r in SWEEP_RNDS for an, a in SWEEP_AXES]


def quant_sweep(Q, inputs, dev, stream, peaks):
    """The quantizer-sweep tensor [8192x4096] (67 MB, fits in L2): GB/s of
    algorithmic bytes (2 B read + 0.5 B codes + 1/16 (NVFP4) or 1/32 (MXFP4)
    B scales per element; the NVFP4 amax pass, counted separately at 2 B per
    element, is taken before the timed launch) for every case. Before every
    launch L2 is evicted by reading a 256 MiB buffer (a reduction that writes
    nothing back to it), so the launch reads its input from DRAM and finds no
    dirty lines left for it to write back."""
    import torch
    T = inputs.workload("sweep", device=dev)["T"]
    R, C = T.shape
    flush = torch.ones((64 << 20,), dtype=torch.float32, device=dev)  # 256 MiB
    ws = torch.empty((Q.quantize_workspace_bytes(),), dtype=torch.uint8, device=dev)
    seed = Q.make_seed(5, 6, 1, 2)
    res = {}

    def timed(fn, n=6):
        times = []
        for it in range(n + 2):
            flush.sum()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize()
            if it >= 2:
                times.append(e0.elapsed_time(e1))
        return statistics.median(times)

    for name, fmt, rnd, had, axis in sweep_cases():
        rows, k = (R, C) if axis == Q.ROW else (C, R)
        q = Q.empty_qtensor(fmt, rows, k, dev)
        # a pre-computed amax isolates the one-pass quantizer kernel
        am = Q.amax(T, had, axis, seed, workspace=ws, stream=stream) if fmt == Q.NVFP4 else None
        ms = timed(lambda: Q.quantize(T, fmt, rnd, had, axis, seed, amax_in=am, out=q, workspace=ws, stream=stream))
        byts = R * C * (2 + 0.5 + (1 / 16 if fmt == Q.NVFP4 else 1 / 32))
        gbs = byts / (ms * 1e-3) / 1e9
        res[name] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_of_measured_hbm": round(gbs / peaks["hbm_gbs"], 3)}
        del q
    am = torch.empty((1,), dtype=torch.float32, device=dev)
    for hn, had in (("none", Q.HAD_NONE), ("rand16", Q.HAD_RAND16), ("rand32", Q.HAD_RAND32)):
        for an, axis in SWEEP_AXES:
            ms = timed(lambda: Q.amax(T, had, axis, seed, out=am, workspace=ws, stream=stream))
            gbs = R * C * 2 / (ms * 1e-3) / 1e9
            res[f"amax_{hn}_{an}"] = {"ms": round(ms, 4), "GB/s": round(gbs, 1),
                                      "frac_of_measured_hbm": round(gbs / peaks["hbm_gbs"], 3)}
    Q.status()
    summary = {}
    for rn, _ in SWEEP_RNDS:
        fr = [v["frac_of_measured_hbm"] for k, v in res.items() if f"_{rn}_" in k]
        summary[rn] = {"min": min(fr), "median": statistics.median(fr), "max": max(fr), "cases": len(fr)}
    return {"workload": "quantizer sweep tensor [8192x4096] bf16, Student-t(3)*0.02*LogNormal(0,1) column gains",
            "bytes_per_elem": "2 read + 0.5 codes + 1/16 (NVFP4) or 1/32 (MXFP4) scales; amax pass 2 read",
            "l2": "a 256 MiB buffer read (summed) before every launch: L2 evicted, no dirty lines left",
            "unit": "GB/s", "frac_summary_by_rounding": summary, "cases": res}


def quant_large(Q, T, stream, peaks):
    """Quantizer and amax kernels on a tensor far larger than L2 (the layer's
    dY, [16384 x 28672] bf16, 940 MB): steady-state GB/s of algorithmic bytes
    (2 B read + 0.5 B codes + 1/16 B (NVFP4) or 1/32 B (MXFP4) scales per
    element; amax: 2 B read)."""
    import torch
    R, C = T.shape
    dev = T.device
    ws = torch.empty((Q.quantize_workspace_bytes(),), dtype=torch.uint8, device=dev)
    seed = Q.make_seed(7, 8)
    res = {}

    def timeit(fn, n=5):
        for _ in range(2):
            fn()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(n):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / n

    for name, fmt, rnd, had, axis in (("nvfp4_rtn_none_row", Q.NVFP4, Q.RTN, Q.HAD_NONE, Q.ROW),
                                      ("nvfp4_rtn_rand16_row", Q.NVFP4, Q.RTN, Q.HAD_RAND16, Q.ROW),
                                      ("nvfp4_rtn_rand16_col", Q.NVFP4, Q.RTN, Q.HAD_RAND16, Q.COL),
                                      ("nvfp4_sr_rand16_row", Q.NVFP4, Q.SR, Q.HAD_RAND16, Q.ROW),
                                      ("nvfp4_q2_rand16_row", Q.NVFP4, Q.QUARTET2, Q.HAD_RAND16, Q.ROW),
                                      ("nvfp4_q2_rand16_col", Q.NVFP4, Q.QUARTET2, Q.HAD_RAND16, Q.COL),
                                      ("mxfp4_rtn_det32_col", Q.MXFP4, Q.RTN, Q.HAD_DET32, Q.COL),
                                      ("mxfp4ru_rtn_det32_col", Q.MXFP4_RU, Q.RTN, Q.HAD_DET32, Q.COL)):
        rows, k = (R, C) if axis == Q.ROW else (C, R)
        q = Q.empty_qtensor(fmt, rows, k, dev)
        am = Q.amax(T, had, axis, seed, workspace=ws, stream=stream) if fmt == Q.NVFP4 else None
        ms = timeit(lambda: Q.quantize(T, fmt, rnd, had, axis, seed, amax_in=am, out=q, workspace=ws,
                                       stream=stream))
        gbs = R * C * (2 + 0.5 + (1 / 16 if fmt == Q.NVFP4 else 1 / 32)) / (ms * 1e-3) / 1e9
        res[name] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_of_measured_hbm": round(gbs / peaks["hbm_gbs"], 3)}
        del q
    for name, axis in (("amax_rand16_row", Q.ROW), ("amax_rand16_col", Q.COL)):
        am = torch.empty((1,), dtype=torch.float32, device=dev)
        ms = timeit(lambda: Q.amax(T, Q.HAD_RAND16, axis, seed, out=am, workspace=ws, stream=stream))
        gbs = R * C * 2 / (ms * 1e-3) / 1e9
        res[name] = {"ms": round(ms, 4), "GB/s": round(gbs, 1), "frac_of_measured_hbm": round(gbs / peaks["hbm_gbs"], 3)}
    Q.status()
    return {"workload": f"dY [{R}x{C}] bf16 N(0,1e-3), 940 MB (larger than L2; no flush)", "unit": "GB/s",
            "cases": res}


def mxfp4_wgrad_study(Q, X, dY, stream):
    """Relative Frobenius error of the MXFP4 Wgrad product dY^T X (both
    operands quantized along the tokens, RTN) against the fp32 product of the
    bf16 inputs, for the Hadamard sizes the AMD MXFP4 page's experiments use
    (none, 16, 32; deterministic) and for the floor and the round-up shared
    exponent. A quality figure of the variants, not part of the timed path."""
    import torch
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    ref = dY.t().float() @ X.float()
    torch.backends.cuda.matmul.allow_tf32 = prev
    nref = torch.linalg.vector_norm(ref).item()
    seed = Q.make_seed(9, 10)
    res = {}
    for hname, had in (("none", Q.HAD_NONE), ("det16", Q.HAD_DET16), ("det32", Q.HAD_DET32)):
        for ename, fmt in (("floor", Q.MXFP4), ("round_up", Q.MXFP4_RU)):
            A = Q.quantize(dY, fmt, Q.RTN, had, Q.COL, seed, stream=stream)
            B = Q.quantize(X, fmt, Q.RTN, had, Q.COL, seed, stream=stream)
            D = Q.gemm(A, B, torch.float32, stream=stream)
            res[f"{hname}_{ename}"] = round(torch.linalg.vector_norm(D - ref).item() / nref, 5)
            del A, B, D
    Q.status()
    del ref
    return {"mxfp4_wgrad_rel_err": res,
            "what": "||dW_fp4 - dW_fp32|| / ||dW_fp32||, dW = dY^T X of the MLP up/gate workload, MXFP4 RTN along "
                    "the tokens, deterministic Hadamard none/16/32, floor vs round-up shared exponent"}


def linear_api_time(Q, X, W, dY, rec, seed, args, stream, dev):
    import torch
    M, K = X.shape
    N = W.shape[0]
    wsf = torch.empty((Q.linear_workspace_bytes(False, M, N, K, rec),), dtype=torch.uint8, device=dev)
    wsb = torch.empty((Q.linear_workspace_bytes(True, M, N, K, rec),), dtype=torch.uint8, device=dev)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device=dev)
    dW = torch.empty((N, K), dtype=torch.float32, device=dev)
    for _ in range(2):
        Q.linear_fwd(X, W, rec, seed, Y=Y, workspace=wsf, stream=stream)
        Q.linear_bwd(dY, X, W, rec, seed, dX=dX, dW=dW, workspace=wsb, stream=stream)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(3, args.steps // 2)
    e0.record(stream)
    for _ in range(n):
        Q.linear_fwd(X, W, rec, seed, Y=Y, workspace=wsf, stream=stream)
        Q.linear_bwd(dY, X, W, rec, seed, dX=dX, dW=dW, workspace=wsb, stream=stream)
    e1.record(stream)
    torch.cuda.synchronize()
    Q.status()
    return e0.elapsed_time(e1) / n


def e2e_time(Q, X, W, dY, rec, seed, args, stream, dev, world):
    """qfp4_linear_fwd/bwd with host buffers: every step copies its inputs
    (X, W, dY) from pinned host memory and its results (Y, dX, dW) back, inside
    the timed region. Steps are pipelined over three streams with
    double-buffered device buffers, as a training loop would run them: step
    i + 1's inputs go up while step i computes and step i - 1's results come
    down (PCIe carries both directions at once). The time covers the first
    step's upload through the last step's download."""
    import torch
    M, K = X.shape
    N = W.shape[0]
    hX, hW, hdY = (t.cpu().pin_memory() for t in (X, W, dY))
    hout = [[torch.empty((M, N), dtype=torch.bfloat16).pin_memory(),
             torch.empty((M, K), dtype=torch.bfloat16).pin_memory(),
             torch.empty((N, K), dtype=torch.float32).pin_memory()] for _ in range(2)]
    din = [[torch.empty_like(X), torch.empty_like(W), torch.empty_like(dY)] for _ in range(2)]
    dout = [[torch.empty((M, N), dtype=torch.bfloat16, device=dev), torch.empty((M, K), dtype=torch.bfloat16, device=dev),
             torch.empty((N, K), dtype=torch.float32, device=dev)] for _ in range(2)]
    wsf = torch.empty((Q.linear_workspace_bytes(False, M, N, K, rec),), dtype=torch.uint8, device=dev)
    wsb = torch.empty((Q.linear_workspace_bytes(True, M, N, K, rec),), dtype=torch.uint8, device=dev)
    # three side streams (the legacy default stream would serialise them)
    s_in, s_cmp, s_out = (torch.cuda.Stream(device=dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_cmp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def issue(i):
        b = i & 1
        xd, wd, dyd = din[b]
        yd, dxd, dwd = dout[b]
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_cmp[b])  # step i - 2 is done with these inputs
            xd.copy_(hX, non_blocking=True)
            wd.copy_(hW, non_blocking=True)
            dyd.copy_(hdY, non_blocking=True)
            ev_in[b].record(s_in)
        s_cmp.wait_event(ev_in[b])
        if i >= 2:
            s_cmp.wait_event(ev_out[b])  # step i - 2's results have been read back
        Q.linear_fwd(xd, wd, rec, seed, Y=yd, workspace=wsf, stream=s_cmp)
        Q.linear_bwd(dyd, xd, wd, rec, seed, dX=dxd, dW=dwd, workspace=wsb, stream=s_cmp)
        ev_cmp[b].record(s_cmp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_cmp[b])
            for h, d in zip(hout[b], dout[b]):
                h.copy_(d, non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(2):
        issue(i)
    torch.cuda.synchronize()
    n = max(4, min(args.steps, 20))  # fill and drain (one upload, one download) amortised over the run
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(n):
        issue(i)
    e1.record(s_out)
    torch.cuda.synchronize()
    Q.status()
    ms = max_over_ranks(e0.elapsed_time(e1) / n, world, dev)
    h2d = (M * K + N * K + M * N) * 2
    d2h = M * N * 2 + M * K * 2 + N * K * 4
    return {"value": round(world * 6.0 * M * N * K / (ms * 1e-3) / 1e12, 2), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 3), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
            "pipelining": "3 streams (upload, compute, download), double-buffered device buffers; "
                          f"{n} steps from the first upload to the last download"}


# ---------------------------------------------------------------------------
def oracle_sample(m_rows: int, n_rows: int, steps: int = 1):
    """The CPU oracle on a bounded sample of the workload: the linear fwd+bwd of
    the first m_rows tokens and n_rows output features (all six quantizations
    and the three fp64 GEMMs of that sub-layer, full K). Returns (seconds per
    sample step, flops of the sample, threads)."""
    import oracle as O
    from fp4_precision_b200 import inputs
    wl = inputs.workload(WORKLOAD, device="cpu", M=m_rows)
    X, W, dY = wl["X"], wl["W"][:n_rows].contiguous(), wl["dY"][:, :n_rows].contiguous()
    M, K = X.shape
    N = W.shape[0]
    r = O.preset(RECIPE)
    t0 = time.perf_counter()
    for _ in range(steps):
        O.linear_fwd(X, W, r, 1, 2)
        O.linear_bwd(dY, X, W, r, 1, 2)
    dt = (time.perf_counter() - t0) / steps
    return dt, 6.0 * M * N * K, os.cpu_count()


def cpu_baseline_obj(m_rows=256, n_rows=16384):
    dt, flops, cores = oracle_sample(m_rows, n_rows)
    return {"value": round(flops / dt / 1e12, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
            "sample": f"linear fwd+bwd of the first {m_rows} tokens x {n_rows} output features (full K = 4096) of "
                      f"the MLP up/gate workload: six quantizations (fp32 decisions) + three fp64 GEMMs; {dt:.1f} s"}


def cpu_quantize_modes():
    """The oracle's quantizer (plain C, OpenMP over rows) on the whole quantizer
    sweep tensor [8192 x 4096], once per mode: NVFP4 and MXFP4 x Hadamard
    none / det16 / det32 / rand16 / rand32 x RTN / SR / Quartet II x row /
    column (60 modes; the NVFP4 amax pass included). GB/s of the same
    algorithmic bytes as the GPU sweep."""
    import oracle as O
    from fp4_precision_b200 import inputs
    T = inputs.workload("sweep", device="cpu")["T"]
    R, C = T.shape
    res = {}
    t_all = time.perf_counter()
    for name, fmt, rnd, had, axis in sweep_cases():
        if fmt == 2:  # the round-up variant costs what MXFP4 does
            continue
        t0 = time.perf_counter()
        O.quantize(T, fmt, rnd, had, axis, 1, 0, 2, 0)
        dt = time.perf_counter() - t0
        byts = R * C * (2 + 0.5 + (1 / 16 if fmt == 0 else 1 / 32))
        res[name] = {"s": round(dt, 3), "GB/s": round(byts / dt / 1e9, 4)}
    return {"kind": "oracle", "cores": os.cpu_count(), "unit": "GB/s", "seconds": round(time.perf_counter() - t_all, 1),
            "sample": "the whole quantizer sweep tensor [8192x4096] per mode (60 modes)", "cases": res}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    m_rows, n_rows = 64, 2048
    times = []
    for _ in range(args.warmup):
        oracle_sample(m_rows, n_rows)
    for _ in range(args.steps):
        dt, flops, cores = oracle_sample(m_rows, n_rows)
        times.append(dt)
    ms = statistics.mean(times) * 1e3
    value = flops / (ms * 1e-3) / 1e12
    return {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(ms, 2), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": {"workload": "Llama-3.1-8B MLP up/gate linear fwd+bwd, X[16384x4096] W[28672x4096] "
                                   "dY[16384x28672], NVFP4 Quartet II recipe", "recipe": RECIPE,
                       "sample_tokens": m_rows, "sample_out_features": n_rows},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                             "sample": f"linear fwd+bwd of {m_rows} tokens x {n_rows} output features (full K) "
                                       f"per step"},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def run_profile(kind: str):
    """One kernel, three launches, on a case larger than L2 that holds a few GB
    at most: each of the MLP up/gate layer's three GEMMs (Fprop, Dgrad, Wgrad
    operands quantized as in the step), or a quantizer / amax pass (NVFP4 with
    Quartet II rounding, or per-element SR for the ``quant_sr_*`` cases, after a
    random 16x16 Hadamard) over a [16384 x 8192] bf16 tensor (268 MB)."""
    import torch

    from fp4_precision_b200 import inputs
    from fp4_precision_b200 import qfp4 as Q
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    seed = Q.make_seed(3, 4)
    if kind.startswith("gemm"):
        wl = inputs.workload(WORKLOAD, device=dev)
        rec = Q.recipe(RECIPE)
        c = {"gemm_fprop": rec.fprop, "gemm_dgrad": rec.dgrad, "gemm_wgrad": rec.wgrad}[kind]
        if kind == "gemm_fprop":
            A = Q.quantize(wl["X"], c.fmt, c.rnd_a, c.had, Q.ROW, seed)
            B = Q.quantize(wl["W"], c.fmt, c.rnd_b, c.had, Q.ROW, seed)
            out_dtype = torch.bfloat16
        elif kind == "gemm_dgrad":
            A = Q.quantize(wl["dY"], c.fmt, c.rnd_a, c.had, Q.ROW, seed)
            B = Q.quantize(wl["W"], c.fmt, c.rnd_b, c.had, Q.COL, seed)
            out_dtype = torch.bfloat16
        else:
            A = Q.quantize(wl["dY"], c.fmt, c.rnd_a, c.had, Q.COL, seed)
            B = Q.quantize(wl["X"], c.fmt, c.rnd_b, c.had, Q.COL, seed)
            out_dtype = torch.float32
        del wl
        D = torch.empty((A.rows, B.rows), dtype=out_dtype, device=dev)
        for _ in range(3):
            Q.gemm(A, B, out_dtype, out=D)
    else:
        T = inputs.normal((16384, 8192), 1e-3, 5, "prof", device=dev)
        axis = Q.ROW if kind.endswith("row") else Q.COL
        if kind == "amax_rowcol":  # both orientations' rotated amax from one read
            for _ in range(3):
                Q.amax_rowcol(T, Q.HAD_RAND16, seed, Q.make_seed(3, 4, 1, 2))
        elif kind.startswith("amax"):
            for _ in range(3):
                Q.amax(T, Q.HAD_RAND16, axis, seed)
        else:
            am = Q.amax(T, Q.HAD_RAND16, axis, seed)
            rnd = Q.SR if kind.startswith("quant_sr") else Q.QUARTET2
            for _ in range(3):
                Q.quantize(T, Q.NVFP4, rnd, Q.HAD_RAND16, axis, seed, amax_in=am)
    torch.cuda.synchronize()
    Q.status()


def main():
    args = parse()
    if args.profile:
        run_profile(args.profile)
        return 0
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.gpus != world and world == 1 and args.gpus > 1:
        print(json.dumps({"error": "launch with torchrun for --gpus > 1"}))
        return 2
    if args.impl == "reference":
        out = run_reference(args, rank, world)
        if out is not None:
            print(json.dumps(out))
        return 0
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    out = run_ours(args, rank, world, local_rank)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline_obj()
        out["cpu_baseline_quantize"] = cpu_quantize_modes()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(out))
    return 0


if __name__ == "__main__":
    sys.exit(main())
