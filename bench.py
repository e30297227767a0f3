#!/usr/bin/env python
"""Benchmark of the rank-r W4A4 linear layer (H-SVDQuant forward) on B200.

One step = one pass of the hot path over one batch: for every linear of the
workload, the fused activation step (hsq_quantize_act) followed by the INT4
GEMM + low-rank/bias epilogue (hsq_linear_forward), weights pre-packed (packing
is offline).  Default workload: the FLUX.1 double-stream block linears
(M = 4608 tokens; QKV 3072->9216, MLP up 3072->12288, MLP down 12288->3072;
rank 4; group-64 INT4), synthetic seeded inputs.

Prints ONE JSON line (rank 0).  ``--impl reference`` times the CPU oracle on a
bounded sample of the same workload instead.

Multi-GPU (torchrun, one rank per GPU): every rank runs the whole workload on
its own batch (token-parallel replicas, no data-path collective); the step time
is the max over ranks and ``value`` aggregates all ranks' work.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from w4a4_rank_assisted_b200.synth import WORKLOADS, make_layer  # noqa: E402

L2_BYTES = 126 * 2 ** 20
METRIC = "W4A4 rank-4 linear TOPS & tokens/s at FLUX/SANA/Qwen3 shapes; % of roofline"
INT8_OVER_BF16_NOMINAL = 2.0  # dense INT8 (4.5 POPS) over dense BF16 (2.25 PFLOP/s), nominal

# DRAM bytes (read + write) per GEMM launch, averaged over the step's layers,
# from one ncu capture of the current kernel (profiles/w4a4_gemm_kernel_flux_mlp_up.md
# gives the command and the per-layer counters).  A workload without a capture,
# or whose GEMM changed after its capture, reports null.
NCU_TRAFFIC_PER_LAUNCH = {
    "flux_block_r4": (45407488 + 40368896 + 55537408 + 66134528 + 215083776 + 19456512) / 3,
}


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return dict(hbm_gbs=float(p["hbm_gbs"]), bf16=float(p["bf16_tflops"]),
                    bf16_sustained=float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                    source="measured")
    except Exception:
        return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


def layer_ops(spec):
    """Algorithmic operations of one layer call: the INT4 product (2MNK) plus the
    rank-r branch (2MKr down-projection, 2MNr up-projection)."""
    return 2 * spec.M * spec.N * spec.K + 2 * spec.M * spec.K * spec.r + 2 * spec.M * spec.N * spec.r


def layer_gemm_bytes(spec):
    """Algorithmic HBM bytes of one hsq_linear_forward call (each operand once)."""
    M, N, K, r, gs = spec.M, spec.N, spec.K, spec.r, spec.group
    G = -(-K // gs)
    Kp = gs * G
    return (M * Kp // 2 + 4 * M * G + 4 * M * r      # x codes, scales, U
            + N * Kp // 2 + 4 * N * G + 2 * r * N    # w codes, scales, L2
            + 2 * M * N)                             # Y (bf16)


def layer_fused_bytes(spec):
    """Algorithmic HBM bytes of one hsq_linear_forward_fused call: X, s, L1, the
    packed weights and their scales, L2 and Y (the activation codes, scales and U
    stay on chip)."""
    M, N, K, r, gs = spec.M, spec.N, spec.K, spec.r, spec.group
    G = -(-K // gs)
    Kp = gs * G
    return 2 * M * K + 4 * K + 2 * K * r + N * Kp // 2 + 4 * N * G + 2 * r * N + 2 * M * N


def layer_act_bytes(spec):
    M, K, r, gs = spec.M, spec.K, spec.r, spec.group
    G = -(-K // gs)
    return 2 * M * K + M * gs * G // 2 + 4 * M * G + 4 * M * r + 4 * K + 2 * K * r


class ClockSampler:
    """nvidia-smi clocks and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for nm, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def _dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return rank, world, local


def _max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device="cuda" if torch.cuda.is_available() else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------------ CPU oracle leg
def oracle_timing(specs, budget_s: float = 12.0, seed_rows: int = 4):
    """Time the CPU oracle (as it stands) on a bounded row sample of every layer
    with pre-packed weights; returns (ops/s, cores, sample description)."""
    from oracle import hsq_oracle as O
    try:
        from threadpoolctl import threadpool_info
        cores = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:
        cores = os.cpu_count() or 1
    packed = []
    for spec in specs:
        lay = make_layer(spec)
        Wn, sn = lay.W.float().numpy(), lay.s.numpy()
        L1n = lay.L1.float().numpy() if spec.r else None
        L2n = lay.L2.float().numpy() if spec.r else None
        wc, ws = O.pack_weights(Wn, sn, L1n, L2n, spec.group)
        packed.append((spec, lay.X.float().numpy(), sn, L1n, L2n, wc, ws))

    def run(rows):
        t0 = time.perf_counter()
        ops = 0
        for spec, X, sn, L1n, L2n, wc, ws in packed:
            m = min(rows, spec.M)
            xc, xs, U = O.quantize_act(X[:m], sn, L1n, spec.group)
            O.linear_forward(xc, xs, U, wc, ws, L2n, None, spec.group)
            ops += layer_ops(spec) * m / spec.M
        return time.perf_counter() - t0, ops

    rows = seed_rows
    max_rows = min(s.M for s in specs)
    dt, ops = run(rows)
    while dt < budget_s / 2 and rows < max_rows:
        rows = min(max_rows, rows * 2)
        dt, ops = run(rows)
    return ops / dt, cores, f"first {rows} token rows of each layer, weights pre-packed ({dt:.1f} s of CPU work)", dt


def run_reference(args, specs, wl_name, rank, world):
    if rank != 0:
        return
    per_step = []
    sample = None
    cores = 1
    for i in range(args.warmup + args.steps):
        v, cores, sample, dt = oracle_timing(specs, budget_s=max(2.0, 60.0 / max(1, args.steps + args.warmup)))
        if i >= args.warmup:
            per_step.append((v, dt))
    v = statistics.median([p[0] for p in per_step])
    tops = v / 1e12
    line = {
        "impl": "reference", "metric": METRIC, "value": tops,
        "unit": "TOPS", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": statistics.median([p[1] for p in per_step]) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; layer shapes of the pages' backbones)",
        "config": {"workload": wl_name, "layers": [s.name for s in specs]},
        "cpu_baseline": {"value": tops, "unit": "TOPS", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": tops, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU leg
def run_gpu(args, specs, wl_name, rank, world, local):
    from w4a4_rank_assisted_b200 import hsq

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    d = lambda t: None if t is None else t.to(dev).contiguous()
    host_layers = [make_layer(spec) for spec in specs]

    def build_layers():
        out = []
        for spec, lay in zip(specs, host_layers):
            pl = hsq.PackedLinear(d(lay.W), d(lay.s), d(lay.L1) if spec.r else None,
                                  d(lay.L2) if spec.r else None, None, group=spec.group)
            X = d(lay.X)
            act = hsq.ActBuffers(spec.M, spec.K, spec.r, dev, group=spec.group)
            Y = torch.empty((spec.M, spec.N), dtype=torch.bfloat16, device=dev)
            out.append(dict(spec=spec, pl=pl, X=X, act=act, Y=Y, ws=pl.workspace(spec.M)))
        return out

    layers = build_layers()
    for L, lay in zip(layers, host_layers):
        L["X_host"] = lay.X.pin_memory()
        L["Y_host"] = torch.empty((L["spec"].M, L["spec"].N), dtype=torch.bfloat16).pin_memory()
    # Working sets smaller than 2 x L2 (decode sizes): the layers are replicated
    # (distinct packed weights, activations, outputs and workspaces) and the timed
    # steps and kernels cycle through the replicas, so that every launch reads
    # inputs that are not in L2 (inputs larger than L2, as a model's many layers
    # are).  Enough replicas that even one layer's launches span 2 x L2.
    ws_bytes = sum(layer_act_bytes(L["spec"]) + layer_gemm_bytes(L["spec"]) for L in layers)
    min_layer = min(layer_act_bytes(L["spec"]) + layer_gemm_bytes(L["spec"]) for L in layers)
    nrep = 1 if ws_bytes >= 2 * L2_BYTES else min(128, -(-2 * L2_BYTES // min_layer))
    replicas = [layers] + [build_layers() for _ in range(nrep - 1)]
    torch.cuda.synchronize()
    if hsq.hsq_get_device_status() != hsq.HSQ_OK:
        raise RuntimeError("device status not clean after packing")

    def launch_act(L, st):
        s = L["spec"]
        hsq.hsq_quantize_act(L["X"], L["pl"].s, L["pl"].L1, s.M, s.K, s.r, L["act"].x_codes,
                             L["act"].x_scales, L["act"].U, group=s.group, stream=st)

    def launch_gemm(L, st):
        s = L["spec"]
        hsq.hsq_linear_forward(L["act"].x_codes, L["act"].x_scales, L["act"].U, L["pl"].w_codes,
                               L["pl"].w_scales, L["pl"].L2, None, s.M, s.N, s.K, s.r, L["Y"],
                               workspace=L["ws"], ws_bytes=0 if L["ws"] is None else L["ws"].numel(),
                               group=s.group, stream=st)

    # decode sizes the single-launch forward takes (up to 4 tokens, r in {0,1,2,4}):
    # the activation step runs inside the weight-stream kernel
    fused = all(hsq.fused_supported(s.M, s.K, s.r, s.group) for s in specs)

    def launch_fused(L, st):
        s = L["spec"]
        hsq.hsq_linear_forward_fused(L["X"], L["pl"].s, L["pl"].L1, L["pl"].w_codes, L["pl"].w_scales,
                                     L["pl"].L2, None, s.M, s.N, s.K, s.r, L["Y"], group=s.group, stream=st)

    def step(st, rep=0):
        for L in replicas[rep]:
            if fused:
                launch_fused(L, st)
            else:
                launch_act(L, st)
                launch_gemm(L, st)

    # End to end: every step copies each layer's X from pinned host memory and its
    # Y back.  The copies run on their own streams (host-to-device and device-to-
    # host use the two directions of the link at once) and overlap the other
    # layers' kernels; the step ends on the compute stream once its outputs landed.
    copy_in = torch.cuda.Stream(device=dev)
    copy_out = torch.cuda.Stream(device=dev)

    def step_e2e():
        copy_in.wait_stream(stream)  # the previous step is done with the input buffers
        arrived = []
        with torch.cuda.stream(copy_in):
            for L in layers:
                L["X"].copy_(L["X_host"], non_blocking=True)
                ev = torch.cuda.Event()
                ev.record(copy_in)
                arrived.append(ev)
        for L, ev in zip(layers, arrived):
            stream.wait_event(ev)
            if fused:
                hsq.forward_fused(L["pl"], L["X"], L["Y"], stream=stream)
            else:
                hsq.forward(L["pl"], L["X"], L["act"], L["Y"], workspace=L["ws"], stream=stream)
            done = torch.cuda.Event()
            done.record(stream)
            copy_out.wait_event(done)
            with torch.cuda.stream(copy_out):
                L["Y_host"].copy_(L["Y"], non_blocking=True)
        stream.wait_stream(copy_out)  # outputs on the host before the step counts as done

    # A step (one replica's layers) is captured once into a CUDA graph and
    # replayed: at decode sizes a kernel runs for a few microseconds, less than
    # its host-side launch.
    gstream = torch.cuda.Stream(device=dev)
    gstream.wait_stream(stream)
    with torch.cuda.stream(gstream):
        for i in range(nrep):
            step(gstream, i)
    torch.cuda.synchronize()
    def capture(fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=gstream):
            fn(gstream)
        return g

    g_steps = [capture(lambda st, i=i: step(st, i)) for i in range(nrep)]
    with torch.cuda.stream(gstream):
        for k in range(max(args.warmup, nrep)):
            g_steps[k % nrep].replay()
    torch.cuda.synchronize()

    def replay_ms(g, n):
        # CUDAGraph.replay() launches on the current stream: make it gstream
        with torch.cuda.stream(gstream):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(gstream)
            for _ in range(n):
                g.replay()
            b.record(gstream)
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    # ---- timed region: exactly K steps
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    _barrier(world)
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(gstream):
        t0.record(gstream)
        for k in range(args.steps):
            g_steps[k % nrep].replay()
        t1.record(gstream)
    torch.cuda.synchronize()
    _barrier(world)
    clk = clocks.stop()
    ms_total = t0.elapsed_time(t1)
    ms_total = _max_over_ranks(ms_total, world)
    ms_step = ms_total / args.steps
    if hsq.hsq_get_device_status() != hsq.HSQ_OK:
        raise RuntimeError("a kernel reported a timeout during the timed region")

    # ---- per-kernel device time: each kernel alone, REPS launches per graph
    # (cycling through the replicas), CUDA events on the replaying stream
    def kernel_us(fn, li):
        reps = max(20, nrep)
        g = capture(lambda st: [fn(replicas[j % nrep][li], st) for j in range(reps)])
        with torch.cuda.stream(gstream):
            g.replay()
        torch.cuda.synchronize()
        return replay_ms(g, 3) * 1e3 / (3 * reps)

    if fused:  # one kernel per layer: its time is reported as the GEMM's, the activation step's as 0
        gemm_us = [kernel_us(launch_fused, li) for li in range(len(layers))]
        act_us = [0.0 for _ in layers]
    else:
        gemm_us = [kernel_us(launch_gemm, li) for li in range(len(layers))]
        act_us = [kernel_us(launch_act, li) for li in range(len(layers))]

    # ---- end to end through the public API with host buffers (no graph)
    for _ in range(max(1, args.warmup // 2)):
        step_e2e()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        step_e2e()
    e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = _max_over_ranks(e0.elapsed_time(e1) / args.steps, world)

    ops_step = sum(layer_ops(L["spec"]) for L in layers)
    tokens_step = specs[0].M
    tops = ops_step * world / (ms_step * 1e-3) / 1e12
    tops_e2e = ops_step * world / (ms_e2e * 1e-3) / 1e12
    h2d = sum(L["X_host"].numel() * 2 for L in layers)
    d2h = sum(L["Y_host"].numel() * 2 for L in layers)

    # ---- roofline of the dominant kernel (the GEMM, all layers of the step):
    # tensor-bound when its INT8 time floor exceeds its HBM floor, else HBM-bound
    peaks = _peaks()
    int8_peak = peaks["bf16_sustained"] * INT8_OVER_BF16_NOMINAL
    gemm_ops = sum(2 * L["spec"].M * L["spec"].N * L["spec"].K + 2 * L["spec"].M * L["spec"].N * L["spec"].r
                   for L in layers)
    gemm_bytes = sum((layer_fused_bytes if fused else layer_gemm_bytes)(L["spec"]) for L in layers)
    gemm_time = sum(gemm_us) * 1e-6
    # hsq_linear_forward launches two operand expansions ahead of the GEMM when
    # the codes are pre-expanded (more than 256 tokens, or more than 64 at groups
    # of 128): its time (and so the roofline) includes them
    large = [L["spec"].M > 256 or (L["spec"].M > 64 and L["spec"].group == 128) for L in layers]
    # up to 8 tokens the forward is the CUDA-core weight stream (its shared-memory
    # limit is far above these shapes' K)
    gemm_label = ("w4a4_gemm_kernel (+ 2 expand_e4m3_kernel: one hsq_linear_forward)" if any(large)
                  else "w4a4_gemv_kernel, activation step fused in (one hsq_linear_forward_fused)" if fused
                  else "w4a4_gemv_kernel" if all(L["spec"].M <= 8 for L in layers) else "w4a4_gemm_kernel")
    t_tensor = gemm_ops / (int8_peak * 1e12)
    t_hbm = gemm_bytes / (peaks["hbm_gbs"] * 1e9)
    if t_tensor >= t_hbm:
        achieved = gemm_ops / gemm_time / 1e12
        roofline = {"bound": "tensor", "kernel": gemm_label, "achieved": achieved, "peak": int8_peak,
                    "unit": "TFLOP/s", "frac": achieved / int8_peak,
                    "traffic": NCU_TRAFFIC_PER_LAUNCH.get(wl_name),
                    "peak_source": f"{peaks['source']}: bf16 sustained {peaks['bf16_sustained']} TFLOP/s x nominal "
                                   f"INT8/BF16 ratio {INT8_OVER_BF16_NOMINAL}",
                    "frac_of_spec_4500": achieved / 4500.0}
    else:
        achieved = gemm_bytes / gemm_time / 1e9
        roofline = {"bound": "hbm", "kernel": gemm_label, "achieved": achieved, "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                    "traffic": NCU_TRAFFIC_PER_LAUNCH.get(wl_name),
                    "peak_source": f"{peaks['source']} copy bandwidth", "frac_of_spec_8000": achieved / 8000.0}
    roofline["algorithmic_per_launch"] = {"ops": gemm_ops / len(layers), "bytes": gemm_bytes / len(layers)}
    layer_detail = []
    for L, g, a in zip(layers, gemm_us, act_us):
        s = L["spec"]
        gops = 2 * s.M * s.N * s.K + 2 * s.M * s.N * s.r
        layer_detail.append({"layer": s.name, "M": s.M, "K": s.K, "N": s.N, "r": s.r,
                             "gemm_us": g, "act_us": a,
                             "gemm_tops": gops / (g * 1e-6) / 1e12,
                             "gemm_gbs": (layer_fused_bytes if fused else layer_gemm_bytes)(s) / (g * 1e-6) / 1e9,
                             "act_gbs": layer_act_bytes(s) / (a * 1e-6) / 1e9 if a > 0 else None})

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample, _ = oracle_timing(specs)
        cpu = {"value": v / 1e12, "unit": "TOPS", "cores": cores, "kind": "oracle", "sample": sample}

    if rank == 0:
        line = {
            "metric": METRIC, "value": tops, "unit": "TOPS",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int4 codes on i8/e4m3 tensor cores, f32 accumulate",
            "data": "synthetic (seeded; layer shapes of the pages' backbones, random weights)",
            "config": {"workload": wl_name, "layers": [s.name for s in specs], "tokens_per_step": tokens_step,
                       "r": specs[0].r, "group": specs[0].group, "parallelism": f"replicas x{world}",
                       "fused_activation_step": fused,
                       "l2": (f"inputs larger than L2: {nrep} replicas of the step's layers (distinct weights, "
                              f"activations, outputs), steps and per-kernel launches cycle through them; "
                              f"{nrep * ws_bytes / 2**20:.0f} MiB in all, {ws_bytes / 2**20:.1f} MiB per step"
                              if nrep > 1 else
                              f"no flush; per-step working set {ws_bytes / 2**20:.0f} MiB > 2 x 126 MiB L2")},
            "tokens_per_s": tokens_step * world / (ms_step * 1e-3),
            "e2e": {"value": tops_e2e, "unit": "TOPS", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": ms_e2e},
            "gpu_launches": sum(1 if fused else 4 if big else 2 for big in large) * args.steps,
            "graph": "one step captured in a CUDA graph, replayed K times",
            "roofline": roofline,
            "layers": layer_detail,
            "cpu_baseline": cpu,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="hsq", choices=["hsq", "reference"])
    ap.add_argument("--workload", default="flux_block_r4", choices=sorted(WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl != "reference":
        args.warmup = 3
    rank, world, local = _dist_init()
    specs = WORKLOADS[args.workload]
    try:
        if args.impl == "reference":
            run_reference(args, specs, args.workload, rank, world)
        else:
            run_gpu(args, specs, args.workload, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
