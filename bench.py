#!/usr/bin/env python
"""Benchmark of the rank-r W4A4 linear layer (H-SVDQuant forward) on B200.

One step = one pass of the hot path over one batch: for every linear of the
workload, the fused activation step followed by the INT4 GEMM + low-rank/bias
epilogue, as one hsq_linear_forward_x call (X in, Y out; the same bits as
hsq_quantize_act + hsq_linear_forward), or one hsq_linear_forward_fused launch
at decode sizes; weights pre-packed, and for many tokens their E4M3 copy made
once, offline (packing is offline).  Default workload: the FLUX.1 double-stream block linears
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
FP4_OVER_BF16_NOMINAL = 4.0   # dense FP4 (9 PFLOP/s) over dense BF16, nominal

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
            + (2 * N if spec.bias else 0)            # bias (bf16; the stated workloads have none)
            + 2 * M * N)                             # Y (bf16)


def layer_fused_bytes(spec):
    """Algorithmic HBM bytes of one hsq_linear_forward_fused call: X, s, L1, the
    packed weights and their scales, L2 and Y (the activation codes, scales and U
    stay on chip)."""
    M, N, K, r, gs = spec.M, spec.N, spec.K, spec.r, spec.group
    G = -(-K // gs)
    Kp = gs * G
    return (2 * M * K + 4 * K + 2 * K * r + N * Kp // 2 + 4 * N * G + 2 * r * N + (2 * N if spec.bias else 0)
            + 2 * M * N)


def layer_act_bytes(spec):
    M, K, r, gs = spec.M, spec.K, spec.r, spec.group
    G = -(-K // gs)
    return 2 * M * K + M * gs * G // 2 + 4 * M * G + 4 * M * r + 4 * K + 2 * K * r


def _cu(res):
    """Unpack a cuda-python driver call's result, raising on an error code."""
    err, *rest = res if isinstance(res, tuple) else (res,)
    if int(err) != 0:
        raise RuntimeError(f"CUDA driver call failed: {err}")
    return rest[0] if len(rest) == 1 else rest


def time_kernel_nodes(launch, stream, name_part: str, calls: int, repeats: int = 3):
    """Device time of one kind of kernel inside a multi-kernel library call.

    ``launch(i, stream)`` issues call i (all of its kernels) on ``stream``.  The
    ``calls`` calls are captured into one CUDA graph; every kernel node whose
    name does not contain ``name_part`` is removed and the remaining nodes are
    chained in launch order, so they run one after another exactly as launched
    (same grid, arguments and inputs: the removed kernels' outputs are already
    in memory from earlier calls).  The graph is replayed ``repeats`` times
    between CUDA events on ``stream``; returns (microseconds per kept node,
    kept nodes per call)."""
    from cuda.bindings import driver as cu
    hs = cu.CUstream(stream.cuda_stream)
    _cu(cu.cuStreamBeginCapture(hs, cu.CUstreamCaptureMode.CU_STREAM_CAPTURE_MODE_RELAXED))
    try:
        for i in range(calls):
            launch(i, stream)
    finally:
        graph = _cu(cu.cuStreamEndCapture(hs))
    try:
        n = _cu(cu.cuGraphGetNodes(graph, 0))[1]
        nodes = _cu(cu.cuGraphGetNodes(graph, n))[0]
        key = lambda nd: int(nd)

        def node_deps(nd):
            # with edge data: a call whose kernels start early has programmatic edges,
            # which the plain query refuses to report
            n_d = _cu(cu.cuGraphNodeGetDependencies_v2(nd, 0))[2]
            return _cu(cu.cuGraphNodeGetDependencies_v2(nd, n_d))[0] if n_d else []

        deps = {key(nd): {key(d) for d in node_deps(nd)} for nd in nodes}
        order, placed = [], set()
        while len(order) < len(nodes):  # launch order (the capture is a chain)
            for nd in nodes:
                k = key(nd)
                if k not in placed and deps[k] <= placed:
                    order.append(nd)
                    placed.add(k)
        kept = []
        for nd in order:
            name = ""
            if _cu(cu.cuGraphNodeGetType(nd)) == cu.CUgraphNodeType.CU_GRAPH_NODE_TYPE_KERNEL:
                prm = _cu(cu.cuGraphKernelNodeGetParams(nd))
                if int(prm.func):
                    name = _cu(cu.cuFuncGetName(prm.func))
                elif int(prm.kern):
                    name = _cu(cu.cuKernelGetName(prm.kern))
                name = name.decode() if isinstance(name, bytes) else str(name)
            if name_part in name:
                kept.append(nd)
            else:
                _cu(cu.cuGraphDestroyNode(nd))
        for a, b in zip(kept[:-1], kept[1:]):  # chain the kept nodes (edges not already there)
            have = node_deps(b)
            if int(a) not in {int(x) for x in have}:
                _cu(cu.cuGraphAddDependencies(graph, [a], [b], 1))
        exe = _cu(cu.cuGraphInstantiate(graph, 0))
        try:
            _cu(cu.cuGraphLaunch(exe, hs))
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            for _ in range(repeats):
                _cu(cu.cuGraphLaunch(exe, hs))
            e1.record(stream)
            torch.cuda.synchronize()
        finally:
            _cu(cu.cuGraphExecDestroy(exe))
    finally:
        _cu(cu.cuGraphDestroy(graph))
    if not kept:
        raise RuntimeError(f"no kernel named like {name_part!r} in the call")
    return e0.elapsed_time(e1) * 1e3 / (repeats * len(kept)), len(kept) / calls


def _sms() -> int:
    return torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count


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
    from oracle import nvfp4_oracle as F
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
        if spec.fmt == "nvfp4":
            wq = F.nvfp4_pack_weights(Wn, sn, L1n, L2n)
        else:
            wq = O.pack_weights(Wn, sn, L1n, L2n, spec.group)
        packed.append((spec, lay.X.float().numpy(), sn, L1n, L2n, wq))

    def run(rows):
        t0 = time.perf_counter()
        ops = 0
        for spec, X, sn, L1n, L2n, wq in packed:
            m = min(rows, spec.M)
            if spec.fmt == "nvfp4":
                xc, xs, xg, U = F.nvfp4_quantize_act(X[:m], sn, L1n)
                F.nvfp4_linear_forward(xc, xs, xg, U, *wq, L2n, None, spec.K)
            else:
                xc, xs, U = O.quantize_act(X[:m], sn, L1n, spec.group)
                O.linear_forward(xc, xs, U, *wq, L2n, None, spec.group)
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
def _sources_sha() -> str:
    """Hash of the CUDA sources: an ncu traffic figure is reported only for the
    build it was captured from."""
    import hashlib
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "w4a4_rank_assisted_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        if f.endswith((".cu", ".cuh")):
            with open(os.path.join(csrc, f), "rb") as fh:
                h.update(f.encode() + fh.read())
    return h.hexdigest()[:16]


# DRAM read + write bytes per launch of the dominant kernel (mean over the
# step's layers) from one ncu capture, keyed by workload, with the hash of the
# CUDA sources it was captured from; any other build reports null.
NCU_TRAFFIC = {
    # w4a4_gemm_kernel, FLUX.1 block: 85.7 / 121.2 / 237.3 MB for qkv / MLP up / MLP down.  Captured on
    # sources whose only difference from these is the host's choice of kernels for ranks of 17 and more:
    # the rank-4 kernel this workload runs is the same code.
    "flux_block_r4": ("69c28b250e6de097", 148059904.0),
}


class Workload:
    """One workload on one GPU: packed layers, their replicas (decode sizes),
    one CUDA graph per replica step, and the launch helpers of the public API."""

    def __init__(self, hsq, specs, dev, host_buffers=False, fused=None):
        self.hsq, self.specs, self.dev = hsq, specs, dev
        d = lambda t: None if t is None else t.to(dev).contiguous()
        host_layers = [make_layer(spec) for spec in specs]

        def build_layers():
            out = []
            for spec, lay in zip(specs, host_layers):
                L1 = d(lay.L1) if spec.r else None
                L2 = d(lay.L2) if spec.r else None
                if spec.fmt == "nvfp4":
                    pl = hsq.Fp4Linear(d(lay.W), d(lay.s), L1, L2, None)
                    act = hsq.Fp4ActBuffers(spec.M, spec.K, spec.r, dev)
                else:
                    pl = hsq.PackedLinear(d(lay.W), d(lay.s), L1, L2, None, group=spec.group)
                    if self.expands(spec):
                        pl.expand()  # the weights' E4M3 copy, made once (offline), as a deployment would
                    act = hsq.ActBuffers(spec.M, spec.K, spec.r, dev, group=spec.group)
                Y = torch.empty((spec.M, spec.N), dtype=torch.bfloat16, device=dev)
                wsx = pl.workspace_x(spec.M) if spec.fmt == "int4" else None
                out.append(dict(spec=spec, pl=pl, X=d(lay.X), act=act, Y=Y, ws=pl.workspace(spec.M), wsx=wsx))
            return out

        self.layers = build_layers()
        if host_buffers:
            for L, lay in zip(self.layers, host_layers):
                L["X_host"] = lay.X.pin_memory()
                L["Y_host"] = torch.empty((L["spec"].M, L["spec"].N), dtype=torch.bfloat16).pin_memory()
        # Working sets smaller than 2 x L2 (decode sizes): the layers are replicated
        # (distinct packed weights, activations, outputs and workspaces) and the timed
        # steps and kernels cycle through the replicas, so that every launch reads
        # inputs that are not in L2 (inputs larger than L2, as a model's many layers
        # are).  Enough replicas that even one layer's launches span 2 x L2.
        self.ws_bytes = sum(layer_act_bytes(L["spec"]) + layer_gemm_bytes(L["spec"]) for L in self.layers)
        min_layer = min(layer_act_bytes(L["spec"]) + layer_gemm_bytes(L["spec"]) for L in self.layers)
        self.nrep = 1 if self.ws_bytes >= 2 * L2_BYTES else min(128, -(-2 * L2_BYTES // min_layer))
        self.replicas = [self.layers] + [build_layers() for _ in range(self.nrep - 1)]
        # decode sizes the single-launch forward takes: the activation step runs
        # inside the forward's kernel
        self.fp4 = all(s.fmt == "nvfp4" for s in specs)
        takes = not self.fp4 and all(hsq.fused_supported(s.M, s.K, s.r, s.group, N=s.N) for s in specs)
        self.fused = takes if fused is None else (bool(fused) and takes)
        torch.cuda.synchronize()
        if hsq.hsq_get_device_status() != hsq.HSQ_OK:
            raise RuntimeError("device status not clean after packing")
        self.gstream = torch.cuda.Stream(device=dev)

    # the public API's calls, one layer at a time
    def launch_act(self, L, st):
        s = L["spec"]
        if s.fmt == "nvfp4":
            a = L["act"]
            self.hsq.hsq_fp4_quantize_act(L["X"], L["pl"].s, L["pl"].L1, s.M, s.K, s.r, a.x_codes, a.x_sf, a.x_gs,
                                          a.U, stream=st)
            return
        self.hsq.hsq_quantize_act(L["X"], L["pl"].s, L["pl"].L1, s.M, s.K, s.r, L["act"].x_codes,
                                  L["act"].x_scales, L["act"].U, group=s.group, stream=st)

    def launch_gemm(self, L, st):
        s = L["spec"]
        if s.fmt == "nvfp4":
            a, pl = L["act"], L["pl"]
            self.hsq.hsq_fp4_linear_forward(a.x_codes, a.x_sf, a.x_gs, a.U, pl.w_codes, pl.w_sf, pl.w_gs, pl.L2, None,
                                            s.M, s.N, s.K, s.r, L["Y"], stream=st)
            return
        if L["pl"].w_e4m3 is not None:
            self.hsq.hsq_linear_forward_pre(L["act"].x_codes, L["act"].x_scales, L["act"].U, L["pl"].w_codes,
                                            L["pl"].w_scales, L["pl"].w_e4m3, L["pl"].L2, None, s.M, s.N, s.K, s.r,
                                            L["Y"], workspace=L["ws"],
                                            ws_bytes=0 if L["ws"] is None else L["ws"].numel(),
                                            group=s.group, stream=st)
            return
        self.hsq.hsq_linear_forward(L["act"].x_codes, L["act"].x_scales, L["act"].U, L["pl"].w_codes,
                                    L["pl"].w_scales, L["pl"].L2, None, s.M, s.N, s.K, s.r, L["Y"],
                                    workspace=L["ws"], ws_bytes=0 if L["ws"] is None else L["ws"].numel(),
                                    group=s.group, stream=st)

    def launch_x(self, L, st):
        """The activation step and the forward in one call (hsq_linear_forward_x)."""
        s = L["spec"]
        self.hsq.hsq_linear_forward_x(L["X"], L["pl"].s, L["pl"].L1, L["pl"].w_codes, L["pl"].w_scales,
                                      L["pl"].w_e4m3, L["pl"].L2, None, s.M, s.N, s.K, s.r, L["Y"],
                                      workspace=L["wsx"], ws_bytes=L["wsx"].numel(), group=s.group, stream=st)

    def launch_fused(self, L, st):
        s = L["spec"]
        self.hsq.hsq_linear_forward_fused(L["X"], L["pl"].s, L["pl"].L1, L["pl"].w_codes, L["pl"].w_scales,
                                          L["pl"].L2, None, s.M, s.N, s.K, s.r, L["Y"], group=s.group, stream=st)

    def step(self, st, rep=0):
        for L in self.replicas[rep]:
            if self.fused:
                self.launch_fused(L, st)
            elif L["spec"].fmt == "int4":
                self.launch_x(L, st)
            else:
                self.launch_act(L, st)
                self.launch_gemm(L, st)

    def capture(self, fn):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.gstream):
            fn(self.gstream)
        return g

    def replay_ms(self, g, n):
        # CUDAGraph.replay() launches on the current stream: make it gstream
        with torch.cuda.stream(self.gstream):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(self.gstream)
            for _ in range(n):
                g.replay()
            b.record(self.gstream)
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    def prepare_steps(self, warmup):
        """One CUDA graph per replica step (at decode sizes a kernel runs for a few
        microseconds, less than its host-side launch), warmed up."""
        self.gstream.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(self.gstream):
            for i in range(self.nrep):
                self.step(self.gstream, i)
        torch.cuda.synchronize()
        self.g_steps = [self.capture(lambda st, i=i: self.step(st, i)) for i in range(self.nrep)]
        with torch.cuda.stream(self.gstream):
            for k in range(max(warmup, self.nrep)):
                self.g_steps[k % self.nrep].replay()
        torch.cuda.synchronize()

    def timed_steps_ms(self, steps):
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.gstream):
            t0.record(self.gstream)
            for k in range(steps):
                self.g_steps[k % self.nrep].replay()
            t1.record(self.gstream)
        torch.cuda.synchronize()
        return t0.elapsed_time(t1)

    def launches_per_step(self):
        """Kernels of this library launched by one step (an NVFP4 activation step
        is two kernels and a tiny pad-zeroing kernel when M is not a multiple of 128)."""
        n = 0
        for L in self.layers:
            s = L["spec"]
            if self.fused:
                n += 1
            elif s.fmt == "nvfp4":
                n += 2 + (1 if s.M % 128 else 0) + 1
            else:
                n += 2 + (0 if not self.expands(s) else
                          (1 if s.M % 128 else 0) if self.x_tiles(s) else 1)
        return n

    @staticmethod
    def x_tiles(s):
        """hsq_linear_forward_x's activation kernel writes the GEMM's E4M3 tiles
        itself (no expansion launch; a pad-zeroing launch when M is not a
        multiple of 128): many rows, ranks 0, 1, 2, 4."""
        return s.M >= 24 * _sms() and s.r in (0, 1, 2, 4)

    @staticmethod
    def expands(s):
        """For more than 256 tokens, or more than 64 at groups of 128, the GEMM
        reads E4M3-expanded operands: the weights' copy is made once at load
        (PackedLinear.expand), the activations' per call (one more launch)."""
        return s.fmt == "int4" and (s.M > 256 or (s.M > 64 and s.group == 128))

    def kernel_times(self):
        """Per layer: device microseconds of each kernel, each timed alone over
        >= 20 launches in a CUDA graph (cycling through the replicas), CUDA events
        on the replaying stream.  For calls of several kernels the GEMM kernel and
        the expansions are also timed apart (time_kernel_nodes)."""
        reps = max(20, self.nrep)
        out = []
        for li, L in enumerate(self.layers):
            def per_call(fn):
                g = self.capture(lambda st: [fn(self.replicas[j % self.nrep][li], st) for j in range(reps)])
                with torch.cuda.stream(self.gstream):
                    g.replay()
                torch.cuda.synchronize()
                return self.replay_ms(g, 3) * 1e3 / (3 * reps)
            d = {}
            if self.fused:
                d["call_us"] = per_call(self.launch_fused)
                d["gemm_kernel_us"] = d["call_us"]
                d["act_us"] = 0.0
            elif L["spec"].fmt == "int4":
                # one call (activation step + forward): its kernels timed apart
                d["call_us"] = per_call(self.launch_x)
                call = lambda i, st: self.launch_x(self.replicas[i % self.nrep][li], st)
                d["gemm_kernel_us"], _ = time_kernel_nodes(call, self.gstream, "w4a4_gem", reps)
                d["act_us"], _ = time_kernel_nodes(call, self.gstream, "quantize_act", reps)
                if self.expands(L["spec"]) and (L["spec"].M % 128 or not self.x_tiles(L["spec"])):
                    e_us, e_n = time_kernel_nodes(call, self.gstream, "e4m3", reps)
                    d["expand_us"] = e_us * e_n  # expansion or pad-zeroing launches of one call
            else:
                d["call_us"] = per_call(self.launch_gemm)
                d["act_us"] = per_call(self.launch_act)
                d["gemm_kernel_us"] = d["call_us"]
            out.append(d)
        return out

    def roofline(self, kt, peaks, wl_name):
        """Roofline of the dominant kernel (the forward's GEMM, or the weight
        stream at decode sizes) over the step's layers, against the measured
        peaks: tensor-bound when its INT8 time floor exceeds its HBM floor."""
        specs = [L["spec"] for L in self.layers]
        # each kernel is timed alone in a short graph: the burst peaks apply; the
        # INT4 codes run on the 8-bit tensor pipe, the NVFP4 variant on the FP4 one
        ratio = FP4_OVER_BF16_NOMINAL if self.fp4 else INT8_OVER_BF16_NOMINAL
        int8_peak = peaks["bf16"] * ratio
        gemm_ops = sum(2 * s.M * s.N * s.K + 2 * s.M * s.N * s.r for s in specs)
        gemm_bytes = sum((layer_fused_bytes if self.fused else layer_gemm_bytes)(s) for s in specs)
        gemm_time = sum(d["gemm_kernel_us"] for d in kt) * 1e-6
        label = ("fp4_gemm_kernel (kind::mxf4nvf4 block-scaled)" if self.fp4
                 else "w4a4_gemv_kernel, activation step fused in (one hsq_linear_forward_fused)" if self.fused
                 else "w4a4_gemv_kernel" if all(s.M <= 8 for s in specs) else "w4a4_gemm_kernel")
        t_tensor = gemm_ops / (int8_peak * 1e12)
        t_hbm = gemm_bytes / (peaks["hbm_gbs"] * 1e9)
        tr = NCU_TRAFFIC.get(wl_name)
        traffic = tr[1] if tr and tr[0] == _sources_sha() else None
        if t_tensor >= t_hbm:
            achieved = gemm_ops / gemm_time / 1e12
            r = {"bound": "tensor", "kernel": label, "achieved": achieved, "peak": int8_peak, "unit": "TFLOP/s",
                 "frac": achieved / int8_peak, "traffic": traffic,
                 "peak_source": (f"{peaks['source']}: bf16 burst {peaks['bf16']} TFLOP/s x nominal "
                                 f"{'FP4' if self.fp4 else 'INT8'}/BF16 ratio {ratio} (each kernel timed alone)"),
                 f"frac_of_spec_{int(2250 * ratio)}": achieved / (2250.0 * ratio)}
        else:
            achieved = gemm_bytes / gemm_time / 1e9
            r = {"bound": "hbm", "kernel": label, "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                 "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                 "peak_source": f"{peaks['source']} copy bandwidth", "frac_of_spec_8000": achieved / 8000.0}
        r["algorithmic_per_launch"] = {"ops": gemm_ops / len(specs), "bytes": gemm_bytes / len(specs)}
        r["time_per_launch_us"] = gemm_time * 1e6 / len(specs)
        return r

    def layer_detail(self, kt):
        out = []
        for L, d in zip(self.layers, kt):
            s = L["spec"]
            gops = 2 * s.M * s.N * s.K + 2 * s.M * s.N * s.r
            g = d["gemm_kernel_us"]
            row = {"layer": s.name, "M": s.M, "K": s.K, "N": s.N, "r": s.r, "group": s.group,
                   "call_us": d["call_us"], "gemm_kernel_us": g, "act_us": d["act_us"],
                   "gemm_tops": gops / (g * 1e-6) / 1e12,
                   "gemm_gbs": (layer_fused_bytes if self.fused else layer_gemm_bytes)(s) / (g * 1e-6) / 1e9,
                   "act_gbs": layer_act_bytes(s) / (d["act_us"] * 1e-6) / 1e9 if d["act_us"] > 0 else None}
            if "expand_us" in d:
                row["expand_us"] = d["expand_us"]
            out.append(row)
        return out

    def l2_note(self):
        if self.nrep > 1:
            return (f"inputs larger than L2: {self.nrep} replicas of the step's layers (distinct weights, "
                    f"activations, outputs), steps and per-kernel launches cycle through them; "
                    f"{self.nrep * self.ws_bytes / 2**20:.0f} MiB in all, {self.ws_bytes / 2**20:.1f} MiB per step")
        return f"no flush; per-step working set {self.ws_bytes / 2**20:.0f} MiB > 2 x 126 MiB L2"


def run_gpu(args, specs, wl_name, rank, world, local):
    from w4a4_rank_assisted_b200 import hsq

    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    stream = torch.cuda.current_stream()
    W = Workload(hsq, specs, dev, host_buffers=True, fused=False if args.no_fused else None)
    layers = W.layers
    W.prepare_steps(args.warmup)

    # ---- timed region: exactly K steps
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    _barrier(world)
    torch.cuda.synchronize()
    ms_total = W.timed_steps_ms(args.steps)
    _barrier(world)
    clk = clocks.stop()
    ms_total = _max_over_ranks(ms_total, world)
    ms_step = ms_total / args.steps
    if hsq.hsq_get_device_status() != hsq.HSQ_OK:
        raise RuntimeError("a kernel reported a timeout during the timed region")

    kt = W.kernel_times()

    # ---- end to end through the public API with host buffers (no graph): every
    # step copies each layer's X from pinned host memory and its Y back.  The
    # copies run on their own streams (host-to-device and device-to-host use the
    # two directions of the link at once) and overlap the other layers' kernels;
    # the step ends on the compute stream once its outputs landed.
    copy_in = torch.cuda.Stream(device=dev)
    copy_out = torch.cuda.Stream(device=dev)

    # Steps are pipelined as a serving loop would run them: a layer's next input
    # copy waits only until its compute has read X, and its next compute only
    # until its previous Y is on the host, so one step's output copies overlap
    # the next step's input copies (both PCIe directions busy).  Every step still
    # copies all its inputs in and all its outputs out inside the timed region,
    # which ends once the last step's outputs are on the host.
    nl = len(layers)
    x_free, y_free = [None] * nl, [None] * nl

    def step_e2e():
        arrived = []
        for i, L in enumerate(layers):
            if x_free[i] is not None:
                copy_in.wait_event(x_free[i])
            with torch.cuda.stream(copy_in):
                L["X"].copy_(L["X_host"], non_blocking=True)
            ev = torch.cuda.Event()
            ev.record(copy_in)
            arrived.append(ev)
        for i, (L, ev) in enumerate(zip(layers, arrived)):
            stream.wait_event(ev)
            if y_free[i] is not None:
                stream.wait_event(y_free[i])
            if W.fused:
                hsq.forward_fused(L["pl"], L["X"], L["Y"], stream=stream)
            elif W.fp4:
                hsq.fp4_forward(L["pl"], L["X"], L["act"], L["Y"], stream=stream)
            else:
                hsq.forward_x(L["pl"], L["X"], L["Y"], L["wsx"], stream=stream)
            done = torch.cuda.Event()
            done.record(stream)
            x_free[i] = done
            copy_out.wait_event(done)
            with torch.cuda.stream(copy_out):
                L["Y_host"].copy_(L["Y"], non_blocking=True)
            out_done = torch.cuda.Event()
            out_done.record(copy_out)
            y_free[i] = out_done

    for _ in range(max(1, args.warmup // 2)):
        step_e2e()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    copy_in.wait_stream(stream)
    copy_out.wait_stream(stream)
    for _ in range(args.steps):
        step_e2e()
    stream.wait_stream(copy_out)  # the last step's outputs are on the host
    stream.wait_stream(copy_in)
    e1.record(stream)
    torch.cuda.synchronize()
    ms_e2e = _max_over_ranks(e0.elapsed_time(e1) / args.steps, world)

    ops_step = sum(layer_ops(L["spec"]) for L in layers)
    tokens_step = specs[0].M
    tops = ops_step * world / (ms_step * 1e-3) / 1e12
    tops_e2e = ops_step * world / (ms_e2e * 1e-3) / 1e12
    h2d = sum(L["X_host"].numel() * 2 for L in layers)
    d2h = sum(L["Y_host"].numel() * 2 for L in layers)
    peaks = _peaks()
    roofline = W.roofline(kt, peaks, wl_name)

    # ---- other workloads timed the same way (their own step graphs, cycling
    # through replicas where the step is smaller than 2 x L2; per-kernel times;
    # roofline): the decode-sized Qwen3-8B layers (1 and 16 tokens) and the FLUX.1
    # block in the NVFP4 variant
    def sub_measure(name, fused=None):
        D = Workload(hsq, WORKLOADS[name], dev, fused=fused)
        D.prepare_steps(args.warmup)
        dsteps = max(50, args.steps)
        d_ms = _max_over_ranks(D.timed_steps_ms(dsteps), world) / dsteps
        dkt = D.kernel_times()
        dops = sum(layer_ops(L["spec"]) for L in D.layers)
        out = {"ms_per_step": d_ms, "tops": dops * world / (d_ms * 1e-3) / 1e12,
               "tokens_per_s": D.specs[0].M * world / (d_ms * 1e-3),
               "fused_activation_step": D.fused, "gpu_launches_per_step": D.launches_per_step(),
               "l2": D.l2_note(), "roofline": D.roofline(dkt, peaks, name), "layers": D.layer_detail(dkt)}
        del D
        torch.cuda.empty_cache()
        if hsq.hsq_get_device_status() != hsq.HSQ_OK:
            raise RuntimeError(f"a kernel reported a timeout in the {name} measurements")
        return out

    def decode_measure(name):
        # where the single launch takes the cooperative decode tiles (form 2), it is
        # not always the faster form: time both, report the faster, keep the other
        specs_d = WORKLOADS[name]
        if not any(hsq.hsq_fused_form(s.M, s.N, s.K, s.r, s.group) == 2 for s in specs_d):
            return sub_measure(name)
        a, b = sub_measure(name, fused=True), sub_measure(name, fused=False)
        best, other = (a, b) if a["ms_per_step"] <= b["ms_per_step"] else (b, a)
        best["alternative"] = {k: other[k] for k in ("ms_per_step", "tokens_per_s", "fused_activation_step",
                                                     "gpu_launches_per_step")}
        best["alternative"]["layers"] = [{"layer": L["layer"], "call_us": L["call_us"]} for L in other["layers"]]
        return best

    decode = None if args.no_decode else {d: decode_measure(d) for d in ("qwen3_8b_m1", "qwen3_8b_m16")}
    nvfp4 = None
    if not args.no_decode and wl_name == "flux_block_r4":
        nvfp4 = {"workload": "flux_block_r4_nvfp4", **sub_measure("flux_block_r4_nvfp4")}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample, _ = oracle_timing(specs)
        cpu = {"value": v / 1e12, "unit": "TOPS", "cores": cores, "kind": "oracle", "sample": sample}

    if rank == 0:
        line = {
            "metric": METRIC, "value": tops, "unit": "TOPS",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": ("e2m1 codes, e4m3 block scales on fp4 tensor cores, f32 accumulate" if W.fp4
                      else "int4 codes on i8/e4m3 tensor cores, f32 accumulate"),
            "data": "synthetic (seeded; layer shapes of the pages' backbones, random weights)",
            "config": {"workload": wl_name, "layers": [s.name for s in specs], "tokens_per_step": tokens_step,
                       "r": specs[0].r, "group": specs[0].group, "parallelism": f"replicas x{world}",
                       "fused_activation_step": W.fused, "l2": W.l2_note()},
            "tokens_per_s": tokens_step * world / (ms_step * 1e-3),
            "e2e": {"value": tops_e2e, "unit": "TOPS", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "ms_per_step": ms_e2e},
            "gpu_launches": W.launches_per_step() * args.steps,
            "graph": "one step captured in a CUDA graph, replayed K times",
            "roofline": roofline,
            "layers": W.layer_detail(kt),
            "decode": decode,
            "nvfp4": nvfp4,
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
    ap.add_argument("--no-decode", action="store_true", help="skip the decode-size sub-measurements")
    ap.add_argument("--no-fused", action="store_true",
                    help="time the two calls (activation step, forward) even where the single launch applies")
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
