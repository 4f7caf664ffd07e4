#!/usr/bin/env python
"""Throughput of the fused weighted GNN aggregation step on B200.

A step is one pass of the whole per-call hot path over one batch of inputs on
a lowered (fixed) topology: forward Y = A_w X, feature gradient
dX = A_w^T dY and weight gradient dw_e = dot(X[src_e], dY[dst_e]), through
ag_step (the forward pass and the fused backward pass of ag_backward in one
call, the two overlapped).  ag_spmm_fwd and ag_backward, and the separate
ag_spmm_dx and ag_sddmm_dw entry points, are timed after the step for the
per-kernel breakdown.  The default workload is
the R-MAT scale-22 graph (4,194,304 nodes, 67,108,864 edges, H = 128, bf16
features with fp32 accumulation), whose inputs (X and dY are 1 GiB each) are
larger than L2, so no flush is needed between steps.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs an independent replica (the path has no
exchange step); the reported value is the sum over ranks of the E*H per step
divided by the slowest rank's time.  --impl reference times the fp64 CPU
oracle on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import datetime
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

import workloads  # noqa: E402

METRIC = "E·H/s for SpMM fwd, dX and SDDMM dw; achieved HBM GB/s as % of B200 peak"
UNIT = "E*H/s"
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=["ours", "reference"], default="ours")
    p.add_argument("--workload", default="rmat22", choices=list(workloads.CONFIGS))
    p.add_argument("--seed", type=int, default=1)
    p.add_argument("--rmat-scale", type=int, default=None,
                   help="override the R-MAT scale (smaller cases for profiling)")
    p.add_argument("--e2e-steps", type=int, default=None, help="steps of the host-buffer measurement")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-rows", action="store_true",
                   help="skip the timings of mean, GCN weights and attention reported beside the step")
    p.add_argument("--cpu-seconds", type=float, default=12.0, help="target oracle time per sample")
    p.add_argument("--profile-once", action="store_true",
                   help="lower the graph once and call every entry point once, without timing "
                        "(a short launch sequence for profilers)")
    return p.parse_args()


# ----------------------------------------------------------------------------- helpers

def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def algorithmic_bytes(N, E, H, elem):
    """Minimal bytes of one call: CSR + order map + weights + input rows read
    once + output rows written once (dw: both index arrays, dw, X and dY once;
    fused backward: transpose CSR + order map + w + dw + X and dY read once +
    dX written once)."""
    spmm = 4 * (N + 1) + 4 * E + 4 * E + 4 * E + 2 * N * H * elem
    dw = 8 * E + 4 * E + 2 * N * H * elem
    backward = 4 * (N + 1) + 4 * E + 4 * E + 4 * E + 4 * E + 3 * N * H * elem
    return {"fwd": spmm, "dx": spmm, "dw": dw, "backward": backward}


def row_bytes(N, E, H, elem):
    """Minimal bytes of one call of the further aggregators: mean as the
    weighted sum; GCN weights read the forward row pointers and both COO
    index arrays and write the weights; attention forward reads the forward
    CSR (row pointers, columns, order map), Q, K and V once and writes Y and
    alpha; its backward reads both CSRs, alpha, Q, K, V and dY once and writes
    dQ, dK and dV."""
    algo = algorithmic_bytes(N, E, H, elem)
    csr = 4 * (N + 1) + 8 * E
    return {"mean_fwd": algo["fwd"], "mean_backward": algo["backward"],
            "gcn_norm": 4 * (N + 1) + 8 * E + 4 * E,
            "attn_fwd": csr + 4 * E + 4 * N * H * elem,
            "attn_backward": 2 * csr + 4 * E + 7 * N * H * elem}


def launches_per_step_of(st, wl):
    """Kernels one step (ag_step) launches, the same as ag_spmm_fwd followed by
    ag_backward: forward = weight regroup + tile walk (+ fixup when rows span
    tiles); backward on the single-walk shapes (the whole width in one lane
    group pass, as for H=128) = weight regroup + fused walk (+ fixup) + dw
    regroup back to COO order."""
    if wl.E == 0:
        return int(wl.N > 0) * 2
    fwd = 2 + int(st["spanning_rows_f"] > 0)
    bwd = 3 + int(st["spanning_rows_t"] > 0)
    return fwd + bwd


STEP_SOURCES = ("aggregate.cu", "device_common.cuh", "internal.h", "lower.cu")


def code_only(text):
    """C/C++ source without comments, trailing blanks or empty lines: the part
    of a file the compiler sees."""
    out, i, n = [], 0, len(text)
    while i < n:
        c = text[i]
        if text.startswith("//", i):
            i = text.find("\n", i)
            i = n if i < 0 else i
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
            out.append(" ")
        elif c in "\"'":
            j = i + 1
            while j < n and text[j] != c:
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(c)
            i += 1
    lines = (ln.rstrip() for ln in "".join(out).splitlines())
    return "\n".join(ln for ln in lines if ln)


def source_hash():
    """Hash of the code (comments left out) of the step's kernels and of the
    schedule they walk: a traffic record taken on other code is not reported."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "gnn_sparse_aggregation_b200", "csrc")
    for fn in STEP_SOURCES:
        with open(os.path.join(csrc, fn), encoding="utf-8") as f:
            h.update(fn.encode() + code_only(f.read()).encode())
    return h.hexdigest()[:16]


def dram_frac(dram_bytes, ms, peak_gbs):
    """Measured DRAM bytes per call over the call's time, as a fraction of the peak."""
    return dram_bytes / (ms / 1e3) / 1e9 / peak_gbs


def traffic_key(args):
    return args.workload if args.rmat_scale is None else f"{args.workload}@scale{args.rmat_scale}"


def ncu_record(workload, kernel_op):
    """The committed ncu record of one entry point, if it was taken on the
    current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            d = json.load(f)
        rec = d.get(workload, {}).get(kernel_op)
        if rec and rec.get("source_hash") == source_hash():
            return rec
    except Exception:
        pass
    return None


def ncu_traffic(workload, kernel_op):
    """DRAM bytes per launch from a committed ncu capture (else None)."""
    rec = ncu_record(workload, kernel_op)
    return rec.get("bytes_per_launch") if rec else None


def ncu_l2_hit(workload, kernel_op):
    """L2 sector hit rate of the entry point's walk from the committed
    small-case capture (R-MAT scale 20: the counter takes several passes),
    with the kernel and the case it was taken on (else None)."""
    rec = ncu_record(workload, kernel_op)
    return rec.get("l2_hit") if rec else None


class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons during the timed
    region: sampled every 20 ms, and only the samples whose timestamps fall
    between the region's first launch and its end are kept (the sampler
    starts early and stops late; its samples of the idle GPU around the
    region would otherwise dilute the median under load)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.t0 = self.t1 = None
        self.out = tempfile.NamedTemporaryFile(prefix="clocks", suffix=".csv", delete=False)

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=self.out, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def begin(self):
        """Marks the start of the region (call right before its first launch)."""
        self.t0 = datetime.datetime.now()

    def end(self):
        """Marks the end of the region (call after its final synchronize)."""
        self.t1 = datetime.datetime.now()

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        self.out.flush()
        try:
            rows = [ln.split(",") for ln in open(self.out.name).read().splitlines() if ln.strip()]
        finally:
            os.unlink(self.out.name)
        parsed = []
        for r in rows:
            r = [x.strip() for x in r]
            if len(r) < 10:
                continue
            try:
                stamp = datetime.datetime.strptime(r[0], "%Y/%m/%d %H:%M:%S.%f")
                parsed.append((stamp, float(r[2]), float(r[3]), r[6:10]))
            except ValueError:
                continue
        window = "timed region"
        inside = [p for p in parsed if self.t0 and self.t1 and self.t0 <= p[0] <= self.t1]
        if not inside:  # a region shorter than the sampling interval
            inside, window = parsed, "around the timed region"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "window": window}
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = {name for p in inside for name, val in zip(names, p[3]) if val.lower().startswith("active")}
        return {"sm_mhz": statistics.median(p[1] for p in inside), "sm_max_mhz": max(p[2] for p in inside),
                "reasons": sorted(reasons), "samples": len(inside), "window": window}


def max_over_ranks(x: float, device) -> float:
    """The slowest rank's value (every rank calls this at the same point)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(world: int, units_per_step: int, steps: int, ms: float) -> float:
    """Units all ranks processed divided by the slowest rank's time."""
    return world * units_per_step * steps / (ms / 1e3)


# ----------------------------------------------------------------------------- oracle timing

def oracle_sample(wl, target_seconds: float):
    """A bounded sample of the workload for the fp64 CPU oracle: the first S
    COO edges with their endpoints relabelled compactly (the per-edge work is
    unchanged; only untouched rows are dropped).  S is chosen so that one
    fwd + dX + dw pass takes about target_seconds on one core."""
    import oracle
    H = wl.H
    # calibrate on a small prefix
    def make(S):
        src = wl.src[:S].cpu().numpy()
        dst = wl.dst[:S].cpu().numpy()
        nodes, inv = np.unique(np.concatenate([src, dst]), return_inverse=True)
        s_loc = inv[:S].astype(np.int32)
        d_loc = inv[S:].astype(np.int32)
        idx = torch.from_numpy(nodes).to(wl.X.device).long()
        X = wl.X[idx].float().cpu().numpy()
        dY = wl.dY[idx].float().cpu().numpy()
        w = wl.w[:S].cpu().numpy()
        return int(nodes.size), s_loc, d_loc, w, X, dY

    def run(sample):
        n, s, d, w, X, dY = sample
        t0 = time.perf_counter()
        oracle.fwd(s, d, n, w, X)
        oracle.dx(s, d, n, w, dY)
        oracle.dw(s, d, n, X, dY)
        return time.perf_counter() - t0

    S = min(wl.E, 1 << 16)
    t = run(make(S))
    if S < wl.E:
        S = int(min(wl.E, max(S, S * target_seconds / max(t, 1e-6))))
    sample = make(S)
    return S, sample, run


# ----------------------------------------------------------------------------- arms

def reference_arm(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    device = "cuda" if torch.cuda.is_available() else "cpu"
    wl = workloads.make(args.workload, seed=args.seed, device=device, rmat_scale=args.rmat_scale)
    S, sample, run = oracle_sample(wl, args.cpu_seconds / max(1, args.steps) * 2)
    for _ in range(args.warmup):
        run(sample)
    t = [run(sample) for _ in range(args.steps)]
    total = sum(t)
    value = S * wl.H * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": workload_config(wl, args),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": 1, "host_cores": os.cpu_count(), "kind": "oracle",
                         "sample": f"first {S} of {wl.E} COO edges (endpoints relabelled), "
                                   f"fwd+dX+dw per step, H={wl.H}"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(wl, args):
    name = wl.name if args.rmat_scale is None else f"{wl.name} at R-MAT scale {args.rmat_scale}"
    return {"workload": f"{name}: N={wl.N}, E={wl.E}, H={wl.H}, "
                        f"features {str(wl.feature_dtype).replace('torch.', '')}",
            "N": wl.N, "E": wl.E, "H": wl.H,
            "feature_dtype": str(wl.feature_dtype).replace("torch.", ""),
            "weights": "fp32, COO order", "seed": args.seed,
            "l2": "inputs larger than L2 (X and dY exceed 126 MB), no flush" if wl.N * wl.H * (
                2 if wl.feature_dtype == torch.bfloat16 else 4) > (126 << 20) else
                  "inputs smaller than L2: warm-L2 numbers",
            "l2_persistence": "not set (no access policy window, default L2 set-aside)",
            "step": "ag_step: forward (ag_spmm_fwd) and fused backward (ag_backward: dX and dw) in one call, "
                    "the two passes overlapped, on a lowered graph; value = E*H per step / step time"}


def profile_once(args):
    """One lowering, then each entry point once (step calls, the separate
    gradients, mean, GCN weights weighted and unweighted, attention forward
    and backward), in that order, with a synchronize at the end."""
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (there is no CPU fallback)")
    from __graft_entry__ import build_library
    build_library()
    import gnn_sparse_aggregation_b200 as agb
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = workloads.make(args.workload, seed=args.seed, device=dev, rmat_scale=args.rmat_scale)
    g = agb.ag_graph_lower(wl.src, wl.dst, wl.N)
    Y, dX = torch.empty_like(wl.X), torch.empty_like(wl.dY)
    dw, wn = torch.empty_like(wl.w), torch.empty_like(wl.w)
    mk = lambda s: workloads.features(wl.N, wl.H, wl.feature_dtype, 11000 + s, dev)
    Q, Kf, V = mk(1), mk(2), mk(3)
    Ya, dQ, dK, dV = (torch.empty_like(wl.X) for _ in range(4))
    alpha = torch.empty(wl.E, dtype=torch.float32, device=dev)
    scale = 1.0 / wl.H ** 0.5
    agb.ag_spmm_fwd(g, wl.w, wl.X, Y)
    agb.ag_backward(g, wl.w, wl.X, wl.dY, dX, dw)
    agb.ag_spmm_dx(g, wl.w, wl.dY, dX)
    agb.ag_sddmm_dw(g, wl.X, wl.dY, dw)
    agb.ag_mean_fwd(g, wl.w, wl.X, Y)
    agb.ag_mean_backward(g, wl.w, wl.X, wl.dY, dX, dw)
    agb.ag_gcn_norm(g, wl.w, wn)
    agb.ag_gcn_norm(g, None, wn)
    agb.ag_attn_fwd(g, Q, Kf, V, scale, Ya, alpha)
    agb.ag_attn_backward(g, Q, Kf, V, scale, alpha, wl.dY, dQ, dK, dV)
    torch.cuda.synchronize()
    print(f"profile-once done: {wl.name} N={wl.N} E={wl.E} H={wl.H}", flush=True)
    g.close()
    return 0


def our_arm(args):
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (there is no CPU fallback)")
    torch.cuda.set_device(local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    from __graft_entry__ import build_library
    if rank == 0 or world == 1:
        build_library()
    if world > 1:
        dist.barrier()
    import gnn_sparse_aggregation_b200 as agb

    dev = torch.device("cuda", local)
    wl = workloads.make(args.workload, seed=args.seed, device=dev, rmat_scale=args.rmat_scale)
    stream = torch.cuda.current_stream(dev)

    # lowering (once per topology; reported, not part of the step).  The first
    # call also pays the library's one-time CUDA module loading, so it is
    # timed separately from a second, warm lowering of the same topology.  The
    # first graph is released before the second lowering, so that its
    # workspace comes from torch's cache rather than from a new device
    # allocation, whose time varies from run to run.
    lower_ms = []
    g = None
    for _ in range(2):
        if g is not None:
            g.close()
            g = None
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        g = agb.ag_graph_lower(wl.src, wl.dst, wl.N)
        lower_ms.append(1e3 * (time.perf_counter() - t0))
    st = g.stats

    Y = torch.empty_like(wl.X)
    dX = torch.empty_like(wl.dY)
    dw = torch.empty(wl.E, dtype=torch.float32, device=dev)
    g.scratch(wl.H)

    ops = ("fwd", "backward")
    agb.ag_step(g, wl.w, wl.X, wl.dY, Y, dX, dw)  # allocates the step's scratch once

    def step():
        # forward + fused backward in one call (the two passes overlapped)
        agb.ag_step(g, wl.w, wl.X, wl.dY, Y, dX, dw)

    for _ in range(max(3, args.warmup)):
        step()
    torch.cuda.synchronize()

    K = args.steps
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk:
        clk.begin()
        start.record(stream)
        for k in range(K):
            step()
        end.record(stream)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        clk.end()
    clocks = clk.summary()
    ms = start.elapsed_time(end)
    ms = max_over_ranks(ms, dev)

    # the entry points of the step one by one, and the separate gradient
    # entry points, for the per-kernel breakdown (not in the step)
    def timed(fn, reps):
        for _ in range(2):
            fn()
        e = [torch.cuda.Event(enable_timing=True) for _ in range(reps + 1)]
        torch.cuda.synchronize()
        e[0].record(stream)
        for i in range(reps):
            fn()
            e[i + 1].record(stream)
        torch.cuda.synchronize()
        return [e[i].elapsed_time(e[i + 1]) for i in range(reps)]

    per_op = {}
    per_op["fwd"] = timed(lambda: agb.ag_spmm_fwd(g, wl.w, wl.X, Y), K)
    per_op["backward"] = timed(lambda: agb.ag_backward(g, wl.w, wl.X, wl.dY, dX, dw), K)
    per_op["dx"] = timed(lambda: agb.ag_spmm_dx(g, wl.w, wl.dY, dX), K)
    per_op["dw"] = timed(lambda: agb.ag_sddmm_dw(g, wl.X, wl.dY, dw), K)

    # the further aggregators on the same graph (reported beside the step, not in it)
    rows = {}
    if not args.no_rows:
        Kr = max(3, min(K, 10))
        mk = lambda s: workloads.features(wl.N, wl.H, wl.feature_dtype, 11000 + s, dev)
        Q, Kf, V = mk(1), mk(2), mk(3)
        Ya, dQ, dK, dV = (torch.empty_like(wl.X) for _ in range(4))
        alpha = torch.empty(wl.E, dtype=torch.float32, device=dev)
        scale = 1.0 / wl.H ** 0.5
        wn = torch.empty_like(wl.w)
        calls = {
            "mean_fwd": lambda: agb.ag_mean_fwd(g, wl.w, wl.X, Y),
            "mean_backward": lambda: agb.ag_mean_backward(g, wl.w, wl.X, wl.dY, dX, dw),
            "gcn_norm": lambda: agb.ag_gcn_norm(g, None, wn),
            "attn_fwd": lambda: agb.ag_attn_fwd(g, Q, Kf, V, scale, Ya, alpha),
            "attn_backward": lambda: agb.ag_attn_backward(g, Q, Kf, V, scale, alpha, wl.dY, dQ, dK, dV),
        }
        rb = row_bytes(wl.N, wl.E, wl.H, wl.X.element_size())
        for name, fn in calls.items():
            t = timed(fn, Kr)
            avg_ms = sum(t) / len(t)
            gbs = rb[name] / (avg_ms / 1e3) / 1e9
            rows[name] = {"ms": avg_ms, "algorithmic_bytes": rb[name], "GB_per_s": gbs,
                          "frac_of_peak": gbs / peaks()[0], "calls": Kr}
        del Q, Kf, V, Ya, dQ, dK, dV, alpha, wn

    # end to end from host buffers, copies inside the timed region
    e2e = None
    Ke = args.e2e_steps if args.e2e_steps is not None else min(K, 20)
    if Ke > 0:
        hw, hX, hdY = (t.cpu().pin_memory() for t in (wl.w, wl.X, wl.dY))
        # two staging buffers, two streams and two sets of host outputs, used
        # in turn: a step's copies in wait only for the backward pass two
        # steps back, so they overlap the previous step's compute and copies
        # out (each call orders its own copies on its stream)
        outs = [(torch.empty_like(hX).pin_memory(), torch.empty_like(hX).pin_memory(),
                 torch.empty_like(hw).pin_memory()) for _ in range(2)]
        nbytes = agb.ag_step_staging_bytes(g, wl.H, wl.X.dtype)
        stagings = [torch.empty(nbytes, dtype=torch.uint8, device=dev) for _ in range(2)]
        streams = [torch.cuda.Stream(dev) for _ in range(2)]

        def host_step(i):
            b = i % 2
            hY, hdX, hdw = outs[b]
            agb.ag_step_host_pipelined(g, hw, hX, hdY, hY, hdX, hdw, stagings[b], stream=streams[b])

        for i in range(2):
            host_step(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(stream)
        for s in streams:
            s.wait_stream(stream)
        for i in range(Ke):
            host_step(i)
        for s in streams:
            stream.wait_stream(s)
        e1.record(stream)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1), dev)
        elem = hX.element_size()
        e2e = {"value": whole_job_rate(world, wl.E * wl.H, Ke, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": hw.numel() * 4 + 2 * hX.numel() * elem,
               "d2h_bytes_per_step": 2 * hX.numel() * elem + outs[0][2].numel() * 4,
               "steps": Ke, "ms_per_step": e_ms / Ke,
               "api": "ag_step_host_pipelined, two staging buffers on two streams in turn"}
        del stagings, outs, hw, hX, hdY

    hbm, peak_kind = peaks()
    elem = wl.X.element_size()
    algo = algorithmic_bytes(wl.N, wl.E, wl.H, elem)
    avg = {op: sum(v) / len(v) for op, v in per_op.items()}
    dominant = max(ops, key=avg.get)
    kernels = {}
    for op in per_op:
        gbs = algo[op] / (avg[op] / 1e3) / 1e9
        kernels[op] = {"ms": avg[op], "EH_per_s": wl.E * wl.H / (avg[op] / 1e3),
                       "algorithmic_bytes": algo[op], "GB_per_s": gbs, "frac_of_peak": gbs / hbm}
        dram = ncu_traffic(traffic_key(args), op)
        if dram:  # measured DRAM bytes of the call (ncu) over its live time: the DRAM fraction
            kernels[op]["dram_bytes"] = dram
            kernels[op]["dram_frac_of_peak"] = dram_frac(dram, avg[op], hbm)
        hit = ncu_l2_hit(traffic_key(args), op)
        if hit:
            kernels[op]["l2_hit"] = hit
    traffic = ncu_traffic(traffic_key(args), dominant)
    launches_per_step = launches_per_step_of(st, wl)
    line = {
        "metric": METRIC,
        "value": whole_job_rate(world, wl.E * wl.H, K, ms),
        "unit": UNIT,
        "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms / K,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": workload_config(wl, args),
        "roofline": {"bound": "hbm", "kernel": dominant,
                     "achieved": algo[dominant] / (avg[dominant] / 1e3) / 1e9,
                     "peak": hbm, "unit": "GB/s",
                     "frac": algo[dominant] / (avg[dominant] / 1e3) / 1e9 / hbm,
                     "peak_source": f"{peak_kind} hbm_gbs",
                     "traffic": traffic,
                     "dram_frac": dram_frac(traffic, avg[dominant], hbm) if traffic else None,
                     "l2_hit": ncu_l2_hit(traffic_key(args), dominant)},
        "kernels": kernels,
        "lowering_ms": lower_ms[1], "lowering_first_call_ms": lower_ms[0],
        "schedule": {k: st[k] for k in ("tile_edges", "tiles", "spanning_rows_f", "long_spanning_rows_f",
                                        "spanning_rows_t", "long_spanning_rows_t", "max_degree_f",
                                        "max_degree_t")},
        "gpu_launches": launches_per_step * K,
        "rows": rows,
        "clocks": clocks,
        "e2e": e2e,
    }
    if world > 1:
        dist.barrier()

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        S, sample, run = oracle_sample(wl, args.cpu_seconds)
        secs = run(sample)
        line["cpu_baseline"] = {"value": S * wl.H / secs, "unit": UNIT, "cores": 1, "host_cores": os.cpu_count(),
                                "kind": "oracle",
                                "sample": f"first {S} of {wl.E} COO edges (endpoints relabelled), "
                                          f"one fwd+dX+dw pass, H={wl.H}, {secs:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    g.close()
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    if args.impl == "reference":
        return reference_arm(args)
    if args.profile_once:
        return profile_once(args)
    return our_arm(args)


if __name__ == "__main__":
    sys.exit(main())
