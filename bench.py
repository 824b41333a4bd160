#!/usr/bin/env python
"""Benchmark of one Laplacian-kernel Nystrom attention call (forward) on a B200.

Workload: the PVT stage-1 shape (B=32, heads=1, 56x56 grid so N=3136, d=64, 8x8 pooled
landmarks so m=49, lambda=4, eps=1e-6, T=20, bf16 Q/V/O), synthetic inputs from
laplacian_nystr_attention_avg_b200.inputs. The fused kernel computes distances and exp in fp32,
multiplies bf16 operands on the tensor cores with fp32 accumulation and runs Newton-Schulz in
split TF32; the line's "dtype" says so.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lfa|reference]

Prints ONE JSON line (rank 0). Under torchrun each rank runs its own full batch on its
own GPU (independent units, no data-path collective: weak scaling); the step time is the
max over ranks. ``--impl reference`` times the CPU oracle instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "tokens/s per Laplacian-Nyström attention call (N=3136,d=64,m=49); % of roofline"
L2_BYTES = 126 * 1024 * 1024
CLOCK_QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
               "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
               "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=4000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["lfa", "reference"], default="lfa")
    ap.add_argument("--workload", default="pvt1")
    ap.add_argument("--whiten", choices=["unit", "batch", "full"], default="unit",
                    help="column statistics per (batch, head) unit; 'batch': pooled per head over the "
                         "batch; 'full': Reading B, the columns of the whole Nystrom matrix (both on the "
                         "per-stage kernels, no CPU baseline)")
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0,
                    help="approximate CPU work of the oracle baseline sample")
    ap.add_argument("--backward", action="store_true",
                    help="time forward + backward steps instead (1 GPU; e.g. --workload long)")
    ap.add_argument("--seqsplit", action="store_true",
                    help="split every unit's grid rows over the ranks (bands; NCCL all-reduces and "
                         "neighbour exchanges); default workload long")
    return ap.parse_args()


def max_over_ranks(values, world, device=None):
    """Element-wise maximum of per-rank timings over all ranks (identity on one rank).

    Every rank calls it at the same point; with NCCL the tensor lives on the rank's GPU.
    """
    if world == 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t]


def job_tokens_per_s(world, units, N, steps, total_ms):
    """Whole-job throughput: every rank processes its own units x N tokens per step."""
    return world * units * N * steps / (total_ms * 1e-3)


def workload_config(wl, extra=None):
    cfg = {"workload": f"{wl.name}: B={wl.B} heads={wl.heads} grid={wl.H}x{wl.W} N={wl.N} d={wl.d} "
                       f"r={wl.r} m={wl.m} lambda={wl.lam:g} eps={wl.eps:g} T={wl.T} {wl.dtype} "
                       f"Q~{wl.qdist}",
           "B": wl.B, "heads": wl.heads, "H": wl.H, "W": wl.W, "N": wl.N, "d": wl.d, "r": wl.r,
           "m": wl.m, "lambda": wl.lam, "eps": wl.eps, "T": wl.T, "storage": wl.dtype,
           "whiten": "unit"}
    if extra:
        cfg.update(extra)
    return cfg


def dtype_label(path: str, kernel: str = "") -> str:
    """The arithmetic of the call (storage type aside), by the path and pass-2 kernel that serve it."""
    if path == "fused":
        return ("bf16-operand MMA (tcgen05 kind::f16), fp32 accumulate; fp32 l1 distances and exp; "
                "split-TF32 Newton-Schulz (3 tcgen05 kind::tf32 products per step)")
    if kernel == "k_stream_pass2":
        return ("fp32 l1 distances and exp; bf16-operand C^T V and C M' on tcgen05 (kind::f16), fp32 accumulate; "
                "split-TF32 tcgen05 Newton-Schulz")
    return "fp32 SIMT distances and products; split-TF32 tcgen05 Newton-Schulz"


def workspace_report(lfa, wl):
    """Device workspace of this config and of the same config at N / 4 and 4 N (grid sides halved
    and doubled, m fixed by scaling r): the linear-in-N memory claim checked on the planner."""
    import dataclasses

    rows = []
    for f in (0.5, 1, 2):
        H, W, r = int(wl.H * f), int(wl.W * f), max(1, int(wl.r * f))
        if H % r or W % r:
            continue
        w2 = dataclasses.replace(wl, H=H, W=W, r=r)
        rows.append({"N": w2.N, "m": w2.m, "bytes": lfa.workspace_size(lfa.make_config(w2))})
    return rows


def solver_report(lfa, dev):
    """Newton-Schulz (the forward's solver) against conjugate gradients on the device, both fp32, on
    synthetic SPD landmark systems with condition number 50 (m = 49, 64 right-hand sides, 3 systems):
    median relative error ||Y - W^-1 B||_F / ||W^-1 B||_F after the given steps."""
    import numpy as np
    import torch

    from laplacian_nystr_attention_avg_b200.inputs import make_spd_systems

    W, B = make_spd_systems(49, 50.0, 3, 64, seed=0)
    Wd = torch.from_numpy(W.astype(np.float32)).to(dev)
    Bd = torch.from_numpy(B.astype(np.float32)).to(dev)
    W32, B32 = W.astype(np.float32).astype(np.float64), B.astype(np.float32).astype(np.float64)
    Y = np.stack([np.linalg.solve(W32[u], B32[u]) for u in range(3)])

    def rel(Z):
        return float(np.median([np.linalg.norm(Z[u] - Y[u]) / np.linalg.norm(Y[u]) for u in range(3)]))

    out = {}
    for T in (10, 20):
        X, _ = lfa.ns_solve(Wd, T)
        out[f"ns_T{T}"] = rel(X.double().cpu().numpy() @ B32)
    for k in (10, 20, 30, 49):
        out[f"cg_{k}"] = rel(lfa.cg_solve(Wd, Bd, k).double().cpu().numpy())
    out["note"] = "median relative error of Y over 3 systems; one NS step ~ 2 m^3 multiply-adds, one CG step m^2 x 64"
    return out


def read_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f), "measured"
    except OSError:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "sm_max_mhz": 1965.0}, "fallback"


def kernel_traffic(kernel: str, workload: str):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, if its source is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    try:
        lines = open(path).read().splitlines()
    except OSError:
        return None, None
    for ln in lines:
        if ln.startswith("#") or not ln.strip():
            continue
        kv = dict(tok.split("=", 1) for tok in ln.split() if "=" in tok)
        if kv.get("kernel") != kernel or kv.get("workload") != workload:
            continue
        src = os.path.join(ROOT, kv.get("source", ""))
        try:
            sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        except OSError:
            return None, None
        if sha != kv.get("source_sha"):
            return None, "stale"
        return float(kv["dram_bytes_per_launch"]), kv.get("note")
    return None, None


class ClockSampler:
    def __init__(self, device_index: int):
        self.proc = None
        fd, self.path = tempfile.mkstemp(prefix=f"lfa_clocks_rank{device_index}_", suffix=".csv")
        os.close(fd)
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={CLOCK_QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(device_index)], stdout=self.fh, stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.fh.close()
        rows = []
        text = open(self.path).read()
        try:
            os.unlink(self.path)
        except OSError:
            pass
        for ln in text.splitlines():
            f = [c.strip() for c in ln.split(",")]
            if len(f) >= 9:
                rows.append(f)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = set()
        for r in rows:
            for i, n in enumerate(names):
                if r[5 + i].lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


def run_reference(args):
    """The CPU oracle, as it stands, on a bounded sample of units per step (rank 0 only)."""
    if int(os.environ.get("RANK", "0")) != 0:
        return
    from laplacian_nystr_attention_avg_b200.inputs import WORKLOADS, make_inputs
    from oracle import lfa_oracle as O

    wl = WORKLOADS[args.workload]
    x = make_inputs(wl)
    Q, V, w = x.Q.numpy(), x.V.numpy(), x.dwc.numpy()
    cores = os.cpu_count() or 1
    O.set_threads(cores)
    per_step = 1  # units per step: keeps --steps K --warmup W within a few minutes
    units = [u % wl.units for u in range(per_step)]
    for _ in range(args.warmup):
        O.forward(Q, V, w, wl, units=units, keep_units=False)
    t0 = time.perf_counter()
    for k in range(args.steps):
        O.forward(Q, V, w, wl, units=[(k + u) % wl.units for u in range(per_step)], keep_units=False)
    dt = time.perf_counter() - t0
    tokens = per_step * wl.N * args.steps
    value = tokens / dt
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": workload_config(wl, {"sample": f"{per_step} of {wl.units} units per step"}),
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": f"{per_step} (batch, head) unit of {wl.N} tokens per step, "
                                       f"{args.steps} steps"},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def cpu_baseline(wl, x, seconds):
    from oracle import lfa_oracle as O

    cores = os.cpu_count() or 1
    O.set_threads(cores)
    Q, V, w = x.Q.numpy(), x.V.numpy(), x.dwc.numpy()
    t0 = time.perf_counter()
    O.forward(Q, V, w, wl, units=[0], keep_units=False)
    one = time.perf_counter() - t0
    n = max(1, min(wl.units, int(seconds / max(one, 1e-3))))
    t0 = time.perf_counter()
    O.forward(Q, V, w, wl, units=list(range(n)), keep_units=False)
    dt = time.perf_counter() - t0
    # the same oracle on one core: one distance thread and one BLAS thread, a single unit
    from threadpoolctl import threadpool_limits
    O.set_threads(1)
    with threadpool_limits(limits=1):
        t0 = time.perf_counter()
        O.forward(Q, V, w, wl, units=[0], keep_units=False)
        dt1 = time.perf_counter() - t0
    O.set_threads(cores)
    return {"value": n * wl.N / dt, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{n} of {wl.units} (batch, head) units of the same workload ({n * wl.N} tokens), "
                      f"float64 numpy, {dt:.1f} s",
            "one_thread": {"value": wl.N / dt1, "unit": "tokens/s", "cores": 1,
                           "sample": f"1 unit ({wl.N} tokens), distance and BLAS threads limited to 1, "
                                     f"{dt1:.1f} s"}}


def run_backward(args):
    """Secondary measurement: one step = lfa_forward + lfa_backward (dQ, dV) on resident inputs."""
    import torch

    from laplacian_nystr_attention_avg_b200 import lfa
    from laplacian_nystr_attention_avg_b200.inputs import WORKLOADS, make_inputs

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = WORKLOADS[args.workload]
    x = make_inputs(wl, with_dO=True)
    mod = lfa.LaplacianNystromAttention(lfa.make_config(wl), x.dwc, str(dev))
    Q, V, dO = x.Q_store.to(dev), x.V_store.to(dev), x.dO_store.to(dev)
    O, dQ, dV = mod.new_output(), mod.new_output(), mod.new_output()
    for _ in range(args.warmup):
        mod.forward(Q, V, O)
        mod.backward(Q, V, dO, dQ, dV)
    torch.cuda.synchronize()
    K = args.steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    fwd_ms = bwd_ms = 0.0
    for _ in range(K):
        ev[0].record()
        mod.forward(Q, V, O)
        ev[1].record()
        mod.backward(Q, V, dO, dQ, dV)
        ev[2].record()
        torch.cuda.synchronize()
        fwd_ms += ev[0].elapsed_time(ev[1])
        bwd_ms += ev[1].elapsed_time(ev[2])
    st, _ = mod.info()
    if st != lfa.LFA_OK:
        raise RuntimeError(f"device status: {lfa.status_string(st)}")
    step_ms = (fwd_ms + bwd_ms) / K
    print(json.dumps({
        "metric": "tokens/s per forward + backward call", "value": wl.units * wl.N / (step_ms * 1e-3),
        "unit": "tokens/s", "n_gpus": 1, "steps": K, "warmup": args.warmup, "ms_per_step": step_ms,
        "forward_ms": fwd_ms / K, "backward_ms": bwd_ms / K, "higher_is_better": True,
        "dtype": dtype_label(mod.path, mod.dominant_kernel) + "; backward: fp32 SIMT main pass, split-TF32 tcgen05 reverse products",
        "data": "synthetic", "config": workload_config(wl, {"path": mod.path, "inputs": "resident, no L2 flush"}),
    }), flush=True)


def run_seqsplit(args):
    """One step = one forward of the whole workload with every unit's grid rows split over the ranks
    (laplacian_nystr_attention_avg_b200.seqsplit: band calls of the library, NCCL exchanges).
    Total work is fixed as ranks are added (strong scaling); value = all tokens / max-over-ranks time."""
    import datetime

    import torch
    import torch.distributed as dist

    from laplacian_nystr_attention_avg_b200 import lfa, seqsplit
    from laplacian_nystr_attention_avg_b200.inputs import WORKLOADS, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    wl = WORKLOADS[args.workload if args.workload != "pvt1" else "long"]
    x = make_inputs(wl)
    y0, ny = seqsplit.band_rows(wl.H, world, rank)
    band = lfa.SeqSplitBand(lfa.make_config(wl), y0, ny, x.dwc, str(dev))
    sl = slice(y0 * wl.W, (y0 + ny) * wl.W)
    Qh = x.Q_store[:, :, sl].contiguous().pin_memory()
    Vh = x.V_store[:, :, sl].contiguous().pin_memory()
    Q, V = Qh.to(dev), Vh.to(dev)
    O = torch.empty_like(Q)
    comm = seqsplit.TorchComm(rank, world)
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        seqsplit.forward_rank(band, Q, V, O, comm, wl.W)
    K = args.steps
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    clocks = ClockSampler(local)
    time.sleep(0.3)
    t0.record(stream)
    for _ in range(K):
        seqsplit.forward_rank(band, Q, V, O, comm, wl.W)
    t1.record(stream)
    barrier()
    clk = clocks.stop()
    ms = max_over_ranks([t0.elapsed_time(t1)], world, dev)[0]
    # end to end: this band's Q, V from pinned host memory and O back, every step
    Oh = torch.empty(Qh.shape, dtype=Qh.dtype).pin_memory()
    E = max(1, args.e2e_steps // 10)
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(E):
        Q.copy_(Qh, non_blocking=True)
        V.copy_(Vh, non_blocking=True)
        seqsplit.forward_rank(band, Q, V, O, comm, wl.W)
        Oh.copy_(O, non_blocking=True)
    e1.record(stream)
    barrier()
    e2e_ms = max_over_ranks([e0.elapsed_time(e1)], world, dev)[0]
    tokens = wl.units * wl.N
    if rank == 0:
        nbytes = Qh.numel() * Qh.element_size()
        print(json.dumps({
            "metric": f"tokens/s per Laplacian-Nyström attention call (N={wl.N},d={wl.d},m={wl.m}), "
                      f"grid rows split over ranks", "value": tokens * K / (ms * 1e-3), "unit": "tokens/s",
            "n_gpus": world, "steps": K, "warmup": args.warmup, "ms_per_step": ms / K, "higher_is_better": True,
            "scaling": "strong", "vs_baseline": None,
            "dtype": dtype_label("generic", "k_stream_pass2" if wl.dtype == "bf16" and wl.d == 64 else ""),
            "data": "synthetic",
            "config": workload_config(wl, {"path": "generic (band calls)", "parallelism": f"seqsplit{world}",
                                           "bands": [seqsplit.band_rows(wl.H, world, k) for k in range(world)],
                                           "l2": "inputs resident; no flush"}),
            "e2e": {"value": tokens * E / (e2e_ms * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": 2 * nbytes * world, "d2h_bytes_per_step": nbytes * world},
            "gpu_launches": K * int(band.lib.lfa_launches_per_forward(band.handle)), "clocks": clk}), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


def main():
    args = parse_args()
    if args.impl == "reference":
        run_reference(args)
        return
    if args.backward:
        run_backward(args)
        return
    if args.seqsplit:
        run_seqsplit(args)
        return
    import torch
    import torch.distributed as dist

    from laplacian_nystr_attention_avg_b200 import lfa
    from laplacian_nystr_attention_avg_b200.inputs import WORKLOADS, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    wl = WORKLOADS[args.workload]
    x = make_inputs(wl, seed=rank)
    mod = lfa.LaplacianNystromAttention(lfa.make_config(wl, True if args.whiten == "unit" else args.whiten),
                                        x.dwc, str(dev))
    set_bytes = 3 * wl.units * wl.N * wl.d * x.Q_store.element_size()
    n_sets = max(2, math.ceil(1.8 * L2_BYTES / set_bytes))
    Qs = [x.Q_store.to(dev) for _ in range(n_sets)]
    Vs = [x.V_store.to(dev) for _ in range(n_sets)]
    Os = [mod.new_output() for _ in range(n_sets)]
    stream = torch.cuda.current_stream()

    for k in range(args.warmup):
        mod.forward(Qs[k % n_sets], Vs[k % n_sets], Os[k % n_sets])
    st, info = mod.info()
    if st != lfa.LFA_OK:
        raise RuntimeError(f"device status after warm-up: {lfa.status_string(st)}")
    kappas = sorted(float(i.kappa) for i in info)

    K = args.steps
    t_begin = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier()
    clocks = ClockSampler(local)
    time.sleep(0.3)
    t_begin.record(stream)
    for k in range(K):
        mod.forward(Qs[k % n_sets], Vs[k % n_sets], Os[k % n_sets])
    t_end.record(stream)
    barrier()
    # the dominant kernel's launch duration: a second pass with the library's timing hook armed
    # (events recorded around that one kernel on the launching stream), kept out of `value`
    Kk = min(K, 1000)
    kb = [torch.cuda.Event(enable_timing=True) for _ in range(Kk)]
    ke = [torch.cuda.Event(enable_timing=True) for _ in range(Kk)]
    for k in range(Kk):
        mod.set_profile_events(kb[k], ke[k])
        mod.forward(Qs[k % n_sets], Vs[k % n_sets], Os[k % n_sets])
    barrier()
    clk = clocks.stop()
    mod.set_profile_events(None, None)
    total_ms = t_begin.elapsed_time(t_end)
    kern_ms = statistics.fmean(kb[k].elapsed_time(ke[k]) for k in range(Kk))
    total_ms, kern_ms = max_over_ranks([total_ms, kern_ms], world, dev)
    ms_per_step = total_ms / K
    value = job_tokens_per_s(world, wl.units, wl.N, K, total_ms)

    # end to end through the host-buffer entry point: pinned host Q, V -> device -> O -> host, every
    # step. Two handles on two streams take alternate steps (lfa_forward_host_async), each with its own
    # pinned host and device buffers, so one step's copies overlap the other's forward and copies; the
    # timed region ends when both streams have drained.
    mod2 = lfa.LaplacianNystromAttention(lfa.make_config(wl, True if args.whiten == "unit" else args.whiten),
                                         x.dwc, str(dev))
    mods = (mod, mod2)
    streams = (stream, torch.cuda.Stream(device=dev))
    host = [(x.Q_store.pin_memory(), x.V_store.pin_memory(), torch.empty(x.Q_store.shape,
                                                                         dtype=x.Q_store.dtype).pin_memory())
            for _ in range(2)]
    devb = [(Qs[i % n_sets], Vs[i % n_sets], Os[i % n_sets]) for i in range(2)]

    def e2e_steps(n):
        for k in range(n):
            i = k % 2
            mods[i].forward_host_async(*host[i], *devb[i], stream=streams[i])

    E = args.e2e_steps
    e2e_steps(4)
    barrier()
    e_b = torch.cuda.Event(enable_timing=True)
    e_e = torch.cuda.Event(enable_timing=True)
    e_b.record(streams[0])
    streams[1].wait_event(e_b)
    e2e_steps(E)
    streams[0].wait_stream(streams[1])
    e_e.record(streams[0])
    barrier()
    e2e_ms = max_over_ranks([e_b.elapsed_time(e_e)], world, dev)[0]
    e2e_value = job_tokens_per_s(world, wl.units, wl.N, E, e2e_ms)
    del mod2
    nbytes = wl.units * wl.N * wl.d * x.Q_store.element_size()

    if rank == 0:
        peaks, peak_kind = read_peaks()
        props = torch.cuda.get_device_properties(dev)
        sms = props.multi_processor_count
        f_max = float(peaks.get("sm_max_mhz", 1965.0)) * 1e6
        alu_peak = sms * 128 * f_max                      # FP32-pipe lane-instructions / s
        alg_instr = 2.0 * wl.units * wl.N * wl.m * wl.d   # one |q - l| sub + abs-add per element
        achieved = alg_instr / (kern_ms * 1e-3)
        traffic, tnote = kernel_traffic(mod.dominant_kernel, wl.name)
        hbm = float(peaks["hbm_gbs"]) * 1e9
        io_bytes = 3.0 * nbytes
        t_roof = max(alg_instr / alu_peak, io_bytes / hbm)
        line = {
            "metric": METRIC if wl.name == "pvt1" else
            f"tokens/s per Laplacian-Nyström attention call (N={wl.N},d={wl.d},m={wl.m}); % of roofline",
            "value": value, "unit": "tokens/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": dtype_label(mod.path, mod.dominant_kernel), "data": "synthetic",
            "config": workload_config(wl, {
                "path": mod.path, "whiten": args.whiten,
                "parallelism": f"replicas{world}" if world > 1 else "single",
                "l2": f"{n_sets} rotating input/output sets of {set_bytes / 2**20:.1f} MiB "
                      f"({n_sets * set_bytes / 2**20:.0f} MiB > 126 MiB L2), no flush",
                "call_roofline_frac": t_roof / (ms_per_step * 1e-3),
                "call_roofline_us": t_roof * 1e6}),
            "roofline": {"bound": "alu", "kernel": mod.dominant_kernel, "achieved": achieved / 1e12,
                         "peak": alu_peak / 1e12, "unit": "Tinstr/s", "frac": achieved / alu_peak,
                         "traffic": traffic,
                         "peak_note": f"{sms} SMs x 128 FP32 lanes x {f_max / 1e6:.0f} MHz "
                                      f"(sm_max_mhz, {peak_kind}); algorithmic work = 2 B*heads*N*m*d "
                                      f"FP32 instructions per launch",
                         "kernel_us": kern_ms * 1e3},
            "e2e": {"value": e2e_value, "unit": "tokens/s", "h2d_bytes_per_step": 2 * nbytes,
                    "d2h_bytes_per_step": nbytes,
                    "note": "lfa_forward_host_async from pinned host buffers, steps alternating over two "
                            "handles and streams"},
            "gpu_launches": K * mod.launches_per_forward,
            "clocks": clk,
            "side_reports": {
                "kappa_W_eps": {"min": kappas[0], "median": statistics.median(kappas), "max": kappas[-1],
                                "note": "kappa_2(W + eps I) per unit after the forward: ||W||_2 (power "
                                        "iteration) x ||X_T||_2 with X_T ~ (W + eps I)^-1"},
                "workspace_bytes": workspace_report(lfa, wl),
                "solvers_kappa50": solver_report(lfa, dev),
            },
        }
        if world == 1 and not args.no_cpu_baseline and args.whiten == "unit":
            line["cpu_baseline"] = cpu_baseline(wl, x, args.cpu_seconds)
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
