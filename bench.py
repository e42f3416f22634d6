#!/usr/bin/env python
"""Benchmark of the fused attention forward + JVP on B200.

One step = one call of the whole path (one kernel launch) over one batch of a
named synthetic workload (default: T2V self-attention, B=1 H=40 L=32760
d=128, the largest single-GPU configuration).  Prints ONE JSON line on rank 0.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                  [--impl ours|reference] [--no-cpu-baseline]

Metric: TFLOP/s counted as 12 * Lq * Lk * d per (b, h), over the valid keys.
Multi-GPU (torchrun): every rank runs its own copy of the workload (seed =
rank), no collective on the data path ("weak" scaling); value = all ranks'
FLOPs / the slowest rank's time.

``--impl reference`` times the fp64 CPU oracle on the host cores on a bounded
row sample of the same workload (rank 0 only).

The roofline object names the bound from the workload's arithmetic intensity
(FLOPs performed over algorithmic bytes) against the ridge point of the two
measured peaks, and carries both the tensor and the HBM fraction.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import math
import os
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = ("attention fwd+JVP TFLOP/s (12·Lq·Lk·d/head) and % of B200 BF16 "
          "dense peak")
UNIT = "TFLOP/s"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"bf16_tflops": 1590.0, "hbm_gbs": 6650.0}
# the sources each timed kernel is built from (a traffic record counts only
# while their hash is unchanged)
KERNEL_SOURCES = ["attention_jvp_fwd_b200/csrc/attn_jvp_fwd.cu",
                  "attention_jvp_fwd_b200/csrc/sm100.cuh"]
LOSS_SOURCES = ["attention_jvp_fwd_b200/csrc/scm_loss.cu", "attention_jvp_fwd_b200/csrc/sm100.cuh"]
QKV_SOURCES = ["attention_jvp_fwd_b200/csrc/qkv_prologue.cu", "attention_jvp_fwd_b200/csrc/sm100.cuh"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: about 10 s of kernel time for the workload)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="t2v_self")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle baseline sample")
    ap.add_argument("--e2e-steps", type=int, default=0, help="0 = min(steps, 100)")
    ap.add_argument("--no-split", action="store_true",
                    help="walk every query tile whole (no last-wave key split)")
    args = ap.parse_args(argv)
    if args.steps is None:
        args.steps = DEFAULT_STEPS.get(args.workload, 1000)
    return args


# default timed steps per workload: about 10 s of kernel time (T2V is 54 ms
# a launch), 1000 launches elsewhere
DEFAULT_STEPS = {"t2v_self": 200}


# ----------------------------------------------------------------- helpers

def kernel_source_hash(sources=None) -> str:
    h = hashlib.sha256()
    for p in sources or KERNEL_SOURCES:
        with open(os.path.join(ROOT, p), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def load_peaks():
    """(burst bf16 TFLOP/s, sustained bf16 TFLOP/s or None, HBM GB/s, source)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            pk = json.load(f)
        sus = pk.get("bf16_tflops_sustained")
        return (float(pk["bf16_tflops"]), float(sus) if sus else None, float(pk["hbm_gbs"]),
                "measured")
    except (OSError, KeyError, ValueError):
        return FALLBACK_PEAKS["bf16_tflops"], None, FALLBACK_PEAKS["hbm_gbs"], "fallback"


# A timed region this long runs the GPU into its power cap, like the
# seconds-long cuBLAS loop behind the sustained peak.
SUSTAINED_MS = 500.0


def measured_traffic(workload: str, sources=None):
    """DRAM bytes per launch from a committed ncu capture, if it was taken on
    the current kernel source (else None)."""
    try:
        with open(TRAFFIC_FILE) as f:
            t = json.load(f)
    except (OSError, ValueError):
        return None
    e = t.get(workload)
    if not e or e.get("source_sha256") != kernel_source_hash(sources):
        return None
    return e.get("dram_bytes_per_launch")


def algorithmic_bytes(w) -> float:
    """Bytes the method must move per launch: read Q, Q' and the valid rows of
    K, K', V, V' once (K, V only when K' = V' = 0), write O, O' (bf16) and
    lse (fp32)."""
    BH = w.B * w.H
    n_valid = (np.clip(w.kv_len, 0, w.Lk).astype(np.int64) * w.H).sum() if w.kv_len is not None \
        else BH * w.Lk
    kv_tensors = 2 if w.zero_kv_dot else 4
    return float(2 * w.d * (2 * BH * w.Lq + kv_tensors * n_valid) + 4 * BH * w.Lq * w.d
                 + 4 * BH * w.Lq)


class ClockSampler:
    """nvidia-smi sampling of SM clock and throttle reasons during the timed region."""
    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        # nvidia-smi numbers GPUs without regard to CUDA_VISIBLE_DEVICES, so
        # the device is named by its UUID (else its PCI bus id)
        self.gpu_id = smi_device_id(device)
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(prefix="bench_clocks_", suffix=".csv")
            self.f = os.fdopen(fd, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_id}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.f.close()
        rows = []
        with open(self.path) as f:
            lines = f.readlines()
        try:
            os.unlink(self.path)
        except OSError:
            pass
        for line in lines:
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                rows.append({"sm": float(parts[2]), "max": float(parts[3]),
                             "power": float(parts[4]),
                             "hw": parts[6], "hw_th": parts[7], "sw_th": parts[8],
                             "sw_pc": parts[9]})
            except ValueError:
                continue
        if not rows:
            return None
        load = [r for r in rows if r["power"] > 200.0] or rows
        reasons = set()
        for r in load:
            for k, name in (("hw", "hw_slowdown"), ("hw_th", "hw_thermal_slowdown"),
                            ("sw_th", "sw_thermal_slowdown"), ("sw_pc", "sw_power_cap")):
                if r[k].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": float(np.median([r["sm"] for r in load])),
                "sm_max_mhz": float(max(r["max"] for r in rows)),
                "reasons": sorted(reasons), "samples": len(load), "gpu": self.gpu_id}


def smi_device_id(device) -> str:
    """The nvidia-smi --id of a torch CUDA device: 'GPU-<uuid>', else the PCI
    bus id, else the CUDA ordinal."""
    import torch
    props = torch.cuda.get_device_properties(device)
    uuid = str(getattr(props, "uuid", "") or "")
    if uuid:
        return uuid if uuid.startswith("GPU-") else "GPU-" + uuid
    if hasattr(props, "pci_bus_id"):
        return "%08x:%02x:%02x.0" % (props.pci_domain_id, props.pci_bus_id, props.pci_device_id)
    return str(torch.device(device).index or 0)


def roofline_bound(flops: float, nbytes: float, peak_tf: float, peak_hbm_gbs: float) -> str:
    """'tensor' when the arithmetic intensity (FLOP per algorithmic byte) is
    above the ridge point of the two peaks, else 'hbm'."""
    ridge = peak_tf * 1e12 / (peak_hbm_gbs * 1e9)
    return "tensor" if flops / nbytes > ridge else "hbm"


# ----------------------------------------------------------------- distributed

def dist_setup():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def aggregate(local_ms: float, local_flops: float, group_active: bool, device=None):
    """Max of the per-rank times and sum of the per-rank FLOPs across ranks."""
    if not group_active:
        return local_ms, local_flops
    import torch
    import torch.distributed as dist
    t = torch.tensor([local_ms], dtype=torch.float64, device=device)
    f = torch.tensor([local_flops], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    dist.all_reduce(f, op=dist.ReduceOp.SUM)
    return float(t.item()), float(f.item())


E2E_NOTE = ("pipelined stream: every step copies its inputs host->device (pinned) and its "
            "outputs device->host; two device buffer sets and three CUDA streams let step i+1's "
            "input copies and step i-1's output copies overlap step i")


def stream_e2e(dev, host_ins, out_like, call, steps, group):
    """End-to-end time (ms) of a streaming loop through the public API.

    Every step copies its inputs from pinned host memory to the device, runs
    `call(dev_inputs, dev_outputs, stream)` and copies its outputs back to
    pinned host memory.  Two device buffer sets and three streams (input
    copies, compute, output copies) let the next step's inputs and the
    previous step's outputs cross PCIe, in both directions at once, while a
    step computes, as a user streaming batches would.  The timed region runs
    from the first input copy to the last output copy."""
    import torch
    import torch.distributed as dist
    slots_in = [[torch.empty(h.shape, dtype=h.dtype, device=dev) for h in host_ins] for _ in range(2)]
    slots_out = [[torch.empty_like(o) for o in out_like] for _ in range(2)]
    host_out = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in out_like]
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_comp = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]
    torch.cuda.synchronize(dev)
    if group:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(steps):
        k = i % 2
        if i >= 2:
            s_in.wait_event(ev_comp[k])  # step i-2's kernel has read these inputs
        with torch.cuda.stream(s_in):
            for dst, src in zip(slots_in[k], host_ins):
                dst.copy_(src, non_blocking=True)
        ev_in[k].record(s_in)
        s_comp.wait_event(ev_in[k])
        if i >= 2:
            s_comp.wait_event(ev_out[k])  # step i-2's outputs have left the device
        call(slots_in[k], slots_out[k], s_comp)
        ev_comp[k].record(s_comp)
        s_out.wait_event(ev_comp[k])
        with torch.cuda.stream(s_out):
            for dst, src in zip(host_out, slots_out[k]):
                dst.copy_(src, non_blocking=True)
        ev_out[k].record(s_out)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    return e0.elapsed_time(e1)


# ----------------------------------------------------------------- CPU oracle

# The oracle runs the whole workload when a probe says that takes at most
# this long; otherwise it runs a row sample and its rate stands for the rest.
FULL_ORACLE_S = 60.0


def time_oracle(w, seconds: float, seed: int = 123):
    """Time the fp64 oracle: the whole workload if the probe's estimate is at
    most FULL_ORACLE_S, else a random row sample sized for about `seconds`.
    Returns (TFLOP/s, cores, rows run, seconds, sample description)."""
    import oracle
    rng = np.random.default_rng(seed)
    total_rows = w.B * w.H * w.Lq
    cores = oracle.max_threads()
    probe = min(total_rows, max(cores * 4, 64))
    rows = np.sort(rng.choice(total_rows, size=probe, replace=False)).astype(np.int64)
    t0 = time.perf_counter()
    oracle.attn_jvp(*w.inputs(), w.scale, kv_len=w.kv_len, rows=rows)
    dt = max(time.perf_counter() - t0, 1e-6)
    est_full = dt * total_rows / probe
    if est_full <= FULL_ORACLE_S:
        t0 = time.perf_counter()
        oracle.attn_jvp(*w.inputs(), w.scale, kv_len=w.kv_len)
        dt = time.perf_counter() - t0
        v = w.flops_valid() / dt / 1e12
        return v, cores, total_rows, dt, f"full run of {w.name} ({total_rows} query rows), {dt:.1f} s"
    n = int(min(total_rows, max(probe, probe * seconds / dt)))
    rows = np.sort(rng.choice(total_rows, size=n, replace=False)).astype(np.int64)
    t0 = time.perf_counter()
    oracle.attn_jvp(*w.inputs(), w.scale, kv_len=w.kv_len, rows=rows)
    dt = time.perf_counter() - t0
    v = row_flops(w, rows) / dt / 1e12
    full_s = w.flops_valid() / (v * 1e12)
    return v, cores, n, dt, (f"{n} random query rows of {w.name} (of {total_rows}, all keys of each), "
                             f"{dt:.1f} s; a full run would take about {full_s:.0f} s at this rate "
                             f"(extrapolated, not run)")


def row_flops(w, rows) -> float:
    b = (np.asarray(rows) // (w.H * w.Lq)).astype(np.int64)
    n = np.full(b.shape, w.Lk, np.int64) if w.kv_len is None else \
        np.clip(w.kv_len.astype(np.int64)[b], 0, w.Lk)
    return float(12.0 * w.d * n.sum())


def run_reference(args):
    ws, rank, _ = dist_setup()
    if rank != 0:
        return 0
    import oracle
    from attention_jvp_fwd_b200 import workloads as W
    w = W.make(args.workload, seed=args.seed)
    total_rows = w.B * w.H * w.Lq
    cores = oracle.max_threads()
    rng = np.random.default_rng(7)
    # calibrate the cost of one row, then size every step so the whole
    # warm-up + timed run stays near `budget` seconds
    probe = np.sort(rng.choice(total_rows, size=min(total_rows, 2 * cores), replace=False))
    t0 = time.perf_counter()
    oracle.attn_jvp(*w.inputs(), w.scale, kv_len=w.kv_len, rows=probe)
    per_row = (time.perf_counter() - t0) / len(probe)
    budget = 120.0
    rows_per_step = int(max(1, min(total_rows, budget / (args.steps + args.warmup) / per_row)))
    samples = [np.sort(rng.choice(total_rows, size=rows_per_step, replace=False))
               for _ in range(args.steps + args.warmup)]
    for s in samples[:args.warmup]:
        oracle.attn_jvp(*w.inputs(), w.scale, kv_len=w.kv_len, rows=s)
    flops = 0.0
    t0 = time.perf_counter()
    for s in samples[args.warmup:]:
        oracle.attn_jvp(*w.inputs(), w.scale, kv_len=w.kv_len, rows=s)
        flops += row_flops(w, s)
    dt = time.perf_counter() - t0
    value = flops / dt / 1e12
    sample = (f"{rows_per_step} random query rows per step of {args.workload} "
              f"(of {total_rows}), all keys of each row; fp64 oracle, OpenMP")
    line = {"metric": METRIC, "value": value, "unit": UNIT, "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": workload_config(w, args),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def workload_config(w, args):
    in_bytes = 2 * w.d * (2 * w.B * w.H * w.Lq + (2 if w.zero_kv_dot else 4) * w.B * w.H * w.Lk)
    return {"workload": w.name, "B": w.B, "H": w.H, "Lq": w.Lq, "Lk": w.Lk, "d": w.d,
            "scale": w.scale, "kv_len": None if w.kv_len is None else w.kv_len.tolist(),
            "seed": args.seed, "input_bytes": in_bytes,
            "l2": ("inputs exceed L2 (%.0f MB > 126 MB), no flush" % (in_bytes / 1e6))
            if in_bytes > L2_BYTES else "L2 flushed between steps"}


# ----------------------------------------------------------------- our arm

def run_ours(args):
    import torch
    import torch.distributed as dist

    ws, rank, local = dist_setup()
    group = ws > 1
    if group:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)

    from attention_jvp_fwd_b200.build import build
    if rank == 0 or not group:
        build()
    if group:
        dist.barrier()
    import attention_jvp_fwd_b200 as A
    from attention_jvp_fwd_b200 import workloads as W

    w = W.make(args.workload, seed=args.seed + rank)
    # with K' = V' = 0 for every batch the call passes None for them and the
    # library runs its zero-tangent kernel; those tensors are never copied
    zkv = w.zero_kv_dot
    host = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory()
            for i, x in enumerate(w.inputs()) if not (zkv and i in (4, 5))]
    ins = [h.to(dev, non_blocking=True) for h in host]
    kv = torch.from_numpy(w.kv_len).to(dev) if w.kv_len is not None else None
    B, H, Lq, d = w.B, w.H, w.Lq, w.d
    o = torch.empty((B, H, Lq, d), dtype=torch.bfloat16, device=dev)
    od = torch.empty_like(o)
    lse = torch.empty((B, H, Lq), dtype=torch.float32, device=dev)
    in_bytes = sum(x.numel() * 2 for x in ins)
    flush = None
    if in_bytes <= L2_BYTES:
        flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=dev)
    stream = torch.cuda.Stream(dev)
    flops_step = w.flops_valid()

    call_ins = ins[:4] + [None, None] if zkv else ins
    # the last-wave key split's workspace, allocated once outside the timed region
    ws_bytes = 0 if args.no_split else A.attn_jvp_workspace_bytes(B, H, Lq, w.Lk, d, device=dev)
    split_ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else None

    def step():
        A.attn_jvp_fwd(*call_ins, scale=w.scale, kv_len=kv, out=(o, od, lse), stream=stream, workspace=split_ws,
                       split=not args.no_split)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
            if flush is not None:
                flush.zero_()
    torch.cuda.synchronize(dev)
    st, site = A.attn_jvp_check(stream)
    if st != 0:
        raise RuntimeError(f"device status {st} at site {site} after warm-up")

    sampler = ClockSampler(dev)
    sampler.start()
    time.sleep(0.6)
    if group:
        dist.barrier()
    torch.cuda.synchronize(dev)
    ev = []
    if flush is None:
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        with torch.cuda.stream(stream):
            for _ in range(args.steps):
                step()
        e1.record(stream)
        torch.cuda.synchronize(dev)
        kernel_ms_total = e0.elapsed_time(e1)
    else:
        with torch.cuda.stream(stream):
            for _ in range(args.steps):
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                flush.zero_()
                a.record(stream)
                step()
                b.record(stream)
                ev.append((a, b))
        torch.cuda.synchronize(dev)
        kernel_ms_total = sum(a.elapsed_time(b) for a, b in ev)
    if group:
        dist.barrier()
    clocks = sampler.stop()
    st, site = A.attn_jvp_check(stream)
    if st != 0:
        raise RuntimeError(f"device status {st} at site {site} in the timed region")

    local_ms = kernel_ms_total
    max_ms, total_flops = aggregate(local_ms, flops_step * args.steps, group, dev)
    value = total_flops / (max_ms * 1e-3) / 1e12

    # end to end: pinned host inputs -> device, kernel, outputs -> pinned host
    e2e_steps = args.e2e_steps or min(args.steps, 100)

    def e2e_call(di, do, st):
        ci = di[:4] + [None, None] if zkv else di
        A.attn_jvp_fwd(*ci, scale=w.scale, kv_len=kv, out=tuple(do), stream=st, workspace=split_ws,
                       split=not args.no_split)

    e2e_local = stream_e2e(dev, host, (o, od, lse), e2e_call, e2e_steps, group)
    e2e_ms, e2e_flops = aggregate(e2e_local, flops_step * e2e_steps, group, dev)
    e2e_value = e2e_flops / (e2e_ms * 1e-3) / 1e12
    h2d = in_bytes
    d2h = (o.numel() + od.numel()) * 2 + lse.numel() * 4

    burst_tf, sustained_tf, peak_hbm, peak_src = load_peaks()
    if sustained_tf is not None and local_ms >= SUSTAINED_MS:
        peak_tf, peak_kind = sustained_tf, "sustained"
    else:
        peak_tf, peak_kind = burst_tf, "burst"
    per_launch_ms = local_ms / args.steps
    # the roofline counts what the kernel performs: 8 units with K' = V' = 0
    achieved = w.flops_performed() / (per_launch_ms * 1e-3) / 1e12
    traffic = measured_traffic(args.workload)
    alg_bytes = algorithmic_bytes(w)
    achieved_gbs = alg_bytes / (per_launch_ms * 1e-3) / 1e9
    bound = roofline_bound(w.flops_performed(), alg_bytes, peak_tf, peak_hbm)
    tensor_side = {"achieved": achieved, "peak": peak_tf, "unit": UNIT, "frac": achieved / peak_tf,
                   "frac_of_burst_peak": achieved / burst_tf,
                   "peak_source": f"{peak_src} bf16 dense ({peak_kind}; timed region {local_ms:.0f} ms)"}
    hbm_side = {"achieved": achieved_gbs, "peak": peak_hbm, "unit": "GB/s",
                "frac": achieved_gbs / peak_hbm, "peak_source": f"{peak_src} HBM copy bandwidth"}
    main_side, other_side = (tensor_side, hbm_side) if bound == "tensor" else (hbm_side, tensor_side)
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": workload_config(w, args),
        "gpu_launches": args.steps,
        "roofline": {"bound": bound, **main_side,
                     "traffic": traffic,
                     "algorithmic_bytes": alg_bytes,
                     "flops_per_launch": w.flops_performed(),
                     "intensity_flop_per_byte": w.flops_performed() / alg_bytes,
                     "ridge_flop_per_byte": peak_tf * 1e12 / (peak_hbm * 1e9),
                     "tensor" if bound == "hbm" else "hbm": other_side,
                     "kernel": f"attn_jvp_fwd_kernel<{d}>"},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": e2e_steps, "how": E2E_NOTE},
        "clocks": clocks,
    }
    line["config"]["last_wave_split_workspace_bytes"] = ws_bytes
    if w.kv_len is not None:
        line["config"]["flops_nominal_per_step"] = w.flops_nominal()
    if zkv:
        line["config"]["zero_kv_dot"] = True
        line["config"]["note"] = ("K' = V' = 0 for every batch: the zero-tangent kernel runs 8 of "
                                  "the 12 FLOP units; value counts the metric's 12 units, "
                                  "roofline.achieved the 8 performed")
    if rank == 0 and not group and not args.no_cpu_baseline:
        v, cores, n, dt, sample = time_oracle(w, args.cpu_seconds)
        line["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle",
                                "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if group:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------- sCM loss

LOSS_METRIC = "sCM tangent-normalised loss GB/s (f, f_ema, g read once, grad written)"
# T2V latents: Wan2.1 480p, 832x480x81 frames -> 16 channels x 21 x 60 x 104
LOSS_SHAPE = (16, 16, 21, 60, 104)


def loss_inputs(seed: int):
    from attention_jvp_fwd_b200.workloads import bf16_round_bits
    r = np.random.default_rng([seed, 11])
    fe = r.standard_normal(LOSS_SHAPE, dtype=np.float32)
    f = fe + np.float32(0.1) * r.standard_normal(LOSS_SHAPE, dtype=np.float32)
    g = r.standard_normal(LOSS_SHAPE, dtype=np.float32)
    return [bf16_round_bits(x) for x in (f, fe, g)]


def run_loss(args):
    """``--workload scm_loss``: the tangent-normalised sCM loss kernel, an
    HBM-bound streaming reduction, on T2V-sized latents."""
    import torch
    import torch.distributed as dist

    ws, rank, local = dist_setup()
    group = ws > 1
    if group:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from attention_jvp_fwd_b200.build import build
    if rank == 0 or not group:
        build()
    if group:
        dist.barrier()
    import attention_jvp_fwd_b200 as A

    bits = loss_inputs(args.seed + rank)
    host = [torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).pin_memory() for b in bits]
    ins = [h.to(dev, non_blocking=True) for h in host]
    B = LOSS_SHAPE[0]
    N = int(np.prod(LOSS_SHAPE[1:]))
    loss = torch.empty(B, dtype=torch.float32, device=dev)
    grad = torch.empty_like(ins[0])
    stream = torch.cuda.Stream(dev)
    bytes_step = 4.0 * B * N * 2 + 4 * B  # inputs > L2, so no flush is needed

    def step():
        A.scm_tangent_loss(*ins, out=(loss, grad), stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize(dev)
    sampler = ClockSampler(dev)
    sampler.start()
    time.sleep(0.6)
    if group:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    local_ms = e0.elapsed_time(e1)
    clocks = sampler.stop()
    max_ms, total_bytes = aggregate(local_ms, bytes_step * args.steps, group, dev)
    value = total_bytes / (max_ms * 1e-3) / 1e9

    e2e_steps = args.e2e_steps or min(args.steps, 100)

    def e2e_call(di, do, st):
        A.scm_tangent_loss(*di, out=tuple(do), stream=st)

    e2e_local = stream_e2e(dev, host, (loss, grad), e2e_call, e2e_steps, group)
    e2e_ms, e2e_bytes = aggregate(e2e_local, bytes_step * e2e_steps, group, dev)

    _, _, hbm, peak_src = load_peaks()
    achieved = bytes_step / (local_ms / args.steps * 1e-3) / 1e9
    line = {
        "metric": LOSS_METRIC, "value": value, "unit": "GB/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "scm_loss", "shape": list(LOSS_SHAPE), "c": 0.1, "seed": args.seed,
                   "l2": "inputs exceed L2 (%.0f MB > 126 MB), no flush" % (3 * B * N * 2 / 1e6)
                   if 3 * B * N * 2 > L2_BYTES else "inputs fit in L2: the number is L2-assisted"},
        "gpu_launches": args.steps,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": hbm,
                     "peak_source": f"{peak_src} HBM copy bandwidth", "unit": "GB/s",
                     "frac": achieved / hbm, "traffic": measured_traffic("scm_loss", LOSS_SOURCES),
                     "algorithmic_bytes": bytes_step,
                     "kernel": "scm_loss_kernel<1>"},
        "e2e": {"value": e2e_bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": 3 * B * N * 2, "d2h_bytes_per_step": B * N * 2 + 4 * B,
                "steps": e2e_steps, "how": E2E_NOTE},
        "clocks": clocks,
    }
    if rank == 0 and not group and not args.no_cpu_baseline:
        from oracle import scm_loss
        t0 = time.perf_counter()
        n = 0
        while time.perf_counter() - t0 < min(args.cpu_seconds, 10.0) or n == 0:
            scm_loss.scm_tangent_loss(*[b[n % B:n % B + 1].reshape(1, -1) for b in bits])
            n += 1
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": n * 4.0 * N * 2 / dt / 1e9, "unit": "GB/s", "cores": 1,
                                "kind": "oracle",
                                "sample": f"{n} single-sample calls of numpy fp64, {dt:.1f} s"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if group:
        dist.barrier()
        dist.destroy_process_group()
    return 0


# ----------------------------------------------------------------- QKV prologue

QKV_METRIC = "QKV projection + RMSNorm forward-and-tangent TFLOP/s (2 GEMMs, 2*2*T*D*3*H*d)"
# Cosmos-Predict2-2B-like layer on the T2I tokens: D = 2048, 16 heads of 128
QKV_SHAPE = dict(B=2, L=4096, H=16, D=2048, d=128)


def qkv_inputs(seed: int):
    """Seeded bf16 bits of x, x' [T, D] (N(0, 1)) and W [3Hd, D] (N(0, 1/D))."""
    from attention_jvp_fwd_b200.workloads import bf16_round_bits
    B, L, H, D, d = (QKV_SHAPE[k] for k in ("B", "L", "H", "D", "d"))
    T = B * L
    r = np.random.default_rng([seed, 13])
    return [bf16_round_bits(r.standard_normal((T, D), dtype=np.float32)),
            bf16_round_bits(r.standard_normal((T, D), dtype=np.float32)),
            bf16_round_bits((r.standard_normal((3 * H * d, D)) / np.sqrt(D)).astype(np.float32))]


def time_qkv_oracle(bits, seconds: float):
    """The fp64 prologue oracle on the first `n` tokens per call (all heads),
    n sized for about `seconds`; returns (TFLOP/s, tokens per call, calls, s)."""
    from oracle import qkv_prologue
    H, D, d = QKV_SHAPE["H"], QKV_SHAPE["D"], QKV_SHAPE["d"]
    x, xd, w = bits
    one = np.ones(d)
    n, calls, dt = 16, 0, 0.0
    while True:
        t0 = time.perf_counter()
        qkv_prologue.qkv_rmsnorm_jvp(x[:n], xd[:n], w, one, one, 1, n, H, d)
        dt1 = time.perf_counter() - t0
        if dt1 > seconds / 8 or n >= x.shape[0]:
            break
        n = min(x.shape[0], n * 2)
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds or calls == 0:
        qkv_prologue.qkv_rmsnorm_jvp(x[:n], xd[:n], w, one, one, 1, n, H, d)
        calls += 1
    dt = time.perf_counter() - t0
    flops = 2.0 * 2 * n * D * 3 * H * d * calls
    return flops / dt / 1e12, n, calls, dt


def run_reference_qkv(args):
    """``--impl reference --workload qkv_t2i``: the fp64 oracle of the prologue
    on the host cores, on bounded token samples of the same layer."""
    _, rank, _ = dist_setup()
    if rank != 0:
        return 0
    bits = qkv_inputs(args.seed)
    per_step = max(1.0, min(20.0, 120.0 / (args.steps + args.warmup)))
    time_qkv_oracle(bits, per_step * args.warmup / max(1, args.steps))  # warm-up
    v, n, calls, dt = time_qkv_oracle(bits, per_step * args.steps)
    sample = (f"first {n} tokens of the layer (all {3 * QKV_SHAPE['H']} head tiles) per call, "
              f"{calls} calls, {dt:.1f} s; numpy fp64")
    line = {"metric": QKV_METRIC, "value": v, "unit": "TFLOP/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "qkv_t2i", **QKV_SHAPE, "seed": args.seed},
            "cpu_baseline": {"value": v, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": v, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_reference_loss(args):
    """``--impl reference --workload scm_loss``: the fp64 oracle of the loss on
    the host cores, one sample per call."""
    _, rank, _ = dist_setup()
    if rank != 0:
        return 0
    from oracle import scm_loss
    bits = loss_inputs(args.seed)
    B = LOSS_SHAPE[0]
    N = int(np.prod(LOSS_SHAPE[1:]))
    budget = max(1.0, min(20.0, 120.0 / (args.steps + args.warmup)))
    for i in range(args.warmup):
        scm_loss.scm_tangent_loss(*[b[i % B:i % B + 1].reshape(1, -1) for b in bits])
    n = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget * args.steps or n == 0:
        scm_loss.scm_tangent_loss(*[b[n % B:n % B + 1].reshape(1, -1) for b in bits])
        n += 1
    dt = time.perf_counter() - t0
    v = n * (4.0 * N * 2 + 4) / dt / 1e9
    line = {"metric": LOSS_METRIC, "value": v, "unit": "GB/s", "impl": "reference",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": dt * 1e3 / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": "scm_loss", "shape": list(LOSS_SHAPE), "c": 0.1, "seed": args.seed},
            "cpu_baseline": {"value": v, "unit": "GB/s", "cores": 1, "kind": "oracle",
                             "sample": f"{n} single-sample calls ({N} elements each), {dt:.1f} s; numpy fp64"},
            "e2e": {"value": v, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_qkv(args):
    """``--workload qkv_t2i``: the prologue kernel (a tensor-core GEMM pair with
    an RMSNorm-JVP epilogue) on a T2I-sized layer."""
    import torch
    import torch.distributed as dist

    ws, rank, local = dist_setup()
    group = ws > 1
    if group:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    from attention_jvp_fwd_b200.build import build
    if rank == 0 or not group:
        build()
    if group:
        dist.barrier()
    import attention_jvp_fwd_b200 as A

    B, L, H, D, d = (QKV_SHAPE[k] for k in ("B", "L", "H", "D", "d"))
    T = B * L
    bits = qkv_inputs(args.seed + rank)
    host = [torch.from_numpy(b.view(np.int16)).view(torch.bfloat16).pin_memory() for b in bits]
    x, xd, w = (h.to(dev, non_blocking=True) for h in host)
    gq = torch.ones(d, dtype=torch.float32, device=dev)
    gk = torch.ones(d, dtype=torch.float32, device=dev)
    outs = tuple(torch.empty((B, H, L, d), dtype=torch.bfloat16, device=dev) for _ in range(6))
    stream = torch.cuda.Stream(dev)
    flops_step = 2.0 * 2 * T * D * 3 * H * d

    def step():
        A.qkv_rmsnorm_jvp(x, xd, w, gq, gk, B, L, H, out=outs, stream=stream)

    with torch.cuda.stream(stream):
        for _ in range(args.warmup):
            step()
    torch.cuda.synchronize(dev)
    st, site = A.qkv_prologue_check(stream)
    if st != 0:
        raise RuntimeError(f"device status {st} at site {site}")
    sampler = ClockSampler(dev)
    sampler.start()
    time.sleep(0.6)
    if group:
        dist.barrier()
    torch.cuda.synchronize(dev)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    with torch.cuda.stream(stream):
        for _ in range(args.steps):
            step()
    e1.record(stream)
    torch.cuda.synchronize(dev)
    local_ms = e0.elapsed_time(e1)
    clocks = sampler.stop()
    max_ms, total = aggregate(local_ms, flops_step * args.steps, group, dev)
    value = total / (max_ms * 1e-3) / 1e12

    e2e_steps = args.e2e_steps or min(args.steps, 100)

    def e2e_call(di, do, st):
        A.qkv_rmsnorm_jvp(di[0], di[1], di[2], gq, gk, B, L, H, out=tuple(do), stream=st)

    e2e_local = stream_e2e(dev, host, outs, e2e_call, e2e_steps, group)
    e2e_ms, e2e_fl = aggregate(e2e_local, flops_step * e2e_steps, group, dev)

    burst_tf, sustained_tf, _, peak_src = load_peaks()
    if sustained_tf is not None and local_ms >= SUSTAINED_MS:
        peak_tf, kind = sustained_tf, "sustained"
    else:
        peak_tf, kind = burst_tf, "burst"
    achieved = flops_step / (local_ms / args.steps * 1e-3) / 1e12
    in_bytes = sum(h.numel() * 2 for h in host)
    line = {
        "metric": QKV_METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": ws, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": max_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": "qkv_t2i", **QKV_SHAPE, "seed": args.seed,
                   "l2": "inputs %.0f MB; weights fit in L2 and are reused across token tiles, "
                         "no flush" % (in_bytes / 1e6)},
        "gpu_launches": args.steps,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak_tf,
                     "peak_source": f"{peak_src} bf16 dense ({kind}; timed region {local_ms:.0f} ms)",
                     "unit": "TFLOP/s", "frac": achieved / peak_tf, "frac_of_burst_peak": achieved / burst_tf,
                     "traffic": measured_traffic("qkv_t2i", QKV_SOURCES), "flops_per_launch": flops_step,
                     "kernel": "qkv_prologue_kernel<128>"},
        "e2e": {"value": e2e_fl / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOP/s", "h2d_bytes_per_step": in_bytes,
                "d2h_bytes_per_step": sum(o.numel() * 2 for o in outs), "steps": e2e_steps,
                "how": E2E_NOTE},
        "clocks": clocks,
    }
    if rank == 0 and not group and not args.no_cpu_baseline:
        v, n, calls, dt = time_qkv_oracle(bits, min(args.cpu_seconds, 10.0))
        line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": os.cpu_count(), "kind": "oracle",
                                "sample": f"first {n} tokens (all head tiles) per call, {calls} calls, "
                                          f"{dt:.1f} s; numpy fp64"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if group:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main(argv=None):
    args = parse_args(argv)
    if args.workload == "qkv_t2i":
        return run_reference_qkv(args) if args.impl == "reference" else run_qkv(args)
    if args.workload == "scm_loss":
        return run_reference_loss(args) if args.impl == "reference" else run_loss(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
