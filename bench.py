#!/usr/bin/env python
"""Selective-scan benchmark: state-updates/s (B*L*D*N per second) of the
fused forward scan on B200, with its roofline fraction.

One "step" is one ssm_scan_fwd call over one batch of synthetic input (the
whole hot path: softplus, discretisation, scan, readout, skip, gate).  The
default workload is the Mamba-130M layer shape (B=8, L=2048, D=1536, N=16,
bf16 in/out, fp32 state, gate on).  Inputs are resident in HBM before the
timed region; two input sets (304 MB together, more than the 126 MB L2)
alternate between steps so every step reads cold inputs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU: one process per GPU (torchrun); every rank runs an independent
replica of the workload (the scan has no cross-GPU exchange), the timed
region is bracketed by barriers and the slowest rank's time is used.
``--impl reference`` times the CPU oracle (fp64, all host cores) on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

MUFU_PER_CLK_PER_SM = 16        # ex2/lg2/rcp results per clock per SM (CUDA throughput table)
NOMINAL_SMS = 148
NOMINAL_SM_MHZ = 1965.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="mamba130m_layer",
                    choices=["tiny_fp32", "mamba130m_layer", "mamba1p4b_layer", "long_seq",
                             "decode"])
    ap.add_argument("--e2e-steps", type=int, default=50)
    ap.add_argument("--cpu-budget-s", type=float, default=60.0,
                    help="CPU seconds (summed over threads) for the oracle baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--lpc", type=int, default=0)
    ap.add_argument("--warps", type=int, default=0)
    ap.add_argument("--grid", type=int, default=0)
    ap.add_argument("--tile-t", type=int, default=0)
    ap.add_argument("--bwd", action="store_true",
                    help="time the backward pass (ssm_scan_bwd) instead of the forward")
    ap.add_argument("--zoh", action="store_true",
                    help="zero-order-hold input matrix (exp(Delta A) - 1)/A * B instead of Delta * B")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# algorithmic work per step
# ---------------------------------------------------------------------------

def algorithmic_counts(inp):
    """Per-call algorithmic work of the fused forward scan.
    bytes: inputs read once, outputs written once, state only at the ends.
    mufu: one exp per state update, plus per token and channel exp+log for
    softplus and exp+reciprocal for the silu gate."""
    B, L, D, N = inp.Bsz, inp.L, inp.D, inp.N
    es_in = 2 if inp.in_dtype == "bf16" else 4
    es_out = 2 if inp.out_dtype == "bf16" else 4
    n_bld = (2 + (inp.z is not None)) * B * L * D
    byt = es_in * n_bld + es_out * B * L * D + es_in * 2 * B * L * N
    byt += 4 * D * N + 4 * D * ((inp.Dskip is not None) + (inp.delta_bias is not None))
    byt += 4 * B * D * N * ((inp.h0 is not None) + bool(inp.want_h_last))
    mufu = B * L * D * N + (2 * B * L * D if inp.delta_softplus else 0) + \
        (2 * B * L * D if inp.z is not None else 0)
    return {"updates": B * L * D * N, "bytes": byt, "mufu": mufu}


# sources that define the forward kernel and its launch shape: a committed
# ncu summary's traffic figure is used only while these are unchanged
FWD_KERNEL_SOURCES = ("device_common.cuh", "scan_params.h", "scan_fwd_kernel.cuh",
                      "scan_fwd_bf16.cu", "scan_fwd_f32.cu", "scan_fwd_bf16_f32.cu",
                      "scan_fwd_dispatch.cu")


STEP_KERNEL_SOURCES = ("device_common.cuh", "scan_params.h", "scan_step.cu")


def source_hash(sources=FWD_KERNEL_SOURCES):
    h = hashlib.sha256()
    for name in sources:
        with open(os.path.join(ROOT, "selective_state_space_31_b200", "csrc", name), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def profiled_traffic(workload, kernel="fwd_kernel", sources=FWD_KERNEL_SOURCES):
    """dram bytes per launch of a kernel from its committed ncu summary
    (profiles/<kernel>_<workload>.md), or None when the summary was taken on
    other source code."""
    path = os.path.join(ROOT, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    kv = {}
    for line in open(path):
        if ":" in line and line.strip().startswith("- "):
            k, v = line.strip()[2:].split(":", 1)
            kv[k.strip()] = v.strip().strip("`")
    if kv.get("source_sha256") != source_hash(sources):
        return None
    try:
        return int(float(kv["dram_bytes_per_launch"]))
    except (KeyError, ValueError):
        return None


# ---------------------------------------------------------------------------
# multi-GPU replicas: slowest rank decides, work adds up
# ---------------------------------------------------------------------------

def max_over_ranks(values, device=None):
    """Max of each value over all ranks (identity when not distributed).
    Works with NCCL (CUDA tensors) and gloo (CPU tensors)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return [float(v) for v in values]
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def replica_throughput(updates_per_rank, world, ms_per_step_max):
    """Whole-job state-updates/s: every rank runs its own replica of the
    workload, so the work adds up and the slowest rank's time counts."""
    return updates_per_rank * world / (ms_per_step_max * 1e-3)


# ---------------------------------------------------------------------------
# clocks (NVML, read-only) sampled during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, torch_device, period_s=0.002):
        self.samples, self.reasons, self.ok = [], set(), False
        self.period, self._stop, self._t = period_s, threading.Event(), None
        self.max_mhz = None
        try:
            import pynvml as nv
            nv.nvmlInit()
            self.nv = nv
            import torch
            props = torch.cuda.get_device_properties(torch_device)
            h = None
            bus = getattr(props, "pci_bus_id", None)
            if bus is not None:
                dom = getattr(props, "pci_domain_id", 0)
                devid = getattr(props, "pci_device_id", 0)
                try:
                    h = nv.nvmlDeviceGetHandleByPciBusId(f"{dom:08x}:{bus:02x}:{devid:02x}.0")
                except Exception:
                    h = None
            if h is None:
                vis = os.environ.get("CUDA_VISIBLE_DEVICES")
                idx = torch_device.index or 0
                if vis:
                    idx = int(vis.split(",")[idx])
                h = nv.nvmlDeviceGetHandleByIndex(idx)
            self.h = h
            self.max_mhz = nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # NVML unavailable: report no clocks
            self.err = repr(e)

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                r = get_r(self.h)
                for bit, name in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def start(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()

    def stop(self):
        if self._t:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


# ---------------------------------------------------------------------------
# CPU oracle timing (reported baseline)
# ---------------------------------------------------------------------------

def oracle_sample_rate(inp, budget_cpu_s, threads=None):
    """Time the fp64 oracle over channel rows of the workload on all host
    cores.  Rows are taken in order (b, d) until the estimated CPU-seconds
    budget is used.  Returns (updates/s, cores, description)."""
    import concurrent.futures as cf

    import numpy as np

    import oracle
    orc = oracle.get()
    threads = threads or os.cpu_count() or 1
    # calibrate on one row
    t0 = time.perf_counter()
    oracle.fwd_rows(inp.x, inp.delta, inp.A, inp.B, inp.C, [(0, 0)], D=inp.Dskip, z=inp.z,
                    delta_bias=inp.delta_bias, h0=inp.h0, delta_softplus=inp.delta_softplus,
                    oracle=orc, zoh=inp.zoh)
    per_row = max(time.perf_counter() - t0, 1e-6)
    n_rows = int(min(inp.Bsz * inp.D, max(threads, budget_cpu_s / per_row)))
    rows = [(r // inp.D, r % inp.D) for r in range(n_rows)]
    chunks = [rows[i::threads] for i in range(threads)]

    def work(ch):
        if ch:
            oracle.fwd_rows(inp.x, inp.delta, inp.A, inp.B, inp.C, ch, D=inp.Dskip, z=inp.z,
                            delta_bias=inp.delta_bias, h0=inp.h0,
                            delta_softplus=inp.delta_softplus, oracle=orc, zoh=inp.zoh)

    t0 = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(work, chunks))
    dt = time.perf_counter() - t0
    upd = n_rows * inp.L * inp.N
    desc = (f"{n_rows} of {inp.Bsz * inp.D} channel rows (full length L={inp.L}, N={inp.N}) "
            f"of {inp.name}, fp64 oracle, {threads} threads")
    return upd / dt, threads, desc, upd


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------

def run_ours(args, rank, world, device):
    import numpy as np
    import torch

    from selective_state_space_31_b200 import binding as bnd
    from selective_state_space_31_b200 import synth

    torch.cuda.set_device(device)
    make = synth.FWD_WORKLOADS[args.workload]
    inp = make()
    inp_b = make(seed={"tiny_fp32": 0, "mamba130m_layer": 1, "mamba1p4b_layer": 2,
                       "long_seq": 3}[args.workload] + 1000 + rank)
    inp.zoh = inp_b.zoh = bool(args.zoh)
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}

    def up(a, dt):
        return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(device, dt)

    def upload(s):
        return dict(x=up(s.x, tdt[s.in_dtype]), delta=up(s.delta, tdt[s.in_dtype]),
                    z=up(s.z, tdt[s.in_dtype]), B=up(s.B, tdt[s.in_dtype]),
                    C=up(s.C, tdt[s.in_dtype]), A=up(s.A, torch.float32),
                    D=up(s.Dskip, torch.float32), delta_bias=up(s.delta_bias, torch.float32),
                    h0=up(s.h0, torch.float32))

    sets = [upload(inp), upload(inp_b)]
    flags = bnd.flags_for(z=inp.z, D=inp.Dskip, delta_bias=inp.delta_bias, h0=inp.h0,
                          delta_softplus=inp.delta_softplus, want_h_last=True, zoh=inp.zoh)
    plan = bnd.Plan(inp.Bsz, inp.L, inp.D, inp.N, tdt[inp.in_dtype], tdt[inp.out_dtype], flags,
                    device)
    if args.lpc or args.warps or args.grid or args.tile_t:
        plan.set_config(args.lpc, args.warps, args.grid, args.tile_t)
    outs = [(torch.empty((inp.Bsz, inp.L, inp.D), dtype=tdt[inp.out_dtype], device=device),
             torch.empty((inp.Bsz, inp.D, inp.N), dtype=torch.float32, device=device))
            for _ in range(2)]

    def step(i):
        s, (y, hl) = sets[i & 1], outs[i & 1]
        if args.bwd:   # y doubles as dL/dy (any values of the output dtype)
            plan.bwd(s["x"], s["delta"], s["A"], s["B"], s["C"], y, D=s["D"], z=s["z"],
                     delta_bias=s["delta_bias"], h0=s["h0"], dh_last=hl)
            return
        plan.fwd(s["x"], s["delta"], s["A"], s["B"], s["C"], D=s["D"], z=s["z"],
                 delta_bias=s["delta_bias"], h0=s["h0"], y=y, h_last=hl)

    stream = torch.cuda.current_stream(device)
    if args.bwd:   # real outputs as dL/dy
        for i in range(2):
            s, (y, hl) = sets[i], outs[i]
            plan.fwd(s["x"], s["delta"], s["A"], s["B"], s["C"], D=s["D"], z=s["z"],
                     delta_bias=s["delta_bias"], h0=s["h0"], y=y, h_last=hl)
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize(device)
    assert plan.status() == 0

    sampler = ClockSampler(device)
    K = args.steps
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(K)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    sampler.start()
    t_start.record(stream)
    for i in range(K):
        ev[i][0].record(stream)
        step(i)
        ev[i][1].record(stream)
    t_end.record(stream)
    torch.cuda.synchronize(device)
    sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    total_ms = t_start.elapsed_time(t_end)
    kern_ms = statistics.mean(a.elapsed_time(b) for a, b in ev)
    st = plan.status()
    if st != 0:
        raise RuntimeError(f"device status {st} after the timed region")
    total_ms, kern_ms = max_over_ranks([total_ms, kern_ms], device)
    ms_per_step = total_ms / K

    counts = algorithmic_counts(inp)
    if args.bwd:
        # the backward evaluates every exp three times: checkpoint pass, chunk
        # recomputation and the reverse walk
        counts["mufu"] *= 3
    value = replica_throughput(counts["updates"], world, ms_per_step)

    # e2e through the public API: pinned host inputs copied in, y/h_last copied out
    e2e = None
    if args.e2e_steps > 0 and not args.bwd:
        def pinned(a, dt):
            return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dt).pin_memory()
        host = dict(x=pinned(inp.x, tdt[inp.in_dtype]), delta=pinned(inp.delta, tdt[inp.in_dtype]),
                    z=pinned(inp.z, tdt[inp.in_dtype]), B=pinned(inp.B, tdt[inp.in_dtype]),
                    C=pinned(inp.C, tdt[inp.in_dtype]), h0=pinned(inp.h0, torch.float32))
        dev_in = {k: (torch.empty_like(v, device=device) if v is not None else None)
                  for k, v in host.items()}
        y_h = torch.empty((inp.Bsz, inp.L, inp.D), dtype=tdt[inp.out_dtype]).pin_memory()
        hl_h = torch.empty((inp.Bsz, inp.D, inp.N), dtype=torch.float32).pin_memory()
        y_d, hl_d = outs[0]
        h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
        d2h = y_h.numel() * y_h.element_size() + hl_h.numel() * 4
        par = sets[0]

        def e2e_step():
            for k, v in host.items():
                if v is not None:
                    dev_in[k].copy_(v, non_blocking=True)
            plan.fwd(dev_in["x"], dev_in["delta"], par["A"], dev_in["B"], dev_in["C"], D=par["D"],
                     z=dev_in["z"], delta_bias=par["delta_bias"], h0=dev_in["h0"], y=y_d,
                     h_last=hl_d)
            y_h.copy_(y_d, non_blocking=True)
            hl_h.copy_(hl_d, non_blocking=True)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize(device)
        if world > 1:
            torch.distributed.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(args.e2e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize(device)
        e_ms = a.elapsed_time(b) / args.e2e_steps
        e_ms = max_over_ranks([e_ms], device)[0]
        e2e = {"value": replica_throughput(counts["updates"], world, e_ms), "unit": "state-updates/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
               "steps": args.e2e_steps}

    info = plan.info()
    clocks = sampler.summary()
    peak_mufu = MUFU_PER_CLK_PER_SM * NOMINAL_SMS * NOMINAL_SM_MHZ * 1e6
    achieved_mufu = counts["mufu"] / (kern_ms * 1e-3)
    hbm_gbs = counts["bytes"] / (kern_ms * 1e-3) / 1e9
    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except Exception:
        pass
    hbm_peak = peaks.get("hbm_gbs", 6650.0)
    traffic = profiled_traffic(args.workload)

    result = {
        "metric": "selective-scan state-updates/s (B*L*D*N)",
        "value": value,
        "unit": "state-updates/s",
        "n_gpus": world,
        "steps": K,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if inp.in_dtype == "bf16" else "f32",
        "data": "synthetic (seeded normal draws, shapes and distributions of the workload)",
        "config": {"workload": inp.name, "batch": inp.Bsz, "seqlen": inp.L, "dim": inp.D,
                   "dstate": inp.N, "in_dtype": inp.in_dtype, "out_dtype": inp.out_dtype,
                   "state_dtype": "f32", "gate": inp.z is not None, "h0": inp.h0 is not None,
                   "discretisation": "zoh" if inp.zoh else "delta_B",
                   "pass": "backward" if args.bwd else "forward",
                   "l2": "two input sets alternate between steps (2x inputs > 126 MB L2)",
                   "parallelism": f"replicas x{world}",
                   "launch": {k: info[k] for k in ("lanes_per_chan", "warps_per_cta",
                                                    "tile_t", "chans_per_cta", "grid",
                                                    "rows", "units")}},
        "roofline": {"bound": "alu", "achieved": achieved_mufu / 1e9, "peak": peak_mufu / 1e9,
                     "unit": "G MUFU-op/s (ex2, lg2, rcp)", "frac": achieved_mufu / peak_mufu,
                     "traffic": traffic,
                     "peak_basis": "16 MUFU results/clk/SM x 148 SMs x 1965 MHz (nominal)",
                     "kernel_ms": kern_ms,
                     "hbm": {"achieved_gbs": hbm_gbs, "peak_gbs": hbm_peak,
                             "frac": hbm_gbs / hbm_peak, "algorithmic_bytes": counts["bytes"]}},
        "gpu_launches": K,
        "clocks": clocks,
        "e2e": e2e,
    }
    if clocks.get("sm_mhz"):
        result["roofline"]["frac_at_sampled_clock"] = achieved_mufu / (
            MUFU_PER_CLK_PER_SM * NOMINAL_SMS * clocks["sm_mhz"] * 1e6)

    if rank == 0 and world == 1 and not args.no_cpu_baseline and not args.bwd:
        rate, cores, desc, _ = oracle_sample_rate(inp, args.cpu_budget_s)
        result["cpu_baseline"] = {"value": rate, "unit": "state-updates/s", "cores": cores,
                                  "kind": "oracle", "sample": desc}
    plan.close()
    return result


# ---------------------------------------------------------------------------
# decode: one token step over a (256, 5120, 16) fp32 state
# ---------------------------------------------------------------------------

def run_decode(args, rank, world, device):
    """One step = one ssm_scan_step over the whole (B, D, N) state.  Three
    independent states (3 x 84 MB, more than the 126 MB L2) take turns and
    32 distinct token inputs rotate, so every step streams its state from
    HBM.  96 steps (all combinations) are captured in one CUDA graph."""
    import numpy as np
    import torch

    from selective_state_space_31_b200 import binding as bnd
    from selective_state_space_31_b200 import synth

    torch.cuda.set_device(device)
    dec = synth.make_decode(steps=32, seed=4 + rank)
    bf, f32 = torch.bfloat16, torch.float32
    up = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(device, dt)
    toks = [dec.token(t) for t in range(32)]
    tin = [{k: up(v, bf) for k, v in tk.items()} for tk in toks]
    A, D, bias = up(dec.A, f32), up(dec.Dskip, f32), up(dec.delta_bias, f32)
    states = [up(dec.h0, f32) for _ in range(3)]
    ys = [torch.empty((dec.Bsz, dec.D), dtype=bf, device=device) for _ in range(3)]
    flags = bnd.flags_for(z=1, D=1, delta_bias=1, delta_softplus=True, want_h_last=False)
    plan = bnd.Plan(dec.Bsz, 1, dec.D, dec.N, bf, bf, flags, device)

    def step(i):
        t, s = tin[i % 32], i % 3
        plan.step(states[s], t["x"], t["delta"], A, t["B"], t["C"], D=D, z=t["z"],
                  delta_bias=bias, y=ys[s])

    G = 96
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        for i in range(G):   # warm-up outside capture (also loads the module)
            step(i)
    torch.cuda.synchronize(device)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(G):
            step(i)
    reps = max(1, args.steps // G)
    for _ in range(max(1, args.warmup // G)):
        graph.replay()
    torch.cuda.synchronize(device)
    sampler = ClockSampler(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(device)
    sampler.start()
    a.record(torch.cuda.current_stream(device))
    for _ in range(reps):
        graph.replay()
    b.record(torch.cuda.current_stream(device))
    torch.cuda.synchronize(device)
    sampler.stop()
    if world > 1:
        torch.distributed.barrier()
    steps = reps * G
    ms_per_step = max_over_ranks([a.elapsed_time(b) / steps], device)[0]
    upd = dec.Bsz * dec.D * dec.N
    Bz, Dm, N = dec.Bsz, dec.D, dec.N
    byt = 8 * Bz * Dm * N + 3 * 2 * Bz * Dm + 2 * 2 * Bz * N + 2 * Bz * Dm + 4 * Dm * N + 8 * Dm
    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except Exception:
        pass
    hbm_peak = peaks.get("hbm_gbs", 6650.0)
    gbs = byt / (ms_per_step * 1e-3) / 1e9
    # e2e: a token's inputs come from pinned host memory, y goes back
    host = [{k: v.to(bf).cpu().pin_memory() for k, v in t.items()} for t in tin[:4]]
    y_h = torch.empty((Bz, Dm), dtype=bf).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host[0].values())
    d2h = y_h.numel() * y_h.element_size()
    s0 = torch.cuda.current_stream(device)
    e1, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    E = max(8, min(args.e2e_steps, 200))
    e1.record(s0)
    for i in range(E):
        for k, v in host[i % 4].items():
            tin[0][k].copy_(v, non_blocking=True)
        step(0)
        y_h.copy_(ys[0], non_blocking=True)
    e2.record(s0)
    torch.cuda.synchronize(device)
    e_ms = max_over_ranks([e1.elapsed_time(e2) / E], device)[0]
    res = {
        "metric": "selective-scan state-updates/s (B*L*D*N)",
        "value": replica_throughput(upd, world, ms_per_step),
        "unit": "state-updates/s", "n_gpus": world, "steps": steps,
        "warmup": max(1, args.warmup // G) * G, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded normal draws, shapes and distributions of the workload)",
        "config": {"workload": "decode", "batch": Bz, "dim": Dm, "dstate": N,
                   "step": "one token for the whole state", "graph": f"{G} steps per CUDA graph",
                   "l2": "3 independent 84 MB states take turns (252 MB > 126 MB L2)",
                   "parallelism": f"replicas x{world}"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": gbs / hbm_peak,
                     "traffic": profiled_traffic("decode", "step_kernel", STEP_KERNEL_SOURCES),
                     "algorithmic_bytes": byt},
        "gpu_launches": steps,
        "clocks": sampler.summary(),
        "e2e": {"value": replica_throughput(upd, world, e_ms), "unit": "state-updates/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms},
    }
    del graph
    plan.close()
    return res


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle on a bounded sample of the same workload
# ---------------------------------------------------------------------------

def oracle_decode_rate(dec, budget_cpu_s, threads):
    """Time the fp64 oracle's decode step on the first channels of the
    (B, D, N) state, sized to the CPU-seconds budget, on all host cores."""
    import concurrent.futures as cf

    import oracle
    orc = oracle.get()
    tok = dec.token(0)
    t0 = time.perf_counter()
    orc.step(dec.h0[:1, :64], tok["x"][:1, :64], tok["delta"][:1, :64], dec.A[:64], tok["B"][:1],
             tok["C"][:1], D=dec.Dskip[:64], z=tok["z"][:1, :64], delta_bias=dec.delta_bias[:64])
    per_chan = max((time.perf_counter() - t0) / 64, 1e-9)
    n_b = int(min(dec.Bsz, max(threads, budget_cpu_s / per_chan / dec.D)))

    def work(b):
        orc.step(dec.h0[b:b + 1], tok["x"][b:b + 1], tok["delta"][b:b + 1], dec.A, tok["B"][b:b + 1],
                 tok["C"][b:b + 1], D=dec.Dskip, z=tok["z"][b:b + 1], delta_bias=dec.delta_bias)

    t0 = time.perf_counter()
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        list(ex.map(work, range(n_b)))
    dt = time.perf_counter() - t0
    upd = n_b * dec.D * dec.N
    return upd / dt, upd, (f"{n_b} of {dec.Bsz} batch rows of one decode step "
                           f"(D={dec.D}, N={dec.N}), fp64 oracle, {threads} threads")


def run_reference(args):
    from selective_state_space_31_b200 import synth
    if args.workload == "decode":
        dec = synth.make_decode(steps=1)
        threads = os.cpu_count() or 1
        per_step = args.cpu_budget_s * threads / max(1, args.steps + args.warmup)
        for _ in range(args.warmup):
            oracle_decode_rate(dec, per_step, threads)
        upd_total, t_total, desc = 0, 0.0, ""
        for _ in range(args.steps):
            rate, upd, desc = oracle_decode_rate(dec, per_step, threads)
            upd_total += upd
            t_total += upd / rate
        value = upd_total / t_total
        return {"impl": "reference", "metric": "selective-scan state-updates/s (B*L*D*N)",
                "value": value, "unit": "state-updates/s", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup,
                "ms_per_step": t_total / max(1, args.steps) * 1e3, "higher_is_better": True,
                "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic (seeded normal draws, shapes and distributions of the workload)",
                "config": {"workload": "decode", "batch": dec.Bsz, "dim": dec.D, "dstate": dec.N},
                "cpu_baseline": {"value": value, "unit": "state-updates/s", "cores": threads,
                                 "kind": "oracle", "sample": "per step: " + desc},
                "e2e": {"value": value, "unit": "state-updates/s", "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}}
    inp = synth.FWD_WORKLOADS[args.workload]()
    inp.zoh = bool(args.zoh)
    threads = os.cpu_count() or 1
    total_budget = args.cpu_budget_s * threads   # CPU-seconds for warmup + timed steps
    per_step = total_budget / max(1, args.steps + args.warmup)
    for _ in range(args.warmup):
        oracle_sample_rate(inp, per_step, threads)
    upd_total, t_total, desc = 0, 0.0, ""
    for _ in range(args.steps):
        rate, cores, desc, upd = oracle_sample_rate(inp, per_step, threads)
        upd_total += upd
        t_total += upd / rate
    value = upd_total / t_total
    return {
        "impl": "reference",
        "metric": "selective-scan state-updates/s (B*L*D*N)",
        "value": value,
        "unit": "state-updates/s",
        "n_gpus": args.gpus,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": t_total / max(1, args.steps) * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic (seeded normal draws, shapes and distributions of the workload)",
        "config": {"workload": inp.name, "batch": inp.Bsz, "seqlen": inp.L, "dim": inp.D,
                   "dstate": inp.N},
        "cpu_baseline": {"value": value, "unit": "state-updates/s", "cores": threads,
                         "kind": "oracle", "sample": "per step: " + desc},
        "e2e": {"value": value, "unit": "state-updates/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    import datetime

    import torch
    device = torch.device("cuda", local)
    if world > 1:
        torch.cuda.set_device(device)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        res = (run_decode if args.workload == "decode" else run_ours)(args, rank, world, device)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
