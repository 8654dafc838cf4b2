#!/usr/bin/env python
"""Selective-scan benchmark: state-updates/s (B*L*D*N per second) of the
fused forward scan on B200, with its roofline fraction.

One "step" is one ssm_scan_fwd call over one batch of synthetic input (the
whole hot path: softplus, discretisation, scan, readout, skip, gate).  The
headline workload is the largest single-GPU one, the long sequence
(B=1, L=131072, D=2560, N=16, bf16 in/out, fp32 state, gate on).  Inputs are
resident in HBM before the timed region and larger than the 126 MB L2 (or,
for the smaller workloads, two input sets alternate between steps).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-sweep]

At N = 1 the same run also measures every other standard workload (the tiny
fp32 scan, the Mamba-130M and 1.4B layer shapes, the decode step) and puts one
record per workload under "workloads", each with its roofline, CPU-oracle
baselines and end-to-end figure.  The roofline peaks are measured in the run:
ex2.approx and FMA throughput probes of the library, at the SM clock sampled
while they run, and the HBM copy bandwidth from MEASURED_PEAKS.json.

Multi-GPU: one process per GPU (torchrun); every rank runs an independent
replica of the workload (the scan has no cross-GPU exchange), the timed
region is bracketed by barriers and the slowest rank's time is used.
``--impl reference`` times the CPU oracle (fp64, all host cores) on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import copy
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
FFMA_PER_CLK_PER_SM = 128
NOMINAL_SMS = 148
NOMINAL_SM_MHZ = 1965.0
L2_BYTES = 126 * 2 ** 20
WORKLOADS = ["tiny_fp32", "mamba130m_layer", "mamba1p4b_layer", "long_seq", "decode"]
SEEDS = {"tiny_fp32": 0, "mamba130m_layer": 1, "mamba1p4b_layer": 2, "long_seq": 3, "decode": 4}
METRIC = "selective-scan state-updates/s (B*L*D*N)"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long_seq", choices=WORKLOADS)
    ap.add_argument("--no-sweep", action="store_true",
                    help="measure only --workload (no per-workload records)")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-budget-s", type=float, default=2.5,
                    help="wall seconds per CPU-oracle timing (4 timings per workload)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--lpc", type=int, default=0)
    ap.add_argument("--warps", type=int, default=0)
    ap.add_argument("--grid", type=int, default=0)
    ap.add_argument("--tile-t", type=int, default=0)
    ap.add_argument("--bwd", action="store_true",
                    help="time the backward pass (ssm_scan_bwd) instead of the forward")
    ap.add_argument("--zoh", action="store_true",
                    help="zero-order-hold input matrix (exp(Delta A) - 1)/A * B instead of Delta * B")
    ap.add_argument("--shape", default="",
                    help="B,L,D: a resized copy of --workload (profiling on smaller inputs)")
    ap.add_argument("--segments", type=int, default=0, help="segments per row (launch override)")
    ap.add_argument("--kc", type=int, default=0, help="channels per lane (launch override)")
    return ap.parse_args(argv)


# ---------------------------------------------------------------------------
# algorithmic work per step
# ---------------------------------------------------------------------------

def algorithmic_counts(inp, backward=False):
    """Per-call algorithmic work of the fused scan (forward, or backward).

    Forward bytes: inputs read once, outputs written once, the state only at
    the ends.  mufu: one exp per state update, plus per token and channel
    exp+log for softplus and exp+reciprocal for the silu gate.

    Backward bytes: the forward inputs and dy read once, the fp32 gradients
    dx, ddelta, dz (B,L,D) and dB, dC (B,L,N) written once, the per-8-token
    stage-start states (B,D,L/8,N) fp32 written and read once, dA/dD/dbias
    and h0/dh_last/dh0 once.  mufu: the state's exp is evaluated three times
    (checkpoint pass, recomputation, reverse walk), the per-token ones twice."""
    B, L, D, N = inp.Bsz, inp.L, inp.D, inp.N
    es_in = 2 if inp.in_dtype == "bf16" else 4
    es_out = 2 if inp.out_dtype == "bf16" else 4
    has_z = inp.z is not None
    n_bld = (2 + has_z) * B * L * D
    per_tok = (2 * B * L * D if inp.delta_softplus else 0) + (2 * B * L * D if has_z else 0)
    params = 4 * D * N + 4 * D * ((inp.Dskip is not None) + (inp.delta_bias is not None))
    if not backward:
        byt = es_in * n_bld + es_out * B * L * D + es_in * 2 * B * L * N + params
        byt += 4 * B * D * N * ((inp.h0 is not None) + bool(inp.want_h_last))
        mufu = B * L * D * N + per_tok
    else:
        byt = es_in * n_bld + es_out * B * L * D + es_in * 2 * B * L * N   # inputs + dy
        byt += 4 * n_bld + 4 * 2 * B * L * N                             # dx, ddelta, dz, dB, dC
        byt += 2 * 4 * B * D * ((L + 7) // 8) * N                       # stage starts out + in
        byt += 2 * params + 4 * B * D * N * (1 + 2 * (inp.h0 is not None))
        mufu = 3 * B * L * D * N + 2 * per_tok
    return {"updates": B * L * D * N, "bytes": byt, "mufu": mufu}


# sources that define the forward kernel and its launch shape: a committed
# ncu summary's traffic figure is used only while these are unchanged
FWD_KERNEL_SOURCES = ("device_common.cuh", "scan_params.h", "scan_fwd_kernel.cuh",
                      "scan_fwd_variants.h", "scan_fwd_dispatch.cu")
STEP_KERNEL_SOURCES = ("device_common.cuh", "scan_params.h", "scan_step.cu")


def source_hash(sources=FWD_KERNEL_SOURCES):
    h = hashlib.sha256()
    for name in sources:
        path = os.path.join(ROOT, "selective_state_space_31_b200", "csrc", name)
        if os.path.exists(path):
            with open(path, "rb") as fh:
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


def measured_hbm_peak():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            v = json.load(f).get("hbm_gbs")
            if v:
                return float(v), "MEASURED_PEAKS.json (copy)"
    except Exception:
        pass
    return 6650.0, "fallback (earlier copy measurement on this pool)"


def workload_config(inp):
    """The workload as both arms name it."""
    return {"workload": inp.name, "batch": inp.Bsz, "seqlen": inp.L, "dim": inp.D,
            "dstate": inp.N, "in_dtype": inp.in_dtype, "out_dtype": inp.out_dtype,
            "state_dtype": "f32", "gate": inp.z is not None, "h0": inp.h0 is not None,
            "discretisation": "zoh" if inp.zoh else "delta_B"}


def input_sets(inp):
    """1 when one input set is larger than 3x the L2 (every step reads cold
    inputs anyway), else 2 sets that alternate between steps."""
    es_in = 2 if inp.in_dtype == "bf16" else 4
    set_bytes = es_in * (3 * inp.Bsz * inp.L * inp.D + 2 * inp.Bsz * inp.L * inp.N)
    return 1 if set_bytes > 3 * L2_BYTES else 2


def arm_config(inp, world, backward=False):
    """The run's config as both arms report it (the reference arm times the
    oracle on the same workload)."""
    n_sets = input_sets(inp)
    return dict(workload_config(inp),
                **{"pass": "backward" if backward else "forward",
                   "l2": ("inputs larger than L2 (one set)" if n_sets == 1 else
                          "two input sets alternate between steps (2x inputs > 126 MB L2)"),
                   "parallelism": f"replicas x{world}"})


def decode_config(dec):
    return {"workload": "decode", "batch": dec.Bsz, "dim": dec.D, "dstate": dec.N,
            "in_dtype": "bf16", "out_dtype": "bf16", "state_dtype": "f32", "gate": True,
            "step": "one token for the whole (B, D, N) state"}


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
# clocks (NVML, read-only) sampled during a timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
               0x2: "applications_clocks_setting", 0x1: "gpu_idle"}

    def __init__(self, torch_device, period_s=0.0005):
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
# measured peaks: the library's ex2 and FMA throughput probes
# ---------------------------------------------------------------------------

def measure_peaks(device, sms):
    """ex2.approx and fp32 FMA throughput of the whole GPU, from the library's
    probe kernels (8 CTAs of 256 threads per SM, 8 independent chains per
    thread), timed with CUDA events with the SM clock sampled meanwhile.
    Returns results/s and results/clk/SM at the sampled clock."""
    import torch

    from selective_state_space_31_b200 import binding as bnd
    blocks = sms * 8
    sink = torch.zeros(blocks, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    out = {}
    for kind, name, iters in ((0, "ex2", 1500), (1, "ffma", 12000)):
        for _ in range(2):
            bnd.probe_peak(kind, max(1, iters // 10), blocks, sink)
        torch.cuda.synchronize(device)
        sampler = ClockSampler(device)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        sampler.start()
        a.record(stream)
        ops = 0
        for _ in range(3):
            ops += bnd.probe_peak(kind, iters, blocks, sink)
        b.record(stream)
        torch.cuda.synchronize(device)
        sampler.stop()
        sec = a.elapsed_time(b) * 1e-3
        clk = sampler.summary()
        mhz = clk["sm_mhz"] or NOMINAL_SM_MHZ
        out[name] = {"ops_per_s": ops / sec, "per_clk_per_sm": ops / sec / (mhz * 1e6) / sms,
                     "sm_mhz": clk["sm_mhz"], "clock_samples": clk["samples"],
                     "reasons": clk["reasons"], "ms": sec * 1e3}
    return out


# ---------------------------------------------------------------------------
# CPU oracle timing (reported baselines)
# ---------------------------------------------------------------------------

def oracle_rate(inp, budget_s, threads, fp32=False):
    """Time the oracle over whole channels (full length L) of the workload,
    blocks of channels taken in order (b, d), for about ``budget_s`` wall
    seconds, on ``threads`` host threads (oracle.fwd_blocks: the C loop runs
    without the GIL).  fp32 selects the fp32-accumulate build of the same
    loop.  Returns (updates/s, updates timed, description)."""
    import oracle
    orc = oracle.get_fp32() if fp32 else oracle.get()
    width = max(1, min(64, (1 << 21) // max(inp.L, 1)))
    blocks = oracle.channel_blocks(inp.Bsz, inp.D, width)
    kw = dict(D=inp.Dskip, z=inp.z, delta_bias=inp.delta_bias, h0=inp.h0,
              delta_softplus=inp.delta_softplus, zoh=inp.zoh, oracle=orc)
    sink = lambda blk, y, h: None
    # calibrate on one block
    t0 = time.perf_counter()
    oracle.fwd_blocks(inp.x, inp.delta, inp.A, inp.B, inp.C, blocks[:1], sink, threads=1, **kw)
    per_block = max(time.perf_counter() - t0, 1e-6)
    n = int(min(len(blocks), max(threads, budget_s * threads / per_block)))
    todo = blocks[:n]
    t0 = time.perf_counter()
    oracle.fwd_blocks(inp.x, inp.delta, inp.A, inp.B, inp.C, todo, sink, threads=threads, **kw)
    dt = time.perf_counter() - t0
    chans = sum(d1 - d0 for _, d0, d1 in todo)
    upd = chans * inp.L * inp.N
    desc = (f"{chans} of {inp.Bsz * inp.D} channels (full length L={inp.L}, N={inp.N}) of "
            f"{inp.name}, {'fp32-accumulate' if fp32 else 'fp64'} oracle, {threads} thread(s)")
    return upd / dt, upd, desc


def cpu_baselines(inp, budget_s):
    """The oracle as it stands, fp64 and fp32-accumulate builds, on one host
    thread and on all host threads.  The headline baseline is fp64, all
    threads."""
    allt = os.cpu_count() or 1
    out = {}
    for fp32 in (False, True):
        for th in (1, allt):
            rate, upd, desc = oracle_rate(inp, budget_s, th, fp32=fp32)
            out[f"{'fp32acc' if fp32 else 'fp64'}_{'1thread' if th == 1 else 'all'}"] = {
                "value": rate, "threads": th, "sample": desc}
    main = out["fp64_all"]
    return {"value": main["value"], "unit": "state-updates/s", "cores": allt, "kind": "oracle",
            "sample": main["sample"], "variants": out, "cpu": _cpu_model()}


def _cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return None


# ---------------------------------------------------------------------------
# our arm: one forward workload
# ---------------------------------------------------------------------------

def run_fwd(name, steps, warmup, args, rank, world, device, peaks, e2e_steps,
            want_cpu=True):
    import numpy as np
    import torch

    from selective_state_space_31_b200 import binding as bnd
    from selective_state_space_31_b200 import synth

    torch.cuda.set_device(device)
    shape = tuple(int(v) for v in args.shape.split(",")) if args.shape and \
        name == args.workload else None
    make = lambda **kw: synth.FWD_WORKLOADS[name](shape=shape, **kw)
    inp = make()
    inp.zoh = bool(args.zoh)
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16}
    n_sets = input_sets(inp)

    def up(a, dt):
        return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(device, dt)

    def upload(s):
        return dict(x=up(s.x, tdt[s.in_dtype]), delta=up(s.delta, tdt[s.in_dtype]),
                    z=up(s.z, tdt[s.in_dtype]), B=up(s.B, tdt[s.in_dtype]),
                    C=up(s.C, tdt[s.in_dtype]), A=up(s.A, torch.float32),
                    D=up(s.Dskip, torch.float32), delta_bias=up(s.delta_bias, torch.float32),
                    h0=up(s.h0, torch.float32))

    sets = [upload(inp)]
    if n_sets == 2:
        other = make(seed=SEEDS[name] + 1000 + rank)
        other.zoh = inp.zoh
        sets.append(upload(other))
        del other
    flags = bnd.flags_for(z=inp.z, D=inp.Dskip, delta_bias=inp.delta_bias, h0=inp.h0,
                          delta_softplus=inp.delta_softplus, want_h_last=True, zoh=inp.zoh)
    plan = bnd.Plan(inp.Bsz, inp.L, inp.D, inp.N, tdt[inp.in_dtype], tdt[inp.out_dtype], flags,
                    device)
    if args.lpc or args.warps or args.grid or args.tile_t or args.segments or args.kc:
        plan.set_config(args.lpc, args.warps, args.grid, args.tile_t, args.kc, args.segments)
    outs = [(torch.empty((inp.Bsz, inp.L, inp.D), dtype=tdt[inp.out_dtype], device=device),
             torch.empty((inp.Bsz, inp.D, inp.N), dtype=torch.float32, device=device))
            for _ in range(n_sets)]

    def step(i):
        s, (y, hl) = sets[i % n_sets], outs[i % n_sets]
        if args.bwd:   # y doubles as dL/dy (any values of the output dtype)
            plan.bwd(s["x"], s["delta"], s["A"], s["B"], s["C"], y, D=s["D"], z=s["z"],
                     delta_bias=s["delta_bias"], h0=s["h0"], dh_last=hl)
            return
        plan.fwd(s["x"], s["delta"], s["A"], s["B"], s["C"], D=s["D"], z=s["z"],
                 delta_bias=s["delta_bias"], h0=s["h0"], y=y, h_last=hl)

    stream = torch.cuda.current_stream(device)
    if args.bwd:   # real outputs as dL/dy
        for i in range(n_sets):
            s, (y, hl) = sets[i], outs[i]
            plan.fwd(s["x"], s["delta"], s["A"], s["B"], s["C"], D=s["D"], z=s["z"],
                     delta_bias=s["delta_bias"], h0=s["h0"], y=y, h_last=hl)
    for i in range(warmup):
        step(i)
    torch.cuda.synchronize(device)
    assert plan.status() == 0

    sampler = ClockSampler(device)
    K = steps
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

    counts = algorithmic_counts(inp, backward=args.bwd)
    value = replica_throughput(counts["updates"], world, ms_per_step)

    # e2e through the public API: pinned host inputs copied in, y/h_last copied out
    e2e = None
    if e2e_steps > 0 and not args.bwd:
        def pinned(a, dt):
            return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(dt).pin_memory()
        host = dict(x=pinned(inp.x, tdt[inp.in_dtype]), delta=pinned(inp.delta, tdt[inp.in_dtype]),
                    z=pinned(inp.z, tdt[inp.in_dtype]), B=pinned(inp.B, tdt[inp.in_dtype]),
                    C=pinned(inp.C, tdt[inp.in_dtype]), h0=pinned(inp.h0, torch.float32),
                    A=pinned(inp.A, torch.float32), D=pinned(inp.Dskip, torch.float32),
                    delta_bias=pinned(inp.delta_bias, torch.float32))
        y_h = torch.empty((inp.Bsz, inp.L, inp.D), dtype=tdt[inp.out_dtype]).pin_memory()
        hl_h = torch.empty((inp.Bsz, inp.D, inp.N), dtype=torch.float32).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in host.values() if v is not None)
        d2h = y_h.numel() * y_h.element_size() + hl_h.numel() * 4

        def e2e_step():  # the C-ABI call on host buffers: chunked copy-in / scan / copy-out
            plan.fwd_host(host["x"], host["delta"], host["A"], host["B"], host["C"],
                          D=host["D"], z=host["z"], delta_bias=host["delta_bias"],
                          h0=host["h0"], y=y_h, h_last=hl_h, stream=stream)

        for _ in range(2):
            e2e_step()
        torch.cuda.synchronize(device)
        if world > 1:
            torch.distributed.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(e2e_steps):
            e2e_step()
        b.record(stream)
        torch.cuda.synchronize(device)
        e_ms = a.elapsed_time(b) / e2e_steps
        e_ms = max_over_ranks([e_ms], device)[0]
        e2e = {"value": replica_throughput(counts["updates"], world, e_ms),
               "unit": "state-updates/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": e_ms, "steps": e2e_steps,
               "note": "ssm_scan_fwd_host on pinned host buffers: inputs in and y/h_last out "
                       "over PCIe each step, overlapped with the scan chunk by chunk"}
        del host, y_h, hl_h

    info = plan.info()
    clocks = sampler.summary()
    hbm_peak, hbm_basis = measured_hbm_peak()
    achieved_mufu = counts["mufu"] / (kern_ms * 1e-3)
    hbm_gbs = counts["bytes"] / (kern_ms * 1e-3) / 1e9
    nominal_mufu = MUFU_PER_CLK_PER_SM * NOMINAL_SMS * NOMINAL_SM_MHZ * 1e6
    if peaks and "ex2" in peaks:
        # the probe's rate per clock, at the clock sampled during this workload
        per_clk = peaks["ex2"]["per_clk_per_sm"]
        mhz = clocks.get("sm_mhz") or peaks["ex2"]["sm_mhz"] or NOMINAL_SM_MHZ
        peak_mufu = per_clk * NOMINAL_SMS * mhz * 1e6
        basis = (f"measured ex2.approx probe: {per_clk:.2f} results/clk/SM x {NOMINAL_SMS} SMs "
                 f"x {mhz:.0f} MHz (SM clock sampled during this workload)")
    else:
        peak_mufu, basis = nominal_mufu, "16 MUFU results/clk/SM x 148 SMs x 1965 MHz (nominal)"
    traffic = None if args.bwd else profiled_traffic(name)
    launches_per_call = int(info.get("launches_per_call", 1) or 1)
    if args.bwd:  # fused backward: (the map pass,) the kernel and the row-tile sum of dB / dC
        launches_per_call = ((3 if info.get("bwd_segments", 1) > 1 else 2)
                             if info.get("bwd_warps_per_cta") else 1)

    result = {
        "metric": METRIC,
        "value": value,
        "unit": "state-updates/s",
        "n_gpus": world,
        "steps": K,
        "warmup": warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if inp.in_dtype == "bf16" else "f32",
        "data": "synthetic (seeded normal draws, shapes and distributions of the workload)",
        "config": arm_config(inp, world, args.bwd),
        "launch": {k: info[k] for k in ("lanes_per_chan", "chans_per_lane", "warps_per_cta",
                                        "tile_t", "chans_per_cta", "grid", "rows", "units",
                                        "parts_per_row", "segments", "stages_per_segment",
                                        "carry_grid", "launches_per_call", "scan_loop",
                                        "carry_lanes_per_chan", "carry_loop",
                                        "bwd_warps_per_cta", "bwd_segments") if k in info},
        "roofline": {"bound": "alu", "achieved": achieved_mufu / 1e9, "peak": peak_mufu / 1e9,
                     "unit": "G MUFU-op/s (ex2, lg2, rcp)", "frac": achieved_mufu / peak_mufu,
                     "traffic": traffic, "peak_basis": basis,
                     "frac_of_nominal": achieved_mufu / nominal_mufu,
                     "algorithmic_mufu_per_launch": counts["mufu"],
                     "kernel_ms": kern_ms,
                     "hbm": {"achieved_gbs": hbm_gbs, "peak_gbs": hbm_peak, "peak_basis": hbm_basis,
                             "frac": hbm_gbs / hbm_peak, "algorithmic_bytes": counts["bytes"]}},
        "gpu_launches": K * launches_per_call,
        "clocks": clocks,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and want_cpu and not args.no_cpu_baseline and not args.bwd:
        result["cpu_baseline"] = cpu_baselines(inp, args.cpu_budget_s)
    plan.close()
    del sets, outs
    torch.cuda.empty_cache()
    return result


# ---------------------------------------------------------------------------
# decode: one token step over a (256, 5120, 16) fp32 state
# ---------------------------------------------------------------------------

def run_decode(steps, warmup, args, rank, world, device, e2e_steps, want_cpu=True):
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
    reps = max(1, steps // G)
    for _ in range(max(1, warmup // G)):
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
    nsteps = reps * G
    ms_per_step = max_over_ranks([a.elapsed_time(b) / nsteps], device)[0]
    upd = dec.Bsz * dec.D * dec.N
    Bz, Dm, N = dec.Bsz, dec.D, dec.N
    byt = 8 * Bz * Dm * N + 3 * 2 * Bz * Dm + 2 * 2 * Bz * N + 2 * Bz * Dm + 4 * Dm * N + 8 * Dm
    hbm_peak, hbm_basis = measured_hbm_peak()
    gbs = byt / (ms_per_step * 1e-3) / 1e9
    # e2e through the C-ABI host-buffer step: a token's inputs come from
    # pinned host memory and y goes back, the state stays on the device
    host = [{k: v.to(bf).cpu().pin_memory() for k, v in t.items()} for t in tin[:4]]
    y_h = torch.empty((Bz, Dm), dtype=bf).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host[0].values())
    d2h = y_h.numel() * y_h.element_size()
    s0 = torch.cuda.current_stream(device)

    def e2e_step(i):
        t = host[i % 4]
        plan.step_host(states[0], t["x"], t["delta"], A, t["B"], t["C"], D=D, z=t["z"],
                       delta_bias=bias, y=y_h, stream=s0)

    for i in range(3):
        e2e_step(i)
    torch.cuda.synchronize(device)
    e1, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    E = max(8, min(e2e_steps * 10, 200))
    e1.record(s0)
    for i in range(E):
        e2e_step(i)
    e2.record(s0)
    torch.cuda.synchronize(device)
    e_ms = max_over_ranks([e1.elapsed_time(e2) / E], device)[0]
    res = {
        "metric": METRIC,
        "value": replica_throughput(upd, world, ms_per_step),
        "unit": "state-updates/s", "n_gpus": world, "steps": nsteps,
        "warmup": max(1, warmup // G) * G, "ms_per_step": ms_per_step,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded normal draws, shapes and distributions of the workload)",
        "config": dict(decode_config(dec), parallelism=f"replicas x{world}"),
        "timing": {"graph": f"{G} steps per CUDA graph",
                   "l2": "3 independent 84 MB states take turns (252 MB > 126 MB L2)"},
        "roofline": {"bound": "hbm", "achieved": gbs, "peak": hbm_peak, "unit": "GB/s",
                     "frac": gbs / hbm_peak, "peak_basis": hbm_basis,
                     "traffic": profiled_traffic("decode", "step_kernel", STEP_KERNEL_SOURCES),
                     "algorithmic_bytes": byt},
        "gpu_launches": nsteps,
        "clocks": sampler.summary(),
        "e2e": {"value": replica_throughput(upd, world, e_ms), "unit": "state-updates/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms,
                "note": "ssm_scan_step_host: token inputs in and y out over PCIe each step, "
                        "overlapped with the step by batch chunks; the state stays on the device"},
    }
    if rank == 0 and world == 1 and want_cpu and not args.no_cpu_baseline:
        res["cpu_baseline"] = decode_cpu_baselines(synth.make_decode(steps=1), args.cpu_budget_s)
    del graph
    plan.close()
    torch.cuda.empty_cache()
    return res


# ---------------------------------------------------------------------------
# CPU oracle: decode step
# ---------------------------------------------------------------------------

def oracle_decode_rate(dec, budget_s, threads):
    """Time the fp64 oracle's decode step on whole batch rows of the
    (B, D, N) state, sized to about ``budget_s`` wall seconds, on ``threads``
    host threads."""
    import concurrent.futures as cf

    import oracle
    orc = oracle.get()
    tok = dec.token(0)
    t0 = time.perf_counter()
    orc.step(dec.h0[:1, :64], tok["x"][:1, :64], tok["delta"][:1, :64], dec.A[:64], tok["B"][:1],
             tok["C"][:1], D=dec.Dskip[:64], z=tok["z"][:1, :64], delta_bias=dec.delta_bias[:64])
    per_chan = max((time.perf_counter() - t0) / 64, 1e-9)
    n_b = int(min(dec.Bsz, max(threads, budget_s * threads / per_chan / dec.D)))

    def work(b):
        orc.step(dec.h0[b:b + 1], tok["x"][b:b + 1], tok["delta"][b:b + 1], dec.A, tok["B"][b:b + 1],
                 tok["C"][b:b + 1], D=dec.Dskip, z=tok["z"][b:b + 1], delta_bias=dec.delta_bias)

    t0 = time.perf_counter()
    if threads == 1:
        for b in range(n_b):
            work(b)
    else:
        with cf.ThreadPoolExecutor(max_workers=threads) as ex:
            list(ex.map(work, range(n_b)))
    dt = time.perf_counter() - t0
    upd = n_b * dec.D * dec.N
    return upd / dt, upd, (f"{n_b} of {dec.Bsz} batch rows of one decode step "
                           f"(D={dec.D}, N={dec.N}), fp64 oracle, {threads} thread(s)")


def decode_cpu_baselines(dec, budget_s):
    allt = os.cpu_count() or 1
    out = {}
    for th in (1, allt):
        rate, _, desc = oracle_decode_rate(dec, budget_s, th)
        out[f"fp64_{'1thread' if th == 1 else 'all'}"] = {"value": rate, "threads": th,
                                                          "sample": desc}
    main = out["fp64_all"]
    return {"value": main["value"], "unit": "state-updates/s", "cores": allt, "kind": "oracle",
            "sample": main["sample"], "variants": out, "cpu": _cpu_model()}


# ---------------------------------------------------------------------------
# reference arm: the CPU oracle on a bounded sample of the same workload
# ---------------------------------------------------------------------------

def run_reference(args):
    from selective_state_space_31_b200 import synth
    threads = os.cpu_count() or 1
    # wall seconds per step, so that warm-up and timed steps end within minutes
    per_step = max(0.1, min(4.0 * args.cpu_budget_s, 120.0 / max(1, args.steps + args.warmup)))
    if args.workload == "decode":
        dec = synth.make_decode(steps=1)
        for _ in range(args.warmup):
            oracle_decode_rate(dec, per_step, threads)
        upd_total, t_total, desc = 0, 0.0, ""
        for _ in range(args.steps):
            rate, upd, desc = oracle_decode_rate(dec, per_step, threads)
            upd_total += upd
            t_total += upd / rate
        cfg = dict(decode_config(dec), parallelism=f"replicas x{args.gpus}")
    else:
        inp = synth.FWD_WORKLOADS[args.workload]()
        inp.zoh = bool(args.zoh)
        for _ in range(args.warmup):
            oracle_rate(inp, per_step, threads)
        upd_total, t_total, desc = 0, 0.0, ""
        for _ in range(args.steps):
            rate, upd, desc = oracle_rate(inp, per_step, threads)
            upd_total += upd
            t_total += upd / rate
        cfg = arm_config(inp, args.gpus, False)
    value = upd_total / t_total
    return {
        "impl": "reference",
        "metric": METRIC,
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
        "config": cfg,
        "cpu_baseline": {"value": value, "unit": "state-updates/s", "cores": threads,
                         "kind": "oracle", "sample": "per step: " + desc},
        "e2e": {"value": value, "unit": "state-updates/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ---------------------------------------------------------------------------

def sweep_steps(name):
    """Timed and warm-up steps of a per-workload record: about 0.3-0.5 s of
    timed GPU work each, so the clock sampler sees hundreds of samples."""
    return {"tiny_fp32": (2000, 50), "mamba130m_layer": (2000, 20), "mamba1p4b_layer": (400, 10),
            "long_seq": (100, 5), "decode": (9600, 192)}[name]


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
    torch.cuda.set_device(device)
    if world > 1:
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=device)
    try:
        sms = torch.cuda.get_device_properties(device).multi_processor_count
        peaks = measure_peaks(device, sms)
        if args.workload == "decode":
            res = run_decode(args.steps, args.warmup, args, rank, world, device, args.e2e_steps)
        else:
            res = run_fwd(args.workload, args.steps, args.warmup, args, rank, world, device,
                          peaks, args.e2e_steps)
        res["peaks"] = peaks
        if world == 1 and not args.no_sweep and not args.bwd and not args.zoh:
            res["workloads"] = {}
            for name in WORKLOADS:
                if name == args.workload:
                    continue
                k, w = sweep_steps(name)
                if name == "decode":
                    sub = run_decode(k, w, args, rank, world, device, args.e2e_steps)
                else:
                    sub = run_fwd(name, k, w, args, rank, world, device, peaks,
                                  args.e2e_steps)
                res["workloads"][name] = sub
            # the backward pass (ssm_scan_bwd) on the 130M layer, about 0.5 s timed
            bargs = copy.copy(args)
            bargs.bwd = True
            res["workloads"]["mamba130m_layer_backward"] = run_fwd(
                "mamba130m_layer", 500, 10, bargs, rank, world, device, peaks, 0)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
