"""Benchmark of the chunkwise gated delta-rule forward on B200.

Default workload: the Gated DeltaNet layer with 1.3B-class head geometry,
B=4, H=16, T=4096, d_k=d_v=128, chunk 64, bf16 q/k/v/o, fp32 alpha/beta and
S_T, exact blocked inversion.  One step = one gdn_chunk_fwd call over the
whole batch (every step of the hot path: staging, gate scans, Gram, inverse,
WY products, state passing, output).  Inputs are synthetic (seeded), resident
in HBM when the timed region starts.

  python bench.py [--gpus N --steps K --warmup W] [--impl reference] [--batch B]
                  [--mode exact|neumann|residual] [--decode] [--bwd]

``--batch B`` replaces the batch size (a smaller case for profiler captures).
``--decode`` times one-token decode steps; ``--bwd`` times the backward pass
(gradients of q, k, v, alpha, beta) on the same workload.  The default line
also carries a short backward timing in its ``backward`` object
(``--bwd-steps``, 0 to skip).

Under torchrun each rank runs its own independent batch (weak scaling, no
collective on the data path); the time is the max over ranks.
``--impl reference`` times the fp64 CPU oracle on a bounded sample of the
same workload (rank 0 only).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

WORKLOAD = "gdn_bf16"
METRIC = "tokens/s (fwd, bf16, H=16, d=128, T=4096) and % of roofline on 1 B200"
UNIT = "tokens/s"


# --------------------------------------------------------------------- utils

def env_int(name, default):
    try:
        return int(os.environ.get(name, default))
    except ValueError:
        return default


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        d = json.load(open(path))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16_tflops=float(d["bf16_tflops"]),
                    bf16_tflops_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16_tflops=1590.0, bf16_tflops_sustained=1400.0,
                source="fallback")


def algorithmic_bytes(w, o_bytes):
    """Bytes the method must move once: q, k, v, alpha, beta, o per token-head,
    S0 (if given) and S_T per (batch, head)."""
    in_b = 2 if w.io == "bf16" else 4
    per_th = 2 * w.dk * in_b + w.dv * in_b + w.dv * o_bytes
    per_th += 4 if w.decay in ("scalar", "weak") else (4 * w.dk if w.decay == "channel" else 0)
    per_th += 4 if w.beta else 0
    per_th += (w.dk + w.dv) * in_b if w.gates else 0
    state = w.dk * w.dv * 4 * (2 if w.s0_std > 0 else 1)
    return w.token_heads * per_th + w.B * w.H * state


def algorithmic_flops(w):
    """Per chunk-head (C tokens, triangular structure exploited): K K^T strict
    lower C(C-1)dk, Q K^T incl. diagonal C(C+1)dk, triangular inverse C^3/3,
    U and W 2C(C-1)d, W h, Q h, K^T Delta 3*2*C*dk*dv, P Delta C(C+1)dv."""
    C, dk, dv = w.chunk, w.dk, w.dv
    f = C * (C - 1) * dk + C * (C + 1) * dk + C ** 3 / 3 + C * (C - 1) * (dk + dv) \
        + 6 * C * dk * dv + C * (C + 1) * dv
    chunks = -(-w.T // C)
    return f * chunks * w.B * w.H


FWD_SOURCES = ("gdn_fused.cu", "gdn_tc_common.cuh", "sm100.cuh", "gdn_internal.cuh")
SPLIT_SOURCES = ("gdn_tc.cu", "gdn_tc_common.cuh", "sm100.cuh", "gdn_internal.cuh")
SIMT_SOURCES = ("gdn_simt.cu", "gdn_internal.cuh")
DECODE_SOURCES = ("gdn_recurrent.cu", "gdn_internal.cuh")
COUNTERS = os.path.join(ROOT, "profiles", "counters.json")


def kernel_source_sha(files=None):
    """sha256 prefix over the given kernel sources (all of csrc when None)."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "chunked_gated_delta_14_b200", "csrc")
    for fn in sorted(os.listdir(csrc)):
        if fn.endswith((".cu", ".cuh")) and (files is None or fn in files):
            h.update(open(os.path.join(csrc, fn), "rb").read())
    return h.hexdigest()[:16]


def profile_traffic(key, files, units=None):
    """DRAM read+write bytes per launch for ``key`` (kernel@workload) from the
    committed counter file, if its capture was taken on the current kernel
    sources.  A capture taken on a smaller case is scaled by ``units`` (the
    launch's units over the captured units) when given."""
    if not os.path.exists(COUNTERS):
        return None
    d = json.load(open(COUNTERS)).get(key)
    if not d or d.get("kernel_source_sha") != kernel_source_sha(files):
        return None
    t = float(d["traffic_bytes_per_launch"])
    if units is not None and d.get("units"):
        t *= units / float(d["units"])
    return t


def max_over_ranks(ms, world, device=None):
    """Slowest rank's time: every rank contributes its own event time and all
    ranks receive the maximum (an all-reduce, so the collective is the same on
    every rank)."""
    if world <= 1:
        return float(ms)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(ms)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank_step, world, steps, ms_max):
    """Whole-job rate: the units all ranks processed over the slowest rank's time."""
    return units_per_rank_step * world * steps / (ms_max / 1e3)


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.samples = []
        self.proc = None
        self.marks = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.samples.append((time.time(), line.strip()))

    def mark(self, t0, t1):
        self.marks = (t0, t1)

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        rows = self.samples
        if self.marks:
            inside = [r for r in rows if self.marks[0] <= r[0] <= self.marks[1]]
            rows = inside or rows
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for _, line in rows:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return dict(sm_mhz=None, sm_max_mhz=None, reasons=[], samples=0)
        return dict(sm_mhz=float(np.median(sm)), sm_max_mhz=float(max(smax)),
                    reasons=sorted(reasons), samples=len(sm))


def pipelined_e2e(host_in, run, steps, dev, warm=2, barrier=None):
    """End-to-end steps through the public API, timed on the device clock.

    Per step, every pinned host tensor of ``host_in`` is copied to the device,
    ``run(dev_in, slot)`` computes on the current stream and returns the device
    tensors to read back, and those are copied into pinned host buffers.
    Uploads run on one copy stream and readbacks on another, with two slots of
    device inputs: step i's compute and readback overlap step i+1's upload,
    and every step still moves all of its own bytes.  Events order each reuse
    of a slot (an upload waits for the compute that read the slot's previous
    inputs; a compute waits for the readback of the slot's previous outputs).
    Returns (ms per step, bytes uploaded per step, bytes read back per step).
    """
    import torch
    comp = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    dev_in = [{k: torch.empty_like(v, device=dev) for k, v in host_in.items()} for _ in range(2)]
    in_done = [torch.cuda.Event(), torch.cuda.Event()]
    comp_done = [torch.cuda.Event(), torch.cuda.Event()]
    out_done = [torch.cuda.Event(), torch.cuda.Event()]
    host_out = [None, None]
    used = [False, False]
    nbytes = dict(h2d=sum(v.numel() * v.element_size() for v in host_in.values()), d2h=0)

    def step(i):
        b = i & 1
        with torch.cuda.stream(s_in):
            if used[b]:
                s_in.wait_event(comp_done[b])
            for k, v in host_in.items():
                dev_in[b][k].copy_(v, non_blocking=True)
            in_done[b].record(s_in)
        comp.wait_event(in_done[b])
        if used[b]:
            comp.wait_event(out_done[b])
        res = run(dev_in[b], b)
        comp_done[b].record(comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(comp_done[b])
            if host_out[b] is None:
                host_out[b] = {k: torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for k, t in res.items()}
            for k, t in res.items():
                t.record_stream(s_out)
                host_out[b][k].copy_(t, non_blocking=True)
            out_done[b].record(s_out)
        used[b] = True
        nbytes["d2h"] = sum(t.numel() * t.element_size() for t in res.values())

    for i in range(warm):
        step(i)
    torch.cuda.synchronize()
    if barrier is not None:
        barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    s_in.wait_event(e0)
    for i in range(steps):
        step(warm + i)
    comp.wait_event(out_done[0])
    comp.wait_event(out_done[1])
    e1.record(comp)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps, nbytes["h2d"], nbytes["d2h"]


def serial_e2e(host_in, run, steps, dev, warm=2, barrier=None):
    """The same end-to-end steps as pipelined_e2e on one stream: upload, compute,
    readback, one after another."""
    import torch
    comp = torch.cuda.current_stream(dev)
    dev_in = {k: torch.empty_like(v, device=dev) for k, v in host_in.items()}
    host_out = {}
    nbytes = dict(h2d=sum(v.numel() * v.element_size() for v in host_in.values()), d2h=0)

    def step():
        for k, v in host_in.items():
            dev_in[k].copy_(v, non_blocking=True)
        res = run(dev_in, 0)
        for k, t in res.items():
            if k not in host_out:
                host_out[k] = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
            host_out[k].copy_(t, non_blocking=True)
        nbytes["d2h"] = sum(t.numel() * t.element_size() for t in res.values())

    for _ in range(warm):
        step()
    torch.cuda.synchronize()
    if barrier is not None:
        barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(comp)
    for _ in range(steps):
        step()
    e1.record(comp)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps, nbytes["h2d"], nbytes["d2h"]


def measure_e2e(host_in, run, steps, dev):
    """pipelined_e2e, or serial_e2e if the pipelined form raises; returns
    (ms per step, h2d bytes, d2h bytes, description).  Single-process runs only:
    a fallback taken by one rank alone would desynchronise the ranks' collectives."""
    try:
        ms, h2d, d2h = pipelined_e2e(host_in, run, steps, dev)
        return ms, h2d, d2h, "uploads, compute and readbacks on three streams, two input slots"
    except Exception as e:   # keep the line: time the steps on one stream instead
        ms, h2d, d2h = serial_e2e(host_in, run, steps, dev)
        return ms, h2d, d2h, f"one stream (pipelined form failed: {type(e).__name__}: {e})"


# ------------------------------------------------------------ our arm (GPU)

WORKLOAD_METRICS = {
    "gdn_bf16": METRIC,
    "plain_fp32": "tokens/s (fwd, fp32 plain delta rule, H=1, d=64, T=256) on 1 B200",
    "long_context": "tokens/s (fwd, bf16, H=16, d=128, T=65536, S0 carried, S_T returned) and % of roofline on 1 B200",
    "neumann": "tokens/s (fwd, bf16, H=16, d=128, T=4096, truncated Neumann inverse) and % of roofline on 1 B200",
    "precond_two_gate": "tokens/s (fwd, bf16, preconditioned two-gate rule, H=16, d=128, T=4096) and % of roofline on 1 B200",
}
KERNEL_NAMES = {1: "simt_prep_kernel+simt_chain_kernel", 2: "fused_kernel", 3: "recurrent_kernel",
                4: "keyside_kernel+chain_kernel"}
KERNEL_SOURCES = {1: SIMT_SOURCES, 2: FWD_SOURCES, 3: DECODE_SOURCES, 4: SPLIT_SOURCES}


def forward_runs(args):
    """(workload name, overrides) of every line this invocation prints."""
    name = args.workload
    chunk = getattr(args, "chunk", 0)
    if name == "neumann":
        return [(name, dict(chunk=c, mode="neumann", neumann_N=n)) for c in ((chunk,) if chunk else (64, 128))
                for n in (2, 3, 4)]
    over = {}
    if args.mode != "exact" and name == "gdn_bf16":
        over = dict(mode=args.mode, neumann_N=args.N)
    if chunk:
        over["chunk"] = chunk
    return [(name, over)]


def workload_text(w, mode, N, S, o_name):
    inv = {"exact": "exact inverse", "neumann": f"masked Neumann inverse N={N}",
           "residual": f"masked Neumann inverse N={N} + {S} residual terms"}[mode]
    extra = []
    if w.s0_std > 0:
        extra.append(f"S0~N(0,{w.s0_std}^2)")
    if w.gates:
        extra.append("erase/write gates, per-channel decay, preconditioned write key")
    return (f"{w.name}: B={w.B} H={w.H} T={w.T} dk={w.dk} dv={w.dv} chunk={w.chunk} {inv}"
            + (", " + ", ".join(extra) if extra else "") + f", o {o_name}")


_ORACLE_CACHE = {}


def oracle_reference(w, x):
    """fp64 oracle output (o, S_T) of the whole workload (cached per workload shape)."""
    import oracle
    key = (w.name, w.B, w.H, w.T, w.dk, w.dv)
    if key not in _ORACLE_CACHE:
        _ORACLE_CACHE[key] = oracle.gated_delta_fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"],
                                                    nthreads=len(os.sched_getaffinity(0)))
    return _ORACLE_CACHE[key]


def max_rel_rms(got, ref):
    rms = float(np.sqrt(np.mean(ref ** 2)))
    return float(np.abs(got - ref).max() / rms), float(np.sqrt(np.mean((got - ref) ** 2)) / rms)


def forward_line(args, rank, world, local_rank, name, over, timed_steps):
    import torch
    import torch.distributed as dist
    import chunked_gated_delta_14_b200 as gdn
    from chunked_gated_delta_14_b200.inputs import make_inputs, workload

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    kw = dict(over)
    if args.batch:
        kw["B"] = args.batch
    w = workload(name, **kw)
    mode = w.mode if name in ("neumann",) or "mode" in over else args.mode
    N = w.neumann_N if "neumann_N" in over else args.N
    x = make_inputs(w, seed=rank)   # each rank its own batch
    d = {k: (None if v is None else v.to(dev)) for k, v in x.items()}
    f32 = w.io == "f32"
    o_dt = torch.float32 if f32 else torch.bfloat16
    o = torch.empty((w.B, w.T, w.H, w.dv), device=dev, dtype=o_dt)
    S_T = torch.empty((w.B, w.H, w.dk, w.dv), device=dev, dtype=torch.float32)
    stream = torch.cuda.current_stream(dev)
    ptr = lambda t: None if t is None else t.data_ptr()
    general = w.gates or w.precond or w.decay == "channel"
    a = gdn.make_args(B=w.B, T=w.T, H=w.H, dk=w.dk, dv=w.dv, chunk=w.chunk, io_dtype=0 if f32 else 1,
                      o_dtype=0 if f32 else 1, q=ptr(d["q"]), k=ptr(d["k"]), v=ptr(d["v"]),
                      alpha=ptr(d["alpha"]), alpha_per_channel=int(w.decay == "channel"),
                      beta=ptr(d["beta"]), erase=ptr(d["erase"]), write=ptr(d["write"]),
                      precond=int(bool(w.precond)), S0=ptr(d["S0"]), o=o.data_ptr(),
                      S_T=S_T.data_ptr(), mode={"exact": 0, "neumann": 1, "residual": 2}[mode],
                      neumann_N=N, residual_S=args.S, kernel=gdn.gdn.KERNELS[args.kernel],
                      seq_segments=getattr(args, "segments", 0))
    ws = gdn.workspace_for(a, dev)
    if ws is not None:
        a.workspace = ws.data_ptr()
        a.workspace_bytes = ws.numel()
    kernel_id = gdn.select_kernel(a)
    kernel_name = KERNEL_NAMES.get(kernel_id, "?")
    # split tensor-core path: key side + chain (chunk 128: the band-corner kernel first
    # when there is a second half); SIMT path: prep + chain, plus the two scan kernels
    # of the preconditioner's running average
    pair = kernel_id == 4 and w.chunk == 128 and w.T > 64
    # the two-gate rule on the split path: the SIMT prep writes fp16 rows, the
    # tensor-core chain reads them (no key-side kernel)
    gen = kernel_id == 4 and general
    if pair:
        kernel_name = "pair_corner_kernel+" + kernel_name
    if gen:
        kernel_name = "simt_prep_kernel+chain_kernel"
    scans = 2 if (w.precond and general) else 0    # the preconditioner's running-average kernels
    launches_per_call = {4: 3 if pair else 2 + scans, 1: 2 + scans}.get(kernel_id, 1)
    segments = gdn.select_segments(a) if kernel_id == 4 else 1
    if segments == 3:
        # three key-side launches, five chain runs (two passes), the identity and the composition
        launches_per_call = 10
        kernel_name += "+seg_identity_kernel+seg_compose_kernel (3 sequence segments)"
    sh = stream.cuda_stream

    def step():
        gdn.call(a, sh)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    steps = timed_steps
    if steps is None:
        # a line other than the headline: about two seconds of timed calls
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        step()
        t1.record(stream)
        torch.cuda.synchronize()
        steps = int(min(args.steps, max(3, 2000.0 / max(t0.elapsed_time(t1), 1e-3))))
        if world > 1:
            steps = int(max_over_ranks(steps, world, dev))

    clocks = ClockSampler(local_rank)
    if rank == 0:
        clocks.start()
        time.sleep(1.0)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if world > 1:
        dist.barrier()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    clocks.mark(t_wall0, t_wall1)
    time.sleep(0.3)
    clocks.stop()
    gdn.device_check(sh)

    ms_step = ms / steps
    tokens_step = w.B * w.T
    value = job_throughput(tokens_step, world, steps, ms)

    # end to end through the public API: pinned host inputs -> device -> kernel -> host o and S_T
    e2e = None
    if args.e2e_steps > 0:
        host = {k: v.pin_memory() for k, v in x.items() if v is not None}
        outs = [torch.empty_like(o) for _ in range(2)]
        finals = [torch.empty_like(S_T) for _ in range(2)]

        def run(di, slot):
            gdn.chunk_fwd(di["q"], di["k"], di["v"], di.get("alpha"), di.get("beta"), erase=di.get("erase"),
                          write=di.get("write"), precond=int(bool(w.precond)), S0=di.get("S0"), chunk=w.chunk,
                          o_dtype=o_dt, out=outs[slot], mode=mode, N=N, S=args.S, S_T=finals[slot],
                          segments=getattr(args, "segments", 0),
                          kernel=args.kernel)
            return {"o": outs[slot], "S_T": finals[slot]}

        n_e2e = args.e2e_steps if timed_steps is not None else max(2, min(args.e2e_steps, steps))
        if world > 1:
            # every rank takes the same collective steps: no fallback that one rank alone could take
            ems, h2d, d2h = pipelined_e2e(host, run, n_e2e, dev, barrier=dist.barrier)
            how = "uploads, compute and readbacks on three streams, two input slots"
        else:
            ems, h2d, d2h, how = measure_e2e(host, run, n_e2e, dev)
        ems = max_over_ranks(ems, world, dev)
        e2e = dict(value=job_throughput(tokens_step, world, 1, ems), unit=UNIT,
                   h2d_bytes_per_step=int(h2d), d2h_bytes_per_step=int(d2h), ms_per_step=ems,
                   pipeline=how)

    pk = peaks()
    bytes_launch = algorithmic_bytes(w, o_bytes=4 if f32 else 2)
    achieved = bytes_launch / (ms_step / 1e3) / 1e9
    flops = algorithmic_flops(w)
    sources = SPLIT_SOURCES + SIMT_SOURCES if gen else KERNEL_SOURCES.get(kernel_id, ())
    traffic = profile_traffic(f"{kernel_name}@{name}", sources, units=w.B)
    roof = dict(bound="hbm", achieved=achieved, peak=pk["hbm_gbs"], unit="GB/s",
                frac=achieved / pk["hbm_gbs"], traffic=traffic,
                peak_source=pk["source"] + " (burst copy bandwidth)",
                algorithmic_bytes_per_launch=bytes_launch,
                tensor_tflops=flops / (ms_step / 1e3) / 1e12,
                tensor_frac_of_bf16_peak=flops / (ms_step / 1e3) / 1e12 / pk["bf16_tflops"],
                roofline_ms=max(bytes_launch / (pk["hbm_gbs"] * 1e9),
                                flops / (pk["bf16_tflops"] * 1e12)) * 1e3)
    if kernel_id == 1 or gen:
        # the SIMT path computes in fp32 on the CUDA cores: its bound is the fp32
        # arithmetic of the chunk algebra, not HBM (the HBM figures stay alongside);
        # so does the two-gate rule's prep, the larger part of its split path
        alu_peak = fp32_alu_peak_tflops(1965.0)
        ach = flops / (ms_step / 1e3) / 1e12
        roof = dict(bound="alu", achieved=ach, peak=alu_peak, unit="TFLOP/s", frac=ach / alu_peak,
                    traffic=traffic, peak_source="derived: 148 SMs x 128 fp32 lanes x 2 flops x max SM clock",
                    algorithmic_flops_per_launch=flops, algorithmic_bytes_per_launch=bytes_launch,
                    hbm_gbs=achieved, hbm_frac=achieved / pk["hbm_gbs"],
                    roofline_ms=max(flops / (alu_peak * 1e12), bytes_launch / (pk["hbm_gbs"] * 1e9)) * 1e3)
    if name == "plain_fp32":
        roof["note"] = "0.3 MB per call: launch-latency bound, the fractions are only reported"

    clk = clocks.summary() if rank == 0 else dict(sm_max_mhz=None)
    accuracy = None
    if mode == "neumann" and rank == 0 and world == 1 and not general:
        # the truncated series against exact inversion (same kernel family, exact mode)
        # and against the fp64 oracle, on this whole workload; o in fp32 here, so
        # that the bf16 rounding of the output is not counted as method error
        o32 = torch.empty((w.B, w.T, w.H, w.dv), device=dev, dtype=torch.float32)
        a.o, a.o_dtype = o32.data_ptr(), 0
        step()
        torch.cuda.synchronize()
        o_n = o32.double().cpu().numpy()
        s_n = S_T.double().cpu().numpy()
        a.mode, a.neumann_N = 0, 0
        ws_x = gdn.workspace_for(a, dev)    # exact inversion may run on another kernel
        if ws_x is not None:
            a.workspace, a.workspace_bytes = ws_x.data_ptr(), ws_x.numel()
        exact_kernel = KERNEL_NAMES.get(gdn.select_kernel(a), "?")
        step()
        torch.cuda.synchronize()
        o_x = o32.double().cpu().numpy()
        s_x = S_T.double().cpu().numpy()
        o_ref, s_ref = oracle_reference(w, x)
        m_o, r_o = max_rel_rms(o_n, o_x)
        m_s, r_s = max_rel_rms(s_n, s_x)
        mo_o, ro_o = max_rel_rms(o_n, o_ref)
        mo_s, ro_s = max_rel_rms(s_n, s_ref)
        accuracy = dict(
            vs_exact_inverse=dict(o_max_rel_rms=m_o, o_rms_rel=r_o, S_T_max_rel_rms=m_s, S_T_rms_rel=r_s,
                                  exact_kernel=exact_kernel),
            vs_exact_oracle=dict(o_max_rel_rms=mo_o, o_rms_rel=ro_o, S_T_max_rel_rms=mo_s, S_T_rms_rel=ro_s),
            note="the truncated series' method error against exact inversion (this library in exact "
                 "mode) and against the fp64 token recurrence, o in fp32; parity with the masked-series "
                 "oracle (max|err| <= 2e-2 * rms) is the tests' check, not this one")

    backward = None
    if name == "gdn_bf16" and args.bwd_steps > 0 and world == 1:
        try:
            backward = backward_side_measure(w, x, rank, world, dev, args.bwd_steps, 3, clk["sm_max_mhz"])
        except Exception as e:   # the forward line is printed either way, with the reason
            backward = dict(error=f"{type(e).__name__}: {e}")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(w, x, budget_s=args.cpu_budget)

    if rank == 0:
        line = dict(metric=WORKLOAD_METRICS[name], value=value, unit=UNIT, n_gpus=world, steps=steps,
                    warmup=args.warmup, ms_per_step=ms_step, higher_is_better=True,
                    scaling="weak", vs_baseline=None, dtype="f32" if f32 else "bf16",
                    compute=("fp32 CUDA cores" if kernel_id == 1 else
                             "fp32 CUDA-core prep; fp16 tensor-core chain operands, fp32 accumulate and state"
                             if gen else
                             "bf16 q/k/v in HBM; fp16 tensor-core operands, fp32 accumulate and state"),
                    data="synthetic (seeded; Gated DeltaNet layer shapes)",
                    parity=("o and S_T meet max|err| <= 2e-2 * rms(oracle) with an fp32 o (the parity tests); "
                            "the bf16 o timed here adds its own rounding, 2^-9 |o|, checked as "
                            "|err| <= 2e-2 * rms + 2^-8 |ref|" if not f32 else
                            "o and S_T against the fp64 oracle at max|err| <= 1e-4 (the parity tests)"),
                    config=dict(workload=workload_text(w, mode, N, args.S, "fp32" if f32 else "bf16"),
                                global_batch=w.B * world, seq_len=w.T,
                                parallelism=f"independent batch per GPU x{world}",
                                l2=(f"no flush: inputs+outputs {bytes_launch / 1e6:.0f} MB per step > 126 MB L2"
                                    if bytes_launch > 126e6 else
                                    f"no flush: {bytes_launch / 1e6:.1f} MB per step (fits L2)"),
                                kernel=kernel_name),
                    clocks=clk,
                    e2e=e2e, gpu_launches=steps * launches_per_call, roofline=roof,
                    cpu_baseline=cpu)
        if accuracy is not None:
            line["accuracy"] = accuracy
        if backward is not None:
            line["backward"] = backward
        if world > 1:
            line["note"] = "multi-rank run: the backward object is measured in single-GPU runs only"
        print(json.dumps(line), flush=True)


def run_gpu(args, rank, world, local_rank):
    for i, (name, over) in enumerate(forward_runs(args)):
        headline = name == "gdn_bf16"
        forward_line(args, rank, world, local_rank, name, over, args.steps if headline else None)


DECODE_METRIC = "decode tokens/s (bf16, H=16, d=128, one token per sequence, state in place) and % of HBM roofline on 1 B200"


def decode_bytes(w):
    """Per step: the fp32 state read and written, q, k, v in and o out (bf16), alpha, beta."""
    return w.B * w.H * (2 * w.dk * w.dv * 4 + (2 * w.dk + w.dv) * 2 + w.dv * 2 + 8)


def run_decode(args, rank, world, local_rank):
    """One decode step per call: T = 1 for B sequences, the state updated in place."""
    import torch
    import chunked_gated_delta_14_b200 as gdn
    from chunked_gated_delta_14_b200.inputs import make_inputs, workload

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workload(WORKLOAD, B=args.batch or 256, T=1, s0_std=0.02)
    x = make_inputs(w, seed=rank)
    d = {k: (None if v is None else v.to(dev)) for k, v in x.items()}
    state = d["S0"].clone()
    o = torch.empty((w.B, 1, w.H, w.dv), device=dev, dtype=torch.bfloat16)
    ptr = lambda t: None if t is None else t.data_ptr()
    a = gdn.make_args(B=w.B, T=1, H=w.H, dk=w.dk, dv=w.dv, chunk=w.chunk, io_dtype=1, o_dtype=1,
                      q=ptr(d["q"]), k=ptr(d["k"]), v=ptr(d["v"]), alpha=ptr(d["alpha"]),
                      beta=ptr(d["beta"]), S0=state.data_ptr(), o=o.data_ptr(), S_T=state.data_ptr(),
                      mode=0, kernel=0)
    assert gdn.select_kernel(a) == 3, "decode steps run on the recurrent kernel"
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    for _ in range(args.warmup):
        gdn.call(a, sh)
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    if rank == 0:
        clocks.start()
        time.sleep(1.0)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        gdn.call(a, sh)
    e1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    clocks.mark(t_wall0, t_wall1)
    time.sleep(0.3)
    clocks.stop()
    ms_step = ms / args.steps
    value = job_throughput(w.B, world, args.steps, ms)

    # end to end: this step's q, k, v, alpha, beta from pinned host memory, o back
    host = {k: x[k].pin_memory() for k in ("q", "k", "v", "alpha", "beta")}
    o_host = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
    h2d = sum(t.numel() * t.element_size() for t in host.values())
    d2h = o_host.numel() * o_host.element_size()

    def e2e_step():
        for k, t in host.items():
            d[k].copy_(t, non_blocking=True)
        gdn.call(a, sh)
        o_host.copy_(o, non_blocking=True)

    for _ in range(3):
        e2e_step()
    torch.cuda.synchronize()
    f0 = torch.cuda.Event(enable_timing=True)
    f1 = torch.cuda.Event(enable_timing=True)
    n_e2e = max(1, args.e2e_steps * 10)
    f0.record(stream)
    for _ in range(n_e2e):
        e2e_step()
    f1.record(stream)
    torch.cuda.synchronize()
    ems = max_over_ranks(f0.elapsed_time(f1), world, dev)
    e2e = dict(value=job_throughput(w.B, world, n_e2e, ems), unit=UNIT, h2d_bytes_per_step=int(h2d),
               d2h_bytes_per_step=int(d2h), ms_per_step=ems / n_e2e)

    pk = peaks()
    bytes_step = decode_bytes(w)
    achieved = bytes_step / (ms_step / 1e3) / 1e9
    traffic = profile_traffic("recurrent_kernel@decode", DECODE_SOURCES, units=w.B)
    roof = dict(bound="hbm", achieved=achieved, peak=pk["hbm_gbs"], unit="GB/s",
                frac=achieved / pk["hbm_gbs"], traffic=traffic,
                peak_source=pk["source"] + " (burst copy bandwidth)",
                algorithmic_bytes_per_launch=bytes_step,
                roofline_ms=bytes_step / (pk["hbm_gbs"] * 1e9) * 1e3)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        cores = len(os.sched_getaffinity(0))
        n, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < min(args.cpu_budget, 3.0):
            oracle.gated_delta_fwd(x["q"], x["k"], x["v"], x["alpha"], x["beta"], x["S0"], nthreads=cores)
            n += 1
        el = time.perf_counter() - t0
        cpu = dict(value=w.B * n / el, unit=UNIT, cores=cores, kind="oracle",
                   sample=f"{n} decode steps of all {w.B} x {w.H} heads, fp64 C oracle, {el:.1f} s")
    if rank == 0:
        line = dict(metric=DECODE_METRIC, value=value, unit=UNIT, n_gpus=world, steps=args.steps,
                    warmup=args.warmup, ms_per_step=ms_step, higher_is_better=True, scaling="weak",
                    vs_baseline=None, dtype="bf16",
                    compute="bf16 q/k/v/o in HBM; fp32 state, fp32 arithmetic",
                    data="synthetic (seeded; Gated DeltaNet layer shapes)",
                    config=dict(workload=f"decode: B={w.B} H={w.H} T=1 dk={w.dk} dv={w.dv}, state in place",
                                global_batch=w.B * world, seq_len=1,
                                parallelism=f"independent batch per GPU x{world}",
                                l2=f"no flush: state {w.B * w.H * w.dk * w.dv * 4 / 1e6:.0f} MB read and "
                                   f"written per step > 126 MB L2",
                                kernel="recurrent_kernel"),
                    clocks=clocks.summary(), e2e=e2e, gpu_launches=args.steps, roofline=roof,
                    cpu_baseline=cpu)
        print(json.dumps(line), flush=True)


BWD_METRIC = "backward tokens/s (bf16 in, fp32 gradients, H=16, d=128, T=4096) and % of fp32 roofline on 1 B200"
BWD_SOURCES = ("gdn_bwd.cu", "gdn_bwd_kernels.cuh", "gdn_bwd_params.cuh")


def fp32_alu_peak_tflops(sm_mhz=1965.0):
    """CUDA-core fp32 peak: 148 SMs x 128 fp32 lanes x 2 flops (FMA) x clock."""
    return 148 * 128 * 2 * sm_mhz * 1e6 / 1e12


def algorithmic_flops_bwd(w):
    """Per chunk-head, the products of the chunked backward (fp32):
    8 state-sized products 2*C*dk*dv (Delta = U - W h, the state update; dDelta's
    K dh', the two terms of dh; dO h^T, Y h^T, Delta dh'^T), the score-sized ones
    C^2 (9 dk + 5 dv) (Gram and scores twice, W and U, M^T dO and T^T dDelta,
    dO Delta^T and Y Delta^T, the four score-times-key products of dq and dk)
    and the triangular inverse C^3 / 3."""
    C, dk, dv = w.chunk, w.dk, w.dv
    f = 16 * C * dk * dv + C * C * (9 * dk + 5 * dv) + C ** 3 / 3
    return f * -(-w.T // C) * w.B * w.H


def bwd_bytes(w):
    """Bytes the backward must move once: q, k, v, grad_o read (io dtype), alpha,
    beta read (fp32); dq, dk, dv, dalpha, dbeta written (fp32)."""
    in_b = 2 if w.io == "bf16" else 4
    per_th = (2 * w.dk + 2 * w.dv) * in_b + 8 + (2 * w.dk + w.dv) * 4 + 8
    return w.token_heads * per_th


def bwd_setup(w, x, c, dev, mode="exact", N=3, S=8):
    """Device copies of the inputs and dL/do, fp32 gradient buffers and the
    gdn_bwd_args (with workspace) of one backward call over the whole batch
    (``mode`` "neumann": the gradient of the masked truncated series of order N;
    "residual": of that series with S correction terms).
    The args hold raw pointers: the returned dict keeps every tensor they point
    to alive."""
    import torch
    import chunked_gated_delta_14_b200 as gdn
    d = {k: (None if v is None else v.to(dev)) for k, v in x.items()}
    grad_o = c["grad_o"].to(dev)
    f32 = dict(device=dev, dtype=torch.float32)
    g = dict(dq=torch.empty((w.B, w.T, w.H, w.dk), **f32), dk=torch.empty((w.B, w.T, w.H, w.dk), **f32),
             dv=torch.empty((w.B, w.T, w.H, w.dv), **f32), da=torch.empty((w.B, w.T, w.H), **f32),
             db=torch.empty((w.B, w.T, w.H), **f32))
    ptr = lambda t: None if t is None else t.data_ptr()
    a = gdn.make_bwd_args(B=w.B, T=w.T, H=w.H, dk=w.dk, dv=w.dv, chunk=w.chunk, io_dtype=1,
                          do_dtype=1, q=ptr(d["q"]), k=ptr(d["k"]), v=ptr(d["v"]),
                          alpha=ptr(d["alpha"]), beta=ptr(d["beta"]), grad_o=ptr(grad_o),
                          grad_q=ptr(g["dq"]), grad_k=ptr(g["dk"]), grad_v=ptr(g["dv"]),
                          grad_alpha=ptr(g["da"]), grad_beta=ptr(g["db"]),
                          mode={"exact": 0, "neumann": 1, "residual": 2}[mode],
                          neumann_N=int(N) if mode != "exact" else 0, residual_S=int(S) if mode == "residual" else 0)
    ws = gdn.workspace_for(a, dev)
    a.workspace, a.workspace_bytes = ws.data_ptr(), ws.numel()
    g["inputs"], g["grad_o"] = d, grad_o
    return a, g, ws


def bwd_roofline(w, ms_step, sm_max_mhz, neumann=False):
    """ALU roofline of one backward call.  With the masked series the FLOP count is
    the exact mode's (the adjoint kernel's C x C products are not counted) and no
    traffic is reported (the committed capture is of the exact mode)."""
    pk = peaks()
    alu_peak = fp32_alu_peak_tflops(sm_max_mhz or 1965.0)
    flops = algorithmic_flops_bwd(w)
    achieved = flops / (ms_step / 1e3) / 1e12
    nbytes = bwd_bytes(w)
    return dict(bound="alu", achieved=achieved, peak=alu_peak, unit="TFLOP/s", frac=achieved / alu_peak,
                traffic=None if neumann else profile_traffic("backward@gdn_bf16", BWD_SOURCES, units=w.B),
                peak_source="derived: 148 SMs x 128 fp32 lanes x 2 flops x max SM clock",
                algorithmic_flops_per_launch=flops, algorithmic_bytes_per_launch=nbytes,
                hbm_gbs=nbytes / (ms_step / 1e3) / 1e9, hbm_frac=nbytes / (ms_step / 1e3) / 1e9 / pk["hbm_gbs"],
                roofline_ms=max(flops / (alu_peak * 1e12), nbytes / (pk["hbm_gbs"] * 1e9)) * 1e3)


def backward_side_measure(w, x, rank, world, dev, steps, warmup, sm_max_mhz):
    """The backward pass timed on the forward's workload (for the forward line's
    ``backward`` object): one gdn_chunk_bwd call per step, CUDA events, max over
    ranks."""
    import torch
    import chunked_gated_delta_14_b200 as gdn
    from chunked_gated_delta_14_b200.inputs import make_cotangents
    c = make_cotangents(w, seed=rank, grad_state=False)
    a, g, ws = bwd_setup(w, x, c, dev)
    stream = torch.cuda.current_stream(dev)
    for _ in range(warmup):
        gdn.call_bwd(a, stream.cuda_stream)
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        gdn.call_bwd(a, stream.cuda_stream)
    e1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    ms_step = ms / steps
    out = dict(metric=BWD_METRIC, value=job_throughput(w.B * w.T, world, steps, ms), unit=UNIT,
               steps=steps, warmup=warmup, ms_per_step=ms_step, dtype="f32",
               gpu_launches=4 * steps, roofline=bwd_roofline(w, ms_step, sm_max_mhz),
               note="gradients of q, k, v, alpha, beta on the same workload; full line: bench.py --bwd")
    del a, g, ws
    return out


def run_bwd(args, rank, world, local_rank):
    """One gdn_chunk_bwd call per step over the whole batch."""
    import torch
    import torch.distributed as dist
    import chunked_gated_delta_14_b200 as gdn
    from chunked_gated_delta_14_b200.inputs import make_cotangents, make_inputs, workload

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workload(WORKLOAD, **({"B": args.batch} if args.batch else {}))
    x = make_inputs(w, seed=rank)
    c = make_cotangents(w, seed=rank, grad_state=False)
    neumann = args.mode in ("neumann", "residual")
    a, g, ws = bwd_setup(w, x, c, dev, mode=args.mode, N=args.N, S=args.S)
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    for _ in range(args.warmup):
        gdn.call_bwd(a, sh)
    torch.cuda.synchronize()
    clocks = ClockSampler(local_rank)
    if rank == 0:
        clocks.start()
        time.sleep(1.0)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    e0.record(stream)
    for _ in range(args.steps):
        gdn.call_bwd(a, sh)
    e1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    ms = max_over_ranks(e0.elapsed_time(e1), world, dev)
    clocks.mark(t_wall0, t_wall1)
    time.sleep(0.3)
    clocks.stop()
    ms_step = ms / args.steps
    tokens_step = w.B * w.T
    value = job_throughput(tokens_step, world, args.steps, ms)

    # end to end through chunk_bwd: pinned host inputs and grad_o in, gradients back out
    e2e = None
    if args.e2e_steps > 0:
        host = {k: x[k].pin_memory() for k in ("q", "k", "v", "alpha", "beta")}
        host["grad_o"] = c["grad_o"].pin_memory()

        def run(di, slot):
            r = gdn.chunk_bwd(di["q"], di["k"], di["v"], di["alpha"], di["beta"], di["grad_o"],
                              mode=args.mode, N=args.N, S=args.S,
                              chunk=w.chunk, want_S0=False)
            return {k: r[k] for k in ("dq", "dk", "dv", "dalpha", "dbeta")}

        n_e2e = max(1, args.e2e_steps // 4)
        if world > 1:
            # every rank takes the same collective steps: no fallback that one rank alone could take
            ems, h2d, d2h = pipelined_e2e(host, run, n_e2e, dev, barrier=dist.barrier)
            how = "uploads, compute and readbacks on three streams, two input slots"
        else:
            ems, h2d, d2h, how = measure_e2e(host, run, n_e2e, dev)
        ems = max_over_ranks(ems, world, dev)
        e2e = dict(value=job_throughput(tokens_step, world, 1, ems), unit=UNIT,
                   h2d_bytes_per_step=int(h2d), d2h_bytes_per_step=int(d2h), ms_per_step=ems,
                   pipeline=how)

    clk = clocks.summary()
    nbytes = bwd_bytes(w)
    roof = bwd_roofline(w, ms_step, clk["sm_max_mhz"], neumann=neumann)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        cores = len(os.sched_getaffinity(0))
        Ts = min(w.T, 256 if neumann else 1024)
        sl = lambda t: None if t is None else t[0:1, :Ts].contiguous()
        n, t0 = 0, time.perf_counter()
        while True:
            if neumann:
                from oracle import chunk_grad
                chunk_grad.neumann_bwd(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["alpha"]), sl(x["beta"]), None,
                                       sl(c["grad_o"]), None, chunk=w.chunk, N=args.N,
                                       S=args.S if args.mode == "residual" else None)
            else:
                oracle.gated_delta_bwd(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["alpha"]), sl(x["beta"]),
                                   None, sl(c["grad_o"]), None, nthreads=cores)
            n += 1
            if time.perf_counter() - t0 >= min(args.cpu_budget, 10.0):
                break
        el = time.perf_counter() - t0
        how = "fp64 autograd of the series' chunk model (torch CPU ops)" if neumann else "fp64 C adjoint"
        cpu = dict(value=Ts * n / el, unit=UNIT, cores=torch.get_num_threads() if neumann else cores, kind="oracle",
                   sample=f"{n} x (tokens [0,{Ts}) of one batch row, all {w.H} heads), {how}, {el:.1f} s")
    if rank == 0:
        line = dict(metric=BWD_METRIC, value=value, unit=UNIT, n_gpus=world, steps=args.steps,
                    warmup=args.warmup, ms_per_step=ms_step, higher_is_better=True, scaling="weak",
                    vs_baseline=None, dtype="f32",
                    compute="bf16 q/k/v/grad_o in HBM; fp32 arithmetic on CUDA cores; fp32 gradients",
                    data="synthetic (seeded; Gated DeltaNet layer shapes)",
                    config=dict(workload=f"{WORKLOAD} backward: B={w.B} H={w.H} T={w.T} dk={w.dk} "
                                f"dv={w.dv} chunk={w.chunk} "
                                + ("exact inverse" if not neumann else
                                   f"masked truncated Neumann inverse N={args.N}"
                                   + (f" with {args.S} residual-correction terms" if args.mode == "residual" else "")),
                                global_batch=w.B * world, seq_len=w.T,
                                parallelism=f"independent batch per GPU x{world}",
                                l2=f"no flush: inputs+gradients {nbytes / 1e6:.0f} MB + workspace "
                                   f"{ws.numel() / 1e6:.0f} MB per step > 126 MB L2",
                                kernel="bwd_prep_kernel+bwd_state_fwd_kernel+bwd_state_rev_kernel+"
                                       + ("bwd_neumann_kernel+" if neumann else "") + "bwd_grad_kernel"),
                    clocks=clk, e2e=e2e, gpu_launches=args.steps * (5 if neumann else 4), roofline=roof,
                    cpu_baseline=cpu)
        print(json.dumps(line), flush=True)


def cpu_baseline(w, x, budget_s=12.0):
    """The fp64 oracle as it stands, timed on this host's cores, on whole
    (batch, head) sequences of the same workload until ~budget_s seconds."""
    import oracle
    cores = len(os.sched_getaffinity(0))
    H = w.H
    done_th = 0
    t0 = time.time()
    b = 0
    two_gate = w.gates or w.precond or w.decay == "channel"
    while True:
        sl = lambda t: None if t is None else t[b:b + 1]
        if two_gate:
            oracle.precond_two_gate_fwd(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["alpha"]), sl(x["erase"]),
                                        sl(x["write"]), precond=int(bool(w.precond)), h0=sl(x["S0"]),
                                        nthreads=cores)
        else:
            oracle.gated_delta_fwd(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["alpha"]),
                                   sl(x["beta"]), sl(x["S0"]), nthreads=cores)
        done_th += w.T * H
        b = (b + 1) % w.B
        if time.time() - t0 >= budget_s:
            break
    el = time.time() - t0
    return dict(value=done_th / H / el, unit=UNIT, cores=cores, kind="oracle",
                sample=f"{done_th // (w.T * H)} x (batch row of {H} heads x {w.T} tokens) "
                       f"of {w.name}, fp64 C oracle, {el:.1f} s")


# ------------------------------------------------- reference arm (the oracle)

def run_reference(args, rank, world):
    if rank != 0:
        return
    import oracle
    from chunked_gated_delta_14_b200.inputs import make_inputs, workload
    name = args.workload
    w = workload(name, **({"B": args.batch} if args.batch else {}))
    two_gate = w.gates or w.precond or w.decay == "channel"
    x = make_inputs(w)
    cores = len(os.sched_getaffinity(0))
    # per-step sample: a prefix of one (batch, head) row group sized so that
    # warmup + steps fit in about args.ref_budget seconds
    total_steps = max(1, args.steps + args.warmup)
    per_step_s = args.ref_budget / total_steps
    probe_T = 256
    t0 = time.time()
    sl = lambda t, b, n: None if t is None else t[b:b + 1, :n].contiguous()
    def run_oracle(b, n):
        if two_gate:
            oracle.precond_two_gate_fwd(sl(x["q"], b, n), sl(x["k"], b, n), sl(x["v"], b, n),
                                        sl(x["alpha"], b, n), sl(x["erase"], b, n), sl(x["write"], b, n),
                                        precond=int(bool(w.precond)), h0=x["S0"][b:b + 1] if x["S0"] is not None
                                        else None, nthreads=cores)
        else:
            oracle.gated_delta_fwd(sl(x["q"], b, n), sl(x["k"], b, n), sl(x["v"], b, n), sl(x["alpha"], b, n),
                                   sl(x["beta"], b, n), x["S0"][b:b + 1] if x["S0"] is not None else None,
                                   nthreads=cores)
    run_oracle(0, probe_T)
    rate = probe_T / max(time.time() - t0, 1e-6)           # tokens (all heads) per second
    Ts = int(min(w.T, max(16, rate * per_step_s)))
    def step(i):
        run_oracle(i % w.B, Ts)
    for i in range(args.warmup):
        step(i)
    t0 = time.perf_counter()
    for i in range(args.steps):
        step(i)
    el = time.perf_counter() - t0
    value = Ts * args.steps / el
    sample = f"tokens [0,{Ts}) of one batch row (all {w.H} heads) of {name} per step"
    line = dict(impl="reference", metric=WORKLOAD_METRICS[name], value=value, unit=UNIT, n_gpus=world,
                steps=args.steps, warmup=args.warmup, ms_per_step=el / args.steps * 1e3,
                higher_is_better=True, scaling="weak", vs_baseline=None, dtype="f64",
                data="synthetic (seeded; Gated DeltaNet layer shapes)",
                config=dict(workload=workload_text(w, "exact" if name != "neumann" else "neumann",
                                                   w.neumann_N, args.S, "fp32" if w.io == "f32" else "bf16"),
                            global_batch=w.B, seq_len=w.T,
                            parallelism="CPU oracle, rank 0 only"),
                cpu_baseline=dict(value=value, unit=UNIT, cores=cores, kind="oracle",
                                  sample=sample),
                e2e=dict(value=value, unit=UNIT, h2d_bytes_per_step=0, d2h_bytes_per_step=0))
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--e2e-steps", type=int, default=20)
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--ref-budget", type=float, default=60.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=0, help="replace the batch size B (profiler case)")
    ap.add_argument("--workload", default="gdn_bf16", choices=sorted(WORKLOAD_METRICS),
                    help="gdn_bf16 (the headline, default), plain_fp32, long_context, neumann "
                         "(one line per chunk 64/128 x N 2/3/4 with its error against exact inversion "
                         "and the oracle) or precond_two_gate")
    ap.add_argument("--mode", default="exact", choices=["exact", "neumann", "residual"],
                    help="inverse: exact (the headline workload), masked Neumann series "
                         "(order --N), or the series with --S residual-correction terms")
    ap.add_argument("--decode", action="store_true",
                    help="decode steps (T = 1, state in place, B = 256 unless --batch)")
    ap.add_argument("--bwd", action="store_true",
                    help="the backward pass (gradients) on the same workload")
    ap.add_argument("--bwd-steps", type=int, default=20,
                    help="backward calls timed for the forward line's 'backward' object (0: none)")
    ap.add_argument("--segments", type=int, default=0, choices=[0, 1, 3],
                    help="sequence segments of the split tensor-core path (0: the library's choice)")
    ap.add_argument("--kernel", default="auto", choices=["auto", "simt", "tc", "tc_split"],
                    help="force one forward kernel (auto: the library's choice)")
    ap.add_argument("--chunk", type=int, default=0,
                    help="chunk length (0: the workload's own; for --workload neumann, the lines of that chunk only)")
    ap.add_argument("--N", type=int, default=3)
    ap.add_argument("--S", type=int, default=8)
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    world = env_int("WORLD_SIZE", 1)
    rank = env_int("RANK", 0)
    local_rank = env_int("LOCAL_RANK", 0)
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        if args.decode:
            run_decode(args, rank, world, local_rank)
        elif args.bwd:
            run_bwd(args, rank, world, local_rank)
        else:
            run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
