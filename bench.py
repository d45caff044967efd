"""Benchmark of the fused selective-scan forward (one B200 per rank).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]
    python bench.py --op step [--workload step_...]     (the recurrent decode step)

A step is one pass of the whole hot path (ss_scan_fwd: discretise, scan,
read out, gate, store y and the final state) over one batch of the workload.
With `--op step` a step is one ss_scan_step call: every sequence of the batch
advances its carried state by one token.
Rank 0 prints one JSON line.  Multi-GPU runs (torchrun, one rank per GPU)
shard nothing: every rank scans its own full batch of the workload, with no
data-path collective (weak scaling); the only collectives are the timing
barrier and the max over ranks.

`--impl reference` times the fp64 CPU oracle on the host cores instead (the
reference arm): each step is a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from selective_state_space_ss_b200 import inputs as I  # noqa: E402

# the largest single-GPU workload: the million-token sequence
DEFAULT_WORKLOAD = "b1_l1048576_d1536_n16_bf16"
# the backward is measured on the B8 L2048 D1536 N16 workload (its own checkpoints fit easily)
BWD_DEFAULT_WORKLOAD = "b8_l2048_d1536_n16_bf16"
METRIC = "selective-scan fwd (B·L·D) elements/s and % of HBM/SFU roofline"
UNIT = "elements/s"
L2_BYTES = 126 * 1024 * 1024
NUM_SMS = 148
MUFU_EX2_PER_CLK_PER_SM = 16  # ex2 results per clock per SM (special-function unit)
_CSRC = "selective_state_space_ss_b200/csrc/"
# Sources each kernel's traffic record is keyed to: its device code and its own
# host code (a change to another entry point leaves the record valid).
_COMMON = ("pointwise.cuh", "scan_common.cuh", "host_common.cuh")
KERNEL_SOURCES = tuple(_CSRC + f for f in _COMMON + ("scan_fwd_chunked.cuh", "scan_fix.cuh",
                                                     "fwd_host.cuh"))
BWD_KERNEL_SOURCES = tuple(_CSRC + f for f in _COMMON + ("scan_bwd.cuh", "bwd_host.cuh"))
STEP_KERNEL_SOURCES = tuple(_CSRC + f for f in _COMMON + ("scan_step.cuh", "step_host.cuh"))


def peaks():
    p = {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0, "source": "fallback"}
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            m = json.load(f)
        p.update(hbm_gbs=float(m["hbm_gbs"]), sm_max_mhz=float(m.get("sm_max_mhz", 1965.0)),
                 source="measured")
    return p


def _code_only(text: str) -> str:
    """A source file without its comments and blank lines (the sources hold no
    string with "//" or "/*"), so that a record outlives edits of comments."""
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    lines = (ln.split("//", 1)[0].rstrip() for ln in text.splitlines())
    return "\n".join(ln for ln in lines if ln)


def kernel_hash(sources=KERNEL_SOURCES) -> str:
    """Hash of the code (not the comments) of a kernel's sources."""
    h = hashlib.sha256()
    for rel in sources:
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def profiled_traffic(workload: str, sources=KERNEL_SOURCES):
    """DRAM bytes per launch from a committed ncu summary, if taken on this kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(workload)
    if not rec or rec.get("kernel_hash") != kernel_hash(sources):
        return None
    return rec.get("dram_bytes_per_launch")


# ------------------------------------------------------------- clocks ------

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, index: int, period_s: float = 0.005):
        self.samples, self.reasons = [], set()
        self.period = period_s
        self._stop = threading.Event()
        self.max_mhz = None
        try:
            import pynvml

            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:  # NVML missing: report no clocks rather than fail the bench
            self.nv = None

    def _sample(self):
        self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
        r = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        for bit, name in self.REASONS.items():
            if r & bit:
                self.reasons.add(name)

    def _run(self):
        while not self._stop.is_set():
            self._sample()
            time.sleep(self.period)

    def __enter__(self):
        if self.nv:
            self._sample()
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.nv:
            self._stop.set()
            self.t.join()
            self._sample()

    def summary(self):
        if not self.nv or not self.samples:
            return None
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "samples": len(self.samples), "reasons": sorted(self.reasons)}


# ---------------------------------------------------------- GPU arm --------

def _dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def rank_seed(rank: int, s: int) -> int:
    """Seed of input set s on `rank`: every rank scans its own batch (weak scaling)."""
    return 1000 + 17 * rank + s


def max_over_ranks(ms: float, world: int, device) -> float:
    """Largest elapsed time over all ranks (the job ends with the slowest rank)."""
    import torch

    t = torch.tensor([ms], dtype=torch.float64, device=device)
    if world > 1:
        import torch.distributed as dist

        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(elements_per_rank: int, world: int, steps: int, ms_max: float) -> float:
    """Whole-job elements per second: all ranks' work over the slowest rank's time."""
    return elements_per_rank * world * steps / (ms_max * 1e-3)


def run_gpu_arm(args, w: I.Workload):
    import torch
    import torch.distributed as dist

    from selective_state_space_ss_b200 import (load_library, ss_scan_fwd, ss_scan_fwd_conv,
                                               ss_scan_fwd_zoh)

    world, rank, local = _dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    load_library()
    stream = torch.cuda.current_stream(dev)

    # inputs: rotate over enough sets that each step reads data last touched
    # more than one L2 capacity ago (flushing is not needed then)
    per_set = w.algorithmic_bytes()
    nsets = max(1, -(-4 * L2_BYTES // per_set))
    host = [I.make_inputs(w, seed=rank_seed(rank, s)) for s in range(nsets)]

    def to_dev(x):
        out = {}
        for k, v in x.items():
            if v is None:
                out[k] = None
            elif v.dtype == np.uint16:
                out[k] = torch.from_numpy(v.view(np.int16)).view(torch.bfloat16).to(dev)
            else:
                out[k] = torch.from_numpy(v).to(dev)
        return out

    sets = [to_dev(x) for x in host]
    ys = [torch.empty((w.batch, w.dim, w.seqlen), dtype=torch.float32, device=dev) for _ in sets]
    hs = [torch.empty((w.batch, w.dim, w.dstate), dtype=torch.float32, device=dev) for _ in sets]
    conv = None
    if args.conv:  # u = SiLU(conv1d(x)) inside the kernel; x takes u's place
        cw, cb = I.make_conv(w.dim, args.conv, seed=rank_seed(rank, 99))
        conv = (torch.from_numpy(cw).to(dev), torch.from_numpy(cb).to(dev))
        host[0]["conv"] = (cw, cb)

    if args.zoh:
        host[0]["zoh"] = True

    def scan(x, y_out, h_out, st=stream):
        if conv is None:
            fn = ss_scan_fwd_zoh if args.zoh else ss_scan_fwd
            return fn(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
                      delta_bias=x["delta_bias"], softplus=w.softplus, y_out=y_out,
                      last_state_out=h_out, stream=st)
        return ss_scan_fwd_conv(x["u"], conv[0], x["delta"], x["A"], x["B"], x["C"], D=x["D"],
                                z=x["z"], delta_bias=x["delta_bias"], conv_bias=conv[1],
                                softplus=w.softplus, y_out=y_out, last_state_out=h_out, stream=st)

    def step(i):
        s = i % nsets
        scan(sets[s], ys[s], hs[s])

    def barrier():
        if world > 1:
            dist.barrier()

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        e0.record(stream)
        for i in range(args.steps):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize()
    barrier()
    torch.cuda.synchronize()
    ms_max = max_over_ranks(e0.elapsed_time(e1), world, dev)
    ms_per_step = ms_max / args.steps
    value = job_throughput(w.elements, world, args.steps, ms_max)

    # end to end through the public call: every step copies its inputs from
    # pinned host memory to the device, scans, and copies y and the final state
    # back.  Three streams pipeline consecutive steps (step i+1's upload runs
    # while step i scans and step i-1 downloads; PCIe carries both directions at
    # once), with two device buffer sets so that no copy overwrites data in use.
    ex = host[0]
    pinned = {}
    for k, v in ex.items():
        if k in ("conv", "zoh"):
            continue
        if v is None:
            pinned[k] = None
        else:
            src = torch.from_numpy(v.view(np.int16)).view(torch.bfloat16) if v.dtype == np.uint16 \
                else torch.from_numpy(v)
            pinned[k] = src.pin_memory()
    # (one buffer set, no overlap, for workloads of several GB per step)
    nbuf = 2 if w.algorithmic_bytes() < (2 << 30) else 1
    y_host = [torch.empty((w.batch, w.dim, w.seqlen), dtype=torch.float32).pin_memory()
              for _ in range(nbuf)]
    h_host = [torch.empty((w.batch, w.dim, w.dstate), dtype=torch.float32).pin_memory()
              for _ in range(nbuf)]
    dbuf = [{k: (None if v is None else torch.empty_like(v, device=dev)) for k, v in pinned.items()}
            for _ in range(nbuf)]
    ye = [ys[0]] + [torch.empty_like(ys[0]) for _ in range(nbuf - 1)]
    he = [hs[0]] + [torch.empty_like(hs[0]) for _ in range(nbuf - 1)]
    h2d = sum(v.numel() * v.element_size() for v in pinned.values() if v is not None)
    d2h = y_host[0].numel() * 4 + h_host[0].numel() * 4
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    ev = lambda: torch.cuda.Event()
    in_done, comp_done, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for e in comp_done + out_done:
        e.record(stream)

    def e2e_step(i):
        j = i % nbuf
        s_in.wait_event(comp_done[j])  # dbuf[j] was read by step i-2's scan
        with torch.cuda.stream(s_in):
            for k, v in pinned.items():
                if v is not None:
                    dbuf[j][k].copy_(v, non_blocking=True)
        in_done[j].record(s_in)
        stream.wait_event(in_done[j])
        stream.wait_event(out_done[j])  # ye[j], he[j] were read by step i-2's download
        scan(dbuf[j], ye[j], he[j])
        comp_done[j].record(stream)
        s_out.wait_event(comp_done[j])
        with torch.cuda.stream(s_out):
            y_host[j].copy_(ye[j], non_blocking=True)
            h_host[j].copy_(he[j], non_blocking=True)
        out_done[j].record(s_out)

    e2e_steps = max(3, min(args.steps, 20))
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(s_in)
    for i in range(e2e_steps):
        e2e_step(i)
    f1.record(s_out)
    torch.cuda.synchronize()
    barrier()
    e2e_value = job_throughput(w.elements, world, e2e_steps,
                               max_over_ranks(f0.elapsed_time(f1), world, dev))

    if world > 1:
        dist.destroy_process_group()
    from selective_state_space_ss_b200 import SS_BF16, SS_F32, ss_debug_fwd_kernels

    # kernels one forward call launches for this shape: the scan, and the
    # carry-in correction when the sequence is cut into segments
    kernels = ss_debug_fwd_kernels(w.batch, w.dim, w.seqlen, w.dstate,
                                   SS_BF16 if w.dtype == "bf16" else SS_F32)
    return dict(ms_per_step=ms_per_step, value=value, world=world, rank=rank,
                kernels_per_step=kernels, clocks=clk.summary(), e2e=dict(value=e2e_value, unit=UNIT, h2d_bytes_per_step=h2d,
                                                d2h_bytes_per_step=d2h, steps=e2e_steps),
                nsets=nsets, host=host[0])


STEP_METRIC = "selective-scan decode step (B·D) channel-steps/s and % of HBM roofline"
STEP_UNIT = "channel-steps/s"


def run_step_arm(args, w: I.Workload):
    """One decode step per timed iteration; the state stays on the device."""
    import torch

    from selective_state_space_ss_b200 import load_library, ss_scan_step

    _, rank, local = _dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    load_library()
    stream = torch.cuda.current_stream(dev)
    nsets = max(1, -(-4 * L2_BYTES // I.step_bytes(w)))
    host = [I.make_step_inputs(w, seed=rank_seed(rank, s)) for s in range(nsets)]

    def to_dev(x):
        return {k: (None if v is None else
                    (torch.from_numpy(v.view(np.int16)).view(torch.bfloat16) if v.dtype == np.uint16
                     else torch.from_numpy(v)).to(dev)) for k, v in x.items()}

    sets = [to_dev(x) for x in host]
    ys = [torch.empty((w.batch, w.dim), dtype=torch.float32, device=dev) for _ in sets]

    def step(i, st):
        s = i % nsets
        x = sets[s]
        ss_scan_step(x["state"], x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"], z=x["z"],
                     delta_bias=x["delta_bias"], softplus=w.softplus, y_out=ys[s], stream=st)

    for i in range(args.warmup):
        step(i, stream)
    torch.cuda.synchronize()
    # a step takes tens of microseconds, about what one Python call costs: the
    # timed steps replay a CUDA graph of one step per input set, so the GPU
    # never waits on the host
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(nsets):
            step(i, None)  # the capture stream
    torch.cuda.synchronize()
    reps = max(1, -(-args.steps // nsets))
    steps = reps * nsets
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        e0.record(stream)
        for _ in range(reps):
            graph.replay()
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps

    # end to end: each token's inputs from pinned host memory, the step, y back;
    # the carried state lives on the device between tokens.  Uploads and
    # downloads run on their own streams with two buffer sets, so token i+1's
    # upload and token i-1's download overlap token i's step.
    tok_keys = ("u", "delta", "z", "B", "C")
    pinned = {k: (torch.from_numpy(host[0][k].view(np.int16)).view(torch.bfloat16)
                  if host[0][k].dtype == np.uint16 else torch.from_numpy(host[0][k])).pin_memory()
              for k in tok_keys if host[0][k] is not None}
    y_host = [torch.empty((w.batch, w.dim), dtype=torch.float32).pin_memory() for _ in range(2)]
    x0 = sets[0]
    dbuf = [{k: torch.empty_like(v, device=dev) for k, v in pinned.items()} for _ in range(2)]
    ye = [ys[0], torch.empty_like(ys[0])]
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    in_done = [torch.cuda.Event(), torch.cuda.Event()]
    comp_done = [torch.cuda.Event(), torch.cuda.Event()]
    out_done = [torch.cuda.Event(), torch.cuda.Event()]
    for e in comp_done + out_done:
        e.record(stream)

    def e2e_step(i):
        j = i % 2
        s_in.wait_event(comp_done[j])  # dbuf[j] was read by token i-2's step
        with torch.cuda.stream(s_in):
            for k, v in pinned.items():
                dbuf[j][k].copy_(v, non_blocking=True)
        in_done[j].record(s_in)
        stream.wait_event(in_done[j])
        stream.wait_event(out_done[j])  # ye[j] was read by token i-2's download
        d = dbuf[j]
        ss_scan_step(x0["state"], d["u"], d["delta"], x0["A"], d["B"], d["C"], D=x0["D"],
                     z=d.get("z"), delta_bias=x0["delta_bias"], softplus=w.softplus, y_out=ye[j],
                     stream=stream)
        comp_done[j].record(stream)
        s_out.wait_event(comp_done[j])
        with torch.cuda.stream(s_out):
            y_host[j].copy_(ye[j], non_blocking=True)
        out_done[j].record(s_out)

    n_e2e = max(3, min(args.steps, 50))
    for i in range(2):
        e2e_step(i)
    torch.cuda.synchronize()
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(s_in)
    for i in range(n_e2e):
        e2e_step(i)
    f1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = f0.elapsed_time(f1) / n_e2e
    chans = w.batch * w.dim
    p = peaks()
    achieved = I.step_bytes(w) / (ms * 1e-3) / 1e9
    line = {"metric": STEP_METRIC, "value": chans / (ms * 1e-3), "unit": STEP_UNIT, "n_gpus": 1,
            "steps": steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": w.name, "batch": w.batch, "dim": w.dim, "dstate": w.dstate,
                       "in_dtype": w.dtype, "state_dtype": "f32", "y_dtype": "f32",
                       "l2": "inputs and states rotated over sets totalling >= 4x L2; no flush"},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": p["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / p["hbm_gbs"],
                         "traffic": profiled_traffic(w.name, STEP_KERNEL_SOURCES),
                         "bytes_per_step": I.step_bytes(w), "peak_source": f"HBM copy, {p['source']}"},
            "e2e": {"value": chans / (e2e_ms * 1e-3), "unit": STEP_UNIT,
                    "h2d_bytes_per_step": sum(v.numel() * v.element_size() for v in pinned.values()),
                    "d2h_bytes_per_step": y_host[0].numel() * 4},
            "gpu_launches": steps, "clocks": clk.summary()}
    if not args.no_cpu_baseline:
        import oracle

        x = host[0]
        cores = os.cpu_count() or 1
        reps, t0 = 0, time.perf_counter()
        while reps < 1 or (time.perf_counter() - t0 < 5.0 and reps < 50):
            oracle.scan_step(x["state"], x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"],
                             x["delta_bias"], softplus=w.softplus, nthreads=cores)
            reps += 1
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": reps * chans / dt, "unit": STEP_UNIT, "cores": cores,
                                "kind": "oracle",
                                "sample": f"{reps} full steps of {chans} channels, fp64, {cores} threads"}
    return line


BWD_METRIC = "selective-scan backward (B·L·D) elements/s and % of SFU roofline"


def bwd_bytes(w: I.Workload) -> int:
    """Bytes a backward must move: the forward's inputs and dy once; du, ddelta,
    dz, dB, dC, dA, dD and the bias gradient once (fp32)."""
    es = 4 if w.dtype == "f32" else 2
    el = w.elements
    rd = (3 * el + 2 * w.batch * w.dstate * w.seqlen) * es + el * 4 + w.dim * (w.dstate + 2) * 4
    wr = 3 * el * 4 + 2 * w.batch * w.dstate * w.seqlen * 4 + w.dim * (w.dstate + 2) * 4
    return rd + wr


def run_bwd_arm(args, w: I.Workload):
    """One backward per step (states recomputed inside), inputs rotated."""
    import torch

    from selective_state_space_ss_b200 import load_library, ss_scan_bwd, ss_scan_bwd_workspace_bytes

    _, rank, local = _dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    load_library()
    stream = torch.cuda.current_stream(dev)
    nsets = max(1, -(-4 * L2_BYTES // bwd_bytes(w)))
    host = [I.make_inputs(w, seed=rank_seed(rank, s)) for s in range(nsets)]

    def to_dev(x):
        return {k: (None if v is None else
                    (torch.from_numpy(v.view(np.int16)).view(torch.bfloat16) if v.dtype == np.uint16
                     else torch.from_numpy(v)).to(dev)) for k, v in x.items()}

    sets = [to_dev(x) for x in host]
    dys = [torch.from_numpy(I.fill(rank_seed(rank, s), 12, (w.batch, w.dim, w.seqlen))).to(dev)
           for s in range(nsets)]
    ws = torch.empty(ss_scan_bwd_workspace_bytes(w.batch, w.dim, w.seqlen, w.dstate),
                     dtype=torch.uint8, device=dev)

    cks = [None] * nsets
    if args.ckpt:  # checkpoints from the training forward (not timed: the forward's work)
        from selective_state_space_ss_b200 import ss_scan_fwd_train

        for s_ in range(nsets):
            x = sets[s_]
            _, _, cks[s_] = ss_scan_fwd_train(x["u"], x["delta"], x["A"], x["B"], x["C"], D=x["D"],
                                              z=x["z"], delta_bias=x["delta_bias"],
                                              softplus=w.softplus, stream=stream)

    def step(i):
        x = sets[i % nsets]
        ss_scan_bwd(x["u"], x["delta"], x["A"], x["B"], x["C"], dys[i % nsets], D=x["D"], z=x["z"],
                    delta_bias=x["delta_bias"], softplus=w.softplus, checkpoints=cks[i % nsets],
                    workspace=ws, stream=stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(local) as clk:
        e0.record(stream)
        for i in range(args.steps):
            step(i)
        e1.record(stream)
        torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / args.steps
    p = peaks()
    sfu_rate = NUM_SMS * MUFU_EX2_PER_CLK_PER_SM * p["sm_max_mhz"] * 1e6
    exps = 2 * w.exps()  # a recomputing backward evaluates exp(Delta A) forward and backward
    achieved = exps / (ms * 1e-3) / 1e9
    line = {"metric": BWD_METRIC, "value": w.elements / (ms * 1e-3), "unit": UNIT, "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": dict(config_of(w, 1), op="backward",
                           checkpoints="from the training forward" if args.ckpt
                           else "computed by the backward"),
            "roofline": {"bound": "alu", "achieved": achieved, "peak": sfu_rate / 1e9, "unit": "Gexp2/s",
                         "frac": achieved * 1e9 / sfu_rate,
                         "traffic": profiled_traffic(w.name + ("+bwdck" if args.ckpt else "+bwd"),
                                                     BWD_KERNEL_SOURCES),
                         "exps_per_step": exps, "hbm_bytes_per_step": bwd_bytes(w),
                         "hbm_frac": bwd_bytes(w) / (ms * 1e-3) / 1e9 / p["hbm_gbs"]},
            "gpu_launches": args.steps, "clocks": clk.summary()}
    if not args.no_cpu_baseline:
        # the oracle's reverse sweep sums dB, dC over every channel of a row, so
        # the sample is the first batch row with its first channels, full L
        import dataclasses

        import oracle

        x = host[0]
        cores = os.cpu_count() or 1
        dims = w.dim
        ws_ = dataclasses.replace(w, batch=1, dim=dims)
        xs = {k: (None if v is None else np.ascontiguousarray(
            v[:1, :dims] if k in ("u", "delta", "z") else v[:1] if k in ("B", "C")
            else v[:dims])) for k, v in x.items()}
        dy = I.fill(7, 12, (1, dims, w.seqlen)).astype(np.float64)
        reps, t0 = 0, time.perf_counter()
        while reps < 1 or (time.perf_counter() - t0 < 10.0 and reps < 100):
            oracle.scan_bwd(xs["u"], xs["delta"], xs["A"], xs["B"], xs["C"], xs["D"], xs["z"],
                            xs["delta_bias"], softplus=w.softplus, dy=dy, nthreads=cores)
            reps += 1
        dt = time.perf_counter() - t0
        line["cpu_baseline"] = {"value": reps * ws_.elements / dt, "unit": UNIT, "cores": cores,
                                "kind": "oracle",
                                "sample": f"batch row 0 of {w.batch} ({dims} channels x full "
                                          f"L={w.seqlen}), {reps} runs, fp64 reverse sweep, "
                                          f"{cores} threads, {dt:.1f} s"}
    return line


def roofline(w: I.Workload, kernel_ms: float, variant: str = ""):
    p = peaks()
    t_hbm = w.algorithmic_bytes() / (p["hbm_gbs"] * 1e9)
    sfu_rate = NUM_SMS * MUFU_EX2_PER_CLK_PER_SM * p["sm_max_mhz"] * 1e6  # ex2 per second
    t_sfu = w.exps() / sfu_rate
    s = kernel_ms * 1e-3
    if t_sfu >= t_hbm:
        achieved = w.exps() / s / 1e9
        peak = sfu_rate / 1e9
        r = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "Gexp2/s"}
    else:
        achieved = w.algorithmic_bytes() / s / 1e9
        r = {"bound": "hbm", "achieved": achieved, "peak": p["hbm_gbs"], "unit": "GB/s"}
    r["frac"] = r["achieved"] / r["peak"]
    r["traffic"] = profiled_traffic(w.name + variant)
    r["peak_source"] = (f"SFU: {NUM_SMS} SMs x {MUFU_EX2_PER_CLK_PER_SM} ex2/clk x "
                        f"{p['sm_max_mhz']:.0f} MHz" if r["bound"] == "alu"
                        else f"HBM copy, {p['source']}")
    r["hbm_bound_us"] = t_hbm * 1e6
    r["sfu_bound_us"] = t_sfu * 1e6
    r["hbm_frac"] = (w.algorithmic_bytes() / s / 1e9) / p["hbm_gbs"]
    return r


# ---------------------------------------------------------- CPU oracle -----

def oracle_sample(w: I.Workload, x: dict, target_s: float):
    """Time the fp64 oracle on a bounded sample of channels (full sequence each)."""
    import oracle

    cores = os.cpu_count() or 1
    nch = w.batch * w.dim
    rng = np.random.default_rng(0)
    take = min(nch, max(cores, 64))
    while True:
        ch = np.sort(rng.choice(nch, take, replace=False))
        t0 = time.perf_counter()
        cw, cb = x.get("conv", (None, None))
        oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"], x["delta_bias"],
                        softplus=w.softplus, channels=ch, nthreads=cores, conv_weight=cw,
                        conv_bias=cb, zoh=x.get("zoh", False))
        dt = time.perf_counter() - t0
        if dt >= target_s or take == nch:
            return take, dt, cores
        take = min(nch, int(take * max(2.0, 1.2 * target_s / max(dt, 1e-3))))


def run_reference_arm(args, w: I.Workload):
    world, rank, _ = _dist_env()
    if world > 1:
        # the ranks meet once (gloo, host only), then rank 0 alone times the oracle
        import datetime

        import torch.distributed as dist

        dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=120))
        # one write per message (text and newline together), so that the
        # ranks' lines do not interleave on the shared stream
        sys.stderr.write(f"reference arm: rank {rank} of {world} joined\n")
        sys.stderr.flush()
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return None
    import oracle

    cores = os.cpu_count() or 1
    rng = np.random.default_rng(1)

    def sample(k):
        # k channels of batch row 0, full sequence each (only their rows are drawn)
        dims = np.sort(rng.choice(w.dim, k, replace=False))
        return I.make_row_inputs(w, 1000, 0, dims)

    def oracle_time(x):
        t0 = time.perf_counter()
        oracle.scan_fwd(x["u"], x["delta"], x["A"], x["B"], x["C"], x["D"], x["z"], x["delta_bias"],
                        softplus=w.softplus, nthreads=cores)
        return time.perf_counter() - t0

    # size one step to ~2 s of oracle work so that warmup + steps stay within minutes
    k0 = min(w.dim, cores)
    per_ch = oracle_time(sample(k0)) / k0
    take = int(min(w.dim, max(k0, 2.0 / max(per_ch, 1e-9))))
    nch = w.batch * w.dim
    x = sample(take)  # one sample, rescanned every step
    times = []
    for i in range(args.warmup + args.steps):
        dt = oracle_time(x)
        if i >= args.warmup:
            times.append(dt)
    tot = sum(times)
    value = take * w.seqlen * len(times) / tot
    desc = (f"{take} of {nch} channels (batch row 0) x full L={w.seqlen} per step, fp64, "
            f"{cores} threads")
    return {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot / len(times),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(w, world),
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle",
                             "sample": desc},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def config_of(w: I.Workload, world: int, conv: int = 0, zoh: bool = False):
    return {"workload": w.name + (f"+conv{conv}" if conv else "") + ("+zoh" if zoh else ""),
            "b_bar": "exact zoh" if zoh else "delta*B", "batch": w.batch,
            "seqlen": w.seqlen, "dim": w.dim, "dstate": w.dstate,
            "in_dtype": w.dtype, "state_dtype": "f32", "y_dtype": "f32", "conv_width": conv,
            "parallelism": f"replicas x{world} (independent batch per GPU, no collective)",
            "l2": "inputs rotated over sets totalling >= 4x L2 (126 MB); no flush"}


def _free_port() -> int:
    import socket

    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as so:
        so.bind(("127.0.0.1", 0))
        return so.getsockname()[1]


def launch_ranks(n: int) -> int:
    """Re-run this command as n ranks (one process per GPU) under
    torch.distributed.run on this node; returns the launcher's exit code."""
    import subprocess

    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={n}",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}",
           os.path.abspath(__file__), *sys.argv[1:]]
    env = dict(os.environ, SS_BENCH_LAUNCHED="1")
    return subprocess.call(cmd, env=env)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1,
                    help="ranks on this node, one per GPU (started here unless a launcher did)")
    ap.add_argument("--steps", type=int, default=50, help="timed steps")
    ap.add_argument("--warmup", type=int, default=5, help="untimed steps before them")
    ap.add_argument("--op", default="scan", choices=["scan", "step", "bwd"],
                    help="the forward scan, the recurrent decode step, or the backward")
    ap.add_argument("--workload", default=None,
                    choices=sorted(I.WORKLOADS) + sorted(I.STEP_WORKLOADS))
    ap.add_argument("--seqlen", type=int, default=None,
                    help="override the workload's sequence length (a shorter proxy of the same "
                         "batch, width and distributions, for profiling captures)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"],
                    help="reference: time the fp64 CPU oracle on a bounded sample instead")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip timing the fp64 oracle beside the GPU line")
    ap.add_argument("--zoh", action="store_true", help="exact zero-order-hold B_bar")
    ap.add_argument("--ckpt", action="store_true",
                    help="--op bwd: start from checkpoints written by the training forward")
    ap.add_argument("--conv", type=int, default=0,
                    help="fuse the short causal conv1d + SiLU of this width (1-4) into the scan")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.gpus < 1:
        ap.error("--gpus must be >= 1")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        # `python bench.py --gpus N` without a launcher: start the N ranks here
        if os.environ.get("SS_BENCH_LAUNCHED"):
            ap.error("rank launch failed: WORLD_SIZE is not set under the launcher")
        sys.exit(launch_ranks(args.gpus))
    if world != args.gpus:
        ap.error(f"--gpus {args.gpus} but the launcher started {world} ranks")
    if args.conv and args.zoh:
        ap.error("--conv and --zoh are separate kernel variants")
    if args.op == "step":
        if args.impl != "native" or args.gpus != 1:
            ap.error("--op step runs the native arm on one GPU")
        w = I.STEP_WORKLOADS[args.workload or "step_b128_d8192_n16_bf16"]
        print(json.dumps(run_step_arm(args, w)), flush=True)
        return
    if args.workload in I.STEP_WORKLOADS:
        ap.error("decode-step workloads run with --op step")
    if args.op == "bwd":
        if args.impl != "native" or args.gpus != 1:
            ap.error("--op bwd runs the native arm on one GPU")
        print(json.dumps(run_bwd_arm(args, I.WORKLOADS[args.workload or BWD_DEFAULT_WORKLOAD])),
              flush=True)
        return
    w = I.WORKLOADS[args.workload or DEFAULT_WORKLOAD]
    if args.seqlen:
        import dataclasses

        w = dataclasses.replace(w, name=w.name.replace(f"_l{w.seqlen}_", f"_l{args.seqlen}_"),
                                seqlen=args.seqlen)

    if args.impl == "reference":
        line = run_reference_arm(args, w)
        if line is not None:
            print(json.dumps(line), flush=True)
        return

    r = run_gpu_arm(args, w)
    if r["rank"] != 0:
        return
    roof = roofline(w, r["ms_per_step"], f"+conv{args.conv}" if args.conv else ("+zoh" if args.zoh else ""))
    line = {"metric": METRIC, "value": r["value"], "unit": UNIT, "n_gpus": r["world"],
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": r["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic", "config": config_of(w, r["world"], args.conv, args.zoh),
            "roofline": roof,
            "e2e": r["e2e"], "gpu_launches": args.steps * r["kernels_per_step"],
            "clocks": r["clocks"]}
    if r["world"] == 1 and not args.no_cpu_baseline:
        take, dt, cores = oracle_sample(w, r["host"], target_s=10.0)
        line["cpu_baseline"] = {"value": take * w.seqlen / dt, "unit": UNIT, "cores": cores,
                                "kind": "oracle",
                                "sample": f"{take} of {w.batch * w.dim} channels x full L={w.seqlen}, "
                                          f"fp64, {cores} threads, {dt:.1f} s"}
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
