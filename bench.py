#!/usr/bin/env python
"""Throughput benchmark of HaloNet blocked local self-attention on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl halo|reference]

One step = one pass of the whole fused operation (block + halo gather,
content and relative logits, masked softmax, A.V, NHWC store) over one batch
of the stage-1 HaloNet layer: N=32, 64x64 map, 8 heads x dim_head 16, block 8,
halo 3 (14x14 window), stride 1, bf16 in / fp32 accumulate, seeded synthetic
inputs already resident in HBM.  The metric is output pixels/s (TFLOP/s
reported beside it).

Multi-GPU (torchrun, one process per GPU): every rank runs its own batch of
independent images (weak scaling, no data-path collective); timing is the max
over ranks.  --impl reference times the CPU oracle (the slow double-precision
reference) on the host cores instead, on rank 0 only.
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

import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "halo-attention output pixels/s and TFLOP/s, % of bf16 tensor/HBM roofline"
PROFILES = os.path.join(ROOT, "profiles")
L2_BYTES = 126 * 1024 * 1024


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["halo", "reference"], default="halo")
    ap.add_argument("--workload", default=workloads.BENCH_WORKLOAD,
                    choices=sorted(workloads.WORKLOADS) + sorted(workloads.NEXT_WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every step from Python instead of replaying captured CUDA graphs")
    ap.add_argument("--min-timed-s", type=float, default=0.5,
                    help="repeat the K-step timed region until about this much time is covered (median reported)")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip timing every workload for the per_config object")
    ap.add_argument("--pass", dest="which", choices=["fwd", "bwd", "masked", "fused"], default="fwd",
                    help="what one step runs: the forward (default), the backward (halo_attn_bwd, one launch per "
                         "step from Python), the SASA-masked forward with a 2*halo+1 window, or the forward with "
                         "the q, k, v projections fused in (halo_attn_fused; workloads with a fused form)")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip timing the backward and the SASA-masked forward (next_rows object)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def dist_init(world):
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Max of a per-rank timing over all ranks (the only collective: timing)."""
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(wl, rank: int) -> int:
    """Each rank draws its own batch of independent images (weak scaling)."""
    return wl.seed + 1000 * rank


def dist_done(world):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi clocks / throttle reasons sampled every 100 ms in the background."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100",
                 "-i", str(self.index), "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.4)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def cleanup(self):
        try:
            if self.path:
                os.unlink(self.path)
        except OSError:
            pass

    def summary(self, t0: float, t1: float, keep: bool = False) -> dict:
        rows = []
        try:
            with open(self.path) as f:
                for line in f:
                    parts = [p.strip() for p in line.split(",")]
                    if len(parts) < 10:
                        continue
                    try:
                        ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                        ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                    except (ValueError, IndexError):
                        continue
                    rows.append((ts, parts))
            if not keep:
                os.unlink(self.path)
        except OSError:
            pass
        inside = [p for ts, p in rows if t0 - 0.15 <= ts <= t1 + 0.15]
        use = inside if inside else [p for _, p in rows]
        if not use:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm = [float(p[2]) for p in use if p[2].replace(".", "").isdigit()]
        mx = [float(p[3]) for p in use if p[3].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for p in use for i in range(4) if p[6 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(inside), "power_w_max": max(
                    (float(p[4]) for p in use if p[4].replace(".", "").isdigit()), default=None)}


# ---------------------------------------------------------------------------
# roofline helpers
# ---------------------------------------------------------------------------

def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "source": "fallback"}


def kernel_source_hash(kernel: str) -> str:
    """Hash of the source of one kernel family (its header and the headers it
    includes, comments and blank space removed), so that a profile summary
    stays attached to the code it measured.  `kernel` is a name as the
    kernel-name queries report it, e.g. "halo_fwd_tc2<16,14>",
    "halo_bwd_tc<16,14>" or "halo_fused_tc<16,14,128>"."""
    import re
    m = re.match(r"halo_(fwd_|bwd_|)(\w+?)<", kernel or "")
    if not m:
        return ""
    kind, fam = m.groups()
    if kind == "fwd_":
        first = "halo_%s.cuh" % fam                                   # halo_fwd_tc4 -> halo_tc4.cuh
    elif kind == "bwd_":
        first = "halo_bwd_tc.cuh" if fam == "tc" else "halo_bwd.cuh"  # tensor-core / CUDA-core backward
    else:
        first = "halo_%s.cuh" % fam.split("_")[0]                     # halo_fused_tc -> halo_fused.cuh
    csrc = os.path.join(ROOT, "blocked_local_self_b200", "csrc")
    seen, todo = set(), [first]
    while todo:
        name = todo.pop()
        if name in seen or not os.path.exists(os.path.join(csrc, name)):
            continue
        seen.add(name)
        with open(os.path.join(csrc, name)) as f:
            todo += re.findall(r'^#include "([^"/]+)"', f.read(), flags=re.M)
    h = hashlib.sha256()
    for name in sorted(seen):
        with open(os.path.join(csrc, name)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(workload: str, kernel: str):
    """DRAM bytes per launch (dram__bytes_read.sum + dram__bytes_write.sum)
    from a committed ncu summary under profiles/ that names this workload,
    only while the kernel's sources still hash to the value it records."""
    import glob
    import re
    for path in sorted(glob.glob(os.path.join(PROFILES, "*.md"))):
        with open(path) as f:
            text = f.read()
        fields = dict(re.findall(r"^- (\w+): `?([^`\n]+?)`?\s*$", text, flags=re.M))
        if fields.get("workload") != workload or "dram_bytes_per_launch" not in fields:
            continue
        family = (kernel or "").split("<")[0]
        if "kernel" in fields and family and family + "<" not in fields["kernel"]:
            continue  # a summary of another kernel on the same workload (e.g. the backward)
        if fields.get("kernel_source_sha") != kernel_source_hash(kernel):
            return None
        return float(fields["dram_bytes_per_launch"])
    return None


# ---------------------------------------------------------------------------
# CPU oracle baseline
# ---------------------------------------------------------------------------

def cpu_baseline(wl, inputs_cpu) -> dict:
    """The oracle on the host cores over a bounded sample of the workload:
    the first n images (n sized so one pass takes about two seconds),
    repeated until about ten seconds have passed."""
    import oracle
    kw = dict(block=wl.block, halo=wl.halo, stride=wl.stride)
    img_px = wl.out_hw[0] * wl.out_hw[1]
    t0 = time.perf_counter()
    oracle.halo_attention(*[t[:1] if t.dim() == 4 else t for t in inputs_cpu], **kw)
    t1 = time.perf_counter() - t0
    n = max(1, min(wl.N, int(2.0 / max(t1, 1e-3))))
    sample = [t[:n].contiguous() if t.dim() == 4 else t for t in inputs_cpu]
    t0 = time.perf_counter()
    reps = 0
    while True:
        oracle.halo_attention(*sample, **kw)
        reps += 1
        el = time.perf_counter() - t0
        if el >= 10.0:
            break
    return {"value": reps * n * img_px / el, "unit": "pixels/s", "cores": oracle.max_threads(),
            "kind": "oracle",
            "sample": f"{n} of the {wl.N} images of {wl.name} ({n * img_px} output pixels) x {reps}, "
                      f"{el:.1f} s wall"}


def oracle_rate(wl, inputs_cpu) -> dict:
    """The oracle's output pixels/s on this workload's first image (all host
    cores; the tiny workload also on one thread), for the per-config table."""
    import oracle
    kw = dict(block=wl.block, halo=wl.halo, stride=wl.stride)
    one = [t[:1].contiguous() if t.dim() == 4 else t for t in inputs_cpu]
    img_px = wl.out_hw[0] * wl.out_hw[1]
    t0 = time.perf_counter()
    oracle.halo_attention(*one, **kw)
    el = time.perf_counter() - t0
    res = {"oracle_pixels_per_s": img_px / el, "oracle_cores": oracle.max_threads()}
    if wl.N * wl.H * wl.W <= 4096:
        t0 = time.perf_counter()
        oracle.halo_attention(*one, threads=1, **kw)
        res["oracle_pixels_per_s_1thread"] = img_px / (time.perf_counter() - t0)
    return res


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    wl = {**workloads.WORKLOADS, **workloads.NEXT_WORKLOADS}[args.workload]
    inputs = workloads.make_inputs(wl)
    # each step: one image of the workload (a bounded sample of the batch)
    n_img = 1
    sl = [t[:n_img].contiguous() if t.dim() == 4 else t for t in inputs]
    px = n_img * wl.out_hw[0] * wl.out_hw[1]
    for _ in range(args.warmup):
        oracle.halo_attention(*sl, block=wl.block, halo=wl.halo, stride=wl.stride)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.halo_attention(*sl, block=wl.block, halo=wl.halo, stride=wl.stride)
    el = time.perf_counter() - t0
    value = args.steps * px / el
    sample = f"one image ({px} output pixels) of {wl.name} per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "pixels/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, **wl.describe(), "sample_per_step": sample},
        "cpu_baseline": {"value": value, "unit": "pixels/s", "cores": oracle.max_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "pixels/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# main (CUDA path)
# ---------------------------------------------------------------------------

def make_device_sets(wl, inputs_cpu, n_sets=None):
    """Input sets on the device, enough of them that the step's inputs are not
    L2-resident when it runs (each set holds q, k, v of the whole batch);
    `n_sets` = 1 gives the warm-L2 case (the same inputs every step)."""
    in_bytes = sum(t.numel() * t.element_size() for t in inputs_cpu[:3])
    if n_sets is None:
        n_sets = max(2, -(-3 * L2_BYTES // in_bytes))
    sets = []
    for i in range(n_sets):
        if i == 0:
            sets.append([t.cuda() for t in inputs_cpu])
        else:
            sets.append([(t.cuda() * 1.0).roll(i, dims=0) if t.dim() == 4 else t.cuda() for t in inputs_cpu])
    return sets, in_bytes


class DeviceBench:
    """Times `halo_attn` on one workload: CUDA graphs of the per-step launches
    (inputs rotating over sets larger than L2) replayed on one stream, CUDA
    events on that stream."""

    def __init__(self, halo, wl, inputs_cpu, stream, use_graph=True, n_sets=None):
        self.halo, self.wl, self.stream, self.use_graph = halo, wl, stream, use_graph
        self.sets, self.in_bytes = make_device_sets(wl, inputs_cpu, n_sets)
        self.n_sets = len(self.sets)
        OH, OW = wl.out_hw
        self.outs = [torch.empty((wl.N, OH, OW, wl.C), dtype=wl.torch_dtype, device="cuda")
                     for _ in range(self.n_sets)]
        self.kernel = halo.kernel_name(wl.N, wl.H, wl.W, wl.heads, wl.dim_head, wl.block, wl.halo, wl.stride,
                                       wl.torch_dtype)
        self.graphs = []

    def step(self, i):
        wl, s = self.wl, self.sets[i % self.n_sets]
        self.halo.attn(*s, block=wl.block, halo=wl.halo, stride=wl.stride, out=self.outs[i % self.n_sets],
                       stream=self.stream)

    def warmup(self, n):
        with torch.cuda.stream(self.stream):
            for i in range(n):
                self.step(i)
        torch.cuda.synchronize()

    def prepare(self, steps):
        """Capture the timed steps: a graph of `per` steps replayed steps // per
        times, then one graph of the remaining steps."""
        self.steps = steps
        self.graphs = []
        if not self.use_graph:
            return
        per = self.n_sets * max(1, -(-64 // self.n_sets))
        plan = [(per, steps // per), (steps % per, 1)]
        start = 0
        for n, reps in plan:
            if n == 0 or reps == 0:
                continue
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=self.stream):
                for i in range(n):
                    self.step(start + i)
            self.graphs.append((g, reps))
            start += n
        with torch.cuda.stream(self.stream):
            for g, _ in self.graphs:
                g.replay()
        torch.cuda.synchronize()

    def region(self):
        """One timed region of exactly `steps` steps; returns milliseconds."""
        ev0 = torch.cuda.Event(enable_timing=True)
        ev1 = torch.cuda.Event(enable_timing=True)
        ev0.record(self.stream)
        with torch.cuda.stream(self.stream):
            if self.graphs:
                for g, reps in self.graphs:
                    for _ in range(reps):
                        g.replay()
            else:
                for i in range(self.steps):
                    self.step(i)
        ev1.record(self.stream)
        ev1.synchronize()
        return ev0.elapsed_time(ev1)

    def release(self):
        self.graphs = []
        self.sets = []
        self.outs = []


def time_flushed_launches(halo, wl, inputs_cpu, stream, launches=200):
    """For a workload whose inputs fit in L2 many times over (the tiny float32
    case): each launch timed on its own with CUDA events, a 256 MiB buffer
    written between launches (outside the events) so that none starts with its
    inputs in L2 (the buffer is twice the L2 size).  Returns the median launch
    time in ms."""
    dev = [t.cuda() for t in inputs_cpu]
    OH, OW = wl.out_hw
    out = torch.empty((wl.N, OH, OW, wl.C), dtype=wl.torch_dtype, device="cuda")
    flush = torch.empty(2 * L2_BYTES, dtype=torch.uint8, device="cuda")
    times = []
    with torch.cuda.stream(stream):
        for i in range(launches + 5):
            flush.fill_(i & 0xff)
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            halo.attn(*dev, block=wl.block, halo=wl.halo, stride=wl.stride, out=out, stream=stream)
            e1.record(stream)
            e1.synchronize()
            if i >= 5:
                times.append(e0.elapsed_time(e1))
    return statistics.median(times)


def roofline_entry(wl, launch_s, peaks, traffic):
    """HBM and tensor fractions of one launch of `wl` taking `launch_s` seconds."""
    gbs = wl.bytes() / launch_s * 1e-9
    tflops = wl.flops() / launch_s * 1e-12
    return {"achieved_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"], "tflops": tflops,
            "tensor_frac": (tflops / peaks["bf16_tflops"]) if wl.dtype == "bf16" else None,
            "traffic": traffic, "algorithmic_bytes": wl.bytes(), "flops": wl.flops()}


def per_config(halo, stream, sampler, peaks, seconds=0.5):
    """Every workload, timed in this run: ms per launch, pixels/s, HBM and
    tensor fractions of the measured peaks, the kernel, ncu traffic when the
    committed summary matches the kernel's sources, and the clocks seen."""
    res = {}
    for name, wl in workloads.WORKLOADS.items():
        res[name] = time_forward(halo, wl, stream, peaks, seconds)
    return res


def time_forward(halo, wl, stream, peaks, seconds=0.5):
    """One workload's forward: ms per launch, pixels/s, roofline fractions,
    kernel, ncu traffic (when the committed summary matches the kernel's
    sources) and the host-time window for the clock summary."""
    inputs_cpu = workloads.make_inputs(wl)
    kernel = halo.kernel_name(wl.N, wl.H, wl.W, wl.heads, wl.dim_head, wl.block, wl.halo, wl.stride,
                              wl.torch_dtype)
    t0 = time.time()
    if wl.N * wl.H * wl.W * wl.C * wl.elem_bytes * 3 < L2_BYTES // 4:
        ms = time_flushed_launches(halo, wl, inputs_cpu, stream)
        how, steps, reps = "each launch alone after a 252 MiB (2x L2) flush; median of 200", 1, 200
    else:
        b = DeviceBench(halo, wl, inputs_cpu, stream)
        b.warmup(10)
        b.prepare(20)
        est = b.region() / 20
        steps = max(20, int(seconds * 1e3 / max(est, 1e-3)))
        b.prepare(steps)
        regions = [b.region() / steps for _ in range(3)]
        ms = statistics.median(regions)
        reps = 3
        how = (f"median of 3 regions of {steps} graph-replayed launches, inputs rotating over "
               f"{b.n_sets} sets ({b.n_sets * b.in_bytes / 2**20:.0f} MiB) > L2")
        b.release()
    # warm L2: the same inputs every step (those that fit the L2 stay resident)
    w = DeviceBench(halo, wl, inputs_cpu, stream, n_sets=1)
    w.warmup(5)
    w.prepare(20)
    wsteps = max(20, int(seconds * 1e3 / max(w.region() / 20, 1e-3)))
    w.prepare(wsteps)
    warm_ms = statistics.median([w.region() / wsteps for _ in range(3)])
    w.release()
    t1 = time.time()
    torch.cuda.synchronize()
    err = halo.get_last_error()
    if err != 0:
        raise RuntimeError(f"device error flag {err} after timing {wl.name}")
    entry = {"kernel": kernel, "ms": ms, "value": wl.out_pixels / (ms * 1e-3), "unit": "pixels/s",
             "timing": how, "warm_ms": warm_ms,
             "warm_timing": "same inputs every step (L2-resident where they fit), graph-replayed, median of 3",
             "clocks": (t0, t1)}  # summarised once the sampler has stopped
    entry.update(oracle_rate(wl, inputs_cpu))
    entry.update(roofline_entry(wl, ms * 1e-3, peaks, ncu_traffic(wl.name, kernel)))
    torch.cuda.empty_cache()
    return entry


# float32 FMA peak of the CUDA cores (148 SMs x 128 lanes x 2 FLOP x 1.965 GHz),
# for kernels that run on them (the backward).
FP32_CUDA_CORE_TFLOPS = 148 * 128 * 2 * 1.965e9 * 1e-12


def bwd_bytes(wl) -> float:
    """Unavoidable HBM traffic of the backward: q, k, v, out, dout read once,
    dq, dk, dv written once (the tables are negligible)."""
    e = wl.elem_bytes
    inp = wl.N * wl.H * wl.W * wl.C * e
    outp = wl.out_pixels * wl.C * e
    return float(3 * inp + 2 * outp + 3 * inp)


def bwd_flops(wl) -> float:
    """Algorithmic FLOPs of the backward: the five window products per output
    pixel and head (q.k again, dout.v, p dout, dz q, dz k), 2 d w^2 each."""
    w = wl.window
    return 10.0 * wl.dim_head * w * w * wl.heads * wl.out_pixels


def time_extra(halo, stream, sampler, peaks, seconds=0.5):
    """The NEXT rows measured in the same run: the backward on the stage-1 and
    stride-2 workloads, and the SASA-masked forward (7 x 7 centred window,
    the paper's comparison) and the fused-projection form on the stage-1
    workload, and the block-32 workloads.  Inputs rotate over sets larger than
    L2 as for the forward."""
    res = {}
    for name in ("stage1_bf16", "stride2_bf16"):
        wl = workloads.WORKLOADS[name]
        inputs_cpu = workloads.make_inputs(wl)
        sets, in_bytes = make_device_sets(wl, inputs_cpu)
        OH, OW = wl.out_hw
        outs = [halo.attn(*st, block=wl.block, halo=wl.halo, stride=wl.stride) for st in sets]
        g = torch.Generator().manual_seed(7)
        douts = [torch.randn((wl.N, OH, OW, wl.C), generator=g).to(wl.torch_dtype).cuda() for _ in sets]
        grads = [tuple(torch.empty_like(t) for t in st) for st in sets]
        nbytes = halo.bwd_workspace_size(wl.N, wl.H, wl.W, wl.heads, wl.dim_head, wl.block, wl.halo, wl.stride, 0,
                                         wl.torch_dtype)
        ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")

        def step(i):
            j = i % len(sets)
            halo.attn_bwd(*sets[j], outs[j], douts[j], block=wl.block, halo=wl.halo, stride=wl.stride,
                          grads=grads[j], workspace=ws, stream=stream)

        with torch.cuda.stream(stream):
            for i in range(3):
                step(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        with torch.cuda.stream(stream):
            step(0)
        e1.record(stream)
        e1.synchronize()
        est = e0.elapsed_time(e1)
        steps = max(3, int(seconds * 1e3 / max(est, 1e-3)))
        t0 = time.time()
        e0.record(stream)
        with torch.cuda.stream(stream):
            for i in range(steps):
                step(i)
        e1.record(stream)
        e1.synchronize()
        t1 = time.time()
        ms = e0.elapsed_time(e1) / steps
        launch_s = ms * 1e-3
        gbs = bwd_bytes(wl) / launch_s * 1e-9
        tf = bwd_flops(wl) / launch_s * 1e-12
        kname = halo.bwd_kernel_name(wl.N, wl.H, wl.W, wl.heads, wl.dim_head, wl.block, wl.halo, wl.stride, 0,
                                     wl.torch_dtype)
        res["bwd_" + name] = {
            "what": "halo_attn_bwd: dq, dk, dv, drel_h, drel_w (workspace zeroing, the kernel, finalize)",
            "kernel": kname, "ms": ms, "value": wl.out_pixels / launch_s, "unit": "pixels/s",
            "timing": f"{steps} back-to-back calls, inputs rotating over {len(sets)} sets > L2",
            "achieved_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes": bwd_bytes(wl),
            "tflops": tf, "flops": bwd_flops(wl),
            "compute_frac": tf / (peaks["bf16_tflops"] if "_tc<" in kname else FP32_CUDA_CORE_TFLOPS),
            "compute_peak": "bf16 tensor (measured)" if "_tc<" in kname else "float32 CUDA cores (nominal)",
            "clocks": (t0, t1)}
        del sets, outs, douts, grads, ws
        torch.cuda.empty_cache()
        halo_err = halo.get_last_error()
        if halo_err != 0:
            raise RuntimeError(f"device error flag {halo_err} after the backward of {name}")
    # SASA-masked forward, 7 x 7 centred window on the stage-1 layer
    wl = workloads.WORKLOADS["stage1_bf16"]
    inputs_cpu = workloads.make_inputs(wl)
    b = DeviceBench(halo, wl, inputs_cpu, stream)
    kern = 7

    def sstep(i):
        st = b.sets[i % b.n_sets]
        halo.attn_masked(*st, block=wl.block, halo=wl.halo, kernel=kern, stride=wl.stride,
                         out=b.outs[i % b.n_sets], stream=stream)

    b.step = sstep
    b.warmup(10)
    b.prepare(20)
    est = b.region() / 20
    steps = max(20, int(seconds * 1e3 / max(est, 1e-3)))
    b.prepare(steps)
    t0 = time.time()
    ms = statistics.median([b.region() / steps for _ in range(3)])
    t1 = time.time()
    kname = halo.masked_kernel_name(wl.N, wl.H, wl.W, wl.heads, wl.dim_head, wl.block, wl.halo, wl.stride, kern,
                                    wl.torch_dtype)
    entry = {"what": "halo_attn_masked, kernel 7 (SASA's 7 x 7 centred window) on the stage-1 layer",
             "kernel": kname, "ms": ms, "value": wl.out_pixels / (ms * 1e-3), "unit": "pixels/s",
             "timing": f"median of 3 regions of {steps} graph-replayed launches", "clocks": (t0, t1)}
    entry.update(roofline_entry(wl, ms * 1e-3, peaks, None))
    res["sasa_k7_stage1_bf16"] = entry
    b.release()
    torch.cuda.empty_cache()
    res.update(time_fused(halo, stream, peaks, seconds))
    # block 32: global attention on a 32x32 map, and block 32 with halo 3
    for name, wl in workloads.NEXT_WORKLOADS.items():
        res[name] = time_forward(halo, wl, stream, peaks, seconds)
    return res


def fused_bytes(wl, c_in) -> float:
    """Unavoidable HBM traffic of the fused form: x read once, out written
    once (the weights and tables are a few KB)."""
    return float(wl.N * wl.H * wl.W * c_in * wl.elem_bytes + wl.out_pixels * wl.C * wl.elem_bytes)


def fused_flops(wl, c_in) -> float:
    """Algorithmic FLOPs of the fused form: the three projections (2 c_in
    FLOPs per output channel of q, k and v at every pixel) plus the
    operation's q.k and p.v."""
    return 2.0 * c_in * 3 * wl.C * wl.N * wl.H * wl.W + wl.flops()


def time_fused(halo, stream, peaks, seconds=0.5):
    """The fused-projection form on the stage-1 layer (c_in = 128), and, for
    context, the same result computed unfused: three cuBLAS projections into
    bf16 q, k, v, then ``halo_attn``.  Graph-replayed, inputs rotating over
    sets larger than L2."""
    res = {}
    for name, (wl, c_in) in workloads.FUSED_WORKLOADS.items():
        inputs_cpu = workloads.make_fused_inputs(wl, c_in)
        b = DeviceBench(halo, wl, inputs_cpu, stream)

        def fstep(i, b=b, wl=wl):
            x, wq, wkv, rh, rw = b.sets[i % b.n_sets]
            halo.attn_fused(x, wq, wkv, rh, rw, heads=wl.heads, block=wl.block, halo=wl.halo,
                            out=b.outs[i % b.n_sets], stream=stream)

        b.step = fstep
        b.warmup(10)
        b.prepare(20)
        est = b.region() / 20
        steps = max(20, int(seconds * 1e3 / max(est, 1e-3)))
        b.prepare(steps)
        t0 = time.time()
        ms = statistics.median([b.region() / steps for _ in range(3)])
        t1 = time.time()
        # unfused, for context: q, k, v projected by cuBLAS, then halo_attn
        shape = (wl.N, wl.H, wl.W, wl.C)
        q, k, v = (torch.empty(shape, dtype=wl.torch_dtype, device="cuda") for _ in range(3))

        def ustep(i, b=b, wl=wl):
            x, wq, wkv, rh, rw = b.sets[i % b.n_sets]
            torch.matmul(x, wq.t(), out=q)
            torch.matmul(x, wkv[:wl.C].t(), out=k)
            torch.matmul(x, wkv[wl.C:].t(), out=v)
            halo.attn(q, k, v, rh, rw, block=wl.block, halo=wl.halo, out=b.outs[i % b.n_sets], stream=stream)

        b.step = ustep
        b.warmup(5)
        b.prepare(steps)
        ums = statistics.median([b.region() / steps for _ in range(3)])
        torch.cuda.synchronize()
        err = halo.get_last_error()
        if err != 0:
            raise RuntimeError(f"device error flag {err} after timing {name}")
        launch_s = ms * 1e-3
        gbs = fused_bytes(wl, c_in) / launch_s * 1e-9
        tf = fused_flops(wl, c_in) / launch_s * 1e-12
        kname = halo.fused_kernel_name(wl.N, wl.H, wl.W, c_in, wl.heads, wl.dim_head, wl.block, wl.halo,
                                       wl.stride, wl.torch_dtype)
        res["fused_" + wl.name] = {
            "what": f"halo_attn_fused: q, k, v projected from x (c_in {c_in}) inside the kernel, then the "
                    "operation, on the stage-1 layer",
            "kernel": kname, "ms": ms, "value": wl.out_pixels / launch_s, "unit": "pixels/s",
            "timing": f"median of 3 regions of {steps} graph-replayed launches, inputs rotating over "
                      f"{b.n_sets} sets > L2",
            "achieved_gbs": gbs, "hbm_frac": gbs / peaks["hbm_gbs"], "algorithmic_bytes": fused_bytes(wl, c_in),
            "tflops": tf, "tensor_frac": tf / peaks["bf16_tflops"], "flops": fused_flops(wl, c_in),
            "unfused_ms": ums,
            "unfused": "three cuBLAS projections (torch.matmul into bf16 q, k, v) + halo_attn, graph-replayed",
            "clocks": (t0, t1)}
        b.release()
        del q, k, v
        torch.cuda.empty_cache()
    return res


def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dist_init(world)
    import blocked_local_self_b200 as halo
    halo.load()

    wl = {**workloads.WORKLOADS, **workloads.NEXT_WORKLOADS}[args.workload]
    c_in = 0
    if args.which == "fused":
        forms = [ci for (fw, ci) in workloads.FUSED_WORKLOADS.values() if fw.name == wl.name]
        if not forms:
            raise SystemExit(f"--pass fused: {wl.name} has no fused form (see workloads.FUSED_WORKLOADS)")
        c_in = forms[0]
        inputs_cpu = workloads.make_fused_inputs(wl, c_in, seed=rank_seed(wl, rank))
    else:
        inputs_cpu = workloads.make_inputs(wl, seed=rank_seed(wl, rank))
    use_graph = not args.no_graph and args.which != "bwd"
    stream = torch.cuda.Stream() if use_graph else torch.cuda.current_stream()
    bench = DeviceBench(halo, wl, inputs_cpu, stream, use_graph=use_graph)
    kernel = bench.kernel
    if args.which == "masked":
        kmask = 2 * wl.halo + 1

        def masked_step(i, b=bench):
            st = b.sets[i % b.n_sets]
            halo.attn_masked(*st, block=wl.block, halo=wl.halo, kernel=kmask, stride=wl.stride,
                             out=b.outs[i % b.n_sets], stream=stream)

        bench.step = masked_step
        kernel = halo.masked_kernel_name(wl.N, wl.H, wl.W, wl.heads, wl.dim_head, wl.block, wl.halo, wl.stride,
                                         kmask, wl.torch_dtype)
    elif args.which == "fused":
        def fused_step(i, b=bench):
            x, wq, wkv, rh, rw = b.sets[i % b.n_sets]
            halo.attn_fused(x, wq, wkv, rh, rw, heads=wl.heads, block=wl.block, halo=wl.halo,
                            out=b.outs[i % b.n_sets], stream=stream)

        bench.step = fused_step
        kernel = halo.fused_kernel_name(wl.N, wl.H, wl.W, c_in, wl.heads, wl.dim_head, wl.block, wl.halo,
                                        wl.stride, wl.torch_dtype)
    elif args.which == "bwd":
        with torch.cuda.stream(stream):
            fwd_outs = [halo.attn(*st, block=wl.block, halo=wl.halo, stride=wl.stride) for st in bench.sets]
        g = torch.Generator().manual_seed(7)
        douts = [torch.randn(o.shape, generator=g).to(o.dtype).cuda() for o in fwd_outs]
        grads = [tuple(torch.empty_like(t) for t in st) for st in bench.sets]
        ws = torch.empty(halo.bwd_workspace_size(wl.N, wl.H, wl.W, wl.heads, wl.dim_head, wl.block, wl.halo,
                                                 wl.stride, 0, wl.torch_dtype), dtype=torch.uint8, device="cuda")

        def bwd_step(i, b=bench):
            j = i % b.n_sets
            halo.attn_bwd(*b.sets[j], fwd_outs[j], douts[j], block=wl.block, halo=wl.halo, stride=wl.stride,
                          grads=grads[j], workspace=ws, stream=stream)

        bench.step = bwd_step
        kernel = halo.bwd_kernel_name(wl.N, wl.H, wl.W, wl.heads, wl.dim_head, wl.block, wl.halo, wl.stride, 0,
                                      wl.torch_dtype)
    bench.warmup(args.warmup)
    # The timed steps replay CUDA graphs of the same launches (one kernel per
    # step, inputs rotating as above), so that the host's per-call cost
    # (tensor-map encoding, argument checks) does not pace the GPU.
    bench.prepare(args.steps)
    # A short run (few steps) is timed as several regions of exactly K steps
    # each, bracketed like the first, and the median region is reported.
    est = bench.region()
    repeats = max(1, min(100, int(math.ceil(args.min_timed_s * 1e3 / max(est, 1e-3)))))
    sampler = ClockSampler(local)
    sampler.start()
    regions = []
    t_host0 = time.time()
    for _ in range(repeats):
        barrier(world)
        torch.cuda.synchronize()
        r = bench.region()
        torch.cuda.synchronize()
        barrier(world)
        regions.append(r)
    t_host1 = time.time()
    ms_local = statistics.median(regions)
    ms = max_over_ranks(ms_local, world)
    err = halo.get_last_error()
    if err != 0:
        raise RuntimeError(f"device error flag {err} after the timed region")
    peaks = measured_peaks()
    configs = None
    if rank == 0 and world == 1 and not args.no_per_config:
        bench.release()
        torch.cuda.empty_cache()
        configs = per_config(halo, stream, sampler, peaks)
    extra = None
    if rank == 0 and world == 1 and not args.no_extra:
        extra = time_extra(halo, stream, sampler, peaks)
    # nvidia-smi buffers its file output: read the samples once it has stopped
    sampler.stop()
    clocks = sampler.summary(t_host0, t_host1, keep=True)
    for entry in list((configs or {}).values()) + list((extra or {}).values()):
        entry["clocks"] = sampler.summary(*entry["clocks"], keep=True)
    sampler.cleanup()

    # end to end through the host entry point: H2D inputs, kernel, D2H output
    OH, OW = wl.out_hw
    h2d = sum(t.numel() * t.element_size() for t in inputs_cpu)
    d2h = wl.out_pixels * wl.C * wl.elem_bytes
    e2e = None
    if args.e2e_steps > 0 and args.which == "fwd":
        pinned = [t.pin_memory() for t in inputs_cpu]
        out_h = torch.empty((wl.N, OH, OW, wl.C), dtype=wl.torch_dtype).pin_memory()
        staging = dict(zip(("q", "k", "v", "rel_h", "rel_w"), [torch.empty_like(t, device="cuda")
                                                              for t in inputs_cpu]))
        staging["out"] = torch.empty((wl.N, OH, OW, wl.C), dtype=wl.torch_dtype, device="cuda")
        for _ in range(2):
            halo.attn_host(*pinned, out_h, staging, block=wl.block, halo=wl.halo, stride=wl.stride, stream=stream)
        torch.cuda.synchronize()
        barrier(world)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.e2e_steps):
            halo.attn_host(*pinned, out_h, staging, block=wl.block, halo=wl.halo, stride=wl.stride,
                           stream=stream)
        e1.record(stream)
        e1.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
        e2e = {"value": wl.out_pixels * world / (e2e_ms * 1e-3 / args.e2e_steps), "unit": "pixels/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": args.e2e_steps}

    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.which != "fused":
        base = cpu_baseline(wl, inputs_cpu)
    barrier(world)
    dist_done(world)
    if rank != 0:
        return 0

    per_step_s = ms * 1e-3 / args.steps
    pixels = wl.out_pixels * world
    value = pixels / per_step_s
    step_flops = {"bwd": bwd_flops(wl), "fused": fused_flops(wl, c_in)}.get(args.which, wl.flops())
    step_bytes = {"bwd": bwd_bytes(wl), "fused": fused_bytes(wl, c_in)}.get(args.which, wl.bytes())
    tflops = step_flops * world / per_step_s * 1e-12
    launch_s = ms_local * 1e-3 / args.steps  # one step per launch sequence on this stream
    achieved_gbs = step_bytes / launch_s * 1e-9
    traffic = ncu_traffic(wl.name, kernel)
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "pixels/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "repeats": repeats,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if wl.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": {"workload": f"{wl.name}: N={wl.N} per GPU, {wl.H}x{wl.W}, heads={wl.heads}, "
                               f"dim_head={wl.dim_head}, block={wl.block}, halo={wl.halo}, stride={wl.stride}",
                   "global_batch": wl.N * world, "parallelism": f"replicas x{world} (batch sharding)",
                   "l2": f"inputs rotate over {bench.n_sets} sets ({bench.n_sets * bench.in_bytes / 2**20:.0f} MiB) > L2",
                   "launch": ("one call per step from Python" if not use_graph else
                              "CUDA graphs of the per-step launches, replayed"),
                   "timing": f"median of {repeats} timed regions of exactly {args.steps} steps each, "
                             "each bracketed by a barrier and a device synchronisation",
                   "pass": args.which,
                   "kernel": kernel},
        "tflops": tflops,
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved_gbs / peaks["hbm_gbs"], "traffic": traffic,
                     "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json hbm_gbs)" if peaks["source"] ==
                     "measured" else "fallback 6.65 TB/s",
                     "algorithmic_bytes_per_launch": step_bytes,
                     "tensor_frac": tflops / world / peaks["bf16_tflops"]},
        "e2e": e2e,
        # one kernel per forward step; the backward launches its kernel and the finalize kernel
        "gpu_launches": args.steps * repeats * (2 if args.which == "bwd" else 1),
        "clocks": clocks,
        "cpu_baseline": base,
        "per_config": configs,
        "next_rows": extra,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
