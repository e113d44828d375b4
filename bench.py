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
    ap.add_argument("--workload", default=workloads.BENCH_WORKLOAD, choices=sorted(workloads.WORKLOADS))
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="launch every step from Python instead of replaying captured CUDA graphs")
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

    def summary(self, t0: float, t1: float) -> dict:
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
    stays attached to the code it measured.  `kernel` is a name as
    halo_kernel_name reports it, e.g. "halo_fwd_tc2<16,14>"."""
    import re
    m = re.match(r"halo_fwd_(\w+?)<", kernel or "")
    if not m:
        return ""
    csrc = os.path.join(ROOT, "blocked_local_self_b200", "csrc")
    seen, todo = set(), ["halo_%s.cuh" % m.group(1)]
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


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    import oracle
    wl = workloads.WORKLOADS[args.workload]
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

def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)
    rank, world, local = dist_env()
    torch.cuda.set_device(local)
    dist_init(world)
    import blocked_local_self_b200 as halo
    halo.load()

    wl = workloads.WORKLOADS[args.workload]
    inputs_cpu = workloads.make_inputs(wl, seed=rank_seed(wl, rank))
    in_bytes = sum(t.numel() * t.element_size() for t in inputs_cpu[:3])
    # rotate among enough input sets that the step's inputs are not L2-resident
    n_sets = max(2, -(-3 * L2_BYTES // in_bytes))
    sets = []
    for i in range(n_sets):
        if i == 0:
            sets.append([t.cuda() for t in inputs_cpu])
        else:
            sets.append([(t.cuda() * 1.0).roll(i, dims=0) if t.dim() == 4 else t.cuda() for t in inputs_cpu])
    OH, OW = wl.out_hw
    outs = [torch.empty((wl.N, OH, OW, wl.C), dtype=wl.torch_dtype, device="cuda") for _ in range(n_sets)]
    stream = torch.cuda.Stream() if not args.no_graph else torch.cuda.current_stream()

    def step(i):
        s = sets[i % n_sets]
        halo.attn(*s, block=wl.block, halo=wl.halo, stride=wl.stride, out=outs[i % n_sets], stream=stream)

    kernel = halo.kernel_name(wl.N, wl.H, wl.W, wl.heads, wl.dim_head, wl.block, wl.halo, wl.stride,
                              wl.torch_dtype)
    with torch.cuda.stream(stream):
        for i in range(args.warmup):
            step(i)
    torch.cuda.synchronize()
    # The timed steps replay CUDA graphs of the same launches (one kernel per
    # step, inputs rotating as above), so that the host's per-call cost
    # (tensor-map encoding, argument checks) does not pace the GPU: a graph of
    # `per` steps replayed steps // per times, then one of the remaining steps.
    graphs = []
    if not args.no_graph:
        per = n_sets * max(1, -(-64 // n_sets))
        plan = [(per, args.steps // per), (args.steps % per, 1)]
        start = 0
        for n, reps in plan:
            if n == 0 or reps == 0:
                continue
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=stream):
                for i in range(n):
                    step(start + i)
            graphs.append((g, reps))
            start += n
        with torch.cuda.stream(stream):
            for g, _ in graphs:
                g.replay()
        torch.cuda.synchronize()
    barrier(world)
    sampler = ClockSampler(local)
    sampler.start()
    torch.cuda.synchronize()
    barrier(world)
    ev0 = torch.cuda.Event(enable_timing=True)
    ev1 = torch.cuda.Event(enable_timing=True)
    t_host0 = time.time()
    ev0.record(stream)
    with torch.cuda.stream(stream):
        if graphs:
            for g, reps in graphs:
                for _ in range(reps):
                    g.replay()
        else:
            for i in range(args.steps):
                step(i)
    ev1.record(stream)
    ev1.synchronize()
    torch.cuda.synchronize()
    t_host1 = time.time()
    barrier(world)
    sampler.stop()
    ms_local = ev0.elapsed_time(ev1)
    ms = max_over_ranks(ms_local, world)
    err = halo.get_last_error()
    if err != 0:
        raise RuntimeError(f"device error flag {err} after the timed region")
    clocks = sampler.summary(t_host0, t_host1)

    # end to end through the host entry point: H2D inputs, kernel, D2H output
    h2d = sum(t.numel() * t.element_size() for t in inputs_cpu)
    d2h = wl.out_pixels * wl.C * wl.elem_bytes
    e2e = None
    if args.e2e_steps > 0:
        pinned = [t.pin_memory() for t in inputs_cpu]
        out_h = torch.empty((wl.N, OH, OW, wl.C), dtype=wl.torch_dtype).pin_memory()
        staging = dict(zip(("q", "k", "v", "rel_h", "rel_w"), sets[0]))
        staging["out"] = outs[0]
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
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(wl, inputs_cpu)
    barrier(world)
    dist_done(world)
    if rank != 0:
        return 0

    per_step_s = ms * 1e-3 / args.steps
    pixels = wl.out_pixels * world
    value = pixels / per_step_s
    tflops = wl.flops() * world / per_step_s * 1e-12
    peaks = measured_peaks()
    launch_s = ms_local * 1e-3 / args.steps  # one launch per step on this stream
    achieved_gbs = wl.bytes() / launch_s * 1e-9
    traffic = ncu_traffic(wl.name, kernel)
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "pixels/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms / args.steps,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if wl.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": {"workload": f"{wl.name}: N={wl.N} per GPU, {wl.H}x{wl.W}, heads={wl.heads}, "
                               f"dim_head={wl.dim_head}, block={wl.block}, halo={wl.halo}, stride={wl.stride}",
                   "global_batch": wl.N * world, "parallelism": f"replicas x{world} (batch sharding)",
                   "l2": f"inputs rotate over {n_sets} sets ({n_sets * in_bytes / 2**20:.0f} MiB) > L2",
                   "launch": ("one launch per step from Python" if args.no_graph else
                              "CUDA graphs of the per-step launches, replayed"),
                   "kernel": kernel},
        "tflops": tflops,
        "roofline": {"bound": "hbm", "achieved": achieved_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved_gbs / peaks["hbm_gbs"], "traffic": traffic,
                     "peak_source": f"{peaks['source']} (MEASURED_PEAKS.json hbm_gbs)" if peaks["source"] ==
                     "measured" else "fallback 6.65 TB/s",
                     "algorithmic_bytes_per_launch": wl.bytes(),
                     "tensor_frac": tflops / world / peaks["bf16_tflops"]},
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clocks,
        "cpu_baseline": base,
    }
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
