"""Seeded synthetic workloads for blocked local self-attention with haloing.

This module only *describes* workloads and *draws* their inputs.  It holds none
of the method's arithmetic, so both the CPU oracle tests and the CUDA path may
use it without sharing any computation.

Input recipe (HaloNet, "Scaling Local Self-Attention for Parameter Efficient
Visual Backbones", section 2.2 and the blog page's ``RelPosEmb`` module):
  * one CPU ``torch.Generator`` seeded with ``seed`` (0 by default);
  * ``randn`` in float32 drawn in the fixed order q, k, v, rel_h, rel_w;
  * the relative tables are multiplied by ``dim_head ** -0.5`` (the blog's
    ``RelPosEmb.__init__`` initialisation), then everything is cast to the
    workload dtype (round-to-nearest-even for bf16);
  * q, k, v are NHWC ``[N, H, W, heads * dim_head]`` (channel = head * d + e),
    rel_h and rel_w are ``[2 * (block + 2 * halo) - 1, dim_head]``.

The five named workloads mirror the shapes HaloNet uses: a stage-1 layer
(b=8, h=3, 14x14 window, d=16), a deeper stage (32x32 map, d=64), the
strided attention-downsampling layer (stride 2), and a large-resolution
layer (b=16, h=4, 24x24 window).  The paper's own numbers are TPU training
step times with the values lost, so these seeded tensors are the workload.
"""
from __future__ import annotations

from dataclasses import dataclass, asdict

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    N: int
    H: int
    W: int
    heads: int
    dim_head: int
    block: int
    halo: int
    stride: int
    dtype: str  # "f32" or "bf16"
    seed: int = 0

    @property
    def C(self) -> int:
        return self.heads * self.dim_head

    @property
    def window(self) -> int:
        return self.block + 2 * self.halo

    @property
    def rel_rows(self) -> int:
        return 2 * self.window - 1

    @property
    def out_hw(self) -> tuple[int, int]:
        return self.H // self.stride, self.W // self.stride

    @property
    def out_pixels(self) -> int:
        oh, ow = self.out_hw
        return self.N * oh * ow

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    @property
    def torch_dtype(self) -> torch.dtype:
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def flops(self) -> float:
        """Algorithmic FLOPs: q.k and p.v over the full w x w window, per
        output pixel and head (2 FLOPs per multiply-add)."""
        w = self.window
        return 4.0 * self.dim_head * w * w * self.heads * self.out_pixels

    def rel_flops(self) -> float:
        """FLOPs of the two factorised relative dot products (rows and
        columns of the window), reported separately from ``flops``."""
        w = self.window
        return 4.0 * self.dim_head * w * self.heads * self.out_pixels

    def bytes(self) -> float:
        """Unavoidable HBM traffic: q (only the strided pixels at stride 2),
        k and v read once, out written once.  Halo re-reads and the tiny
        relative tables are not counted."""
        e = self.elem_bytes
        q = self.out_pixels * self.C * e
        kv = 2 * self.N * self.H * self.W * self.C * e
        out = self.out_pixels * self.C * e
        return float(q + kv + out)

    def valid_key_fraction(self) -> float:
        """Fraction of window keys that fall inside the image."""
        b, h, w = self.block, self.halo, self.window
        tot = 0
        val = 0
        for by in range(self.H // b):
            ry = sum(1 for kr in range(w) if 0 <= by * b - h + kr < self.H)
            for bx in range(self.W // b):
                rx = sum(1 for kc in range(w) if 0 <= bx * b - h + kc < self.W)
                tot += w * w
                val += ry * rx
        return val / tot

    def describe(self) -> dict:
        d = asdict(self)
        d["window"] = self.window
        d["C"] = self.C
        return d


WORKLOADS: dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("tiny_f32", N=1, H=16, W=16, heads=2, dim_head=32, block=4, halo=1, stride=1, dtype="f32"),
        Workload("stage1_bf16", N=32, H=64, W=64, heads=8, dim_head=16, block=8, halo=3, stride=1, dtype="bf16"),
        Workload("deep_bf16", N=64, H=32, W=32, heads=8, dim_head=64, block=8, halo=3, stride=1, dtype="bf16"),
        Workload("stride2_bf16", N=64, H=64, W=64, heads=8, dim_head=32, block=8, halo=3, stride=2, dtype="bf16"),
        Workload("large_bf16", N=16, H=128, W=128, heads=8, dim_head=32, block=16, halo=4, stride=1, dtype="bf16"),
    ]
}

# The workload the throughput benchmark times (the stage-1 layer).
BENCH_WORKLOAD = "stage1_bf16"

# Shapes measured beside the five above: global attention at the smallest
# resolution (block = the whole 32x32 map, halo 0; section 2.2 and the deep
# stages of section 4), the block-32, halo-3 setting of the detection
# backbones (section 4.5, Table 5), and the stage-1 layer in float32.
NEXT_WORKLOADS: dict[str, Workload] = {
    w.name: w
    for w in [
        Workload("global32_bf16", N=64, H=32, W=32, heads=8, dim_head=32, block=32, halo=0, stride=1, dtype="bf16"),
        Workload("block32_h3_bf16", N=4, H=128, W=128, heads=8, dim_head=32, block=32, halo=3, stride=1,
                 dtype="bf16"),
        # the stage-1 layer in float32 (the float32 path at a full-size shape)
        Workload("stage1_f32", N=32, H=64, W=64, heads=8, dim_head=16, block=8, halo=3, stride=1, dtype="f32"),
    ]
}


def make_inputs(wl: Workload, seed: int | None = None):
    """Draw (q, k, v, rel_h, rel_w) on the CPU for workload ``wl``.

    Returns contiguous CPU tensors in the workload dtype.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.seed if seed is None else seed)
    shape = (wl.N, wl.H, wl.W, wl.C)
    q = torch.randn(shape, generator=g, dtype=torch.float32)
    k = torch.randn(shape, generator=g, dtype=torch.float32)
    v = torch.randn(shape, generator=g, dtype=torch.float32)
    rel_h = torch.randn((wl.rel_rows, wl.dim_head), generator=g, dtype=torch.float32)
    rel_w = torch.randn((wl.rel_rows, wl.dim_head), generator=g, dtype=torch.float32)
    scale = wl.dim_head ** -0.5
    rel_h = rel_h * scale
    rel_w = rel_w * scale
    dt = wl.torch_dtype
    return tuple(t.to(dt).contiguous() for t in (q, k, v, rel_h, rel_w))


# The fused-projection form (the blog page's HaloAttention: to_q and to_kv are
# bias-free linear layers of the layer's input map x) on the stage-1 layer,
# with c_in = heads * dim_head = 128 input channels.
FUSED_WORKLOADS: dict[str, tuple[Workload, int]] = {
    "stage1_fused_bf16": (WORKLOADS["stage1_bf16"], 128),
}


def make_fused_inputs(wl: Workload, c_in: int, seed: int | None = None):
    """Draw (x, wq, wkv, rel_h, rel_w) on the CPU for the fused form.

    One CPU generator seeded with ``seed`` (default the workload's); ``randn``
    in float32 in the order x [N, H, W, c_in], wq [heads*d, c_in],
    wkv [2*heads*d, c_in] (key rows, then value rows), rel_h, rel_w; the
    weights are scaled by ``c_in ** -0.5`` (so q, k, v have unit variance),
    the tables by ``dim_head ** -0.5``; then everything is cast to the
    workload dtype."""
    g = torch.Generator(device="cpu")
    g.manual_seed(wl.seed if seed is None else seed)
    x = torch.randn((wl.N, wl.H, wl.W, c_in), generator=g, dtype=torch.float32)
    wq = torch.randn((wl.C, c_in), generator=g, dtype=torch.float32) * c_in ** -0.5
    wkv = torch.randn((2 * wl.C, c_in), generator=g, dtype=torch.float32) * c_in ** -0.5
    rel_h = torch.randn((wl.rel_rows, wl.dim_head), generator=g, dtype=torch.float32) * wl.dim_head ** -0.5
    rel_w = torch.randn((wl.rel_rows, wl.dim_head), generator=g, dtype=torch.float32) * wl.dim_head ** -0.5
    dt = wl.torch_dtype
    return tuple(t.to(dt).contiguous() for t in (x, wq, wkv, rel_h, rel_w))


def custom(name: str = "custom", **kw) -> Workload:
    """A workload with explicit sizes (used by the parity and edge-case tests)."""
    base = dict(N=1, H=16, W=16, heads=2, dim_head=16, block=4, halo=1, stride=1, dtype="bf16")
    base.update(kw)
    return Workload(name, **base)
