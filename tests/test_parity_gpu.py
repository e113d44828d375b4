"""GPU parity: libhalo (through its C ABI) against the CPU oracle, element by
element on the same seeded inputs.

Tolerances (max-abs): 1e-4 for float32 inputs, 2e-2 for bf16 inputs with
float32 accumulation.  The five full-size workloads are compared on every
output pixel (the multi-threaded oracle takes a few seconds each); smaller
cases that span many blocks, heads and a ragged number of work items are
compared in full too, and so are the numerics stress cases (large relative
tables, strongly negative logits at the image border).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from workloads import WORKLOADS, custom, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def _lib():
    import blocked_local_self_b200 as h
    h.load()
    return h


def _run(wl, inputs, **kw):
    h = _lib()
    dev = [t.cuda() for t in inputs]
    out = h.attn(*dev, block=wl.block, halo=wl.halo, stride=wl.stride, **kw)
    torch.cuda.synchronize()
    assert h.get_last_error() == 0
    return out


def _compare(got, want, tol, what=""):
    got = got.detach().cpu().to(torch.float64).numpy()
    err = np.abs(got - want)
    assert np.all(np.isfinite(got)), f"{what}: non-finite outputs"
    assert err.max() <= tol, f"{what}: max abs err {err.max():.3e} > {tol} (mean {err.mean():.2e})"
    print(f"[parity] {what}: max abs err {err.max():.3e} (mean {err.mean():.2e}, tol {tol})")
    return err.max()


def _samples(wl, count, seed=0):
    """Border rows/columns, the four corners of every image and random pixels."""
    rng = np.random.default_rng(seed)
    OH, OW = wl.out_hw
    pts = set()
    for n in {0, wl.N - 1}:
        for oy, ox in [(0, 0), (0, OW - 1), (OH - 1, 0), (OH - 1, OW - 1)]:
            pts.add((n, oy, ox))
        for ox in range(0, OW, max(1, OW // 8)):
            pts.add((n, 0, ox))
            pts.add((n, OH - 1, ox))
        for oy in range(0, OH, max(1, OH // 8)):
            pts.add((n, oy, 0))
            pts.add((n, oy, OW - 1))
    while len(pts) < count:
        pts.add((int(rng.integers(wl.N)), int(rng.integers(OH)), int(rng.integers(OW))))
    return np.array(sorted(pts), dtype=np.int32)


# ---------------------------------------------------------------------------
# full-size workloads
# ---------------------------------------------------------------------------

def test_tiny_f32_full():
    wl = WORKLOADS["tiny_f32"]
    inputs = make_inputs(wl)
    got = _run(wl, inputs)
    want = oracle.halo_attention(*inputs, block=wl.block, halo=wl.halo, stride=wl.stride)
    _compare(got, want, TOL["f32"], wl.name)


@pytest.mark.parametrize("name", ["stage1_bf16", "deep_bf16", "stride2_bf16", "large_bf16"])
def test_full_size_every_pixel(name):
    """The full-size workload in the launch configuration the benchmark times
    (one launch over the whole batch), every output pixel against the oracle."""
    wl = WORKLOADS[name]
    inputs = make_inputs(wl)
    got = _run(wl, inputs)
    want = oracle.halo_attention(*inputs, block=wl.block, halo=wl.halo, stride=wl.stride)
    _compare(got, want, TOL[wl.dtype], name)


@pytest.mark.parametrize("name", ["stage1_bf16", "large_bf16"])
def test_full_size_sampled_pixels_match_full_oracle(name):
    """The oracle's sampled form (used by smaller checks) agrees with its full
    form on the GPU output's pixels: borders, corners and random pixels."""
    wl = WORKLOADS[name]
    inputs = make_inputs(wl)
    got = _run(wl, inputs)
    smp = _samples(wl, 384)
    want = oracle.halo_attention_samples(*inputs, smp, block=wl.block, halo=wl.halo, stride=wl.stride)
    g = got[smp[:, 0], smp[:, 1], smp[:, 2]]
    _compare(g, want, TOL[wl.dtype], name + " sampled")


@pytest.mark.parametrize("name,kernel", [("stage1_bf16", "tc_bf16"), ("deep_bf16", "tc_bf16"),
                                         ("stride2_bf16", "tc_bf16"), ("large_bf16", "tc_bf16"),
                                         ("tiny_f32", "simt_f32")])
def test_kernel_selection(name, kernel):
    h = _lib()
    wl = WORKLOADS[name]
    assert h.kernel_for(wl.N, wl.H, wl.W, wl.heads, wl.dim_head, wl.block, wl.halo, wl.stride,
                        wl.torch_dtype) == kernel


# ---------------------------------------------------------------------------
# smaller cases compared in full: every tensor-core instantiation family
# ---------------------------------------------------------------------------

CASES = []
for d in (16, 32, 64):
    for halo in (0, 1, 2, 3):
        for stride in (1, 2):
            CASES.append(dict(N=2, H=24, W=40, heads=8 if d < 64 else 4, dim_head=d, block=8, halo=halo,
                              stride=stride))
# odd head counts at stride 1 (d = 16, 32): with an odd number of block rows
# the one-head-per-item kernel, with an even number the two-block kernel
CASES += [
    dict(N=2, H=24, W=24, heads=3, dim_head=16, block=8, halo=3, stride=1),
    dict(N=2, H=24, W=24, heads=3, dim_head=32, block=8, halo=2, stride=1),
    dict(N=2, H=16, W=24, heads=3, dim_head=16, block=8, halo=3, stride=1),
    dict(N=2, H=16, W=24, heads=3, dim_head=32, block=8, halo=2, stride=1),
]
# an even number of block rows: the kernel that pairs two vertically adjacent
# blocks (every head size and window, one pair and several pairs)
for d in (16, 32, 64):
    for halo in (0, 1, 2, 3):
        CASES.append(dict(N=2, H=32, W=24, heads=3, dim_head=d, block=8, halo=halo, stride=1))
CASES.append(dict(N=3, H=16, W=40, heads=2, dim_head=64, block=8, halo=3, stride=1))
# 16x16 query blocks (windows 16..24): every window of the block-16 kernel, both head sizes
for d in (16, 32):
    for halo in (0, 1, 2, 3, 4):
        CASES.append(dict(N=2, H=32, W=48, heads=3, dim_head=d, block=16, halo=halo, stride=1))
# 32x32 query blocks (windows 32..38): global attention on a 32x32 map and
# haloed 32x32 blocks, both head sizes, every window
for d in (16, 32):
    for halo in (0, 1, 2, 3):
        CASES.append(dict(N=1, H=64, W=32 if halo else 64, heads=2, dim_head=d, block=32, halo=halo, stride=1))
CASES += [
    dict(N=3, H=32, W=32, heads=3, dim_head=32, block=32, halo=0, stride=1),  # global attention, several items per CTA
    dict(N=1, H=32, W=96, heads=1, dim_head=16, block=32, halo=3, stride=1),  # one block row
]
CASES += [
    dict(N=1, H=16, W=16, heads=2, dim_head=32, block=16, halo=4, stride=1),  # block = map, halo all outside
    dict(N=3, H=16, W=80, heads=1, dim_head=16, block=16, halo=4, stride=1),  # one block row, one head
    dict(N=1, H=8, W=8, heads=8, dim_head=16, block=8, halo=0, stride=1),    # global attention
    dict(N=1, H=8, W=8, heads=2, dim_head=32, block=8, halo=3, stride=1),    # block = map, halo all outside
    dict(N=3, H=16, W=8, heads=4, dim_head=64, block=8, halo=0, stride=2),   # isolated blocks, stride 2
    dict(N=5, H=8, W=56, heads=8, dim_head=16, block=8, halo=3, stride=1),   # one block row, ragged items
    dict(N=1, H=64, W=8, heads=2, dim_head=32, block=8, halo=3, stride=2),   # one block column
    # several items per CTA with both softmax warpgroups and every stage cycling
    dict(N=8, H=32, W=48, heads=8, dim_head=16, block=8, halo=3, stride=1),
    dict(N=8, H=32, W=48, heads=4, dim_head=16, block=8, halo=2, stride=1),
]
# stride 2 with about five items per CTA, every window: both warpgroups, both
# V buffers and (d = 32, four heads per tile) the per-pair Q/K barriers cycle
for d in (16, 32):
    for halo in (0, 1, 2, 3):
        CASES.append(dict(N=16, H=32, W=48, heads=8, dim_head=d, block=8, halo=halo, stride=2))
# four heads (one tile per block), more items than CTAs
CASES.append(dict(N=8, H=32, W=48, heads=4, dim_head=32, block=8, halo=3, stride=2))
CASES.append(dict(N=8, H=32, W=48, heads=4, dim_head=16, block=8, halo=2, stride=2))


@pytest.mark.parametrize("case", CASES, ids=lambda c: "d{dim_head}_h{halo}_s{stride}_{H}x{W}_n{N}_heads{heads}".format(**c))
def test_small_full_bf16(case):
    wl = custom("case", dtype="bf16", **case)
    inputs = make_inputs(wl, seed=hash(tuple(case.values())) % 1000)
    h = _lib()
    assert h.kernel_for(wl.N, wl.H, wl.W, wl.heads, wl.dim_head, wl.block, wl.halo, wl.stride,
                        torch.bfloat16) == "tc_bf16"
    got = _run(wl, inputs)
    want = oracle.halo_attention(*inputs, block=wl.block, halo=wl.halo, stride=wl.stride)
    _compare(got, want, TOL["bf16"], str(case))


def test_stage1_shape_in_float32_every_pixel():
    """The float32 path (window staged in shared memory) at the stage-1
    layer's full size, every output pixel against the oracle at 1e-4."""
    wl = workloads.NEXT_WORKLOADS["stage1_f32"]
    h = _lib()
    assert h.kernel_name(wl.N, wl.H, wl.W, wl.heads, wl.dim_head, wl.block, wl.halo, wl.stride,
                         wl.torch_dtype) == "halo_fwd_win<float,16>"
    inputs = make_inputs(wl)
    got = _run(wl, inputs)
    want = oracle.halo_attention(*inputs, block=wl.block, halo=wl.halo, stride=wl.stride)
    _compare(got, want, TOL["f32"], wl.name)


SIMT_CASES = [
    dict(N=2, H=12, W=20, heads=3, dim_head=8, block=4, halo=2, stride=1, dtype="f32"),
    dict(N=1, H=16, W=16, heads=2, dim_head=40, block=4, halo=1, stride=2, dtype="f32"),
    dict(N=1, H=9, W=9, heads=1, dim_head=16, block=3, halo=1, stride=1, dtype="f32"),
    dict(N=1, H=32, W=32, heads=2, dim_head=128, block=16, halo=2, stride=1, dtype="f32"),
    dict(N=2, H=32, W=32, heads=4, dim_head=40, block=16, halo=4, stride=1, dtype="bf16"),
    dict(N=1, H=16, W=16, heads=1, dim_head=16, block=8, halo=3, stride=2, dtype="bf16"),
    dict(N=2, H=24, W=16, heads=4, dim_head=16, block=8, halo=4, stride=1, dtype="bf16"),
    # window staged in shared memory: every dim_head it takes, both strides, ragged passes
    dict(N=2, H=16, W=24, heads=3, dim_head=64, block=8, halo=3, stride=1, dtype="f32"),
    dict(N=1, H=32, W=32, heads=2, dim_head=128, block=8, halo=2, stride=2, dtype="f32"),
    dict(N=1, H=32, W=32, heads=2, dim_head=16, block=32, halo=0, stride=1, dtype="f32"),  # 1024 queries, 4 passes
    dict(N=2, H=16, W=16, heads=2, dim_head=8, block=16, halo=3, stride=2, dtype="f32"),
    dict(N=1, H=24, W=24, heads=2, dim_head=32, block=12, halo=5, stride=1, dtype="bf16"),
]


@pytest.mark.parametrize("case", SIMT_CASES, ids=lambda c: "{dtype}_d{dim_head}_b{block}_h{halo}_s{stride}".format(**c))
def test_small_full_simt(case):
    wl = custom("case", **case)
    inputs = make_inputs(wl, seed=7)
    got = _run(wl, inputs)
    want = oracle.halo_attention(*inputs, block=wl.block, halo=wl.halo, stride=wl.stride)
    _compare(got, want, TOL[wl.dtype], str(case))


# ---------------------------------------------------------------------------
# numerics edge cases
# ---------------------------------------------------------------------------

def test_saturated_softmax_and_constant_values():
    """Large logits (one key dominates) and constant v (output = v exactly up
    to bf16 rounding)."""
    wl = custom("sat", N=2, H=16, W=16, heads=8, dim_head=16, block=8, halo=3, stride=1, dtype="bf16")
    q, k, v, rh, rw = make_inputs(wl, seed=3)
    q8, k8 = (q.float() * 8).to(torch.bfloat16), (k.float() * 8).to(torch.bfloat16)
    got = _run(wl, (q8, k8, v, rh, rw))
    want = oracle.halo_attention(q8, k8, v, rh, rw, block=8, halo=3)
    _compare(got, want, TOL["bf16"], "saturated")
    vc = torch.full_like(v, 0.75)
    got = _run(wl, (q, k, vc, rh, rw))
    assert torch.all(got == 0.75)


@pytest.mark.parametrize("scale", [2.0, 4.0, 8.0])
def test_block16_running_maximum(scale):
    """Scaled q and k make later key chunks exceed earlier maxima by a wide
    margin, which exercises the block-16 kernel's rescaling of the
    accumulator; the scale-2 case moves the maximum only sometimes."""
    wl = custom("sat16", N=2, H=32, W=32, heads=2, dim_head=32, block=16, halo=4, stride=1, dtype="bf16")
    q, k, v, rh, rw = make_inputs(wl, seed=13)
    qs, ks = (q.float() * scale).to(torch.bfloat16), (k.float() * scale).to(torch.bfloat16)
    # A peaked softmax passes single values of v through: v is halved so that
    # |out| stays below ~2.5, where rounding the output to bf16 costs at most
    # 0.0078 of the 2e-2 budget (above 4 it alone would cost 0.0156).
    v = (v.float() * 0.5).to(torch.bfloat16)
    got = _run(wl, (qs, ks, v, rh, rw))
    want = oracle.halo_attention(qs, ks, v, rh, rw, block=16, halo=4)
    _compare(got, want, TOL["bf16"], f"block16 scale {scale}")


# One case per tensor-core kernel family (the kernel name prefix it must
# select), used by the large-relative-table stress test.
FAMILY_CASES = {
    "halo_fwd_tc4<16,": dict(N=2, H=32, W=24, heads=3, dim_head=16, block=8, halo=3, stride=1),
    "halo_fwd_tc4<32,": dict(N=2, H=32, W=24, heads=3, dim_head=32, block=8, halo=3, stride=1),
    "halo_fwd_tc4<64,": dict(N=2, H=32, W=24, heads=2, dim_head=64, block=8, halo=3, stride=1),
    "halo_fwd_tc2<16,": dict(N=2, H=24, W=24, heads=4, dim_head=16, block=8, halo=3, stride=1),
    "halo_fwd_tc2<32,": dict(N=2, H=24, W=24, heads=2, dim_head=32, block=8, halo=2, stride=1),
    "halo_fwd_tc<64,14,1,1>": dict(N=2, H=24, W=24, heads=2, dim_head=64, block=8, halo=3, stride=1),
    "halo_fwd_tc<16,14,2,4>": dict(N=2, H=32, W=32, heads=8, dim_head=16, block=8, halo=3, stride=2),
    "halo_fwd_tc<32,14,2,4>": dict(N=2, H=32, W=32, heads=4, dim_head=32, block=8, halo=3, stride=2),
    "halo_fwd_tc<32,14,2,2>": dict(N=2, H=32, W=32, heads=2, dim_head=32, block=8, halo=3, stride=2),
    "halo_fwd_tc3<16,": dict(N=1, H=32, W=32, heads=2, dim_head=16, block=16, halo=3, stride=1),
    "halo_fwd_tc3<32,": dict(N=1, H=32, W=48, heads=2, dim_head=32, block=16, halo=4, stride=1),
    "halo_fwd_tc3<16,38,32>": dict(N=1, H=64, W=32, heads=2, dim_head=16, block=32, halo=3, stride=1),
    "halo_fwd_tc3<32,32,32>": dict(N=2, H=32, W=32, heads=2, dim_head=32, block=32, halo=0, stride=1),
}


def _scaled(t, f):
    """Multiply a bf16 tensor by a power of two (exact)."""
    return (t.float() * f).to(t.dtype)


@pytest.mark.parametrize("rel_scale", [8.0, 32.0, 64.0])
@pytest.mark.parametrize("family", sorted(FAMILY_CASES))
def test_large_relative_tables(family, rel_scale):
    """Relative tables scaled by 8..64 and q by 4: the relative logits span
    tens to hundreds of log2 units, so the two-block kernel's bound of the row
    maximum overshoots by more than the exponential's range (its exact
    maximum must take over), the block-16 kernel moves its running maximum
    and rescales, and the per-chunk maxima of the other kernels see chunks
    far below the row's maximum.  v is halved so that the near one-hot
    outputs stay where rounding the output to bf16 fits the bar."""
    case = FAMILY_CASES[family]
    wl = custom("bigrel", dtype="bf16", **case)
    h = _lib()
    assert h.kernel_name(wl.N, wl.H, wl.W, wl.heads, wl.dim_head, wl.block, wl.halo, wl.stride,
                         wl.torch_dtype).startswith(family)
    q, k, v, rh, rw = make_inputs(wl, seed=21)
    q, rh, rw, v = _scaled(q, 4.0), _scaled(rh, rel_scale), _scaled(rw, rel_scale), _scaled(v, 0.5)
    got = _run(wl, (q, k, v, rh, rw))
    want = oracle.halo_attention(q, k, v, rh, rw, block=wl.block, halo=wl.halo, stride=wl.stride)
    _compare(got, want, TOL["bf16"], f"{family} rel x{rel_scale:g}")


@pytest.mark.parametrize("family", sorted(FAMILY_CASES))
def test_strongly_negative_logits_at_border(family):
    """q and k anti-aligned (q = a u + noise, k = -a u + noise per head): every
    in-image logit is strongly negative (about -150 log2 units and below),
    while the zero-filled out-of-image keys of a border window give S = 0.
    The two-block kernel's cheap bound of the row maximum then lies far above
    the exact one; the output must still match."""
    case = FAMILY_CASES[family]
    wl = custom("antialign", dtype="bf16", **case)
    q, k, v, rh, rw = make_inputs(wl, seed=22)
    g = torch.Generator().manual_seed(23)
    u = torch.randn((wl.heads, wl.dim_head), generator=g)
    a = 6.0
    base = (a * u).reshape(1, 1, 1, wl.C)
    qa = (base + q.float()).to(torch.bfloat16)
    ka = (-base + k.float()).to(torch.bfloat16)
    v = _scaled(v, 0.5)
    got = _run(wl, (qa, ka, v, rh, rw))
    want = oracle.halo_attention(qa, ka, v, rh, rw, block=wl.block, halo=wl.halo, stride=wl.stride)
    _compare(got, want, TOL["bf16"], f"{family} anti-aligned")


def test_deterministic():
    wl = WORKLOADS["stage1_bf16"]
    inputs = [t.cuda() for t in make_inputs(wl)]
    h = _lib()
    a = h.attn(*inputs, block=wl.block, halo=wl.halo)
    b = h.attn(*inputs, block=wl.block, halo=wl.halo)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


@pytest.mark.parametrize("name", ["stage1_bf16", "stride2_bf16", "tiny_f32"])
def test_no_writes_outside_output(name):
    """Guard bands before and after `out` keep their canary value."""
    wl = WORKLOADS[name]
    h = _lib()
    inputs = [t.cuda() for t in make_inputs(wl)]
    OH, OW = wl.out_hw
    n_out = wl.N * OH * OW * wl.C
    guard = 4096
    buf = torch.full((n_out + 2 * guard,), 12345.0, dtype=wl.torch_dtype, device="cuda")
    out = buf[guard:guard + n_out].view(wl.N, OH, OW, wl.C)
    h.attn(*inputs, block=wl.block, halo=wl.halo, stride=wl.stride, out=out)
    torch.cuda.synchronize()
    assert torch.all(buf[:guard] == 12345.0) and torch.all(buf[guard + n_out:] == 12345.0)


def test_host_entry_point_matches_device_entry_point():
    wl = custom("e2e", N=2, H=32, W=32, heads=8, dim_head=16, block=8, halo=3, stride=1, dtype="bf16")
    inputs = [t.pin_memory() for t in make_inputs(wl, seed=5)]
    h = _lib()
    staging = {n: torch.empty_like(t, device="cuda") for n, t in zip(("q", "k", "v", "rel_h", "rel_w"), inputs)}
    staging["out"] = torch.empty((wl.N, wl.H, wl.W, wl.C), dtype=torch.bfloat16, device="cuda")
    out_h = torch.empty((wl.N, wl.H, wl.W, wl.C), dtype=torch.bfloat16).pin_memory()
    h.attn_host(*inputs, out_h, staging, block=8, halo=3)
    torch.cuda.synchronize()
    ref = h.attn(*[t.cuda() for t in inputs], block=8, halo=3)
    torch.cuda.synchronize()
    assert torch.equal(out_h, ref.cpu())


@pytest.mark.parametrize("n", [5, 13])
def test_host_entry_point_pipelined_chunks(n):
    """The host entry point splits the batch into chunks on two library
    streams: ragged chunk sizes give the same result as the device entry
    point, and work queued on the caller's stream afterwards sees it all."""
    wl = custom("e2e", N=n, H=16, W=24, heads=4, dim_head=32, block=8, halo=2, stride=1, dtype="bf16")
    inputs = [t.pin_memory() for t in make_inputs(wl, seed=n)]
    h = _lib()
    staging = {nm: torch.empty_like(t, device="cuda") for nm, t in zip(("q", "k", "v", "rel_h", "rel_w"), inputs)}
    staging["out"] = torch.empty((wl.N, wl.H, wl.W, wl.C), dtype=torch.bfloat16, device="cuda")
    out_h = torch.empty((wl.N, wl.H, wl.W, wl.C), dtype=torch.bfloat16).pin_memory()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        h.attn_host(*inputs, out_h, staging, block=8, halo=2)
        after = staging["out"].float() * 1.0  # queued on the caller's stream after the call
    s.synchronize()
    ref = h.attn(*[t.cuda() for t in inputs], block=8, halo=2)
    torch.cuda.synchronize()
    assert torch.equal(out_h, ref.cpu())
    assert torch.equal(after, ref.float())


def test_side_stream():
    wl = custom("stream", N=2, H=16, W=24, heads=8, dim_head=32, block=8, halo=2, stride=1, dtype="bf16")
    inputs = make_inputs(wl, seed=11)
    h = _lib()
    s = torch.cuda.Stream()
    dev = [t.cuda() for t in inputs]
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        out = h.attn(*dev, block=8, halo=2)
    s.synchronize()
    want = oracle.halo_attention(*inputs, block=8, halo=2)
    _compare(out, want, TOL["bf16"], "side stream")


def test_rejects_bad_arguments_on_device():
    h = _lib()
    from blocked_local_self_b200 import _native as n
    wl = custom("bad", N=1, H=16, W=16, heads=2, dim_head=16, block=8, halo=3, dtype="bf16")
    q, k, v, rh, rw = [t.cuda() for t in make_inputs(wl)]
    with pytest.raises(h.HaloError) as e:
        h.attn(q, k, v, rh, rw, block=6, halo=3)
    assert e.value.code == n.HALO_ERR_DIVISIBILITY
    with pytest.raises(h.HaloError) as e:
        h.attn(q, k, v, rh, rw, block=8, halo=3, out=q)
    assert e.value.code == n.HALO_ERR_ALIAS


def test_timeout_path_reports_and_device_stays_usable():
    """A bounded device wait that nothing satisfies ends with HALO_ERR_TIMEOUT
    and the context keeps working."""
    h = _lib()
    from blocked_local_self_b200 import _native as n
    assert h.get_last_error() == 0
    assert h.debug_wait_timeout(2000) == n.HALO_ERR_TIMEOUT
    assert h.debug_wait_timeout(2000) == n.HALO_ERR_TIMEOUT  # its own flag starts clear each call
    assert h.get_last_error() == 0  # the self test does not set the operation's flag
    wl = WORKLOADS["tiny_f32"]
    inputs = make_inputs(wl)
    got = _run(wl, inputs)
    want = oracle.halo_attention(*inputs, block=wl.block, halo=wl.halo)
    _compare(got, want, TOL["f32"], "after timeout")
