"""GPU parity of the fused-projection form (``halo_attn_fused`` through the C
ABI) against the CPU oracle's ``halo_attention_fused`` on the same seeded
inputs: the projections q = x wq^T and [k | v] = x wkv^T (rounded to bf16, as
a pipeline that stored them would), then the operation.

Tolerance 2e-2 max-abs on outputs of unit scale, the forward's bf16 bar: the
kernel accumulates the projections in float32 where the oracle is exact, so a
projection may round to the neighbouring bf16 value; that moves an output by
far less than the bar.
"""
import numpy as np
import pytest
import torch

import oracle
from workloads import FUSED_WORKLOADS, custom, make_fused_inputs

pytestmark = pytest.mark.gpu

TOL = 2e-2


def _lib():
    import blocked_local_self_b200 as h
    h.load()
    return h


def _check(got, want, what):
    got = got.detach().cpu().to(torch.float64).numpy()
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = float(np.abs(got - want).max())
    print(f"[fused parity] {what}: max abs err {err:.3e}")
    assert err <= TOL, f"{what}: max abs err {err:.3e} > {TOL}"


CASES = [
    dict(N=1, H=16, W=16, heads=2, dim_head=16, c_in=64, halo=3),
    dict(N=2, H=16, W=24, heads=3, dim_head=16, c_in=128, halo=3),    # odd head count
    dict(N=1, H=32, W=16, heads=1, dim_head=16, c_in=128, halo=2),    # one head
    dict(N=2, H=16, W=16, heads=2, dim_head=32, c_in=64, halo=3),
    dict(N=1, H=32, W=32, heads=4, dim_head=32, c_in=64, halo=1),
    dict(N=1, H=16, W=40, heads=2, dim_head=16, c_in=128, halo=0),    # window = block
    dict(N=3, H=48, W=8, heads=2, dim_head=32, c_in=64, halo=2),      # one block column
    dict(N=9, H=64, W=64, heads=2, dim_head=16, c_in=128, halo=3),    # several block pairs per CTA
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "N{N}_{H}x{W}_h{heads}_d{dim_head}_c{c_in}_halo{halo}".format(**c))
def test_fused_small_full(case):
    c_in = case.pop("c_in")
    wl = custom("fused", block=8, stride=1, dtype="bf16", **case)
    h = _lib()
    assert h.fused_kernel_name(wl.N, wl.H, wl.W, c_in, wl.heads, wl.dim_head, 8, wl.halo, 1, torch.bfloat16) == \
        f"halo_fused_tc<{wl.dim_head},{wl.window},{c_in}>"
    inputs = make_fused_inputs(wl, c_in, seed=11)
    dev = [t.cuda() for t in inputs]
    out = h.attn_fused(*dev, heads=wl.heads, block=8, halo=wl.halo)
    torch.cuda.synchronize()
    assert h.get_last_error() == 0
    want = oracle.halo_attention_fused(*inputs, block=8, halo=wl.halo, heads=wl.heads)
    _check(out, want, str(case) + f" c_in={c_in}")


def test_fused_matches_projection_then_attn():
    """The unfused pipeline on the GPU: q, k, v projected (float64 on the CPU,
    rounded to bf16) and passed to ``halo_attn``; the two library paths agree
    to the bar."""
    wl = custom("fused", N=2, H=32, W=32, heads=4, dim_head=16, block=8, halo=3, dtype="bf16")
    h = _lib()
    x, wq, wkv, rh, rw = make_fused_inputs(wl, 128, seed=12)
    xd = x.double()
    q = (xd @ wq.double().T).to(torch.bfloat16)
    kv = (xd @ wkv.double().T).to(torch.bfloat16)
    k, v = kv[..., :wl.C].contiguous(), kv[..., wl.C:].contiguous()
    ref = h.attn(q.cuda(), k.cuda(), v.cuda(), rh.cuda(), rw.cuda(), block=8, halo=3)
    got = h.attn_fused(x.cuda(), wq.cuda(), wkv.cuda(), rh.cuda(), rw.cuda(), heads=wl.heads, block=8, halo=3)
    torch.cuda.synchronize()
    err = (got.float() - ref.float()).abs().max().item()
    assert err <= TOL, err


def test_fused_full_size():
    """The benchmark's launch (stage-1 layer, c_in 128, the whole batch);
    images 0 and N-1 compared with the oracle element by element, and every
    image against the unfused library path as a property at full size."""
    wl, c_in = FUSED_WORKLOADS["stage1_fused_bf16"]
    h = _lib()
    inputs = make_fused_inputs(wl, c_in)
    dev = [t.cuda() for t in inputs]
    out = h.attn_fused(*dev, heads=wl.heads, block=wl.block, halo=wl.halo)
    torch.cuda.synchronize()
    assert h.get_last_error() == 0
    sel = [0, wl.N - 1]
    want = oracle.halo_attention_fused(inputs[0][sel].contiguous(), *inputs[1:], block=wl.block, halo=wl.halo,
                                       heads=wl.heads)
    _check(out[sel], want, "stage1_fused_bf16 images 0, N-1")
    x, wq, wkv = dev[:3]
    q = (x.float() @ wq.float().T).to(torch.bfloat16)
    kv = (x.float() @ wkv.float().T).to(torch.bfloat16)
    ref = h.attn(q, kv[..., :wl.C].contiguous(), kv[..., wl.C:].contiguous(), dev[3], dev[4], block=wl.block,
                 halo=wl.halo)
    err = (out.float() - ref.float()).abs().max().item()
    assert err <= TOL, f"full batch vs projection + halo_attn: {err:.3e}"


@pytest.mark.parametrize("stress", ["large_tables", "anti_aligned"])
def test_fused_stress(stress):
    """The forward's numerics stress cases through the fused path: tables x32
    with the query weights x4 (near one-hot rows, the bound's exact fallback),
    and query and key weights that make every in-image logit strongly negative
    next to the zero keys of the border."""
    wl = custom("fstress", N=1, H=16, W=24, heads=2, dim_head=16, block=8, halo=3, dtype="bf16")
    h = _lib()
    x, wq, wkv, rh, rw = make_fused_inputs(wl, 64, seed=13)
    sc = lambda t, f: (t.float() * f).to(torch.bfloat16)
    if stress == "large_tables":
        wq, rh, rw = sc(wq, 4.0), sc(rh, 32.0), sc(rw, 32.0)
    else:
        # a constant channel in x carries a large offset: q = +6u, k = -6u per head
        x = x.clone()
        x[..., 0] = 1.0
        g = torch.Generator().manual_seed(14)
        u = torch.randn((wl.C,), generator=g)
        wq, wkv = wq.clone(), wkv.clone()
        wq[:, 0] = (6.0 * u).to(torch.bfloat16)
        wkv[:wl.C, 0] = (-6.0 * u).to(torch.bfloat16)
    inputs = (x, wq, wkv, rh, rw)
    out = h.attn_fused(*[t.cuda() for t in inputs], heads=wl.heads, block=8, halo=3)
    torch.cuda.synchronize()
    assert h.get_last_error() == 0
    want = oracle.halo_attention_fused(*inputs, block=8, halo=3, heads=wl.heads)
    _check(out, want, f"fused {stress}")


def test_fused_unsupported_shape_raises():
    h = _lib()
    from blocked_local_self_b200 import _native as n
    wl = custom("fu", N=1, H=16, W=16, heads=2, dim_head=16, block=8, halo=3, dtype="bf16")
    x, wq, wkv, rh, rw = [t.cuda() for t in make_fused_inputs(wl, 96)]
    with pytest.raises(h.HaloError) as e:
        h.attn_fused(x, wq, wkv, rh, rw, heads=2, block=8, halo=3)
    assert e.value.code == n.HALO_ERR_UNSUPPORTED
