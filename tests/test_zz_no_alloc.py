"""The backward's no-allocation entry point, ``halo_attn_bwd_noalloc``,
called through the C ABI (ctypes), against the workspace-taking entry point
``halo_attn_bwd`` on the same inputs.

Some callers cannot call cudaMalloc when they run the backward: code whose
device memory all belongs to a caching allocator, or latency-critical paths
where an allocation's device-wide synchronisation is not acceptable.  For
them the library keeps the backward's float32 accumulators in a built-in
16 MiB device array.  This file is collected last (its name sorts after the
other test files), so a run that stops at the first failure has run every
other test before it.  It passes alone in a fresh process as well.

Tolerance: the backward tests' bar, tol * max(1, max |reference|) per
gradient, tol = 2e-2 for bf16 and 1e-4 for float32; the two entry points run
the same kernels, so they differ only by the order of float32 atomic sums.
"""
import ctypes

import pytest
import torch

from workloads import custom, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def _lib():
    import blocked_local_self_b200 as h
    h.load()
    return h


def _noalloc(lib, wl, dev, out, dout, kernel=0):
    grads = [torch.empty_like(dev[0]), torch.empty_like(dev[1]), torch.empty_like(dev[2]),
             torch.empty_like(dev[3]), torch.empty_like(dev[4])]
    code = 1 if wl.dtype == "bf16" else 0
    stream = torch.cuda.current_stream().cuda_stream
    rc = lib.halo_attn_bwd_noalloc(*[ctypes.c_void_p(t.data_ptr()) for t in (*dev, out, dout, *grads)],
                                   wl.N, wl.H, wl.W, wl.heads, wl.dim_head, wl.block, wl.halo, wl.stride,
                                   kernel, code, ctypes.c_void_p(stream))
    return rc, grads


@pytest.mark.parametrize("case", [
    dict(N=2, H=16, W=24, heads=3, dim_head=16, block=8, halo=3, stride=1, dtype="bf16"),
    dict(N=1, H=16, W=16, heads=2, dim_head=32, block=4, halo=1, stride=2, dtype="f32"),
], ids=["bf16_b8h3", "f32_b4h1_s2"])
def test_noalloc_matches_workspace_entry_point_twice(case):
    """Two calls in a row, on different inputs: the second must not see the
    first call's sums left in the shared array."""
    h = _lib()
    from blocked_local_self_b200 import _native
    lib = _native.lib()
    wl = custom("noalloc", **case)
    for seed in (1, 2):
        dev = [t.cuda() for t in make_inputs(wl, seed=seed)]
        out = h.attn(*dev, block=wl.block, halo=wl.halo, stride=wl.stride)
        g = torch.Generator().manual_seed(seed + 10)
        dout = torch.randn(out.shape, generator=g).to(out.dtype).cuda()
        rc, got = _noalloc(lib, wl, dev, out, dout)
        assert rc == 0, _native.strerror(rc)
        want = h.attn_bwd(*dev, out, dout, block=wl.block, halo=wl.halo, stride=wl.stride)
        torch.cuda.synchronize()
        assert h.get_last_error() == 0
        for a, b, name in zip(got, want, ("dq", "dk", "dv", "drel_h", "drel_w")):
            a, b = a.double(), b.double()
            scale = max(1.0, b.abs().max().item())
            err = (a - b).abs().max().item()
            assert err <= TOL[wl.dtype] * scale, f"call {seed} {name}: {err:.3e}"


def test_noalloc_rejects_shapes_beyond_its_scratch():
    """The stage-1 layer's full batch needs about 134 MB of accumulators,
    more than the 16 MiB array: a clear error, no device work."""
    from blocked_local_self_b200 import _native
    lib = _native.lib()
    nul = ctypes.c_void_p(16)
    rc = lib.halo_attn_bwd_noalloc(*([nul] * 12), 32, 64, 64, 8, 16, 8, 3, 1, 0, 1, None)
    assert rc == _native.HALO_ERR_SCRATCH_LIMIT
    assert "16 MiB" in _native.strerror(rc)
