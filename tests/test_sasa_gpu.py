"""GPU parity of the SASA-masked variant (``halo_attn_masked`` through the C
ABI) against the CPU oracle: each query keeps only the k x k keys centred on
it (HaloNet paper, section 2.2, the paragraph after Figure 1).  Tolerances as
for the unmasked op: max-abs 1e-4 for float32, 2e-2 for bf16."""
import numpy as np
import pytest
import torch

import oracle
from workloads import custom, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


def _lib():
    import blocked_local_self_b200 as h
    h.load()
    return h


SASA_CASES = [
    # the paper's comparison: block 8, halo 3, 7 x 7 centred window
    dict(N=2, H=32, W=24, heads=3, dim_head=16, block=8, halo=3, stride=1, dtype="bf16", kernel=7),
    dict(N=2, H=32, W=24, heads=2, dim_head=32, block=8, halo=3, stride=1, dtype="bf16", kernel=7),
    dict(N=1, H=16, W=16, heads=2, dim_head=64, block=8, halo=3, stride=1, dtype="bf16", kernel=5),
    dict(N=2, H=24, W=24, heads=2, dim_head=16, block=8, halo=2, stride=1, dtype="bf16", kernel=5),
    dict(N=1, H=16, W=16, heads=2, dim_head=32, block=8, halo=3, stride=2, dtype="bf16", kernel=7),
    dict(N=1, H=32, W=32, heads=2, dim_head=32, block=16, halo=4, stride=1, dtype="bf16", kernel=9),
    dict(N=1, H=16, W=16, heads=2, dim_head=32, block=4, halo=1, stride=1, dtype="f32", kernel=3),
    dict(N=1, H=16, W=16, heads=2, dim_head=16, block=8, halo=3, stride=1, dtype="f32", kernel=1),
]


@pytest.mark.parametrize("case", SASA_CASES,
                         ids=lambda c: "{dtype}_d{dim_head}_b{block}_h{halo}_s{stride}_k{kernel}".format(**c))
def test_sasa_matches_oracle(case):
    case = dict(case)
    kernel = case.pop("kernel")
    wl = custom("sasa", **case)
    inputs = make_inputs(wl, seed=17)
    h = _lib()
    out = h.attn_masked(*[t.cuda() for t in inputs], block=wl.block, halo=wl.halo, kernel=kernel,
                        stride=wl.stride)
    torch.cuda.synchronize()
    assert h.get_last_error() == 0
    want = oracle.halo_attention_masked(*inputs, block=wl.block, halo=wl.halo, kernel=kernel, stride=wl.stride)
    got = out.cpu().to(torch.float64).numpy()
    err = float(np.abs(got - want).max())
    assert np.all(np.isfinite(got)) and err <= TOL[wl.dtype], f"max abs err {err:.3e}"
    print(f"[sasa parity] {case} k={kernel}: max abs err {err:.3e}")


def test_sasa_rejects_bad_kernel_sizes():
    h = _lib()
    from blocked_local_self_b200 import _native as n
    wl = custom("bad", N=1, H=16, W=16, heads=2, dim_head=16, block=8, halo=3, dtype="bf16")
    dev = [t.cuda() for t in make_inputs(wl)]
    for k in (0, 4, 9):
        with pytest.raises(h.HaloError) as e:
            h.attn_masked(*dev, block=8, halo=3, kernel=k)
        assert e.value.code == n.HALO_ERR_KERNEL
