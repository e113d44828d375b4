"""Pins for the oracle's fused-projection form (the blog page's HaloAttention:
to_q and to_kv are bias-free linear maps of the input map x, k and v the two
halves of to_kv's output; HaloNet appendix D fuses around the op):
  * identity weights (c_in = heads*d) reduce it exactly to the op on x;
  * the projection done independently with a numpy matmul (rounded to the
    dtype as an unfused pipeline stores it) followed by the pinned forward
    oracle gives the same result (pins the weight layout and the k / v
    halves);
  * zero query weights make every logit zero, so each output is the mean of v
    over the query's in-image window keys (closed form);
  * swapping the k and v halves changes the result (the pin is not vacuous).
"""
import numpy as np
import pytest

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def _randn(rng, *shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float32)


def _setup(seed, N=1, H=8, W=8, c_in=6, heads=2, d=4, b=4, h=1):
    rng = _rng(seed)
    x = _randn(rng, N, H, W, c_in)
    wq = _randn(rng, heads * d, c_in, scale=c_in ** -0.5)
    wkv = _randn(rng, 2 * heads * d, c_in, scale=c_in ** -0.5)
    w = b + 2 * h
    rh, rw = _randn(rng, 2 * w - 1, d, scale=0.5), _randn(rng, 2 * w - 1, d, scale=0.5)
    return x, wq, wkv, rh, rw


def test_identity_weights_reduce_to_the_op_on_x():
    heads, d = 2, 4
    x, _, _, rh, rw = _setup(50, c_in=heads * d, heads=heads, d=d)
    eye = np.eye(heads * d, dtype=np.float32)
    got = oracle.halo_attention_fused(x, eye, np.concatenate([eye, eye]), rh, rw, block=4, halo=1, heads=heads)
    want = oracle.halo_attention(x, x, x, rh, rw, block=4, halo=1)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("b,h,S", [(4, 1, 1), (4, 2, 2), (8, 3, 1)])
def test_matmul_projection_then_forward_oracle(b, h, S):
    heads, d, c_in = 2, 4, 6
    x, wq, wkv, rh, rw = _setup(51, H=16, W=8, c_in=c_in, heads=heads, d=d, b=b, h=h)
    xd = x.astype(np.float64)
    q = (xd @ wq.T.astype(np.float64)).astype(np.float32)
    kv = xd @ wkv.T.astype(np.float64)
    k, v = kv[..., :heads * d].astype(np.float32), kv[..., heads * d:].astype(np.float32)
    want = oracle.halo_attention(np.ascontiguousarray(q), np.ascontiguousarray(k), np.ascontiguousarray(v), rh, rw,
                                 block=b, halo=h, stride=S)
    got = oracle.halo_attention_fused(x, wq, wkv, rh, rw, block=b, halo=h, heads=heads, stride=S)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
    swapped = np.concatenate([wkv[heads * d:], wkv[:heads * d]])
    other = oracle.halo_attention_fused(x, wq, swapped, rh, rw, block=b, halo=h, heads=heads, stride=S)
    assert np.abs(other - want).max() > 1e-2


def test_zero_query_weights_average_v_over_the_window():
    heads, d, c_in, b, h = 1, 4, 5, 4, 1
    x, wq, wkv, rh, rw = _setup(52, c_in=c_in, heads=heads, d=d, b=b, h=h)
    got = oracle.halo_attention_fused(x, np.zeros_like(wq), wkv, rh, rw, block=b, halo=h, heads=heads)
    v = (x.astype(np.float64) @ wkv[heads * d:].T.astype(np.float64)).astype(np.float32).astype(np.float64)
    H, W = x.shape[1:3]
    for y in range(H):
        for xx in range(W):
            y0, x0 = (y // b) * b - h, (xx // b) * b - h
            ys = slice(max(y0, 0), min(y0 + b + 2 * h, H))
            xs = slice(max(x0, 0), min(x0 + b + 2 * h, W))
            want = v[0, ys, xs].reshape(-1, d).mean(axis=0)
            np.testing.assert_allclose(got[0, y, xx], want, rtol=0, atol=1e-12)


def test_fused_bf16_rounds_projections_like_a_stored_pipeline():
    """bf16 inputs: the projections are rounded to bf16 (nearest even) before
    the op, exactly as torch rounds a float32 tensor to bf16."""
    import torch
    heads, d, c_in = 2, 8, 16
    x, wq, wkv, rh, rw = _setup(53, H=16, W=16, c_in=c_in, heads=heads, d=d, b=8, h=3)
    tb = lambda a: torch.from_numpy(a).to(torch.bfloat16)
    xb, wqb, wkvb, rhb, rwb = map(tb, (x, wq, wkv, rh, rw))
    xd = xb.double()
    q = (xd @ wqb.double().T).float().to(torch.bfloat16)
    kv = (xd @ wkvb.double().T).float().to(torch.bfloat16)
    want = oracle.halo_attention(q.contiguous(), kv[..., :heads * d].contiguous(), kv[..., heads * d:].contiguous(),
                                 rhb, rwb, block=8, halo=3)
    got = oracle.halo_attention_fused(xb, wqb, wkvb, rhb, rwb, block=8, halo=3, heads=heads)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)
