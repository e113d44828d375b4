"""Pins for the oracle's backward (gradients of L = sum(out * dout) with
respect to q, k, v, rel_h, rel_w).

The pages train this layer (HaloNet paper, section 2.2 and Figure 3: the
speed-ups are training step times) but print no gradient, so the backward
is pinned to the forward oracle and to the mathematics, never to its own
formula retyped:
  * central finite differences of the forward oracle, element by element, on
    tiny inputs (stride 1 and 2, with and without halo, SASA mask);
  * closed-form identities of the sums: the v-gradient over all keys equals
    the dout sum (softmax rows sum to one), every table gradient sums to
    zero over its rows (softmax gradients sum to zero per query), and
    Euler's identity for the bilinear logits (sum q.dq equals
    sum k.dk + sum rel_h.drel_h + sum rel_w.drel_w);
  * block = H = W with halo 0 (global attention with a relative bias,
    section 2.2) against torch autograd of a dense formulation.
A planted sign error in a gradient is caught by the finite differences.
"""
import math

import numpy as np
import pytest
import torch

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def _randn(rng, *shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float32)


def _inputs(seed, N, H, W, heads, d, b, h, S):
    rng = _rng(seed)
    w = b + 2 * h
    q, k, v = (_randn(rng, N, H, W, heads * d) for _ in range(3))
    rel_h, rel_w = _randn(rng, 2 * w - 1, d, scale=0.5), _randn(rng, 2 * w - 1, d, scale=0.5)
    dout = _randn(rng, N, H // S, W // S, heads * d)
    return [q, k, v, rel_h, rel_w], dout


def _loss(x, dout, b, h, S, kernel):
    if kernel:
        out = oracle.halo_attention_masked(*x, block=b, halo=h, kernel=kernel, stride=S)
    else:
        out = oracle.halo_attention(*x, block=b, halo=h, stride=S)
    return float(np.sum(out * dout.astype(np.float64)))


def _finite_differences(x, dout, b, h, S, kernel, which, eps=2.0 ** -14):
    """Central differences of L over every element of input `which`.  The
    quotient divides by the step actually stored in float32 (x + eps and
    x - eps are rounded where they cross a power of two)."""
    base = x[which]
    fd = np.zeros(base.shape, dtype=np.float64)
    flat = base.reshape(-1)
    for i in range(flat.size):
        keep = flat[i]
        flat[i] = keep + np.float32(eps)
        xp = float(flat[i])
        lp = _loss(x, dout, b, h, S, kernel)
        flat[i] = keep - np.float32(eps)
        xm = float(flat[i])
        lm = _loss(x, dout, b, h, S, kernel)
        flat[i] = keep
        fd.reshape(-1)[i] = (lp - lm) / (xp - xm)
    return fd


FD_CASES = [
    # N, H, W, heads, d, b, h, S, kernel
    (1, 8, 8, 2, 3, 4, 1, 1, 0),
    (1, 8, 4, 1, 4, 4, 2, 1, 0),
    (1, 8, 8, 1, 3, 4, 1, 2, 0),
    (1, 6, 6, 2, 2, 2, 0, 1, 0),
    (1, 8, 8, 1, 3, 4, 2, 1, 3),
]


@pytest.mark.parametrize("case", FD_CASES, ids=lambda c: "H{1}W{2}_b{5}h{6}_S{7}_k{8}".format(*c))
def test_gradients_match_finite_differences(case):
    N, H, W, heads, d, b, h, S, kernel = case
    x, dout = _inputs(31, N, H, W, heads, d, b, h, S)
    grads = oracle.halo_attention_bwd(*x, dout, block=b, halo=h, stride=S, kernel=kernel)
    for which, name in enumerate(["dq", "dk", "dv", "drel_h", "drel_w"]):
        fd = _finite_differences(x, dout, b, h, S, kernel, which)
        scale = max(1.0, np.abs(fd).max())
        np.testing.assert_allclose(grads[which], fd, rtol=0, atol=2e-6 * scale, err_msg=name)


def test_finite_differences_catch_a_planted_sign_error():
    """The pin is not vacuous: a sign slip in one table's gradient (planted
    here in the oracle's result) fails it."""
    N, H, W, heads, d, b, h, S, kernel = FD_CASES[0]
    x, dout = _inputs(31, N, H, W, heads, d, b, h, S)
    grads = list(oracle.halo_attention_bwd(*x, dout, block=b, halo=h, stride=S))
    fd = _finite_differences(x, dout, b, h, S, 0, 4)
    assert np.abs(grads[4] - fd).max() < 1e-5
    assert np.abs(-grads[4] - fd).max() > 1e-2
    # and a swap of the two tables' gradients fails too
    assert np.abs(grads[3] - fd).max() > 1e-2


@pytest.mark.parametrize("b,h,S,kernel", [(4, 1, 1, 0), (8, 3, 1, 0), (8, 3, 2, 0), (4, 2, 1, 5), (8, 0, 1, 0)])
def test_closed_form_identities(b, h, S, kernel):
    x, dout = _inputs(32, 2, 16, 24, 3, 8, b, h, S)
    q, k, v, rel_h, rel_w = [t.astype(np.float64) for t in x]
    dq, dk, dv, drh, drw = oracle.halo_attention_bwd(*x, dout, block=b, halo=h, stride=S, kernel=kernel)
    C = q.shape[-1]
    # sum over every key pixel of dv = sum over every query of dout (per image and channel)
    np.testing.assert_allclose(dv.sum(axis=(1, 2)), dout.astype(np.float64).sum(axis=(1, 2)), rtol=0, atol=1e-9)
    # table gradients sum to zero over their rows
    np.testing.assert_allclose(drh.sum(axis=0), 0.0, atol=1e-9)
    np.testing.assert_allclose(drw.sum(axis=0), 0.0, atol=1e-9)
    # Euler: the logits are bilinear in q and (k, rel_h, rel_w)
    lhs = float(np.sum(q * dq))
    rhs = float(np.sum(k * dk) + np.sum(rel_h * drh) + np.sum(rel_w * drw))
    assert abs(lhs - rhs) <= 1e-9 * max(1.0, abs(lhs))
    # queries only at the strided pixels: dq vanishes elsewhere
    if S == 2:
        mask = np.zeros(q.shape[1:3], bool)
        mask[::2, ::2] = True
        assert np.all(dq[:, ~mask] == 0.0)
    assert C == 24


def _dense_global_torch(q, k, v, rel_h, rel_w, heads):
    """Global attention with the relative bias B[i, j] = q_i . (rel_h[r_j -
    r_i + H - 1] + rel_w[c_j - c_i + W - 1]), written densely in torch."""
    _, H, W, C = q.shape
    d = C // heads
    ys, xs = torch.meshgrid(torch.arange(H), torch.arange(W), indexing="ij")
    ys, xs = ys.reshape(-1), xs.reshape(-1)
    ih = ys[None, :] - ys[:, None] + H - 1
    iw = xs[None, :] - xs[:, None] + W - 1
    outs = []
    for hd in range(heads):
        sl = slice(hd * d, (hd + 1) * d)
        Q = q[0, :, :, sl].reshape(H * W, d)
        K = k[0, :, :, sl].reshape(H * W, d)
        V = v[0, :, :, sl].reshape(H * W, d)
        B = torch.einsum("id,ijd->ij", Q, rel_h[ih] + rel_w[iw])
        P = torch.softmax((Q @ K.T + B) / math.sqrt(d), dim=1)
        outs.append(P @ V)
    return torch.cat(outs, dim=1).reshape(1, H, W, C)


def test_global_attention_gradients_match_autograd():
    H = W = 6
    heads, d = 2, 4
    x, dout = _inputs(33, 1, H, W, heads, d, H, 0, 1)
    tx = [torch.tensor(t, dtype=torch.float64, requires_grad=True) for t in x]
    out = _dense_global_torch(*tx, heads)
    want = torch.autograd.grad((out * torch.tensor(dout, dtype=torch.float64)).sum(), tx)
    got = oracle.halo_attention_bwd(*x, dout, block=H, halo=0)
    for g, wv, name in zip(got, want, ["dq", "dk", "dv", "drel_h", "drel_w"]):
        np.testing.assert_allclose(g, wv.numpy(), rtol=0, atol=1e-12, err_msg=name)


def test_bwd_rejects_bad_arguments():
    x, dout = _inputs(34, 1, 8, 8, 1, 4, 4, 1, 1)
    with pytest.raises(ValueError):
        oracle.halo_attention_bwd(*x, dout, block=3, halo=1)
    with pytest.raises(ValueError):
        oracle.halo_attention_bwd(*x, dout, block=4, halo=1, kernel=5)  # kernel // 2 > halo
