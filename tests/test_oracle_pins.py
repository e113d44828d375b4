"""Pins for the CPU oracle: checks against what the HaloNet pages and the
mathematics fix, never against the oracle's own formula retyped.

Each test names the passage it follows.  The pages print no worked numerical
example, so the pins are: the blog page's relative-position recipe restated
independently (P1), special cases that reduce to dense matrix products (P2,
P2'), closed forms and invariants (P3-P5, golden file), the stride-2
definition (P6), the shift-by-b equivariance statement (P7), the half-channel
factorisation of Appendix A (P8), and a second naive implementation (P9).
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _randn(rng, *shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float32)


# ----------------------------------------------------------------------------
# P1: the blog page's rel_to_abs / relative_logits_1d recipe, restated.
# ----------------------------------------------------------------------------

def _rel_to_abs_recipe(x):
    """Blog page, ``rel_to_abs``: turn logits against the 2w-1 relative offsets
    into logits against the w absolute key positions by padding one zero
    column, flattening, padding (M - L) zeros, reshaping to (L+1, M) and keeping
    the last w columns of the first L rows.  x: [B, L, M] with M = 2w-1."""
    B, L, M = x.shape
    w = (M + 1) // 2
    x = np.concatenate([x, np.zeros((B, L, 1), x.dtype)], axis=2)
    flat = x.reshape(B, L * (M + 1))
    flat = np.concatenate([flat, np.zeros((B, M - L), x.dtype)], axis=1)
    full = flat.reshape(B, L + 1, M)
    return full[:, :L, M - w:]


def _rel_logits_recipe(q_block, rel_h, rel_w):
    """Blog page, ``RelPosEmb.forward``: q_block [b, b, d] (query rows x, cols
    y).  Returns the [b*b, w*w] relative logit matrix, queries in row-major
    (x, y) order and keys in row-major (row i, col j) window order."""
    b = q_block.shape[0]
    w = (rel_h.shape[0] + 1) // 2
    # width part: logits against rel_w along the query's column axis
    lw = np.einsum("xyd,rd->xyr", q_block, rel_w)          # [b(x), b(y), 2w-1]
    lw = _rel_to_abs_recipe(lw.reshape(b, b, -1))           # [b(x), b(y), w(j)]
    # height part: the same along the query's row axis (q transposed)
    lh = np.einsum("xyd,rd->yxr", q_block, rel_h)           # [b(y), b(x), 2w-1]
    lh = _rel_to_abs_recipe(lh.reshape(b, b, -1))           # [b(y), b(x), w(i)]
    out = np.zeros((b, b, w, w))
    for x in range(b):
        for y in range(b):
            out[x, y] = lh[y, x][:, None] + lw[x, y][None, :]
    return out.reshape(b * b, w * w)


@pytest.mark.parametrize("b,h", [(2, 1), (4, 1), (8, 3), (16, 4), (3, 0), (4, 2)])
def test_p1_relative_index_matches_blog_recipe(b, h):
    """The oracle's attention weights for a block whose window lies inside the
    image equal softmax(d^-1/2 * relative logits) with the logits built by the
    blog page's pad/flatten/reshape recipe (section 2.1 content-geometry term,
    appendix A factorisation)."""
    w = b + 2 * h
    H = W = 3 * b
    d = w * w  # one channel per window key, so v can label every key
    rng = _rng(1000 + b * 10 + h)
    q = _randn(rng, 1, H, W, d)
    k = np.zeros((1, H, W, d), np.float32)  # content term vanishes
    rel_h = _randn(rng, 2 * w - 1, d, scale=0.3)
    rel_w = _randn(rng, 2 * w - 1, d, scale=0.3)
    # centre block (1, 1): window rows/cols [b - h, 2b + h) are all in-image
    v = np.zeros((1, H, W, d), np.float32)
    for kr in range(w):
        for kc in range(w):
            v[0, b - h + kr, b - h + kc, kr * w + kc] = 1.0
    samples = [(0, b + qy, b + qx) for qy in range(b) for qx in range(b)]
    got = oracle.halo_attention_samples(q, k, v, rel_h, rel_w, samples, b, h, 1)
    logits = _rel_logits_recipe(q[0, b:2 * b, b:2 * b].astype(np.float64),
                                rel_h.astype(np.float64), rel_w.astype(np.float64))
    z = logits / math.sqrt(d)
    z = z - z.max(axis=1, keepdims=True)
    p = np.exp(z)
    p /= p.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(got, p, rtol=0, atol=1e-12)


def test_p1_recipe_is_not_vacuous():
    """A transposed axis assignment (rows <-> rel_w) must fail P1's check."""
    b, h = 4, 1
    w = b + 2 * h
    rng = _rng(7)
    qb = rng.standard_normal((b, b, 3))
    rh = rng.standard_normal((2 * w - 1, 3))
    rw = rng.standard_normal((2 * w - 1, 3))
    good = _rel_logits_recipe(qb, rh, rw)
    swapped = _rel_logits_recipe(qb, rw, rh)
    assert np.abs(good - swapped).max() > 1e-3


# ----------------------------------------------------------------------------
# P2 / P2': global attention special case (section 2.2: block = whole map).
# ----------------------------------------------------------------------------

def _dense_global(q, k, v, rel_h, rel_w, heads):
    """softmax(d^-1/2 (Q K^T + B)) V over all pixels, one image, by numpy
    matrix products; B is the relative term built with the blog recipe."""
    _, H, W, C = q.shape
    d = C // heads
    out = np.zeros((H * W, C))
    for hd in range(heads):
        sl = slice(hd * d, (hd + 1) * d)
        Q = q[0, :, :, sl].reshape(H * W, d).astype(np.float64)
        K = k[0, :, :, sl].reshape(H * W, d).astype(np.float64)
        V = v[0, :, :, sl].reshape(H * W, d).astype(np.float64)
        B = _rel_logits_recipe(q[0, :, :, sl].astype(np.float64), rel_h.astype(np.float64),
                               rel_w.astype(np.float64))
        Z = (Q @ K.T + B) / math.sqrt(d)
        Z -= Z.max(axis=1, keepdims=True)
        P = np.exp(Z)
        P /= P.sum(axis=1, keepdims=True)
        out[:, sl] = P @ V
    return out.reshape(1, H, W, C)


def test_p2_global_attention_reduction():
    """block = H = W, halo = 0 is global attention with a relative bias."""
    rng = _rng(2)
    H = W = 8
    heads, d = 2, 16
    q, k, v = (_randn(rng, 1, H, W, heads * d) for _ in range(3))
    rel_h = _randn(rng, 2 * H - 1, d, scale=0.25)
    rel_w = _randn(rng, 2 * W - 1, d, scale=0.25)
    got = oracle.halo_attention(q, k, v, rel_h, rel_w, block=H, halo=0)
    want = _dense_global(q, k, v, rel_h, rel_w, heads)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("halo", [1, 2])
def test_p2prime_halo_outside_image_is_masked(halo):
    """block = H = W with halo > 0: every halo key lies outside the image and
    must drop out, leaving global attention with the tables shifted by 3*halo
    rows (window coordinate = image coordinate + halo, window w = H + 2*halo)."""
    rng = _rng(3)
    H = W = 8
    heads, d = 2, 8
    q, k, v = (_randn(rng, 1, H, W, heads * d) for _ in range(3))
    rel_h = _randn(rng, 2 * H - 1, d, scale=0.25)
    rel_w = _randn(rng, 2 * W - 1, d, scale=0.25)
    w = H + 2 * halo
    big_h = _randn(rng, 2 * w - 1, d, scale=5.0)  # rows no in-image key uses
    big_w = _randn(rng, 2 * w - 1, d, scale=5.0)
    big_h[3 * halo:3 * halo + 2 * H - 1] = rel_h
    big_w[3 * halo:3 * halo + 2 * W - 1] = rel_w
    got = oracle.halo_attention(q, k, v, big_h, big_w, block=H, halo=halo)
    want = _dense_global(q, k, v, rel_h, rel_w, heads)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# P3: out-of-image keys get zero weight; the weights sum to one.
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("b,h,stride", [(4, 1, 1), (4, 3, 1), (8, 3, 1), (4, 2, 2)])
def test_p3_weights_sum_to_one_over_in_image_keys(b, h, stride):
    """v = one-hot of the pixel index recovers every query's weights over the
    image.  They must sum to 1 and vanish outside the block's window.  A
    version that zero-padded the border instead of masking it would give
    weight to padding keys (v = 0 there) and the in-image sum would fall
    below 1."""
    H = W = 2 * b
    d = H * W
    rng = _rng(4)
    q = _randn(rng, 1, H, W, d)
    k = _randn(rng, 1, H, W, d, scale=0.3)
    w = b + 2 * h
    rel_h = _randn(rng, 2 * w - 1, d, scale=0.1)
    rel_w = _randn(rng, 2 * w - 1, d, scale=0.1)
    v = np.zeros((1, H, W, d), np.float32)
    for y in range(H):
        for x in range(W):
            v[0, y, x, y * W + x] = 1.0
    got = oracle.halo_attention(q, k, v, rel_h, rel_w, b, h, stride)
    OH, OW = H // stride, W // stride
    for oy in range(OH):
        for ox in range(OW):
            wts = got[0, oy, ox].reshape(H, W)
            assert abs(wts.sum() - 1.0) < 1e-12
            y, x = stride * oy, stride * ox
            by, bx = y // b, x // b
            mask = np.zeros((H, W), bool)
            mask[max(0, by * b - h):min(H, by * b + b + h), max(0, bx * b - h):min(W, bx * b + b + h)] = True
            assert np.all(wts[~mask] == 0.0)
            assert np.all(wts[mask] > 0.0)


def test_p3_values_outside_window_never_read():
    """Changing every pixel outside a block's window (even to NaN) leaves that
    block's outputs unchanged (locality of the haloed neighbourhood)."""
    rng = _rng(5)
    b, h, H, W, d = 4, 1, 16, 16, 8
    q, k, v = (_randn(rng, 1, H, W, d) for _ in range(3))
    w = b + 2 * h
    rel_h, rel_w = _randn(rng, 2 * w - 1, d), _randn(rng, 2 * w - 1, d)
    base = oracle.halo_attention(q, k, v, rel_h, rel_w, b, h)
    by, bx = 1, 2
    k2, v2 = k.copy(), v.copy()
    keep = np.zeros((H, W), bool)
    keep[by * b - h:by * b + b + h, bx * b - h:bx * b + b + h] = True
    k2[0][~keep] = np.nan
    v2[0][~keep] = np.nan
    got = oracle.halo_attention(q, k2, v2, rel_h, rel_w, b, h)
    np.testing.assert_array_equal(got[0, by * b:by * b + b, bx * b:bx * b + b],
                                  base[0, by * b:by * b + b, bx * b:bx * b + b])


# ----------------------------------------------------------------------------
# P4: convex combination and closed forms.
# ----------------------------------------------------------------------------

def _window_pixels(H, W, b, h, y, x):
    by, bx = y // b, x // b
    ys = range(max(0, by * b - h), min(H, by * b + b + h))
    xs = range(max(0, bx * b - h), min(W, bx * b + b + h))
    return ys, xs


@pytest.mark.parametrize("stride", [1, 2])
def test_p4_convex_combination_and_closed_forms(stride):
    rng = _rng(6)
    b, h, H, W, heads, d = 4, 2, 12, 8, 2, 4
    C = heads * d
    q, k, v = (_randn(rng, 1, H, W, C) for _ in range(3))
    w = b + 2 * h
    rel_h, rel_w = _randn(rng, 2 * w - 1, d), _randn(rng, 2 * w - 1, d)
    out = oracle.halo_attention(q, k, v, rel_h, rel_w, b, h, stride)
    for oy in range(H // stride):
        for ox in range(W // stride):
            ys, xs = _window_pixels(H, W, b, h, stride * oy, stride * ox)
            win = v[0, ys.start:ys.stop, xs.start:xs.stop].reshape(-1, C)
            assert np.all(out[0, oy, ox] >= win.min(axis=0) - 1e-12)
            assert np.all(out[0, oy, ox] <= win.max(axis=0) + 1e-12)
    # constant v -> out = v exactly
    vc = np.full_like(v, 0.375)
    out_c = oracle.halo_attention(q, k, vc, rel_h, rel_w, b, h, stride)
    np.testing.assert_allclose(out_c, 0.375, rtol=0, atol=1e-14)
    # q = 0 -> uniform weights -> mean of v over the in-image window
    q0 = np.zeros_like(q)
    out_0 = oracle.halo_attention(q0, k, v, rel_h, rel_w, b, h, stride)
    for oy in range(H // stride):
        for ox in range(W // stride):
            ys, xs = _window_pixels(H, W, b, h, stride * oy, stride * ox)
            mean = v[0, ys.start:ys.stop, xs.start:xs.stop].reshape(-1, C).astype(np.float64).mean(axis=0)
            np.testing.assert_allclose(out_0[0, oy, ox], mean, rtol=0, atol=1e-12)


def _load_golden():
    cases = []
    with open(os.path.join(GOLDEN, "fig1_uniform.txt")) as f:
        for line in f:
            line = line.strip()
            if not line.startswith("case"):
                continue
            head, vals = line.split("|")
            _, name, b, h, s = head.split()
            cases.append((name, int(b), int(h), int(s), [float(t) for t in vals.split()]))
    return cases


@pytest.mark.parametrize("case", _load_golden(), ids=lambda c: c[0])
def test_golden_figure1_uniform_average(case):
    name, b, h, s, want = case
    rng = _rng(8)
    H = W = 4
    q = np.zeros((1, H, W, 1), np.float32)
    k = _randn(rng, 1, H, W, 1)
    v = np.arange(16, dtype=np.float32).reshape(1, H, W, 1)
    w = b + 2 * h
    rel_h, rel_w = _randn(rng, 2 * w - 1, 1), _randn(rng, 2 * w - 1, 1)
    got = oracle.halo_attention(q, k, v, rel_h, rel_w, b, h, s)
    np.testing.assert_allclose(got.reshape(-1), np.array(want), rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# P5: one-hot routing (softmax saturates on the dominant key).
# ----------------------------------------------------------------------------

def test_p5_dominant_key_routes_its_value():
    rng = _rng(9)
    b, h, H, W, d = 4, 1, 8, 8, 8
    q, k, v = (_randn(rng, 1, H, W, d, scale=0.1) for _ in range(3))
    w = b + 2 * h
    rel_h, rel_w = _randn(rng, 2 * w - 1, d, scale=0.01), _randn(rng, 2 * w - 1, d, scale=0.01)
    y, x = 5, 2                # query pixel (block (1, 0))
    Y, X = 3, 4                # a key inside its window (rows 3..8, cols -1..4)
    q[0, y, x] = 1.0
    k[0, Y, X] = 200.0         # logit ~ 200 / sqrt(8) above all others
    got = oracle.halo_attention_samples(q, k, v, rel_h, rel_w, [(0, y, x)], b, h)
    np.testing.assert_allclose(got[0], v[0, Y, X].astype(np.float64), rtol=0, atol=1e-6)


# ----------------------------------------------------------------------------
# P6: stride 2 = stride 1 subsampled (section 2.2, Figure 2: same neighbourhood).
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("b,h", [(4, 1), (8, 3), (2, 0)])
def test_p6_stride2_subsamples_stride1(b, h):
    rng = _rng(10)
    H, W, heads, d = 2 * b, 3 * b, 2, 4
    C = heads * d
    q, k, v = (_randn(rng, 1, H, W, C) for _ in range(3))
    w = b + 2 * h
    rel_h, rel_w = _randn(rng, 2 * w - 1, d), _randn(rng, 2 * w - 1, d)
    s1 = oracle.halo_attention(q, k, v, rel_h, rel_w, b, h, 1)
    s2 = oracle.halo_attention(q, k, v, rel_h, rel_w, b, h, 2)
    np.testing.assert_array_equal(s2, s1[:, ::2, ::2])


# ----------------------------------------------------------------------------
# P7: equivariance only to shifts by b (section 2.2).
# ----------------------------------------------------------------------------

def test_p7_shift_by_block_equivariance():
    rng = _rng(11)
    b, h, H, W, d = 4, 1, 16, 20, 4
    q, k, v = (_randn(rng, 1, H, W, d) for _ in range(3))
    w = b + 2 * h
    rel_h, rel_w = _randn(rng, 2 * w - 1, d), _randn(rng, 2 * w - 1, d)
    base = oracle.halo_attention(q, k, v, rel_h, rel_w, b, h)

    def shifted(s):
        out = []
        for t in (q, k, v):
            u = np.zeros_like(t)
            u[:, :, s:] = t[:, :, :W - s]
            out.append(u)
        return out

    # shift right by b: interior blocks (windows inside both images) move by b
    qs, ks, vs = shifted(b)
    got = oracle.halo_attention(qs, ks, vs, rel_h, rel_w, b, h)
    for by in range(1, H // b - 1):
        for bx in range(1, W // b - 2):
            np.testing.assert_array_equal(got[0, by * b:by * b + b, (bx + 1) * b:(bx + 2) * b],
                                          base[0, by * b:by * b + b, bx * b:bx * b + b])
    # shift by one pixel: block membership changes, outputs do not simply move
    qs, ks, vs = shifted(1)
    got1 = oracle.halo_attention(qs, ks, vs, rel_h, rel_w, b, h)
    diff = np.abs(got1[0, b:2 * b, 1 + b:1 + 2 * b] - base[0, b:2 * b, b:2 * b]).max()
    assert diff > 1e-3


# ----------------------------------------------------------------------------
# P8: appendix A's half-channel factorisation is the zeroed-halves special case.
# ----------------------------------------------------------------------------

def test_p8_half_channel_factorisation():
    """Appendix A splits a head's channels: the first half meets a height
    embedding, the second half a width embedding.  With rel_h zero on the
    second half and rel_w zero on the first, the summed-table reading must
    give exactly that, computed here by dense numpy products."""
    rng = _rng(12)
    H = W = 6
    heads, d = 1, 8
    q, k, v = (_randn(rng, 1, H, W, d) for _ in range(3))
    eh = _randn(rng, 2 * H - 1, d // 2)   # height embedding (d/2 channels)
    ew = _randn(rng, 2 * W - 1, d // 2)   # width embedding (d/2 channels)
    rel_h = np.concatenate([eh, np.zeros_like(eh)], axis=1)
    rel_w = np.concatenate([np.zeros_like(ew), ew], axis=1)
    got = oracle.halo_attention(q, k, v, rel_h, rel_w, block=H, halo=0)
    Q = q[0].reshape(-1, d).astype(np.float64)
    K = k[0].reshape(-1, d).astype(np.float64)
    V = v[0].reshape(-1, d).astype(np.float64)
    B = np.zeros((H * W, H * W))
    for i in range(H * W):
        yi, xi = divmod(i, W)
        for j in range(H * W):
            yj, xj = divmod(j, W)
            B[i, j] = Q[i, :d // 2] @ eh[yj - yi + H - 1] + Q[i, d // 2:] @ ew[xj - xi + W - 1]
    Z = (Q @ K.T + B) / math.sqrt(d)
    P = np.exp(Z - Z.max(axis=1, keepdims=True))
    P /= P.sum(axis=1, keepdims=True)
    np.testing.assert_allclose(got[0].reshape(-1, d), P @ V, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# P9: a second, naive pure-Python implementation at tiny sizes.
# ----------------------------------------------------------------------------

def _naive(q, k, v, rel_h, rel_w, b, h, S, heads):
    _, H, W, C = q.shape
    d = C // heads
    w = b + 2 * h
    out = np.zeros((1, H // S, W // S, C))
    for hd in range(heads):
        for oy in range(H // S):
            for ox in range(W // S):
                y, x = S * oy, S * ox
                top, left = (y // b) * b - h, (x // b) * b - h
                logits, vals = [], []
                for Y in range(top, top + w):
                    for X in range(left, left + w):
                        if not (0 <= Y < H and 0 <= X < W):
                            continue
                        rh = rel_h[(Y - top) - (y - (y // b) * b) + w - 1]
                        rw = rel_w[(X - left) - (x - (x // b) * b) + w - 1]
                        qq = q[0, y, x, hd * d:(hd + 1) * d]
                        logits.append(sum(float(qq[e]) * (float(k[0, Y, X, hd * d + e]) + float(rh[e]) + float(rw[e]))
                                          for e in range(d)) / math.sqrt(d))
                        vals.append(v[0, Y, X, hd * d:(hd + 1) * d].astype(np.float64))
                mx = max(logits)
                ws = [math.exp(z - mx) for z in logits]
                tot = sum(ws)
                out[0, oy, ox, hd * d:(hd + 1) * d] = sum(wt * vv for wt, vv in zip(ws, vals)) / tot
    return out


@pytest.mark.parametrize("b,h,S", [(4, 1, 1), (2, 1, 2), (4, 0, 1), (2, 3, 1)])
def test_p9_naive_python_agrees(b, h, S):
    rng = _rng(13)
    H, W, heads, d = 8, 4, 2, 3
    q, k, v = (_randn(rng, 1, H, W, heads * d) for _ in range(3))
    w = b + 2 * h
    rel_h, rel_w = _randn(rng, 2 * w - 1, d), _randn(rng, 2 * w - 1, d)
    got = oracle.halo_attention(q, k, v, rel_h, rel_w, b, h, S)
    want = _naive(q, k, v, rel_h, rel_w, b, h, S, heads)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


# ----------------------------------------------------------------------------
# bf16 inputs are widened exactly; argument validation.
# ----------------------------------------------------------------------------

def test_bf16_inputs_widen_exactly():
    import torch
    rng = _rng(14)
    b, h, H, W, heads, d = 4, 1, 8, 8, 2, 8
    tensors = [torch.from_numpy(_randn(rng, 1, H, W, heads * d)) for _ in range(3)]
    w = b + 2 * h
    tensors += [torch.from_numpy(_randn(rng, 2 * w - 1, d)) for _ in range(2)]
    bf = [t.to(torch.bfloat16) for t in tensors]
    widened = [t.to(torch.float32) for t in bf]
    a = oracle.halo_attention(*bf, block=b, halo=h)
    c = oracle.halo_attention(*widened, block=b, halo=h)
    np.testing.assert_array_equal(a, c)


def test_oracle_rejects_bad_arguments():
    z = np.zeros((1, 6, 6, 4), np.float32)
    r = np.zeros((7, 4), np.float32)
    with pytest.raises(ValueError):
        oracle.halo_attention(z, z, z, r, r, block=4, halo=0)  # 6 % 4 != 0
    with pytest.raises(ValueError):
        oracle.halo_attention(z, z, z, r, r, block=2, halo=1, stride=3)
