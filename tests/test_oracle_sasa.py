"""Pins for the oracle's SASA-masked variant (HaloNet paper, section 2.2, the
paragraph after Figure 1: SASA uses the same blocking with halo
h = floor(k/2) and an attention mask that emulates a k x k pixel-centred
window, which makes the op translation-equivariant because every pixel only
looks at the square around it).

Pins, none of them the masked formula retyped:
  * k = 1 keeps only the query's own pixel: out = v exactly;
  * pixel-wise neighbourhood extraction is blocked attention with block size
    1 (section 2.2, first paragraph of the blocked local self-attention
    part): the masked op with k = 2h + 1 at any block size equals the
    unmasked op at block 1, with the tables shifted by the change of window;
  * the result does not depend on the block size beyond that table shift;
  * shifting the image by one pixel shifts the output by one pixel wherever
    the k x k neighbourhoods stay inside the image (the unmasked op is only
    equivariant to shifts by the block size);
  * a naive pure-Python pixel-centred implementation at tiny sizes.
"""
import math

import numpy as np
import pytest

import oracle


def _rng(seed):
    return np.random.default_rng(seed)


def _randn(rng, *shape, scale=1.0):
    return (rng.standard_normal(shape) * scale).astype(np.float32)


def _qkv(seed, N, H, W, C):
    rng = _rng(seed)
    return [_randn(rng, N, H, W, C) for _ in range(3)]


def _tables(seed, rows, d, scale=0.5):
    rng = _rng(seed)
    return _randn(rng, rows, d, scale=scale), _randn(rng, rows, d, scale=scale)


def _shifted(table, offset, rows):
    """Rows [offset, offset + len) of a larger table of `rows` rows hold
    `table`; the rest is filled with large values no kept key reads."""
    big = np.full((rows, table.shape[1]), 50.0, np.float32)
    big[offset:offset + table.shape[0]] = table
    return big


def test_kernel_one_returns_the_query_pixels_value():
    q, k, v = _qkv(40, 2, 8, 8, 6)
    rh, rw = _tables(41, 2 * (4 + 2) - 1, 3)
    out = oracle.halo_attention_masked(q, k, v, rh, rw, block=4, halo=1, kernel=1)
    np.testing.assert_array_equal(out, v.astype(np.float64))


@pytest.mark.parametrize("b,h", [(4, 1), (4, 2), (8, 3), (2, 1)])
def test_masked_equals_pixelwise_blocks(b, h):
    """k = 2h + 1 at block b equals the unmasked op at block 1 and halo h.
    Key at offset (dy, dx) from the query: block-1 table row dy + 3h, block-b
    table row dy + b + 3h - 1, so the block-b tables are the block-1 tables
    shifted down by b - 1 rows."""
    H, W, heads, d = 8, 8, 2, 3
    q, k, v = _qkv(42, 1, H, W, heads * d)
    w1 = 1 + 2 * h
    rh1, rw1 = _tables(43, 2 * w1 - 1, d)
    want = oracle.halo_attention(q, k, v, rh1, rw1, block=1, halo=h)
    wb = b + 2 * h
    rhb, rwb = _shifted(rh1, b - 1, 2 * wb - 1), _shifted(rw1, b - 1, 2 * wb - 1)
    got = oracle.halo_attention_masked(q, k, v, rhb, rwb, block=b, halo=h, kernel=2 * h + 1)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("kernel", [3, 5])
def test_masked_result_does_not_depend_on_block_size(kernel):
    H, W, heads, d, h = 16, 16, 1, 4, 2
    q, k, v = _qkv(44, 1, H, W, heads * d)
    base_h, base_w = _tables(45, 2 * h + 1, d)  # rows for offsets -h..h
    outs = []
    for b in (2, 4, 8):
        w = b + 2 * h
        off = b + 2 * h - 1  # table row of offset -h: (-h) + b + 3h - 1
        outs.append(oracle.halo_attention_masked(q, k, v, _shifted(base_h, off, 2 * w - 1),
                                                 _shifted(base_w, off, 2 * w - 1), block=b, halo=h,
                                                 kernel=kernel))
    np.testing.assert_allclose(outs[1], outs[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(outs[2], outs[0], rtol=0, atol=1e-12)


def test_masked_is_equivariant_to_one_pixel_shifts():
    """Shift the inputs by (1, 1): interior outputs shift by (1, 1).  The
    unmasked op (same inputs) is not equivariant to this shift."""
    H = W = 16
    b, h, kernel, d = 4, 2, 5, 4
    q, k, v = _qkv(46, 1, H + 1, W + 1, d)
    rh, rw = _tables(47, 2 * (b + 2 * h) - 1, d)
    a = [t[:, :H, :W].copy() for t in (q, k, v)]
    s = [t[:, 1:, 1:].copy() for t in (q, k, v)]  # the image moved up-left by one pixel
    oa = oracle.halo_attention_masked(*a, rh, rw, block=b, halo=h, kernel=kernel)
    os_ = oracle.halo_attention_masked(*s, rh, rw, block=b, halo=h, kernel=kernel)
    r = kernel // 2
    inner_a = oa[:, 1 + r:H - r, 1 + r:W - r]
    inner_s = os_[:, r:H - r - 1, r:W - r - 1]
    np.testing.assert_allclose(inner_s, inner_a, rtol=0, atol=1e-12)
    ua = oracle.halo_attention(*a, rh, rw, block=b, halo=h)
    us = oracle.halo_attention(*s, rh, rw, block=b, halo=h)
    assert np.abs(us[:, r:H - r - 1, r:W - r - 1] - ua[:, 1 + r:H - r, 1 + r:W - r]).max() > 1e-3


def _naive_centred(q, k, v, rel_h, rel_w, b, h, kernel, S):
    """Pixel-centred k x k attention written directly: key (Y, X) with
    |Y - y|, |X - x| <= k // 2 inside the image, relative rows indexed by the
    offset plus the blocked window's constant b + 3h - 1."""
    _, H, W, C = q.shape
    d = rel_h.shape[1]
    heads = C // d
    r = kernel // 2
    base = b + 3 * h - 1
    out = np.zeros((1, H // S, W // S, C))
    for hd in range(heads):
        sl = slice(hd * d, (hd + 1) * d)
        for oy in range(H // S):
            for ox in range(W // S):
                y, x = S * oy, S * ox
                zs, vs = [], []
                for dy in range(-r, r + 1):
                    for dx in range(-r, r + 1):
                        Y, X = y + dy, x + dx
                        if not (0 <= Y < H and 0 <= X < W):
                            continue
                        qq = q[0, y, x, sl].astype(np.float64)
                        kk = k[0, Y, X, sl].astype(np.float64) + rel_h[dy + base] + rel_w[dx + base]
                        zs.append(float(qq @ kk) / math.sqrt(d))
                        vs.append(v[0, Y, X, sl].astype(np.float64))
                m = max(zs)
                ws = [math.exp(z - m) for z in zs]
                out[0, oy, ox, sl] = sum(wt * vv for wt, vv in zip(ws, vs)) / sum(ws)
    return out


@pytest.mark.parametrize("b,h,kernel,S", [(4, 1, 3, 1), (4, 2, 3, 1), (2, 2, 5, 2), (4, 3, 7, 1)])
def test_naive_centred_agrees(b, h, kernel, S):
    H, W, heads, d = 8, 8, 2, 3
    q, k, v = _qkv(48, 1, H, W, heads * d)
    rh, rw = _tables(49, 2 * (b + 2 * h) - 1, d)
    got = oracle.halo_attention_masked(q, k, v, rh, rw, block=b, halo=h, kernel=kernel, stride=S)
    want = _naive_centred(q, k, v, rh.astype(np.float64), rw.astype(np.float64), b, h, kernel, S)
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-12)


def test_masked_rejects_bad_kernels():
    q, k, v = _qkv(50, 1, 8, 8, 4)
    rh, rw = _tables(51, 2 * 6 - 1, 4)
    for kern in (0, 2, 5):  # not positive, even, larger than 2h + 1
        with pytest.raises(ValueError):
            oracle.halo_attention_masked(q, k, v, rh, rw, block=4, halo=1, kernel=kern)
