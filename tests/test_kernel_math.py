"""CPU checks of the arithmetic the tensor-core kernels use in place of
library calls, against its mathematical definition:

* the polynomial 2^x on the FMA pipe (range reduction x = j + f with
  j = floor(x), a cubic for 2^f on [0, 1) fitted with p(0) = 1, and 2^j added
  into the exponent field) must stay within its stated relative error bound
  of 2^x over the whole range the softmax feeds it (x <= 0), with masked
  logits (x = -inf, clamped to -127) giving exactly 0.

The constants are read from the kernel sources, so these tests check the
values the kernels are built with.
"""
import os
import re

import numpy as np

CSRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "blocked_local_self_b200", "csrc")


def _read(name):
    with open(os.path.join(CSRC, name)) as f:
        return f.read()


def _cubic_coefficients():
    """(c3, c2, c1) of p(f) = ((c3 f + c2) f + c1) f + 1 from exp2_poly2 (the
    packed form: both lanes of every constant must agree)."""
    src = _read("halo_tc2.cuh")
    body = src[src.index("void exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    pair = r"make_float2\(([0-9.e+-]+)f, ([0-9.e+-]+)f\)"
    m = re.search(r"__ffma2_rn\(f, " + pair + ", " + pair + r"\)", body)
    c3a, c3b, c2a, c2b = map(float, m.groups())
    m1 = re.search(r"__ffma2_rn\(q, f, " + pair + r"\)", body)
    c1a, c1b = map(float, m1.groups())
    assert (c3a, c2a, c1a) == (c3b, c2b, c1b)
    assert re.search(r"__ffma2_rn\(q, f, make_float2\(1\.0f, 1\.0f\)\)", body)
    return c3a, c2a, c1a


def _f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def _fma32(a, b, c):
    # a*b is exact in float64 for float32 operands; one rounding to float32
    return _f32(a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64))


def _exp2_poly_emulated(x):
    """The kernel's steps in float32: clamp, floor by a round-down add of
    1.5*2^23, fraction, cubic by three FMAs, exponent insertion."""
    c3, c2, c1 = (_f32(c) for c in _cubic_coefficients())
    x = np.maximum(_f32(x), _f32(-127.0))
    j = np.floor(x.astype(np.float64)).astype(np.float32)  # what add.rm with 1.5*2^23 yields, minus the magic
    f = _f32(x.astype(np.float64) - j.astype(np.float64))
    p = _fma32(f, np.full_like(f, c3), np.full_like(f, c2))
    p = _fma32(p, f, np.full_like(f, c1))
    p = _fma32(p, f, np.ones_like(f))
    bits = p.view(np.int32).astype(np.int64) + (j.astype(np.int64) << 23)
    return bits.astype(np.int32).view(np.float32)


def test_cubic_fixes_the_endpoints():
    c3, c2, c1 = _cubic_coefficients()
    # p(0) = 1 exactly by construction; p(1) close to 2 so the pieces join
    assert abs((c3 + c2 + c1 + 1.0) - 2.0) < 2e-4


def test_exp2_poly_relative_error_bound():
    rng = np.random.default_rng(0)
    # dense grid on [-30, 0] plus random points down to -126 (normal range)
    x = np.concatenate([np.linspace(-30.0, 0.0, 2_000_001), -rng.random(200_000) * 126.0]).astype(np.float32)
    got = _exp2_poly_emulated(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(got - want) / want
    assert rel.max() < 1.0e-4, rel.max()
    # far below a bf16 half-ulp (2^-9): the P rounding dominates, not the polynomial
    assert rel.max() < 2.0 ** -9 / 10


def test_exp2_poly_masked_logits_are_exact_zero():
    got = _exp2_poly_emulated(np.array([-np.inf, -1e30, -127.0], dtype=np.float32))
    assert np.all(got == 0.0)


def test_exp2_poly_at_integers_is_exact():
    x = np.arange(-126, 1, dtype=np.float32)
    assert np.array_equal(_exp2_poly_emulated(x), np.exp2(x.astype(np.float64)).astype(np.float32))
