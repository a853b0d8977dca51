"""Host-side checks of the constants of the prefill softmax's exponential on
the FMA pipe (no GPU).

csrc/flint_prefill.cu computes one pair of exponentials in four with
ex2_fma2: 2^x = 2^j 2^f with j = rint(x), taken from the low bits of
x + 1.5 * 2^23, f = x - j in [-1/2, 1/2], and 2^f the degree-4 polynomial
that interpolates 2^f at the five Chebyshev nodes cos((2k+1) pi / 10) / 2 of
the interval; j joins the exponent field by an integer add.  This test
derives the interpolant in float64, checks that the float coefficients in
the source are its values rounded to float, and bounds the error of the
whole method (float32 arithmetic emulated step by step, each fused
multiply-add rounded once) over the range the softmax uses.  The same
function is compared with the hardware's ex2.approx on the GPU in
tests/test_gpu_ex2.py."""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "long_context_decode_flash_b200", "csrc", "flint_prefill.cu")
F32 = np.float32


def chebyshev_interpolant():
    n = 5
    nodes = 0.5 * np.cos((2 * np.arange(n) + 1) * np.pi / (2 * n))
    return np.linalg.solve(np.vander(nodes, n, increasing=True), np.exp2(nodes))


def source_coefficients():
    """c4, c3, c2, c1 in the order the source's Horner steps use them (each
    written twice, once per lane of the pair)."""
    body = open(SRC).read()
    fn = body[body.index("float2 ex2_fma2(float2 x)"):]
    fn = fn[:fn.index("\n}")]
    seen = []
    for h in re.findall(r"0x1\.[0-9a-f]+p-?\d+f", fn):
        v = float.fromhex(h[:-1])
        if v not in seen:
            seen.append(v)
    return seen


def fma32(a, b, c):
    # the exact product of two floats fits a double; one rounding to float after the add
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(F32)


def emulate(x, c4, c3, c2, c1):
    x = np.maximum(x.astype(F32), F32(-127.0))
    t = (x + F32(12582912.0)).astype(F32)
    f = fma32((t + F32(-12582912.0)).astype(F32), np.full_like(x, -1.0), x)
    full = lambda v: np.full_like(f, F32(v))  # noqa: E731
    q = fma32(full(c4), f, full(c3))
    q = fma32(q, f, full(c2))
    q = fma32(q, f, full(c1))
    q = fma32(q, f, full(1.0))
    bits = (q.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(F32)


def test_ex2_coefficients_are_the_chebyshev_interpolant():
    c = chebyshev_interpolant()
    assert abs(c[0] - 1.0) < 1e-12  # the constant term in the source is 1.0 exactly
    assert source_coefficients() == [float(F32(v)) for v in (c[4], c[3], c[2], c[1])]


def test_ex2_fma_error_bound():
    c4, c3, c2, c1 = source_coefficients()
    x = np.linspace(-125.0, 8.0, 4_000_001).astype(F32)
    y = emulate(x, c4, c3, c2, c1).astype(np.float64)
    rel = np.abs(y / np.exp2(x.astype(np.float64)) - 1.0)
    assert rel.max() < 3.6e-6
    special = emulate(np.array([-np.inf, 0.0, 8.0, -127.0]), c4, c3, c2, c1)
    assert list(special) == [0.0, 1.0, 256.0, 0.0]


def test_the_bound_catches_a_wrong_coefficient():
    """A coefficient off in its last bits of significance (a garbled hex
    digit) breaks the bound."""
    c4, c3, c2, c1 = source_coefficients()
    x = np.linspace(-3.0, 3.0, 200_001).astype(F32)
    y = emulate(x, c4, c3, c2 * (1 + 1e-3), c1).astype(np.float64)
    assert np.abs(y / np.exp2(x.astype(np.float64)) - 1.0).max() > 3.6e-6
