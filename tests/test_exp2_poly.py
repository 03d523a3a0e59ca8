"""Host check of the FMA-pipe exponential the forward and dK/dV kernels use
for half of their softmax terms (ptx::exp2_poly in csrc/ptx.cuh): the same
steps in fp32 (range reduction by the 1.5 * 2^23 rounding constant, the cubic
read from the header, 2^n added to the exponent field) against numpy's exp2 in
fp64.  Pins the error bound stated beside the coefficients and the exact
zero for masked scores."""
import os
import re

import numpy as np

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "branch_attention_speculative_packed_b200", "csrc", "ptx.cuh")


def _coefficients():
    src = open(HDR).read()
    body = src[src.index("float2 exp2_poly(float2 x)"):]
    body = body[:body.index("\n}\n")]
    nums = [float(v) for v in re.findall(r"make_float2\(([0-9.e+-]+)f,", body)]
    # make_float2 constants in order: 1.5*2^23, c3, c2, c1, 1
    big, c3, c2, c1, one = nums
    assert big == 12582912.0 and one == 1.0
    return np.float32(c1), np.float32(c2), np.float32(c3)


def _fma(a, b, c):  # one rounding, as fma.rn.f32 (the fp32 product is exact in fp64)
    return (a.astype(np.float64) * b + c).astype(np.float32)


def exp2_poly(x):
    c1, c2, c3 = _coefficients()
    x = np.maximum(np.asarray(x, np.float32), np.float32(-127.0))
    big = np.float32(12582912.0)
    t = (x + big).astype(np.float32)
    f = (x - (t - big)).astype(np.float32)
    p = _fma(np.full_like(f, c3), f, np.full_like(f, c2))
    p = _fma(p, f, np.full_like(f, c1))
    p = _fma(p, f, np.full_like(f, np.float32(1.0)))
    bits = p.view(np.uint32) + (t.view(np.uint32) << np.uint32(23))
    return bits.view(np.float32)


def test_relative_error_bound():
    x = np.linspace(-126.0, 8.0, 2_000_001, dtype=np.float64).astype(np.float32)
    got = exp2_poly(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() <= 1.05e-4, rel.max()
    # well below bf16 rounding (2^-9), the precision P is stored in
    assert rel.max() < 2.0 ** -9 / 10


def test_special_values():
    got = exp2_poly(np.array([0.0, 1.0, -1.0, 3.0, -127.0, -np.inf, -1e30], np.float32))
    assert got[0] == 1.0 and got[1] == 2.0 and got[2] == 0.5 and got[3] == 8.0
    assert got[4] == 0.0 and got[5] == 0.0 and got[6] == 0.0  # masked scores give exactly 0


def test_monotone_on_a_fine_grid():
    x = np.linspace(-20.0, 8.0, 400_001, dtype=np.float64).astype(np.float32)
    x = np.unique(x)
    y = exp2_poly(x)
    # the cubic is continuous across integer breakpoints to within its error
    assert np.all(np.diff(y.astype(np.float64)) >= -2e-4 * y[1:])
