"""Error bound of the FMA-pipe 2^x the attention softmax uses for one pair in
eight (csrc/common.cuh, exp2_poly2).

The kernel splits x = j + f with j = round(x) (adding and subtracting
1.5 * 2^23 in fp32), evaluates 2^f with a degree-4 polynomial by Horner
steps, and adds j into the exponent field.  This test reads the constants
from the source, replays the same fp32 operations in numpy (each add and
fused multiply-add rounded once to fp32), and checks the result against
exact 2^x in fp64 over the range the softmax feeds it: x <= 8 (the lazily
updated row max lets scores exceed it by at most 2^8) down to the clamp.
P is rounded to bf16 (relative step 2^-8) right after; the bound asked
here, 1e-5, keeps the rounding of P almost always that of the exact value.
"""
import os
import re

import numpy as np

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "block_sparse_long_07_b200", "csrc", "common.cuh")


def _constants():
    text = open(SRC).read()
    body = text[text.index("void exp2_poly2("):]
    body = body[:body.index("\n}\n")]
    nums = [float(x) for x in re.findall(r"(-?\d+\.\d*)f\b", body)]
    # clamp x2, rounding constant x2, its negation x2, then c4 c4 c3 c3 c2 c2 c1 c1 c0 c0
    assert len(nums) == 16, nums
    clamp, magic = nums[0], nums[2]
    c4, c3, c2, c1, c0 = nums[6], nums[8], nums[10], nums[12], nums[14]
    assert nums[4] == -magic
    return clamp, magic, (c4, c3, c2, c1, c0)


def _f32(x):
    return np.asarray(x, dtype=np.float64).astype(np.float32)


def _fma32(a, b, c):
    # one rounding: the fp64 product of two fp32 values is exact
    return _f32(np.asarray(a, np.float64) * np.asarray(b, np.float64) + np.asarray(c, np.float64))


def exp2_poly_np(x):
    clamp, magic, (c4, c3, c2, c1, c0) = _constants()
    x = np.maximum(_f32(x), np.float32(clamp))
    t = _f32(x.astype(np.float64) + magic)
    j = _f32(t.astype(np.float64) - magic)
    f = _f32(x.astype(np.float64) - j.astype(np.float64))
    p = _fma32(np.float32(c4), f, np.float32(c3))
    p = _fma32(p, f, np.float32(c2))
    p = _fma32(p, f, np.float32(c1))
    p = _fma32(p, f, np.float32(c0))
    bits = p.view(np.int32).astype(np.int64) + (t.view(np.int32).astype(np.int64) << 23)
    return (bits & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def test_constants_are_the_fitted_ones():
    clamp, magic, coef = _constants()
    assert clamp == -126.0 and magic == 1.5 * 2.0 ** 23
    # 2^f near f = 0 is 1 + f ln 2 + ...: the fit must be close to the Taylor terms
    c4, c3, c2, c1, c0 = coef
    assert abs(c0 - 1.0) < 1e-5 and abs(c1 - np.log(2)) < 1e-4
    assert abs(c2 - np.log(2) ** 2 / 2) < 1e-3 and abs(c3 - np.log(2) ** 3 / 6) < 1e-3
    assert abs(c4 - np.log(2) ** 4 / 24) < 1e-3


def test_relative_error_bound():
    x = np.linspace(-125.0, 8.0, 2_000_001).astype(np.float32)
    got = exp2_poly_np(x).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < 1e-5, rel.max()


def test_integer_points_and_rounding_ties():
    for k in range(-120, 9):
        for dx in (0.0, 0.5, -0.5, 0.4999999, -0.4999999):
            x = np.array([k + dx], np.float32)
            v = float(exp2_poly_np(x)[0])
            assert abs(v / 2.0 ** float(x[0]) - 1.0) < 1e-5, (k, dx)


def test_below_the_clamp_stays_tiny_and_finite():
    v = exp2_poly_np(np.array([-1e4, -300.0, -126.5, -np.inf], np.float32))
    assert np.all(np.isfinite(v)) and np.all(v >= 0) and np.all(v < 2.0 ** -125)


def _minimax_fit(deg, npts=4001):
    """Coefficients c0..c_deg minimising max |p(f) / 2^f - 1| over npts
    equispaced points of [-1/2, 1/2], as a linear program in (c, t):
    minimise t subject to -t <= p(f_i) / 2^f_i - 1 <= t."""
    from scipy.optimize import linprog
    f = np.linspace(-0.5, 0.5, npts)
    y = 2.0 ** f
    V = np.vstack([f ** k for k in range(deg + 1)]).T / y[:, None]
    n = deg + 1
    ones = np.ones((len(f), 1))
    A = np.vstack([np.hstack([V, -ones]), np.hstack([-V, -ones])])
    b = np.concatenate([np.ones(len(f)), -np.ones(len(f))])
    cost = np.zeros(n + 1)
    cost[-1] = 1.0
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * (n + 1), method="highs")
    assert res.success
    return res.x[:n], res.x[-1]


def test_constants_come_from_the_minimax_fit():
    """Refit the degree-4 polynomial and compare with the source's constants
    (rounded to fp32), so the derivation of the constants is reproducible."""
    _, _, (c4, c3, c2, c1, c0) = _constants()
    coef, err = _minimax_fit(4)
    assert err < 2.7e-6
    got = np.array([c0, c1, c2, c3, c4], np.float64)
    assert np.allclose(got, coef.astype(np.float32).astype(np.float64), rtol=0, atol=2e-7), \
        (got, coef)
