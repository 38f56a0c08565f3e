"""The FMA-pipe 2^x of the attention kernels (sm100.cuh, exp2_fma2): 2^x =
2^j * 2^f with j = rne(x) and f in [-1/2, 1/2], 2^f by a degree-3 polynomial.

The polynomial is the minimax (least maximum relative error) cubic for 2^f on
[-1/2, 1/2], found by the Remez exchange algorithm (Remez 1934).  This test
re-derives it independently, checks the constants compiled into the kernels,
and bounds the error of the whole evaluation -- emulated step by step in fp32
with one rounding per fused multiply-add -- against the exact 2^x over the
range the softmax uses (x = s - m + log2 448 <= log2 448, down to the clamp
at -125)."""
import math
import re
from fractions import Fraction

import numpy as np

import os

HDR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "video_dit_quantized_b200", "csrc",
                   "sm100.cuh")


def _constants():
    txt = open(HDR).read()
    vals = {}
    for name in ("kExp2C0", "kExp2C1", "kExp2C2", "kExp2C3"):
        m = re.search(name + r"\s*=\s*([0-9.eE+-]+)f", txt)
        assert m, name
        vals[name] = float(np.float32(float(m.group(1))))
    return [vals["kExp2C0"], vals["kExp2C1"], vals["kExp2C2"], vals["kExp2C3"]]


def _remez_exp2(deg, iters=40):
    """Minimax polynomial for 2^f on [-1/2, 1/2] in relative error (Remez exchange, fp64)."""
    a, b = -0.5, 0.5
    n = deg
    k = np.arange(n + 2)
    x = 0.5 * (a + b) + 0.5 * (b - a) * np.cos(np.pi * (n + 1 - k) / (n + 1))
    grid = np.linspace(a, b, 100001)
    for _ in range(iters):
        A = np.zeros((n + 2, n + 2))
        for i in range(n + 2):
            A[i, :n + 1] = x[i] ** np.arange(n + 1)
            A[i, n + 1] = (-1) ** i * 2.0 ** x[i]
        sol = np.linalg.solve(A, 2.0 ** x)
        c = sol[:n + 1]
        err = np.polyval(c[::-1], grid) / 2.0 ** grid - 1
        sign = np.sign(err)
        bounds = [0] + list(np.where(np.diff(sign) != 0)[0] + 1) + [len(grid)]
        ext = [lo + int(np.argmax(np.abs(err[lo:hi]))) for lo, hi in zip(bounds[:-1], bounds[1:])]
        if len(ext) == n + 2:
            x = grid[ext]
    return c, float(np.abs(err).max())


def _f32(v):
    return np.float32(v)


def _fma32(a, b, c):
    """fp32 fused multiply-add: the exact a*b + c rounded once to fp32."""
    exact = Fraction(float(a)) * Fraction(float(b)) + Fraction(float(c))
    return np.float32(float(exact)) if abs(exact) < 2 ** 127 else np.float32(math.inf)


def _exp2_fma(x):
    """Step-by-step fp32 emulation of exp2_fma2 for one lane."""
    c0, c1, c2, c3 = (_f32(v) for v in _constants())
    x = np.float32(max(np.float32(x), np.float32(-125.0)))
    M = np.float32(12582912.0)
    t = np.float32(x + M)                       # rounds to the nearest integer offset
    jf = np.float32(t - M)                      # exact
    f = np.float32(x - jf)                      # exact
    p = _fma32(f, c3, c2)
    p = _fma32(p, f, c1)
    p = _fma32(p, f, c0)
    bits = (int(np.array(p, np.float32).view(np.uint32)) + ((int(np.array(t, np.float32).view(np.uint32)) << 23) & 0xFFFFFFFF)) & 0xFFFFFFFF
    return float(np.array(bits, np.uint32).view(np.float32))


def test_constants_are_the_minimax_cubic():
    c, e = _remez_exp2(3)
    got = _constants()
    for g, w in zip(got, c):
        assert abs(g - w) <= 2e-7 * max(1.0, abs(w)), (got, c.tolist())
    assert 7.0e-5 < e < 8.0e-5          # the equioscillation level of the cubic


def test_relative_error_bound_over_the_softmax_range():
    rng = np.random.default_rng(7)
    xs = np.concatenate([np.linspace(-125.0, 8.807354922057604, 4001), rng.uniform(-30, 8.8, 2000),
                         np.arange(-20, 9, 0.5), np.arange(-20, 9) + 0.5 - 1e-6])
    worst = 0.0
    for x in xs.astype(np.float32):
        got = _exp2_fma(x)
        want = 2.0 ** float(x)
        worst = max(worst, abs(got / want - 1.0))
    # the cubic's 7.48e-5 plus a few fp32 roundings
    assert worst <= 7.6e-5, worst


def test_exact_at_integer_arguments_up_to_the_polynomial_value_at_zero():
    c0 = _constants()[0]
    for j in range(-120, 9):
        assert _exp2_fma(np.float32(j)) == float(np.float32(c0)) * 2.0 ** j


def test_clamp_keeps_the_result_a_tiny_normal_number():
    for x in (-126.0, -200.0, -1e4):
        got = _exp2_fma(np.float32(x))
        assert 0 < got < 2.0 ** -124
        assert math.isfinite(got)
