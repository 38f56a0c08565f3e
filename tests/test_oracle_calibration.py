"""Pins of the oracle's per-layer error and full-precision layer selection
(page 1 of the TMAP write-up, "Attention performance optimisation / Keeping
video quality": the attention error of every layer at every denoising
iteration decides which layers keep the original precision).

The relative L2 error is pinned by closed forms on bf16 data whose scaling is
exact (a = 2b gives 1, a = b/2 gives 1/2, a = 0 gives 1, a = b gives 0), the
zero-denominator cases, the independent fp64 norm on random data, and
invariance under a common exact scaling; the selection by a hand-built table
whose two rules give different answers."""
import math

import numpy as np
import pytest

import oracle


def _bf16(x):
    """fp32 values exactly representable in bf16 -> uint16 bits."""
    x = np.asarray(x, np.float32)
    bits = x.view(np.uint32)
    assert np.all(bits & 0xFFFF == 0)
    return (bits >> 16).astype(np.uint16)


def _rand_bf16(n, seed):
    r = np.random.default_rng(seed).standard_normal(n).astype(np.float32)
    return _bf16((r.view(np.uint32) & 0xFFFF0000).view(np.float32))


def test_rel_l2_closed_forms():
    b = _rand_bf16(5000, 1)
    bf = (b.astype(np.uint32) << 16).view(np.float32)
    assert oracle.rel_l2(b, b) == 0.0
    assert oracle.rel_l2(_bf16(2 * bf), b) == 1.0          # |a - b| = |b|
    assert oracle.rel_l2(_bf16(bf / 2), b) == 0.5
    assert oracle.rel_l2(_bf16(-bf), b) == 2.0
    assert oracle.rel_l2(np.zeros_like(b), b) == 1.0
    # (3b)^2 sums round differently from 9 * sum b^2: equal to fp64 rounding
    assert math.isclose(oracle.rel_l2(_bf16(4 * bf), b), 3.0, rel_tol=1e-14)


def test_rel_l2_zero_denominator():
    z = np.zeros(64, np.uint16)
    assert oracle.rel_l2(z, z) == 0.0
    assert math.isinf(oracle.rel_l2(_rand_bf16(64, 2), z))


def test_rel_l2_against_an_independent_norm():
    a, b = _rand_bf16(100000, 3), _rand_bf16(100000, 4)
    af = (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    bf = (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    want = np.linalg.norm(af - bf) / np.linalg.norm(bf)
    assert abs(oracle.rel_l2(a, b) - want) <= 1e-12 * want
    # symmetric error terms, asymmetric denominator
    assert abs(oracle.rel_l2(b, a) - np.linalg.norm(af - bf) / np.linalg.norm(af)) <= 1e-12 * want


def test_rel_l2_is_invariant_under_a_common_power_of_two_scale():
    a, b = _rand_bf16(4096, 5), _rand_bf16(4096, 6)
    f = lambda x: (x.astype(np.uint32) << 16).view(np.float32)
    assert oracle.rel_l2(_bf16(f(a) * 8), _bf16(f(b) * 8)) == oracle.rel_l2(a, b)


def test_select_layers_hand_table():
    err = [[0.10, 0.40],      # mean 0.25 > 0.2, but not above 0.2 at every iteration
           [0.25, 0.22],      # above 0.2 at every iteration
           [0.05, 0.06],      # never
           [0.21, 0.20]]      # 0.20 is not above 0.2
    assert oracle.select_layers(err, 0.2, oracle.SELECT_EVERY_ITERATION) == [1]
    assert oracle.select_layers(err, 0.2, oracle.SELECT_MEAN) == [0, 1, 3]
    assert oracle.select_layers(err, 0.0, oracle.SELECT_EVERY_ITERATION) == [0, 1, 2, 3]
    assert oracle.select_layers(err, 0.5, oracle.SELECT_MEAN) == []
    # one iteration: the two rules agree
    one = [[0.3], [0.1]]
    assert oracle.select_layers(one, 0.2, 0) == oracle.select_layers(one, 0.2, 1) == [0]


def test_select_layers_rejects_bad_input():
    with pytest.raises(ValueError):
        oracle.select_layers([[float("nan")]], 0.1)
    with pytest.raises(ValueError):
        oracle.select_layers([[0.1]], 0.1, rule=7)
    with pytest.raises(ValueError):
        oracle.select_layers([0.1, 0.2], 0.1)
