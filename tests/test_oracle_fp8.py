"""Pins the oracle's FP8 e4m3 codec to the OCP FP8 definition.

The quantized P.V product of the SageAttention-style path (page 1 of the TMAP
write-up, "Attention performance optimisation") runs in FP8 e4m3; the oracle's
encoder/decoder is checked here against the published special values, against
an exhaustive round trip, against ties-to-even at every midpoint, and against
torch's own float8_e4m3fn cast (a library routine) for in-range values.
"""
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "e4m3_ocp_points.txt")


def _golden():
    pts = []
    for line in open(GOLDEN):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        h, v = line.split()
        pts.append((int(h, 16), float(v)))
    return pts


def test_published_special_values():
    for code, val in _golden():
        got = oracle.e4m3_decode(code)
        if math.isnan(val):
            assert math.isnan(got)
        else:
            assert got == val and math.copysign(1.0, got) == math.copysign(1.0, val), hex(code)
            assert oracle.e4m3_encode(val) == code, hex(code)


def test_decode_monotone_and_symmetric():
    t = oracle.e4m3_decode_table()
    pos = t[:0x7F]                      # 0x00..0x7E, all finite
    assert np.all(np.isfinite(pos))
    assert np.all(np.diff(pos) > 0)
    assert np.array_equal(t[0x80:0xFF], -pos)
    # 8 subnormal steps of 2^-9, then each binade holds 8 values
    assert np.allclose(pos[:8], np.arange(8) * 2.0 ** -9)
    for e in range(1, 16):
        binade = pos[8 * e: 8 * e + 8]
        if len(binade) == 8:
            assert np.allclose(binade, (1 + np.arange(8) / 8) * 2.0 ** (e - 7))


def test_round_trip_every_code():
    t = oracle.e4m3_decode_table()
    for c in range(256):
        if math.isnan(t[c]):
            continue
        assert oracle.e4m3_encode(t[c]) == c, hex(c)


def test_midpoints_round_to_even_and_saturate():
    t = oracle.e4m3_decode_table()[:0x7F]
    for c in range(0x7E):
        mid = (t[c] + t[c + 1]) / 2.0          # exact in fp32 (few significant bits)
        want = c if c % 2 == 0 else c + 1      # even code <=> even mantissa here
        assert oracle.e4m3_encode(np.float32(mid)) == want, hex(c)
        assert oracle.e4m3_encode(np.float32(-mid)) == want | 0x80
        # just off the midpoint goes to the nearer neighbour
        lo = np.nextafter(np.float32(mid), np.float32(0))
        hi = np.nextafter(np.float32(mid), np.float32(1000))
        assert oracle.e4m3_encode(lo) == c and oracle.e4m3_encode(hi) == c + 1
    for x in (448.0, 449.0, 464.0, 1e6, float("inf")):
        assert oracle.e4m3_encode(x) == 0x7E
        assert oracle.e4m3_encode(-x) == 0xFE


def test_matches_torch_float8_cast_in_range():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.uniform(-448, 448, 4000),
        rng.standard_normal(4000) * 0.05,
        rng.standard_normal(2000) * 2.0 ** -8,
    ]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = np.array([oracle.e4m3_encode(v) for v in x], dtype=np.uint8)
    assert np.array_equal(got, ref)
