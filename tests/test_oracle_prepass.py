"""Pins the oracle's quantization prepass (K mean, K smoothing, per-block INT8
for Q and K, per-channel FP8 for V) to exact arithmetic and to the properties
the scheme must have.

Method: page 1 of the TMAP write-up, "Attention performance optimisation":
SageAttention operator, plus the fix for the per-channel quantization
coefficient that divided by zero on an all-zero channel ("operator details").
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
import synth


def f32(x) -> float:
    """Nearest fp32 (RNE) of an exact rational or float."""
    return float(np.float32(float(x))) if not isinstance(x, Fraction) else _frac_to_f32(x)


def _frac_to_f32(fr: Fraction) -> float:
    # RNE of a rational to fp32: pick the nearer of the two bracketing floats
    a = np.float32(float(fr))          # float() is RNE to fp64; refine exactly below
    cands = {np.float32(a), np.nextafter(a, np.float32(np.inf)), np.nextafter(a, np.float32(-np.inf))}
    best = None
    for c in cands:
        err = abs(Fraction(float(c)) - fr)
        if best is None or err < best[0] or (err == best[0] and (np.float32(c).view(np.uint32) & 1) == 0):
            best = (err, c)
    return float(best[1])


def _tiny_tensor(seed, B, H, N, d, **kw):
    w = synth.Workload("t", B, H, N, d, seed=seed, **kw)
    return synth.qkv_numpy(w), w


def test_k_mean_is_exact_sum_then_fp64_divide():
    (q, k, v), w = _tiny_tensor(3, 1, 2, 300, 16)
    kf = synth.bf16_bits_to_f32(k).astype(np.float64)
    mean = oracle.k_mean(k)
    for h in range(2):
        for c in range(16):
            exact = sum(Fraction(float(x)) for x in kf[0, h, :, c])
            # divide by N rounded to fp64, then to fp32 (the stated order)
            want = np.float32(float(exact / 300))
            assert mean[0, h, c] == want
            # and the fp64 partial sums really were exact: fp64 mean agrees
            assert np.float64(kf[0, h, :, c].sum()) == float(exact)


def test_k_mean_constant_channel_and_numpy():
    k = np.full((1, 1, 257, 4), 0, dtype=np.uint16)
    vals = np.array([1.5, -2.25, 0.0, 3.0], dtype=np.float32)
    k[...] = (vals.view(np.uint32) >> 16).astype(np.uint16)
    assert np.array_equal(oracle.k_mean(k)[0, 0], vals)
    (q, k2, v), _ = _tiny_tensor(5, 2, 3, 1000, 8)
    ref = synth.bf16_bits_to_f32(k2).astype(np.float64).mean(axis=2).astype(np.float32)
    np.testing.assert_array_equal(oracle.k_mean(k2), ref)


def _check_int8_block_properties(xs: np.ndarray, codes: np.ndarray, scale: float):
    """xs: fp32 values of one block (already smoothed), codes: its INT8 codes."""
    amax = float(np.abs(xs).max())
    if amax == 0.0:
        assert scale == 0.0 and not codes.any()
        return
    assert scale == f32(Fraction(amax) / 127)
    assert np.abs(codes.astype(int)).max() <= 127
    # the absmax element maps to +-127
    i = np.unravel_index(np.argmax(np.abs(xs)), xs.shape)
    assert abs(int(codes[i])) == 127 and np.sign(codes[i]) == np.sign(xs[i])
    # each code is the nearest integer to x * 127/amax: within half a step plus fp32 slack
    t = xs.astype(np.float64) * 127.0 / amax
    assert np.all(np.abs(codes - t) <= 0.5 + 1e-5)
    # exact rational brute force of rne(fl32(x * fl32(127/amax)))
    inv = f32(Fraction(127) / Fraction(amax))
    for x, c in zip(xs.ravel()[:200], codes.ravel()[:200]):
        prod = Fraction(f32(Fraction(float(x)) * Fraction(inv)))
        fl = prod.numerator // prod.denominator
        r = prod - fl
        want = fl + (1 if r > Fraction(1, 2) or (r == Fraction(1, 2) and fl % 2 == 1) else 0)
        assert int(c) == max(-127, min(127, want))


def test_q_blocks_int8():
    (q, k, v), w = _tiny_tensor(11, 1, 2, 300, 32)
    codes, scale = oracle.quant_int8_blocks(q)
    assert scale.shape == (1, 2, 3)
    qf = synth.bf16_bits_to_f32(q)
    for h in range(2):
        for b in range(3):
            sl = slice(b * 128, min(300, b * 128 + 128))
            _check_int8_block_properties(qf[0, h, sl], codes[0, h, sl], float(scale[0, h, b]))


def test_k_smoothing_int8():
    (q, k, v), w = _tiny_tensor(12, 1, 2, 300, 32, k_off_std=3.0)
    mean = oracle.k_mean(k)
    codes, scale = oracle.quant_int8_blocks(k, mean)
    kf = synth.bf16_bits_to_f32(k)
    ks = (kf - mean[:, :, None, :]).astype(np.float32)   # fp32 subtraction
    for h in range(2):
        for b in range(3):
            sl = slice(b * 128, min(300, b * 128 + 128))
            _check_int8_block_properties(ks[0, h, sl], codes[0, h, sl], float(scale[0, h, b]))
    # smoothing removes the offset: smoothed channel means are ~0
    assert np.abs(ks.mean(axis=2)).max() < 1e-5


def test_zero_channel_and_zero_block_guard():
    # all-zero K channel (the NaN bug of the pages), all-zero Q block, all-zero V channel
    (q, k, v), w = _tiny_tensor(13, 1, 1, 260, 16, zero_k_channel=5)
    q = q.copy()
    v = v.copy()
    q[0, 0, 128:256] = 0
    v[0, 0, :, 3] = 0
    pre = oracle.prepass(q, k, v)
    for name in ("k_mean", "q_scale", "k_scale", "v_scale"):
        assert np.all(np.isfinite(pre[name])), name
    assert pre["q_scale"][0, 0, 1] == 0.0 and not pre["q_i8"][0, 0, 128:256].any()
    assert pre["k_mean"][0, 0, 5] == 0.0 and not pre["k_i8"][0, 0, :, 5].any()
    assert pre["v_scale"][0, 0, 3] == 0.0 and not pre["v_f8"][0, 0, :, 3].any()
    # a K block that is exactly its mean smooths to zero -> scale 0, codes 0
    kc = np.zeros((1, 1, 128, 8), dtype=np.uint16)
    kc[...] = np.uint16(0x3F80)                         # 1.0 everywhere
    m = oracle.k_mean(kc)
    c, s = oracle.quant_int8_blocks(kc, m)
    assert s[0, 0, 0] == 0.0 and not c.any()


def test_v_fp8_per_channel():
    (q, k, v), w = _tiny_tensor(14, 1, 2, 333, 16)
    codes, scale = oracle.quant_v_fp8(v)
    table = oracle.e4m3_decode_table()
    vf = synth.bf16_bits_to_f32(v).astype(np.float64)
    for h in range(2):
        for c in range(16):
            col = vf[0, h, :, c]
            amax = np.abs(col).max()
            assert scale[0, h, c] == f32(Fraction(float(amax)) / 448)
            cc = codes[0, h, :, c]
            # channel absmax maps to +-448
            i = int(np.argmax(np.abs(col)))
            assert cc[i] & 0x7F == 0x7E
            deq = table[cc] * float(scale[0, h, c])
            # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 in the normal range,
            # absolute error <= 2^-10 * scale in the subnormal range
            tol = np.maximum(np.abs(col) * 2.0 ** -4, 2.0 ** -10 * amax / 448) * 1.0001
            assert np.all(np.abs(deq - col) <= tol + 1e-12)
            # encoding agrees with an independent nearest-value search over the code table
            inv = np.float32(f32(Fraction(448) / Fraction(float(amax))))
            t = (col.astype(np.float32) * inv).astype(np.float64)
            finite = table[:0x7F]
            for x, code in zip(t[:64], cc[:64]):
                dist = np.abs(finite - abs(x))
                best = np.flatnonzero(dist == dist.min())
                want = best[0] if len(best) == 1 else [b for b in best if b % 2 == 0][0]
                assert code & 0x7F == want


def test_rows_quantizer_generalises_the_block_one():
    (q, k, v), w = _tiny_tensor(15, 2, 2, 300, 64)
    a = oracle.quant_int8_blocks(q)
    b = oracle.quant_int8_rows(q, 128)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1].view(np.uint32), b[1].view(np.uint32))
    mean = oracle.k_mean(k)
    a = oracle.quant_int8_blocks(k, mean)
    b = oracle.quant_int8_rows(k, 128, mean)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1].view(np.uint32), b[1].view(np.uint32))


def test_per_token_q_int8():
    (q, k, v), w = _tiny_tensor(16, 1, 2, 70, 32)
    q = q.copy()
    q[0, 1, 5] = 0                                       # an all-zero token
    codes, scale = oracle.quant_int8_rows(q, 1)
    assert scale.shape == (1, 2, 70)
    qf = synth.bf16_bits_to_f32(q)
    for h in range(2):
        for n in range(70):
            _check_int8_block_properties(qf[0, h, n:n + 1], codes[0, h, n:n + 1], float(scale[0, h, n]))
    assert scale[0, 1, 5] == 0.0 and not codes[0, 1, 5].any()
