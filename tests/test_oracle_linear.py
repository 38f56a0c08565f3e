"""Pins the oracle's W8A8 linear layer with 128x128 block scales (page 1 of the
TMAP write-up, "FFN performance optimisation": 8-bit weights and activations
with a 128x128 per-block quantization operator)."""
from fractions import Fraction

import numpy as np

import oracle


def bf16(x):
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def f(b):
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f32_rne(r: Fraction) -> np.float32:
    """The fp32 nearest to the rational r, ties to even (no double rounding through float64)."""
    c = np.float32(float(r))
    cands = [c, np.nextafter(c, np.float32(np.inf)), np.nextafter(c, np.float32(-np.inf))]
    best = min(abs(Fraction(float(x)) - r) for x in cands)
    near = [x for x in cands if abs(Fraction(float(x)) - r) == best]
    return min(near, key=lambda x: int(np.array(x).view(np.uint32)) & 1)


def test_block_quantizer_matches_the_attention_one_per_block():
    rng = np.random.default_rng(0)
    x = bf16(rng.standard_normal((300, 256)).astype(np.float32) * 2)
    x[130:140, 128:256] = 0
    x[256:300, :128] = 0                                           # one all-zero block
    codes, scales = oracle.quant_blocks_2d(x)
    assert scales.shape == (3, 2)
    for rb in range(3):
        for kb in range(2):
            blk = x[rb * 128:(rb + 1) * 128, kb * 128:(kb + 1) * 128]
            # the same block as a [1, 1, rows, 128] tensor through the pinned per-block quantizer
            c1, s1 = oracle.quant_int8_rows(np.ascontiguousarray(blk)[None, None], 128)
            assert scales[rb, kb] == s1[0, 0, 0]
            assert np.array_equal(codes[rb * 128:(rb + 1) * 128, kb * 128:(kb + 1) * 128], c1[0, 0])
    assert scales[2, 0] == 0.0 and not codes[256:300, :128].any()


def test_linear_is_the_exact_block_scaled_sum():
    rng = np.random.default_rng(1)
    M, N, K = 130, 140, 256
    x = bf16(rng.standard_normal((M, K)).astype(np.float32))
    w = bf16(rng.standard_normal((N, K)).astype(np.float32) * 0.1)
    b = bf16(rng.standard_normal(N).astype(np.float32))
    xq, sx = oracle.quant_blocks_2d(x)
    wq, sw = oracle.quant_blocks_2d(w)
    rows = [0, 1, 127, 128, 129]
    y, yb = oracle.linear_w8a8(xq, sx, wq, sw, b, rows)
    for i, m in enumerate(rows):
        for n in (0, 5, 127, 128, 139):
            acc = np.float32(0)
            for kb in range(2):
                s = int(np.dot(xq[m, kb * 128:(kb + 1) * 128].astype(np.int64), wq[n, kb * 128:(kb + 1) * 128].astype(np.int64)))
                sc = np.float32(sx[m // 128, kb]) * np.float32(sw[n // 128, kb])
                # fused multiply-add: the exact rational sc * s + acc, rounded once to fp32
                acc = f32_rne(Fraction(float(sc)) * s + Fraction(float(acc)))
            acc = f32_rne(Fraction(float(acc)) + Fraction(float(f(b[n:n + 1])[0])))
            assert y[i, n] == acc
    # and it approximates the exact bf16 product within the INT8 quantization error
    exact = f(x)[rows] @ f(w).T + f(b)
    rel = np.linalg.norm(y - exact) / np.linalg.norm(exact)
    assert rel < 2e-2


def test_linear_special_cases():
    # identity-like weights: W = c * e_j rows -> Y = dequantized X columns
    K = 128
    x = bf16(np.linspace(-1, 1, 4 * K).reshape(4, K).astype(np.float32))
    w = np.zeros((K, K), dtype=np.float32)
    np.fill_diagonal(w, 0.5)
    xq, sx = oracle.quant_blocks_2d(x)
    wq, sw = oracle.quant_blocks_2d(bf16(w))
    assert np.all(wq[np.arange(K), np.arange(K)] == 127)
    y, _ = oracle.linear_w8a8(xq, sx, wq, sw)
    deq = xq.astype(np.float64) * sx[0, 0]
    np.testing.assert_allclose(y, deq * 0.5, rtol=1e-6)


def test_linear_within_the_quantization_error_bound():
    # |x - sx*xq| <= sx/2 and |w - sw*wq| <= sw/2 elementwise, so per output
    # |Y - X W^T| <= sum_k (|w| sx/2 + |x| sw/2 + sx sw/4) plus fp32 summation slack
    rng = np.random.default_rng(2)
    M, N, K = 64, 96, 384
    x = bf16(rng.standard_normal((M, K)).astype(np.float32) * np.exp(rng.standard_normal((1, K))).astype(np.float32))
    w = bf16(rng.standard_normal((N, K)).astype(np.float32) * 0.05)
    xq, sx = oracle.quant_blocks_2d(x)
    wq, sw = oracle.quant_blocks_2d(w)
    y, yb = oracle.linear_w8a8(xq, sx, wq, sw)
    X, W = f(x), f(w)
    exact = X @ W.T
    SX = np.repeat(sx.astype(np.float64), 128, axis=1)[0]      # [K] (one row block)
    SW = np.repeat(sw.astype(np.float64), 128, axis=1)[0]
    slack = 1e-5 * (np.abs(X) @ np.abs(W).T)
    err = np.abs(y - exact)
    per = (np.abs(X) @ (SW / 2))[:, None] + (SX / 2) @ np.abs(W).T + (SX * SW / 4).sum()
    assert np.all(err <= per + slack)
    # the largest code in each block is +-127 (the argmax element maps to the end of the range)
    for kb in range(3):
        assert np.abs(xq[:, kb * 128:(kb + 1) * 128]).max() == 127
    # bf16 output bits are the RNE of the fp32 values
    np.testing.assert_array_equal(yb, bf16(y))


def test_quantizer_is_rational_rne_on_a_tiny_block():
    x = bf16(np.array([[0.3, -1.7, 2.5, 0.0] * 32, [1.0, 0.25, -0.125, 3.0] * 32], dtype=np.float32))
    codes, scales = oracle.quant_blocks_2d(x)
    amax = Fraction(3)
    assert scales[0, 0] == np.float32(3.0) / np.float32(127.0)
    inv = Fraction(float(np.float32(127.0) / np.float32(3.0)))         # fl(127/amax), a correctly rounded fp32
    for r in range(2):
        for c in range(4):
            v = Fraction(float(f(x[r:r + 1, c:c + 1])[0, 0]))
            prod = Fraction(float(np.float32(float(v * inv))))   # fp32 product, RNE
            want = round(prod)                                    # Python's round is half-to-even
            assert codes[r, c] == max(-127, min(127, want))
    assert amax == 3


def test_dequant_closed_form_and_round_trip():
    # a block whose codes are all +-127 dequantizes to +-amax (scale * 127 = amax up to one fp32 rounding)
    rng = np.random.default_rng(5)
    w = bf16(rng.standard_normal((256, 256)).astype(np.float32) * 0.05)
    codes, scales = oracle.quant_blocks_2d(w)
    deq = oracle.dequant_blocks_2d(codes, scales)
    for rb in range(2):
        for kb in range(2):
            c = codes[rb * 128:(rb + 1) * 128, kb * 128:(kb + 1) * 128].astype(np.int64)
            d = f(deq[rb * 128:(rb + 1) * 128, kb * 128:(kb + 1) * 128])
            sc = np.float32(scales[rb, kb])
            for cv in (-127, -3, 0, 1, 64, 127):
                m = c == cv
                if m.any():
                    want = f(bf16(np.array([np.float32(sc) * np.float32(cv)], dtype=np.float32)))[0]
                    assert np.all(d[m] == want)
    # dequantized weights approximate the originals within half a step plus bf16 rounding
    W = f(w)
    S = np.repeat(np.repeat(scales.astype(np.float64), 128, 0), 128, 1)
    assert np.all(np.abs(f(deq) - W) <= S / 2 + np.abs(W) * 2.0 ** -8 + 1e-12)
    # all-zero block: zeros
    z = np.zeros((128, 128), dtype=np.uint16)
    assert not oracle.dequant_blocks_2d(*oracle.quant_blocks_2d(z)).any()


def test_linear_bf16_is_the_exact_product():
    # small integers: every product and sum is exact, so the fp64 result is exact
    rng = np.random.default_rng(6)
    x = bf16(rng.integers(-8, 9, (5, 256)).astype(np.float32))
    w = bf16(rng.integers(-8, 9, (7, 256)).astype(np.float32))
    b = bf16(rng.integers(-8, 9, 7).astype(np.float32))
    y = oracle.linear_bf16(x, w, b)
    X, W, B = (f(a).astype(np.int64) for a in (x, w, b))
    assert np.array_equal(y, (X @ W.T + B[None, :]).astype(np.float64))
    assert np.array_equal(oracle.linear_bf16(x, w, None, rows=[4, 0]), (X @ W.T)[[4, 0]].astype(np.float64))
