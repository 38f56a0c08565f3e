"""Pins the oracle's attention (O1 exact fp64, O2 emulation of the quantized
scheme) to brute force, closed forms and invariants of softmax attention.

The op is the DiT full-sequence self-attention that page 1 of the TMAP
write-up profiles ("Attention performance optimisation / Background":
aten.scaled_dot_product_flash_attention, 73.76% of FLOPs) and then replaces
with SageAttention ("attention quantization").
"""
import numpy as np
import pytest

import oracle
import synth

TABLE = oracle.e4m3_decode_table()


def bf16(x: np.ndarray) -> np.ndarray:
    """fp32 values -> bf16 bits (RNE); used only to build exact test inputs."""
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def f(b):
    return synth.bf16_bits_to_f32(b).astype(np.float64)


def cos(a, b):
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    return float(a @ b / np.linalg.norm(a) / np.linalg.norm(b))


def textbook(q, k, v):
    """softmax(q k^T / sqrt(d)) v in numpy longdouble, straight from the definition."""
    Q, K, V = (f(x).astype(np.longdouble) for x in (q, k, v))
    d = Q.shape[-1]
    s = np.einsum("bhic,bhjc->bhij", Q, K) / np.sqrt(np.longdouble(d))
    e = np.exp(s - s.max(axis=-1, keepdims=True))
    p = e / e.sum(axis=-1, keepdims=True)
    return np.einsum("bhij,bhjc->bhic", p, V)


@pytest.mark.parametrize("N", [1, 2, 5, 8])
def test_exact_matches_textbook_brute_force(N):
    w = synth.Workload("t", 2, 2, N, 16, seed=N)
    q, k, v = synth.qkv_numpy(w)
    got = oracle.attn_exact(q, k, v)
    want = textbook(q, k, v).astype(np.float64)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_exact_special_cases():
    w = synth.Workload("t", 1, 1, 1, 32, seed=1)
    q, k, v = synth.qkv_numpy(w)
    # N = 1: the output is the only V row
    np.testing.assert_array_equal(oracle.attn_exact(q, k, v)[0, 0, 0], f(v)[0, 0, 0])
    # Q = 0: uniform weights -> column mean of V
    w = synth.Workload("t", 1, 1, 200, 32, seed=2)
    q, k, v = synth.qkv_numpy(w)
    q0 = np.zeros_like(q)
    got = oracle.attn_exact(q0, k, v, rows=[0, 7, 199])
    np.testing.assert_allclose(got[0, 0], np.broadcast_to(f(v)[0, 0].mean(0), (3, 32)), atol=1e-13)
    # one-hot scores: q . k_j = 64 for the chosen j and 0 otherwise -> row j of V
    d, N = 64, 6
    K = np.eye(N, d, dtype=np.float32) * 8.0
    Q = np.zeros((N, d), dtype=np.float32)
    Q[np.arange(N), (np.arange(N) + 2) % N] = 8.0 * 100
    V = np.random.default_rng(0).standard_normal((N, d)).astype(np.float32)
    out = oracle.attn_exact(bf16(Q)[None, None], bf16(K)[None, None], bf16(V)[None, None])[0, 0]
    np.testing.assert_allclose(out, f(bf16(V))[(np.arange(N) + 2) % N], atol=1e-12)


def test_exact_smoothing_invariance():
    # K with integer entries and an integer per-channel offset: K - offset is exact in bf16
    rng = np.random.default_rng(3)
    N, d = 300, 32
    Kc = rng.integers(-8, 9, (1, 1, N, d)).astype(np.float32)
    off = rng.integers(-20, 21, (1, 1, 1, d)).astype(np.float32)
    Q = rng.standard_normal((1, 1, N, d)).astype(np.float32) * 0.3
    V = rng.standard_normal((1, 1, N, d)).astype(np.float32)
    q, v = bf16(Q), bf16(V)
    a = oracle.attn_exact(q, bf16(Kc + off), v)
    b = oracle.attn_exact(q, bf16(Kc), v)
    np.testing.assert_allclose(a, b, rtol=1e-10, atol=1e-12)


def test_convex_hull_and_zero_channel_finite():
    w = synth.WORKLOADS["tiny"]
    q, k, v = synth.qkv_numpy(w)
    rows = synth.sample_rows(5, w.N, 48)
    o1 = oracle.attn_exact(q, k, v, rows)
    pre = oracle.prepass(q, k, v)
    o2, _ = oracle.attn_emul(pre, rows)
    V = f(v)
    lo, hi = V.min(axis=2)[:, :, None], V.max(axis=2)[:, :, None]
    for o in (o1, o2.astype(np.float64)):
        assert np.all(np.isfinite(o))
        assert np.all(o >= lo - 1e-6 * np.abs(lo)) and np.all(o <= hi + 1e-6 * np.abs(hi))


def test_qk_tile_matches_int64_matmul():
    w = synth.Workload("t", 1, 2, 300, 64, seed=4)
    q, k, v = synth.qkv_numpy(w)
    pre = oracle.prepass(q, k, v)
    q8 = pre["q_i8"].astype(np.int64)
    k8 = pre["k_i8"].astype(np.int64)
    for bh, qb, kb in [(0, 0, 0), (1, 2, 1), (1, 0, 2), (0, 2, 2)]:
        tile = oracle.qk_tile(pre["q_i8"], pre["k_i8"], bh, qb, kb)
        qs = np.zeros((128, 64), np.int64)
        ks = np.zeros((128, 64), np.int64)
        qr = q8[0, bh, qb * 128:(qb + 1) * 128]
        kr = k8[0, bh, kb * 128:(kb + 1) * 128]
        qs[:len(qr)] = qr
        ks[:len(kr)] = kr
        np.testing.assert_array_equal(tile, qs @ ks.T)


def test_emulation_converges_to_exact_as_quantization_is_removed():
    w = synth.Workload("t", 1, 2, 700, 64, seed=6)
    q, k, v = synth.qkv_numpy(w)
    pre = oracle.prepass(q, k, v)
    rows = synth.sample_rows(7, w.N, 40)
    o1 = oracle.attn_exact(q, k, v, rows)
    allx = oracle.EMUL_P_FP32 | oracle.EMUL_V_EXACT | oracle.EMUL_QK_EXACT
    # no quantization left: fp32 online softmax == fp64 attention to fp32 accuracy
    o_none, _ = oracle.attn_emul(pre, rows, allx, q, k, v)
    np.testing.assert_allclose(o_none, o1, rtol=2e-5, atol=2e-6)
    # the single-tile (non-online) variant agrees with the tiled one to fp32 rounding
    o_one, _ = oracle.attn_emul(pre, rows, allx | oracle.EMUL_ONE_TILE, q, k, v)
    np.testing.assert_allclose(o_none, o_one, rtol=2e-5, atol=2e-6)
    # switching each quantization on moves the result away from O1 monotonically-ish,
    # but every stage stays close
    errs = []
    for flags in (allx, oracle.EMUL_P_FP32 | oracle.EMUL_V_EXACT, oracle.EMUL_P_FP32, 0):
        o, _ = oracle.attn_emul(pre, rows, flags, q, k, v)
        errs.append(1 - cos(o, o1))
    assert errs[0] < 1e-10
    assert errs[-1] > errs[0]
    assert all(e < 5e-3 for e in errs)


def test_emulation_special_cases():
    # N = 1: p = 1 -> P8 = 448 exactly -> O = dequantized V row
    w = synth.Workload("t", 1, 1, 1, 64, seed=8)
    q, k, v = synth.qkv_numpy(w)
    pre = oracle.prepass(q, k, v)
    o, _ = oracle.attn_emul(pre)
    deq = TABLE[pre["v_f8"][0, 0, 0]] * pre["v_scale"][0, 0]
    np.testing.assert_allclose(o[0, 0, 0], deq, rtol=1e-6)
    # Q = 0: every score is 0 -> uniform weights -> mean of dequantized V
    w = synth.Workload("t", 1, 1, 300, 64, seed=9)
    q, k, v = synth.qkv_numpy(w)
    q = np.zeros_like(q)
    pre = oracle.prepass(q, k, v)
    assert not pre["q_scale"].any()
    o, _ = oracle.attn_emul(pre, [0, 150, 299])
    deq = TABLE[pre["v_f8"][0, 0]] * pre["v_scale"][0, 0][None, :]
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(deq.mean(0), (3, 64)), rtol=1e-5, atol=1e-6)


def test_emulation_quality_on_tiny_with_zero_channel():
    w = synth.WORKLOADS["tiny"]
    q, k, v = synth.qkv_numpy(w)
    pre = oracle.prepass(q, k, v)
    o1 = oracle.attn_exact(q, k, v)
    o2, ob = oracle.attn_emul(pre)
    assert np.all(np.isfinite(o2))
    assert cos(o2, o1) >= 0.995
    # bf16 output bits are the RNE of the fp32 values
    np.testing.assert_array_equal(ob, bf16(o2))


def test_layer_schedule():
    modes = oracle.layer_schedule(40, synth.LAYER_STACK_FULL_PRECISION)
    assert modes.tolist() == [0 if l % 8 == 0 else 1 for l in range(40)]
    assert oracle.layer_schedule(3, [1, 1]).tolist() == [1, 0, 1]
    assert oracle.layer_schedule(0, []).tolist() == []
    with pytest.raises(ValueError):
        oracle.layer_schedule(4, [4])
    with pytest.raises(ValueError):
        oracle.layer_schedule(4, [-1])


def test_per_token_q_scale_emulation():
    # every row of a block shares its absmax -> per-token scales equal the block scale,
    # so the per-token emulation must equal the per-block one exactly
    w = synth.Workload("t", 1, 2, 256, 64, seed=17)
    q, k, v = synth.qkv_numpy(w)
    Q = synth.bf16_bits_to_f32(q).copy()
    Q = np.clip(Q, -3.0, 3.0)
    Q[..., 0] = 4.0
    q = bf16(Q)
    pre_b = oracle.prepass(q, k, v)
    pre_t = oracle.prepass(q, k, v, q_per_token=True)
    assert np.array_equal(pre_b["q_i8"], pre_t["q_i8"])
    assert np.all(pre_t["q_scale"] == pre_b["q_scale"][0, 0, 0])
    rows = [0, 5, 130, 255]
    ob, _ = oracle.attn_emul(pre_b, rows)
    ot, _ = oracle.attn_emul(pre_t, rows, flags=oracle.EMUL_Q_PER_TOKEN)
    np.testing.assert_array_equal(ob, ot)
    # on ordinary inputs the per-token scheme stays close to exact attention
    w = synth.Workload("t", 1, 2, 700, 128, seed=18, outlier_frac=0.01)
    q, k, v = synth.qkv_numpy(w)
    rows = synth.sample_rows(4, w.N, 64)
    o1 = oracle.attn_exact(q, k, v, rows)
    ot, _ = oracle.attn_emul(oracle.prepass(q, k, v, q_per_token=True), rows, flags=oracle.EMUL_Q_PER_TOKEN)
    assert cos(ot, o1) >= 0.995
