"""The seeded input generator (synth/) against its stated recipe.

synth/ is shared by both sides (it draws numbers only), so the parity tests
rest on it producing what the input recipe says: splitmix64 counters, Box-Muller
normals, Q, V ~ N(0, 1), K ~ N(0, 1) plus a per-(b, h, c) offset ~ N(0, 9),
round(0.01 * H * d) outlier (h, c) pairs scaled x20 in Q and K alike, an
optional all-zero K channel, bf16 by round-to-nearest-even, and determinism.
The splitmix64 mixer is pinned to the published sequence of the generator
seeded with 0 (Steele, Lea & Flood, OOPSLA 2014)."""
import ctypes
import math

import numpy as np

import synth

M64 = (1 << 64) - 1
GAMMA = 0x9E3779B97F4A7C15


def _splitmix64(x: int) -> int:
    x = (x + GAMMA) & M64
    x = ((x ^ (x >> 30)) * 0xBF58476D1CE4E5B9) & M64
    x = ((x ^ (x >> 27)) * 0x94D049BB133111EB) & M64
    return x ^ (x >> 31)


def _normal(seed: int, tensor: int, e: int) -> float:
    key = _splitmix64(_splitmix64(seed) ^ ((tensor * 0xD1B54A32D192ED03) & M64))
    u1 = (_splitmix64((key + 2 * e) & M64) >> 11) * 2.0 ** -53
    u2 = (_splitmix64((key + 2 * e + 1) & M64) >> 11) * 2.0 ** -53
    return math.sqrt(-2.0 * math.log(1.0 - u1)) * math.cos(2.0 * math.pi * u2)


def test_splitmix64_published_sequence():
    # the generator seeded with 0 yields e220a8397b1dcdaf, 6e789e6aa1b965f4, 06c45d188009454f, ...
    state, out = 0, []
    for _ in range(3):
        out.append(_splitmix64(state))
        state = (state + GAMMA) & M64
    assert out == [0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4, 0x06C45D188009454F]


def test_normals_follow_the_counter_definition():
    lib = synth._load()
    for seed, tensor, e in [(0, 1, 0), (0, 2, 12345), (7, 3, 2 ** 33 + 5), (123456789, 4, 99)]:
        assert abs(lib.synth_normal(seed, tensor, e) - _normal(seed, tensor, e)) < 1e-12


def test_q_v_standard_normal_and_k_offsets():
    w = synth.Workload("recipe", 1, 8, 4096, 64, seed=3)
    q, k, v = (synth.bf16_bits_to_f32(a).astype(np.float64) for a in synth.qkv_numpy(w))
    n = q.size
    for t in (q, v):
        assert abs(t.mean()) < 5 / math.sqrt(n)
        assert abs(t.std() - 1.0) < 0.01
    # K = N(0,1) + off[b,h,c]: token means per channel spread like N(0, 9), within-channel spread ~ 1
    means = k.mean(axis=2).ravel()                  # [B*H*d] channel offsets (+ O(1/sqrt(N)) noise)
    assert abs(means.std() - 3.0) < 0.35            # 512 draws of N(0, 9)
    assert abs((k - k.mean(axis=2, keepdims=True)).std() - 1.0) < 0.01


def test_outlier_pairs_are_shared_by_q_and_k():
    w = synth.Workload("recipe_out", 1, 40, 2048, 128, seed=11, outlier_frac=0.01)
    assert w.n_outlier == 51                        # round(0.01 * 40 * 128)
    mask = np.zeros(w.H * w.d, dtype=np.uint8)
    assert synth._load().synth_outlier_pairs(w.seed, w.H, w.d, w.n_outlier,
                                             mask.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8))) == 0
    mask = mask.reshape(w.H, w.d).astype(bool)
    assert mask.sum() == 51
    q, k, _ = (synth.bf16_bits_to_f32(a).astype(np.float64) for a in synth.qkv_numpy(w))
    q_std = q[0].std(axis=1)                        # [H, d] per-channel spread over tokens
    k_std = k[0].std(axis=1)
    assert np.all(np.abs(q_std[mask] - 20.0) < 2.0) and np.all(np.abs(q_std[~mask] - 1.0) < 0.15)
    assert np.all(np.abs(k_std[mask] - 20.0) < 2.0) and np.all(np.abs(k_std[~mask] - 1.0) < 0.15)


def test_zero_k_channel_bf16_rounding_and_determinism():
    w = synth.Workload("recipe_zero", 2, 3, 300, 128, seed=5, zero_k_channel=7)
    q, k, v = synth.qkv_numpy(w)
    assert not k[..., 7].any()                      # all-zero bit patterns
    assert k[..., 6].any()
    # bf16 = RNE of the fp32 value of the fp64 normal (Q stream = tensor 1, element e = row * d + c)
    for e in (0, 1, 777, q.size - 1):
        f = np.float32(_normal(w.seed, 1, e))
        bits = int(np.array(f).view(np.uint32))
        rne = (bits + 0x7FFF + ((bits >> 16) & 1)) >> 16
        assert int(q.reshape(-1)[e]) == rne
    again = synth.qkv_numpy(w)
    assert all(np.array_equal(a, b) for a, b in zip((q, k, v), again))
    other = synth.qkv_numpy(w.with_seed(6))
    assert not np.array_equal(q, other[0])


def test_linear_operands_recipe():
    """X ~ N(0,1) with round(0.01 K) outlier channels x20, W ~ N(0, 1/K), bias ~ 0.02 N(0,1)."""
    lw = synth.LinearWorkload("recipe_lin", 4096, 384, 1024, seed=9)
    assert lw.n_outlier == 10
    x, wt, b = (synth.bf16_bits_to_f32(a).astype(np.float64) for a in synth.linear_numpy(lw))
    col_std = x.std(axis=0)
    out = col_std > 5.0
    assert out.sum() == 10
    assert np.all(np.abs(col_std[out] - 20.0) < 1.5) and np.all(np.abs(col_std[~out] - 1.0) < 0.1)
    assert abs(x[:, ~out].mean()) < 5 / math.sqrt(x[:, ~out].size)
    assert abs(wt.std() * math.sqrt(lw.K) - 1.0) < 0.01
    assert abs(b.std() / 0.02 - 1.0) < 0.15          # 384 draws
    assert np.array_equal(synth.linear_numpy(lw)[0], synth.linear_numpy(lw)[0])


def test_sampled_rows_cover_the_edges():
    """Parity samples always hold row 0, row N-1 and the first row of the tail tile; sorted, distinct."""
    for seed, N, n in [(0, 75600, 48), (3, 17776, 16), (5, 129, 8), (1, 100, 500), (2, 1, 4)]:
        rows = synth.sample_rows(seed, N, n)
        assert len(rows) == min(n, N)
        assert np.all(np.diff(rows) > 0) and rows[0] >= 0 and rows[-1] < N
        assert {0, N - 1, (N - 1) // 128 * 128} <= set(rows.tolist())
    assert np.array_equal(synth.sample_rows(7, 5000, 20), synth.sample_rows(7, 5000, 20))
