"""The tcgen05 operand paths the attention kernels are built from, one tile at
a time: INT8 QK^T (bit-exact against the oracle's integer tile), FP8 P.V with
P written into tensor memory, BF16 QK^T and BF16 P.V with an MN-major V."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu

E4M3 = oracle.e4m3_decode_table()


def _dev(a, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


@pytest.mark.parametrize("w", [synth.WORKLOADS["tiny"], synth.Workload("d64", 1, 3, 700, 64, seed=31),
                               synth.Workload("ragged", 2, 1, 300, 128, seed=32, outlier_frac=0.01)],
                         ids=lambda w: w.name)
def test_qk_int8_tiles_bit_exact(w, cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    q, k, v = synth.qkv_numpy(w)
    pre = oracle.prepass(q, k, v)
    nT = (w.N + 127) // 128
    npad = nT * 128
    q8 = np.zeros((w.B, w.H, npad, w.d), np.int8)
    k8 = np.zeros((w.B, w.H, npad, w.d), np.int8)
    q8[:, :, :w.N] = pre["q_i8"]
    k8[:, :, :w.N] = pre["k_i8"]
    tiles = []
    for b in range(w.B):
        for h in range(w.H):
            tiles += [(b, h, 0, 0), (b, h, nT - 1, nT - 1), (b, h, 0, nT - 1), (b, h, nT - 1, 0)]
    got = sage.dbg_qk_tiles(_dev(q8, cuda_dev), _dev(k8, cuda_dev), w.N, tiles).cpu().numpy()
    torch.cuda.synchronize()
    for i, (b, h, qb, kb) in enumerate(tiles):
        want = oracle.qk_tile(pre["q_i8"], pre["k_i8"], b * w.H + h, qb, kb)
        np.testing.assert_array_equal(got[i], want, err_msg=str((b, h, qb, kb)))


@pytest.mark.parametrize("d", [128, 64])
def test_pv_fp8_tile(d, cuda_dev):
    from video_dit_quantized_b200 import sage
    rng = np.random.default_rng(d)
    p = rng.integers(0, 0x7F, (128, 128)).astype(np.uint8)            # e4m3 in [0, 448]
    p[:, 100:] = 0                                                     # masked keys
    vt = rng.integers(0, 256, (d, 128)).astype(np.uint8)
    vt[(vt & 0x7F) == 0x7F] = 0x38                                     # no NaN codes
    got = sage.dbg_pv_tile(_dev(p, cuda_dev), _dev(vt, cuda_dev), sage.MODE_INT8_FP8).cpu().numpy()
    P, V = E4M3[p], E4M3[vt].T                                         # [128,128], [128,d]
    want = P @ V
    scale = np.abs(P) @ np.abs(V)
    assert np.all(np.abs(got - want) <= 1e-6 * scale + 1e-30)


@pytest.mark.parametrize("d", [128, 64])
def test_pv_bf16_tile_mn_major_v(d, cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    g = torch.Generator().manual_seed(d)
    p = torch.rand((128, 128), generator=g).to(torch.bfloat16)
    vv = torch.randn((128, d), generator=g).to(torch.bfloat16)
    got = sage.dbg_pv_tile(p.to(cuda_dev), vv.to(cuda_dev), sage.MODE_BF16).cpu().numpy()
    P, V = p.double().numpy(), vv.double().numpy()
    want = P @ V
    assert np.all(np.abs(got - want) <= 1e-5 * (np.abs(P) @ np.abs(V)) + 1e-30)


@pytest.mark.parametrize("d", [128, 64])
def test_qk_bf16_tile(d, cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    g = torch.Generator().manual_seed(100 + d)
    q = torch.randn((128, d), generator=g).to(torch.bfloat16)
    k = (torch.randn((128, d), generator=g) * 3).to(torch.bfloat16)
    got = sage.dbg_qk_bf16_tile(q.to(cuda_dev), k.to(cuda_dev)).cpu().numpy()
    Q, K = q.double().numpy(), k.double().numpy()
    want = Q @ K.T
    assert np.all(np.abs(got - want) <= 1e-5 * (np.abs(Q) @ np.abs(K).T) + 1e-30)


def test_mma_throughput_probe(cuda_dev):
    """Dense tcgen05 rates per SM per clock: 8192 MACs for kind::i8 and kind::f8f6f4, 4096 for kind::f16
    (twice the bf16 rate for 8-bit, as the datasheet's 4.5 vs 2.25 PFLOP/s), at N = 128 and 256."""
    from video_dit_quantized_b200 import sage
    for kind, want in ((sage.MMA_I8, 8192), (sage.MMA_E4M3, 8192), (sage.MMA_BF16, 4096)):
        for n in (128, 256):
            r = sage.dbg_mma_peak(kind, n, iters=2000)
            assert 0.95 * want <= r["mac_per_clk_per_sm"] <= 1.01 * want, (kind, n, r)
