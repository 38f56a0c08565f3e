"""Per-layer error calibration for the selective-quantization table (page 1
of the TMAP write-up, "keeping video quality": per-layer attention error over
the denoising iterations decides which layers keep the original precision).

The error-statistics kernel is checked against numpy's fp64 sums, and the
whole calibration on a synthetic 4-layer stack whose layers 1 and 3 carry
heavy outlier channels (5% of (h, c) pairs x60, versus 1% x20 elsewhere):
the layers it selects must be the ones the oracle's emulation puts above the
same threshold against exact attention."""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("shape", [(1, 3, 1000, 128), (2, 2, 777, 64)])
def test_error_stats_match_numpy(shape, cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    g = torch.Generator().manual_seed(sum(shape))
    a = torch.randn(shape, generator=g).to(torch.bfloat16)
    b = (a.float() + 0.05 * torch.randn(shape, generator=g)).to(torch.bfloat16)
    st = sage.error_stats(a.to(cuda_dev), b.to(cuda_dev)).cpu().numpy()
    A = a.double().numpy().reshape(shape[0] * shape[1], -1)
    Bm = b.double().numpy().reshape(shape[0] * shape[1], -1)
    want = np.stack([((A - Bm) ** 2).sum(1), (Bm ** 2).sum(1), (A * Bm).sum(1), (A ** 2).sum(1)], 1)
    np.testing.assert_allclose(st, want, rtol=1e-10)
    # deterministic
    st2 = sage.error_stats(a.to(cuda_dev), b.to(cuda_dev)).cpu().numpy()
    assert np.array_equal(st, st2)


def test_calibration_selects_the_outlier_layers(cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    bad = {1, 3}
    layers, oracle_err = [], []
    for l in range(4):
        per_layer, per_oracle = [], []
        for it in range(2):
            w = synth.Workload(f"l{l}", 1, 2, 2048, 128, seed=100 * l + it,
                               outlier_frac=0.05 if l in bad else 0.01, outlier_scale=60.0 if l in bad else 20.0)
            q, k, v = synth.qkv_numpy(w)
            per_layer.append(tuple(torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(cuda_dev) for a in (q, k, v)))
            rows = synth.sample_rows(it, w.N, 128)
            pre = oracle.prepass(q, k, v)
            o2, _ = oracle.attn_emul(pre, rows)
            o1 = oracle.attn_exact(q, k, v, rows)
            per_oracle.append(float(np.sqrt(((o2 - o1) ** 2).sum() / (o1 ** 2).sum())))
        layers.append(per_layer)
        oracle_err.append(per_oracle)
    err = np.array(sage.layer_errors(layers))
    assert np.all(np.isfinite(err)) and err.shape == (4, 2)
    threshold = 0.11
    oracle_pick = [l for l in range(4) if np.mean(oracle_err[l]) > threshold]
    assert oracle_pick == sorted(bad)
    picked = sage.select_full_precision_layers(err, threshold)
    assert picked == oracle_pick
    # the GPU error tracks the oracle's error layer by layer
    np.testing.assert_allclose(err.mean(1), np.mean(oracle_err, 1), rtol=0.35)
    modes = sage.layer_schedule(4, picked)
    assert modes == [sage.MODE_INT8_FP8, sage.MODE_BF16, sage.MODE_INT8_FP8, sage.MODE_BF16]


def test_linear_layer_selection_matches_the_oracle(cuda_dev):
    """Selective W8A8 -> W8A16 for linear layers: on a synthetic stack where two layers carry strong
    activation outlier channels (per-block X scales inflated by 100x outliers), the layers whose
    W8A8-vs-W8A16 error exceeds the threshold are the ones the oracle's errors select."""
    import torch
    from video_dit_quantized_b200 import sage
    L, iters = 6, 2
    heavy = {2, 5}
    layers, oracle_err = [], []
    for l in range(L):
        row, orow = [], []
        for it in range(iters):
            lw = synth.LinearWorkload("cal", 256, 256, 512, seed=100 * l + it,
                                      outlier_frac=0.02, outlier_scale=100.0 if l in heavy else 3.0)
            x, wt, b = synth.linear_numpy(lw)
            dev = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(cuda_dev)
            wq, sw = sage.quantize_blocks_2d(dev(wt))
            row.append((dev(x), wq, sw, dev(b)))
            # oracle: W8A8 (fp32, then bf16) against W8A16 (exact product of the dequantized weights)
            xq_o, sx_o = oracle.quant_blocks_2d(x)
            wq_o, sw_o = oracle.quant_blocks_2d(wt)
            _, y8 = oracle.linear_w8a8(xq_o, sx_o, wq_o, sw_o, b)
            y16 = oracle.linear_bf16(x, oracle.dequant_blocks_2d(wq_o, sw_o), b)
            y16 = torch.from_numpy(y16).to(torch.bfloat16).double().numpy()    # both outputs are bf16
            a = synth.bf16_bits_to_f32(y8).astype(np.float64)
            orow.append(float(np.linalg.norm(a - y16) / np.linalg.norm(y16)))
        layers.append(row)
        oracle_err.append(orow)
    err = sage.linear_layer_errors(layers)
    # the same errors: the W8A8 outputs are bit-exact; the W8A16 ones differ only by fp32 summation order
    np.testing.assert_allclose(err, oracle_err, rtol=0.02)
    light = [np.mean(oracle_err[l]) for l in range(L) if l not in heavy]
    strong = [np.mean(oracle_err[l]) for l in heavy]
    assert min(strong) > 2 * max(light)                         # the synthetic stack separates the two kinds
    thr = float(np.sqrt(max(light) * min(strong)))
    picked = sage.select_full_precision_layers(err, thr)
    assert picked == sorted(heavy)
    assert picked == [l for l in range(L) if np.mean(oracle_err[l]) > thr]
