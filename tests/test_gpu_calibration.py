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
