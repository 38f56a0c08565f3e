"""Per-layer error calibration for the selective-quantization table (page 1
of the TMAP write-up, "keeping video quality": per-layer attention error over
the denoising iterations decides which layers keep the original precision).

The error-statistics kernel is checked against numpy's fp64 sums, the
device relative L2 error against the oracle's, and the whole calibration on a
synthetic 4-layer stack whose layers 1 and 3 carry heavy outlier channels (5%
of (h, c) pairs x60, versus 1% x20 elsewhere): the library's per-layer errors
equal the oracle's relative L2 of the GPU's own INT8/FP8 and BF16 outputs
(rtol 1e-9), its selection equals the oracle's selection on them under both
rules, and the layers it selects are the ones the oracle's emulation puts
above the same threshold against exact attention."""
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


def _bits(t):
    """torch bf16 tensor -> uint16 numpy bits (host)."""
    import torch
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


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
    # the library's per-layer error is the oracle's relative L2 of the GPU's own INT8/FP8 and BF16 outputs
    for l in range(4):
        for it in range(2):
            q, k, v = layers[l][it]
            oq = sage.attn_fwd(q, k, v, sage.MODE_INT8_FP8)
            ob = sage.attn_fwd(q, k, v, sage.MODE_BF16)
            want = oracle.rel_l2(_bits(oq), _bits(ob))
            np.testing.assert_allclose(err[l, it], want, rtol=1e-9)
    threshold = 0.11
    for rule in (sage.SELECT_EVERY_ITERATION, sage.SELECT_MEAN):
        picked = sage.select_full_precision_layers(err, threshold, rule)
        assert picked == oracle.select_layers(err, threshold, rule)
        # the scheme's own error (emulation against exact attention) puts the same layers above the threshold
        assert oracle.select_layers(oracle_err, threshold, rule) == sorted(bad)
        assert picked == sorted(bad)
    modes = sage.layer_schedule(4, sorted(bad))
    assert modes == [sage.MODE_INT8_FP8, sage.MODE_BF16, sage.MODE_INT8_FP8, sage.MODE_BF16]


def test_rel_l2_matches_the_oracle(cuda_dev):
    """sage_attn_rel_l2 on random bf16 tensors (several heads, ragged N) against the oracle's fp64 sums."""
    import torch
    from video_dit_quantized_b200 import sage
    for shape in [(1, 3, 1000, 128), (2, 2, 777, 64), (1, 1, 1, 8)]:
        g = torch.Generator().manual_seed(sum(shape))
        a = torch.randn(shape, generator=g).to(torch.bfloat16)
        b = (a.float() + 0.05 * torch.randn(shape, generator=g)).to(torch.bfloat16)
        got = float(sage.rel_l2(a.to(cuda_dev), b.to(cuda_dev)).cpu())
        np.testing.assert_allclose(got, oracle.rel_l2(_bits(a), _bits(b)), rtol=1e-9)
    z = torch.zeros((1, 1, 16, 64), dtype=torch.bfloat16, device=cuda_dev)
    assert float(sage.rel_l2(z, z).cpu()) == 0.0


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
    # the library's error is the oracle's relative L2 of the GPU's own W8A8 and W8A16 outputs
    for l in range(L):
        for it in range(iters):
            x, wq, sw, b = layers[l][it]
            xq, sx = sage.quantize_blocks_2d(x)
            y8 = sage.linear_w8a8(xq, sx, wq, sw, b)
            y16 = sage.linear_w8a16(x, wq, sw, b)
            np.testing.assert_allclose(err[l][it], oracle.rel_l2(_bits(y8), _bits(y16)), rtol=1e-9)
    # and close to the oracle's own: the W8A8 outputs are bit-exact; the W8A16 ones differ only by fp32
    # summation order
    np.testing.assert_allclose(err, oracle_err, rtol=0.02)
    light = [np.mean(oracle_err[l]) for l in range(L) if l not in heavy]
    strong = [np.mean(oracle_err[l]) for l in heavy]
    assert min(strong) > 2 * max(light)                         # the synthetic stack separates the two kinds
    thr = float(np.sqrt(max(light) * min(strong)))
    for rule in (sage.SELECT_EVERY_ITERATION, sage.SELECT_MEAN):
        picked = sage.select_full_precision_layers(err, thr, rule)
        assert picked == sorted(heavy)
        assert picked == oracle.select_layers(oracle_err, thr, rule)
