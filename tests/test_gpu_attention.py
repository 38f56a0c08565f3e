"""GPU attention (INT8/FP8 and BF16 modes) against the oracle.

Quantized mode: cosine >= 0.9999 and max-abs <= 5e-3 * max|V| (per head)
against the scalar emulation, cosine >= 0.995 against fp64 exact attention.
BF16 mode: relative L2 <= 4e-3 against fp64 exact attention.  Small ragged
shapes are checked on every row; the full-size CogVideoX / Wan shapes in the
launch configuration of the benchmark on sampled rows of three heads.
The op: full-sequence self-attention of a video DiT (page 1 of the TMAP
write-up, "Attention performance optimisation").
"""
import numpy as np
import pytest

import oracle
import synth
from _util import (COS_EMUL, COS_EXACT, MAXABS_EMUL, REL_L2_BF16, bf16_to_np, cos, emul_and_exact, heads,
                   rel_l2, small_workloads)

pytestmark = pytest.mark.gpu


def _dev(a, device):
    import torch
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)


def check_quant(got, o2, o1, vf, label):
    """got: GPU [B,H',R,d] fp32 (bf16 values); o2/o1 oracle; vf: V fp32 [B,H',N,d]."""
    assert np.all(np.isfinite(got)), label
    c2 = cos(got, o2)
    c1 = cos(got, o1)
    vmax = np.abs(vf).max(axis=(2, 3))                         # [B,H']
    err = np.abs(got - o2).max(axis=(2, 3))
    assert c2 >= COS_EMUL, f"{label}: cos vs emulation {c2}"
    assert np.all(err <= MAXABS_EMUL * vmax), f"{label}: max-abs {err.max()} vs {MAXABS_EMUL} * {vmax.min()}"
    assert c1 >= COS_EXACT, f"{label}: cos vs exact {c1}"


@pytest.mark.parametrize("w", small_workloads(), ids=lambda w: w.name)
def test_quantized_small_all_rows(w, cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    q, k, v = synth.qkv_numpy(w)
    rows = np.arange(w.N, dtype=np.int32)
    _, o2, o1 = emul_and_exact(q, k, v, rows)
    qd, kd, vd = _dev(q, cuda_dev), _dev(k, cuda_dev), _dev(v, cuda_dev)
    ws = sage.alloc_workspace(w.B, w.H, w.N, w.d, sage.MODE_INT8_FP8)
    o = sage.attn_fwd(qd, kd, vd, sage.MODE_INT8_FP8, workspace=ws)
    assert sage.status(ws) == sage.OK
    got = bf16_to_np(o)
    check_quant(got, o2, o1, synth.bf16_bits_to_f32(v), w.name)
    # the two-call form (prepass, then attention on its outputs) is the same computation
    pre = sage.quantize_qk(qd, kd, vd)
    o_b = sage.attn_quantized(pre, w.N)
    torch.cuda.synchronize()
    assert torch.equal(o_b.view(torch.int16), o.view(torch.int16))


@pytest.mark.parametrize("w", small_workloads(), ids=lambda w: w.name)
def test_bf16_small_all_rows(w, cuda_dev):
    from video_dit_quantized_b200 import sage
    q, k, v = synth.qkv_numpy(w)
    o1 = oracle.attn_exact(q, k, v)
    ws = sage.alloc_workspace(w.B, w.H, w.N, w.d, sage.MODE_BF16)
    o = sage.attn_fwd(_dev(q, cuda_dev), _dev(k, cuda_dev), _dev(v, cuda_dev), sage.MODE_BF16, workspace=ws)
    assert sage.status(ws) == sage.OK
    got = bf16_to_np(o)
    assert np.all(np.isfinite(got))
    assert rel_l2(got, o1) <= REL_L2_BF16, rel_l2(got, o1)


def test_all_zero_inputs_give_zero_output(cuda_dev):
    from video_dit_quantized_b200 import sage
    z = np.zeros((1, 2, 333, 128), dtype=np.uint16)
    for mode in (sage.MODE_INT8_FP8, sage.MODE_BF16):
        o = sage.attn_fwd(_dev(z, cuda_dev), _dev(z, cuda_dev), _dev(z, cuda_dev), mode)
        got = bf16_to_np(o)
        assert np.all(got == 0.0), mode


def test_repeated_calls_are_deterministic(cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.Workload("det", 1, 4, 1500, 128, seed=41, outlier_frac=0.01)
    q, k, v = (_dev(a, cuda_dev) for a in synth.qkv_numpy(w))
    for mode in (sage.MODE_INT8_FP8, sage.MODE_BF16):
        a = sage.attn_fwd(q, k, v, mode)
        b = sage.attn_fwd(q, k, v, mode)
        torch.cuda.synchronize()
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("name", ["cogvideox2b", "wan1.3b_480p", "wan14b_720p"])
def test_full_size_sampled_rows(name, cuda_dev, big_inputs):
    """The benchmark's launch (one sage_attn_fwd over all heads); 48 sampled rows of three heads checked."""
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.WORKLOADS[name]
    q, k, v, qd, kd, vd = big_inputs(name)
    hs = sorted({0, w.H // 2, w.H - 1})
    rows = synth.sample_rows(w.seed + 99, w.N, 48)
    qh, kh, vh = heads(q, hs), heads(k, hs), heads(v, hs)
    _, o2, o1 = emul_and_exact(qh, kh, vh, rows)
    # quantized
    ws = sage.alloc_workspace(w.B, w.H, w.N, w.d, sage.MODE_INT8_FP8)
    o = sage.attn_fwd(qd, kd, vd, sage.MODE_INT8_FP8, workspace=ws)
    assert sage.status(ws) == sage.OK
    got = bf16_to_np(o[:, hs][:, :, torch.from_numpy(rows).long().to(cuda_dev)])
    check_quant(got, o2, o1, synth.bf16_bits_to_f32(vh), name)
    del o, ws
    # bf16
    ws = sage.alloc_workspace(w.B, w.H, w.N, w.d, sage.MODE_BF16)
    o = sage.attn_fwd(qd, kd, vd, sage.MODE_BF16, workspace=ws)
    assert sage.status(ws) == sage.OK
    got = bf16_to_np(o[:, hs][:, :, torch.from_numpy(rows).long().to(cuda_dev)])
    assert rel_l2(got, o1) <= REL_L2_BF16, rel_l2(got, o1)


def test_layer_stack_schedule(cuda_dev):
    """40 consecutive calls at the Wan-1.3B shape with H=40, seed = layer; layers
    0, 8, 16, 24, 32 in BF16 (per-layer selective quantization), the rest INT8/FP8.
    Every BF16 layer and INT8/FP8 layers 1, 20 and 39 are checked against the oracle
    on sampled rows of the first and last head."""
    import torch
    from video_dit_quantized_b200 import sage
    base = synth.WORKLOADS["layer_stack"]
    modes = sage.layer_schedule(synth.LAYER_STACK_LAYERS, synth.LAYER_STACK_FULL_PRECISION)
    assert modes == oracle.layer_schedule(synth.LAYER_STACK_LAYERS, synth.LAYER_STACK_FULL_PRECISION).tolist()
    ws = sage.alloc_workspace(base.B, base.H, base.N, base.d, sage.MODE_INT8_FP8)
    # every BF16 layer and three INT8/FP8 layers (first, middle, last) against the oracle
    checked = set(synth.LAYER_STACK_FULL_PRECISION) | {1, 20, 39}
    for layer, mode in enumerate(modes):
        w = base.with_seed(layer)
        q, k, v = synth.qkv_numpy(w)
        o = sage.attn_fwd(_dev(q, cuda_dev), _dev(k, cuda_dev), _dev(v, cuda_dev), mode, workspace=ws)
        assert torch.isfinite(o.float()).all(), layer
        if layer in checked:
            hs = [0, base.H - 1]
            rows = synth.sample_rows(layer, w.N, 16)
            got = bf16_to_np(o[:, hs][:, :, torch.from_numpy(rows).long().to(cuda_dev)])
            qh, kh, vh = heads(q, hs), heads(k, hs), heads(v, hs)
            if mode == sage.MODE_BF16:
                o1 = oracle.attn_exact(qh, kh, vh, rows)
                assert rel_l2(got, o1) <= REL_L2_BF16
            else:
                _, o2, o1 = emul_and_exact(qh, kh, vh, rows)
                check_quant(got, o2, o1, synth.bf16_bits_to_f32(vh), f"layer {layer}")
    assert sage.status(ws) == sage.OK


def _emul_tok(q, k, v, rows):
    pre = oracle.prepass(q, k, v, q_per_token=True)
    o2, _ = oracle.attn_emul(pre, rows, flags=oracle.EMUL_Q_PER_TOKEN)
    return o2, oracle.attn_exact(q, k, v, rows)


@pytest.mark.parametrize("w", small_workloads(), ids=lambda w: w.name)
def test_quantized_per_token_q_small_all_rows(w, cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    q, k, v = synth.qkv_numpy(w)
    o2, o1 = _emul_tok(q, k, v, np.arange(w.N, dtype=np.int32))
    qd, kd, vd = _dev(q, cuda_dev), _dev(k, cuda_dev), _dev(v, cuda_dev)
    ws = sage.alloc_workspace(w.B, w.H, w.N, w.d, sage.MODE_INT8_FP8_QTOKEN)
    o = sage.attn_fwd(qd, kd, vd, sage.MODE_INT8_FP8_QTOKEN, workspace=ws)
    assert sage.status(ws) == sage.OK
    check_quant(bf16_to_np(o), o2, o1, synth.bf16_bits_to_f32(v), w.name + " per-token Q")
    pre = sage.quantize_qk(qd, kd, vd, q_per_token=True)
    o_b = sage.attn_quantized(pre, w.N)
    torch.cuda.synchronize()
    assert torch.equal(o_b.view(torch.int16), o.view(torch.int16))


@pytest.mark.parametrize("name", ["cogvideox2b", "wan1.3b_480p", "wan14b_720p"])
def test_quantized_per_token_q_full_size_sampled(name, cuda_dev, big_inputs):
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.WORKLOADS[name]
    q, k, v, qd, kd, vd = big_inputs(name)
    hs = [0, w.H - 1]
    rows = synth.sample_rows(w.seed + 98, w.N, 32)
    o2, o1 = _emul_tok(heads(q, hs), heads(k, hs), heads(v, hs), rows)
    o = sage.attn_fwd(qd, kd, vd, sage.MODE_INT8_FP8_QTOKEN)
    got = bf16_to_np(o[:, hs][:, :, torch.from_numpy(rows).long().to(cuda_dev)])
    check_quant(got, o2, o1, synth.bf16_bits_to_f32(heads(v, hs)), name + " per-token Q")
