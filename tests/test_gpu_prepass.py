"""GPU prepass (K mean, K smoothing + per-block INT8, per-block INT8 Q,
per-channel FP8 V) against the oracle: bit-exact codes, equal fp32 scales and
means, zero padding.  Scheme: page 1 of the TMAP write-up, "Attention
performance optimisation" (SageAttention, zero-channel fix)."""
import numpy as np
import pytest

import oracle
import synth
from _util import heads, small_workloads

pytestmark = pytest.mark.gpu


def _dev(a, device):
    import torch
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)


def _f32bits(t):
    return t.detach().cpu().numpy().view(np.uint32)


def compare_prepass(pre_g: dict, pre_o: dict, N: int, hs=None):
    """pre_g: GPU tensors for all heads; pre_o: oracle arrays for heads hs (all if None)."""
    sel = (lambda t: t.detach().cpu().numpy()) if hs is None else (lambda t: t.detach().cpu().numpy()[:, list(hs)])
    q8, k8, vt = sel(pre_g["q_i8"]), sel(pre_g["k_i8"]), sel(pre_g["v_f8t"])
    np.testing.assert_array_equal(q8[:, :, :N], pre_o["q_i8"])
    np.testing.assert_array_equal(k8[:, :, :N], pre_o["k_i8"])
    assert not q8[:, :, N:].any() and not k8[:, :, N:].any(), "padding rows must be zero"
    v8 = np.swapaxes(vt, 2, 3)
    np.testing.assert_array_equal(v8[:, :, :N], pre_o["v_f8"])
    assert not v8[:, :, N:].any(), "padding tokens must be zero"
    for name in ("q_scale", "k_scale", "k_mean", "v_scale"):
        g = sel(pre_g[name]).view(np.uint32)
        np.testing.assert_array_equal(g, pre_o[name].view(np.uint32), err_msg=name)


@pytest.mark.parametrize("w", small_workloads(), ids=lambda w: w.name)
def test_prepass_bit_exact_small(w, cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    q, k, v = synth.qkv_numpy(w)
    pre_o = oracle.prepass(q, k, v)
    pre_g = sage.quantize_qk(_dev(q, cuda_dev), _dev(k, cuda_dev), _dev(v, cuda_dev))
    torch.cuda.synchronize()
    compare_prepass(pre_g, pre_o, w.N)
    # zero guard: no NaN anywhere
    for name in ("q_scale", "k_scale", "k_mean", "v_scale"):
        assert torch.isfinite(pre_g[name]).all()


def test_prepass_all_zero_inputs(cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    z = np.zeros((1, 2, 300, 128), dtype=np.uint16)
    pre_g = sage.quantize_qk(_dev(z, cuda_dev), _dev(z, cuda_dev), _dev(z, cuda_dev))
    torch.cuda.synchronize()
    for name in ("q_i8", "k_i8", "v_f8t", "q_scale", "k_scale", "k_mean", "v_scale"):
        assert not pre_g[name].bool().any(), name


@pytest.mark.parametrize("name", ["cogvideox2b", "wan1.3b_480p", "wan14b_720p"])
def test_prepass_bit_exact_full_size(name, cuda_dev, big_inputs):
    """Full-size call on the device; three heads re-derived by the oracle."""
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.WORKLOADS[name]
    q, k, v, qd, kd, vd = big_inputs(name)
    pre_g = sage.quantize_qk(qd, kd, vd)
    torch.cuda.synchronize()
    hs = sorted({0, w.H // 2, w.H - 1})
    pre_o = oracle.prepass(heads(q, hs), heads(k, hs), heads(v, hs))
    compare_prepass(pre_g, pre_o, w.N, hs)


@pytest.mark.parametrize("w", small_workloads(), ids=lambda w: w.name)
def test_prepass_per_token_q_bit_exact(w, cuda_dev):
    """The finer Q granularity: one INT8 scale per token (amax of its d channels / 127)."""
    import torch
    from video_dit_quantized_b200 import sage
    q, k, v = synth.qkv_numpy(w)
    pre_o = oracle.prepass(q, k, v, q_per_token=True)
    pre_g = sage.quantize_qk(_dev(q, cuda_dev), _dev(k, cuda_dev), _dev(v, cuda_dev), q_per_token=True)
    torch.cuda.synchronize()
    qs = pre_g["q_scale"].cpu().numpy()
    np.testing.assert_array_equal(qs[:, :, :w.N].view(np.uint32), pre_o["q_scale"].view(np.uint32))
    assert not qs[:, :, w.N:].any()
    np.testing.assert_array_equal(pre_g["q_i8"].cpu().numpy()[:, :, :w.N], pre_o["q_i8"])
    # K and V are the same as in the per-block prepass
    ref = oracle.prepass(q, k, v)
    for name in ("k_scale", "k_mean", "v_scale"):
        np.testing.assert_array_equal(pre_g[name].cpu().numpy().view(np.uint32), ref[name].view(np.uint32))
