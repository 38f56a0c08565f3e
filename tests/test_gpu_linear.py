"""GPU W8A8 linear layer (128 x 128 block scales) against the oracle.

The quantizer's codes and scales are bit-exact; the GEMM output is bit-exact
too (bf16 and fp32): the integer block products are exact on both sides and
both take the same fp32 roundings in the same order (block scale product,
one fused multiply-add per K block in ascending order, bias add, bf16 RNE).
The op: the DiT's linear layers in 8 bits with a 128 x 128 per-block
quantization operator (page 1 of the TMAP write-up, "FFN performance
optimisation / linear-layer quantization").
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu


def _bf16_dev(a, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def _bits(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _case(w, device):
    x, wt, b = synth.linear_numpy(w)
    return x, wt, b, _bf16_dev(x, device), _bf16_dev(wt, device), _bf16_dev(b, device)


def test_quantize_blocks_2d_bit_exact_ragged(cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.LINEAR_WORKLOADS["lin_tiny"]
    x, _, _ = synth.linear_numpy(w, "x")
    x = x.copy()
    x[128:256, 256:384] = 0                                  # one all-zero block
    codes, scales = sage.quantize_blocks_2d(_bf16_dev(x, cuda_dev))
    torch.cuda.synchronize()
    c_o, s_o = oracle.quant_blocks_2d(x)
    np.testing.assert_array_equal(codes.cpu().numpy(), c_o)
    np.testing.assert_array_equal(scales.cpu().numpy().view(np.uint32), s_o.view(np.uint32))
    assert scales[1, 2].item() == 0.0


@pytest.mark.parametrize("name", ["lin_tiny", "lin_multi"])
@pytest.mark.parametrize("with_bias", [True, False])
def test_linear_bit_exact(name, with_bias, cuda_dev):
    """Every output of the ragged case; sampled rows of the multi-wave case (more tiles than SMs)."""
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.LINEAR_WORKLOADS[name]
    x, wt, b, xd, wd, bd = _case(w, cuda_dev)
    xq, sx = sage.quantize_blocks_2d(xd)
    wq, sw = sage.quantize_blocks_2d(wd)
    st = torch.zeros(64, dtype=torch.int32, device=cuda_dev)
    y16 = sage.linear_w8a8(xq, sx, wq, sw, bd if with_bias else None, status=st)
    y32 = sage.linear_w8a8(xq, sx, wq, sw, bd if with_bias else None, out_dtype=torch.float32, status=st)
    assert sage.status(st) == sage.OK
    xq_o, sx_o = oracle.quant_blocks_2d(x)
    wq_o, sw_o = oracle.quant_blocks_2d(wt)
    rows = np.arange(w.M, dtype=np.int32) if w.M <= 512 else synth.sample_rows(w.seed + 5, w.M, 96)
    y_o, yb_o = oracle.linear_w8a8(xq_o, sx_o, wq_o, sw_o, b if with_bias else None, rows)
    ridx = torch.from_numpy(rows).long().to(cuda_dev)
    np.testing.assert_array_equal(y32[ridx].cpu().numpy().view(np.uint32), y_o.view(np.uint32))
    np.testing.assert_array_equal(_bits(y16[ridx]), yb_o)


def test_linear_long_k_scale_windows(cuda_dev):
    """K = 13824 (the FFN-down depth: 108 K blocks, so the per-lane scale windows roll over three
    times), ragged M and an odd multiple of 128 in N; every output, fp32 and bf16."""
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.LinearWorkload("long_k", 200, 384, 13824, seed=11)
    x, wt, b, xd, wd, bd = _case(w, cuda_dev)
    xq, sx = sage.quantize_blocks_2d(xd)
    wq, sw = sage.quantize_blocks_2d(wd)
    y32 = sage.linear_w8a8(xq, sx, wq, sw, bd, out_dtype=torch.float32)
    y16 = sage.linear_w8a8(xq, sx, wq, sw, bd)
    torch.cuda.synchronize()
    xq_o, sx_o = oracle.quant_blocks_2d(x)
    wq_o, sw_o = oracle.quant_blocks_2d(wt)
    np.testing.assert_array_equal(sx.cpu().numpy().view(np.uint32), sx_o.view(np.uint32))
    y_o, yb_o = oracle.linear_w8a8(xq_o, sx_o, wq_o, sw_o, b)
    np.testing.assert_array_equal(y32.cpu().numpy().view(np.uint32), y_o.view(np.uint32))
    np.testing.assert_array_equal(_bits(y16), yb_o)


def test_linear_minimal_shape_and_determinism(cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.LinearWorkload("one", 1, 128, 128, seed=9)
    x, wt, b, xd, wd, bd = _case(w, cuda_dev)
    xq, sx = sage.quantize_blocks_2d(xd)
    wq, sw = sage.quantize_blocks_2d(wd)
    y1 = sage.linear_w8a8(xq, sx, wq, sw, bd, out_dtype=torch.float32)
    y2 = sage.linear_w8a8(xq, sx, wq, sw, bd, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2)
    y_o, _ = oracle.linear_w8a8(*oracle.quant_blocks_2d(x), *oracle.quant_blocks_2d(wt), b)
    np.testing.assert_array_equal(y1.cpu().numpy().view(np.uint32), y_o.view(np.uint32))


def test_linear_zero_operands(cuda_dev):
    """All-zero X: every block scale 0, every output equals the bias."""
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.LINEAR_WORKLOADS["lin_tiny"]
    _, wt, b = synth.linear_numpy(w)
    xd = torch.zeros((w.M, w.K), dtype=torch.bfloat16, device=cuda_dev)
    xq, sx = sage.quantize_blocks_2d(xd)
    wq, sw = sage.quantize_blocks_2d(_bf16_dev(wt, cuda_dev))
    y = sage.linear_w8a8(xq, sx, wq, sw, _bf16_dev(b, cuda_dev))
    torch.cuda.synchronize()
    assert not sx.bool().any()
    assert np.array_equal(_bits(y), np.broadcast_to(b, (w.M, w.N)))


def test_linear_full_size_sampled_rows(cuda_dev):
    """The Wan2.1-14B projection shape (75600 x 5120 x 5120), the benchmark's launch; 24 sampled rows."""
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.LINEAR_WORKLOADS["wan14b_720p_proj"]
    x, wt, b, xd, wd, bd = _case(w, cuda_dev)
    xq, sx = sage.quantize_blocks_2d(xd)
    wq, sw = sage.quantize_blocks_2d(wd)
    y = sage.linear_w8a8(xq, sx, wq, sw, bd)
    torch.cuda.synchronize()
    rows = synth.sample_rows(w.seed + 6, w.M, 24)
    blocks = np.unique(rows // 128)
    # the oracle quantizes only the row blocks that hold sampled rows (the scales are per block)
    xs = np.concatenate([x[r * 128:(r + 1) * 128] for r in blocks])
    xq_o, sx_o = oracle.quant_blocks_2d(xs)
    wq_o, sw_o = oracle.quant_blocks_2d(wt)
    local = np.array([np.searchsorted(blocks, r // 128) * 128 + r % 128 for r in rows], dtype=np.int32)
    _, yb_o = oracle.linear_w8a8(xq_o, sx_o, wq_o, sw_o, b, local)
    got = _bits(y[torch.from_numpy(rows).long().to(cuda_dev)])
    np.testing.assert_array_equal(got, yb_o)
    # the quantized codes of those rows and every weight code match as well
    ridx = torch.from_numpy(rows).long().to(cuda_dev)
    np.testing.assert_array_equal(xq[ridx].cpu().numpy(), xq_o[local])
    np.testing.assert_array_equal(wq.cpu().numpy(), wq_o)


def test_linear_forced_timeout_reports_and_recovers(cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.LINEAR_WORKLOADS["lin_tiny"]
    _, _, _, xd, wd, bd = _case(w, cuda_dev)
    xq, sx = sage.quantize_blocks_2d(xd)
    wq, sw = sage.quantize_blocks_2d(wd)
    st = torch.zeros(64, dtype=torch.int32, device=cuda_dev)
    sage.dbg_linear_forced_timeout(xq, sx, wq, sw, st, timeout_cycles=2_000_000, bias=bd)
    assert sage.status(st) == sage.ETIMEOUT
    assert sage.status(st) == sage.OK                        # read-and-clear
    y = sage.linear_w8a8(xq, sx, wq, sw, bd, status=st)      # the context is still usable
    torch.cuda.synchronize()
    assert sage.status(st) == sage.OK
    assert torch.isfinite(y.float()).all()
