"""GPU W8A16 and bf16 linear layers against the oracle.

The weight dequantization is bit-exact.  The bf16 GEMM sums fp32 products
on the tensor cores in an unspecified order, so each output is checked
against the exact (fp64) product within the recursive-summation bound
K * 2^-24 * sum_k |x_k w_k| (plus one fp32 rounding of the bias add and,
for bf16 output, half a bf16 ulp); a structural error (a dropped K step, a
wrong tile) exceeds it by orders of magnitude.  The relative L2 error over
all outputs must also stay within 16 * sqrt(K) * 2^-24, the statistical
size of fp32 summation error (random-walk growth) with a wide margin.  The op: the FFN section of the TMAP
write-up, whose quality fallback keeps the weights in 8 bits and computes
with 16-bit activations (W8A16).
"""
import numpy as np
import pytest

import oracle
import synth

pytestmark = pytest.mark.gpu


def _bf16_dev(a, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def _f(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _check(got32, got16, x, w, b, rows, K):
    """got32 fp32 [R, N], got16 bf16 bits [R, N] for the given rows of X."""
    exact = oracle.linear_bf16(x, w, b, rows)
    X = _f(x)[rows]
    W = _f(w)
    mag = np.abs(X) @ np.abs(W).T + (np.abs(_f(b))[None, :] if b is not None else 0)
    bound = (K + 2) * 2.0 ** -24 * mag + 1e-30
    err32 = np.abs(got32.astype(np.float64) - exact)
    assert np.all(err32 <= bound), float((err32 / bound).max())
    rel = np.linalg.norm(got32 - exact) / np.linalg.norm(exact)
    assert rel < 16 * np.sqrt(K) * 2.0 ** -24, rel
    g16 = _f(got16)
    assert np.all(np.abs(g16 - exact) <= bound + np.abs(g16) * 2.0 ** -8)


def test_dequant_bit_exact_ragged(cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.LinearWorkload("dq", 300, 128, 384, seed=21)
    _, wt, _ = synth.linear_numpy(w, "w")          # W [128, 384] -> treat as [R=128, K=384]
    x, _, _ = synth.linear_numpy(w, "x")            # X [300, 384]: ragged rows
    for a in (wt, x):
        codes, scales = oracle.quant_blocks_2d(a)
        got = sage.dequant_blocks_2d(torch.from_numpy(codes).to(cuda_dev), torch.from_numpy(scales).to(cuda_dev))
        torch.cuda.synchronize()
        np.testing.assert_array_equal(got.view(torch.int16).cpu().numpy().view(np.uint16),
                                      oracle.dequant_blocks_2d(codes, scales))


@pytest.mark.parametrize("shape", [(333, 384, 512), (1, 128, 64), (8197, 1280, 1024), (200, 384, 13824)],
                         ids=lambda s: "x".join(map(str, s)))
def test_linear_bf16_within_summation_bound(shape, cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    M, N, K = shape
    w = synth.LinearWorkload("bf", M, N, K, seed=M + N)
    x, wt, b = synth.linear_numpy(w)
    xd, wd, bd = _bf16_dev(x, cuda_dev), _bf16_dev(wt, cuda_dev), _bf16_dev(b, cuda_dev)
    st = torch.zeros(64, dtype=torch.int32, device=cuda_dev)
    y32 = sage.linear_bf16(xd, wd, bd, out_dtype=torch.float32, status=st)
    y16 = sage.linear_bf16(xd, wd, bd, status=st)
    assert sage.status(st) == sage.OK
    rows = np.arange(M) if M <= 512 else synth.sample_rows(w.seed + 3, M, 64)
    ridx = torch.from_numpy(np.asarray(rows)).long().to(cuda_dev)
    _check(y32[ridx].cpu().numpy(), y16[ridx].view(torch.int16).cpu().numpy().view(np.uint16), x, wt, b, rows, K)
    # no bias: the same products
    y0 = sage.linear_bf16(xd, wd, None, out_dtype=torch.float32)
    torch.cuda.synchronize()
    _check(y0[ridx].cpu().numpy(), y0[ridx].to(torch.bfloat16).view(torch.int16).cpu().numpy().view(np.uint16),
           x, wt, None, rows, K)


def test_linear_w8a16_equals_dequant_then_bf16(cuda_dev):
    """The W8A16 layer is the bf16 linear against the dequantized weights (bitwise, same kernel),
    and within the summation bound of the oracle's exact product."""
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.LINEAR_WORKLOADS["lin_multi"]
    x, wt, b = synth.linear_numpy(w)
    xd, bd = _bf16_dev(x, cuda_dev), _bf16_dev(b, cuda_dev)
    wq, sw = sage.quantize_blocks_2d(_bf16_dev(wt, cuda_dev))
    y = sage.linear_w8a16(xd, wq, sw, bd, out_dtype=torch.float32)
    deq = sage.dequant_blocks_2d(wq, sw)
    y_ref = sage.linear_bf16(xd, deq, bd, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(y, y_ref)
    wq_o, sw_o = oracle.quant_blocks_2d(wt)
    deq_o = oracle.dequant_blocks_2d(wq_o, sw_o)
    np.testing.assert_array_equal(deq.view(torch.int16).cpu().numpy().view(np.uint16), deq_o)
    rows = synth.sample_rows(w.seed + 4, w.M, 64)
    ridx = torch.from_numpy(rows).long().to(cuda_dev)
    got = y[ridx].cpu().numpy()
    _check(got, y[ridx].to(torch.bfloat16).view(torch.int16).cpu().numpy().view(np.uint16), x, deq_o, b, rows, w.K)
    # W8A16 is closer to the bf16 layer than W8A8 (only the weights are quantized)
    ex = oracle.linear_bf16(x, wt, b, rows)
    y8 = sage.linear_w8a8(*sage.quantize_blocks_2d(xd), wq, sw, bd, out_dtype=torch.float32)
    torch.cuda.synchronize()
    e16 = np.linalg.norm(got - ex) / np.linalg.norm(ex)
    e8 = np.linalg.norm(y8[ridx].cpu().numpy() - ex) / np.linalg.norm(ex)
    assert e16 < e8


def test_linear_bf16_full_size_sampled_rows(cuda_dev):
    """The Wan2.1-14B projection shape (75600 x 5120 x 5120), the benchmark's launch; 16 sampled rows."""
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.LINEAR_WORKLOADS["wan14b_720p_proj"]
    x, wt, b = synth.linear_numpy(w)
    xd, bd = _bf16_dev(x, cuda_dev), _bf16_dev(b, cuda_dev)
    wq, sw = sage.quantize_blocks_2d(_bf16_dev(wt, cuda_dev))
    y = sage.linear_w8a16(xd, wq, sw, bd, out_dtype=torch.float32)
    torch.cuda.synchronize()
    rows = synth.sample_rows(w.seed + 8, w.M, 16)
    deq_o = oracle.dequant_blocks_2d(*oracle.quant_blocks_2d(wt))
    got = y[torch.from_numpy(rows).long().to(cuda_dev)].cpu().numpy()
    got16 = torch.from_numpy(got).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    _check(got, got16, x, deq_o, b, rows, w.K)


def test_linear_bf16_forced_timeout_reports_and_recovers(cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.LINEAR_WORKLOADS["lin_tiny"]
    x, wt, b = synth.linear_numpy(w)
    xd, wd, bd = _bf16_dev(x, cuda_dev), _bf16_dev(wt, cuda_dev), _bf16_dev(b, cuda_dev)
    st = torch.zeros(64, dtype=torch.int32, device=cuda_dev)
    sage.dbg_linear_bf16_forced_timeout(xd, wd, st, timeout_cycles=2_000_000, bias=bd)
    assert sage.status(st) == sage.ETIMEOUT
    assert sage.status(st) == sage.OK
    y = sage.linear_bf16(xd, wd, bd, out_dtype=torch.float32, status=st)     # the context is still usable
    torch.cuda.synchronize()
    assert sage.status(st) == sage.OK
    _check(y.cpu().numpy(), y.to(torch.bfloat16).view(torch.int16).cpu().numpy().view(np.uint16), x, wt, b,
           np.arange(w.M), w.K)
