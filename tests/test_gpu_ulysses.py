"""Ulysses layout copies and the fused sequence-parallel attention on the GPU, and the whole
exchange emulated on one GPU.

The four row copies of sage_ulysses_permute equal independent torch
reshape/permute references bit for bit, dense and with a strided [P] side.
sage_attn_fwd_seqpar, which reads q, k, v from the exchange layout
[P][B][Nl][Hl][d] and writes O into it (the quantization prepass walks the
chunks, the attention epilogue scatters its rows), gives the same bits as
sage_attn_fwd on the gathered heads, in every mode, with ragged chunks.  With
P ranks emulated on one device (the all-to-all done by slicing the P send
buffers), the sequence-parallel path gives the same bits as one attention
call over all heads: attention has no cross-head term and the kernels treat
every (b, h) alike.  The pattern is the DeepSpeed-Ulysses sequence
parallelism of the TMAP write-up ("Optimising multi-GPU parallelism").
"""
import numpy as np
import pytest

import synth
from _util import ulysses_ref_permute

pytestmark = pytest.mark.gpu


def _bf16(a, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


@pytest.mark.parametrize("B,Nl,H,d,P", [(1, 96, 8, 128, 1), (1, 100, 8, 128, 2), (2, 37, 12, 64, 4),
                                        (1, 1181, 40, 128, 8)])
def test_permutes_match_reference(B, Nl, H, d, P, cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    g = torch.Generator(device="cpu").manual_seed(B * 1000 + Nl + H + P)
    Hl, N = H // P, P * Nl
    shapes_in = {0: (B, Nl, H, d), 1: (P, B, Nl, Hl, d), 2: (P, B, Nl, Hl, d), 3: (B, Hl, N, d)}
    shapes_out = {0: (P, B, Nl, Hl, d), 1: (B, Nl, H, d), 2: (B, Hl, N, d), 3: (P, B, Nl, Hl, d)}
    for op in range(4):
        src = torch.randn(shapes_in[op], generator=g).to(torch.bfloat16).to(cuda_dev)
        got = torch.empty(shapes_out[op], dtype=torch.bfloat16, device=cuda_dev)
        sage.ulysses_permute(src, got, B, Nl, H, d, P, op)
        want = ulysses_ref_permute(src, torch.empty_like(got), B, Nl, H, d, P, op)
        torch.cuda.synchronize()
        assert torch.equal(got.view(torch.int16), want.view(torch.int16)), op
    # strided [P] side: q, k, v interleaved as [P][3][B][Nl][Hl][d]
    dense = B * Hl * Nl
    x = torch.randn((3, B, Nl, H, d), generator=g).to(torch.bfloat16).to(cuda_dev)
    buf = torch.zeros((P, 3, B, Nl, Hl, d), dtype=torch.bfloat16, device=cuda_dev)
    for t in range(3):
        sage.ulysses_permute(x[t], buf, B, Nl, H, d, P, sage.ULYSSES_SEND, chunk_rows=3 * dense, base_rows=t * dense)
    back = torch.empty_like(x)
    for t in range(3):
        want = ulysses_ref_permute(x[t], torch.empty((P, B, Nl, Hl, d), dtype=torch.bfloat16, device=cuda_dev),
                                   B, Nl, H, d, P, 0)
        assert torch.equal(buf[:, t].view(torch.int16), want.view(torch.int16))
        sage.ulysses_permute(buf, back[t], B, Nl, H, d, P, sage.ULYSSES_RECV_O, chunk_rows=3 * dense,
                             base_rows=t * dense)
    torch.cuda.synchronize()
    assert torch.equal(back.view(torch.int16), x.view(torch.int16))       # RECV_O inverts SEND


@pytest.mark.parametrize("mode_name,P,Nl,Hl,d,B", [("int8_fp8", 8, 1181, 2, 128, 1), ("int8_fp8", 3, 333, 3, 64, 1),
                                                   ("int8_fp8_qtoken", 4, 257, 2, 128, 1),
                                                   ("bf16", 8, 1181, 2, 128, 1), ("bf16", 1, 640, 4, 64, 1),
                                                   ("int8_fp8", 1, 1000, 3, 128, 1), ("int8_fp8", 2, 300, 3, 64, 2),
                                                   ("int8_fp8_qtoken", 3, 129, 1, 128, 3), ("bf16", 2, 200, 2, 128, 2)])
def test_seqpar_equals_plain_attention(mode_name, P, Nl, Hl, d, B, cuda_dev):
    """The fused chunk-layout call gives bitwise the plain call's output on the gathered heads
    (several batch elements too: the chunk rows interleave b and the local heads)."""
    import torch
    from video_dit_quantized_b200 import sage
    mode = {"int8_fp8": sage.MODE_INT8_FP8, "int8_fp8_qtoken": sage.MODE_INT8_FP8_QTOKEN,
            "bf16": sage.MODE_BF16}[mode_name]
    N, H = P * Nl, P * Hl
    w = synth.Workload("sp", B, Hl, N, d, seed=P * 10 + Hl, outlier_frac=0.01)
    q, k, v = (_bf16(a, cuda_dev) for a in synth.qkv_numpy(w))             # plain [B, Hl, N, d]
    scat = lambda t: ulysses_ref_permute(t, torch.empty((P, B, Nl, Hl, d), dtype=t.dtype, device=cuda_dev),
                                         B, Nl, H, d, P, 3)
    qc, kc, vc = scat(q), scat(k), scat(v)
    ws = sage.alloc_seqpar_workspace(P, B, Nl, Hl, d, mode, cuda_dev)
    oc = sage.attn_fwd_seqpar(qc, kc, vc, mode, P=P, workspace=ws)
    assert sage.status(ws) == sage.OK
    ref = sage.attn_fwd(q, k, v, mode)
    torch.cuda.synchronize()
    assert torch.equal(oc.view(torch.int16), scat(ref).view(torch.int16))


@pytest.mark.parametrize("mode_name,P", [("int8_fp8", 4), ("bf16", 2), ("int8_fp8", 8), ("int8_fp8", 1)])
def test_emulated_ranks_equal_one_call(mode_name, P, cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    from video_dit_quantized_b200.ulysses import UlyssesAttention
    mode = {"int8_fp8": sage.MODE_INT8_FP8, "bf16": sage.MODE_BF16}[mode_name]
    w = synth.Workload("uly", 1, 8, 8 * 160, 128, seed=5 + P, outlier_frac=0.01)
    q, k, v = (_bf16(a, cuda_dev) for a in synth.qkv_numpy(w))            # [B, H, N, d]
    ref = sage.attn_fwd(q, k, v, mode)
    Nl = w.N // P
    seq = [t.permute(0, 2, 1, 3).contiguous() for t in (q, k, v)]         # [B, N, H, d]

    # P ranks on one device; the all-to-all is done by hand once every rank has sent
    sent = {}

    def make_a2a(rank):
        def a2a(out, inp):
            sent[(rank, id(out))] = (out, inp)
            return None
        return a2a

    ranks = [UlyssesAttention(w.B, Nl, w.H, w.d, P, mode=mode, device=cuda_dev, a2a=make_a2a(r))
             for r in range(P)]

    def exchange():
        # rank r receives chunk r of every rank's send buffer, in rank order
        # (one rank sends nothing: its exchange is the identity)
        if not sent:
            return
        outs = {}
        for (r, _), (out, inp) in sent.items():
            outs.setdefault(r, []).append((out, inp))
        for slot in range(len(outs[0])):
            for r in range(P):
                out_r = outs[r][slot][0]
                for src in range(P):
                    out_r[src].copy_(outs[src][slot][1][r])
        sent.clear()

    for r, ua in enumerate(ranks):
        for t, x in zip("qkv", seq):
            ua.send(t, x[:, r * Nl:(r + 1) * Nl].contiguous())
    exchange()
    for ua in ranks:
        ua.attend_local()
    exchange()
    outs = [ua.finish().clone() for ua in ranks]
    torch.cuda.synchronize()
    got = torch.cat(outs, dim=1).permute(0, 2, 1, 3)                      # back to [B, H, N, d]
    assert torch.equal(got.contiguous().view(torch.int16), ref.view(torch.int16))


def test_single_rank_nccl_exchange(cuda_dev):
    """A one-rank NCCL group: the layer runs with no collective (the exchange of one rank is the
    identity) and equals one attention call; the default exchange itself, an asynchronous
    all_to_all_single on the group, moves a buffer in the layer's send layout unchanged."""
    import os
    import socket

    import torch
    import torch.distributed as dist
    from video_dit_quantized_b200 import sage
    from video_dit_quantized_b200.ulysses import UlyssesAttention
    w = synth.Workload("uly1", 1, 4, 640, 128, seed=9, outlier_frac=0.01)
    q, k, v = (_bf16(a, cuda_dev) for a in synth.qkv_numpy(w))
    ref = sage.attn_fwd(q, k, v, sage.MODE_INT8_FP8)
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    store = dist.TCPStore("127.0.0.1", port, 1, True)
    group_made = False
    try:
        if not dist.is_initialized():
            dist.init_process_group("nccl", store=store, rank=0, world_size=1, device_id=cuda_dev)
            group_made = True
        ua = UlyssesAttention(w.B, w.N, w.H, w.d, 1, mode=sage.MODE_INT8_FP8, device=cuda_dev)
        out = ua(*(t.permute(0, 2, 1, 3).contiguous() for t in (q, k, v)))
        torch.cuda.synchronize()
        assert torch.equal(out.permute(0, 2, 1, 3).contiguous().view(torch.int16), ref.view(torch.int16))
        from video_dit_quantized_b200.ulysses import _default_a2a
        src = q.permute(0, 2, 1, 3).contiguous().view(1, w.B, w.N, w.H, w.d)
        dst = torch.empty_like(src)
        _default_a2a(None)(dst, src).wait()
        torch.cuda.synchronize()
        assert torch.equal(dst.view(torch.int16), src.view(torch.int16))
    finally:
        if group_made:
            dist.destroy_process_group()
