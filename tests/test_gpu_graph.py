"""The device entry points can be captured into a CUDA graph and replayed.

After one eager call per device (which sets the kernels' shared-memory
attributes), sage_attn_fwd (INT8/FP8 and BF16), sage_linear_w8a8 and
sage_linear_w8a16 enqueue only kernels on the caller's stream: no
allocation, no synchronisation.  Captured once and replayed, they must give
the same bits as the eager calls, on fresh inputs copied into the captured
buffers too.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


def _dev(a, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def test_attention_and_linear_replay_from_a_graph(cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.Workload("g", 1, 4, 1500, 128, seed=31, outlier_frac=0.01)
    q, k, v = (_dev(a, cuda_dev) for a in synth.qkv_numpy(w))
    lw = synth.LINEAR_WORKLOADS["lin_tiny"]
    x, wt, b = (_dev(a, cuda_dev) for a in synth.linear_numpy(lw))
    ws8 = sage.alloc_workspace(w.B, w.H, w.N, w.d, sage.MODE_INT8_FP8, cuda_dev)
    ws16 = sage.alloc_workspace(w.B, w.H, w.N, w.d, sage.MODE_BF16, cuda_dev)
    o8, o16 = torch.empty_like(q), torch.empty_like(q)
    xq = torch.empty((lw.M, lw.K), dtype=torch.int8, device=cuda_dev)
    sx = torch.empty(((lw.M + 127) // 128, lw.K // 128), dtype=torch.float32, device=cuda_dev)
    wq, sw = sage.quantize_blocks_2d(wt)
    y8 = torch.empty((lw.M, lw.N), dtype=torch.bfloat16, device=cuda_dev)
    y16 = torch.empty_like(y8)
    wsl = torch.empty(int(sage.LIB.sage_linear_w8a16_workspace_bytes(lw.N, lw.K)), dtype=torch.uint8,
                      device=cuda_dev)
    st = torch.zeros(64, dtype=torch.int32, device=cuda_dev)

    def run(stream=None):
        sage.attn_fwd(q, k, v, sage.MODE_INT8_FP8, o=o8, workspace=ws8, stream=stream)
        sage.attn_fwd(q, k, v, sage.MODE_BF16, o=o16, workspace=ws16, stream=stream)
        sage.quantize_blocks_2d(x, xq, sx, stream=stream)
        sage.linear_w8a8(xq, sx, wq, sw, b, y=y8, status=st, stream=stream)
        sage.linear_w8a16(x, wq, sw, b, y=y16, workspace=wsl, status=st, stream=stream)

    run()                                                    # eager: sets kernel attributes
    torch.cuda.synchronize()
    ref = [t.clone() for t in (o8, o16, y8, y16)]
    for t in (o8, o16, y8, y16):
        t.zero_()
    g = torch.cuda.CUDAGraph()
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            run(stream=side)
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    for a, r in zip((o8, o16, y8, y16), ref):
        assert torch.equal(a.view(torch.int16), r.view(torch.int16))
    assert sage.status(ws8) == sage.OK and sage.status(ws16) == sage.OK and sage.status(st) == sage.OK

    # new inputs copied into the captured buffers: the replay follows them
    w2 = w.with_seed(32)
    for dst, src in zip((q, k, v), synth.qkv_numpy(w2)):
        dst.copy_(_dev(src, cuda_dev))
    run()
    torch.cuda.synchronize()
    ref2 = [t.clone() for t in (o8, o16)]
    g.replay()
    torch.cuda.synchronize()
    for a, r in zip((o8, o16), ref2):
        assert torch.equal(a.view(torch.int16), r.view(torch.int16))
    assert not torch.equal(ref2[0].view(torch.int16), ref[0].view(torch.int16))
