"""sage_attn_fwd_host: the call from pinned host memory, pipelined over chunks of
heads (copies of one chunk overlap the attention of another).  Every statistic
of the scheme is per head, so the result must equal the device call bit for bit."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("w", [synth.WORKLOADS["tiny"], synth.Workload("mid", 2, 5, 1500, 64, seed=61, outlier_frac=0.01),
                               synth.Workload("mid128", 1, 7, 2100, 128, seed=62)], ids=lambda w: w.name)
@pytest.mark.parametrize("chunk", [0, 1, 3])
def test_host_pipeline_matches_device_call(w, chunk, cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    qh, kh, vh = synth.qkv_torch(w, pin=True)
    qd, kd, vd = (t.to(cuda_dev) for t in (qh, kh, vh))
    for mode in (sage.MODE_INT8_FP8, sage.MODE_BF16, sage.MODE_INT8_FP8_QTOKEN):
        ref = sage.attn_fwd(qd, kd, vd, mode)
        oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
        sage.attn_fwd_host(qh, kh, vh, oh, mode, chunk_heads=chunk)
        torch.cuda.synchronize()
        assert torch.equal(oh.view(torch.int16), ref.cpu().view(torch.int16)), (mode, chunk)


def test_host_pipeline_rejects_small_workspace(cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.WORKLOADS["tiny"]
    qh, kh, vh = synth.qkv_torch(w, pin=True)
    oh = torch.empty_like(qh)
    ws = torch.zeros(256, dtype=torch.uint8, device=cuda_dev)
    with pytest.raises(sage.SageError) as e:
        sage.attn_fwd_host(qh, kh, vh, oh, sage.MODE_INT8_FP8, workspace=ws, chunk_heads=1)
    assert e.value.code == sage.EWORKSPACE
    # one chunk's workspace is not enough: two chunks are in flight
    one = sage.workspace_bytes(1, 1, w.N, w.d, sage.MODE_INT8_FP8)
    assert sage.host_workspace_bytes(w.B, w.H, w.N, w.d, sage.MODE_INT8_FP8, 1) == 2 * ((one + 255) // 256 * 256)
    ws = torch.zeros(one, dtype=torch.uint8, device=cuda_dev)
    with pytest.raises(sage.SageError) as e:
        sage.attn_fwd_host(qh, kh, vh, oh, sage.MODE_INT8_FP8, workspace=ws, chunk_heads=1)
    assert e.value.code == sage.EWORKSPACE


def test_host_pipeline_one_workspace_for_every_mode(cuda_dev):
    """A layer stack alternates modes on one host workspace (sized for the largest mode, per-token
    INT8/FP8): every call must find its chunks' status words where the previous call of another mode
    left them clean."""
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.Workload("stackmix", 1, 6, 1100, 128, seed=63)
    qh, kh, vh = synth.qkv_torch(w, pin=True)
    qd, kd, vd = (t.to(cuda_dev) for t in (qh, kh, vh))
    ws = sage.alloc_host_workspace(w.B, w.H, w.N, w.d, sage.MODE_INT8_FP8_QTOKEN, 2, cuda_dev)
    staging = tuple(torch.empty(qh.shape, dtype=torch.bfloat16, device=cuda_dev) for _ in range(4))
    for mode in (sage.MODE_INT8_FP8, sage.MODE_BF16, sage.MODE_INT8_FP8, sage.MODE_INT8_FP8_QTOKEN, sage.MODE_BF16):
        ref = sage.attn_fwd(qd, kd, vd, mode)
        oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
        sage.attn_fwd_host(qh, kh, vh, oh, mode, staging=staging, workspace=ws, chunk_heads=2)
        torch.cuda.synchronize()
        assert torch.equal(oh.view(torch.int16), ref.cpu().view(torch.int16)), mode
