"""Failure detection without a GPU fault: the attention kernel's bounded waits.

A test hook makes the MMA thread wait on a barrier no one arrives on, with a
short limit (about 10 ms of SM clocks).  The kernel must record SAGE_ETIMEOUT
in the status word, drain its in-flight copies, free tensor memory and
return; the context stays usable and the next call is correct.
"""
import numpy as np
import pytest

import synth
from _util import bf16_to_np

pytestmark = pytest.mark.gpu


def _dev(a, device):
    import torch
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)


def test_forced_timeout_reports_and_recovers(cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.WORKLOADS["tiny"]
    q, k, v = (_dev(a, cuda_dev) for a in synth.qkv_numpy(w))
    pre = sage.quantize_qk(q, k, v)
    status = torch.zeros(64, dtype=torch.int32, device=cuda_dev)
    sage.dbg_attn_forced_timeout(pre, w.N, status, timeout_cycles=20_000_000)
    assert sage.status(status) == sage.ETIMEOUT
    assert sage.status(status) == sage.OK          # read-and-clear
    # the context is still usable and results are right
    ref = sage.attn_quantized(pre, w.N, status=status)
    again = sage.attn_fwd(q, k, v, sage.MODE_INT8_FP8)
    torch.cuda.synchronize()
    assert sage.status(status) == sage.OK
    assert torch.equal(ref.view(torch.int16), again.view(torch.int16))
    assert np.all(np.isfinite(bf16_to_np(again)))


def test_host_side_errors_do_not_touch_the_device(cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    q = torch.zeros((1, 1, 128, 96), dtype=torch.bfloat16, device=cuda_dev)
    with pytest.raises(sage.SageError) as e:
        sage.attn_fwd(q, q, q, sage.MODE_BF16, workspace=torch.zeros(256, dtype=torch.uint8, device=cuda_dev))
    assert e.value.code == sage.EUNSUPPORTED
    q = torch.zeros((1, 1, 128, 128), dtype=torch.bfloat16, device=cuda_dev)
    with pytest.raises(sage.SageError) as e:
        sage.attn_fwd(q, q, q, sage.MODE_INT8_FP8, workspace=torch.zeros(256, dtype=torch.uint8, device=cuda_dev))
    assert e.value.code == sage.EWORKSPACE
    torch.cuda.synchronize()
