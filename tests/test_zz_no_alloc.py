"""sage_quantize_qk_noalloc: the quantization prepass for callers that must not
allocate device memory while they run (a service that reserved all of HBM for
its own pool, or a latency-critical loop that cannot take the implicit
synchronisation of cudaMalloc / cudaFree).  Its scratch is a fixed array
inside the library; the caller passes only inputs and outputs.

Checked through the C ABI against the allocating entry point
(sage_quantize_qk): bit-exact, as every prepass result is, on two calls in a
row -- a larger problem, then a smaller one, so that anything the second call
wrongly took from the first call's leftovers in the shared array would show.
This file is collected last so that a run stopping at the first failure has
already run every other test.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


def _dev(a, device):
    import torch
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)


def _outputs_like(ref: dict):
    import torch
    return {k: torch.full_like(v, 0x55 if v.dtype in (torch.int8, torch.uint8) else float("nan"))
            for k, v in ref.items() if not k.startswith("_")}


def _assert_same(got: dict, ref: dict):
    import torch
    for name, r in ref.items():
        if name.startswith("_"):
            continue
        g = got[name]
        if g.dtype == torch.float32:
            assert torch.equal(g.view(torch.int32), r.view(torch.int32)), name
        else:
            assert torch.equal(g, r), name


def test_noalloc_prepass_matches_allocating_entry_point_twice(cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    workloads = [synth.Workload("first", 1, 6, 3000, 128, seed=51, outlier_frac=0.01, zero_k_channel=3),
                 synth.Workload("second", 2, 2, 700, 64, seed=52)]
    for w in workloads:
        q, k, v = (_dev(a, cuda_dev) for a in synth.qkv_numpy(w))
        ref = sage.quantize_qk(q, k, v)
        torch.cuda.synchronize()
        out = _outputs_like(ref)
        rc = sage.quantize_qk_noalloc(q, k, v, out)
        assert rc == sage.OK, sage.strerror(rc)
        torch.cuda.synchronize()
        _assert_same(out, ref)


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    B, H, N, d = 1, 40, 75600, 128
    assert sage.prepass_scratch_bytes(B, H, N, d) > sage.NOALLOC_SCRATCH_BYTES
    # validation happens before any pointer is used; 16-byte aligned dummies suffice
    t = torch.zeros(64, dtype=torch.uint8, device=cuda_dev)
    p = t.data_ptr()
    import ctypes
    args = [ctypes.c_void_p(p)] * 3 + [B, H, N, d] + [ctypes.c_void_p(p)] * 7 + [None]
    assert sage.LIB.sage_quantize_qk_noalloc(*args) == sage.EWORKSPACE
