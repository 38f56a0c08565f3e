"""The debug build (libsage_debug.so: the same sources with SAGE_DEBUG, device-side
bounds checks that record a failure instead of trapping, entry points that
synchronise and return EBOUNDS) on small odd shapes.

Its checks must stay silent on every valid call and change no result: each
call through the debug build returns OK and equals the release build bit for
bit.  The one check that fails on purpose (the self-test kernel, which touches
no memory) must come back as EBOUNDS with its site and index."""
import contextlib
import ctypes

import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu

ODD = [synth.Workload(f"odd_n{n}_d{d}", 2, 3, n, d, seed=70 + n + d, outlier_frac=0.02)
       for n in (1, 127, 129, 385, 1000) for d in (64, 128)]


@contextlib.contextmanager
def debug_build():
    """Routes the binding's calls through libsage_debug.so."""
    from video_dit_quantized_b200 import sage
    old = sage.LIB
    sage.LIB = sage.debug_library()
    try:
        yield sage
    finally:
        sage.LIB = old


def _dev(a, device):
    import torch
    return torch.from_numpy(a.view(np.int16)).view(torch.bfloat16).to(device)


def _same(a, b):
    import torch
    torch.cuda.synchronize()
    return torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a,
                       b.view(torch.int16) if b.dtype == torch.bfloat16 else b)


def test_selftest_reports_its_site_and_index(cuda_dev):
    from video_dit_quantized_b200 import sage
    dbg = sage.debug_library()
    assert dbg.sage_dbg_bounds_selftest(None) == sage.EBOUNDS
    site, index = ctypes.c_int(), ctypes.c_longlong()
    assert dbg.sage_debug_last_failure(ctypes.byref(site), ctypes.byref(index)) == sage.OK
    assert (site.value, index.value) == (99, 1)
    assert sage.LIB.sage_dbg_bounds_selftest(None) == sage.EUNSUPPORTED
    # the record was cleared: a valid call afterwards is clean
    w = ODD[0]
    q, k, v = (_dev(a, cuda_dev) for a in synth.qkv_numpy(w))
    with debug_build() as s:
        s.attn_fwd(q, k, v, s.MODE_INT8_FP8)


@pytest.mark.parametrize("w", ODD, ids=lambda w: w.name)
def test_attention_and_prepass_clean_and_unchanged(w, cuda_dev):
    from video_dit_quantized_b200 import sage
    q, k, v = (_dev(a, cuda_dev) for a in synth.qkv_numpy(w))
    for mode in (sage.MODE_INT8_FP8, sage.MODE_BF16, sage.MODE_INT8_FP8_QTOKEN):
        ref = sage.attn_fwd(q, k, v, mode)
        with debug_build() as s:
            ws = s.alloc_workspace(w.B, w.H, w.N, w.d, mode)
            got = s.attn_fwd(q, k, v, mode, workspace=ws)           # raises on EBOUNDS
            assert s.status(ws) == s.OK
        assert _same(got, ref), (w.name, mode)
    for qtok in (False, True):
        ref = sage.quantize_qk(q, k, v, q_per_token=qtok)
        with debug_build() as s:
            got = s.quantize_qk(q, k, v, q_per_token=qtok)
        for name in ref:
            if not name.startswith("_"):
                assert _same(got[name], ref[name]), (w.name, qtok, name)


@pytest.mark.parametrize("P", [1, 2, 3])
def test_sequence_parallel_path_and_permutations_clean(P, cuda_dev):
    """The chunked-layout prepass and epilogue, and the four permutations, under the checks."""
    import torch
    from video_dit_quantized_b200 import sage
    B, Nl, Hl, d = 2, 129, 1, 64
    H, N = P * Hl, P * Nl
    g = torch.Generator().manual_seed(5 + P)
    x = torch.randn(B, Nl, H, d, generator=g).to(torch.bfloat16).to(cuda_dev)
    bufs = [torch.randn(P, B, Nl, Hl, d, generator=g).to(torch.bfloat16).to(cuda_dev) for _ in range(3)]
    for mode in (sage.MODE_INT8_FP8, sage.MODE_BF16):
        ref = torch.empty_like(bufs[0])
        sage.attn_fwd_seqpar(*bufs, mode, ref, P)
        out = torch.empty_like(bufs[0])
        with debug_build() as s:
            s.attn_fwd_seqpar(*bufs, mode, out, P)
        assert _same(out, ref), (P, mode)
    cases = [(x, (P, B, Nl, Hl, d), sage.ULYSSES_SEND), (bufs[0], (B, Nl, H, d), sage.ULYSSES_RECV_O),
             (bufs[0], (B, Hl, N, d), sage.ULYSSES_GATHER)]
    for src, shape, op in cases:
        ref = torch.empty(shape, dtype=torch.bfloat16, device=cuda_dev)
        sage.ulysses_permute(src, ref, B, Nl, H, d, P, op)
        got = torch.empty_like(ref)
        with debug_build() as s:
            s.ulysses_permute(src, got, B, Nl, H, d, P, op)
        assert _same(got, ref), op
    y = torch.randn(B, Hl, N, d, generator=g).to(torch.bfloat16).to(cuda_dev)
    ref = torch.empty(P, B, Nl, Hl, d, dtype=torch.bfloat16, device=cuda_dev)
    sage.ulysses_permute(y, ref, B, Nl, H, d, P, sage.ULYSSES_SCATTER)
    got = torch.empty_like(ref)
    with debug_build() as s:
        s.ulysses_permute(y, got, B, Nl, H, d, P, sage.ULYSSES_SCATTER)
    assert _same(got, ref)


def test_host_pipeline_and_no_alloc_prepass_clean(cuda_dev):
    import torch
    from video_dit_quantized_b200 import sage
    w = synth.Workload("odd_host", 1, 5, 385, 128, seed=77, outlier_frac=0.02)
    qh, kh, vh = synth.qkv_torch(w, pin=True)
    qd, kd, vd = (t.to(cuda_dev) for t in (qh, kh, vh))
    ref = sage.attn_fwd(qd, kd, vd, sage.MODE_INT8_FP8).cpu()
    oh = torch.empty(qh.shape, dtype=torch.bfloat16).pin_memory()
    with debug_build() as s:
        s.attn_fwd_host(qh, kh, vh, oh, s.MODE_INT8_FP8, chunk_heads=2)
    assert torch.equal(oh.view(torch.int16), ref.view(torch.int16))
    pre = sage.quantize_qk(qd, kd, vd)
    out = {name: torch.empty_like(t) for name, t in pre.items() if not name.startswith("_")}
    with debug_build() as s:
        assert s.quantize_qk_noalloc(qd, kd, vd, out) == s.OK
    for name in out:
        assert _same(out[name], pre[name]), name
