"""Thin ctypes binding of the sage C ABI (include/sage.h).

Argument marshalling only: every step of the attention path runs in the
CUDA kernels of libsage.so.  torch is used for device memory and streams.
There is no fallback: if the library cannot be loaded, importing this module
raises.
"""
from __future__ import annotations

import ctypes
import os
import re

from . import build as _build

MODE_BF16 = 0
MODE_INT8_FP8 = 1
MODE_INT8_FP8_QTOKEN = 2
DTYPE_BF16 = 0
DTYPE_F32 = 1
BLK = 128
P_SCALE = 448.0

OK, EINVAL, EUNSUPPORTED, ELAUNCH, EWORKSPACE, ETIMEOUT, EBOUNDS = 0, -1, -2, -3, -4, -5, -6
SELECT_EVERY_ITERATION, SELECT_MEAN = 0, 1

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "sage.h")


class SageError(RuntimeError):
    def __init__(self, code: int, what: str):
        self.code = code
        super().__init__(f"{what}: {strerror(code)} ({code})")


def load_library(path: str) -> ctypes.CDLL:
    """Loads a build of the library (libsage.so, or libsage_debug.so) with the C prototypes set."""
    if not os.path.exists(path):
        raise ImportError(f"{os.path.basename(path)} is not built ({path}); run video_dit_quantized_b200.build.build()")
    lib = ctypes.CDLL(path)
    vp, i32, sz, ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_longlong
    sig = {
        "sage_workspace_bytes": (sz, [i32, i32, i32, i32, i32]),
        "sage_prepass_scratch_bytes": (sz, [i32, i32, i32, i32]),
        "sage_quantize_qk": (i32, [vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "sage_attn_quantized": (i32, [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, vp]),
        "sage_attn_fwd": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, sz, vp]),
        "attn_layer_schedule": (i32, [i32, vp, i32, vp]),
        "sage_status": (i32, [vp, vp]),
        "sage_strerror": (ctypes.c_char_p, [i32]),
        "sage_device_check": (i32, []),
        "sage_dbg_qk_tiles": (i32, [vp, vp, i32, i32, i32, i32, vp, i32, vp, vp]),
        "sage_dbg_pv_tile": (i32, [vp, vp, i32, i32, vp, vp]),
        "sage_dbg_qk_bf16_tile": (i32, [vp, vp, i32, vp, vp]),
        "sage_dbg_attn_forced_timeout": (i32, [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, ll, vp]),
        "sage_quantize_qk_noalloc": (i32, [vp, vp, vp, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp]),
        "sage_attn_fwd_host": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, sz, i32, vp]),
        "sage_quantize_qk_ex": (i32, [vp, vp, vp, i32, i32, i32, i32, i32, vp, vp, vp, vp, vp, vp, vp, vp, sz, vp]),
        "sage_attn_quantized_ex": (i32, [vp, vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, i32, vp, vp]),
        "sage_error_scratch_bytes": (sz, [i32, i32]),
        "sage_attn_error_stats": (i32, [vp, vp, i32, i32, i32, i32, vp, vp, sz, vp]),
        "sage_attn_rel_l2": (i32, [vp, vp, i32, i32, i32, i32, vp, vp, sz, vp]),
        "sage_select_full_precision_layers": (i32, [vp, i32, i32, ctypes.c_double, i32, vp, vp]),
        "sage_quantize_blocks_2d": (i32, [vp, i32, i32, vp, vp, vp]),
        "sage_linear_w8a8": (i32, [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, vp]),
        "sage_dbg_linear_forced_timeout": (i32, [vp, vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, ll, vp]),
        "sage_dequant_blocks_2d": (i32, [vp, vp, i32, i32, vp, vp]),
        "sage_linear_bf16": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, vp, vp]),
        "sage_linear_w8a16_workspace_bytes": (sz, [i32, i32]),
        "sage_linear_w8a16": (i32, [vp, vp, vp, vp, vp, i32, i32, i32, i32, vp, sz, vp, vp]),
        "sage_ulysses_permute": (i32, [vp, vp, i32, i32, i32, i32, i32, i32, ll, ll, vp]),
        "sage_seqpar_workspace_bytes": (sz, [i32, i32, i32, i32, i32, i32]),
        "sage_attn_fwd_seqpar": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, i32, i32, vp, sz, vp]),
        "sage_host_chunk_heads": (i32, [i32, i32, i32, i32]),
        "sage_host_workspace_bytes": (sz, [i32, i32, i32, i32, i32, i32]),
        "sage_debug_build": (i32, []),
        "sage_debug_last_failure": (i32, [vp, vp]),
        "sage_dbg_bounds_selftest": (i32, [vp]),
        "sage_dbg_mma_peak": (i32, [i32, i32, i32, vp, i32, vp, vp]),
        "sage_dbg_linear_bf16_forced_timeout": (i32, [vp, vp, vp, vp, i32, i32, i32, i32, vp, ll, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(lib, name)
        f.restype = res
        f.argtypes = args
    return lib


LIB = load_library(_build.LIB_PATH)
_DEBUG_LIB = None


def debug_library() -> ctypes.CDLL:
    """libsage_debug.so (the same sources built with SAGE_DEBUG: device-side bounds checks, entry points
    that synchronise and return EBOUNDS), loaded once; raises ImportError if it is not built."""
    global _DEBUG_LIB
    if _DEBUG_LIB is None:
        _DEBUG_LIB = load_library(_build.DEBUG_LIB_PATH)
    return _DEBUG_LIB


def header_functions() -> list[str]:
    """Names of the functions declared in include/sage.h."""
    txt = open(HEADER).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return re.findall(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", txt, flags=re.M)


def strerror(code: int) -> str:
    return LIB.sage_strerror(int(code)).decode()


def _check(rc: int, what: str):
    if rc != OK:
        raise SageError(rc, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dptr(t):
    """Device pointer of a CUDA tensor (None stays None).  The C ABI takes device pointers and cannot tell a
    host address from a device one, so a host tensor is refused here instead of being read by a kernel."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("a tensor passed for device memory is not a CUDA tensor")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, name, dtype, shape=None, optional=False):
    """Checks a tensor argument the C ABI cannot see: dtype, contiguity, shape."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _bhnd(t, name):
    if t.dim() != 4:
        raise ValueError(f"{name} must be [B, H, N, d]")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.shape


def workspace_bytes(B: int, H: int, N: int, d: int, mode: int) -> int:
    return int(LIB.sage_workspace_bytes(B, H, N, d, mode))


def prepass_scratch_bytes(B: int, H: int, N: int, d: int) -> int:
    return int(LIB.sage_prepass_scratch_bytes(B, H, N, d))


def host_workspace_bytes(B: int, H: int, N: int, d: int, mode: int, chunk_heads: int = 0) -> int:
    return int(LIB.sage_host_workspace_bytes(B, H, N, d, int(mode), int(chunk_heads)))


def alloc_host_workspace(B: int, H: int, N: int, d: int, mode: int, chunk_heads: int = 0, device=None):
    """Zero-filled workspace of attn_fwd_host (two chunk workspaces)."""
    import torch
    n = host_workspace_bytes(B, H, N, d, mode, chunk_heads)
    if n == 0:
        raise SageError(EINVAL, "sage_host_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device or "cuda")


def alloc_workspace(B: int, H: int, N: int, d: int, mode: int, device=None):
    import torch
    n = workspace_bytes(B, H, N, d, mode)
    if n == 0:
        raise SageError(EINVAL, "sage_workspace_bytes")
    ws = torch.zeros(n, dtype=torch.uint8, device=device or "cuda")
    return ws


def quantize_qk(q, k, v, stream=None, q_per_token: bool = False):
    """Runs the prepass; returns a dict of device tensors (q_i8, q_scale, k_i8, k_scale, k_mean, v_f8t, v_scale).

    q_per_token: one Q scale per token (q_scale [B,H,nT*128]) instead of per 128-token block.
    """
    import torch
    B, H, N, d = _bhnd(q, "q")
    dev = q.device
    nT = (N + BLK - 1) // BLK
    out = dict(
        q_i8=torch.empty((B, H, nT * BLK, d), dtype=torch.int8, device=dev),
        q_scale=torch.empty((B, H, nT * BLK if q_per_token else nT), dtype=torch.float32, device=dev),
        k_i8=torch.empty((B, H, nT * BLK, d), dtype=torch.int8, device=dev),
        k_scale=torch.empty((B, H, nT), dtype=torch.float32, device=dev),
        k_mean=torch.empty((B, H, d), dtype=torch.float32, device=dev),
        v_f8t=torch.empty((B, H, d, nT * BLK), dtype=torch.uint8, device=dev),
        v_scale=torch.empty((B, H, d), dtype=torch.float32, device=dev),
    )
    nscr = prepass_scratch_bytes(B, H, N, d)
    scratch = torch.empty(max(nscr, 256), dtype=torch.uint8, device=dev)
    _check(LIB.sage_quantize_qk_ex(_dptr(q), _dptr(k), _dptr(v), B, H, N, d, 1 if q_per_token else BLK,
                                   _dptr(out["q_i8"]), _dptr(out["q_scale"]), _dptr(out["k_i8"]), _dptr(out["k_scale"]),
                                   _dptr(out["k_mean"]), _dptr(out["v_f8t"]), _dptr(out["v_scale"]), _dptr(scratch),
                                   scratch.numel(), _stream(stream)), "sage_quantize_qk_ex")
    out["_scratch"] = scratch
    out["_q_per_token"] = bool(q_per_token)
    return out


NOALLOC_SCRATCH_BYTES = 32 << 20


def quantize_qk_noalloc(q, k, v, out: dict, stream=None) -> int:
    """The prepass through sage_quantize_qk_noalloc: its scratch is the library's
    fixed device array, so the call itself allocates nothing.  `out` holds
    caller-allocated outputs with the keys and shapes quantize_qk returns.
    Returns the status code (SAGE_EWORKSPACE if the problem exceeds the array)."""
    B, H, N, d = _bhnd(q, "q")
    return int(LIB.sage_quantize_qk_noalloc(_dptr(q), _dptr(k), _dptr(v), B, H, N, d, _dptr(out["q_i8"]),
                                            _dptr(out["q_scale"]), _dptr(out["k_i8"]), _dptr(out["k_scale"]),
                                            _dptr(out["k_mean"]), _dptr(out["v_f8t"]), _dptr(out["v_scale"]),
                                            _stream(stream)))


def attn_quantized(pre: dict, N: int, o=None, status=None, stream=None):
    """Attention over prepass outputs; returns bf16 O [B,H,N,d]."""
    import torch
    B, H, _, d = pre["q_i8"].shape
    if o is None:
        o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=pre["q_i8"].device)
    if status is None:
        status = torch.zeros(64, dtype=torch.int32, device=o.device)
    gran = 1 if pre.get("_q_per_token", False) else BLK
    _check(LIB.sage_attn_quantized_ex(_dptr(pre["q_i8"]), _dptr(pre["q_scale"]), _dptr(pre["k_i8"]),
                                      _dptr(pre["k_scale"]), _dptr(pre["v_f8t"]), _dptr(pre["v_scale"]), _dptr(o), B, H, N,
                                      d, gran, _dptr(status), _stream(stream)), "sage_attn_quantized_ex")
    return o


def attn_fwd(q, k, v, mode: int, o=None, workspace=None, stream=None):
    """Full-sequence self-attention through sage_attn_fwd; returns bf16 O [B,H,N,d]."""
    import torch
    B, H, N, d = _bhnd(q, "q")
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o)):
        _need(t, name, torch.bfloat16, (B, H, N, d), optional=name == "o")
    if o is None:
        o = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(B, H, N, d, mode, q.device)
    _check(LIB.sage_attn_fwd(_dptr(q), _dptr(k), _dptr(v), _dptr(o), B, H, N, d, int(mode), _dptr(workspace),
                             workspace.numel() * workspace.element_size(), _stream(stream)), "sage_attn_fwd")
    return o


def attn_fwd_host(q_h, k_h, v_h, o_h, mode: int, staging=None, workspace=None, chunk_heads: int = 0, stream=None):
    """sage_attn_fwd_host: host bf16 [B,H,N,d] tensors (pinned for overlap) in, o_h filled on return.

    staging: optional tuple of four device bf16 tensors shaped like q_h; workspace: optional
    zero-filled device buffer of sage_host_workspace_bytes(B, H, N, d, mode, chunk) bytes
    (alloc_host_workspace).
    """
    import torch
    B, H, N, d = _bhnd(q_h, "q_h")
    BH = B * H
    chunk = chunk_heads if chunk_heads > 0 else host_chunk_heads(B, H, N, d)
    chunk = min(chunk, BH)
    if staging is None:
        staging = tuple(torch.empty(q_h.shape, dtype=torch.bfloat16, device="cuda") for _ in range(4))
    if workspace is None:
        workspace = alloc_host_workspace(B, H, N, d, mode, chunk)
    qd, kd, vd, od = staging
    _check(LIB.sage_attn_fwd_host(_ptr(q_h), _ptr(k_h), _ptr(v_h), _ptr(o_h), B, H, N, d, int(mode), _dptr(qd),
                                  _dptr(kd), _dptr(vd), _dptr(od), _dptr(workspace),
                                  workspace.numel() * workspace.element_size(), int(chunk), _stream(stream)),
           "sage_attn_fwd_host")
    return o_h


def error_stats(a, b, stream=None):
    """Per-head fp64 [B*H, 4] = {sum (a-b)^2, sum b^2, sum a*b, sum a^2} of two bf16 [B,H,N,d] tensors (device)."""
    import torch
    B, H, N, d = _bhnd(a, "a")
    stats = torch.empty((B * H, 4), dtype=torch.float64, device=a.device)
    scratch = torch.empty(max(int(LIB.sage_error_scratch_bytes(B, H)), 16), dtype=torch.uint8, device=a.device)
    _check(LIB.sage_attn_error_stats(_dptr(a), _dptr(b), B, H, N, d, _dptr(stats), _dptr(scratch), scratch.numel(),
                                     _stream(stream)), "sage_attn_error_stats")
    return stats


def rel_l2(a, b, out=None, scratch=None, stream=None):
    """sqrt(sum (a-b)^2 / sum b^2) over every element of two bf16 [B,H,N,d] device tensors, computed on the
    device (sage_attn_rel_l2).  out: device fp64 tensor of one element (a view into a larger table works);
    returned."""
    import torch
    B, H, N, d = _bhnd(a, "a")
    _need(b, "b", torch.bfloat16, tuple(a.shape))
    if out is None:
        out = torch.empty((), dtype=torch.float64, device=a.device)
    if scratch is None:
        scratch = torch.empty(max(int(LIB.sage_error_scratch_bytes(B, H)), 16), dtype=torch.uint8, device=a.device)
    _check(LIB.sage_attn_rel_l2(_dptr(a), _dptr(b), B, H, N, d, _dptr(out), _dptr(scratch),
                                scratch.numel() * scratch.element_size(), _stream(stream)), "sage_attn_rel_l2")
    return out


def layer_errors(layers, stream=None):
    """Relative L2 error of the INT8/FP8 output against the BF16 output, per layer and iteration.

    layers: [num_layers][num_iters] of (q, k, v) device bf16 [B,H,N,d] tensors.
    Returns a nested list [num_layers][num_iters] of sqrt(sum (a-b)^2 / sum b^2) over all heads, each
    formed on the device by sage_attn_rel_l2 and read back once at the end.
    """
    import torch
    L = len(layers)
    I = len(layers[0]) if L else 0
    err = None
    for li, per_layer in enumerate(layers):
        if len(per_layer) != I:
            raise ValueError("every layer needs the same number of iterations")
        for ii, (q, k, v) in enumerate(per_layer):
            if err is None:
                err = torch.empty((L, I), dtype=torch.float64, device=q.device)
            oq = attn_fwd(q, k, v, MODE_INT8_FP8, stream=stream)
            ob = attn_fwd(q, k, v, MODE_BF16, stream=stream)
            rel_l2(oq, ob, out=err[li, ii], stream=stream)
    return [] if err is None else err.cpu().tolist()


def linear_layer_errors(layers, stream=None):
    """Relative L2 error of the W8A8 output against the W8A16 output, per linear layer and iteration.

    The FFN section's selective quantization for linear layers: the weights stay 8-bit in both modes,
    so the error measured here is what quantizing the activations costs; the layers whose error stays
    large run W8A16 (select_full_precision_layers on this table).
    layers: [num_layers][num_iters] of (x bf16 [M, K], wq int8 [N, K], sw fp32, bias bf16 [N] or None).
    """
    import torch
    L = len(layers)
    I = len(layers[0]) if L else 0
    err = None
    for li, per_layer in enumerate(layers):
        if len(per_layer) != I:
            raise ValueError("every layer needs the same number of iterations")
        for ii, (x, wq, sw, bias) in enumerate(per_layer):
            if err is None:
                err = torch.empty((L, I), dtype=torch.float64, device=x.device)
            xq, sx = quantize_blocks_2d(x, stream=stream)
            y8 = linear_w8a8(xq, sx, wq, sw, bias, stream=stream)
            y16 = linear_w8a16(x, wq, sw, bias, stream=stream)
            M, N = y8.shape
            rel_l2(y8.view(1, 1, M, N), y16.view(1, 1, M, N), out=err[li, ii], stream=stream)
    return [] if err is None else err.cpu().tolist()


def select_full_precision_layers(layer_err, threshold: float, rule: int = SELECT_EVERY_ITERATION) -> list[int]:
    """Layers kept at full precision from layer_err [layers][iterations]: with SELECT_EVERY_ITERATION those
    whose error is above threshold at every iteration, with SELECT_MEAN those whose mean error is."""
    import numpy as np
    err = np.ascontiguousarray(np.asarray(layer_err, dtype=np.float64))
    if err.ndim != 2:
        raise ValueError("layer_err must be [layers][iterations]")
    L, I = err.shape
    out = (ctypes.c_int * max(L, 1))()
    n = ctypes.c_int(0)
    _check(LIB.sage_select_full_precision_layers(err.ctypes.data_as(ctypes.c_void_p), L, I, float(threshold),
                                                 int(rule), ctypes.cast(out, ctypes.c_void_p), ctypes.byref(n)),
           "sage_select_full_precision_layers")
    return [int(out[i]) for i in range(n.value)]


def quantize_blocks_2d(x, codes=None, scales=None, stream=None):
    """bf16 [R, K] -> (int8 codes [R, K], fp32 scales [ceil(R/128), K/128]), 128 x 128 blocks."""
    import torch
    if x.dim() != 2 or not x.is_contiguous() or x.dtype != torch.bfloat16:
        raise ValueError("x must be a contiguous bf16 [R, K] tensor")
    R, K = x.shape
    if codes is None:
        codes = torch.empty((R, K), dtype=torch.int8, device=x.device)
    if scales is None:
        scales = torch.empty(((R + BLK - 1) // BLK, K // BLK), dtype=torch.float32, device=x.device)
    _check(LIB.sage_quantize_blocks_2d(_dptr(x), R, K, _dptr(codes), _dptr(scales), _stream(stream)),
           "sage_quantize_blocks_2d")
    return codes, scales


def linear_w8a8(xq, sx, wq, sw, bias=None, y=None, out_dtype=None, status=None, stream=None):
    """Y = X W^T + bias from 128 x 128 block-quantized X [M, K] and W [N, K]; returns Y [M, N]."""
    import torch
    M, K = xq.shape
    N = wq.shape[0]
    _need(xq, "xq", torch.int8, (M, K))
    _need(wq, "wq", torch.int8, (N, K))
    _need(sx, "sx", torch.float32, ((M + BLK - 1) // BLK, K // BLK))
    _need(sw, "sw", torch.float32, ((N + BLK - 1) // BLK, K // BLK))
    _need(bias, "bias", torch.bfloat16, (N,), optional=True)
    if out_dtype is None:
        out_dtype = torch.bfloat16 if y is None else y.dtype
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype, device=xq.device)
    if status is None:
        status = torch.zeros(64, dtype=torch.int32, device=xq.device)
    code = DTYPE_F32 if y.dtype == torch.float32 else DTYPE_BF16
    _check(LIB.sage_linear_w8a8(_dptr(xq), _dptr(sx), _dptr(wq), _dptr(sw), _dptr(bias), _dptr(y), code, M, N, K,
                                _dptr(status), _stream(stream)), "sage_linear_w8a8")
    return y


def dequant_blocks_2d(codes, scales, out=None, stream=None):
    """int8 codes [R, K] + block scales -> bf16 [R, K] = bf16(scale * code)."""
    import torch
    R, K = codes.shape
    _need(codes, "codes", torch.int8, (R, K))
    _need(scales, "scales", torch.float32, ((R + BLK - 1) // BLK, K // BLK))
    _need(out, "out", torch.bfloat16, (R, K), optional=True)
    if out is None:
        out = torch.empty((R, K), dtype=torch.bfloat16, device=codes.device)
    _check(LIB.sage_dequant_blocks_2d(_dptr(codes), _dptr(scales), R, K, _dptr(out), _stream(stream)),
           "sage_dequant_blocks_2d")
    return out


def linear_bf16(x, w, bias=None, y=None, out_dtype=None, status=None, stream=None):
    """Y = X W^T + bias for bf16 X [M, K] and W [N, K]; returns Y [M, N]."""
    import torch
    M, K = x.shape
    N = w.shape[0]
    _need(x, "x", torch.bfloat16, (M, K))
    _need(w, "w", torch.bfloat16, (N, K))
    _need(bias, "bias", torch.bfloat16, (N,), optional=True)
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype or torch.bfloat16, device=x.device)
    if status is None:
        status = torch.zeros(64, dtype=torch.int32, device=x.device)
    code = DTYPE_F32 if y.dtype == torch.float32 else DTYPE_BF16
    _check(LIB.sage_linear_bf16(_dptr(x), _dptr(w), _dptr(bias), _dptr(y), code, M, N, K, _dptr(status),
                                _stream(stream)), "sage_linear_bf16")
    return y


def linear_w8a16(x, wq, sw, bias=None, y=None, out_dtype=None, workspace=None, status=None, stream=None):
    """W8A16 layer: bf16 X [M, K] against 128 x 128 block-quantized W (wq int8 [N, K], sw); returns Y [M, N]."""
    import torch
    M, K = x.shape
    N = wq.shape[0]
    _need(x, "x", torch.bfloat16, (M, K))
    _need(wq, "wq", torch.int8, (N, K))
    _need(sw, "sw", torch.float32, ((N + BLK - 1) // BLK, K // BLK))
    _need(bias, "bias", torch.bfloat16, (N,), optional=True)
    if y is None:
        y = torch.empty((M, N), dtype=out_dtype or torch.bfloat16, device=x.device)
    if status is None:
        status = torch.zeros(64, dtype=torch.int32, device=x.device)
    nbytes = int(LIB.sage_linear_w8a16_workspace_bytes(N, K))
    if workspace is None:
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
    code = DTYPE_F32 if y.dtype == torch.float32 else DTYPE_BF16
    _check(LIB.sage_linear_w8a16(_dptr(x), _dptr(wq), _dptr(sw), _dptr(bias), _dptr(y), code, M, N, K, _dptr(workspace),
                                 workspace.numel() * workspace.element_size(), _dptr(status), _stream(stream)),
           "sage_linear_w8a16")
    return y


ULYSSES_SEND, ULYSSES_RECV_O, ULYSSES_GATHER, ULYSSES_SCATTER = 0, 1, 2, 3


def host_chunk_heads(B: int, H: int, N: int, d: int) -> int:
    """Default head chunk of attn_fwd_host (see sage_host_chunk_heads)."""
    return int(LIB.sage_host_chunk_heads(B, H, N, d))


def ulysses_permute(src, dst, B: int, Nl: int, H: int, d: int, P: int, op: int, chunk_rows: int = 0,
                    base_rows: int = 0, stream=None):
    """Row permutation between the Ulysses layouts (see include/sage.h); dst is filled and returned."""
    import torch
    _need(src, "src", torch.bfloat16)
    _need(dst, "dst", torch.bfloat16)
    if P < 1 or H % P:
        raise ValueError(f"H={H} must be a multiple of P={P}")
    dense = B * (H // P) * Nl                     # rows of one [P] chunk
    p_side_rows = base_rows + (P - 1) * (chunk_rows or dense) + dense
    chunked, flat = (dst, src) if op in (ULYSSES_SEND, ULYSSES_SCATTER) else (src, dst)
    if flat.numel() < B * Nl * H * d:
        raise ValueError("the [B, ...] side holds fewer than B * Nl * H rows of d values")
    if chunked.numel() < p_side_rows * d:
        raise ValueError("the [P] side is smaller than base_rows + (P - 1) * chunk_rows + one chunk")
    _check(LIB.sage_ulysses_permute(_dptr(src), _dptr(dst), B, Nl, H, d, P, op, int(chunk_rows), int(base_rows),
                                    _stream(stream)), "sage_ulysses_permute")
    return dst


def seqpar_workspace_bytes(P: int, B: int, Nl: int, Hl: int, d: int, mode: int) -> int:
    return int(LIB.sage_seqpar_workspace_bytes(P, B, Nl, Hl, d, mode))


def alloc_seqpar_workspace(P: int, B: int, Nl: int, Hl: int, d: int, mode: int, device=None):
    """Device workspace of sage_attn_fwd_seqpar (uint8, 256-byte aligned by the allocator)."""
    import torch
    n = seqpar_workspace_bytes(P, B, Nl, Hl, d, mode)
    if n == 0:
        raise SageError(EINVAL, "sage_seqpar_workspace_bytes")
    return torch.zeros(n, dtype=torch.uint8, device=device if device is not None else "cuda")


def attn_fwd_seqpar(q, k, v, mode: int, o=None, P: int = 1, workspace=None, stream=None):
    """Attention on the sequence-parallel exchange layout: q, k, v, o bf16 [P, B, Nl, Hl, d] (chunk p:
    tokens p*Nl .. p*Nl + Nl - 1, token-major).  Returns o."""
    import torch
    if q.dim() != 5 or q.shape[0] != P:
        raise ValueError("q must be [P, B, Nl, Hl, d]")
    shape = tuple(q.shape)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16, shape)
    _, B, Nl, Hl, d = shape
    if o is None:
        o = torch.empty_like(q)
    _need(o, "o", torch.bfloat16, shape)
    if workspace is None:
        workspace = alloc_seqpar_workspace(P, B, Nl, Hl, d, mode, q.device)
    _check(LIB.sage_attn_fwd_seqpar(_dptr(q), _dptr(k), _dptr(v), _dptr(o), P, B, Nl, Hl, d, int(mode),
                                    _dptr(workspace), workspace.numel() * workspace.element_size(), _stream(stream)),
           "sage_attn_fwd_seqpar")
    return o


def status(workspace, stream=None) -> int:
    """Reads and clears the device status word (synchronises the stream); returns a status code."""
    return int(LIB.sage_status(_dptr(workspace), _stream(stream)))


def layer_schedule(num_layers: int, full_precision_layers) -> list[int]:
    """Per-layer modes: MODE_BF16 for the listed layers, MODE_INT8_FP8 for the rest (host only)."""
    fp = list(full_precision_layers)
    arr = (ctypes.c_int * max(len(fp), 1))(*fp)
    modes = (ctypes.c_int8 * max(num_layers, 1))()
    _check(LIB.attn_layer_schedule(int(num_layers), ctypes.cast(arr, ctypes.c_void_p), len(fp),
                                   ctypes.cast(modes, ctypes.c_void_p)), "attn_layer_schedule")
    return [int(modes[i]) for i in range(num_layers)]


def device_check() -> int:
    return int(LIB.sage_device_check())


# ---------------------------------------------------------------- diagnostics

def dbg_qk_tiles(q_i8, k_i8, N: int, tiles, stream=None):
    """int32 QK^T tiles [(b,h,qb,kb)...] -> [n,128,128] through the tcgen05 kind::i8 path."""
    import torch
    B, H, _, d = q_i8.shape
    tl = torch.tensor(tiles, dtype=torch.int32, device=q_i8.device).reshape(-1, 4).contiguous()
    out = torch.empty((tl.shape[0], BLK, BLK), dtype=torch.int32, device=q_i8.device)
    _check(LIB.sage_dbg_qk_tiles(_dptr(q_i8), _dptr(k_i8), B, H, N, d, _dptr(tl), tl.shape[0], _dptr(out),
                                 _stream(stream)), "sage_dbg_qk_tiles")
    return out


def dbg_pv_tile(p, vt, mode: int, stream=None):
    import torch
    d = vt.shape[0] if mode == MODE_INT8_FP8 else vt.shape[1]
    out = torch.empty((BLK, d), dtype=torch.float32, device=p.device)
    _check(LIB.sage_dbg_pv_tile(_dptr(p), _dptr(vt), d, int(mode), _dptr(out), _stream(stream)), "sage_dbg_pv_tile")
    return out


def dbg_qk_bf16_tile(q, k, stream=None):
    import torch
    d = q.shape[1]
    out = torch.empty((BLK, BLK), dtype=torch.float32, device=q.device)
    _check(LIB.sage_dbg_qk_bf16_tile(_dptr(q), _dptr(k), d, _dptr(out), _stream(stream)), "sage_dbg_qk_bf16_tile")
    return out


def dbg_linear_forced_timeout(xq, sx, wq, sw, status, timeout_cycles: int, bias=None, y=None, stream=None):
    import torch
    M, K = xq.shape
    N = wq.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=xq.device)
    code = DTYPE_F32 if y.dtype == torch.float32 else DTYPE_BF16
    _check(LIB.sage_dbg_linear_forced_timeout(_dptr(xq), _dptr(sx), _dptr(wq), _dptr(sw), _dptr(bias), _dptr(y), code, M,
                                              N, K, _dptr(status), int(timeout_cycles), _stream(stream)),
           "sage_dbg_linear_forced_timeout")
    return y


def dbg_linear_bf16_forced_timeout(x, w, status, timeout_cycles: int, bias=None, y=None, stream=None):
    import torch
    M, K = x.shape
    N = w.shape[0]
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    code = DTYPE_F32 if y.dtype == torch.float32 else DTYPE_BF16
    _check(LIB.sage_dbg_linear_bf16_forced_timeout(_dptr(x), _dptr(w), _dptr(bias), _dptr(y), code, M, N, K, _dptr(status),
                                                   int(timeout_cycles), _stream(stream)),
           "sage_dbg_linear_bf16_forced_timeout")
    return y


MMA_BF16, MMA_E4M3, MMA_I8 = 0, 1, 2


def dbg_mma_peak(kind: int, n: int = 256, iters: int = 4000, stream=None) -> dict:
    """Tensor-core probe: MACs per SM per clock of back-to-back tcgen05.mma (slowest SM)."""
    import torch
    sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
    cycles = torch.zeros(sms, dtype=torch.int64, device="cuda")
    status = torch.zeros(64, dtype=torch.int32, device="cuda")
    _check(LIB.sage_dbg_mma_peak(int(kind), int(n), int(iters), _dptr(cycles), sms, _dptr(status), _stream(stream)),
           "sage_dbg_mma_peak")
    torch.cuda.synchronize()
    if int(status[0].item()) != 0:
        raise SageError(ETIMEOUT, "sage_dbg_mma_peak")
    k = 16 if kind == MMA_BF16 else 32
    slowest = int(cycles.max().item())
    return {"mac_per_clk_per_sm": iters * 4 * 128 * n * k / slowest, "cycles": slowest, "sms": sms}


def dbg_attn_forced_timeout(pre: dict, N: int, status, timeout_cycles: int, o=None, stream=None):
    import torch
    B, H, _, d = pre["q_i8"].shape
    if o is None:
        o = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=pre["q_i8"].device)
    _check(LIB.sage_dbg_attn_forced_timeout(_dptr(pre["q_i8"]), _dptr(pre["q_scale"]), _dptr(pre["k_i8"]),
                                            _dptr(pre["k_scale"]), _dptr(pre["v_f8t"]), _dptr(pre["v_scale"]), _dptr(o),
                                            B, H, N, d, _dptr(status), int(timeout_cycles), _stream(stream)),
           "sage_dbg_attn_forced_timeout")
    return o
