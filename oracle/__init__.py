"""CPU oracle for quantized video-DiT self-attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The product library never routes through it and
shares no code with it.

What it computes is stated in ``oracle.c`` (a plain, slow C restatement of the
method of page 1 of the TMAP / Taobao Faxiang image-to-video write-up,
"Attention performance optimisation": SageAttention-style INT8 QK^T with K
smoothing and a zero-scale guard, FP8 P.V, online softmax, and a per-layer
BF16 table).  This module compiles it in-tree and wraps it with numpy.

Every function here is pinned by ``tests/test_oracle_*.py`` against things
other than itself: exact rational brute force, the OCP FP8 code table,
closed-form special cases and invariants of exact softmax attention.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

TILE = 128
# emulation switches (see orc_attn_emul): used only to pin the emulation
EMUL_P_FP32 = 1
EMUL_V_EXACT = 2
EMUL_QK_EXACT = 4
EMUL_ONE_TILE = 8
EMUL_Q_PER_TOKEN = 16


def build(force: bool = False) -> str:
    """Compiles oracle.c into liboracle.so (gcc -O2, OpenMP, no contraction)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                               "-fno-fast-math", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _p(a, ct):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ct))


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            i32, i64 = ctypes.c_int, ctypes.c_long
            P = ctypes.POINTER
            u16, i8, u8, f32, f64, s32 = (P(ctypes.c_uint16), P(ctypes.c_int8), P(ctypes.c_uint8),
                                          P(ctypes.c_float), P(ctypes.c_double), P(ctypes.c_int32))
            lib.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
            lib.orc_e4m3_decode.restype = ctypes.c_double
            lib.orc_e4m3_encode.argtypes = [ctypes.c_float]
            lib.orc_e4m3_encode.restype = ctypes.c_uint8
            lib.orc_k_mean.argtypes = [u16, i32, i32, i32, i32, f32]
            lib.orc_quant_int8_blocks.argtypes = [u16, f32, i32, i32, i32, i32, i8, f32]
            lib.orc_quant_v_fp8.argtypes = [u16, i32, i32, i32, i32, u8, f32]
            lib.orc_quant_int8_rows.argtypes = [u16, f32, i32, i32, i32, i32, i32, i8, f32]
            lib.orc_qk_tile.argtypes = [i8, i8, i32, i32, i64, i32, i32, s32]
            lib.orc_attn_exact.argtypes = [u16, u16, u16, i32, i32, i32, i32, P(i32), i32, f64]
            lib.orc_attn_emul.argtypes = [i8, f32, i8, f32, u8, f32, i32, i32, i32, i32, P(i32), i32, i32,
                                          u16, u16, u16, f32, u16]
            lib.orc_quant_blocks_2d.argtypes = [u16, i32, i32, i8, f32]
            lib.orc_linear_w8a8.argtypes = [i8, f32, i8, f32, u16, i32, i32, i32, P(i32), i32, f32, u16]
            lib.orc_dequant_blocks_2d.argtypes = [i8, f32, i32, i32, u16]
            lib.orc_layer_schedule.argtypes = [i32, P(i32), i32, i8]
            lib.orc_layer_schedule.restype = i32
            lib.orc_rel_l2.argtypes = [u16, u16, i64]
            lib.orc_rel_l2.restype = ctypes.c_double
            lib.orc_select_layers.argtypes = [f64, i32, i32, ctypes.c_double, i32, P(i32)]
            lib.orc_select_layers.restype = i32
            _lib = lib
    return _lib


def _c(a, dtype):
    a = np.ascontiguousarray(a)
    assert a.dtype == dtype, (a.dtype, dtype)
    return a


# ---------------- FP8 e4m3 ----------------

def e4m3_decode(code: int) -> float:
    return _load().orc_e4m3_decode(int(code) & 0xFF)


def e4m3_encode(x: float) -> int:
    return int(_load().orc_e4m3_encode(float(x)))


def e4m3_decode_table() -> np.ndarray:
    """fp64 value of each of the 256 e4m3 codes (NaN for 0x7F / 0xFF)."""
    return np.array([e4m3_decode(i) for i in range(256)], dtype=np.float64)


# ---------------- prepass (a1..a4) ----------------

def k_mean(k: np.ndarray) -> np.ndarray:
    """a1: fp32 [B,H,d] per-channel token mean of bf16 K [B,H,N,d]."""
    k = _c(k, np.uint16)
    B, H, N, d = k.shape
    out = np.empty((B, H, d), dtype=np.float32)
    _load().orc_k_mean(_p(k, ctypes.c_uint16), B, H, N, d, _p(out, ctypes.c_float))
    return out


def quant_int8_blocks(x: np.ndarray, mean: np.ndarray | None = None):
    """a2/a3: per-128-token-block INT8 codes [B,H,N,d] and fp32 scales [B,H,nblk]."""
    x = _c(x, np.uint16)
    B, H, N, d = x.shape
    nb = (N + TILE - 1) // TILE
    codes = np.empty((B, H, N, d), dtype=np.int8)
    scale = np.empty((B, H, nb), dtype=np.float32)
    m = None if mean is None else _c(mean, np.float32)
    _load().orc_quant_int8_blocks(_p(x, ctypes.c_uint16), _p(m, ctypes.c_float), B, H, N, d,
                                  _p(codes, ctypes.c_int8), _p(scale, ctypes.c_float))
    return codes, scale


def quant_int8_rows(x: np.ndarray, rows: int, mean: np.ndarray | None = None):
    """INT8 codes [B,H,N,d] and fp32 scales [B,H,ceil(N/rows)] with a block of `rows` tokens (1: per token)."""
    x = _c(x, np.uint16)
    B, H, N, d = x.shape
    nb = (N + rows - 1) // rows
    codes = np.empty((B, H, N, d), dtype=np.int8)
    scale = np.empty((B, H, nb), dtype=np.float32)
    m = None if mean is None else _c(mean, np.float32)
    _load().orc_quant_int8_rows(_p(x, ctypes.c_uint16), _p(m, ctypes.c_float), B, H, N, d, int(rows),
                                _p(codes, ctypes.c_int8), _p(scale, ctypes.c_float))
    return codes, scale


def quant_v_fp8(v: np.ndarray):
    """a4: e4m3 codes [B,H,N,d] (natural layout) and fp32 per-channel scales [B,H,d]."""
    v = _c(v, np.uint16)
    B, H, N, d = v.shape
    codes = np.empty((B, H, N, d), dtype=np.uint8)
    scale = np.empty((B, H, d), dtype=np.float32)
    _load().orc_quant_v_fp8(_p(v, ctypes.c_uint16), B, H, N, d, _p(codes, ctypes.c_uint8),
                            _p(scale, ctypes.c_float))
    return codes, scale


def prepass(q: np.ndarray, k: np.ndarray, v: np.ndarray, q_per_token: bool = False) -> dict:
    """a1..a4 in order; returns every intermediate the path exposes.

    q_per_token: one Q scale per token instead of per 128-token block (the
    finer granularity; pair it with attn_emul(..., flags=EMUL_Q_PER_TOKEN)).
    """
    mean = k_mean(k)
    q8, qs = quant_int8_rows(q, 1) if q_per_token else quant_int8_blocks(q)
    k8, ks = quant_int8_blocks(k, mean)
    v8, vs = quant_v_fp8(v)
    return dict(k_mean=mean, q_i8=q8, q_scale=qs, k_i8=k8, k_scale=ks, v_f8=v8, v_scale=vs)


def qk_tile(q8: np.ndarray, k8: np.ndarray, bh: int, qb: int, kb: int) -> np.ndarray:
    """a5: exact int32 [128,128] tile of Q_i8 K_i8^T for one (b*H+h, q-block, k-block)."""
    q8 = _c(q8, np.int8)
    k8 = _c(k8, np.int8)
    B, H, N, d = q8.shape
    out = np.empty((TILE, TILE), dtype=np.int32)
    _load().orc_qk_tile(_p(q8, ctypes.c_int8), _p(k8, ctypes.c_int8), N, d, bh, qb, kb,
                        _p(out, ctypes.c_int32))
    return out


# ---------------- attention ----------------

def attn_exact(q, k, v, rows=None) -> np.ndarray:
    """O1: fp64 softmax(Q K^T/sqrt(d)) V for the given query rows, shape [B,H,len(rows),d]."""
    q, k, v = (_c(a, np.uint16) for a in (q, k, v))
    B, H, N, d = q.shape
    rows = np.arange(N, dtype=np.int32) if rows is None else _c(np.asarray(rows, dtype=np.int32), np.int32)
    out = np.empty((B, H, len(rows), d), dtype=np.float64)
    _load().orc_attn_exact(_p(q, ctypes.c_uint16), _p(k, ctypes.c_uint16), _p(v, ctypes.c_uint16),
                           B, H, N, d, _p(rows, ctypes.c_int), len(rows), _p(out, ctypes.c_double))
    return out


def attn_emul(pre: dict, rows=None, flags: int = 0, q=None, k=None, v=None):
    """O2: emulated quantized attention for the given rows.

    Returns (fp32 values [B,H,R,d] before output rounding, bf16 bits [B,H,R,d]).
    """
    q8, k8, v8 = _c(pre["q_i8"], np.int8), _c(pre["k_i8"], np.int8), _c(pre["v_f8"], np.uint8)
    qs, ks, vs = (_c(pre[n], np.float32) for n in ("q_scale", "k_scale", "v_scale"))
    B, H, N, d = q8.shape
    rows = np.arange(N, dtype=np.int32) if rows is None else _c(np.asarray(rows, dtype=np.int32), np.int32)
    out = np.empty((B, H, len(rows), d), dtype=np.float32)
    outb = np.empty((B, H, len(rows), d), dtype=np.uint16)
    qb_, kb_, vb_ = (None if a is None else _c(a, np.uint16) for a in (q, k, v))
    _load().orc_attn_emul(_p(q8, ctypes.c_int8), _p(qs, ctypes.c_float), _p(k8, ctypes.c_int8),
                          _p(ks, ctypes.c_float), _p(v8, ctypes.c_uint8), _p(vs, ctypes.c_float),
                          B, H, N, d, _p(rows, ctypes.c_int), len(rows), int(flags),
                          _p(qb_, ctypes.c_uint16), _p(kb_, ctypes.c_uint16), _p(vb_, ctypes.c_uint16),
                          _p(out, ctypes.c_float), _p(outb, ctypes.c_uint16))
    return out, outb


def quant_blocks_2d(x: np.ndarray):
    """W8A8 operand: INT8 codes [R, K] and fp32 scales [ceil(R/128), K/128] of a bf16 [R, K] matrix."""
    x = _c(x, np.uint16)
    R, K = x.shape
    assert K % 128 == 0
    codes = np.empty((R, K), dtype=np.int8)
    scales = np.empty(((R + 127) // 128, K // 128), dtype=np.float32)
    _load().orc_quant_blocks_2d(_p(x, ctypes.c_uint16), R, K, _p(codes, ctypes.c_int8), _p(scales, ctypes.c_float))
    return codes, scales


def linear_w8a8(xq, sx, wq, sw, bias=None, rows=None):
    """Y = block-scaled INT8 product (+ bias) for the given rows: (fp32 [R, N], bf16 bits [R, N])."""
    xq, wq = _c(xq, np.int8), _c(wq, np.int8)
    sx, sw = _c(sx, np.float32), _c(sw, np.float32)
    M, K = xq.shape
    N = wq.shape[0]
    rows = np.arange(M, dtype=np.int32) if rows is None else _c(np.asarray(rows, dtype=np.int32), np.int32)
    y = np.empty((len(rows), N), dtype=np.float32)
    yb = np.empty((len(rows), N), dtype=np.uint16)
    b = None if bias is None else _c(bias, np.uint16)
    _load().orc_linear_w8a8(_p(xq, ctypes.c_int8), _p(sx, ctypes.c_float), _p(wq, ctypes.c_int8),
                            _p(sw, ctypes.c_float), _p(b, ctypes.c_uint16), M, N, K, _p(rows, ctypes.c_int),
                            len(rows), _p(y, ctypes.c_float), _p(yb, ctypes.c_uint16))
    return y, yb


def dequant_blocks_2d(codes: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """bf16 bits [R, K] of the block-scaled codes: bf16_rne(fl(scale * code))."""
    codes, scales = _c(codes, np.int8), _c(scales, np.float32)
    R, K = codes.shape
    out = np.empty((R, K), dtype=np.uint16)
    _load().orc_dequant_blocks_2d(_p(codes, ctypes.c_int8), _p(scales, ctypes.c_float), R, K,
                                  _p(out, ctypes.c_uint16))
    return out


def linear_bf16(x: np.ndarray, w: np.ndarray, bias=None, rows=None) -> np.ndarray:
    """Y = X W^T (+ bias) for bf16 bits X [M, K], W [N, K]: the exact products summed in fp64
    (a library matmul of the fp64 values), returned in fp64 for the given rows."""
    X = _bf16_f64(np.asarray(x, dtype=np.uint16))
    W = _bf16_f64(np.asarray(w, dtype=np.uint16))
    if rows is not None:
        X = X[np.asarray(rows)]
    y = X @ W.T
    if bias is not None:
        y = y + _bf16_f64(np.asarray(bias, dtype=np.uint16))[None, :]
    return y


def _bf16_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def layer_schedule(num_layers: int, fp_layers) -> np.ndarray:
    """a11: int8 modes [num_layers]: 0 = BF16 for the listed layers, 1 = INT8/FP8 otherwise."""
    fp = np.asarray(list(fp_layers), dtype=np.int32)
    modes = np.empty(max(num_layers, 0), dtype=np.int8)
    rc = _load().orc_layer_schedule(num_layers, _p(fp, ctypes.c_int), len(fp), _p(modes, ctypes.c_int8))
    if rc != 0:
        raise ValueError("layer index out of range")
    return modes


# ---------------- f2: per-layer error and the full-precision layer set ----------------

SELECT_EVERY_ITERATION = 0
SELECT_MEAN = 1


def rel_l2(a: np.ndarray, b: np.ndarray) -> float:
    """sqrt(sum (a-b)^2 / sum b^2) over every element of two bf16 arrays (uint16 bits), fp64 ascending sums."""
    a = _c(a, np.uint16).ravel()
    b = _c(b, np.uint16).ravel()
    if a.size != b.size:
        raise ValueError("a and b differ in size")
    return float(_load().orc_rel_l2(_p(a, ctypes.c_uint16), _p(b, ctypes.c_uint16), a.size))


def select_layers(err, threshold: float, rule: int = SELECT_EVERY_ITERATION) -> list[int]:
    """Layers kept at full precision from err[layer][iteration] (rule 0: above the threshold at every
    iteration; rule 1: mean above it)."""
    e = np.ascontiguousarray(np.asarray(err, dtype=np.float64))
    if e.ndim != 2:
        raise ValueError("err must be [layers][iterations]")
    out = np.zeros(max(e.shape[0], 1), dtype=np.int32)
    n = _load().orc_select_layers(_p(e, ctypes.c_double), e.shape[0], e.shape[1], float(threshold), int(rule),
                                  _p(out, ctypes.c_int))
    if n < 0:
        raise ValueError("bad error table or rule")
    return out[:n].tolist()
