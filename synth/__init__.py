"""Seeded synthetic inputs for the video-DiT self-attention workloads.

Draws numbers only (no attention or quantization arithmetic lives here), so
that the CUDA path and the CPU oracle are fed identical bytes.  The generator
itself is ``synth.c`` (splitmix64 + Box-Muller, counter based); this module
compiles it in-tree on first use and exposes numpy / torch views.

The named workloads follow the shapes that page 1 of the TMAP write-up
("Attention performance optimisation", the FLOP profile of
``aten.scaled_dot_product_flash_attention`` on CogVideoX / Wan DiTs) refers to;
the values are synthetic stand-ins for real activations, which need trained
weights.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading
from dataclasses import dataclass, replace

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "synth.c")
_LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compiles synth.c into libsynth.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            u64, i32, dbl = ctypes.c_uint64, ctypes.c_int, ctypes.c_double
            p16 = ctypes.POINTER(ctypes.c_uint16)
            lib.synth_qkv.argtypes = [u64, i32, i32, i32, i32, dbl, i32, dbl, i32, p16, p16, p16]
            lib.synth_qkv.restype = i32
            lib.synth_sample_rows.argtypes = [u64, i32, i32, ctypes.POINTER(i32)]
            lib.synth_sample_rows.restype = i32
            lib.synth_outlier_pairs.argtypes = [u64, i32, i32, i32, ctypes.POINTER(ctypes.c_uint8)]
            lib.synth_outlier_pairs.restype = i32
            lib.synth_linear.argtypes = [u64, i32, i32, i32, i32, dbl, p16, p16, p16]
            lib.synth_linear.restype = i32
            lib.synth_normal.argtypes = [u64, ctypes.c_uint32, u64]
            lib.synth_normal.restype = dbl
            _lib = lib
    return _lib


@dataclass(frozen=True)
class Workload:
    """One synthetic self-attention call: shapes plus the value recipe."""
    name: str
    B: int
    H: int
    N: int
    d: int
    seed: int = 0
    k_off_std: float = 3.0          # K offset ~ N(0, 9) per (b, h, c)
    outlier_frac: float = 0.0       # fraction of (h, c) pairs scaled as outliers
    outlier_scale: float = 20.0
    zero_k_channel: int = -1        # K channel forced to zero (-1: none)

    @property
    def n_outlier(self) -> int:
        return int(math.floor(self.outlier_frac * self.H * self.d + 0.5))

    @property
    def flops(self) -> float:
        """Attention FLOPs of one call: 4 * B * H * N^2 * d."""
        return 4.0 * self.B * self.H * float(self.N) ** 2 * self.d

    def with_seed(self, seed: int) -> "Workload":
        return replace(self, seed=seed)


WORKLOADS = {
    # 2 heads, 1024 tokens; K channel 5 all zero (the all-zero channel case).
    "tiny": Workload("tiny", 1, 2, 1024, 128, seed=0, zero_k_channel=5),
    # CogVideoX-2B: 13x30x45 video tokens + 226 text tokens, head dim 64.
    "cogvideox2b": Workload("cogvideox2b", 1, 30, 17776, 64, seed=0),
    # Wan2.1-1.3B 480p: 21x30x52 latent patches, 1% outlier channels x20.
    "wan1.3b_480p": Workload("wan1.3b_480p", 1, 12, 32760, 128, seed=0, outlier_frac=0.01),
    # Wan2.1-14B 720p: 21x45x80 latent patches, 1% outlier channels x20.
    "wan14b_720p": Workload("wan14b_720p", 1, 40, 75600, 128, seed=0, outlier_frac=0.01),
    # One layer of the 40-layer stack (seed = layer index).
    "layer_stack": Workload("layer_stack", 1, 40, 32760, 128, seed=0, outlier_frac=0.01),
}

# Layers of the 40-layer stack that stay in BF16.
LAYER_STACK_FULL_PRECISION = (0, 8, 16, 24, 32)
LAYER_STACK_LAYERS = 40


def qkv_numpy(w: Workload, parts: str = "qkv"):
    """Returns (q, k, v) as uint16 arrays of bf16 bits, shape [B, H, N, d]."""
    lib = _load()
    shape = (w.B, w.H, w.N, w.d)
    out = {p: (np.empty(shape, dtype=np.uint16) if p in parts else None) for p in "qkv"}

    def ptr(a):
        return a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)) if a is not None else None

    rc = lib.synth_qkv(w.seed, w.B, w.H, w.N, w.d, w.k_off_std, w.n_outlier, w.outlier_scale,
                       w.zero_k_channel, ptr(out["q"]), ptr(out["k"]), ptr(out["v"]))
    if rc != 0:
        raise ValueError(f"synth_qkv rejected workload {w}")
    return out["q"], out["k"], out["v"]


def qkv_torch(w: Workload, pin: bool = False):
    """Returns (q, k, v) as CPU torch.bfloat16 tensors [B, H, N, d] (optionally pinned)."""
    import torch
    q, k, v = qkv_numpy(w)
    res = []
    for a in (q, k, v):
        t = torch.from_numpy(a.view(np.int16)).view(torch.bfloat16)
        res.append(t.pin_memory() if pin else t)
    return tuple(res)


def sample_rows(seed: int, N: int, n: int) -> np.ndarray:
    """Seeded, sorted sample of n distinct query rows (includes 0, N-1 and the tail tile)."""
    lib = _load()
    rows = np.empty(max(min(n, N), 0), dtype=np.int32)
    cnt = lib.synth_sample_rows(seed, N, n, rows.ctypes.data_as(ctypes.POINTER(ctypes.c_int)))
    return rows[:cnt]


def outlier_pairs(w: Workload) -> np.ndarray:
    """Boolean [H, d] mask of the outlier (h, c) pairs of a workload."""
    lib = _load()
    m = np.zeros((w.H, w.d), dtype=np.uint8)
    rc = lib.synth_outlier_pairs(w.seed, w.H, w.d, w.n_outlier,
                                 m.ctypes.data_as(ctypes.POINTER(ctypes.c_uint8)))
    if rc != 0:
        raise ValueError("bad outlier request")
    return m.astype(bool)


def bf16_bits_to_f32(a: np.ndarray) -> np.ndarray:
    """Widens bf16 bit patterns (uint16) to float32 exactly."""
    return (a.astype(np.uint32) << 16).view(np.float32)


@dataclass(frozen=True)
class LinearWorkload:
    """One synthetic linear layer Y = X W^T + bias: X [M, K], W [N, K]."""
    name: str
    M: int
    N: int
    K: int
    seed: int = 0
    outlier_frac: float = 0.01      # fraction of X channels scaled as outliers
    outlier_scale: float = 20.0

    @property
    def n_outlier(self) -> int:
        return int(math.floor(self.outlier_frac * self.K + 0.5))

    @property
    def flops(self) -> float:
        """GEMM FLOPs of one call: 2 * M * N * K."""
        return 2.0 * self.M * self.N * float(self.K)


# Wan2.1-14B (hidden 5120, FFN 13824) over the 720p video's 75600 tokens, and
# small ragged cases (M not a multiple of 128, N an odd multiple of 128).
LINEAR_WORKLOADS = {
    "lin_tiny": LinearWorkload("lin_tiny", 333, 384, 512, seed=1),
    "lin_multi": LinearWorkload("lin_multi", 8197, 1280, 1024, seed=2),
    "wan14b_720p_proj": LinearWorkload("wan14b_720p_proj", 75600, 5120, 5120, seed=0),
    "wan14b_720p_ffn_up": LinearWorkload("wan14b_720p_ffn_up", 75600, 13824, 5120, seed=0),
    "wan14b_720p_ffn_down": LinearWorkload("wan14b_720p_ffn_down", 75600, 5120, 13824, seed=0),
}


def linear_numpy(w: LinearWorkload, parts: str = "xwb"):
    """Returns (x [M, K], w [N, K], bias [N]) as uint16 arrays of bf16 bits."""
    lib = _load()
    out = {
        "x": np.empty((w.M, w.K), dtype=np.uint16) if "x" in parts else None,
        "w": np.empty((w.N, w.K), dtype=np.uint16) if "w" in parts else None,
        "b": np.empty((w.N,), dtype=np.uint16) if "b" in parts else None,
    }

    def ptr(a):
        return a.ctypes.data_as(ctypes.POINTER(ctypes.c_uint16)) if a is not None else None

    rc = lib.synth_linear(w.seed, w.M, w.N, w.K, w.n_outlier, w.outlier_scale, ptr(out["x"]), ptr(out["w"]),
                          ptr(out["b"]))
    if rc != 0:
        raise ValueError(f"synth_linear rejected workload {w}")
    return out["x"], out["w"], out["b"]
