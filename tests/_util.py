"""Shared helpers of the parity tests: metrics and head-sliced oracle calls."""
from __future__ import annotations

import numpy as np

import oracle
import synth

# Tolerances of the path (quantized vs emulation, quantized vs exact, bf16 vs exact)
COS_EMUL = 0.9999
MAXABS_EMUL = 5e-3          # x max|V| of the head
COS_EXACT = 0.995
REL_L2_BF16 = 4e-3


def cos(a, b) -> float:
    a = np.asarray(a, np.float64).ravel()
    b = np.asarray(b, np.float64).ravel()
    na, nb = np.linalg.norm(a), np.linalg.norm(b)
    if na == 0 and nb == 0:
        return 1.0
    return float(a @ b / (na * nb))


def rel_l2(got, want) -> float:
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    return float(np.linalg.norm(got - want) / np.linalg.norm(want))


def bf16_to_np(t) -> np.ndarray:
    """torch bf16 tensor -> fp32 numpy."""
    import torch
    return t.detach().to("cpu").view(torch.int16).numpy().view(np.uint16).astype(np.uint32).__lshift__(16).view(np.float32)


def heads(a: np.ndarray, hs) -> np.ndarray:
    """Contiguous [B, len(hs), N, d] slice of a [B, H, N, d] array."""
    return np.ascontiguousarray(a[:, list(hs)])


def small_workloads():
    """Ragged and degenerate shapes the oracle finishes in seconds."""
    W = synth.Workload
    return [
        synth.WORKLOADS["tiny"],
        W("n1", 1, 1, 1, 128, seed=21),
        W("n127_d64", 1, 2, 127, 64, seed=22),
        W("n129", 1, 3, 129, 128, seed=23, zero_k_channel=7),
        W("n1000_d64_b2", 2, 2, 1000, 64, seed=24, outlier_frac=0.01),
        W("n640_outlier", 1, 2, 640, 128, seed=25, outlier_frac=0.01),
        W("n385", 1, 1, 385, 128, seed=26, k_off_std=0.0),
    ]


def emul_and_exact(q, k, v, rows):
    """Oracle prepass + O2 (fp32) and O1 (fp64) for the given rows of every head."""
    pre = oracle.prepass(q, k, v)
    o2, _ = oracle.attn_emul(pre, rows)
    o1 = oracle.attn_exact(q, k, v, rows)
    return pre, o2, o1


def ulysses_ref_permute(src, dst, B, Nl, H, d, P, op):
    """The four Ulysses layout copies written with torch reshapes / permutes (dense [P] side).
    Exchange layout [P, B, Nl, Hl, d]: chunk r holds the sender's tokens for heads r*Hl .. r*Hl + Hl - 1."""
    Hl = H // P
    if op == 0:      # send: [B, Nl, H, d] -> [P, B, Nl, Hl, d]
        dst.copy_(src.reshape(B, Nl, P, Hl, d).permute(2, 0, 1, 3, 4))
    elif op == 1:    # receive O: [P, B, Nl, Hl, d] -> [B, Nl, H, d]
        dst.copy_(src.reshape(P, B, Nl, Hl, d).permute(1, 2, 0, 3, 4).reshape(B, Nl, H, d))
    elif op == 2:    # gather: [P, B, Nl, Hl, d] -> [B, Hl, P * Nl, d]
        dst.copy_(src.reshape(P, B, Nl, Hl, d).permute(1, 3, 0, 2, 4).reshape(B, Hl, P * Nl, d))
    else:            # scatter: [B, Hl, P * Nl, d] -> [P, B, Nl, Hl, d]
        dst.copy_(src.reshape(B, Hl, P, Nl, d).permute(2, 0, 3, 1, 4))
    return dst


def attention_seqpar_ref(q, k, v, mode, o, workspace=None):
    """attention_per_head_ref on the [P, B, Nl, Hl, d] exchange layout: gather, attend, scatter."""
    import torch
    P, B, Nl, Hl, d = q.shape
    g = lambda t: t.permute(1, 3, 0, 2, 4).reshape(B, Hl, P * Nl, d)
    out = attention_per_head_ref(g(q), g(k), g(v), mode, torch.empty((B, Hl, P * Nl, d), dtype=o.dtype))
    o.copy_(out.reshape(B, Hl, P, Nl, d).permute(2, 0, 3, 1, 4))
    return o


def attention_per_head_ref(q, k, v, mode, o, workspace=None):
    """softmax(q k^T / sqrt(d)) v per (b, h) in float64, rounded to o's dtype; [B, H, N, d]."""
    import torch
    B, H, N, d = q.shape
    for b in range(B):
        for h in range(H):
            s = (q[b, h].double() @ k[b, h].double().T) / d ** 0.5
            p = torch.softmax(s, dim=-1)
            o[b, h] = (p @ v[b, h].double()).to(o.dtype)
    return o
