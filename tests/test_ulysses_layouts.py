"""Pins the reference Ulysses layout copies (the check the CUDA copies are held to) against
brute-force index loops written from the layout definitions of include/sage.h, and the round trips
the exchange relies on.  DeepSpeed-Ulysses head split: rank r owns heads r*H/P .. (r+1)*H/P - 1 and
tokens r*N/P .. (r+1)*N/P - 1 (TMAP write-up, "Optimising multi-GPU parallelism").  Exchange buffers
are [P][B][Nl][Hl][d]: chunk r holds the sending rank's tokens for heads r*Hl .. r*Hl + Hl - 1."""
import itertools

import pytest
import torch

from _util import attention_per_head_ref, attention_seqpar_ref, ulysses_ref_permute


def _loops(src, B, Nl, H, d, P, op):
    Hl, N = H // P, P * Nl
    out = {0: torch.empty(P, B, Nl, Hl, d), 1: torch.empty(B, Nl, H, d), 2: torch.empty(B, Hl, N, d),
           3: torch.empty(P, B, Nl, Hl, d)}[op]
    for b, hl, n, r in itertools.product(range(B), range(Hl), range(Nl), range(P)):
        if op == 0:     # send: chunk r holds heads of rank r, this rank's tokens
            out[r, b, n, hl] = src[b, n, r * Hl + hl]
        elif op == 1:   # receive O: chunk r holds heads of rank r
            out[b, n, r * Hl + hl] = src[r, b, n, hl]
        elif op == 2:   # gather: chunk r came from rank r, i.e. tokens r*Nl + n
            out[b, hl, r * Nl + n] = src[r, b, n, hl]
        else:           # scatter: chunk r holds the tokens of rank r
            out[r, b, n, hl] = src[b, hl, r * Nl + n]
    return out


@pytest.mark.parametrize("B,Nl,H,d,P", [(1, 3, 4, 2, 2), (2, 2, 6, 1, 3), (1, 5, 8, 3, 4), (1, 4, 4, 2, 1)])
def test_reference_permutes_match_the_definitions(B, Nl, H, d, P):
    g = torch.Generator().manual_seed(B * 100 + Nl * 10 + P)
    Hl, N = H // P, P * Nl
    shapes = {0: (B, Nl, H, d), 1: (P, B, Nl, Hl, d), 2: (P, B, Nl, Hl, d), 3: (B, Hl, N, d)}
    for op in range(4):
        src = torch.randn(shapes[op], generator=g)
        want = _loops(src, B, Nl, H, d, P, op)
        got = ulysses_ref_permute(src, torch.empty_like(want), B, Nl, H, d, P, op)
        assert torch.equal(got, want), op


def test_single_rank_layouts_coincide():
    """At P = 1 the send layout is the input and the O receive layout is the output."""
    B, Nl, H, d = 2, 5, 3, 4
    x = torch.randn(B, Nl, H, d)
    assert torch.equal(ulysses_ref_permute(x, torch.empty(1, B, Nl, H, d), B, Nl, H, d, 1, 0).view(B, Nl, H, d), x)
    assert torch.equal(ulysses_ref_permute(x.view(1, B, Nl, H, d), torch.empty(B, Nl, H, d), B, Nl, H, d, 1, 1), x)


def test_exchange_round_trips():
    """Send then receive with every rank's chunks swapped is the head/sequence re-partition, and the
    O path undoes it: the P ranks' outputs, concatenated over tokens, are the per-head inputs."""
    B, Nl, H, d, P = 1, 3, 6, 2, 3
    Hl, N = H // P, P * Nl
    full = torch.randn(B, N, H, d)                      # [B, N, H, d]
    sends = [ulysses_ref_permute(full[:, r * Nl:(r + 1) * Nl].contiguous(), torch.empty(P, B, Nl, Hl, d),
                                 B, Nl, H, d, P, 0) for r in range(P)]
    # all-to-all: rank r receives chunk r of every rank's send buffer, in rank order
    recvs = [torch.stack([sends[src][r] for src in range(P)]) for r in range(P)]
    local = [ulysses_ref_permute(recvs[r], torch.empty(B, Hl, N, d), B, Nl, H, d, P, 2) for r in range(P)]
    for r in range(P):                                   # rank r now has heads r*Hl.. for all tokens
        assert torch.equal(local[r], full[:, :, r * Hl:(r + 1) * Hl].permute(0, 2, 1, 3))
    o_sends = [ulysses_ref_permute(local[r], torch.empty(P, B, Nl, Hl, d), B, Nl, H, d, P, 3) for r in range(P)]
    o_recvs = [torch.stack([o_sends[src][r] for src in range(P)]) for r in range(P)]
    outs = [ulysses_ref_permute(o_recvs[r], torch.empty(B, Nl, H, d), B, Nl, H, d, P, 1) for r in range(P)]
    assert torch.equal(torch.cat(outs, dim=1), full)     # identity "attention": back to the input


def test_seqpar_reference_is_gather_attend_scatter():
    """The chunk-layout reference attention equals per-head attention on the gathered layout."""
    B, Nl, Hl, d, P = 1, 4, 2, 8, 3
    g = torch.Generator().manual_seed(11)
    q, k, v = (torch.randn(P, B, Nl, Hl, d, generator=g).to(torch.bfloat16) for _ in range(3))
    o = attention_seqpar_ref(q, k, v, 0, torch.empty_like(q))
    gath = lambda t: ulysses_ref_permute(t, torch.empty(B, Hl, P * Nl, d, dtype=t.dtype), B, Nl, P * Hl, d, P, 2)
    want = attention_per_head_ref(gath(q), gath(k), gath(v), 0, torch.empty(B, Hl, P * Nl, d, dtype=q.dtype))
    assert torch.equal(gath(o), want)
