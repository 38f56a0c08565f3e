"""DeepSpeed-Ulysses sequence-parallel attention around the sage kernels.

TMAP write-up, "Optimising multi-GPU parallelism": the sequence of a video
DiT is split over P GPUs.  Before attention an all-to-all gives every GPU the
whole sequence for H/P heads (attention is head-parallel, so the quantized
kernels run unchanged on full sequences), and a second all-to-all returns
the output to the sequence slices.  The all-to-all of q, k and v cost about
2/3 of the attention time there, and the pages hide part of it by starting
each exchange as soon as its tensor is computed, while the next projection
still runs.  `UlyssesAttention.send` does exactly that: each of q, k, v goes
into its send layout and its all-to-all starts at once (asynchronously, on
the communicator's stream); `attend` waits for the three, runs the attention
path on the local heads and brings O back.

Per rank: inputs [B, Nl, H, d] (this rank's Nl = N / P tokens, all heads),
output [B, Nl, H, d].  The exchange buffers are [P][B][Nl][Hl][d] (chunk r:
this rank's tokens, heads r*Hl .. r*Hl + Hl - 1, token-major), so:
  - at P = 1 the input already is the send layout and the exchange of one
    rank is the identity: attention reads the inputs and writes the output
    in place, and no collective runs;
  - at P > 1 the send copy and the O receive copy move contiguous runs of
    Hl * d values (`sage_ulysses_permute`);
  - the attention call `sage_attn_fwd_seqpar` reads q, k and v straight
    from the receive buffers (the quantization prepass walks the chunks) and
    writes O straight into the send buffer of the return exchange.
The collectives are torch.distributed's `all_to_all_single` (NCCL on GPUs).
"""
from __future__ import annotations

from . import sage


def _default_a2a(group):
    import torch.distributed as dist

    def a2a(out, inp):
        return dist.all_to_all_single(out, inp, group=group, async_op=True)
    return a2a


class UlyssesAttention:
    """One attention layer's Ulysses exchange for fixed shapes (buffers allocated once).

    permute(src, dst, B, Nl, H, d, P, op) and attention(q, k, v, mode, o, workspace) default to the
    CUDA kernels (`attention` takes and gives the [P][B][Nl][Hl][d] exchange layout); a2a(out, inp)
    -> handle defaults to an asynchronous all_to_all_single on `group`.
    """

    def __init__(self, B: int, Nl: int, H: int, d: int, world: int, mode: int = sage.MODE_INT8_FP8,
                 device=None, group=None, permute=None, attention=None, a2a=None):
        import torch
        if H % world:
            raise ValueError(f"H={H} is not divisible by the {world} ranks")
        self.B, self.Nl, self.H, self.d, self.P, self.mode = B, Nl, H, d, world, mode
        self.Hl, self.N = H // world, world * Nl
        dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        bf = torch.bfloat16
        chunk = (world, B, Nl, self.Hl, d)
        # at P = 1 the caller's tensor is sent as it is (same layout)
        multi = world > 1
        self.send_buf = {t: torch.empty(chunk, dtype=bf, device=dev) for t in "qkv"} if multi else {}
        self.recv_buf = {t: torch.empty(chunk, dtype=bf, device=dev) for t in "qkv"} if multi else {}
        self.o_send = torch.empty(chunk, dtype=bf, device=dev)
        self.o_recv = torch.empty(chunk, dtype=bf, device=dev) if multi else self.o_send
        self.out = torch.empty((B, Nl, H, d), dtype=bf, device=dev) if multi else self.o_send.view(B, Nl, H, d)
        self.workspace = None
        if attention is None and dev.type == "cuda":
            self.workspace = sage.alloc_seqpar_workspace(world, B, Nl, self.Hl, d, mode, dev)
        self._permute = permute or (lambda src, dst, *g: sage.ulysses_permute(src, dst, *g))
        self._attention = attention or (
            lambda q, k, v, m, o, ws: sage.attn_fwd_seqpar(q, k, v, m, o, world, workspace=ws))
        self._a2a = a2a or _default_a2a(group)
        self._pending = {}
        self._keep = {}

    def _geom(self, op):
        return (self.B, self.Nl, self.H, self.d, self.P, op)

    def send(self, which: str, x):
        """Start the exchange of q, k or v ([B, Nl, H, d] bf16): send layout, then an async all-to-all.
        At P = 1, x itself is sent: it must stay unchanged until attend_local()."""
        if which not in "qkv" or len(which) != 1:
            raise ValueError("which must be 'q', 'k' or 'v'")
        if tuple(x.shape) != (self.B, self.Nl, self.H, self.d):
            raise ValueError(f"{which} must be [B, Nl, H, d] = {(self.B, self.Nl, self.H, self.d)}")
        x = x.contiguous()
        if self.P == 1:
            # the exchange of one rank is the identity: attention reads x itself
            self._keep[which] = x.view(1, self.B, self.Nl, self.H, self.d)
            self._pending[which] = None
            return
        src = self.send_buf[which]
        self._permute(x, src, *self._geom(sage.ULYSSES_SEND))
        self._pending[which] = self._a2a(self.recv_buf[which], src)

    def attend_local(self):
        """Wait for q, k, v, run attention on the local heads (O lands in the send layout) and start
        O's way back."""
        missing = [t for t in "qkv" if t not in self._pending]
        if missing:
            raise RuntimeError(f"send() was not called for {missing}")
        for t in "qkv":
            h = self._pending.pop(t)
            if h is not None:
                h.wait()
        src = self._keep if self.P == 1 else self.recv_buf
        self._attention(src["q"], src["k"], src["v"], self.mode, self.o_send, self.workspace)
        self._keep = {}
        self._pending["o"] = self._a2a(self.o_recv, self.o_send) if self.P > 1 else None

    def finish(self):
        """Wait for O and return it for this rank's tokens, [B, Nl, H, d]."""
        h = self._pending.pop("o")
        if h is not None:
            h.wait()
        if self.P > 1:
            self._permute(self.o_recv, self.out, *self._geom(sage.ULYSSES_RECV_O))
        return self.out

    def attend(self):
        """attend_local() then finish(): O [B, Nl, H, d] for this rank's tokens."""
        self.attend_local()
        return self.finish()

    def __call__(self, q, k, v):
        for t, x in zip("qkv", (q, k, v)):
            self.send(t, x)
        return self.attend()
