"""Head-sharded execution of the op across ranks (one process per GPU), with
the all-to-all exchanges of Ulysses sequence parallelism around it.

Video DeltaNet (arXiv 2609.20744), Section 5, "Other optimizations": the
serving stack shards attention by head with Ulysses sequence parallelism, and
the linear branch runs on the head shards (Section 6.4 measures its scans at
seven heads per rank).  Outside the attention block every rank holds a
contiguous slice of the token sequence for all heads; the branch needs all
tokens of a head, since its scans run over every frame.  So:

  sequence shard  [B, H, S/P, ...]   (S = T * U tokens, frame-major)
      --all-to-all-->  head shard  [B, H/P, S, ...]  -> vda_forward per rank
      --all-to-all-->  sequence shard of the output  [B, H, S/P, d_v]

Every (batch, head) pair of the op is independent, so the per-rank forwards
need no collective; the two exchanges are the only cross-rank traffic, plain
all_to_all_single calls (NCCL over NVLink on GPUs, gloo on the CPU).
Requirements: H % P == 0 and (T * U) % P == 0.  Per-head inputs that are not
token activations (the initial states, the decay gates) are passed as the
rank's head shard.
"""

from __future__ import annotations

import torch
import torch.distributed as dist


def _world(group):
    return dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1


def _a2a(x, group):
    """all_to_all_single over dim 0 (equal splits); 16-bit floats travel as
    their bytes (not every backend carries them)."""
    raw = x.dtype in (torch.bfloat16, torch.float16)
    src = x.contiguous().view(torch.uint8) if raw else x.contiguous()
    out = torch.empty_like(src)
    dist.all_to_all_single(out, src, group=group)
    return out.view(x.dtype) if raw else out


def token_shard(x, rank, world, T, U):
    """The rank's sequence shard of a full tensor [B, H, T, U, ...]: tokens
    [rank * S / P, (rank + 1) * S / P) of the flattened (t, u) order, as
    [B, H, S / P, ...]."""
    B, H = x.shape[:2]
    S = T * U
    if S % world:
        raise ValueError(f"T * U = {S} is not divisible by {world} ranks")
    n = S // world
    return x.reshape(B, H, S, *x.shape[4:])[:, :, rank * n:(rank + 1) * n].contiguous()


def seq_to_heads(x_seq, group=None):
    """[B, H, S/P, ...] (this rank's tokens, every head) -> [B, H/P, S, ...]
    (every token, this rank's heads: [rank * H/P, (rank + 1) * H/P))."""
    P = _world(group)
    B, H, Sr = x_seq.shape[:3]
    rest = x_seq.shape[3:]
    if H % P:
        raise ValueError(f"H = {H} is not divisible by {P} ranks")
    Hp = H // P
    if P == 1:
        return x_seq
    # send block s: the heads of rank s, for this rank's tokens
    send = x_seq.reshape(B, P, Hp, Sr, *rest).transpose(0, 1)
    recv = _a2a(send, group)   # block s: rank s's tokens, for this rank's heads
    dims = list(range(recv.dim()))
    out = recv.permute(1, 2, 0, *dims[3:])   # [B, Hp, P, Sr, ...]
    return out.reshape(B, Hp, P * Sr, *rest)


def heads_to_seq(y_heads, group=None):
    """[B, H/P, S, ...] (this rank's heads) -> [B, H, S/P, ...] (this rank's
    tokens); the inverse of seq_to_heads."""
    P = _world(group)
    B, Hp, S = y_heads.shape[:3]
    rest = y_heads.shape[3:]
    if S % P:
        raise ValueError(f"S = {S} is not divisible by {P} ranks")
    Sr = S // P
    if P == 1:
        return y_heads
    dims = list(range(y_heads.dim() + 1))
    # send block s: this rank's heads, for rank s's tokens
    send = y_heads.reshape(B, Hp, P, Sr, *rest).permute(2, 0, 1, 3, *dims[4:])
    recv = _a2a(send, group)   # block s: rank s's heads, for this rank's tokens
    dims = list(range(recv.dim()))
    return recv.permute(1, 0, 2, *dims[3:]).reshape(B, P * Hp, Sr, *rest)


def vda_forward_ulysses(q, k, v, beta, gate, rms_weight, S0_fwd, S0_rev, T, U, chunk=5, window_chunks=1,
                        group=None, alpha=None, forward=None, **kw):
    """The forward on head shards.  q, k, gate [B, H, S/P, d_k], v [B, H, S/P,
    d_v], beta [B, H, S/P]: this rank's sequence shard (see token_shard).
    S0_fwd, S0_rev [B, H/P, d_v, d_k] and alpha [B, H/P, T, d_k]: this rank's
    heads (or None).  Returns the output's sequence shard [B, H, S/P, d_v].
    `forward` computes the head shard (default: api.vda_forward, the CUDA
    library); its keyword arguments pass through."""
    if forward is None:
        from . import api
        forward = api.vda_forward
    B = q.shape[0]

    def heads(x, d=None):
        y = seq_to_heads(x, group)
        return y.reshape(B, y.shape[1], T, U, *(() if d is None else (d,)))

    qh, kh, gh = heads(q, q.shape[-1]), heads(k, k.shape[-1]), heads(gate, gate.shape[-1])
    vh, bh = heads(v, v.shape[-1]), heads(beta)
    out = forward(qh, kh, vh, bh, gh, rms_weight, S0_fwd, S0_rev, chunk=chunk, window_chunks=window_chunks,
                  alpha=alpha, **kw)
    return heads_to_seq(out.reshape(B, out.shape[1], T * U, out.shape[-1]), group)
