"""Ulysses context parallelism for the fused attention forward + JVP.

Causal-rCM trains with flattened Ulysses context parallelism (section 3.2.1,
"Parallelism"): the flattened video tokens are sharded over P ranks as
[B, H, L/P, C]. An all-to-all turns that into [B, H/P, L, C], local attention
runs over the full sequence for H/P heads, and a second all-to-all returns the
output. Section 3.2.2 ("JVP Ulysses CP") extends this to the JVP: the tangents
follow exactly the communication pattern of their primals, the local attention
is the masked attention JVP kernel, and the output tangent returns through the
same all-to-all as the output.

Here the six inputs travel in one all-to-all and the four outputs in two (the
bf16 pair O, tO and the fp32 pair LSE, tLSE). The mask needs no translation,
because the local call sees the whole packed sequence. Collectives go through
torch.distributed (NCCL over NVLink on GPUs). All arithmetic is in the local
kernel.
"""
from __future__ import annotations

from typing import Callable, Optional

import torch
import torch.distributed as dist


def _world(group) -> int:
    return dist.get_world_size(group) if dist.is_initialized() else 1


def seq_to_head(x: torch.Tensor, group=None) -> torch.Tensor:
    """[S, B, H, Ls, D] sequence-sharded (this rank holds tokens
    [rank*Ls, (rank+1)*Ls)) -> [S, B, H/P, P*Ls, D] head-sharded (this rank holds
    heads [rank*H/P, (rank+1)*H/P) over the whole sequence)."""
    P = _world(group)
    if P == 1:
        return x
    S, B, H, Ls, D = x.shape
    if H % P:
        raise ValueError(f"heads ({H}) must divide evenly over {P} ranks")
    send = x.reshape(S, B, P, H // P, Ls, D).permute(2, 0, 1, 3, 4, 5).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[src] holds the sequence shard of rank src for this rank's heads
    return recv.permute(1, 2, 3, 0, 4, 5).reshape(S, B, H // P, P * Ls, D)


def head_to_seq(y: torch.Tensor, group=None) -> torch.Tensor:
    """Inverse of seq_to_head: [S, B, H/P, N, E] -> [S, B, H, N/P, E]."""
    P = _world(group)
    if P == 1:
        return y
    S, B, Hp, N, E = y.shape
    if N % P:
        raise ValueError(f"sequence length ({N}) must divide evenly over {P} ranks")
    Ls = N // P
    send = y.reshape(S, B, Hp, P, Ls, E).permute(3, 0, 1, 2, 4, 5).contiguous()
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    # recv[src] holds head group src for this rank's sequence shard
    return recv.permute(1, 2, 0, 3, 4, 5).reshape(S, B, P * Hp, Ls, E)


def ulysses_attn_fwd_jvp(q, k, v, tq, tk, tv, mask, scale: Optional[float] = None, group=None,
                         clean_tangent_zero: bool = False,
                         local_fn: Optional[Callable] = None):
    """Context-parallel forward + JVP.

    q..tv: this rank's sequence shard, [B, H, N/P, D], where shard r holds
    tokens [r*N/P, (r+1)*N/P) of the packed sequence described by `mask`.
    Returns (o, to, lse, tlse) for the same shard: [B, H, N/P, D] and
    [B, H, N/P]. local_fn(q, k, v, tq, tk, tv, mask, scale=..., clean_tangent_zero=...)
    computes attention on the head-sharded full sequence. It defaults to the
    fused kernel (masked_attention_jvp_b200.attn_fwd_jvp).
    """
    if local_fn is None:
        from . import attn_fwd_jvp as local_fn
    ins = torch.stack([q, k, v, tq, tk, tv])
    full = seq_to_head(ins, group)
    o, to, lse, tlse = local_fn(*full.unbind(0), mask, scale=scale,
                                clean_tangent_zero=clean_tangent_zero)
    out = head_to_seq(torch.stack([o, to]), group)
    stats = head_to_seq(torch.stack([lse, tlse]).unsqueeze(-1), group).squeeze(-1)
    return out[0], out[1], stats[0], stats[1]
