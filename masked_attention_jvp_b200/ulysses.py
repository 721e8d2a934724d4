"""Ulysses context parallelism for the fused attention forward + JVP.

Causal-rCM trains with flattened Ulysses context parallelism (section 3.2.1,
"Parallelism"): the flattened video tokens are sharded over P ranks as
[B, H, L/P, C]. An all-to-all turns that into [B, H/P, L, C], local attention
runs over the full sequence for H/P heads, and a second all-to-all returns the
output. Section 3.2.2 ("JVP Ulysses CP") extends this to the JVP: the tangents
follow exactly the communication pattern of their primals, the local attention
is the masked attention JVP kernel, and the output tangent returns through the
same all-to-all as the output.

Here the six inputs travel in one all-to-all. The four outputs return one of
two ways:
  - two all-to-alls (the bf16 pair O, tO and the fp32 pair LSE, tLSE), or
  - with fused_output=True, no collective at all: the kernel's epilogue writes
    every output row into the symmetric-memory slice buffers of the rank that
    owns its tokens (caj_attn_fwd_jvp_scatter), over NVLink, and two
    stream-ordered barriers fence the writes.
The mask needs no translation, because the local call sees the whole packed
sequence. Collectives go through torch.distributed (NCCL over NVLink on GPUs).
All arithmetic is in the local kernel.
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


class SliceBuffers:
    """This rank's output slice in symmetric memory, mapped on every rank.

    One allocation holds O, tO [B, H, Ls, D], LSE, tLSE [B, H, Ls] fp32 and a
    pad of signal words for the barrier (regions 256-byte aligned). o[r],
    to[r], lse[r], tlse[r] view rank r's copy: rank r's device memory, reached
    over NVLink for r != this rank."""

    def __init__(self, B: int, H: int, Ls: int, D: int, dtype: torch.dtype, device, group=None):
        import torch.distributed._symmetric_memory as symm_mem

        def up(x):
            return (x + 255) // 256 * 256

        es = torch.empty((), dtype=dtype).element_size()
        n_out, n_st = B * H * Ls * D, B * H * Ls
        offs = [0, up(n_out * es), 2 * up(n_out * es), 2 * up(n_out * es) + up(n_st * 4)]
        pad_off = offs[3] + up(n_st * 4)
        total = pad_off + 256
        self.key = (B, H, Ls, D, dtype, torch.device(device))
        self.buf = symm_mem.empty(total, dtype=torch.uint8, device=device)
        # the signal pad starts at zero before any peer can reach it: the
        # rendezvous below is the first point where peers learn its address
        self.buf.zero_()
        torch.cuda.synchronize(device)
        self.handle = symm_mem.rendezvous(self.buf, group if group is not None else dist.group.WORLD)
        self.rank, self.world = self.handle.rank, self.handle.world_size
        hd = self.handle

        def view(r, off, shape, dt):
            return hd.get_buffer(r, shape, dt, off // torch.empty((), dtype=dt).element_size())

        P = self.world
        self.o = [view(r, offs[0], (B, H, Ls, D), dtype) for r in range(P)]
        self.to = [view(r, offs[1], (B, H, Ls, D), dtype) for r in range(P)]
        self.lse = [view(r, offs[2], (B, H, Ls), torch.float32) for r in range(P)]
        self.tlse = [view(r, offs[3], (B, H, Ls), torch.float32) for r in range(P)]
        self.pads = [view(r, pad_off, (64,), torch.int32).data_ptr() for r in range(P)]
        self.epoch = 0

    def barrier(self, timeout_ms: int = 10000):
        """Stream-ordered barrier over the group's ranks: the library's signal
        kernel over the mapped pads (caj_signal_barrier). A peer that does not
        arrive within timeout_ms makes the kernel record a timeout, which
        masked_attention_jvp_b200.device_status() raises; nothing traps.
        Every rank calls it the same number of times, so the epochs agree."""
        from . import signal_barrier
        self.epoch += 1
        signal_barrier(self.pads, self.rank, self.epoch, timeout_ms)


class _LocalSlices:
    """The one slice of a single process without a process group: ordinary
    device memory, and nothing to wait for."""

    def __init__(self, B: int, H: int, Ls: int, D: int, dtype: torch.dtype, device):
        self.rank, self.world = 0, 1
        self.o = [torch.empty(B, H, Ls, D, dtype=dtype, device=device)]
        self.to = [torch.empty_like(self.o[0])]
        self.lse = [torch.empty(B, H, Ls, dtype=torch.float32, device=device)]
        self.tlse = [torch.empty_like(self.lse[0])]

    def barrier(self, timeout_ms: int = 10000):
        pass


_slice_buffers = {}


def _get_slice_buffers(B, H, Ls, D, dtype, device, group):
    # whether a process group exists, and its size, are part of the key: local
    # slices made before init_process_group never serve a group afterwards
    key = (B, H, Ls, D, dtype, torch.device(device), id(group), dist.is_initialized(), _world(group))
    sb = _slice_buffers.get(key)
    if sb is None:
        if dist.is_initialized():
            sb = SliceBuffers(B, H, Ls, D, dtype, device, group)
        else:
            sb = _LocalSlices(B, H, Ls, D, dtype, device)
        _slice_buffers[key] = sb
    return sb


def ulysses_attn_fwd_jvp(q, k, v, tq, tk, tv, mask, scale: Optional[float] = None, group=None,
                         clean_tangent_zero: bool = False,
                         local_fn: Optional[Callable] = None, fused_output: bool = False):
    """Context-parallel forward + JVP.

    q..tv: this rank's sequence shard, [B, H, N/P, D], where shard r holds
    tokens [r*N/P, (r+1)*N/P) of the packed sequence described by `mask`.
    Returns (o, to, lse, tlse) for the same shard: [B, H, N/P, D] and
    [B, H, N/P]. local_fn(q, k, v, tq, tk, tv, mask, scale=..., clean_tangent_zero=...)
    computes attention on the head-sharded full sequence. It defaults to the
    fused kernel (masked_attention_jvp_b200.attn_fwd_jvp).

    fused_output=True (CUDA tensors, the fused kernel): the output all-to-all
    is done by the kernel's epilogue, which stores each row into the
    symmetric-memory slice buffer of its owner (see SliceBuffers). The
    returned tensors are copies, so the slice buffers are free for the next
    call once every rank has passed its first barrier. Without a process group
    (a single process) the one slice is ordinary device memory. The barriers
    are bounded: a peer that never arrives leaves a timeout status, raised by
    masked_attention_jvp_b200.device_status(), not a trapped GPU.
    """
    ins = torch.stack([q, k, v, tq, tk, tv])
    if fused_output:
        if local_fn is not None:
            raise ValueError("fused_output runs the fused kernel; local_fn does not apply")
        return _ulysses_fused_output(ins, mask, scale, group, clean_tangent_zero)
    if local_fn is None:
        from . import attn_fwd_jvp as local_fn
    full = seq_to_head(ins, group)
    o, to, lse, tlse = local_fn(*full.unbind(0), mask, scale=scale,
                                clean_tangent_zero=clean_tangent_zero)
    out = head_to_seq(torch.stack([o, to]), group)
    stats = head_to_seq(torch.stack([lse, tlse]).unsqueeze(-1), group).squeeze(-1)
    return out[0], out[1], stats[0], stats[1]


def _ulysses_fused_output(ins, mask, scale, group, clean_tangent_zero, slices=None, scatter_fn=None):
    """The fused-output path. `slices` (default: this group's SliceBuffers)
    provides rank, o, to, lse, tlse and barrier(); `scatter_fn` (default: the
    scattering kernel, attn_fwd_jvp_scatter) stores this rank's heads into
    every slice. Both are replaceable so that the multi-rank control flow can
    run on CPU ranks."""
    P = _world(group)
    _, B, H, Ls, D = ins.shape
    if H % P:
        raise ValueError(f"heads ({H}) must divide evenly over {P} ranks")
    full = seq_to_head(ins, group)
    Hp = H // P
    sb = slices if slices is not None else _get_slice_buffers(B, H, Ls, D, ins.dtype, ins.device, group)
    if scatter_fn is None:
        from . import attn_fwd_jvp_scatter as scatter_fn
    # every rank has copied its previous results out of its slice buffer
    sb.barrier()
    scatter_fn(*full.unbind(0), mask, sb.o, sb.to, sb.lse, sb.tlse, head_base=sb.rank * Hp,
               scale=scale, clean_tangent_zero=clean_tangent_zero)
    # every rank's rows have landed in this rank's slice buffer
    sb.barrier()
    me = sb.rank
    return sb.o[me].clone(), sb.to[me].clone(), sb.lse[me].clone(), sb.tlse[me].clone()


def release_slice_buffers() -> None:
    """Drops the cached slice buffers (before the process group goes away)."""
    _slice_buffers.clear()
