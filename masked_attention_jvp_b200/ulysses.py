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
    every output row into the slice buffer of the rank that owns its tokens
    (caj_attn_fwd_jvp_scatter), mapped from that rank by CUDA IPC, over NVLink,
    and two stream-ordered barriers (caj_signal_barrier) fence the writes.
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


class PeerView:
    """A [shape] view of `dtype` elements at a device address mapped from
    another rank (an IPC mapping). It offers what attn_fwd_jvp_scatter reads
    from a slice buffer (shape, dtype, data_ptr) and nothing else: peer memory
    is written by the scattering kernel, never through PyTorch here."""

    is_cuda = True

    def __init__(self, address: int, shape, dtype: torch.dtype):
        self._address = int(address)
        self.shape = torch.Size(shape)
        self.dtype = dtype

    def data_ptr(self) -> int:
        return self._address

    def dim(self) -> int:
        return len(self.shape)

    def is_contiguous(self) -> bool:
        return True


class SliceBuffers:
    """This rank's output slice, mapped by every rank of the group.

    One device allocation holds O, tO [B, H, Ls, D], LSE, tLSE [B, H, Ls] fp32
    and a pad of signal words for the barrier (regions 256-byte aligned). The
    ranks swap CUDA IPC handles of their allocations (one all_gather_object)
    and each maps the others' as plain peer memory: no multicast object is
    created or bound. o[r], to[r], lse[r], tlse[r] are rank r's slice: this
    rank's own tensors for r == rank, PeerView mappings reached over NVLink
    for the others."""

    def __init__(self, B: int, H: int, Ls: int, D: int, dtype: torch.dtype, device, group=None):
        from . import ipc_export, ipc_open

        def up(x):
            return (x + 255) // 256 * 256

        es = torch.empty((), dtype=dtype).element_size()
        n_out, n_st = B * H * Ls * D, B * H * Ls
        offs = [0, up(n_out * es), 2 * up(n_out * es), 2 * up(n_out * es) + up(n_st * 4)]
        pad_off = offs[3] + up(n_st * 4)
        total = pad_off + 256
        self.key = (B, H, Ls, D, dtype, torch.device(device))
        self.rank, self.world = dist.get_rank(group), dist.get_world_size(group)
        # zeroed (the signal pad included) before any peer can learn its address
        self.buf = torch.zeros(total, dtype=torch.uint8, device=device)
        torch.cuda.synchronize(device)
        handles = [None] * self.world
        dist.all_gather_object(handles, ipc_export(self.buf), group=group)
        self._opened = []
        bases = []
        for r in range(self.world):
            if r == self.rank:
                bases.append(self.buf.data_ptr())
            else:
                addr = ipc_open(handles[r])
                self._opened.append(addr)
                bases.append(addr)
        me = self.rank

        def view(r, off, shape, dt):
            if r == me:
                n = 1
                for x in shape:
                    n *= x
                return self.buf[off:off + n * torch.empty((), dtype=dt).element_size()].view(dt).view(shape)
            return PeerView(bases[r] + off, shape, dt)

        P = self.world
        self.o = [view(r, offs[0], (B, H, Ls, D), dtype) for r in range(P)]
        self.to = [view(r, offs[1], (B, H, Ls, D), dtype) for r in range(P)]
        self.lse = [view(r, offs[2], (B, H, Ls), torch.float32) for r in range(P)]
        self.tlse = [view(r, offs[3], (B, H, Ls), torch.float32) for r in range(P)]
        self.pads = [bases[r] + pad_off for r in range(P)]
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

    def close(self):
        """Unmaps the peers' slices (after this rank's last use of them)."""
        from . import ipc_close
        torch.cuda.synchronize(self.buf.device)
        for addr in self._opened:
            ipc_close(addr)
        self._opened = []


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
    slice buffer of its owner, mapped by CUDA IPC (see SliceBuffers). The
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
    """Unmaps and drops the cached slice buffers (before the process group
    goes away)."""
    for sb in _slice_buffers.values():
        close = getattr(sb, "close", None)
        if close is not None:
            close()
    _slice_buffers.clear()
