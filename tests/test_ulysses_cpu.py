"""Ulysses context parallelism on the CPU with gloo ranks: the all-to-all layout
transforms and the whole sequence-sharded forward + JVP, with the fp64 oracle as
the local attention (so no GPU is involved), against the oracle on the unsharded
problem."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from masked_attention_jvp_b200.workloads import MaskDesc


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(B, H, N, D, seed):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(B, H, N, D, generator=g, dtype=torch.float64) for _ in range(6)]


def _oracle_local(q, k, v, tq, tk, tv, mask, scale=None, clean_tangent_zero=False):
    import oracle
    o, to, lse, tlse = oracle.attn_fwd_jvp(q, k, v, tq, tk, tv, mask, scale=scale)
    return tuple(torch.from_numpy(x) for x in (o, to, lse, tlse))


def _worker(rank, world, port, mask, B, H, D, q_out):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from masked_attention_jvp_b200.ulysses import head_to_seq, seq_to_head, ulysses_attn_fwd_jvp
        N = mask.seq_len
        Ls = N // world
        full = _inputs(B, H, N, D, seed=7)
        shard = [x[:, :, rank * Ls:(rank + 1) * Ls].contiguous() for x in full]
        # layout: seq -> head gives this rank's heads over the whole sequence, and back
        st = torch.stack(shard)
        hs = seq_to_head(st)
        Hp = H // world
        want = torch.stack(full)[:, :, rank * Hp:(rank + 1) * Hp]
        layout_ok = torch.equal(hs, want) and torch.equal(head_to_seq(hs), st)
        o, to, lse, tlse = ulysses_attn_fwd_jvp(*shard, mask, local_fn=_oracle_local)
        q_out.put((rank, layout_ok, o.numpy(), to.numpy(), lse.numpy(), tlse.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,mask", [(2, MaskDesc(3, 1, 4, 1)), (2, MaskDesc(5, 1, 4, 0)),
                                        (4, MaskDesc(2, 2, 4, 1))])
def test_ulysses_matches_unsharded_oracle(world, mask):
    import oracle
    B, H, D = 1, 4, 8
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, mask, B, H, D, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = {}
    for _ in range(world):
        rank, layout_ok, o, to, lse, tlse = q.get(timeout=120)
        got[rank] = (layout_ok, o, to, lse, tlse)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    ro, rto, rlse, rtlse = oracle.attn_fwd_jvp(*_inputs(B, H, mask.seq_len, D, seed=7), mask)
    Ls = mask.seq_len // world
    for r in range(world):
        layout_ok, o, to, lse, tlse = got[r]
        assert layout_ok
        sl = slice(r * Ls, (r + 1) * Ls)
        assert np.array_equal(o, ro[:, :, sl]) and np.array_equal(to, rto[:, :, sl])
        assert np.array_equal(lse, rlse[:, :, sl]) and np.array_equal(tlse, rtlse[:, :, sl])


def test_single_rank_is_the_local_call():
    from masked_attention_jvp_b200.ulysses import ulysses_attn_fwd_jvp
    mask = MaskDesc(3, 1, 3, 1)
    xs = _inputs(1, 2, mask.seq_len, 4, seed=3)
    a = ulysses_attn_fwd_jvp(*xs, mask, local_fn=_oracle_local)
    b = _oracle_local(*xs, mask)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


class _HostSlices:
    """Slice buffers of the fused-output path for CPU ranks: shared-memory
    tensors that every rank maps (entry r is rank r's slice), and a gloo barrier
    in place of the stream-ordered one."""

    def __init__(self, rank, o, to, lse, tlse):
        self.rank = rank
        self.o, self.to, self.lse, self.tlse = o, to, lse, tlse

    def barrier(self):
        dist.barrier()


def _oracle_scatter(q, k, v, tq, tk, tv, mask, o, to, lse, tlse, head_base, scale=None,
                    clean_tangent_zero=False):
    """What the scattering kernel does, with the oracle as the arithmetic: this
    rank's heads over the whole sequence, each row stored into the slice that
    owns its token, at the rank's head offset."""
    ro, rto, rlse, rtlse = _oracle_local(q, k, v, tq, tk, tv, mask, scale=scale)
    P, Hp = len(o), q.shape[1]
    Ls = q.shape[2] // P
    hs = slice(head_base, head_base + Hp)
    for r in range(P):
        rows = slice(r * Ls, (r + 1) * Ls)
        o[r][:, hs] = ro[:, :, rows]
        to[r][:, hs] = rto[:, :, rows]
        lse[r][:, hs] = rlse[:, :, rows]
        tlse[r][:, hs] = rtlse[:, :, rows]


def _fused_worker(rank, world, port, mask, B, H, D, slices, q_out):
    import datetime
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        from masked_attention_jvp_b200.ulysses import _ulysses_fused_output
        Ls = mask.seq_len // world
        sb = _HostSlices(rank, *slices)
        outs = []
        for seed in (11, 12):  # the second call reuses the slice buffers
            full = _inputs(B, H, mask.seq_len, D, seed=seed)
            shard = torch.stack([x[:, :, rank * Ls:(rank + 1) * Ls].contiguous() for x in full])
            res = _ulysses_fused_output(shard, mask, None, None, False, slices=sb, scatter_fn=_oracle_scatter)
            outs.append([t.numpy() for t in res])
        q_out.put((rank, outs))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,mask", [(2, MaskDesc(3, 1, 4, 1)), (4, MaskDesc(2, 2, 4, 1))])
def test_fused_output_control_flow_matches_unsharded_oracle(world, mask):
    """The fused-output path at world sizes 2 and 4: input all-to-all, each
    rank's head offset, both barriers and the copy-out, twice over the same
    slice buffers, against the oracle on the unsharded problem."""
    import oracle
    B, H, D = 1, 4, 8
    Ls = mask.seq_len // world
    nan = float("nan")
    slices = tuple([torch.full(shape, nan, dtype=torch.float64).share_memory_() for _ in range(world)]
                   for shape in ((B, H, Ls, D), (B, H, Ls, D), (B, H, Ls), (B, H, Ls)))
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_fused_worker, args=(r, world, port, mask, B, H, D, slices, q))
             for r in range(world)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for call, seed in enumerate((11, 12)):
        want = oracle.attn_fwd_jvp(*_inputs(B, H, mask.seq_len, D, seed=seed), mask)
        for r in range(world):
            sl = slice(r * Ls, (r + 1) * Ls)
            for x, y in zip(got[r][call], want):
                assert np.array_equal(x, y[:, :, sl]), (r, call)


def test_fused_output_without_process_group_is_the_local_call():
    """A single process with no process group: the fused path uses one local
    slice and no barrier, and returns the local attention."""
    from masked_attention_jvp_b200.ulysses import _ulysses_fused_output, release_slice_buffers
    assert not dist.is_initialized()
    mask = MaskDesc(3, 1, 3, 1)
    xs = _inputs(1, 2, mask.seq_len, 4, seed=5)
    try:
        got = _ulysses_fused_output(torch.stack(xs), mask, None, None, False, scatter_fn=_oracle_scatter)
    finally:
        release_slice_buffers()
    o, to, lse, tlse = _oracle_local(*xs, mask)
    assert torch.equal(got[0], o) and torch.equal(got[1], to)
    # the statistics slices are fp32, as the kernel writes them
    assert torch.equal(got[2], lse.float()) and torch.equal(got[3], tlse.float())
