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
