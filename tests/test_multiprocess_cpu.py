"""Multi-process host path of bench.py on the CPU: two gloo ranks, each timing its
own copy of the workload, combine the slowest rank's time with one all-reduce MAX
and report whole-job throughput. No GPU is involved."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        local_ms = [10.0, 12.5][rank]
        slowest = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        value = bench.whole_job_tflops(20_724_000_000_000, world, 4, slowest)
        q.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    for rank, slowest, value in got:
        assert slowest == 12.5
        # 2 ranks x 4 steps x 20.724 TFLOP in 12.5 ms
        assert value == pytest.approx(2 * 4 * 20.724 / 12.5e-3)


def test_single_rank_needs_no_collective():
    import bench
    assert bench.max_over_ranks(3.0, 1, torch.device("cpu")) == 3.0
    assert bench.whole_job_tflops(10**12, 1, 1, 1000.0) == pytest.approx(1.0)


def _split_worker(rank, world, port, q):
    """Each gloo rank takes its share of one problem's heads, 'times' it, and
    reports the whole problem's throughput over the slowest rank."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        h0, h1 = bench.split_heads(12, world, rank)
        local_ms = 1.0 * (h1 - h0)            # time proportional to the heads a rank runs
        slowest = bench.max_over_ranks(local_ms, world, torch.device("cpu"))
        value = bench.strong_tflops(20_724_000_000_000, 4, slowest)
        q.put((rank, h0, h1, slowest, value))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_head_split_reports_the_whole_problem_over_the_slowest_rank(world):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_split_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    got = sorted(q.get(timeout=5) for _ in range(world))
    # the ranks' head ranges tile [0, 12) in order
    assert [g[1] for g in got] == [0] + [g[2] for g in got[:-1]] and got[-1][2] == 12
    for rank, h0, h1, slowest, value in got:
        assert slowest == 12 / world                      # 12 heads split evenly
        # one C2 problem (20.724 TFLOP) per step, 4 steps, in the slowest rank's time
        assert value == pytest.approx(4 * 20.724 / (slowest * 1e-3))


def test_head_split_covers_every_head_once():
    import bench
    for H in (1, 5, 12, 40):
        for world in (1, 2, 3, 4, 8):
            ranges = [bench.split_heads(H, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == H
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 0


def test_tile_split_parts_balance_for_the_bench_workload():
    """The default multi-GPU mode deals C2's 512 query tiles over the ranks by
    cost: with 8 ranks the slowest part carries at most one tile's work more
    than an even share, so the ideal speed-up is close to 8 (the head split
    tops out at 6: 12 heads over 8 GPUs)."""
    import masked_attention_jvp_b200 as caj
    from masked_attention_jvp_b200.workloads import WORKLOADS
    m = WORKLOADS["wan1.3b_tf_framewise"].mask
    N = m.seq_len
    cost = [caj.qtile_key_tiles(m, 128 * t, min(128 * t + 128, N))[0] for t in range((N + 127) // 128)]
    for world in (2, 4, 8):
        loads = [sum(cost[t] for t in caj.part_query_tiles(m, r, world)) for r in range(world)]
        assert sum(cost) / max(loads) >= world * 0.99
