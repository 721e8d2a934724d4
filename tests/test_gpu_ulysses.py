"""Ulysses path on the GPU with the real kernel: a one-rank NCCL group (this
machine gives one GPU per run), so the all-to-alls are identities and the result
must equal the direct call bit for bit. The fused-output form runs through
symmetric memory, its barriers and the scattering kernel on the same group.
Multi-rank layout and arithmetic are covered by the gloo tests on the CPU, and
the scatter over several slices by the emulated ranks of test_gpu_scatter."""
import contextlib
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist

import masked_attention_jvp_b200 as caj
from masked_attention_jvp_b200.ulysses import release_slice_buffers, ulysses_attn_fwd_jvp
from masked_attention_jvp_b200.workloads import MaskDesc, Workload, make_inputs

pytestmark = pytest.mark.gpu


@contextlib.contextmanager
def _one_rank_nccl_group():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("nccl", rank=0, world_size=1, timeout=datetime.timedelta(seconds=60),
                            device_id=torch.device("cuda", 0))
    try:
        yield
    finally:
        release_slice_buffers()
        dist.destroy_process_group()


def test_one_rank_nccl_group_equals_direct_call():
    with _one_rank_nccl_group():
        w = Workload("cp", 1, 4, 128, MaskDesc(100, 1, 4, 1), torch.bfloat16, seed=21)
        ins = make_inputs(w, "cuda")
        a = ulysses_attn_fwd_jvp(*ins, w.mask)
        b = caj.attn_fwd_jvp(*ins, w.mask)
        torch.cuda.synchronize()
        for x, y in zip(a, b):
            assert torch.equal(x, y)


def test_one_rank_fused_output_equals_direct_call():
    with _one_rank_nccl_group():
        # twice: the second call reuses the slice buffers
        for seed in (22, 23):
            w = Workload("cp", 1, 4, 128, MaskDesc(100, 1, 4, 1), torch.bfloat16, seed=seed)
            ins = make_inputs(w, "cuda")
            a = ulysses_attn_fwd_jvp(*ins, w.mask, fused_output=True)
            b = caj.attn_fwd_jvp(*ins, w.mask)
            torch.cuda.synchronize()
            for x, y in zip(a, b):
                assert torch.equal(x, y)
