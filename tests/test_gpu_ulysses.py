"""Ulysses path on the GPU with the real kernel: a one-rank NCCL group (this
machine gives one GPU per run), so the all-to-alls are identities and the result
must equal the direct call bit for bit, and the fp64 oracle within the bf16
tolerances of the parity tests. The fused-output form runs through the IPC
slice buffers, the library's signal barrier and the scattering kernel on the
same group, and through ordinary memory without a process group. Multi-rank layout
and arithmetic are covered by the gloo tests on the CPU, and the scatter over
several slices by the emulated ranks of test_gpu_scatter."""
import contextlib
import datetime
import os
import socket

import pytest
import torch
import torch.distributed as dist

import oracle

import masked_attention_jvp_b200 as caj
from masked_attention_jvp_b200.ulysses import release_slice_buffers, ulysses_attn_fwd_jvp
from masked_attention_jvp_b200.workloads import MaskDesc, Workload, make_inputs
from tests.test_gpu_parity import check_rows

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
        _check_oracle(a, ins, w)


def test_one_rank_fused_output_equals_direct_call():
    with _one_rank_nccl_group():
        # twice: the second call reuses the slice buffers
        for seed in (22, 23):
            w = Workload("cp", 1, 4, 128, MaskDesc(100, 1, 4, 1), torch.bfloat16, seed=seed)
            ins = make_inputs(w, "cuda")
            a = ulysses_attn_fwd_jvp(*ins, w.mask, fused_output=True)
            b = caj.attn_fwd_jvp(*ins, w.mask)
            torch.cuda.synchronize()
            caj.device_status()  # both signal barriers completed in time
            for x, y in zip(a, b):
                assert torch.equal(x, y)
            _check_oracle(a, ins, w)


def _check_oracle(outs, ins, w):
    """The returned shard (here: the whole sequence) against the fp64 oracle."""
    ref = oracle.attn_fwd_jvp_rows(*[t.cpu() for t in ins], w.mask)
    o, to, lse, tlse = outs
    got = (o.reshape(-1, w.D).float().cpu().numpy(), to.reshape(-1, w.D).float().cpu().numpy(),
           lse.reshape(-1).cpu().numpy(), tlse.reshape(-1).cpu().numpy())
    check_rows(got, ref, w.dtype, "ulysses")


def test_fused_output_without_process_group_on_the_device():
    """A single process with no process group: the one slice is ordinary device
    memory, the barriers are no-ops and the scattering kernel writes it."""
    assert not dist.is_initialized()
    torch.cuda.set_device(0)
    for seed in (24, 25):
        w = Workload("cp_local", 1, 4, 128, MaskDesc(100, 1, 4, 1), torch.bfloat16, seed=seed)
        ins = make_inputs(w, "cuda")
        a = ulysses_attn_fwd_jvp(*ins, w.mask, fused_output=True)
        b = caj.attn_fwd_jvp(*ins, w.mask)
        torch.cuda.synchronize()
        for x, y in zip(a, b):
            assert torch.equal(x, y)
        _check_oracle(a, ins, w)
    release_slice_buffers()


def test_signal_barrier_of_one_rank_passes():
    torch.cuda.set_device(0)
    pad = torch.zeros(64, dtype=torch.int32, device="cuda")
    for epoch in (1, 2, 3):
        caj.signal_barrier([pad.data_ptr()], 0, epoch, timeout_ms=1000)
    caj.device_status()
    assert pad[0].item() == 3


def test_signal_barrier_gives_up_on_a_peer_that_never_arrives():
    """Two ranks, but rank 1 never runs: the word it would write on rank 0's pad
    stays 0, so rank 0's wait runs out. The kernel records a timeout (site
    0xF0), returns, and the context stays usable."""
    torch.cuda.set_device(0)
    pads = [torch.zeros(64, dtype=torch.int32, device="cuda") for _ in range(2)]
    caj.signal_barrier([p.data_ptr() for p in pads], 0, 1, timeout_ms=100)
    with pytest.raises(caj.CajError) as ei:
        caj.device_status()
    assert ei.value.status == 4
    assert caj._lib.lib().caj_last_device_error_code() == 0x1F0
    assert pads[0][0].item() == 1 and pads[1][0].item() == 1  # rank 0 signalled both pads
    # the context still works: a normal call afterwards matches the oracle
    w = Workload("after_timeout", 1, 2, 128, MaskDesc(64, 1, 3, 1), torch.bfloat16, seed=26)
    ins = make_inputs(w, "cuda")
    out = caj.attn_fwd_jvp(*ins, w.mask)
    torch.cuda.synchronize()
    caj.device_status()
    _check_oracle(out, ins, w)
