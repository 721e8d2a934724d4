"""CUDA IPC slice buffers for the fused output all-to-all, on one GPU with two
processes.

Process A owns the buffers of sequence slice 1 and exports them
(caj_ipc_export). Process B maps them (caj_ipc_open) and runs the scattering
forward over every head: slice 0 goes to B's own memory, slice 1 through the
IPC mapping into A's memory, which is what a peer rank's slice is on a
multi-GPU run. The processes meet only on the host (a queue), never through a
GPU wait. A then checks its slice against its own direct call, bit for bit,
and against the fp64 oracle."""
import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import masked_attention_jvp_b200 as caj
from masked_attention_jvp_b200.workloads import MaskDesc, make_inputs, small
from tests.test_gpu_parity import check_rows

pytestmark = pytest.mark.gpu

W = small("ipc", 1, 4, 128, MaskDesc(100, 1, 4, 1), torch.bfloat16, seed=41)   # N = 800, slices of 400


def _writer(handles, q):
    """Process B: map slice 1, compute every head, scatter over both slices."""
    try:
        import masked_attention_jvp_b200 as caj2
        from masked_attention_jvp_b200.ulysses import PeerView
        torch.cuda.set_device(0)
        B, H, N, D = W.B, W.H, W.N, W.D
        Ls = N // 2
        ins = make_inputs(W, "cuda")
        mine = [torch.full((B, H, Ls, D), float("nan"), dtype=W.dtype, device="cuda") for _ in range(2)]
        mine += [torch.full((B, H, Ls), float("nan"), device="cuda") for _ in range(2)]
        addrs = [caj2.ipc_open(h) for h in handles]
        # a second open of a mapped handle gives the same address and needs its
        # own close; the first mapping stays usable (the scatter below writes
        # through it)
        again = caj2.ipc_open(handles[0])
        if again != addrs[0]:
            raise AssertionError(f"second open gave {again:#x}, first {addrs[0]:#x}")
        caj2.ipc_close(again)
        shapes = [((B, H, Ls, D), W.dtype)] * 2 + [((B, H, Ls), torch.float32)] * 2
        peer = [PeerView(a, s, dt) for a, (s, dt) in zip(addrs, shapes)]
        caj2.attn_fwd_jvp_scatter(*ins, W.mask, [mine[0], peer[0]], [mine[1], peer[1]],
                                  [mine[2], peer[2]], [mine[3], peer[3]])
        torch.cuda.synchronize()
        caj2.device_status()
        for a in addrs:
            caj2.ipc_close(a)
        # plain numpy arrays: torch tensors would travel as file descriptors that
        # this process must outlive
        q.put(("ok", [t.cpu().view(torch.int16).numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()
                      for t in mine]))
    except BaseException as e:  # report, never hang the parent
        q.put(("error", repr(e)))


def test_ipc_mapped_slice_receives_the_scattered_rows():
    torch.cuda.set_device(0)
    B, H, N, D = W.B, W.H, W.N, W.D
    Ls = N // 2
    theirs = [torch.full((B, H, Ls, D), float("nan"), dtype=W.dtype, device="cuda") for _ in range(2)]
    theirs += [torch.full((B, H, Ls), float("nan"), device="cuda") for _ in range(2)]
    torch.cuda.synchronize()
    handles = [caj.ipc_export(t) for t in theirs]
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    p = ctx.Process(target=_writer, args=(handles, q))
    p.start()
    status, payload = q.get(timeout=300)
    p.join(timeout=60)
    assert status == "ok", payload
    assert p.exitcode == 0
    payload = [torch.from_numpy(a).view(torch.bfloat16) if a.dtype == np.int16 else torch.from_numpy(a)
               for a in payload]
    torch.cuda.synchronize()
    ins = make_inputs(W, "cuda")
    direct = caj.attn_fwd_jvp(*ins, W.mask)
    torch.cuda.synchronize()
    s0, s1 = slice(0, Ls), slice(Ls, N)
    for got, want in zip(theirs, direct):          # slice 1, written through the IPC mapping
        assert torch.equal(got, want[:, :, s1])
    for got, want in zip(payload, direct):         # slice 0, B's own memory
        assert torch.equal(got, want[:, :, s0].cpu())
    full = [torch.cat([a.cpu(), b.cpu()], dim=2) for a, b in zip(payload, theirs)]
    ref = oracle.attn_fwd_jvp_rows(*[t.cpu() for t in ins], W.mask)
    got = (full[0].reshape(-1, D).float().numpy(), full[1].reshape(-1, D).float().numpy(),
           full[2].reshape(-1).numpy(), full[3].reshape(-1).numpy())
    check_rows(got, ref, W.dtype, "ipc slices")


def test_ipc_close_refuses_an_address_it_did_not_open():
    with pytest.raises(caj.CajError):
        caj.ipc_close(0x1000)
