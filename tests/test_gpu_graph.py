"""The hot-path entry points inside CUDA graphs.

Each call enqueues kernels on the caller's stream with everything they need
passed by value (tensor maps and tile orders travel in the kernel parameters)
and allocates nothing, so a call can be captured once and replayed. Each test
captures a call on fixed buffers, refills the inputs in place with fresh
seeded values, replays, and compares every output bit for bit with a direct
call on the fresh values. A replay that read stale inputs, or a launch whose
parameters were baked from the first capture's data, fails the comparison."""
import dataclasses

import pytest
import torch

import masked_attention_jvp_b200 as caj
from masked_attention_jvp_b200.workloads import MaskDesc, make_inputs, small, zero_clean_tangents

pytestmark = pytest.mark.gpu

# teacher-forcing layout, N = 3600: 29 query tiles with a ragged last one
W = small("graph", 1, 3, 128, MaskDesc(300, 1, 6, 1), torch.bfloat16, seed=61, std_tangent=0.5)


def _fresh(seed, ctz=False):
    w = dataclasses.replace(W, seed=seed)
    ins = make_inputs(w, "cuda")
    if ctz:
        zero_clean_tangents(w, *ins[3:])
    return ins


def _outs(q):
    return [torch.empty_like(q), torch.empty_like(q),
            torch.empty(q.shape[:3], device="cuda"), torch.empty(q.shape[:3], device="cuda")]


@pytest.mark.parametrize("ctz", [False, True], ids=["dense", "clean_tangent_zero"])
def test_forward_replays_on_refilled_inputs(ctz):
    torch.cuda.set_device(0)
    ins = _fresh(61, ctz)
    outs = _outs(ins[0])
    caj.attn_fwd_jvp_out(*ins, W.mask, *outs, clean_tangent_zero=ctz)  # per-device set-up outside capture
    torch.cuda.synchronize()
    caj.device_status()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        caj.attn_fwd_jvp_out(*ins, W.mask, *outs, clean_tangent_zero=ctz)
    for seed in (62, 63):
        fresh = _fresh(seed, ctz)
        for t, f in zip(ins, fresh):
            t.copy_(f)
        for t in outs:
            t.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        caj.device_status()
        want = caj.attn_fwd_jvp(*fresh, W.mask, clean_tangent_zero=ctz)
        torch.cuda.synchronize()
        for got, ref in zip(outs, want):
            assert torch.equal(got, ref)
    del g


def test_backward_replays_on_refilled_inputs():
    torch.cuda.set_device(0)

    def operands(seed):
        q, k, v = _fresh(seed)[:3]
        o, _, lse, _ = caj.attn_fwd_jvp(*_fresh(seed), W.mask)
        gen = torch.Generator(device="cuda").manual_seed(seed)
        dout = torch.randn(q.shape, device="cuda", generator=gen).to(torch.bfloat16)
        return [q, k, v, o, dout, lse]

    bufs = operands(61)
    caj.attn_bwd(*bufs, W.mask)
    torch.cuda.synchronize()
    caj.device_status()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        res = caj.attn_bwd(*bufs, W.mask)
    for seed in (62, 63):
        fresh = operands(seed)
        for t, f in zip(bufs, fresh):
            t.copy_(f)
        for t in res:
            t.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        caj.device_status()
        want = caj.attn_bwd(*fresh, W.mask)
        torch.cuda.synchronize()
        for got, ref in zip(res, want):
            assert torch.equal(got, ref)
    del g


def test_output_projection_replays_on_refilled_inputs():
    torch.cuda.set_device(0)
    M, K, C = 1000, 384, 640  # ragged in M and in C against the 256 x 256 tiles

    def operands(seed):
        gen = torch.Generator(device="cuda").manual_seed(seed)
        x = torch.randn((M, K), device="cuda", generator=gen).to(torch.bfloat16)
        tx = torch.randn((M, K), device="cuda", generator=gen).to(torch.bfloat16)
        w = (torch.randn((C, K), device="cuda", generator=gen) * K ** -0.5).to(torch.bfloat16)
        b = torch.randn((C,), device="cuda", generator=gen).to(torch.bfloat16)
        return [x, tx, w, b]

    bufs = operands(61)
    out = (torch.empty((M, C), dtype=torch.bfloat16, device="cuda"),
           torch.empty((M, C), dtype=torch.bfloat16, device="cuda"))
    caj.out_proj_jvp(*bufs, out=out)
    torch.cuda.synchronize()
    caj.device_status()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        caj.out_proj_jvp(*bufs, out=out)
    for seed in (62, 63):
        fresh = operands(seed)
        for t, f in zip(bufs, fresh):
            t.copy_(f)
        for t in out:
            t.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        caj.device_status()
        want = caj.out_proj_jvp(*fresh)
        torch.cuda.synchronize()
        for got, ref in zip(out, want):
            assert torch.equal(got, ref)
    del g
