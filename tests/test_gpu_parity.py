"""GPU parity: the CUDA path (called through the C-ABI) against the fp64 oracle
on the same seeded inputs.

Tolerances: fp32 inputs -> relative Frobenius error <= 1e-5 on O and tO (and
tLSE), max-abs <= 1e-5 on LSE. bf16 inputs with fp32 accumulation -> relative
Frobenius <= 1e-2 and max-abs <= 3e-2 on O and tO, relative Frobenius <= 1e-2 on
tLSE and max-abs <= 1e-2 on LSE. Small cases compare every output element; the
full-size workloads compare 512 seeded random rows per head plus the first and
last row of every chunk."""
import numpy as np
import pytest
import torch

import oracle
import masked_attention_jvp_b200 as caj
from masked_attention_jvp_b200.workloads import (MaskDesc, WORKLOADS, Workload, boundary_rows,
                                                 make_inputs, sample_rows, with_dtype)

pytestmark = pytest.mark.gpu

TOL = {
    torch.float32: dict(fro=1e-5, maxabs=None, lse=1e-5),
    torch.bfloat16: dict(fro=1e-2, maxabs=3e-2, lse=1e-2),
}


def rel_fro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def check_rows(got, ref, dtype, what="", maxabs_relative=False):
    """maxabs_relative: for inputs outside the workloads' distributions (larger
    scale or larger scores, hence larger outputs) the bf16 max-abs bound is taken
    relative to the largest reference magnitude."""
    o, to, lse, tlse = [np.asarray(x, np.float64) for x in got]
    ro, rto, rlse, rtlse = ref
    t = TOL[dtype]
    errs = dict(o_fro=rel_fro(o, ro), to_fro=rel_fro(to, rto), tlse_fro=rel_fro(tlse, rtlse),
                o_max=float(np.max(np.abs(o - ro))), to_max=float(np.max(np.abs(to - rto))),
                lse_max=float(np.max(np.abs(lse - rlse))))
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(to)), what
    assert errs["o_fro"] <= t["fro"], (what, errs)
    assert errs["to_fro"] <= t["fro"], (what, errs)
    assert errs["tlse_fro"] <= t["fro"], (what, errs)
    assert errs["lse_max"] <= t["lse"], (what, errs)
    if t["maxabs"] is not None:
        o_lim = t["maxabs"] * (max(1.0, float(np.max(np.abs(ro)))) if maxabs_relative else 1.0)
        to_lim = t["maxabs"] * (max(1.0, float(np.max(np.abs(rto)))) if maxabs_relative else 1.0)
        assert errs["o_max"] <= o_lim, (what, errs)
        assert errs["to_max"] <= to_lim, (what, errs, to_lim)
    return errs


def run_gpu(w: Workload):
    ins = make_inputs(w, "cuda")
    outs = caj.attn_fwd_jvp(*ins, w.mask, scale=w.scale)
    torch.cuda.synchronize()
    caj.device_status()
    return ins, outs


def gather(outs, rows, D):
    o, to, lse, tlse = outs
    idx = rows.to(o.device)
    return (o.reshape(-1, D)[idx].float().cpu().numpy(), to.reshape(-1, D)[idx].float().cpu().numpy(),
            lse.reshape(-1)[idx].cpu().numpy(), tlse.reshape(-1)[idx].cpu().numpy())


def full_check(w: Workload, maxabs_relative=False):
    ins, outs = run_gpu(w)
    ref = oracle.attn_fwd_jvp_rows(*[t.cpu() for t in ins], w.mask, scale=w.scale)
    rows = torch.arange(w.B * w.H * w.N)
    return check_rows(gather(outs, rows, w.D), ref, w.dtype, w.name, maxabs_relative)


# --------------------------------------------------------------- small, full outputs
def test_tiny_workload_fp32():
    full_check(WORKLOADS["tiny_framewise_fp32"])


def test_tiny_workload_bf16():
    full_check(with_dtype(WORKLOADS["tiny_framewise_fp32"], torch.bfloat16))


SMALL = [
    # (mask, B, H) -- several query/key tiles, ragged tails, both layouts
    (MaskDesc(100, 1, 5, 0), 1, 2),     # N=500, frame-wise, frames straddle tiles
    (MaskDesc(37, 1, 7, 1), 1, 2),      # N=518, TF frame-wise, seam inside a tile
    (MaskDesc(16, 3, 6, 1), 2, 1),      # N=192, TF chunk-wise
    (MaskDesc(1, 1, 300, 0), 1, 1),     # N=300, token-causal (single-key rows)
    (MaskDesc(600, 1, 1, 0), 1, 2),     # N=600, one frame: dense attention
    (MaskDesc(64, 1, 4, 1), 1, 1),      # N=512, tile-aligned TF
    (MaskDesc(5, 1, 3, 1), 1, 3),       # N=30, smaller than one tile
    (MaskDesc(200, 2, 4, 1), 1, 1),     # N=1600, TF chunk-wise, 2 frames per chunk
]


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("case", range(len(SMALL)))
def test_small_shapes_full(case, D, dtype):
    mask, B, H = SMALL[case]
    w = Workload(f"small{case}", B, H, D, mask, dtype, seed=100 + case, std_tangent=0.5)
    full_check(w)


@pytest.mark.parametrize("scale", [0.05, 0.3])
def test_explicit_scale(scale):
    w = Workload("scaled", 1, 2, 128, MaskDesc(50, 1, 6, 1), torch.bfloat16, seed=7, scale=scale)
    full_check(w, maxabs_relative=True)


def test_large_values_exercise_rescaling():
    """std 3 scores make the running max move by more than 2^8 between tiles."""
    w = Workload("wide", 1, 2, 128, MaskDesc(300, 1, 4, 1), torch.bfloat16, seed=8, std_qkv=3.0)
    full_check(w, maxabs_relative=True)


# ------------------------------------------------------ full-size workloads, sampled
@pytest.mark.parametrize("name", ["wan1.3b_framewise_infer", "wan1.3b_tf_framewise",
                                  "wan1.3b_tf_chunkwise", "h40_framewise_infer"])
def test_workload_sampled_rows(name):
    w = WORKLOADS[name]
    ins, outs = run_gpu(w)
    rows = torch.cat([sample_rows(w, 512), boundary_rows(w)])
    rows = torch.unique(rows)
    host = [t.cpu() for t in ins]
    del ins
    ref = oracle.attn_fwd_jvp_rows(*host, w.mask, scale=w.scale, rows=rows)
    check_rows(gather(outs, rows, w.D), ref, w.dtype, name)


# ------------------------------------------------------------------ invariants
def test_future_chunks_leave_earlier_rows_bitwise_unchanged():
    mask = MaskDesc(150, 1, 6, 1)
    w = Workload("inv", 1, 2, 128, mask, torch.bfloat16, seed=9)
    ins = [t.clone() for t in make_inputs(w, "cuda")]
    a = [t.clone() for t in caj.attn_fwd_jvp(*ins, mask)]
    L, G = 6 * 150, 150
    last = torch.cat([torch.arange(L - G, L), torch.arange(2 * L - G, 2 * L)]).cuda()
    g = torch.Generator(device="cpu").manual_seed(1)
    for t in ins:
        t[:, :, last] = (20 * torch.randn(t[:, :, last].shape, generator=g)).to(t.dtype).cuda()
    b = caj.attn_fwd_jvp(*ins, mask)
    keep = torch.ones(2 * L, dtype=torch.bool)
    keep[last.cpu()] = False
    keep = keep.cuda()
    for x, y in zip(a, b):
        assert torch.equal(x[:, :, keep], y[:, :, keep])


def test_repeated_calls_are_bitwise_identical():
    w = Workload("rep", 1, 4, 128, MaskDesc(333, 1, 5, 1), torch.bfloat16, seed=10)
    ins = make_inputs(w, "cuda")
    a = [t.clone() for t in caj.attn_fwd_jvp(*ins, w.mask)]
    b = caj.attn_fwd_jvp(*ins, w.mask)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("dtype", [torch.bfloat16, torch.float32], ids=["bf16", "fp32"])
def test_outputs_fully_overwritten(dtype):
    w = Workload("nan", 2, 3, 64, MaskDesc(70, 1, 4, 1), dtype, seed=11)
    ins = make_inputs(w, "cuda")
    o = torch.full(ins[0].shape, float("nan"), dtype=dtype, device="cuda")
    to = torch.full_like(o, float("nan"))
    lse = torch.full(ins[0].shape[:3], float("nan"), device="cuda")
    tlse = torch.full_like(lse, float("nan"))
    caj.attn_fwd_jvp_out(*ins, w.mask, o, to, lse, tlse)
    torch.cuda.synchronize()
    for t in (o, to, lse, tlse):
        assert torch.isfinite(t).all()


# (mask, B, H, D, dtype, pinned, clean_tangent_zero): head counts that fill 16
# chunks of one head, 14 chunks of 3 heads with a short last chunk, and one head
HOST = [(MaskDesc(90, 1, 4, 1), 1, 2, 128, torch.bfloat16, True, False),
        (MaskDesc(33, 2, 4, 0), 1, 13, 64, torch.bfloat16, True, False),
        (MaskDesc(20, 1, 3, 1), 4, 10, 128, torch.bfloat16, False, False),
        (MaskDesc(45, 2, 4, 1), 1, 3, 128, torch.bfloat16, True, True),
        (MaskDesc(17, 1, 3, 0), 1, 1, 64, torch.float32, True, False)]


@pytest.mark.parametrize("case", range(len(HOST)))
def test_host_entry_matches_device_path(case):
    """The host-buffer entry point (chunked copies overlapped with the kernels)
    gives bitwise the device path's results."""
    mask, B, H, D, dtype, pinned, ctz = HOST[case]
    w = Workload(f"host{case}", B, H, D, mask, dtype, seed=12 + case)
    host = make_inputs(w, "cpu")
    if ctz:
        from masked_attention_jvp_b200.workloads import zero_clean_tangents
        zero_clean_tangents(w, *host[3:])
    if pinned:
        host = [t.pin_memory() for t in host]
    a = caj.attn_fwd_jvp(*host, w.mask, clean_tangent_zero=ctz)
    assert all(not t.is_cuda for t in a)
    b = caj.attn_fwd_jvp(*[t.cuda() for t in host], w.mask, clean_tangent_zero=ctz)
    torch.cuda.synchronize()
    caj.device_status()
    for x, y in zip(a, b):
        assert torch.equal(x, y.cpu())


def test_host_entry_back_to_back_calls_reuse_nothing_stale():
    """Two host calls in a row on different inputs: the second call's results
    are its own (the copies of one call are ordered after the previous one)."""
    w1 = Workload("hostA", 1, 4, 128, MaskDesc(64, 1, 4, 1), torch.bfloat16, seed=31)
    w2 = Workload("hostB", 1, 4, 128, MaskDesc(64, 1, 4, 1), torch.bfloat16, seed=32)
    h1 = [t.pin_memory() for t in make_inputs(w1, "cpu")]
    h2 = [t.pin_memory() for t in make_inputs(w2, "cpu")]
    a1 = caj.attn_fwd_jvp(*h1, w1.mask)
    a2 = caj.attn_fwd_jvp(*h2, w2.mask)
    b2 = caj.attn_fwd_jvp(*[t.cuda() for t in h2], w2.mask)
    torch.cuda.synchronize()
    for x, y in zip(a2, b2):
        assert torch.equal(x, y.cpu())
    assert not torch.equal(a1[0], a2[0])


def test_rejects_mismatched_inputs_without_launch():
    w = Workload("bad", 1, 2, 64, MaskDesc(16, 1, 4, 0), torch.bfloat16, seed=13)
    ins = list(make_inputs(w, "cuda"))
    with pytest.raises(caj.CajError):
        caj.attn_fwd_jvp(*ins, MaskDesc(16, 1, 5, 0))
    ins[2] = ins[2].float()
    with pytest.raises(ValueError):
        caj.attn_fwd_jvp(*ins, w.mask)
    caj.device_status()


# -------------------------------------- clean-tangent-zero teacher forcing (TF-sCM)
CTZ = [(MaskDesc(37, 1, 7, 1), 1, 2, 128), (MaskDesc(16, 3, 6, 1), 2, 1, 64),
       (MaskDesc(200, 2, 4, 1), 1, 1, 128), (MaskDesc(64, 1, 4, 1), 1, 2, 128),
       (MaskDesc(5, 1, 3, 1), 1, 3, 128)]


@pytest.mark.parametrize("case", range(len(CTZ)))
def test_clean_tangent_zero_matches_dense_definition(case):
    """With zero clean tangents the skipping kernel equals the oracle's dense
    definition (and the dense kernel, up to rounding)."""
    from masked_attention_jvp_b200.workloads import zero_clean_tangents
    mask, B, H, D = CTZ[case]
    w = Workload(f"ctz{case}", B, H, D, mask, torch.bfloat16, seed=300 + case, std_tangent=0.5)
    q, k, v, tq, tk, tv = make_inputs(w, "cuda")
    zero_clean_tangents(w, tq, tk, tv)
    outs = caj.attn_fwd_jvp(q, k, v, tq, tk, tv, w.mask, clean_tangent_zero=True)
    torch.cuda.synchronize()
    caj.device_status()
    ref = oracle.attn_fwd_jvp_rows(*[t.cpu() for t in (q, k, v, tq, tk, tv)], w.mask)
    rows = torch.arange(w.B * w.H * w.N)
    check_rows(gather(outs, rows, w.D), ref, w.dtype, w.name)
    L = mask.n_frames * mask.tokens_per_frame
    o, to, lse, tlse = outs
    assert torch.all(to[:, :, :L] == 0) and torch.all(tlse[:, :, :L] == 0)
    dense = caj.attn_fwd_jvp(q, k, v, tq, tk, tv, w.mask)
    assert torch.allclose(outs[0].float(), dense[0].float(), atol=1e-2, rtol=0)
    assert torch.allclose(outs[1].float(), dense[1].float(), atol=1e-2, rtol=0)


@pytest.mark.parametrize("name", ["wan1.3b_tf_framewise", "wan1.3b_tf_chunkwise"])
def test_clean_tangent_zero_full_size_sampled(name):
    from masked_attention_jvp_b200.workloads import zero_clean_tangents
    w = WORKLOADS[name]
    q, k, v, tq, tk, tv = make_inputs(w, "cuda")
    zero_clean_tangents(w, tq, tk, tv)
    outs = caj.attn_fwd_jvp(q, k, v, tq, tk, tv, w.mask, clean_tangent_zero=True)
    torch.cuda.synchronize()
    caj.device_status()
    rows = torch.unique(torch.cat([sample_rows(w, 256), boundary_rows(w)]))
    host = [t.cpu() for t in (q, k, v, tq, tk, tv)]
    del q, k, v, tq, tk, tv
    ref = oracle.attn_fwd_jvp_rows(*host, w.mask, rows=rows)
    check_rows(gather(outs, rows, w.D), ref, w.dtype, name)


def test_clean_tangent_zero_needs_teacher_forcing_layout():
    w = Workload("ctzbad", 1, 1, 64, MaskDesc(16, 1, 4, 0), torch.bfloat16, seed=1)
    ins = make_inputs(w, "cuda")
    with pytest.raises(caj.CajError):
        caj.attn_fwd_jvp(*ins, w.mask, clean_tangent_zero=True)


def test_clean_tangent_zero_repeated_calls_are_bitwise_identical():
    """Both clean-tangent-zero kernels are deterministic (in the primal kernel
    the two softmax warpgroups finish different tiles; their epilogues must
    still see every value product)."""
    from masked_attention_jvp_b200.workloads import zero_clean_tangents
    w = Workload("ctzdet", 1, 4, 128, MaskDesc(200, 2, 6, 1), torch.bfloat16, seed=21)
    ins = make_inputs(w, "cuda")
    zero_clean_tangents(w, *ins[3:])
    first = caj.attn_fwd_jvp(*ins, w.mask, clean_tangent_zero=True)
    for _ in range(3):
        again = caj.attn_fwd_jvp(*ins, w.mask, clean_tangent_zero=True)
        for x, y in zip(first, again):
            assert torch.equal(x, y)
    caj.device_status()


PART_CASES = [(MaskDesc(100, 1, 5, 0), 1, 2, 128, False, False), (MaskDesc(37, 1, 7, 1), 2, 2, 128, False, False),
              (MaskDesc(64, 3, 6, 1), 1, 3, 128, True, False), (MaskDesc(40, 1, 5, 1), 1, 2, 64, False, True),
              (MaskDesc(5, 1, 3, 1), 1, 2, 128, False, False)]


@pytest.mark.parametrize("case", range(len(PART_CASES)))
@pytest.mark.parametrize("nparts", [2, 3, 8])
def test_parts_together_equal_the_whole_call(case, nparts):
    """caj_attn_fwd_jvp_part: run part by part into buffers pre-filled with NaN,
    the parts write every row exactly as the whole call does (bit for bit),
    and a part alone leaves the other parts' rows untouched."""
    from masked_attention_jvp_b200.workloads import zero_clean_tangents
    mask, B, H, D, ctz, tm = PART_CASES[case]
    w = Workload(f"part{case}", B, H, D, mask, torch.bfloat16, seed=700 + case, std_tangent=0.5)
    ins = make_inputs(w, "cuda")
    if ctz:
        zero_clean_tangents(w, *ins[3:])
    whole = caj.attn_fwd_jvp(*ins, w.mask, clean_tangent_zero=ctz, token_major_out=tm)
    shape = whole[0].shape
    outs = [torch.full(shape, float("nan"), dtype=torch.bfloat16, device="cuda") for _ in range(2)] + \
        [torch.full(whole[2].shape, float("nan"), device="cuda") for _ in range(2)]
    for r in range(nparts):
        caj.attn_fwd_jvp_out(*ins, w.mask, *outs, clean_tangent_zero=ctz, token_major_out=tm, part=(r, nparts))
        if r == 0:  # part 0 alone wrote its tiles' rows and nothing else
            torch.cuda.synchronize()
            rows = torch.zeros(w.N, dtype=torch.bool)
            for t in caj.part_query_tiles(w.mask, 0, nparts):
                rows[128 * t:min(128 * t + 128, w.N)] = True
            lse0 = outs[2].cpu()
            assert torch.isfinite(lse0[:, :, rows]).all() and torch.isnan(lse0[:, :, ~rows]).all()
    torch.cuda.synchronize()
    caj.device_status()
    for got, want in zip(outs, whole):
        assert torch.equal(got, want)
