"""The forward + JVP with its output all-to-all in the epilogue
(caj_attn_fwd_jvp_scatter), on one GPU: P ranks of Ulysses context parallelism
(Causal-rCM section 3.2.1 "Parallelism", section 3.2.2 "JVP Ulysses CP") are
emulated as P launches, launch r computing heads [r H/P, (r+1) H/P) over the
whole sequence and storing every row into the slice buffer of the token's
owner. The P slice buffers are local here; on a multi-GPU run they are the
ranks' memory and the same stores cross NVLink. The launches only store, they
never wait on one another. After all P launches slice r must equal rows
[r N/P, (r+1) N/P) of the direct call, bit for bit, for every head. The slices,
put back together, must also match the fp64 oracle within the parity tests'
tolerances (every row for the small cases; 512 seeded rows per head plus the
chunk boundaries at full size), so a layout error shared by the direct and the
scattering kernels cannot pass."""
import ctypes

import pytest
import torch

import oracle

import masked_attention_jvp_b200 as caj
from masked_attention_jvp_b200.workloads import (MaskDesc, boundary_rows, make_inputs, sample_rows, small,
                                                 zero_clean_tangents)
from tests.test_gpu_parity import check_rows, gather

pytestmark = pytest.mark.gpu

bf, f32 = torch.bfloat16, torch.float32

# name, B, H, D, mask, dtype, P, clean_tangent_zero, token_major
CASES = [
    ("tf_p2", 1, 4, 128, MaskDesc(100, 1, 4, 1), bf, 2, False, False),          # N 800, slices of 400
    ("infer_d64_p4_ragged", 2, 4, 64, MaskDesc(75, 1, 8, 0), bf, 4, False, False),  # slices of 150: tiles straddle
    ("tf_ctz_p4", 1, 8, 128, MaskDesc(100, 1, 4, 1), bf, 4, True, False),       # both CTZ launches scatter
    ("tf_chunk_tokmajor_p2", 1, 4, 128, MaskDesc(60, 3, 6, 1), bf, 2, False, True),
    ("tf_ctz_tokmajor_p8", 1, 8, 64, MaskDesc(40, 1, 8, 1), bf, 8, True, True),  # 8 slices of 80 rows
    ("fp32_p2", 1, 2, 64, MaskDesc(16, 1, 4, 0), f32, 2, False, False),          # CUDA-core path
    ("tf_p1", 1, 2, 128, MaskDesc(50, 1, 3, 1), bf, 1, False, False),            # one slice: plain output
]


def _slices(B, H, Ls, D, dtype, P, token_major):
    shp = (B, Ls, H, D) if token_major else (B, H, Ls, D)
    full = lambda s, dt: [torch.full(s, float("nan"), dtype=dt, device="cuda") for _ in range(P)]
    return full(shp, dtype), full(shp, dtype), full((B, H, Ls), f32), full((B, H, Ls), f32)


def _rows(t, rows, token_major):
    return t[:, rows] if token_major else t[:, :, rows]


def _assemble(o, to, lse, tlse, token_major):
    """The P slices put back together as [B, H, N, D] and [B, H, N]."""
    if token_major:
        fo = torch.cat(o, dim=1).permute(0, 2, 1, 3).contiguous()
        fto = torch.cat(to, dim=1).permute(0, 2, 1, 3).contiguous()
    else:
        fo, fto = torch.cat(o, dim=2), torch.cat(to, dim=2)
    return fo, fto, torch.cat(lse, dim=2), torch.cat(tlse, dim=2)


@pytest.mark.parametrize("case", CASES, ids=[c[0] for c in CASES])
def test_scatter_equals_direct_call(case):
    name, B, H, D, mask, dtype, P, ctz, tm = case
    w = small(name, B, H, D, mask, dtype, seed=31)
    ins = make_inputs(w, "cuda")
    if ctz:
        zero_clean_tangents(w, *ins[3:])
    direct = caj.attn_fwd_jvp(*ins, w.mask, clean_tangent_zero=ctz, token_major_out=tm)
    N, Hp = w.N, H // P
    Ls = N // P
    o, to, lse, tlse = _slices(B, H, Ls, D, dtype, P, tm)
    for r in range(P):  # emulated rank r: its heads, every slice
        mine = [x[:, r * Hp:(r + 1) * Hp].contiguous() for x in ins]
        caj.attn_fwd_jvp_scatter(*mine, w.mask, o, to, lse, tlse, head_base=r * Hp,
                                 clean_tangent_zero=ctz, token_major_out=tm)
    torch.cuda.synchronize()
    for r in range(P):
        rows = slice(r * Ls, (r + 1) * Ls)
        assert torch.equal(o[r], _rows(direct[0], rows, tm)), (name, r, "o")
        assert torch.equal(to[r], _rows(direct[1], rows, tm)), (name, r, "to")
        assert torch.equal(lse[r], direct[2][:, :, rows]), (name, r, "lse")
        assert torch.equal(tlse[r], direct[3][:, :, rows]), (name, r, "tlse")
    # every row of the reassembled slices against the oracle
    ref = oracle.attn_fwd_jvp_rows(*[t.cpu() for t in ins], w.mask)
    full = _assemble(o, to, lse, tlse, tm)
    check_rows(gather(full, torch.arange(B * H * N), D), ref, dtype, name)


def test_scatter_writes_only_its_own_heads():
    B, H, D, P = 1, 4, 128, 2
    w = small("own_heads", B, H, D, MaskDesc(100, 1, 4, 1), bf, seed=32)
    ins = make_inputs(w, "cuda")
    direct = caj.attn_fwd_jvp(*ins, w.mask)
    Ls, Hp = w.N // P, H // P
    o, to, lse, tlse = _slices(B, H, Ls, D, bf, P, False)
    mine = [x[:, Hp:].contiguous() for x in ins]  # rank 1 alone
    caj.attn_fwd_jvp_scatter(*mine, w.mask, o, to, lse, tlse, head_base=Hp)
    torch.cuda.synchronize()
    for r in range(P):
        rows = slice(r * Ls, (r + 1) * Ls)
        for got, want in ((o[r], direct[0]), (to[r], direct[1]), (lse[r], direct[2]), (tlse[r], direct[3])):
            assert torch.equal(got[:, Hp:], want[:, Hp:, rows])
            assert torch.isnan(got[:, :Hp].float()).all()  # rank 0's heads untouched


def test_scatter_rejects_bad_slices():
    w = small("bad", 1, 2, 64, MaskDesc(16, 1, 4, 0), bf, seed=33)
    ins = make_inputs(w, "cuda")
    o, to, lse, tlse = _slices(1, 2, 21, 64, bf, 3, False)
    with pytest.raises(ValueError):  # 64 rows do not split in 3
        caj.attn_fwd_jvp_scatter(*ins, w.mask, o, to, lse, tlse)
    o, to, lse, tlse = _slices(1, 2, 32, 64, bf, 2, False)
    with pytest.raises(caj.CajError):  # heads 1, 2 of a 2-head slice
        caj.attn_fwd_jvp_scatter(*ins, w.mask, o, to, lse, tlse, head_base=1)


def test_scatter_at_full_size_equals_direct_call():
    """The bench's scatter configuration at full size: the TF frame-wise
    workload (B=1, H=12, N=65520, D=128) split over 4 emulated ranks of 3 heads,
    slices of 16380 rows (query tiles straddle every slice boundary)."""
    from masked_attention_jvp_b200.workloads import WORKLOADS
    w = WORKLOADS["wan1.3b_tf_framewise"]
    P = 4
    ins = make_inputs(w, "cuda")
    direct = caj.attn_fwd_jvp(*ins, w.mask)
    Hp, Ls = w.H // P, w.N // P
    o, to, lse, tlse = _slices(w.B, w.H, Ls, w.D, w.dtype, P, False)
    for r in range(P):
        mine = [x[:, r * Hp:(r + 1) * Hp].contiguous() for x in ins]
        caj.attn_fwd_jvp_scatter(*mine, w.mask, o, to, lse, tlse, head_base=r * Hp)
        del mine
    torch.cuda.synchronize()
    caj.device_status()
    for r in range(P):
        rows = slice(r * Ls, (r + 1) * Ls)
        assert torch.equal(o[r], direct[0][:, :, rows])
        assert torch.equal(to[r], direct[1][:, :, rows])
        assert torch.equal(lse[r], direct[2][:, :, rows])
        assert torch.equal(tlse[r], direct[3][:, :, rows])
    del direct
    full = _assemble(o, to, lse, tlse, False)
    del o, to, lse, tlse
    rows = torch.unique(torch.cat([sample_rows(w, 512, seed_offset=9), boundary_rows(w)]))
    got = gather(full, rows, w.D)
    host = [t.cpu() for t in ins]
    del ins, full
    ref = oracle.attn_fwd_jvp_rows(*host, w.mask, rows=rows)
    check_rows(got, ref, w.dtype, "scatter full size")


def test_scatter_refuses_host_memory_slices():
    """Slices in host memory are refused before any launch: by the Python
    binding (CPU tensors), and by the library itself for pinned host memory
    given through the C-ABI (device-reachable, so nothing could fault even if
    the check were missing; the status is what is checked)."""
    w = small("host_slices", 1, 2, 64, MaskDesc(16, 1, 4, 0), bf, seed=34)
    ins = make_inputs(w, "cuda")
    o, to, lse, tlse = _slices(1, 2, 32, 64, bf, 2, False)
    cpu_o = [t.cpu() for t in o]
    with pytest.raises(ValueError):
        caj.attn_fwd_jvp_scatter(*ins, w.mask, cpu_o, to, lse, tlse)
    pinned = torch.zeros(1, 2, 32, 64, dtype=bf).pin_memory()
    dst = caj._lib.SeqScatterC()
    dst.shards, dst.head_base, dst.heads_total = 2, 0, 2
    for r in range(2):
        dst.o[r], dst.to[r] = o[r].data_ptr(), to[r].data_ptr()
        dst.lse[r], dst.tlse[r] = lse[r].data_ptr(), tlse[r].data_ptr()
    dst.to[1] = pinned.data_ptr()
    prob = caj._problem(ins[0], None)
    st = caj._lib.lib().caj_attn_fwd_jvp_scatter(*[ctypes.c_void_p(t.data_ptr()) for t in ins],
                                                 ctypes.byref(prob), ctypes.byref(caj._lib.mask_c(w.mask)),
                                                 ctypes.byref(dst), None)
    torch.cuda.synchronize()
    assert st == caj._lib.CAJ_ERR_INVALID_ARG
    assert torch.count_nonzero(pinned.float()) == 0
    assert all(torch.isnan(t.float()).all() for t in o)  # nothing launched
