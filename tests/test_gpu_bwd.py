"""GPU parity of the primal attention backward (dQ, dK, dV, Delta) against the
fp64 oracle, through the C-ABI. The backward takes O and LSE from the fused
forward on the same inputs (as a training step would).

Bounds: relative Frobenius error <= 1e-2 on dV and Delta, <= 2e-2 on dQ and dK.
The pages state no tolerance for the backward. The forward's bf16 bound
(1e-2) is kept where the result is a sum of positive weights times bf16 values
(dV = P^T dO, Delta = <dO, O>). dQ and dK are sums of dS = P (dP - Delta), a
difference of two nearly equal terms whose bf16 rounding of dS (the tensor
cores' operand) does not shrink with it, so their relative error runs about
twice as high; measured: about 2.4e-3 on all four."""
import numpy as np
import pytest
import torch

import oracle
import masked_attention_jvp_b200 as caj
from masked_attention_jvp_b200.workloads import (MaskDesc, Workload, WORKLOADS, boundary_rows, make_inputs,
                                                 sample_rows)

pytestmark = pytest.mark.gpu


def rel_fro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


def run(w, seed_do=99):
    q, k, v, tq, tk, tv = make_inputs(w, "cuda")
    g = torch.Generator().manual_seed(seed_do)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16).cuda()
    o, _, lse, _ = caj.attn_fwd_jvp(q, k, v, tq, tk, tv, w.mask)
    dq, dk, dv, delta = caj.attn_bwd(q, k, v, o, dout, lse, w.mask)
    torch.cuda.synchronize()
    caj.device_status()
    return (q, k, v, o, dout), (dq, dk, dv, delta)


CASES = [(MaskDesc(100, 1, 5, 0), 1, 2, 128), (MaskDesc(37, 1, 7, 1), 1, 2, 128),
         (MaskDesc(16, 3, 6, 1), 2, 1, 64), (MaskDesc(1, 1, 300, 0), 1, 1, 128),
         (MaskDesc(600, 1, 1, 0), 1, 1, 64), (MaskDesc(5, 1, 3, 1), 1, 3, 128),
         (MaskDesc(200, 2, 4, 1), 1, 1, 128), (MaskDesc(64, 1, 4, 1), 1, 2, 64)]


@pytest.mark.parametrize("case", range(len(CASES)))
def test_bwd_matches_oracle(case):
    mask, B, H, D = CASES[case]
    w = Workload(f"bwd{case}", B, H, D, mask, torch.bfloat16, seed=500 + case)
    (q, k, v, o, dout), (dq, dk, dv, delta) = run(w)
    rq, rk, rv, rdelta = oracle.attn_bwd(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), mask)
    errs = dict(dq=rel_fro(dq.float().cpu().numpy(), rq), dk=rel_fro(dk.float().cpu().numpy(), rk),
                dv=rel_fro(dv.float().cpu().numpy(), rv), delta=rel_fro(delta.cpu().numpy(), rdelta))
    print(case, errs)
    assert errs["dv"] <= 1e-2, errs
    assert errs["dq"] <= 2e-2 and errs["dk"] <= 2e-2, errs
    assert errs["delta"] <= 1e-2, errs


def test_bwd_is_deterministic():
    w = Workload("bwddet", 1, 2, 128, MaskDesc(150, 1, 4, 1), torch.bfloat16, seed=7)
    a = run(w)[1]
    b = run(w)[1]
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("name", ["wan1.3b_tf_framewise"])
def test_bwd_full_size_invariants(name):
    """At full size: each row of dS sums to zero, so the keys' dK sum to zero
    (relative to the size of dK); each row of P sums to one, so the keys' dV sum
    to the queries' dO sum."""
    w = WORKLOADS[name]
    (q, k, v, o, dout), (dq, dk, dv, delta) = run(w)
    dk_sum = dk.float().sum(dim=2)
    assert float(dk_sum.norm() / dk.float().norm()) <= 2e-2
    dv_sum, do_sum = dv.float().sum(dim=2), dout.float().sum(dim=2)
    assert float((dv_sum - do_sum).norm() / do_sum.norm()) <= 2e-2
    assert torch.isfinite(dq.float()).all() and torch.isfinite(dk.float()).all()


@pytest.mark.parametrize("name", ["wan1.3b_tf_framewise"])
def test_bwd_full_size_dq_rows_match_oracle(name):
    """At full size, dQ and Delta of 512 seeded rows per head plus the first and
    last row of every chunk, against the oracle's row-wise backward."""
    w = WORKLOADS[name]
    (q, k, v, o, dout), (dq, dk, dv, delta) = run(w)
    del dk, dv
    rows = torch.unique(torch.cat([sample_rows(w, 512, seed_offset=5), boundary_rows(w)]))
    idx = rows.to(dq.device)
    got_dq = dq.reshape(-1, w.D)[idx].float().cpu().numpy()
    got_delta = delta.reshape(-1)[idx].cpu().numpy()
    host = [t.cpu() for t in (q, k, v, dout)]
    del q, k, v, o, dout, dq, delta
    rdq, rdelta = oracle.attn_bwd_dq_rows(*host, w.mask, rows=rows)
    errs = dict(dq=rel_fro(got_dq, rdq), delta=rel_fro(got_delta, rdelta))
    print(name, rows.numel(), errs)
    assert np.all(np.isfinite(got_dq))
    assert errs["dq"] <= 2e-2, errs
    assert errs["delta"] <= 1e-2, errs


def test_bwd_mid_size_teacher_forcing_matches_oracle():
    """dK and dV over every key of a mid-size teacher-forcing case (N = 9360,
    73 query tiles and a ragged tail, 4 heads), against the full oracle: the
    key-major kernel's transposed schedule is checked on every key tile."""
    w = Workload("bwd_mid", 1, 4, 128, MaskDesc(312, 1, 15, 1), torch.bfloat16, seed=520, std_tangent=0.5)
    (q, k, v, o, dout), (dq, dk, dv, delta) = run(w)
    rq, rk, rv, rdelta = oracle.attn_bwd(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), w.mask)
    errs = dict(dq=rel_fro(dq.float().cpu().numpy(), rq), dk=rel_fro(dk.float().cpu().numpy(), rk),
                dv=rel_fro(dv.float().cpu().numpy(), rv), delta=rel_fro(delta.cpu().numpy(), rdelta))
    print(errs)
    assert errs["dv"] <= 1e-2 and errs["delta"] <= 1e-2, errs
    assert errs["dq"] <= 2e-2 and errs["dk"] <= 2e-2, errs
    # per key tile as well: a missed or doubled tile would hide in the global norm
    for name, got, ref in (("dk", dk, rk), ("dv", dv, rv)):
        g = got.float().cpu().numpy()
        for t0 in range(0, w.N, 128):
            a, b = g[:, :, t0:t0 + 128], ref[:, :, t0:t0 + 128]
            assert rel_fro(a, b) <= 5e-2, (name, t0, rel_fro(a, b))
