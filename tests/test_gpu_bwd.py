"""GPU parity of the primal attention backward (dQ, dK, dV, Delta) against the
fp64 oracle, through the C-ABI. The backward takes O and LSE from the fused
forward on the same inputs (as a training step would)."""
import numpy as np
import pytest
import torch

import oracle
import masked_attention_jvp_b200 as caj
from masked_attention_jvp_b200.workloads import MaskDesc, Workload, WORKLOADS, make_inputs

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
