"""GPU parity of the attention-block prologue (RMSNorm + JVP, rotary embedding,
re-layout) against the fp64 oracle, through the C-ABI.

Tolerance: outputs are bf16 rounded from fp32 arithmetic, so each element may be
off by half a bf16 ulp (2^-9 relative) plus fp32 rounding: elementwise
|err| <= 2^-8 |ref| + 1e-3 * rms(ref), relative Frobenius <= 4e-3; v and tv
must equal the permuted inputs bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import masked_attention_jvp_b200 as caj

pytestmark = pytest.mark.gpu


def make(B, N, H, D, seed):
    g = torch.Generator().manual_seed(seed)
    xs = [torch.randn(B, N, H * D, generator=g).to(torch.bfloat16) for _ in range(6)]
    gq = (1 + 0.1 * torch.randn(H * D, generator=g)).float()
    gk = (1 + 0.1 * torch.randn(H * D, generator=g)).float()
    theta = torch.rand(N, D // 2, generator=g) * 100.0
    return xs, gq, gk, torch.cos(theta).float(), torch.sin(theta).float()


@pytest.mark.parametrize("B,N,H,D,per_head", [(1, 37, 2, 128, False), (2, 19, 4, 64, False),
                                              (1, 33, 12, 128, False), (1, 33, 12, 128, True),
                                              (2, 17, 8, 64, True)])
def test_prologue_matches_oracle(B, N, H, D, per_head):
    xs, gq, gk, c, s = make(B, N, H, D, seed=B * 100 + N)
    dev = [t.cuda() for t in xs]
    outs = caj.qk_norm_rope_jvp(*dev, gq.cuda(), gk.cuda(), c.cuda(), s.cuda(), H, eps=1e-6,
                                per_head=per_head)
    torch.cuda.synchronize()
    ref = oracle.qk_norm_rope_jvp(*xs, gq.double(), gk.double(), c.double(), s.double(), H,
                                  eps=1e-6, per_head=per_head)
    for i, (o, r) in enumerate(zip(outs, ref)):
        got = o.float().cpu().numpy().astype(np.float64)
        if i in (2, 5):  # v, tv: pure re-layout
            assert np.array_equal(got, r)
            continue
        err = np.abs(got - r)
        rms = float(np.sqrt(np.mean(r * r)))
        assert np.all(err <= 2.0 ** -8 * np.abs(r) + 1e-3 * rms), (i, float(err.max()))
        assert float(np.linalg.norm(got - r) / np.linalg.norm(r)) <= 4e-3


def test_prologue_feeds_attention():
    """End to end: prologue then fused attention, against the oracle applied to
    the oracle's own prologue outputs (rounded to bf16 like the GPU's)."""
    from masked_attention_jvp_b200.workloads import MaskDesc
    B, H, D = 1, 2, 128
    mask = MaskDesc(40, 1, 3, 1)
    N = mask.seq_len
    xs, gq, gk, c, s = make(B, N, H, D, seed=5)
    outs = caj.qk_norm_rope_jvp(*[t.cuda() for t in xs], gq.cuda(), gk.cuda(), c.cuda(), s.cuda(), H)
    o, to, lse, tlse = caj.attn_fwd_jvp(*outs, mask)
    torch.cuda.synchronize()
    ref_in = [torch.from_numpy(r).to(torch.bfloat16) for r in
              oracle.qk_norm_rope_jvp(*xs, gq.double(), gk.double(), c.double(), s.double(), H)]
    ro, rto, rlse, rtlse = oracle.attn_fwd_jvp(*ref_in, mask)
    rel = lambda a, b: float(np.linalg.norm(a - b) / np.linalg.norm(b))
    assert rel(o.float().cpu().numpy(), ro) <= 1e-2
    assert rel(to.float().cpu().numpy(), rto) <= 1e-2
