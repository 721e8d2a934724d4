"""GPU checks of the attention block's output side in primal-tangent form:
the token-major output layout of the attention kernels, and the output
projection y = x W^T + b, ty = tx W^T against the fp64 oracle.

Tolerances (bf16 inputs, fp32 accumulation, bf16 outputs): relative Frobenius
error <= 1e-2 and max-abs error <= 1e-2 of the largest reference magnitude."""
import numpy as np
import pytest
import torch

import oracle
import masked_attention_jvp_b200 as caj
from masked_attention_jvp_b200.workloads import MaskDesc, Workload, make_inputs, zero_clean_tangents

pytestmark = pytest.mark.gpu


def rel_fro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))


# (mask, B, H, D, dtype, clean_tangent_zero): the dense JVP kernel, both
# clean-tangent-zero kernels, and the fp32 path
TM = [(MaskDesc(37, 1, 7, 1), 2, 3, 128, torch.bfloat16, False),
      (MaskDesc(37, 1, 7, 1), 2, 3, 128, torch.bfloat16, True),
      (MaskDesc(16, 3, 6, 0), 1, 2, 64, torch.bfloat16, False),
      (MaskDesc(17, 1, 3, 0), 2, 2, 64, torch.float32, False)]


@pytest.mark.parametrize("case", range(len(TM)))
def test_token_major_output_is_the_head_major_output_permuted(case):
    mask, B, H, D, dtype, ctz = TM[case]
    w = Workload(f"tm{case}", B, H, D, mask, dtype, seed=40 + case)
    ins = make_inputs(w, "cuda")
    if ctz:
        zero_clean_tangents(w, *ins[3:])
    a = caj.attn_fwd_jvp(*ins, mask, clean_tangent_zero=ctz)
    t = caj.attn_fwd_jvp(*ins, mask, clean_tangent_zero=ctz, token_major_out=True)
    torch.cuda.synchronize()
    caj.device_status()
    assert t[0].shape == (B, w.N, H, D)
    assert torch.equal(t[0], a[0].permute(0, 2, 1, 3))
    assert torch.equal(t[1], a[1].permute(0, 2, 1, 3))
    assert torch.equal(t[2], a[2]) and torch.equal(t[3], a[3])


@pytest.mark.parametrize("M,K,C,with_bias", [(37, 64, 72, True), (1000, 1536, 1536, True),
                                             (4096, 1536, 1536, False), (1, 128, 8, True),
                                             (300, 200, 520, True),     # ragged K block, partial column box
                                             (2000, 40, 1032, False),   # K below one stage, 5 column blocks
                                             (129, 5120, 64, True)])    # long K, one column box
def test_out_proj_matches_oracle(M, K, C, with_bias):
    g = torch.Generator(device="cuda").manual_seed(M + K + C)
    x, tx = (torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16) for _ in range(2))
    wt = (torch.randn(C, K, device="cuda", generator=g) / K ** 0.5).to(torch.bfloat16)
    b = torch.randn(C, device="cuda", generator=g).to(torch.bfloat16) if with_bias else None
    y, ty = caj.out_proj_jvp(x, tx, wt, b)
    torch.cuda.synchronize()
    ry, rty = oracle.out_proj_jvp(x, tx, wt, b)
    for got, ref in ((y, ry), (ty, rty)):
        got = got.float().cpu().numpy()
        assert rel_fro(got, ref) <= 1e-2
        assert float(np.max(np.abs(got - ref))) <= 1e-2 * float(np.max(np.abs(ref)))


def test_out_proj_full_size_rows_match_oracle():
    """The bench's shape: the TF frame-wise workload's tokens (M = 65520, which
    is not a multiple of the 128-row tile), K = C = 1536. Rows sampled across
    the whole range, the last row block of x and of tx included."""
    M, K, C = 65520, 1536, 1536
    g = torch.Generator(device="cuda").manual_seed(9)
    x, tx = (torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16) for _ in range(2))
    wt = (torch.randn(C, K, device="cuda", generator=g) / K ** 0.5).to(torch.bfloat16)
    b = torch.randn(C, device="cuda", generator=g).to(torch.bfloat16)
    y, ty = caj.out_proj_jvp(x, tx, wt, b)
    torch.cuda.synchronize()
    caj.device_status()
    gen = torch.Generator().manual_seed(10)
    rows = torch.unique(torch.cat([torch.randint(0, M, (2048,), generator=gen), torch.arange(M - 200, M),
                                   torch.arange(0, 130)]))
    idx = rows.cuda()
    ry, rty = oracle.out_proj_jvp(x[idx], tx[idx], wt, b)
    for got, ref in ((y[idx], ry), (ty[idx], rty)):
        got = got.float().cpu().numpy()
        assert rel_fro(got, ref) <= 1e-2
        assert float(np.max(np.abs(got - ref))) <= 1e-2 * float(np.max(np.abs(ref)))


def test_out_proj_writes_nothing_past_its_rows_and_columns():
    """Output rows and columns outside [M, C] stay untouched (the tile store
    clips them): a larger buffer around y keeps its sentinel values."""
    M, K, C = 150, 64, 72
    g = torch.Generator(device="cuda").manual_seed(11)
    x, tx = (torch.randn(M, K, device="cuda", generator=g).to(torch.bfloat16) for _ in range(2))
    wt = (torch.randn(C, K, device="cuda", generator=g) / K ** 0.5).to(torch.bfloat16)
    big = torch.full((M + 64, C), 7.0, dtype=torch.bfloat16, device="cuda")
    bigt = torch.full((M + 64, C), 7.0, dtype=torch.bfloat16, device="cuda")
    caj.out_proj_jvp(x, tx, wt, None, out=(big[:M], bigt[:M]))
    torch.cuda.synchronize()
    assert torch.all(big[M:] == 7.0) and torch.all(bigt[M:] == 7.0)
    ry, rty = oracle.out_proj_jvp(x, tx, wt, None)
    assert rel_fro(big[:M].float().cpu().numpy(), ry) <= 1e-2


def test_attention_then_projection_chain():
    """attn_fwd_jvp (token-major) -> out_proj_jvp, against the oracles chained."""
    mask, B, H, D = MaskDesc(40, 1, 5, 1), 1, 4, 64
    w = Workload("chain", B, H, D, mask, torch.bfloat16, seed=77)
    ins = make_inputs(w, "cuda")
    o, to, _, _ = caj.attn_fwd_jvp(*ins, mask, token_major_out=True)
    C = 256
    g = torch.Generator(device="cuda").manual_seed(5)
    wt = (torch.randn(C, H * D, device="cuda", generator=g) / (H * D) ** 0.5).to(torch.bfloat16)
    b = torch.randn(C, device="cuda", generator=g).to(torch.bfloat16)
    y, ty = caj.out_proj_jvp(o, to, wt, b)
    torch.cuda.synchronize()
    assert y.shape == (B, w.N, C)
    ro, rto, _, _ = oracle.attn_fwd_jvp(*[t.cpu() for t in ins], mask)
    # the oracle's attention output in the projection's layout [B*N, H*D]
    xo = np.transpose(ro, (0, 2, 1, 3)).reshape(-1, H * D)
    xto = np.transpose(rto, (0, 2, 1, 3)).reshape(-1, H * D)
    ry, rty = oracle.out_proj_jvp(xo, xto, wt, b)
    for got, ref in ((y, ry), (ty, rty)):
        got = got.float().cpu().numpy().reshape(ref.shape)
        assert rel_fro(got, ref) <= 1e-2
