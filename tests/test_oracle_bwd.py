"""Pins for the fp64 oracle of the primal attention backward (dQ, dK, dV).
CPU only."""
import math

import numpy as np
import pytest
import torch

import oracle
from masked_attention_jvp_b200.workloads import MaskDesc

F64 = torch.float64
MASKS = [MaskDesc(3, 1, 4, 0), MaskDesc(2, 2, 4, 0), MaskDesc(3, 1, 3, 1), MaskDesc(2, 3, 6, 1),
         MaskDesc(1, 1, 7, 0), MaskDesc(5, 1, 1, 0)]


def rand(B, H, N, D, seed, n=4):
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(B, H, N, D, generator=g, dtype=F64) for _ in range(n)]


def loss(q, k, v, dout, mask, scale=None):
    """<dO, O(q, k, v)> with O from the forward oracle."""
    z = torch.zeros_like(q)
    o, _, _, _ = oracle.attn_fwd_jvp(q, k, v, z, z, z, mask, scale=scale)
    return float(np.sum(o * dout.numpy()))


@pytest.mark.parametrize("mask", MASKS)
def test_gradient_matches_central_differences(mask):
    """d/dh <dO, O(x + h u)> at h = 0 equals <dQ, uq> + <dK, uk> + <dV, uv>."""
    q, k, v, dout = rand(1, 2, mask.seq_len, 6, seed=1)
    uq, uk, uv = rand(1, 2, mask.seq_len, 6, seed=2, n=3)
    dq, dk, dv, _ = oracle.attn_bwd(q, k, v, dout, mask)
    h = 1e-6
    fd = (loss(q + h * uq, k + h * uk, v + h * uv, dout, mask) -
          loss(q - h * uq, k - h * uk, v - h * uv, dout, mask)) / (2 * h)
    an = float(np.sum(dq * uq.numpy()) + np.sum(dk * uk.numpy()) + np.sum(dv * uv.numpy()))
    assert abs(fd - an) <= 1e-7 * max(1.0, abs(an))


@pytest.mark.parametrize("mask", MASKS)
def test_adjoint_of_the_jvp(mask):
    """Backward and JVP are adjoint: <dO, tO> = <dQ, tQ> + <dK, tK> + <dV, tV>,
    with tO from the independent JVP oracle."""
    q, k, v, dout = rand(2, 2, mask.seq_len, 8, seed=3)
    tq, tk, tv = rand(2, 2, mask.seq_len, 8, seed=4, n=3)
    _, to, _, _ = oracle.attn_fwd_jvp(q, k, v, tq, tk, tv, mask)
    dq, dk, dv, _ = oracle.attn_bwd(q, k, v, dout, mask)
    lhs = float(np.sum(dout.numpy() * to))
    rhs = float(np.sum(dq * tq.numpy()) + np.sum(dk * tk.numpy()) + np.sum(dv * tv.numpy()))
    assert abs(lhs - rhs) <= 1e-11 * max(1.0, abs(lhs))


@pytest.mark.parametrize("mask", MASKS)
def test_column_sum_invariants(mask):
    """Each row of dS sums to zero, so sum_j dK_j = 0; each row of P sums to one,
    so sum_j dV_j = sum_i dO_i. Delta_i = <dO_i, O_i>."""
    q, k, v, dout = rand(1, 3, mask.seq_len, 5, seed=5)
    dq, dk, dv, delta = oracle.attn_bwd(q, k, v, dout, mask)
    assert np.max(np.abs(dk.sum(axis=2))) <= 1e-12
    assert np.max(np.abs(dv.sum(axis=2) - dout.numpy().sum(axis=2))) <= 1e-12
    z = torch.zeros_like(q)
    o, _, _, _ = oracle.attn_fwd_jvp(q, k, v, z, z, z, mask)
    assert np.max(np.abs(delta - np.sum(o * dout.numpy(), axis=-1))) <= 1e-12


@pytest.mark.parametrize("mask", MASKS)
def test_matches_torch_autograd(mask):
    from tests.test_oracle import dense_mask_from_chunks
    q, k, v, dout = rand(1, 2, mask.seq_len, 8, seed=6)
    m = dense_mask_from_chunks(mask)
    qq, kk, vv = (x.clone().requires_grad_(True) for x in (q, k, v))
    s = (qq @ kk.transpose(-1, -2)) / math.sqrt(8)
    o = torch.softmax(s.masked_fill(~m, float("-inf")), dim=-1) @ vv
    (o * dout).sum().backward()
    dq, dk, dv, _ = oracle.attn_bwd(q, k, v, dout, mask)
    assert np.max(np.abs(dq - qq.grad.numpy())) <= 1e-12
    assert np.max(np.abs(dk - kk.grad.numpy())) <= 1e-12
    assert np.max(np.abs(dv - vv.grad.numpy())) <= 1e-12


def test_single_key_row_has_no_query_gradient():
    """Token-causal row 0 sees only key 0: P = 1, dS = 0, so dQ_0 = 0."""
    mask = MaskDesc(1, 1, 4, 0)
    q, k, v, dout = rand(1, 1, mask.seq_len, 4, seed=7)
    dq, _, _, _ = oracle.attn_bwd(q, k, v, dout, mask)
    assert np.all(dq[0, 0, 0] == 0.0)


@pytest.mark.parametrize("mask", MASKS)
def test_dq_rows_match_central_differences_of_the_forward(mask):
    """dQ of one row from the row-wise oracle equals the central difference of
    <dO, O> when only that row of q moves (the forward oracle, h = 1e-6)."""
    q, k, v, dout = rand(1, 2, mask.seq_len, 6, seed=8)
    (u,) = rand(1, 2, mask.seq_len, 6, seed=9, n=1)
    N = mask.seq_len
    for bh, i in ((0, 0), (1, N - 1), (0, N // 2)):
        e = torch.zeros_like(u)
        e[0, bh, i] = u[0, bh, i]
        dq, _ = oracle.attn_bwd_dq_rows(q, k, v, dout, mask, rows=[bh * N + i])
        h = 1e-6
        fd = (loss(q + h * e, k, v, dout, mask) - loss(q - h * e, k, v, dout, mask)) / (2 * h)
        an = float(np.sum(dq[0] * u[0, bh, i].numpy()))
        assert abs(fd - an) <= 1e-7 * max(1.0, abs(an)), (bh, i, fd, an)


@pytest.mark.parametrize("mask", MASKS)
def test_dq_rows_delta_is_the_output_inner_product(mask):
    """Delta_i = <dO_i, O_i>, with O from the forward oracle; every row's dQ
    also equals that row of the full backward."""
    q, k, v, dout = rand(2, 2, mask.seq_len, 5, seed=10)
    N = mask.seq_len
    rows = torch.arange(4 * N)
    dq, delta = oracle.attn_bwd_dq_rows(q, k, v, dout, mask, rows=rows)
    z = torch.zeros_like(q)
    o, _, _, _ = oracle.attn_fwd_jvp(q, k, v, z, z, z, mask)
    assert np.max(np.abs(delta - np.sum(o * dout.numpy(), axis=-1).reshape(-1))) <= 1e-12
    fdq, _, _, _ = oracle.attn_bwd(q, k, v, dout, mask)
    assert np.max(np.abs(dq - fdq.reshape(-1, 5))) <= 1e-12


def test_dq_rows_single_key_row_is_zero():
    mask = MaskDesc(1, 1, 4, 0)
    q, k, v, dout = rand(1, 1, mask.seq_len, 4, seed=11)
    dq, delta = oracle.attn_bwd_dq_rows(q, k, v, dout, mask, rows=[0])
    assert np.all(dq == 0.0)
    assert abs(delta[0] - float(dout[0, 0, 0] @ v[0, 0, 0])) <= 1e-12
