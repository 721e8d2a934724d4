"""Pins for the fp64 oracle of the layer prologue in primal-tangent form
(RMSNorm with its JVP and the rotary embedding of q and k; re-layout of v).
CPU only."""
import math

import numpy as np
import pytest
import torch

import oracle

F64 = torch.float64


def make(B, N, H, D, seed, dtype=F64):
    g = torch.Generator().manual_seed(seed)
    xs = [torch.randn(B, N, H * D, generator=g, dtype=F64) for _ in range(6)]
    gq = 1 + 0.1 * torch.randn(H * D, generator=g, dtype=F64)
    gk = 1 + 0.1 * torch.randn(H * D, generator=g, dtype=F64)
    theta = torch.rand(N, D // 2, generator=g, dtype=F64) * 6.0
    return [x.to(dtype) for x in xs], gq, gk, torch.cos(theta), torch.sin(theta)


def rel(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


@pytest.mark.parametrize("per_head", [False, True])
def test_tangent_matches_central_differences(per_head):
    B, N, H, D = 2, 5, 3, 8
    xs, gq, gk, c, s = make(B, N, H, D, 1)
    x, t = xs[:3], xs[3:]
    out = oracle.qk_norm_rope_jvp(*x, *t, gq, gk, c, s, H, eps=1e-5, per_head=per_head)
    h = 1e-6
    z = [torch.zeros_like(a) for a in x]
    plus = oracle.qk_norm_rope_jvp(*[a + h * b for a, b in zip(x, t)], *z, gq, gk, c, s, H, 1e-5, per_head)
    minus = oracle.qk_norm_rope_jvp(*[a - h * b for a, b in zip(x, t)], *z, gq, gk, c, s, H, 1e-5, per_head)
    for i in range(3):
        fd = (plus[i] - minus[i]) / (2 * h)
        assert rel(out[3 + i], fd) <= 1e-7


def test_rms_of_normalised_output_closed_form():
    """g = 1 and no rotation: mean over the token of y^2 = ms / (ms + eps)."""
    B, N, H, D = 1, 4, 2, 8
    xs, _, _, _, _ = make(B, N, H, D, 2)
    ones = torch.ones(H * D, dtype=F64)
    c, s = torch.ones(N, D // 2, dtype=F64), torch.zeros(N, D // 2, dtype=F64)
    eps = 0.3
    q = oracle.qk_norm_rope_jvp(*xs, ones, ones, c, s, H, eps=eps)[0]
    y = q.transpose(0, 2, 1, 3).reshape(B, N, H * D)
    ms = (xs[0] ** 2).mean(-1).numpy()
    assert np.allclose((y ** 2).mean(-1), ms / (ms + eps), rtol=0, atol=1e-14)


def test_quarter_turn_rotation():
    """theta = pi/2 maps each pair (a, b) to (-b, a)."""
    B, N, H, D = 1, 3, 2, 4
    xs, gq, gk, _, _ = make(B, N, H, D, 3)
    c0, s0 = torch.ones(N, D // 2, dtype=F64), torch.zeros(N, D // 2, dtype=F64)
    c1, s1 = torch.zeros(N, D // 2, dtype=F64), torch.ones(N, D // 2, dtype=F64)
    a = oracle.qk_norm_rope_jvp(*xs, gq, gk, c0, s0, H)
    b = oracle.qk_norm_rope_jvp(*xs, gq, gk, c1, s1, H)
    for i in (0, 1, 3, 4):  # q, k, tq, tk
        assert np.allclose(b[i][..., 0::2], -a[i][..., 1::2], atol=1e-15)
        assert np.allclose(b[i][..., 1::2], a[i][..., 0::2], atol=1e-15)


def test_rotation_preserves_pair_norms():
    B, N, H, D = 2, 4, 2, 8
    xs, gq, gk, c, s = make(B, N, H, D, 4)
    c0, s0 = torch.ones_like(c), torch.zeros_like(s)
    a = oracle.qk_norm_rope_jvp(*xs, gq, gk, c0, s0, H)
    b = oracle.qk_norm_rope_jvp(*xs, gq, gk, c, s, H)
    for i in (0, 1, 3, 4):
        na = a[i][..., 0::2] ** 2 + a[i][..., 1::2] ** 2
        nb = b[i][..., 0::2] ** 2 + b[i][..., 1::2] ** 2
        assert np.allclose(na, nb, rtol=1e-13, atol=1e-13)


def test_scale_invariance_kills_the_radial_tangent():
    """RMSNorm with eps = 0 is invariant to scaling x, so the tangent along x is 0."""
    B, N, H, D = 1, 3, 2, 8
    xs, gq, gk, c, s = make(B, N, H, D, 5)
    x = xs[:3]
    out = oracle.qk_norm_rope_jvp(*x, *x, gq, gk, c, s, H, eps=0.0)
    assert np.max(np.abs(out[3])) <= 1e-13 and np.max(np.abs(out[4])) <= 1e-13


def test_value_is_only_relaid_out_and_tangent_linear():
    B, N, H, D = 2, 3, 2, 4
    xs, gq, gk, c, s = make(B, N, H, D, 6)
    out = oracle.qk_norm_rope_jvp(*xs, gq, gk, c, s, H)
    assert np.array_equal(out[2], xs[2].reshape(B, N, H, D).permute(0, 2, 1, 3).numpy())
    assert np.array_equal(out[5], xs[5].reshape(B, N, H, D).permute(0, 2, 1, 3).numpy())
    t2 = [2.5 * t for t in xs[3:]]
    out2 = oracle.qk_norm_rope_jvp(*xs[:3], *t2, gq, gk, c, s, H)
    for i in (3, 4, 5):
        assert np.allclose(out2[i], 2.5 * out[i], rtol=1e-13, atol=1e-13)


def test_single_head_per_head_equals_whole_token():
    B, N, H, D = 1, 4, 1, 8
    xs, gq, gk, c, s = make(B, N, H, D, 7)
    a = oracle.qk_norm_rope_jvp(*xs, gq, gk, c, s, H, per_head=False)
    b = oracle.qk_norm_rope_jvp(*xs, gq, gk, c, s, H, per_head=True)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)


@pytest.mark.parametrize("per_head", [False, True])
def test_matches_torch_func_jvp(per_head):
    """Independent torch formulation: torch RMS normalisation, rotation as complex
    multiplication of (even, odd) pairs, tangent by torch.func.jvp."""
    B, N, H, D = 2, 5, 3, 8
    xs, gq, gk, c, s = make(B, N, H, D, 8)
    eps = 1e-4
    rot = torch.complex(c, s)  # [N, D/2]

    def f(x, g):
        if per_head:
            xh = x.reshape(B, N, H, D)
            y = xh * torch.rsqrt(xh.pow(2).mean(-1, keepdim=True) + eps) * g.reshape(H, D)
        else:
            y = (x * torch.rsqrt(x.pow(2).mean(-1, keepdim=True) + eps) * g).reshape(B, N, H, D)
        z = torch.view_as_complex(y.reshape(B, N, H, D // 2, 2).contiguous()) * rot[None, :, None, :]
        return torch.view_as_real(z).reshape(B, N, H, D).permute(0, 2, 1, 3)

    out = oracle.qk_norm_rope_jvp(*xs, gq, gk, c, s, H, eps=eps, per_head=per_head)
    for i, g in ((0, gq), (1, gk)):
        y, ty = torch.func.jvp(lambda x: f(x, g), (xs[i],), (xs[3 + i],))
        assert np.max(np.abs(out[i] - y.numpy())) <= 1e-13
        assert np.max(np.abs(out[3 + i] - ty.numpy())) <= 1e-13
