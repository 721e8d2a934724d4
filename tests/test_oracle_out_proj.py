"""Pins for the oracle of the output projection in primal-tangent form
(y = x W^T + b, ty = tx W^T). CPU only."""
import numpy as np
import torch

import oracle


def rand(shape, seed):
    return torch.randn(*shape, generator=torch.Generator().manual_seed(seed), dtype=torch.float64)


def test_matches_a_brute_force_loop():
    """Element by element from the definition (pins the orientation of W)."""
    M, K, C = 3, 5, 4
    x, tx, w, b = rand((M, K), 1), rand((M, K), 2), rand((C, K), 3), rand((C,), 4)
    y, ty = oracle.out_proj_jvp(x, tx, w, b)
    for m in range(M):
        for c in range(C):
            ref_y = float(b[c]) + sum(float(x[m, k]) * float(w[c, k]) for k in range(K))
            ref_ty = sum(float(tx[m, k]) * float(w[c, k]) for k in range(K))
            assert abs(y[m, c] - ref_y) <= 1e-12 and abs(ty[m, c] - ref_ty) <= 1e-12


def test_tangent_is_the_directional_derivative():
    """ty = d/dh y(x + h tx) at h = 0, exactly (y is affine in x)."""
    x, tx, w, b = rand((7, 16), 5), rand((7, 16), 6), rand((9, 16), 7), rand((9,), 8)
    h = 0.5
    y_p, _ = oracle.out_proj_jvp(x + h * tx, tx, w, b)
    y_m, _ = oracle.out_proj_jvp(x - h * tx, tx, w, b)
    _, ty = oracle.out_proj_jvp(x, tx, w, b)
    assert np.max(np.abs((y_p - y_m) / (2 * h) - ty)) <= 1e-12


def test_tangent_is_linear_and_bias_free():
    x, tx, w, b = rand((6, 8), 9), rand((6, 8), 10), rand((5, 8), 11), rand((5,), 12)
    _, ty1 = oracle.out_proj_jvp(x, tx, w, b)
    _, ty2 = oracle.out_proj_jvp(x, 3.0 * tx, w, None)
    assert np.max(np.abs(3.0 * ty1 - ty2)) <= 1e-12
    _, ty0 = oracle.out_proj_jvp(x, torch.zeros_like(tx), w, b)
    assert np.all(ty0 == 0.0)


def test_identity_weight_adds_the_bias():
    x, b = rand((4, 6), 13), rand((6,), 14)
    y, ty = oracle.out_proj_jvp(x, x, torch.eye(6, dtype=torch.float64), b)
    assert np.max(np.abs(y - (x.numpy() + b.numpy()[None, :]))) <= 1e-15
    assert np.max(np.abs(ty - x.numpy())) <= 1e-15


def test_bf16_inputs_are_widened_exactly():
    x = rand((3, 4), 15).to(torch.bfloat16)
    w = torch.eye(4, dtype=torch.bfloat16)
    y, _ = oracle.out_proj_jvp(x, x, w)
    assert np.array_equal(y, x.to(torch.float64).numpy())
