"""Pins for the fp64 oracle: properties fixed by the mathematics and by the mask
definitions of the Causal-rCM pages, each chosen so that a plausible mistake in
the oracle (a dropped term, a wrong sign, a transposed operand, a wrong chunk
index) fails at least one of them. CPU only."""
import math

import numpy as np
import pytest
import torch

import oracle
from masked_attention_jvp_b200.workloads import MaskDesc
from tests.conftest import load_mask_fixture

F64 = torch.float64


def rand_inputs(B, H, N, D, seed, std_t=1.0, dtype=F64):
    g = torch.Generator().manual_seed(seed)
    xs = [torch.randn(B, H, N, D, generator=g, dtype=F64) for _ in range(3)]
    ts = [std_t * torch.randn(B, H, N, D, generator=g, dtype=F64) for _ in range(3)]
    return [x.to(dtype) for x in xs + ts]


def rel_fro(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


MASKS = [
    MaskDesc(3, 1, 4, 0),   # frame-wise block-causal
    MaskDesc(2, 2, 4, 0),   # chunk-wise block-causal
    MaskDesc(3, 1, 3, 1),   # teacher forcing, frame-wise
    MaskDesc(2, 3, 6, 1),   # teacher forcing, chunk-wise
    MaskDesc(1, 1, 7, 0),   # token-causal
    MaskDesc(5, 1, 1, 0),   # a single frame: dense attention
]


# ---------------------------------------------------------------- mask pins
@pytest.mark.parametrize("name", ["mask_tf_T2_c1_F3.txt", "mask_tf_T1_c2_F4.txt",
                                  "mask_bc_T1_c2_F4.txt", "mask_bc_T3_c1_F3.txt"])
def test_mask_matches_hand_drawn_fixture(name):
    desc, mat = load_mask_fixture(name)
    n = len(mat)
    for i in range(n):
        for j in range(n):
            assert oracle.visible(desc, i, j) == bool(mat[i][j]), (name, i, j)
    assert oracle.visible_pairs(desc) == sum(map(sum, mat))


@pytest.mark.parametrize("T,c,F", [(1, 1, 1), (3, 1, 5), (2, 3, 6), (4, 2, 8), (7, 3, 3)])
def test_visible_pair_count_closed_form(T, c, F):
    # n chunks of G tokens. Block-causal: chunk i sees i+1 chunks -> G^2 n(n+1)/2.
    # TF: the clean half repeats that count; noisy chunk j sees j clean chunks plus
    # itself -> again G^2 n(n+1)/2; total G^2 n(n+1).
    G, n = c * T, F // c
    assert oracle.visible_pairs((T, c, F, 0)) == G * G * n * (n + 1) // 2
    assert oracle.visible_pairs((T, c, F, 1)) == G * G * n * (n + 1)


def test_visible_rejects_out_of_range():
    assert not oracle.visible((2, 1, 3, 0), 6, 0)
    assert not oracle.visible((2, 1, 3, 0), 0, -1)
    assert not oracle.visible((2, 1, 3, 1), 12, 0)


# ------------------------------------------------------- JVP vs finite differences
@pytest.mark.parametrize("mask", MASKS)
@pytest.mark.parametrize("D", [1, 8])
def test_tangent_matches_central_differences(mask, D):
    """(F(x + h t) - F(x - h t)) / 2h with h = 1e-6 agrees with (tO, tLSE) to
    rel. Frobenius 1e-7: the tangent is the derivative of the primal."""
    N = mask.seq_len
    q, k, v, tq, tk, tv = rand_inputs(1, 2, N, D, seed=11 + D)
    h = 1e-6
    o, to, lse, tlse = oracle.attn_fwd_jvp(q, k, v, tq, tk, tv, mask)
    z = [torch.zeros_like(q)] * 3
    op, _, lp, _ = oracle.attn_fwd_jvp(q + h * tq, k + h * tk, v + h * tv, *z, mask)
    om, _, lm, _ = oracle.attn_fwd_jvp(q - h * tq, k - h * tk, v - h * tv, *z, mask)
    fd_o = (op - om) / (2 * h)
    fd_l = (lp - lm) / (2 * h)
    assert rel_fro(to, fd_o) <= 1e-7
    assert rel_fro(tlse, fd_l) <= 1e-7


@pytest.mark.parametrize("scale", [0.3, 2.0])
def test_central_differences_with_explicit_scale(scale):
    mask = MaskDesc(2, 1, 3, 1)
    q, k, v, tq, tk, tv = rand_inputs(1, 1, mask.seq_len, 4, seed=5)
    h = 1e-6
    _, to, _, tlse = oracle.attn_fwd_jvp(q, k, v, tq, tk, tv, mask, scale=scale)
    z = [torch.zeros_like(q)] * 3
    op, _, lp, _ = oracle.attn_fwd_jvp(q + h * tq, k + h * tk, v + h * tv, *z, mask, scale=scale)
    om, _, lm, _ = oracle.attn_fwd_jvp(q - h * tq, k - h * tk, v - h * tv, *z, mask, scale=scale)
    assert rel_fro(to, (op - om) / (2 * h)) <= 1e-7
    assert rel_fro(tlse, (lp - lm) / (2 * h)) <= 1e-7


# ------------------------------------------------------------- exact special cases
def test_linear_in_the_tangent():
    mask = MaskDesc(3, 1, 3, 1)
    q, k, v, a1, a2, a3 = rand_inputs(1, 2, mask.seq_len, 8, seed=3)
    _, _, _, b1, b2, b3 = rand_inputs(1, 2, mask.seq_len, 8, seed=4)
    al, be = 0.7, -1.3
    _, t1, _, l1 = oracle.attn_fwd_jvp(q, k, v, a1, a2, a3, mask)
    _, t2, _, l2 = oracle.attn_fwd_jvp(q, k, v, b1, b2, b3, mask)
    _, t12, _, l12 = oracle.attn_fwd_jvp(q, k, v, al * a1 + be * b1, al * a2 + be * b2,
                                         al * a3 + be * b3, mask)
    assert np.max(np.abs(t12 - (al * t1 + be * t2))) <= 1e-12
    assert np.max(np.abs(l12 - (al * l1 + be * l2))) <= 1e-12


def test_zero_tangent_gives_zero():
    mask = MaskDesc(2, 2, 4, 1)
    q, k, v, _, _, _ = rand_inputs(1, 2, mask.seq_len, 8, seed=6)
    z = torch.zeros_like(q)
    _, to, _, tlse = oracle.attn_fwd_jvp(q, k, v, z, z, z, mask)
    assert np.all(to == 0.0) and np.all(tlse == 0.0)


def test_value_only_tangent_is_attention_of_the_tangent():
    """Tangent (0, 0, tV): tO = P tV (the primal with V replaced by tV), tLSE = 0.
    Tangent (0, 0, V): tO = O."""
    mask = MaskDesc(3, 1, 3, 1)
    q, k, v, _, _, tv = rand_inputs(1, 2, mask.seq_len, 8, seed=7)
    z = torch.zeros_like(q)
    _, to, _, tlse = oracle.attn_fwd_jvp(q, k, v, z, z, tv, mask)
    o_tv, _, _, _ = oracle.attn_fwd_jvp(q, k, tv, z, z, z, mask)
    assert np.max(np.abs(to - o_tv)) <= 1e-13
    assert np.all(tlse == 0.0)
    o, to2, _, _ = oracle.attn_fwd_jvp(q, k, v, z, z, v, mask)
    assert np.max(np.abs(to2 - o)) <= 1e-13


def test_single_visible_key():
    """Token-causal mask (T=1, c=1): row 0 sees only key 0, so O_0 = v_0,
    tO_0 = tv_0, LSE_0 = s_00 and tLSE_0 = ts_00."""
    mask = MaskDesc(1, 1, 5, 0)
    D = 6
    q, k, v, tq, tk, tv = rand_inputs(1, 1, mask.seq_len, D, seed=8)
    o, to, lse, tlse = oracle.attn_fwd_jvp(q, k, v, tq, tk, tv, mask)
    sc = 1 / math.sqrt(D)
    q0, k0 = q[0, 0, 0], k[0, 0, 0]
    assert np.allclose(o[0, 0, 0], v[0, 0, 0].numpy(), rtol=0, atol=1e-15)
    assert np.allclose(to[0, 0, 0], tv[0, 0, 0].numpy(), rtol=0, atol=1e-15)
    assert lse[0, 0, 0] == pytest.approx(sc * float(q0 @ k0), abs=1e-14)
    assert tlse[0, 0, 0] == pytest.approx(sc * float(tq[0, 0, 0] @ k0 + q0 @ tk[0, 0, 0]), abs=1e-14)


def test_two_keys_closed_form():
    """Two visible keys, D = 1: p_1 = sigmoid(s_1 - s_0), so
    O = v_0 + p_1 (v_1 - v_0),
    tO = sigma'(s_1 - s_0) (ts_1 - ts_0)(v_1 - v_0) + (1 - p_1) tv_0 + p_1 tv_1,
    LSE = s_0 + softplus(s_1 - s_0), tLSE = ts_0 + p_1 (ts_1 - ts_0)."""
    mask = MaskDesc(1, 1, 2, 0)  # token-causal, row 1 sees keys 0 and 1
    vals = {"q": [0.0, 1.5], "k": [0.8, -0.4], "v": [2.0, -1.0],
            "tq": [0.0, 0.25], "tk": [-0.5, 0.75], "tv": [0.3, 1.1]}
    ts = [torch.tensor(vals[n], dtype=F64).reshape(1, 1, 2, 1) for n in ("q", "k", "v", "tq", "tk", "tv")]
    o, to, lse, tlse = oracle.attn_fwd_jvp(*ts, mask, scale=1.0)
    q1, tq1 = 1.5, 0.25
    s0, s1 = q1 * 0.8, q1 * -0.4
    ts0, ts1 = tq1 * 0.8 + q1 * -0.5, tq1 * -0.4 + q1 * 0.75
    p1 = 1 / (1 + math.exp(-(s1 - s0)))
    exp_o = 2.0 + p1 * (-1.0 - 2.0)
    exp_to = p1 * (1 - p1) * (ts1 - ts0) * (-3.0) + (1 - p1) * 0.3 + p1 * 1.1
    assert o[0, 0, 1, 0] == pytest.approx(exp_o, abs=1e-14)
    assert to[0, 0, 1, 0] == pytest.approx(exp_to, abs=1e-14)
    assert lse[0, 0, 1] == pytest.approx(s0 + math.log1p(math.exp(s1 - s0)), abs=1e-14)
    assert tlse[0, 0, 1] == pytest.approx(ts0 + p1 * (ts1 - ts0), abs=1e-14)


@pytest.mark.parametrize("mask", [MaskDesc(3, 1, 4, 0), MaskDesc(2, 2, 6, 1), MaskDesc(3, 1, 3, 1)])
def test_future_chunks_do_not_change_earlier_rows(mask):
    """The mask has no tangent and hides future chunks: perturbing every input
    of the last chunk (both copies for TF) leaves all other rows bit-identical."""
    N = mask.seq_len
    xs = rand_inputs(1, 2, N, 4, seed=9)
    G = mask.frames_per_chunk * mask.tokens_per_frame
    L = mask.n_frames * mask.tokens_per_frame
    last = list(range(L - G, L))
    if mask.tf_layout:
        last += list(range(2 * L - G, 2 * L))
    ys = [x.clone() for x in xs]
    g = torch.Generator().manual_seed(99)
    for y in ys:
        y[:, :, last] = 50 * torch.randn(y[:, :, last].shape, generator=g, dtype=F64)
    a = oracle.attn_fwd_jvp(*xs, mask)
    b = oracle.attn_fwd_jvp(*ys, mask)
    keep = [i for i in range(N) if i not in last]
    for x, y in zip(a, b):
        assert np.array_equal(x[:, :, keep], y[:, :, keep])


def test_permuting_keys_inside_a_chunk():
    """Attention is bidirectional inside a chunk: permuting the keys (k, v, tk, tv
    together) within one chunk leaves every output unchanged up to rounding."""
    mask = MaskDesc(4, 1, 3, 1)
    q, k, v, tq, tk, tv = rand_inputs(1, 1, mask.seq_len, 8, seed=12)
    perm = torch.arange(mask.seq_len)
    perm[4:8] = torch.tensor([6, 4, 7, 5])          # clean frame 1
    perm[16:20] = torch.tensor([19, 18, 16, 17])    # noisy frame 1
    a = oracle.attn_fwd_jvp(q, k, v, tq, tk, tv, mask)
    b = oracle.attn_fwd_jvp(q, k[:, :, perm], v[:, :, perm], tq, tk[:, :, perm], tv[:, :, perm], mask)
    for x, y in zip(a, b):
        assert np.max(np.abs(x - y)) <= 1e-13


# ----------------------------------------- cross-checks against torch library routines
def dense_mask_from_chunks(mask: MaskDesc):
    """Independent construction of the boolean mask with torch ops: a chunk id
    and a copy id per token, then the visibility rule as tensor comparisons."""
    T, c, F, tf = mask.as_tuple()
    L = F * T
    tok = torch.arange(L * (2 if tf else 1))
    copy = tok // L                    # 0 = clean, 1 = noisy
    chunk = (tok % L) // (c * T)
    qc, kc = chunk[:, None], chunk[None, :]
    qn, kn = copy[:, None], copy[None, :]
    if not tf:
        return kc <= qc
    clean_q = (qn == 0) & (kn == 0) & (kc <= qc)
    noisy_q = (qn == 1) & (((kn == 0) & (kc < qc)) | ((kn == 1) & (kc == qc)))
    return clean_q | noisy_q


def naive_attention(q, k, v, m, scale):
    s = (q @ k.transpose(-1, -2)) * scale
    s = s.masked_fill(~m, float("-inf"))
    return torch.softmax(s, dim=-1) @ v


@pytest.mark.parametrize("mask", MASKS)
def test_primal_matches_torch_sdpa(mask):
    N, D = mask.seq_len, 8
    q, k, v, tq, tk, tv = rand_inputs(2, 2, N, D, seed=21)
    m = dense_mask_from_chunks(mask)
    ref = torch.nn.functional.scaled_dot_product_attention(q, k, v, attn_mask=m)
    s = (q @ k.transpose(-1, -2)) / math.sqrt(D)
    ref_lse = torch.logsumexp(s.masked_fill(~m, float("-inf")), dim=-1)
    o, _, lse, _ = oracle.attn_fwd_jvp(q, k, v, tq, tk, tv, mask)
    assert np.max(np.abs(o - ref.numpy())) <= 1e-12
    assert np.max(np.abs(lse - ref_lse.numpy())) <= 1e-12


@pytest.mark.parametrize("mask", MASKS)
def test_tangent_matches_torch_func_jvp(mask):
    N, D = mask.seq_len, 8
    q, k, v, tq, tk, tv = rand_inputs(1, 3, N, D, seed=22, std_t=0.5)
    m = dense_mask_from_chunks(mask)
    sc = 1 / math.sqrt(D)

    def f(q_, k_, v_):
        out = naive_attention(q_, k_, v_, m, sc)
        s = (q_ @ k_.transpose(-1, -2)) * sc
        return out, torch.logsumexp(s.masked_fill(~m, float("-inf")), dim=-1)

    (_, _), (t_o, t_lse) = torch.func.jvp(f, (q, k, v), (tq, tk, tv))
    _, to, _, tlse = oracle.attn_fwd_jvp(q, k, v, tq, tk, tv, mask)
    assert np.max(np.abs(to - t_o.numpy())) <= 1e-12
    assert np.max(np.abs(tlse - t_lse.numpy())) <= 1e-12


# ---------------------------------------------------------------- input handling
def test_bf16_and_fp32_inputs_are_widened_exactly():
    mask = MaskDesc(3, 1, 3, 1)
    xs = rand_inputs(1, 2, mask.seq_len, 8, seed=30)
    for dt in (torch.float32, torch.bfloat16):
        ys = [x.to(dt) for x in xs]
        a = oracle.attn_fwd_jvp(*ys, mask)
        b = oracle.attn_fwd_jvp(*[y.to(F64) for y in ys], mask)
        for x, y in zip(a, b):
            assert np.array_equal(x, y)


def test_row_subset_equals_full():
    mask = MaskDesc(5, 1, 4, 1)
    xs = rand_inputs(2, 2, mask.seq_len, 8, seed=31)
    full = oracle.attn_fwd_jvp(*xs, mask)
    rows = torch.tensor([0, 7, 19, 20, 39, 41, 79, 80, 120, 159])
    sub = oracle.attn_fwd_jvp_rows(*xs, mask, rows=rows)
    B, H, N, D = xs[0].shape
    for f, s in zip(full, sub):
        flat = f.reshape(B * H * N, -1)
        assert np.array_equal(flat[rows.numpy()].reshape(s.shape), s)


def test_rejects_inconsistent_sequence_length():
    xs = rand_inputs(1, 1, 10, 4, seed=1)
    with pytest.raises(ValueError):
        oracle.attn_fwd_jvp(*xs, MaskDesc(3, 1, 3, 0))
