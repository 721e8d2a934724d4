"""The autograd binding (attention_jvp): its forward is the fused kernel's,
and backward() gives exactly the backward kernels' dQ, dK, dV for the
upstream gradient of o, while the tangent branch stays stop-gradient."""
import pytest
import torch

import masked_attention_jvp_b200 as caj
from masked_attention_jvp_b200.workloads import MaskDesc, make_inputs, small, zero_clean_tangents

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("ctz", [False, True], ids=["dense", "clean_tangent_zero"])
def test_gradients_are_the_backward_kernels(ctz):
    torch.cuda.set_device(0)
    w = small("autograd", 1, 3, 128, MaskDesc(300, 1, 6, 1), torch.bfloat16, seed=71, std_tangent=0.5)
    q, k, v, tq, tk, tv = make_inputs(w, "cuda")
    if ctz:
        zero_clean_tangents(w, tq, tk, tv)
    leaves = [t.clone().requires_grad_(True) for t in (q, k, v, tq, tk, tv)]
    o, to, lse, tlse = caj.attention_jvp(*leaves, w.mask, clean_tangent_zero=ctz)
    assert o.requires_grad
    assert not (to.requires_grad or lse.requires_grad or tlse.requires_grad)
    want = caj.attn_fwd_jvp(q, k, v, tq, tk, tv, w.mask, clean_tangent_zero=ctz)
    for got, ref in zip((o, to, lse, tlse), want):
        assert torch.equal(got.detach(), ref)
    gen = torch.Generator(device="cuda").manual_seed(72)
    dout = torch.randn(o.shape, device="cuda", generator=gen).to(torch.bfloat16)
    (o.float() * dout.float()).sum().backward()  # upstream gradient of o: dout (exact in bf16)
    dq, dk, dv, _ = caj.attn_bwd(q, k, v, want[0], dout, want[2], w.mask)
    torch.cuda.synchronize()
    caj.device_status()
    for leaf, ref in zip(leaves[:3], (dq, dk, dv)):
        assert torch.equal(leaf.grad, ref)
    for leaf in leaves[3:]:
        assert leaf.grad is None  # stop-gradient tangent branch


def test_rejects_non_bf16_inputs():
    w = small("autograd32", 1, 2, 64, MaskDesc(16, 1, 4, 0), torch.float32, seed=73)
    ins = make_inputs(w, "cuda")
    with pytest.raises(ValueError):
        caj.attention_jvp(*ins, w.mask)
