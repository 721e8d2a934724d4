"""Failure detection on the GPU without a fault: the tensor-core kernels' waits
are bounded. With the library's test hook the producers skip their copies (the
forward's query tiles, every copy of the backward's), so the MMA warp's first
wait can never complete; the kernel must give up after the configured limit,
report CAJ_ERR_DEVICE_TIMEOUT through the device error word, leave the context
usable, and the next normal call must be correct."""
import numpy as np
import pytest
import torch

import oracle
import masked_attention_jvp_b200 as caj
from masked_attention_jvp_b200 import _lib
from masked_attention_jvp_b200.workloads import MaskDesc, Workload, make_inputs

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives():
    L = _lib.lib()
    w = Workload("fault", 1, 1, 128, MaskDesc(64, 1, 2, 0), torch.bfloat16, seed=5)  # one CTA
    ins = make_inputs(w, "cuda")
    caj.device_status()  # clears any earlier error word
    assert L.caj_set_wait_timeout_ms(100.0) == _lib.CAJ_OK
    assert L.caj_debug_set_fault(1) == _lib.CAJ_OK
    try:
        caj.attn_fwd_jvp(*ins, w.mask)
        with pytest.raises(caj.CajError) as err:
            caj.device_status()
        assert err.value.status == _lib.CAJ_ERR_DEVICE_TIMEOUT
        assert L.caj_last_device_error_code() & 0xFF00 == 0x100  # a wait site, not another error
    finally:
        L.caj_debug_set_fault(0)
        L.caj_set_wait_timeout_ms(0.0)
    caj.device_status()  # the error word was cleared by the read above
    o, to, lse, tlse = caj.attn_fwd_jvp(*ins, w.mask)
    caj.device_status()
    ro, rto, rlse, rtlse = oracle.attn_fwd_jvp(*[t.cpu() for t in ins], w.mask)
    rel = lambda a, b: float(np.linalg.norm(a - b) / np.linalg.norm(b))
    assert rel(o.float().cpu().numpy(), ro) <= 1e-2
    assert rel(to.float().cpu().numpy(), rto) <= 1e-2


def test_fault_hook_rejects_unknown_modes():
    L = _lib.lib()
    assert L.caj_debug_set_fault(7) == _lib.CAJ_ERR_INVALID_ARG
    assert L.caj_debug_set_fault(0) == _lib.CAJ_OK


def test_clean_tangent_zero_kernels_time_out_too():
    """Both kernels of the clean-tangent-zero path (the JVP kernel on the noisy
    query tile, the primal-only kernel on the clean one) bound their waits the
    same way."""
    L = _lib.lib()
    from masked_attention_jvp_b200.workloads import zero_clean_tangents
    w = Workload("fault_ctz", 1, 1, 128, MaskDesc(64, 1, 2, 1), torch.bfloat16, seed=6)  # L = 128
    ins = make_inputs(w, "cuda")
    zero_clean_tangents(w, *ins[3:])
    caj.device_status()
    assert L.caj_set_wait_timeout_ms(100.0) == _lib.CAJ_OK
    assert L.caj_debug_set_fault(1) == _lib.CAJ_OK
    try:
        caj.attn_fwd_jvp(*ins, w.mask, clean_tangent_zero=True)
        with pytest.raises(caj.CajError) as err:
            caj.device_status()
        assert err.value.status == _lib.CAJ_ERR_DEVICE_TIMEOUT
        assert L.caj_last_device_error_code() & 0xFF00 == 0x100
    finally:
        L.caj_debug_set_fault(0)
        L.caj_set_wait_timeout_ms(0.0)
    caj.device_status()
    o, to, lse, tlse = caj.attn_fwd_jvp(*ins, w.mask, clean_tangent_zero=True)
    caj.device_status()
    ro, rto, rlse, rtlse = oracle.attn_fwd_jvp(*[t.cpu() for t in ins], w.mask)
    rel = lambda a, b: float(np.linalg.norm(a - b) / np.linalg.norm(b))
    assert rel(o.float().cpu().numpy(), ro) <= 1e-2
    assert rel(to.float().cpu().numpy(), rto) <= 1e-2


def test_backward_kernels_time_out_too():
    """The backward's dQ and dK/dV kernels bound their waits the same way: with
    the hook their producers issue no copies, the MMA warp's first wait runs
    out, and the next normal call is correct."""
    L = _lib.lib()
    w = Workload("fault_bwd", 1, 1, 128, MaskDesc(64, 1, 2, 0), torch.bfloat16, seed=7)  # one tile each
    q, k, v, _, _, _ = make_inputs(w, "cuda")
    g = torch.Generator(device="cpu").manual_seed(8)
    dout = torch.randn(q.shape, generator=g).to(torch.bfloat16).cuda()
    z = torch.zeros_like(q)
    o, _, lse, _ = caj.attn_fwd_jvp(q, k, v, z, z, z, w.mask)
    caj.device_status()
    assert L.caj_set_wait_timeout_ms(100.0) == _lib.CAJ_OK
    assert L.caj_debug_set_fault(1) == _lib.CAJ_OK
    try:
        caj.attn_bwd(q, k, v, o, dout, lse, w.mask)
        with pytest.raises(caj.CajError) as err:
            caj.device_status()
        assert err.value.status == _lib.CAJ_ERR_DEVICE_TIMEOUT
        assert L.caj_last_device_error_code() & 0xFF00 == 0x100
    finally:
        L.caj_debug_set_fault(0)
        L.caj_set_wait_timeout_ms(0.0)
    caj.device_status()
    dq, dk, dv, delta = caj.attn_bwd(q, k, v, o, dout, lse, w.mask)
    caj.device_status()
    rq, rk, rv, rdelta = oracle.attn_bwd(q.cpu(), k.cpu(), v.cpu(), dout.cpu(), w.mask)
    rel = lambda a, b: float(np.linalg.norm(a - b) / np.linalg.norm(b))
    assert rel(dq.float().cpu().numpy(), rq) <= 2e-2
    assert rel(dk.float().cpu().numpy(), rk) <= 2e-2
    assert rel(dv.float().cpu().numpy(), rv) <= 1e-2


def test_output_projection_times_out_too():
    """The projection kernel bounds its waits the same way: with the hook its
    producer issues no copies, the MMA thread's first wait runs out, and the
    next normal call is correct."""
    L = _lib.lib()
    g = torch.Generator(device="cuda").manual_seed(12)
    x, tx = (torch.randn(256, 128, device="cuda", generator=g).to(torch.bfloat16) for _ in range(2))
    wt = (torch.randn(256, 128, device="cuda", generator=g) / 128 ** 0.5).to(torch.bfloat16)
    caj.device_status()
    assert L.caj_set_wait_timeout_ms(100.0) == _lib.CAJ_OK
    assert L.caj_debug_set_fault(1) == _lib.CAJ_OK
    try:
        caj.out_proj_jvp(x, tx, wt)
        with pytest.raises(caj.CajError) as err:
            caj.device_status()
        assert err.value.status == _lib.CAJ_ERR_DEVICE_TIMEOUT
        assert L.caj_last_device_error_code() & 0xFF00 == 0x100
    finally:
        L.caj_debug_set_fault(0)
        L.caj_set_wait_timeout_ms(0.0)
    caj.device_status()
    y, ty = caj.out_proj_jvp(x, tx, wt)
    caj.device_status()
    ry, rty = oracle.out_proj_jvp(x, tx, wt)
    rel = lambda a, b: float(np.linalg.norm(a - b) / np.linalg.norm(b))
    assert rel(y.float().cpu().numpy(), ry) <= 1e-2
    assert rel(ty.float().cpu().numpy(), rty) <= 1e-2
