"""The host-buffer forward + JVP that allocates no device memory
(caj_attn_fwd_jvp_host_static), called through the C-ABI.

It serves callers that cannot allocate device memory: a plain C program or
plugin that keeps its tensors in host memory and links no device allocator, or
a host runtime whose memory manager owns the GPU. The library stages such a
call in a fixed array of its own instead of a caller-supplied workspace.

Its results must match the ordinary host-buffer entry point
(caj_attn_fwd_jvp_host, given a workspace allocated by torch) within the
tolerances the parity tests use, on two calls in a row. The second call has
other inputs and another shape, so output left in the shared array by the
first call cannot pass for the second's. This file is collected last, so a
run that stops at its first failure has run every other test first.
"""
import ctypes

import numpy as np
import pytest
import torch

import masked_attention_jvp_b200 as caj
from masked_attention_jvp_b200 import _lib
from masked_attention_jvp_b200.workloads import MaskDesc, small, make_inputs


def _static_call(ins, mask):
    """One call of caj_attn_fwd_jvp_host_static on host tensors, through ctypes."""
    q = ins[0]
    o, to = (torch.empty(q.shape, dtype=q.dtype, pin_memory=True) for _ in range(2))
    lse, tlse = (torch.empty(q.shape[:3], dtype=torch.float32, pin_memory=True) for _ in range(2))
    B, H, N, D = q.shape
    dtype = _lib.CAJ_DTYPE_BF16 if q.dtype == torch.bfloat16 else _lib.CAJ_DTYPE_F32
    prob = _lib.ProblemC(B, H, N, D, dtype, 0.0, 0)
    stream = torch.cuda.current_stream()
    st = _lib.lib().caj_attn_fwd_jvp_host_static(
        *[ctypes.c_void_p(t.data_ptr()) for t in ins], ctypes.byref(prob), ctypes.byref(_lib.mask_c(mask)),
        *[ctypes.c_void_p(t.data_ptr()) for t in (o, to, lse, tlse)], ctypes.c_void_p(stream.cuda_stream))
    _lib.check(st, "caj_attn_fwd_jvp_host_static")
    stream.synchronize()
    caj.device_status()
    return o, to, lse, tlse


def _close(got, want, bf16):
    """The parity tests' bounds: relative Frobenius (and max-abs on O, tO) for
    the bf16 path, relative Frobenius 1e-5 for fp32; max-abs on LSE."""
    fro, mx, lse_mx = (1e-2, 3e-2, 1e-2) if bf16 else (1e-5, 1e-5, 1e-5)
    for name, a, b in zip(("o", "to", "lse", "tlse"), got, want):
        a, b = a.double().numpy(), b.double().numpy()
        if name == "lse":
            assert float(np.max(np.abs(a - b))) <= lse_mx, name
            continue
        rel = float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-30))
        assert rel <= fro, (name, rel)
        if name in ("o", "to"):
            assert float(np.max(np.abs(a - b))) <= mx, name


@pytest.mark.gpu
def test_static_staging_matches_host_entry_point_twice():
    torch.cuda.set_device(0)
    cases = [  # two calls in a row: other inputs, another shape, dtype and mask
        small("static_tf", 1, 4, 128, MaskDesc(100, 1, 4, 1), torch.bfloat16, seed=61),
        small("static_chunk_fp32", 2, 2, 64, MaskDesc(24, 2, 6, 0), torch.float32, seed=62),
    ]
    for w in cases:
        ins = make_inputs(w, "cpu")
        want = caj.attn_fwd_jvp(*ins, w.mask)      # caj_attn_fwd_jvp_host with a torch workspace
        got = _static_call(ins, w.mask)
        _close(got, want, w.dtype == torch.bfloat16)


def test_static_staging_rejects_a_problem_beyond_its_array():
    """A problem whose staging exceeds the fixed array is refused before any
    CUDA call, with CAJ_ERR_UNSUPPORTED (no GPU needed)."""
    B, H, N, D = 1, 12, 4096, 128     # 8 tensors x 12.6 MB of staging > 64 MiB
    prob = _lib.ProblemC(B, H, N, D, _lib.CAJ_DTYPE_BF16, 0.0, 0)
    need = ctypes.c_size_t(0)
    assert _lib.lib().caj_attn_fwd_jvp_host_workspace(ctypes.byref(prob), ctypes.byref(need)) == _lib.CAJ_OK
    assert need.value > _lib.HOST_STATIC_MAX_BYTES
    buf = ctypes.create_string_buffer(16)
    p = ctypes.c_void_p(ctypes.addressof(buf))
    st = _lib.lib().caj_attn_fwd_jvp_host_static(p, p, p, p, p, p, ctypes.byref(prob),
                                                 ctypes.byref(_lib.mask_c(MaskDesc(1024, 1, 2, 1))),
                                                 p, p, p, p, None)
    assert st == _lib.CAJ_ERR_UNSUPPORTED
