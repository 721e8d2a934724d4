"""fp64 CPU oracle for block-causal attention forward + JVP (test infrastructure).

Only the tests, the package's smoke check and the benchmark's CPU-baseline arm
import this package. The product path never does. The arithmetic lives in
`oracle.c` (plain C, fp64, OpenMP over rows); this module only compiles it with
gcc and marshals arrays through ctypes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

_F64, _F32, _BF16 = 0, 1, 2
_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-Wall",
                        "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, i32, dbl, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_double, ctypes.c_void_p
        lib.oracle_visible.argtypes = [i64, i64, i64, i32, i64, i64]
        lib.oracle_visible.restype = i32
        lib.oracle_visible_pairs.argtypes = [i64, i64, i64, i32]
        lib.oracle_visible_pairs.restype = i64
        lib.oracle_attn_fwd_jvp_rows.argtypes = [vp] * 6 + [i32, i64, i64, i64, dbl,
                                                            i64, i64, i64, i32, vp, i64,
                                                            vp, vp, vp, vp, i32]
        lib.oracle_attn_fwd_jvp_rows.restype = i32
        lib.oracle_qk_norm_rope_jvp.argtypes = [vp] * 6 + [i32, vp, vp, vp, vp, i64, i64, i64, i64,
                                                           dbl, i32] + [vp] * 6
        lib.oracle_qk_norm_rope_jvp.restype = i32
        lib.oracle_attn_bwd.argtypes = [vp] * 4 + [i32, i64, i64, i64, dbl, i64, i64, i64, i32] + [vp] * 4
        lib.oracle_attn_bwd.restype = i32
        lib.oracle_attn_bwd_dq_rows.argtypes = [vp] * 4 + [i32, i64, i64, i64, dbl, i64, i64, i64, i32,
                                                           vp, i64, vp, vp]
        lib.oracle_attn_bwd_dq_rows.restype = i32
        lib.oracle_max_threads.argtypes = []
        lib.oracle_max_threads.restype = i32
        _lib = lib
    return _lib


def max_threads() -> int:
    return _load().oracle_max_threads()


def visible(mask, qi: int, kj: int) -> bool:
    """Whether query token qi may attend to key token kj under `mask`
    (a MaskDesc or a (T, c, F, tf) tuple)."""
    T, c, F, tf = _mask_tuple(mask)
    return bool(_load().oracle_visible(T, c, F, tf, qi, kj))


def visible_pairs(mask) -> int:
    """Visible (query, key) pairs of one head, counted by brute force."""
    T, c, F, tf = _mask_tuple(mask)
    return int(_load().oracle_visible_pairs(T, c, F, tf))


def _mask_tuple(mask):
    if hasattr(mask, "as_tuple"):
        return mask.as_tuple()
    return tuple(int(x) for x in mask)


def _as_host(t: torch.Tensor):
    t = t.detach()
    if t.device.type != "cpu":
        t = t.cpu()
    t = t.contiguous()
    if t.dtype == torch.float64:
        return t, _F64
    if t.dtype == torch.float32:
        return t, _F32
    if t.dtype == torch.bfloat16:
        return t, _BF16
    raise TypeError(f"oracle: unsupported dtype {t.dtype}")


def attn_fwd_jvp_rows(q, k, v, tq, tk, tv, mask, scale=None, rows=None, nthreads=0):
    """fp64 O, tO, LSE, tLSE for selected rows.

    q..tv: [B, H, N, D] tensors of one dtype (fp64, fp32 or bf16; values are
    widened to double exactly). rows: flat ids bh*N + i (default: all rows).
    Returns numpy arrays o [R, D], to [R, D], lse [R], tlse [R] (float64).
    """
    ts = [_as_host(t) for t in (q, k, v, tq, tk, tv)]
    dtypes = {d for _, d in ts}
    if len(dtypes) != 1:
        raise TypeError("oracle: all six inputs must share one dtype")
    dtype = dtypes.pop()
    B, H, N, D = q.shape
    for t, _ in ts:
        if tuple(t.shape) != (B, H, N, D):
            raise ValueError("oracle: shape mismatch")
    T, c, F, tf = _mask_tuple(mask)
    if scale is None:
        scale = 1.0 / float(np.sqrt(D))
    if rows is None:
        rows = torch.arange(B * H * N, dtype=torch.int64)
    rows = torch.as_tensor(rows, dtype=torch.int64).contiguous()
    R = rows.numel()
    o = np.zeros((R, D), np.float64)
    to = np.zeros((R, D), np.float64)
    lse = np.zeros((R,), np.float64)
    tlse = np.zeros((R,), np.float64)
    rc = _load().oracle_attn_fwd_jvp_rows(
        *[t.data_ptr() for t, _ in ts], dtype, B * H, N, D, float(scale),
        T, c, F, tf, rows.data_ptr(), R,
        o.ctypes.data, to.ctypes.data, lse.ctypes.data, tlse.ctypes.data, int(nthreads))
    if rc != 0:
        raise ValueError("oracle: rejected arguments")
    return o, to, lse, tlse


def attn_fwd_jvp(q, k, v, tq, tk, tv, mask, scale=None, nthreads=0):
    """Full outputs shaped like the inputs: o, to [B, H, N, D]; lse, tlse [B, H, N]."""
    B, H, N, D = q.shape
    o, to, lse, tlse = attn_fwd_jvp_rows(q, k, v, tq, tk, tv, mask, scale, None, nthreads)
    return (o.reshape(B, H, N, D), to.reshape(B, H, N, D),
            lse.reshape(B, H, N), tlse.reshape(B, H, N))


def qk_norm_rope_jvp(xq, xk, xv, txq, txk, txv, gq, gk, cos, sin, H, eps=1e-6, per_head=False):
    """fp64 layer prologue: RMSNorm (+ JVP) and rotary embedding of q and k,
    layout change of all six tensors from [B, N, H*D] to [B, H, N, D].
    Returns numpy arrays (q, k, v, tq, tk, tv), each [B, H, N, D] float64."""
    ts = [_as_host(t) for t in (xq, xk, xv, txq, txk, txv)]
    dtypes = {d for _, d in ts}
    if len(dtypes) != 1:
        raise TypeError("oracle: all six inputs must share one dtype")
    dtype = dtypes.pop()
    B, N, C = xq.shape
    D = C // H
    g = [np.ascontiguousarray(torch.as_tensor(x, dtype=torch.float64).cpu().numpy()) for x in (gq, gk)]
    tab = [np.ascontiguousarray(torch.as_tensor(x, dtype=torch.float64).cpu().numpy()) for x in (cos, sin)]
    outs = [np.zeros((B, H, N, D), np.float64) for _ in range(6)]
    rc = _load().oracle_qk_norm_rope_jvp(*[t.data_ptr() for t, _ in ts], dtype,
                                         g[0].ctypes.data, g[1].ctypes.data, tab[0].ctypes.data,
                                         tab[1].ctypes.data, B, N, H, D, float(eps), int(bool(per_head)),
                                         *[o.ctypes.data for o in outs])
    if rc != 0:
        raise ValueError("oracle: rejected arguments")
    return tuple(outs)


def attn_bwd(q, k, v, dout, mask, scale=None):
    """fp64 backward of the masked attention primal: (dq, dk, dv, delta) as numpy
    arrays [B, H, N, D] (delta [B, H, N] = rowsum(P * dP) = <dO, O>)."""
    ts = [_as_host(t) for t in (q, k, v, dout)]
    dtypes = {d for _, d in ts}
    if len(dtypes) != 1:
        raise TypeError("oracle: all four inputs must share one dtype")
    dtype = dtypes.pop()
    B, H, N, D = q.shape
    T, c, F, tf = _mask_tuple(mask)
    if scale is None:
        scale = 1.0 / float(np.sqrt(D))
    dq, dk, dv = (np.zeros((B, H, N, D), np.float64) for _ in range(3))
    delta = np.zeros((B, H, N), np.float64)
    rc = _load().oracle_attn_bwd(*[t.data_ptr() for t, _ in ts], dtype, B * H, N, D, float(scale),
                                 T, c, F, tf, dq.ctypes.data, dk.ctypes.data, dv.ctypes.data,
                                 delta.ctypes.data)
    if rc != 0:
        raise ValueError("oracle: rejected arguments")
    return dq, dk, dv, delta


def attn_bwd_dq_rows(q, k, v, dout, mask, rows, scale=None):
    """fp64 dQ and Delta of selected query rows (flat ids bh*N + i) of the
    masked attention backward. Each row needs only its own softmax, so this
    serves full-size problems where the N x N backward would not finish.
    Returns numpy arrays dq [R, D] and delta [R] (float64)."""
    ts = [_as_host(t) for t in (q, k, v, dout)]
    dtypes = {d for _, d in ts}
    if len(dtypes) != 1:
        raise TypeError("oracle: all four inputs must share one dtype")
    dtype = dtypes.pop()
    B, H, N, D = q.shape
    T, c, F, tf = _mask_tuple(mask)
    if scale is None:
        scale = 1.0 / float(np.sqrt(D))
    rows = torch.as_tensor(rows, dtype=torch.int64).contiguous()
    R = rows.numel()
    dq = np.zeros((R, D), np.float64)
    delta = np.zeros((R,), np.float64)
    rc = _load().oracle_attn_bwd_dq_rows(*[t.data_ptr() for t, _ in ts], dtype, B * H, N, D, float(scale),
                                         T, c, F, tf, rows.data_ptr(), R, dq.ctypes.data, delta.ctypes.data)
    if rc != 0:
        raise ValueError("oracle: rejected arguments")
    return dq, delta


def out_proj_jvp(x, tx, w, bias=None):
    """Output projection of the attention block in primal-tangent form.

    Causal-rCM, section 3.2.2 ("JVP FSDP2"): the JVP runs layer by layer, each
    layer taking and returning a (primal, tangent) pair. The projection after
    attention is linear, so its tangent is the same map without the bias:
        y = x W^T + b,   ty = tx W^T.
    x, tx: [M, K] (tokens x H*D, the attention output in token-major layout);
    w: [C, K] (the layer's weight); bias: [C] or None. Returns (y, ty) as fp64
    numpy arrays [M, C]; the matmul is numpy's, in fp64, on the exact input
    values."""
    def f64(t):  # exact widening of bf16 / fp32 values
        if isinstance(t, torch.Tensor):
            return t.detach().cpu().to(torch.float64).numpy()
        return np.asarray(t, np.float64)

    x64, tx64, w64 = f64(x), f64(tx), f64(w)
    y = x64 @ w64.T
    if bias is not None:
        y = y + f64(bias)[None, :]
    return y, tx64 @ w64.T
