"""Fused forward + forward-mode JVP of block-causal softmax attention on B200.

Public API (a thin layer over the C-ABI library libcausaljvp):

    o, to, lse, tlse = attn_fwd_jvp(q, k, v, tq, tk, tv, mask, scale=None)
    o, to, lse, tlse = attention_jvp(q, k, v, tq, tk, tv, mask)  # o differentiable in q, k, v

q..tv are [B, H, N, D] tensors (bf16 for the tensor-core path, fp32 for the
CUDA-core fp32 path), `mask` a MaskDesc (or a (tokens_per_frame,
frames_per_chunk, n_frames, tf_layout) tuple). With CUDA tensors everything
stays on the device and the call is asynchronous on the current stream. With
CPU tensors the library's host-buffer entry point copies the inputs to the
current CUDA device and the outputs back, overlapping the copies with the
kernels chunk by chunk (the end-to-end path).

The operation is the masked FlashAttention JVP of the Causal-rCM paper
(appendix B, eq. 42-45): O = softmax(scale Q K^T + M) V,
tO = (P o (tS - rowsum(P o tS))) V + P tV with tS = scale (tQ K^T + Q tK^T),
LSE (natural log) and tLSE = rowsum(P o tS).
"""
from __future__ import annotations

import ctypes
from typing import Optional

import torch

from . import _lib
from ._lib import CajError, EXPORTED, LIB_PATH
from .workloads import MaskDesc

__all__ = ["attention_jvp", "attn_fwd_jvp", "attn_fwd_jvp_out", "attn_fwd_jvp_scatter", "attn_fwd_jvp_host_static", "signal_barrier",
           "ipc_export", "ipc_open", "ipc_close", "part_query_tiles", "attn_bwd", "qk_norm_rope_jvp", "out_proj_jvp", "MaskDesc", "CajError", "visible_pairs",
           "row_key_ranges", "qtile_key_tiles", "device_status", "flops", "EXPORTED", "LIB_PATH",
           "BLOCK_M", "BLOCK_N"]

BLOCK_M = 128  # query rows per tile of both kernels
BLOCK_N = 64   # keys per tile of the tensor-core kernel

_DTYPES = {torch.float32: _lib.CAJ_DTYPE_F32, torch.bfloat16: _lib.CAJ_DTYPE_BF16}

from .autograd import attention_jvp  # noqa: E402  (autograd binding: fused forward, backward kernels)


def part_query_tiles(mask, part: int, nparts: int):
    """The 128-row query tiles part `part` of `nparts` runs, heaviest first."""
    n = _lib.lib().caj_part_query_tiles(ctypes.byref(_lib.mask_c(mask)), int(part), int(nparts), None, 0)
    if n < 0:
        raise ValueError("caj_part_query_tiles rejected its arguments")
    buf = (ctypes.c_int32 * max(n, 1))()
    _lib.lib().caj_part_query_tiles(ctypes.byref(_lib.mask_c(mask)), int(part), int(nparts), buf, n)
    return list(buf[:n])


def visible_pairs(mask) -> int:
    """Visible (query, key) pairs of one head (closed form, from the library)."""
    n = _lib.lib().caj_visible_pairs(ctypes.byref(_lib.mask_c(mask)))
    if n < 0:
        raise ValueError(f"invalid mask descriptor {mask}")
    return int(n)


def flops(B: int, H: int, D: int, mask) -> int:
    """Algorithmic floating-point work of one call: 12 D per visible pair per head
    (six products of 2 D flops: S, two for tS, O, two for tO)."""
    return 12 * D * visible_pairs(mask) * B * H


def row_key_ranges(mask, row: int):
    r = (ctypes.c_int32 * 4)()
    _lib.check(_lib.lib().caj_row_key_ranges(ctypes.byref(_lib.mask_c(mask)), int(row), r),
               "caj_row_key_ranges")
    return (r[0], r[1]), (r[2], r[3])


def qtile_key_tiles(mask, q0: int, q1: int, block_n: int = BLOCK_N):
    t = (ctypes.c_int32 * 4)()
    n = _lib.lib().caj_qtile_key_tiles(ctypes.byref(_lib.mask_c(mask)), int(q0), int(q1),
                                       int(block_n), t)
    if n < 0:
        raise ValueError("caj_qtile_key_tiles rejected its arguments")
    return n, (t[0], t[1]), (t[2], t[3])


def device_status(stream: Optional[torch.cuda.Stream] = None):
    """Synchronise the stream and raise CajError if a kernel gave up on a wait."""
    s = (stream or torch.cuda.current_stream()).cuda_stream
    _lib.check(_lib.lib().caj_last_device_status(ctypes.c_void_p(s)), "caj_last_device_status")


def _problem(q: torch.Tensor, scale: Optional[float], clean_tangent_zero: bool = False,
             token_major_out: bool = False) -> _lib.ProblemC:
    B, H, N, D = q.shape
    flags = (_lib.CAJ_FLAG_CLEAN_TANGENT_ZERO if clean_tangent_zero else 0) | \
        (_lib.CAJ_FLAG_TOKEN_MAJOR_OUT if token_major_out else 0)
    return _lib.ProblemC(B, H, N, D, _DTYPES[q.dtype], float(scale) if scale else 0.0, flags)


def attn_fwd_jvp_out(q, k, v, tq, tk, tv, mask, o, to, lse, tlse, scale: Optional[float] = None,
                     stream: Optional[torch.cuda.Stream] = None, clean_tangent_zero: bool = False,
                     token_major_out: bool = False, part=None) -> None:
    """Writes into caller-provided CUDA tensors o, to [B,H,N,D] and lse, tlse [B,H,N] fp32.

    part: None for the whole call, or (r, n): only the query tiles of part r
    of n (cost-balanced, every head; caj_attn_fwd_jvp_part), the way n GPUs
    split one call with no collective. Rows of other parts are left as they are.

    clean_tangent_zero: teacher-forcing layout only; the caller guarantees that
    tq, tk, tv are zero on the clean half, and the kernel skips the products
    that vanish (clean query tiles compute only the primal).
    token_major_out: o and to are [B,N,H,D] (the output projection's input
    layout, see out_proj_jvp) instead of [B,H,N,D]."""
    ins = (q, k, v, tq, tk, tv)
    for t in ins + (o, to, lse, tlse):
        if not t.is_cuda:
            raise ValueError("attn_fwd_jvp_out: all tensors must be CUDA tensors")
        if not t.is_contiguous():
            raise ValueError("attn_fwd_jvp_out: tensors must be contiguous")
    if q.dtype not in _DTYPES or any(t.dtype != q.dtype for t in ins + (o, to)):
        raise ValueError("attn_fwd_jvp_out: q..tv, o, to must share one dtype (bf16 or fp32)")
    B, H, N, D = q.shape
    out_shape = (B, N, H, D) if token_major_out else (B, H, N, D)
    if any(t.shape != q.shape for t in ins) or o.shape != out_shape or to.shape != out_shape:
        raise ValueError("attn_fwd_jvp_out: shape mismatch")
    if lse.dtype != torch.float32 or tlse.dtype != torch.float32 or lse.shape != q.shape[:3] \
            or tlse.shape != q.shape[:3]:
        raise ValueError("attn_fwd_jvp_out: lse/tlse must be fp32 [B,H,N]")
    s = (stream or torch.cuda.current_stream(q.device)).cuda_stream
    prob = _problem(q, scale, clean_tangent_zero, token_major_out)
    outs = [ctypes.c_void_p(t.data_ptr()) for t in (o, to, lse, tlse)]
    if part is None:
        st = _lib.lib().caj_attn_fwd_jvp(*[ctypes.c_void_p(t.data_ptr()) for t in ins],
                                         ctypes.byref(prob), ctypes.byref(_lib.mask_c(mask)), *outs,
                                         ctypes.c_void_p(s))
        _lib.check(st)
    else:
        r, n = part
        st = _lib.lib().caj_attn_fwd_jvp_part(*[ctypes.c_void_p(t.data_ptr()) for t in ins],
                                              ctypes.byref(prob), ctypes.byref(_lib.mask_c(mask)),
                                              int(r), int(n), *outs, ctypes.c_void_p(s))
        _lib.check(st, "caj_attn_fwd_jvp_part")


def attn_fwd_jvp(q, k, v, tq, tk, tv, mask, scale: Optional[float] = None,
                 clean_tangent_zero: bool = False, token_major_out: bool = False):
    """Returns (o, to, lse, tlse). See the module docstring and attn_fwd_jvp_out.

    With CPU tensors the library's host-buffer entry point runs the call: it
    copies head chunks to a device workspace, runs the kernel on each chunk and
    copies the outputs back, with the three overlapped. Outputs are returned
    in pinned host memory; pinned inputs copy fastest."""
    if q.is_cuda:
        ins = [q, k, v, tq, tk, tv]
        B, H, N, D = q.shape
        out_shape = (B, N, H, D) if token_major_out else (B, H, N, D)
        o = torch.empty(out_shape, dtype=q.dtype, device=q.device)
        to = torch.empty(out_shape, dtype=q.dtype, device=q.device)
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
        tlse = torch.empty_like(lse)
        attn_fwd_jvp_out(*ins, mask, o, to, lse, tlse, scale=scale, clean_tangent_zero=clean_tangent_zero,
                         token_major_out=token_major_out)
        return o, to, lse, tlse
    if token_major_out:
        raise ValueError("attn_fwd_jvp: host tensors take the head-major output layout only")
    ins = (q, k, v, tq, tk, tv)
    for t in ins:
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("attn_fwd_jvp: host inputs must be contiguous CPU tensors")
    if q.dtype not in _DTYPES or any(t.dtype != q.dtype or t.shape != q.shape for t in ins):
        raise ValueError("attn_fwd_jvp: q..tv must share one shape and dtype (bf16 or fp32)")
    prob = _problem(q, scale, clean_tangent_zero)
    L = _lib.lib()
    nbytes = ctypes.c_size_t(0)
    _lib.check(L.caj_attn_fwd_jvp_host_workspace(ctypes.byref(prob), ctypes.byref(nbytes)),
               "caj_attn_fwd_jvp_host_workspace")
    dev = torch.device("cuda", torch.cuda.current_device())
    workspace = torch.empty(nbytes.value, dtype=torch.uint8, device=dev)
    o = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    to = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, pin_memory=True)
    tlse = torch.empty(q.shape[:3], dtype=torch.float32, pin_memory=True)
    stream = torch.cuda.current_stream(dev)
    st = L.caj_attn_fwd_jvp_host(*[ctypes.c_void_p(t.data_ptr()) for t in ins], ctypes.byref(prob),
                                 ctypes.byref(_lib.mask_c(mask)),
                                 *[ctypes.c_void_p(t.data_ptr()) for t in (o, to, lse, tlse)],
                                 ctypes.c_void_p(workspace.data_ptr()), nbytes,
                                 ctypes.c_void_p(stream.cuda_stream))
    _lib.check(st, "caj_attn_fwd_jvp_host")
    stream.synchronize()
    return o, to, lse, tlse


def attn_fwd_jvp_host_static(q, k, v, tq, tk, tv, mask, scale: Optional[float] = None,
                             clean_tangent_zero: bool = False):
    """Host tensors in, pinned host tensors out, with no device memory
    allocated anywhere: the library stages the call in a fixed device array of
    its own (caj_attn_fwd_jvp_host_static). This is for callers that cannot
    allocate device memory, e.g. a host runtime whose allocator owns the GPU.
    The problem's staging must fit in HOST_STATIC_MAX_BYTES (64 MiB); calls
    share that array, so calls overlapping on the GPU race. The first call on
    a device looks up the array's address: make it before any stream capture.
    Returns (o, to, lse, tlse) like attn_fwd_jvp on host tensors."""
    ins = (q, k, v, tq, tk, tv)
    for t in ins:
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("attn_fwd_jvp_host_static: inputs must be contiguous CPU tensors")
    if q.dtype not in _DTYPES or any(t.dtype != q.dtype or t.shape != q.shape for t in ins):
        raise ValueError("attn_fwd_jvp_host_static: q..tv must share one shape and dtype (bf16 or fp32)")
    prob = _problem(q, scale, clean_tangent_zero)
    L = _lib.lib()
    o = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    to = torch.empty(q.shape, dtype=q.dtype, pin_memory=True)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, pin_memory=True)
    tlse = torch.empty(q.shape[:3], dtype=torch.float32, pin_memory=True)
    stream = torch.cuda.current_stream(torch.device("cuda", torch.cuda.current_device()))
    st = L.caj_attn_fwd_jvp_host_static(*[ctypes.c_void_p(t.data_ptr()) for t in ins], ctypes.byref(prob),
                                        ctypes.byref(_lib.mask_c(mask)),
                                        *[ctypes.c_void_p(t.data_ptr()) for t in (o, to, lse, tlse)],
                                        ctypes.c_void_p(stream.cuda_stream))
    if st == _lib.CAJ_ERR_UNSUPPORTED:
        raise _lib.CajError(st, "caj_attn_fwd_jvp_host_static: the problem's staging exceeds the "
                                f"library's fixed {_lib.HOST_STATIC_MAX_BYTES >> 20} MiB device array "
                                "(or D is not 64/128)")
    _lib.check(st, "caj_attn_fwd_jvp_host_static")
    stream.synchronize()
    return o, to, lse, tlse


def attn_fwd_jvp_scatter(q, k, v, tq, tk, tv, mask, o, to, lse, tlse, head_base: int = 0,
                         scale: Optional[float] = None, stream: Optional[torch.cuda.Stream] = None,
                         clean_tangent_zero: bool = False, token_major_out: bool = False) -> None:
    """Forward + JVP whose output rows go straight to their sequence slice.

    q..tv: [B, H, N, D] CUDA tensors, this call's H heads over the whole packed
    sequence. o, to, lse, tlse: lists of P tensors, entry r the buffers of
    sequence slice r (token rows [r N/P, (r+1) N/P)): o[r], to[r] are
    [B, Ht, N/P, D] ([B, N/P, Ht, D] with token_major_out), lse[r], tlse[r]
    fp32 [B, Ht, N/P], where Ht >= head_base + H is the heads of a slice. Head h
    of the call fills head head_base + h of every slice; other heads are left
    as they are. In Ulysses context parallelism entry r is rank r's memory
    mapped into this process, and the call is the attention plus the output
    all-to-all (include/causaljvp.h, caj_attn_fwd_jvp_scatter: the caller
    orders the ranks around it)."""
    ins = (q, k, v, tq, tk, tv)
    P = len(o)
    if not 1 <= P <= _lib.MAX_SHARDS or not (len(to) == len(lse) == len(tlse) == P):
        raise ValueError(f"attn_fwd_jvp_scatter: o, to, lse, tlse need one entry per slice (1..{_lib.MAX_SHARDS})")
    for t in ins:
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("attn_fwd_jvp_scatter: q..tv must be contiguous CUDA tensors")
    if q.dtype not in _DTYPES or any(t.dtype != q.dtype or t.shape != q.shape for t in ins):
        raise ValueError("attn_fwd_jvp_scatter: q..tv must share one shape and dtype (bf16 or fp32)")
    B, H, N, D = q.shape
    if N % P:
        raise ValueError(f"attn_fwd_jvp_scatter: sequence length {N} is not a multiple of {P} slices")
    Ht = (o[0].shape[2] if token_major_out else o[0].shape[1]) if o[0].dim() == 4 else -1
    Ls = N // P
    out_shape = (B, Ls, Ht, D) if token_major_out else (B, Ht, Ls, D)
    for r in range(P):
        for t in (o[r], to[r], lse[r], tlse[r]):
            if not t.is_cuda:
                raise ValueError(f"attn_fwd_jvp_scatter: slice {r} buffers must be CUDA tensors "
                                 "(the kernel writes them with device stores)")
        for t in (o[r], to[r]):
            if t.dtype != q.dtype or tuple(t.shape) != out_shape or not t.is_contiguous():
                raise ValueError(f"attn_fwd_jvp_scatter: slice {r} output must be contiguous {out_shape}")
        for t in (lse[r], tlse[r]):
            if t.dtype != torch.float32 or tuple(t.shape) != (B, Ht, Ls) or not t.is_contiguous():
                raise ValueError(f"attn_fwd_jvp_scatter: slice {r} lse/tlse must be contiguous fp32 {(B, Ht, Ls)}")
    dst = _lib.SeqScatterC()
    dst.shards, dst.head_base, dst.heads_total = P, int(head_base), Ht
    for r in range(P):
        dst.o[r], dst.to[r] = o[r].data_ptr(), to[r].data_ptr()
        dst.lse[r], dst.tlse[r] = lse[r].data_ptr(), tlse[r].data_ptr()
    s = (stream or torch.cuda.current_stream(q.device)).cuda_stream
    prob = _problem(q, scale, clean_tangent_zero, token_major_out)
    st = _lib.lib().caj_attn_fwd_jvp_scatter(*[ctypes.c_void_p(t.data_ptr()) for t in ins],
                                             ctypes.byref(prob), ctypes.byref(_lib.mask_c(mask)),
                                             ctypes.byref(dst), ctypes.c_void_p(s))
    _lib.check(st, "caj_attn_fwd_jvp_scatter")


def signal_barrier(pads, rank: int, epoch: int, timeout_ms: float = 0.0,
                   stream: Optional[torch.cuda.Stream] = None) -> None:
    """Stream-ordered barrier of the P ranks of a context-parallel group
    (caj_signal_barrier). pads: P device addresses (ints), entry r rank r's pad
    of MAX_SHARDS uint32 words as mapped in this process, zeroed before the
    first call. epoch: the same nonzero value on every rank, larger than any
    earlier one over these pads. A peer that does not arrive within timeout_ms
    (<= 0: the library's wait limit) makes the kernel record a timeout, which
    device_status() raises; the kernel never traps."""
    P = len(pads)
    arr = (ctypes.c_void_p * max(P, 1))(*[int(p) for p in pads])
    s = (stream or torch.cuda.current_stream()).cuda_stream
    st = _lib.lib().caj_signal_barrier(arr, P, int(rank), ctypes.c_uint32(int(epoch) & 0xFFFFFFFF),
                                       float(timeout_ms), ctypes.c_void_p(s))
    _lib.check(st, "caj_signal_barrier")


def ipc_export(t: torch.Tensor) -> bytes:
    """An IPC handle (bytes) through which another process on this node maps
    the device memory of CUDA tensor `t` (caj_ipc_export). `t` must come from
    PyTorch's default cudaMalloc-backed allocator."""
    if not t.is_cuda:
        raise ValueError("ipc_export: a CUDA tensor is needed")
    h = _lib.IpcHandleC()
    _lib.check(_lib.lib().caj_ipc_export(ctypes.c_void_p(t.data_ptr()), ctypes.byref(h)), "caj_ipc_export")
    return bytes(ctypes.string_at(ctypes.addressof(h), ctypes.sizeof(h)))


def ipc_open(handle: bytes) -> int:
    """Maps a handle from ipc_export of ANOTHER process; returns the device
    address of the exported tensor's first byte in this process."""
    h = _lib.IpcHandleC()
    if len(handle) != ctypes.sizeof(h):
        raise ValueError("ipc_open: not a handle from ipc_export")
    ctypes.memmove(ctypes.addressof(h), handle, len(handle))
    p = ctypes.c_void_p(0)
    _lib.check(_lib.lib().caj_ipc_open(ctypes.byref(h), ctypes.byref(p)), "caj_ipc_open")
    return int(p.value)


def ipc_close(address: int) -> None:
    """Unmaps an address returned by ipc_open."""
    _lib.check(_lib.lib().caj_ipc_close(ctypes.c_void_p(int(address))), "caj_ipc_close")


def out_proj_jvp(x, tx, w, bias=None, out=None):
    """Output projection in primal-tangent form (see include/causaljvp.h):
    y = x W^T + bias, ty = tx W^T.

    x, tx: [..., K] bf16 CUDA tensors (e.g. the attention output [B, N, H, D]
    from attn_fwd_jvp(..., token_major_out=True), K = H*D); w: [C, K] bf16;
    bias: [C] bf16 or None. Returns (y, ty) of shape [..., C]."""
    C, K = w.shape
    # rows of K elements: [..., K] or, for the token-major attention output, [..., H, D]
    if x.shape[-1] == K:
        lead = tuple(x.shape[:-1])
    elif x.dim() >= 2 and x.shape[-2] * x.shape[-1] == K:
        lead = tuple(x.shape[:-2])
    else:
        raise ValueError("out_proj_jvp: x's rows must hold the weight's K elements")
    if tx.shape != x.shape or (bias is not None and tuple(bias.shape) != (C,)):
        raise ValueError("out_proj_jvp: shape mismatch")
    for t in (x, tx, w) + ((bias,) if bias is not None else ()):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == torch.bfloat16):
            raise ValueError("out_proj_jvp: tensors must be contiguous bf16 CUDA tensors")
    M = x.numel() // K
    if out is None:
        out = (torch.empty((M, C), dtype=torch.bfloat16, device=x.device),
               torch.empty((M, C), dtype=torch.bfloat16, device=x.device))
    y, ty = out
    shape = _lib.LinearShapeC(M, K, C)
    s = torch.cuda.current_stream(x.device).cuda_stream
    st = _lib.lib().caj_out_proj_jvp(ctypes.c_void_p(x.data_ptr()), ctypes.c_void_p(tx.data_ptr()),
                                     ctypes.c_void_p(w.data_ptr()),
                                     ctypes.c_void_p(bias.data_ptr() if bias is not None else 0),
                                     ctypes.byref(shape), ctypes.c_void_p(y.data_ptr()),
                                     ctypes.c_void_p(ty.data_ptr()), ctypes.c_void_p(s))
    _lib.check(st, "caj_out_proj_jvp")
    return y.view(*lead, C), ty.view(*lead, C)


def qk_norm_rope_jvp(xq, xk, xv, txq, txk, txv, gq, gk, rope_cos, rope_sin, H: int,
                     eps: float = 1e-6, per_head: bool = False, out=None):
    """Attention-block prologue in primal-tangent form (see include/causaljvp.h).

    xq..txv: [B, N, H*D] bf16 CUDA tensors (projection outputs); gq, gk: [H*D]
    fp32 RMSNorm gains; rope_cos, rope_sin: [N, D/2] fp32. Returns
    (q, k, v, tq, tk, tv), each [B, H, N, D] bf16, ready for attn_fwd_jvp.
    """
    ins = (xq, xk, xv, txq, txk, txv)
    B, N, C = xq.shape
    if C % H:
        raise ValueError("qk_norm_rope_jvp: H must divide the channel count")
    D = C // H
    for t in ins:
        if not (t.is_cuda and t.is_contiguous() and t.dtype == torch.bfloat16 and t.shape == xq.shape):
            raise ValueError("qk_norm_rope_jvp: inputs must be contiguous bf16 CUDA tensors of one shape")
    for t, shape in ((gq, (C,)), (gk, (C,)), (rope_cos, (N, D // 2)), (rope_sin, (N, D // 2))):
        if not (t.is_cuda and t.is_contiguous() and t.dtype == torch.float32 and tuple(t.shape) == shape):
            raise ValueError("qk_norm_rope_jvp: gains [H*D] and rope tables [N, D/2] must be fp32 CUDA tensors")
    if out is None:
        out = [torch.empty((B, H, N, D), dtype=torch.bfloat16, device=xq.device) for _ in range(6)]
    shape = _lib.PrologueShapeC(B, N, H, D, float(eps), 1 if per_head else 0)
    s = torch.cuda.current_stream(xq.device).cuda_stream
    st = _lib.lib().caj_qk_norm_rope_jvp(*[ctypes.c_void_p(t.data_ptr()) for t in ins],
                                         *[ctypes.c_void_p(t.data_ptr()) for t in (gq, gk, rope_cos, rope_sin)],
                                         ctypes.byref(shape), *[ctypes.c_void_p(t.data_ptr()) for t in out],
                                         ctypes.c_void_p(s))
    _lib.check(st, "caj_qk_norm_rope_jvp")
    return tuple(out)


def attn_bwd(q, k, v, o, dout, lse, mask, scale: Optional[float] = None):
    """Backward of the primal masked attention (see include/causaljvp.h).

    q, k, v, o, dout: [B, H, N, D] bf16 CUDA tensors (o and lse from
    attn_fwd_jvp on the same q, k, v). Returns (dq, dk, dv, delta) with
    delta = rowsum(dout * o) in fp32 [B, H, N]."""
    ins = (q, k, v, o, dout)
    for t in ins:
        if not (t.is_cuda and t.is_contiguous() and t.dtype == torch.bfloat16 and t.shape == q.shape):
            raise ValueError("attn_bwd: q, k, v, o, dout must be contiguous bf16 CUDA tensors of one shape")
    if not (lse.is_cuda and lse.dtype == torch.float32 and lse.shape == q.shape[:3] and lse.is_contiguous()):
        raise ValueError("attn_bwd: lse must be a contiguous fp32 CUDA tensor [B, H, N]")
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    delta = torch.empty(q.shape[:3], dtype=torch.float32, device=q.device)
    prob = _problem(q, scale)
    s = torch.cuda.current_stream(q.device).cuda_stream
    st = _lib.lib().caj_attn_bwd(*[ctypes.c_void_p(t.data_ptr()) for t in ins],
                                 ctypes.c_void_p(lse.data_ptr()), ctypes.byref(prob),
                                 ctypes.byref(_lib.mask_c(mask)),
                                 *[ctypes.c_void_p(t.data_ptr()) for t in (dq, dk, dv, delta)],
                                 ctypes.c_void_p(s))
    _lib.check(st, "caj_attn_bwd")
    return dq, dk, dv, delta
