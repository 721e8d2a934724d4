"""Host-side checks of libcausaljvp that need no GPU: the library loads and
exports every symbol its header declares, the closed-form mask / tile schedule
matches brute force over the oracle's independent visibility rule, and argument
validation rejects bad calls before anything is launched."""
import ctypes
import os
import random
import re

import pytest
import torch

import oracle
import masked_attention_jvp_b200 as caj
from masked_attention_jvp_b200 import _lib
from masked_attention_jvp_b200.workloads import MaskDesc, WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MASKS = [MaskDesc(3, 1, 4, 0), MaskDesc(2, 2, 4, 0), MaskDesc(3, 1, 3, 1), MaskDesc(2, 3, 6, 1),
         MaskDesc(1, 1, 7, 0), MaskDesc(5, 1, 1, 0), MaskDesc(37, 1, 5, 1), MaskDesc(100, 1, 3, 0),
         MaskDesc(13, 3, 6, 1), MaskDesc(64, 1, 4, 1), MaskDesc(1, 1, 130, 1)]



# Calls whose arguments pass validation reach the device check: on a machine
# without a GPU they stop there (CAJ_ERR_CUDA); elsewhere they would launch
# with the fake pointers these tests use, so they run only without a GPU.
_NO_GPU = not torch.cuda.is_available()

def test_header_symbols_are_exported():
    hdr = open(os.path.join(ROOT, "include", "causaljvp.h")).read()
    declared = sorted(set(re.findall(r"\b(caj_[a-z_]+)\s*\(", hdr)))
    assert declared == sorted(_lib.EXPORTED)
    L = _lib.lib()
    for name in declared:
        assert hasattr(L, name), name


def test_version_and_status_strings():
    assert _lib.lib().caj_version() >= 100
    names = [_lib.status_string(i) for i in range(5)]
    assert names == ["CAJ_OK", "CAJ_ERR_INVALID_ARG", "CAJ_ERR_UNSUPPORTED", "CAJ_ERR_CUDA",
                     "CAJ_ERR_DEVICE_TIMEOUT"]
    assert _lib.status_string(99) == "CAJ_ERR_UNKNOWN"


@pytest.mark.parametrize("mask", MASKS)
def test_visible_pairs_matches_brute_force(mask):
    assert caj.visible_pairs(mask) == oracle.visible_pairs(mask)


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_visible_pairs_of_the_workloads(name):
    w = WORKLOADS[name]
    m = w.mask
    G, n = m.frames_per_chunk * m.tokens_per_frame, m.n_frames // m.frames_per_chunk
    half = G * G * n * (n + 1) // 2
    assert caj.visible_pairs(m) == (2 * half if m.tf_layout else half)


@pytest.mark.parametrize("mask", MASKS)
def test_row_ranges_match_oracle_visibility(mask):
    N = mask.seq_len
    for i in range(N):
        (a0, b0), (a1, b1) = caj.row_key_ranges(mask, i)
        got = set(range(a0, b0)) | set(range(a1, b1))
        want = {j for j in range(N) if oracle.visible(mask, i, j)}
        assert got == want, (mask, i)


@pytest.mark.parametrize("mask", MASKS)
@pytest.mark.parametrize("bm,bn", [(128, 64), (16, 8), (7, 5), (32, 64)])
def test_query_tile_schedule_matches_brute_force(mask, bm, bn):
    """The kernel visits exactly the key tiles some row of the query tile can see."""
    N = mask.seq_len
    for q0 in range(0, N, bm):
        q1 = min(q0 + bm, N)
        n, (t0, t1), (t2, t3) = caj.qtile_key_tiles(mask, q0, q1, bn)
        assert t0 <= t1 <= t2 <= t3
        tiles = list(range(t0, t1)) + list(range(t2, t3))
        assert n == len(tiles)
        want = sorted({j // bn for i in range(q0, q1) for j in range(N) if oracle.visible(mask, i, j)})
        assert tiles == want, (mask, q0, q1, bn)


@pytest.mark.parametrize("name", [n for n in WORKLOADS if n != "tiny_framewise_fp32"])
def test_schedule_at_full_size_covers_every_row(name):
    """At the workloads' sizes: every row's key ranges lie inside its tile's
    visited tiles, and the visited tiles hold no tile that no row needs (sampled)."""
    m = WORKLOADS[name].mask
    N = m.seq_len
    rng = random.Random(5)
    tiles_q = list(range((N + 127) // 128))
    for qt in rng.sample(tiles_q, 40) + [0, len(tiles_q) - 1]:
        q0, q1 = qt * 128, min(qt * 128 + 128, N)
        n, (t0, t1), (t2, t3) = caj.qtile_key_tiles(m, q0, q1, 64)
        tiles = set(range(t0, t1)) | set(range(t2, t3))
        needed = set()
        for i in range(q0, q1):
            (a0, b0), (a1, b1) = caj.row_key_ranges(m, i)
            for a, b in ((a0, b0), (a1, b1)):
                if b > a:
                    needed |= set(range(a // 64, (b + 63) // 64))
        assert tiles == needed


def _call(q=0x10000, o=0x20000, lse=0x30000, prob=None, mask=None):
    prob = prob or _lib.ProblemC(1, 2, 64, 64, _lib.CAJ_DTYPE_BF16, 0.0, 0)
    mask = mask or _lib.MaskDescC(16, 1, 4, 0)
    vp = ctypes.c_void_p
    return _lib.lib().caj_attn_fwd_jvp(vp(q), vp(q), vp(q), vp(q), vp(q), vp(q),
                                       ctypes.byref(prob), ctypes.byref(mask),
                                       vp(o), vp(o), vp(lse), vp(lse), vp(0))


def test_argument_validation_launches_nothing():
    P, M = _lib.ProblemC, _lib.MaskDescC
    bf = _lib.CAJ_DTYPE_BF16
    INV, UNS = _lib.CAJ_ERR_INVALID_ARG, _lib.CAJ_ERR_UNSUPPORTED
    assert _call(q=0) == INV                                   # null input
    assert _call(q=0x10008) == INV                             # misaligned input
    assert _call(o=0x20004) == INV                             # misaligned output
    assert _call(lse=0x30002) == INV                           # misaligned lse
    assert _call(prob=P(1, 2, 65, 64, bf, 0.0)) == INV         # N != mask length
    assert _call(prob=P(0, 2, 64, 64, bf, 0.0)) == INV         # empty batch
    assert _call(prob=P(1, 2, 64, 64, 7, 0.0)) == INV          # unknown dtype
    assert _call(prob=P(1, 2, 64, 64, bf, -1.0)) == INV        # negative scale
    assert _call(prob=P(1, 2, 64, 64, bf, float("nan"))) == INV
    assert _call(mask=M(16, 3, 4, 0)) == INV                   # frames % chunk != 0
    assert _call(mask=M(16, 1, 4, 2)) == INV                   # bad layout flag
    assert _call(mask=M(0, 1, 4, 0)) == INV                    # empty frame
    if _NO_GPU:  # would launch with these fake pointers on a GPU machine
        assert _call(prob=P(1, 2, 128, 64, bf, 0.0), mask=M(16, 1, 4, 1)) != INV  # TF: N = 2L
    assert _call(prob=P(1, 2, 64, 96, bf, 0.0)) == UNS         # head dim not built
    assert _call(prob=P(700, 100, 64, 64, bf, 0.0)) == UNS     # too many heads
    assert _call(prob=P(1, 2, 64, 64, bf, 0.0, 1)) == INV      # clean-tangent flag needs TF layout
    assert _call(prob=P(1, 2, 64, 64, bf, 0.0, 4)) == INV      # unknown flag bit
    if _NO_GPU:  # would launch with these fake pointers on a GPU machine
        assert _call(prob=P(1, 2, 128, 64, bf, 0.0, 1), mask=M(16, 1, 4, 1)) != INV


def _ws_bytes(prob):
    n = ctypes.c_size_t(0)
    st = _lib.lib().caj_attn_fwd_jvp_host_workspace(ctypes.byref(prob), ctypes.byref(n))
    return st, n.value


def test_host_workspace_size():
    """Six inputs, O and tO of the problem's element size plus LSE and tLSE in
    fp32, each region rounded up to 256 bytes."""
    P = _lib.ProblemC
    up = lambda x: (x + 255) // 256 * 256
    for B, H, N, D, dt, es in [(1, 12, 65520, 128, _lib.CAJ_DTYPE_BF16, 2), (2, 3, 77, 64, _lib.CAJ_DTYPE_F32, 4),
                               (1, 1, 1, 64, _lib.CAJ_DTYPE_BF16, 2)]:
        st, n = _ws_bytes(P(B, H, N, D, dt, 0.0))
        assert st == _lib.CAJ_OK
        assert n == 8 * up(B * H * N * D * es) + 2 * up(B * H * N * 4)
    assert _ws_bytes(P(1, 2, 64, 64, 7, 0.0))[0] == _lib.CAJ_ERR_INVALID_ARG   # unknown dtype
    assert _ws_bytes(P(0, 2, 64, 64, 1, 0.0))[0] == _lib.CAJ_ERR_INVALID_ARG   # empty batch
    n = ctypes.c_size_t(0)
    assert _lib.lib().caj_attn_fwd_jvp_host_workspace(None, ctypes.byref(n)) == _lib.CAJ_ERR_INVALID_ARG


def _host_call(workspace, nbytes, prob=None, mask=None, q=0x1000):
    prob = prob or _lib.ProblemC(1, 2, 64, 64, _lib.CAJ_DTYPE_BF16, 0.0)
    mask = mask or _lib.MaskDescC(16, 1, 4, 0)
    vp = ctypes.c_void_p
    return _lib.lib().caj_attn_fwd_jvp_host(vp(q), vp(q), vp(q), vp(q), vp(q), vp(q), ctypes.byref(prob),
                                            ctypes.byref(mask), vp(q), vp(q), vp(q), vp(q),
                                            vp(workspace), nbytes, vp(0))


def test_host_entry_validation_copies_nothing():
    """Bad arguments are refused before any copy is enqueued (these pointers are
    never dereferenced)."""
    INV, UNS = _lib.CAJ_ERR_INVALID_ARG, _lib.CAJ_ERR_UNSUPPORTED
    _, need = _ws_bytes(_lib.ProblemC(1, 2, 64, 64, _lib.CAJ_DTYPE_BF16, 0.0))
    assert _host_call(0, need) == INV                     # no workspace
    assert _host_call(0x100080, need) == INV              # workspace not 256-byte aligned
    assert _host_call(0x100000, need - 1) == INV          # workspace too small
    assert _host_call(0x100000, need, q=0) == INV         # null input
    assert _host_call(0x100000, need, mask=_lib.MaskDescC(16, 1, 5, 0)) == INV   # N != mask length
    assert _host_call(0x100000, 1 << 40, prob=_lib.ProblemC(1, 2, 64, 96, _lib.CAJ_DTYPE_BF16, 0.0)) == UNS


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_valid_call_without_gpu_reports_cuda_error():
    assert _call() == _lib.CAJ_ERR_CUDA
    assert len(_lib.lib().caj_last_cuda_error()) > 0


def test_mask_queries_reject_bad_arguments():
    M = _lib.MaskDescC
    L = _lib.lib()
    assert L.caj_validate_mask(ctypes.byref(M(16, 1, 4, 0)), 64) == _lib.CAJ_OK
    assert L.caj_validate_mask(ctypes.byref(M(16, 1, 4, 1)), 64) == _lib.CAJ_ERR_INVALID_ARG
    assert L.caj_visible_pairs(ctypes.byref(M(16, 2, 3, 0))) == -1
    r = (ctypes.c_int32 * 4)()
    assert L.caj_row_key_ranges(ctypes.byref(M(4, 1, 2, 0)), 8, r) == _lib.CAJ_ERR_INVALID_ARG
    assert L.caj_qtile_key_tiles(ctypes.byref(M(4, 1, 2, 0)), 4, 4, 64, r) == -1
    assert L.caj_qtile_key_tiles(ctypes.byref(M(4, 1, 2, 0)), 0, 9, 64, r) == -1


def test_flops_count():
    m = WORKLOADS["wan1.3b_tf_framewise"].mask
    assert caj.flops(1, 12, 128, m) == 12 * 128 * 1_124_323_200 * 12


def test_timeout_and_fault_hooks_host_side():
    L = _lib.lib()
    assert L.caj_set_wait_timeout_ms(250.0) == _lib.CAJ_OK
    assert L.caj_set_wait_timeout_ms(0.0) == _lib.CAJ_OK
    assert L.caj_debug_set_fault(2) == _lib.CAJ_ERR_INVALID_ARG
    assert L.caj_debug_set_fault(1) == _lib.CAJ_OK
    assert L.caj_debug_set_fault(0) == _lib.CAJ_OK


def test_prologue_validation_launches_nothing():
    L = _lib.lib()
    S = _lib.PrologueShapeC
    vp = ctypes.c_void_p

    def call(shape, ptr=0x10000, g=0x20000):
        return L.caj_qk_norm_rope_jvp(*[vp(ptr)] * 6, vp(g), vp(g), vp(g), vp(g), ctypes.byref(shape),
                                      *[vp(ptr)] * 6, vp(0))
    assert call(S(1, 8, 12, 128, 1e-6, 0), ptr=0) == _lib.CAJ_ERR_INVALID_ARG
    assert call(S(1, 8, 12, 128, 1e-6, 0), ptr=0x10008) == _lib.CAJ_ERR_INVALID_ARG
    assert call(S(1, 8, 12, 128, 1e-6, 0), g=0x20004) == _lib.CAJ_ERR_INVALID_ARG
    assert call(S(1, 8, 12, 128, -1.0, 0)) == _lib.CAJ_ERR_INVALID_ARG
    assert call(S(1, 8, 12, 128, 1e-6, 2)) == _lib.CAJ_ERR_INVALID_ARG
    assert call(S(0, 8, 12, 128, 1e-6, 0)) == _lib.CAJ_ERR_INVALID_ARG
    assert call(S(1, 8, 12, 96, 1e-6, 0)) == _lib.CAJ_ERR_UNSUPPORTED
    assert call(S(1, 8, 3, 64, 1e-6, 0)) == _lib.CAJ_ERR_UNSUPPORTED     # H*D not a multiple of 256
    assert call(S(1, 8, 128, 128, 1e-6, 0)) == _lib.CAJ_ERR_UNSUPPORTED  # H*D > 8192


@pytest.mark.parametrize("mask", MASKS)
def test_key_ranges_match_oracle_visibility(mask):
    """The transposed mask: queries that see each key, against brute force."""
    L = _lib.lib()
    N = mask.seq_len
    r = (ctypes.c_int32 * 4)()
    for j in range(N):
        assert L.caj_key_query_ranges(ctypes.byref(_lib.mask_c(mask)), j, r) == _lib.CAJ_OK
        got = set(range(r[0], r[1])) | set(range(r[2], r[3]))
        want = {i for i in range(N) if oracle.visible(mask, i, j)}
        assert got == want, (mask, j)


@pytest.mark.parametrize("mask", MASKS)
@pytest.mark.parametrize("bk,bq", [(128, 64), (16, 8), (7, 5), (64, 128)])
def test_key_tile_schedule_matches_brute_force(mask, bk, bq):
    """The key-major backward visits exactly the query tiles that see some key of the tile."""
    L = _lib.lib()
    N = mask.seq_len
    t = (ctypes.c_int32 * 6)()
    for k0 in range(0, N, bk):
        k1 = min(k0 + bk, N)
        n = L.caj_ktile_query_tiles(ctypes.byref(_lib.mask_c(mask)), k0, k1, bq, t)
        tiles = list(range(t[0], t[1])) + list(range(t[2], t[3])) + list(range(t[4], t[5]))
        assert t[0] <= t[1] <= t[2] <= t[3] <= t[4] <= t[5]
        assert n == len(tiles)
        want = sorted({i // bq for j in range(k0, k1) for i in range(N) if oracle.visible(mask, i, j)})
        assert tiles == want, (mask, k0, k1, bk, bq)


def test_out_proj_validation_launches_nothing():
    vp = ctypes.c_void_p
    L = _lib.lib()
    INV, UNS = _lib.CAJ_ERR_INVALID_ARG, _lib.CAJ_ERR_UNSUPPORTED

    def call(M=64, K=128, C=256, x=0x1000, bias=0, y=0x2000):
        shape = _lib.LinearShapeC(M, K, C)
        return L.caj_out_proj_jvp(vp(x), vp(x), vp(x), vp(bias), ctypes.byref(shape), vp(y), vp(y), vp(0))

    assert call(M=0) == INV                  # no rows
    assert call(K=0) == INV
    assert call(K=100) == UNS                # rows not whole 16-byte units
    assert call(C=36) == UNS
    assert call(x=0) == INV                  # null input
    assert call(x=0x1008) == INV             # misaligned input
    assert call(bias=0x3004) == INV          # misaligned bias
    assert L.caj_out_proj_jvp(vp(1), vp(1), vp(1), vp(0), None, vp(1), vp(1), vp(0)) == INV


def test_token_major_flag_validation():
    P, M = _lib.ProblemC, _lib.MaskDescC
    bf, tm, ctz = _lib.CAJ_DTYPE_BF16, _lib.CAJ_FLAG_TOKEN_MAJOR_OUT, _lib.CAJ_FLAG_CLEAN_TANGENT_ZERO
    if _NO_GPU:  # would launch with these fake pointers on a GPU machine
        assert _call(prob=P(1, 2, 64, 64, bf, 0.0, tm)) != _lib.CAJ_ERR_INVALID_ARG      # accepted
    if _NO_GPU:  # would launch with these fake pointers on a GPU machine
        assert _call(prob=P(1, 2, 128, 64, bf, 0.0, tm | ctz), mask=M(16, 1, 4, 1)) != _lib.CAJ_ERR_INVALID_ARG
    assert _call(prob=P(1, 2, 64, 64, bf, 0.0, 8)) == _lib.CAJ_ERR_INVALID_ARG       # unknown bit
    # the host-buffer form copies head-major chunks only
    _, need = _ws_bytes(P(1, 2, 64, 64, bf, 0.0))
    assert _host_call(0x100000, need, prob=P(1, 2, 64, 64, bf, 0.0, tm)) == _lib.CAJ_ERR_INVALID_ARG


def _scatter_call(shards=2, head_base=0, heads_total=4, prob=None, mask=None, o=0x20000, lse=0x30000,
                  null_slice=None):
    prob = prob or _lib.ProblemC(1, 2, 64, 64, _lib.CAJ_DTYPE_BF16, 0.0, 0)
    mask = mask or _lib.MaskDescC(16, 1, 4, 0)
    d = _lib.SeqScatterC()
    d.shards, d.head_base, d.heads_total = shards, head_base, heads_total
    for r in range(_lib.MAX_SHARDS):
        step = 0 if r == null_slice else 1
        d.o[r], d.to[r] = step * (o + 0x1000 * r), step * (o + 0x1000 * r + 0x800)
        d.lse[r], d.tlse[r] = step * (lse + 0x1000 * r), step * (lse + 0x1000 * r + 0x800)
    vp = ctypes.c_void_p
    return _lib.lib().caj_attn_fwd_jvp_scatter(*[vp(0x10000)] * 6, ctypes.byref(prob), ctypes.byref(mask),
                                               ctypes.byref(d), vp(0))


def test_scatter_validation_launches_nothing():
    P = _lib.ProblemC
    bf, INV = _lib.CAJ_DTYPE_BF16, _lib.CAJ_ERR_INVALID_ARG
    vp = ctypes.c_void_p
    L = _lib.lib()
    prob, mask = P(1, 2, 64, 64, bf, 0.0, 0), _lib.MaskDescC(16, 1, 4, 0)
    assert L.caj_attn_fwd_jvp_scatter(*[vp(0x10000)] * 6, ctypes.byref(prob), ctypes.byref(mask),
                                      None, vp(0)) == INV                    # no descriptor
    assert _scatter_call(shards=0) == INV                                    # no slice
    assert _scatter_call(shards=_lib.MAX_SHARDS + 1) == INV                  # more slices than the map holds
    assert _scatter_call(shards=3) == INV                                    # 64 rows do not split in 3
    assert _scatter_call(head_base=-1) == INV                                # head range below 0
    assert _scatter_call(head_base=3, heads_total=4) == INV                  # heads 3, 4 of 4
    assert _scatter_call(heads_total=1) == INV                               # fewer heads than the call
    assert _scatter_call(o=0x20008) == INV                                   # misaligned O slice
    assert _scatter_call(lse=0x30002) == INV                                 # misaligned LSE slice
    assert _scatter_call(null_slice=1) == INV                                # a used slice is null
    if _NO_GPU:  # would launch with these fake pointers on a GPU machine
        assert _scatter_call(shards=1, null_slice=1) != INV                      # an unused one may be
    assert _scatter_call(prob=P(1, 2, 64, 64, bf, 0.0, 1)) == INV            # clean-tangent needs TF
    assert _scatter_call(prob=P(1, 2, 64, 96, bf, 0.0)) == _lib.CAJ_ERR_UNSUPPORTED
    for ok in (dict(shards=8, head_base=2), dict(shards=4, heads_total=2),
               dict(prob=P(1, 2, 64, 64, bf, 0.0, _lib.CAJ_FLAG_TOKEN_MAJOR_OUT))):
        if _NO_GPU:  # would launch with these fake pointers on a GPU machine
            assert _scatter_call(**ok) != INV, ok


def test_signal_barrier_validation_launches_nothing():
    L = _lib.lib()
    INV = _lib.CAJ_ERR_INVALID_ARG
    vp = ctypes.c_void_p

    def call(pads, shards, rank, epoch):
        arr = (vp * max(len(pads), 1))(*pads)
        return L.caj_signal_barrier(arr, shards, rank, epoch, 0.0, vp(0))

    assert L.caj_signal_barrier(None, 1, 0, 1, 0.0, vp(0)) == INV         # no pad list
    assert call([0x1000], 0, 0, 1) == INV                                  # no rank
    assert call([0x1000] * 9, 9, 0, 1) == INV                              # more ranks than a pad holds
    assert call([0x1000, 0x2000], 2, 2, 1) == INV                          # rank out of range
    assert call([0x1000, 0x2000], 2, -1, 1) == INV
    assert call([0x1000, 0x2000], 2, 0, 0) == INV                          # epoch 0 is the pads' start value
    assert call([0x1000, 0], 2, 0, 1) == INV                               # null pad
    assert call([0x1000, 0x2002], 2, 0, 1) == INV                          # misaligned pad
    if _NO_GPU:
        assert call([0x1000, 0x2000], 2, 1, 7) == _lib.CAJ_ERR_CUDA        # valid: stops at the device check


def test_ipc_entry_points_validate_without_a_gpu():
    L = _lib.lib()
    INV = _lib.CAJ_ERR_INVALID_ARG
    h = _lib.IpcHandleC()
    p = ctypes.c_void_p(0)
    assert L.caj_ipc_export(None, ctypes.byref(h)) == INV
    assert L.caj_ipc_export(ctypes.c_void_p(0x1000), None) == INV
    assert L.caj_ipc_open(None, ctypes.byref(p)) == INV
    assert L.caj_ipc_open(ctypes.byref(h), None) == INV
    assert L.caj_ipc_close(ctypes.c_void_p(0x1000)) == INV          # never opened here
    assert L.caj_ipc_close(None) == INV
    assert ctypes.sizeof(_lib.IpcHandleC) == 72


@pytest.mark.parametrize("mask", [MaskDesc(1560, 1, 21, 1), MaskDesc(1560, 3, 21, 1), MaskDesc(3600, 1, 21, 0),
                                  MaskDesc(37, 1, 7, 1), MaskDesc(5, 1, 3, 1)])
def test_parts_deal_every_query_tile_once_and_balance_the_work(mask):
    """caj_part_query_tiles: the parts of one call cover every 128-row query
    tile exactly once, each part's work (visited key tiles) is within one
    tile's work of every other part's, and each part is in heaviest-first
    order; one part is the whole call."""
    N = mask.seq_len
    n_tiles = (N + 127) // 128
    cost = {t: caj.qtile_key_tiles(mask, 128 * t, min(128 * t + 128, N))[0] for t in range(n_tiles)}
    whole = caj.part_query_tiles(mask, 0, 1)
    assert sorted(whole) == list(range(n_tiles))
    for nparts in (2, 3, 4, 8):
        parts = [caj.part_query_tiles(mask, r, nparts) for r in range(nparts)]
        assert sorted(t for p in parts for t in p) == list(range(n_tiles))
        loads = [sum(cost[t] for t in p) for p in parts]
        assert max(loads) - min(loads) <= max(cost.values())
        for p in parts:
            assert [cost[t] for t in p] == sorted((cost[t] for t in p), reverse=True)


def test_part_entry_validation_launches_nothing():
    L = _lib.lib()
    INV, UNS = _lib.CAJ_ERR_INVALID_ARG, _lib.CAJ_ERR_UNSUPPORTED
    vp = ctypes.c_void_p
    mask = _lib.MaskDescC(16, 1, 4, 0)

    def call(part, nparts, dtype=_lib.CAJ_DTYPE_BF16):
        prob = _lib.ProblemC(1, 2, 64, 64, dtype, 0.0, 0)
        return L.caj_attn_fwd_jvp_part(*[vp(0x10000)] * 6, ctypes.byref(prob), ctypes.byref(mask), part, nparts,
                                       vp(0x20000), vp(0x20000), vp(0x30000), vp(0x30000), vp(0))

    assert call(0, 0) == INV
    assert call(2, 2) == INV
    assert call(-1, 2) == INV
    assert call(0, 2, _lib.CAJ_DTYPE_F32) == UNS          # the fp32 path runs whole calls only
    assert L.caj_part_query_tiles(ctypes.byref(mask), 1, 1, None, 0) == -1
    assert L.caj_part_query_tiles(None, 0, 1, None, 0) == -1
    if _NO_GPU:
        assert call(1, 2) == _lib.CAJ_ERR_CUDA             # valid: stops at the device check
