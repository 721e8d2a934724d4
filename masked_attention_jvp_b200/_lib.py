"""ctypes binding of libcausaljvp (include/causaljvp.h). Argument marshalling only:
every step of the computation runs in the library's CUDA kernels."""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcausaljvp.so")

CAJ_OK, CAJ_ERR_INVALID_ARG, CAJ_ERR_UNSUPPORTED, CAJ_ERR_CUDA, CAJ_ERR_DEVICE_TIMEOUT = range(5)
CAJ_DTYPE_F32, CAJ_DTYPE_BF16 = 0, 1

# Every symbol include/causaljvp.h declares.
EXPORTED = [
    "caj_attn_fwd_jvp", "caj_last_device_status", "caj_last_device_error_code",
    "caj_status_string", "caj_last_cuda_error", "caj_validate_mask", "caj_visible_pairs",
    "caj_row_key_ranges", "caj_qtile_key_tiles", "caj_version", "caj_set_wait_timeout_ms",
    "caj_debug_set_fault", "caj_qk_norm_rope_jvp", "caj_key_query_ranges", "caj_ktile_query_tiles",
    "caj_attn_bwd", "caj_attn_fwd_jvp_host_workspace", "caj_attn_fwd_jvp_host", "caj_out_proj_jvp",
    "caj_attn_fwd_jvp_scatter", "caj_attn_fwd_jvp_host_static", "caj_signal_barrier",
    "caj_ipc_export", "caj_ipc_open", "caj_ipc_close", "caj_attn_fwd_jvp_part", "caj_part_query_tiles",
]


MAX_SHARDS = 8  # CAJ_MAX_SHARDS
HOST_STATIC_MAX_BYTES = 64 << 20  # CAJ_HOST_STATIC_MAX_BYTES


class SeqScatterC(ctypes.Structure):
    _fields_ = [("shards", ctypes.c_int32), ("head_base", ctypes.c_int32), ("heads_total", ctypes.c_int32),
                ("o", ctypes.c_void_p * MAX_SHARDS), ("to", ctypes.c_void_p * MAX_SHARDS),
                ("lse", ctypes.c_void_p * MAX_SHARDS), ("tlse", ctypes.c_void_p * MAX_SHARDS)]


class IpcHandleC(ctypes.Structure):
    _fields_ = [("handle", ctypes.c_ubyte * 64), ("offset", ctypes.c_uint64)]


class LinearShapeC(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int64), ("K", ctypes.c_int32), ("C", ctypes.c_int32)]


class MaskDescC(ctypes.Structure):
    _fields_ = [("tokens_per_frame", ctypes.c_int32), ("frames_per_chunk", ctypes.c_int32),
                ("n_frames", ctypes.c_int32), ("tf_layout", ctypes.c_int32)]


class ProblemC(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32),
                ("D", ctypes.c_int32), ("dtype", ctypes.c_int32), ("scale", ctypes.c_float),
                ("flags", ctypes.c_int32)]


CAJ_FLAG_CLEAN_TANGENT_ZERO = 1
CAJ_FLAG_TOKEN_MAJOR_OUT = 2


class PrologueShapeC(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("N", ctypes.c_int32), ("H", ctypes.c_int32),
                ("D", ctypes.c_int32), ("eps", ctypes.c_float), ("norm_per_head", ctypes.c_int32)]


class CajError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(msg)
        self.status = status


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library. Raises if the CUDA extension has not been built:
    there is no fallback implementation."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(
                f"libcausaljvp.so is missing at {LIB_PATH}; build it with "
                "`python -m masked_attention_jvp_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
        L.caj_attn_fwd_jvp.argtypes = [vp] * 6 + [ctypes.POINTER(ProblemC), ctypes.POINTER(MaskDescC),
                                                  vp, vp, vp, vp, vp]
        L.caj_attn_fwd_jvp.restype = ctypes.c_int
        L.caj_last_device_status.argtypes = [vp]
        L.caj_last_device_status.restype = ctypes.c_int
        L.caj_last_device_error_code.argtypes = []
        L.caj_last_device_error_code.restype = ctypes.c_uint32
        L.caj_status_string.argtypes = [ctypes.c_int]
        L.caj_status_string.restype = ctypes.c_char_p
        L.caj_last_cuda_error.argtypes = []
        L.caj_last_cuda_error.restype = ctypes.c_char_p
        L.caj_validate_mask.argtypes = [ctypes.POINTER(MaskDescC), i32]
        L.caj_validate_mask.restype = ctypes.c_int
        L.caj_visible_pairs.argtypes = [ctypes.POINTER(MaskDescC)]
        L.caj_visible_pairs.restype = i64
        L.caj_row_key_ranges.argtypes = [ctypes.POINTER(MaskDescC), i32, ctypes.POINTER(i32)]
        L.caj_row_key_ranges.restype = ctypes.c_int
        L.caj_qtile_key_tiles.argtypes = [ctypes.POINTER(MaskDescC), i32, i32, i32, ctypes.POINTER(i32)]
        L.caj_qtile_key_tiles.restype = i32
        L.caj_set_wait_timeout_ms.argtypes = [ctypes.c_double]
        L.caj_set_wait_timeout_ms.restype = ctypes.c_int
        L.caj_debug_set_fault.argtypes = [ctypes.c_int32]
        L.caj_debug_set_fault.restype = ctypes.c_int
        L.caj_qk_norm_rope_jvp.argtypes = [vp] * 10 + [ctypes.POINTER(PrologueShapeC)] + [vp] * 7
        L.caj_qk_norm_rope_jvp.restype = ctypes.c_int
        L.caj_key_query_ranges.argtypes = [ctypes.POINTER(MaskDescC), i32, ctypes.POINTER(i32)]
        L.caj_key_query_ranges.restype = ctypes.c_int
        L.caj_ktile_query_tiles.argtypes = [ctypes.POINTER(MaskDescC), i32, i32, i32, ctypes.POINTER(i32)]
        L.caj_ktile_query_tiles.restype = i32
        L.caj_attn_bwd.argtypes = [vp] * 6 + [ctypes.POINTER(ProblemC), ctypes.POINTER(MaskDescC)] + [vp] * 5
        L.caj_attn_bwd.restype = ctypes.c_int
        L.caj_attn_fwd_jvp_host_workspace.argtypes = [ctypes.POINTER(ProblemC), ctypes.POINTER(ctypes.c_size_t)]
        L.caj_attn_fwd_jvp_host_workspace.restype = ctypes.c_int
        L.caj_attn_fwd_jvp_host.argtypes = [vp] * 6 + [ctypes.POINTER(ProblemC), ctypes.POINTER(MaskDescC)] + \
            [vp] * 5 + [ctypes.c_size_t, vp]
        L.caj_attn_fwd_jvp_host.restype = ctypes.c_int
        L.caj_attn_fwd_jvp_host_static.argtypes = [vp] * 6 + [ctypes.POINTER(ProblemC),
                                                    ctypes.POINTER(MaskDescC)] + [vp] * 5
        L.caj_attn_fwd_jvp_host_static.restype = ctypes.c_int
        L.caj_out_proj_jvp.argtypes = [vp] * 4 + [ctypes.POINTER(LinearShapeC), vp, vp, vp]
        L.caj_out_proj_jvp.restype = ctypes.c_int
        L.caj_attn_fwd_jvp_scatter.argtypes = [vp] * 6 + [ctypes.POINTER(ProblemC), ctypes.POINTER(MaskDescC),
                                                ctypes.POINTER(SeqScatterC), vp]
        L.caj_attn_fwd_jvp_scatter.restype = ctypes.c_int
        L.caj_signal_barrier.argtypes = [ctypes.POINTER(vp), i32, i32, ctypes.c_uint32, ctypes.c_double, vp]
        L.caj_signal_barrier.restype = ctypes.c_int
        L.caj_ipc_export.argtypes = [vp, ctypes.POINTER(IpcHandleC)]
        L.caj_ipc_export.restype = ctypes.c_int
        L.caj_ipc_open.argtypes = [ctypes.POINTER(IpcHandleC), ctypes.POINTER(vp)]
        L.caj_ipc_open.restype = ctypes.c_int
        L.caj_ipc_close.argtypes = [vp]
        L.caj_ipc_close.restype = ctypes.c_int
        L.caj_attn_fwd_jvp_part.argtypes = [vp] * 6 + [ctypes.POINTER(ProblemC), ctypes.POINTER(MaskDescC),
                                                 i32, i32] + [vp] * 5
        L.caj_attn_fwd_jvp_part.restype = ctypes.c_int
        L.caj_part_query_tiles.argtypes = [ctypes.POINTER(MaskDescC), i32, i32, ctypes.POINTER(i32), i32]
        L.caj_part_query_tiles.restype = i32
        L.caj_version.argtypes = []
        L.caj_version.restype = i32
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().caj_status_string(status).decode()


def check(status: int, what: str = "caj_attn_fwd_jvp"):
    if status != CAJ_OK:
        msg = f"{what}: {status_string(status)}"
        if status == CAJ_ERR_CUDA:
            msg += f" ({lib().caj_last_cuda_error().decode()})"
        if status == CAJ_ERR_DEVICE_TIMEOUT:
            msg += f" (device code {lib().caj_last_device_error_code():#x})"
        raise CajError(status, msg)


def mask_c(mask) -> MaskDescC:
    t = mask.as_tuple() if hasattr(mask, "as_tuple") else tuple(mask)
    return MaskDescC(*[int(x) for x in t])
