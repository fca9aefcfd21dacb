"""ctypes binding of libst_attn.so: the C ABI declared in include/st_attn.h, same names.

Argument marshalling only.  Every step of the attention path runs in the library's kernels;
there is no Python or CPU fallback, and loading fails loudly when the library is missing.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libst_attn.so")

ST_OK = 0
ST_ERR_DEVICE_TIMEOUT = 7
STATUS_NAMES = {
    0: "ST_OK", 1: "ST_ERR_INVALID_ARG", 2: "ST_ERR_UNSUPPORTED", 3: "ST_ERR_ALIGNMENT",
    4: "ST_ERR_NOT_UPLOADED", 5: "ST_ERR_CUDA", 6: "ST_ERR_OOM", 7: "ST_ERR_DEVICE_TIMEOUT",
    8: "ST_ERR_WORKSPACE", 9: "ST_ERR_INTERNAL",
}
ST_STRIDED, ST_FIXED = 1, 2
ST_PER_HEAD_ALTERNATING, ST_MERGED, ST_SINGLE_A1, ST_SINGLE_A2 = 1, 2, 3, 4
ST_BF16, ST_FP32 = 1, 2
ST_KIND_SA1, ST_KIND_SA2, ST_KIND_SU, ST_KIND_FA1, ST_KIND_FA2, ST_KIND_FU = 1, 2, 3, 4, 5, 6

# every symbol include/st_attn.h declares
EXPORTED = (
    "st_layout_build", "st_layout_upload", "st_layout_head_kind", "st_layout_export",
    "st_layout_info", "st_layout_exec_row", "st_layout_check", "st_selftest_wait_timeout",
    "st_layout_destroy",
    "st_attn_fwd_workspace_bytes", "st_attn_bwd_workspace_bytes", "st_attn_fwd", "st_attn_bwd",
    "st_attn_bwd_prepare", "st_attn_bwd_main", "st_attn_bwd_finish", "st_attn_bwd_noalloc",
    "st_attn_decode_workspace_bytes", "st_attn_decode", "st_decode_row_keys",
    "st_status_string", "st_version",
)


class StError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


class st_pattern_t(ctypes.Structure):
    _fields_ = [("family", ctypes.c_int32), ("head_mode", ctypes.c_int32),
                ("num_heads", ctypes.c_int32), ("a2_offset_step", ctypes.c_int32)]


class st_desc_t(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("heads", ctypes.c_int64), ("n", ctypes.c_int64),
                ("d", ctypes.c_int64), ("dtype", ctypes.c_int32), ("dv", ctypes.c_int32)]


class st_layout_info_t(ctypes.Structure):
    _fields_ = [("fwd_items", ctypes.c_int64), ("exec_tiles", ctypes.c_int64),
                ("bwd_items", ctypes.c_int64), ("allowed_pairs", ctypes.c_int64),
                ("passes", ctypes.c_int32), ("split_passes", ctypes.c_int32),
                ("dq_direct_heads", ctypes.c_int32), ("reserved", ctypes.c_int32)]


_lib = None


def load() -> ctypes.CDLL:
    """Load libst_attn.so (building it first when it is missing or older than its sources)."""
    global _lib
    if _lib is not None:
        return _lib
    from . import build as _build
    if _build._stale():
        if not os.path.exists(_build.NVCC):
            raise RuntimeError(f"{LIB_PATH} is missing or stale and nvcc is not available")
        _build.build()
    lib = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    i32, i64, sz = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    pp = ctypes.POINTER
    lib.st_layout_build.argtypes = [pp(st_pattern_t), i64, i32, i32, i32, pp(P)]
    lib.st_layout_upload.argtypes = [P, P]
    lib.st_layout_head_kind.argtypes = [P, i32, pp(i32), pp(i32)]
    lib.st_layout_export.argtypes = [P, i32, pp(P), pp(P), pp(P), pp(P), pp(i32), pp(i32), pp(i32)]
    lib.st_layout_info.argtypes = [P, pp(st_layout_info_t)]
    lib.st_layout_exec_row.argtypes = [P, i32, i64, P, pp(i64)]
    lib.st_layout_check.argtypes = [P, P]
    lib.st_selftest_wait_timeout.argtypes = [P, P]
    lib.st_layout_destroy.argtypes = [P]
    lib.st_layout_destroy.restype = None
    lib.st_attn_fwd_workspace_bytes.argtypes = [pp(st_desc_t), P]
    lib.st_attn_fwd_workspace_bytes.restype = sz
    lib.st_attn_bwd_workspace_bytes.argtypes = [pp(st_desc_t), P]
    lib.st_attn_bwd_workspace_bytes.restype = sz
    lib.st_attn_fwd.argtypes = [P, P, P, P, P, P, P, sz, pp(st_desc_t), P]
    lib.st_attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, P, P, sz, pp(st_desc_t), P]
    lib.st_attn_bwd_prepare.argtypes = [P, P, P, P, P, P, sz, pp(st_desc_t), P]
    lib.st_attn_bwd_main.argtypes = [P, P, P, P, P, P, P, P, P, P, sz, pp(st_desc_t), P]
    lib.st_attn_bwd_finish.argtypes = [P, P, P, sz, pp(st_desc_t), P]
    lib.st_attn_bwd_noalloc.argtypes = [P, P, P, P, P, P, P, P, P, P, pp(st_desc_t), P]
    lib.st_attn_bwd_noalloc.restype = i32
    lib.st_attn_decode_workspace_bytes.argtypes = [pp(st_desc_t), P]
    lib.st_attn_decode_workspace_bytes.restype = sz
    lib.st_attn_decode.argtypes = [P, P, P, P, i64, P, P, P, sz, pp(st_desc_t), P]
    lib.st_decode_row_keys.argtypes = [P, i32, i64, P, pp(i64)]
    lib.st_status_string.argtypes = [i32]
    lib.st_status_string.restype = ctypes.c_char_p
    lib.st_version.restype = ctypes.c_char_p
    for name in ("st_layout_build", "st_layout_upload", "st_layout_head_kind", "st_layout_export",
                 "st_layout_info", "st_layout_exec_row", "st_layout_check", "st_selftest_wait_timeout",
                 "st_attn_fwd",
                 "st_attn_bwd", "st_attn_bwd_prepare", "st_attn_bwd_main", "st_attn_bwd_finish",
                 "st_attn_decode", "st_decode_row_keys"):
        getattr(lib, name).restype = i32
    _lib = lib
    return lib


def check(status: int, where: str) -> None:
    if status != ST_OK:
        raise StError(status, where)
