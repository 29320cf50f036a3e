"""ctypes view of the C ABI in include/attn_jvp.h (marshalling only)."""
from __future__ import annotations

import ctypes
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libattn_jvp.so")
HEADER_PATH = os.path.join(os.path.dirname(_PKG), "include", "attn_jvp.h")

OK = 0
ERR_INVALID_ARGUMENT = 1
ERR_UNSUPPORTED = 2
ERR_MISALIGNED = 3
ERR_CUDA = 4
ERR_DEVICE_TIMEOUT = 5
ERR_NO_DEVICE = 6

DTYPE_BF16 = 0
DTYPE_F32 = 1


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("L", ctypes.c_int64), ("H", ctypes.c_int64),
                ("d", ctypes.c_int64), ("dtype", ctypes.c_int32), ("scale", ctypes.c_float)]


class Mask(ctypes.Structure):
    _fields_ = [("mode", ctypes.c_int32), ("chunk_tokens", ctypes.c_int32),
                ("n_chunks", ctypes.c_int32)]


MAX_GROUPS = 512


class Group(ctypes.Structure):
    _fields_ = [("row_end", ctypes.c_int32), ("k0_begin", ctypes.c_int32),
                ("k0_end", ctypes.c_int32), ("k1_begin", ctypes.c_int32),
                ("k1_end", ctypes.c_int32)]


def group_array(groups):
    """A ctypes array of Group from (row_end, k0_begin, k0_end, k1_begin, k1_end) tuples."""
    arr = (Group * max(1, len(groups)))()
    for i, g in enumerate(groups):
        arr[i] = Group(*(int(x) for x in g))
    return arr


_lib = None
_lock = threading.Lock()


def load(path: str = None) -> ctypes.CDLL:
    """Load the in-tree CUDA library (or the library at `path`, e.g. the trace
    build, which then serves every later call); raise if it is missing."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        path = path or os.environ.get("ATTN_JVP_LIB") or LIB_PATH
        if not os.path.exists(path):
            raise RuntimeError(
                f"CUDA library not built: {path} is missing "
                "(run `python -m attention_jvp_attn_b200.build`)")
        lib = ctypes.CDLL(path)
        vp = ctypes.c_void_p
        lib.attn_jvp_fwd.argtypes = [ctypes.POINTER(Shape), vp, vp, vp, vp, vp, vp, Mask,
                                     vp, vp, vp, vp]
        lib.attn_jvp_fwd.restype = ctypes.c_int
        lib.attn_jvp_fwd_host.argtypes = [ctypes.POINTER(Shape), vp, vp, vp, vp, vp, vp, Mask,
                                          vp, vp, vp, vp, vp]
        lib.attn_jvp_fwd_host.restype = ctypes.c_int
        lib.attn_jvp_host_staging_bytes.argtypes = [ctypes.POINTER(Shape)]
        lib.attn_jvp_host_staging_bytes.restype = ctypes.c_int64
        lib.attn_jvp_sync_status.argtypes = [vp]
        lib.attn_jvp_sync_status.restype = ctypes.c_int
        lib.attn_jvp_status_string.argtypes = [ctypes.c_int]
        lib.attn_jvp_status_string.restype = ctypes.c_char_p
        lib.attn_jvp_unmasked_pairs.argtypes = [Mask]
        lib.attn_jvp_unmasked_pairs.restype = ctypes.c_int64
        lib.attn_jvp_schedule_tiles.argtypes = [Mask, ctypes.c_int64, ctypes.c_int32,
                                                ctypes.c_int32, ctypes.c_int32,
                                                ctypes.POINTER(ctypes.c_int32),
                                                ctypes.POINTER(ctypes.c_uint8), ctypes.c_int32]
        lib.attn_jvp_schedule_tiles.restype = ctypes.c_int32
        lib.attn_jvp_key_tile_query_bounds.argtypes = [
            Mask, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
            ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_int32)]
        lib.attn_jvp_key_tile_query_bounds.restype = ctypes.c_int32
        lib.attn_jvp_fwd_noalloc.argtypes = [ctypes.POINTER(Shape), vp, vp, vp, vp, vp, vp,
                                             Mask, vp, vp, vp, vp]
        lib.attn_jvp_fwd_noalloc.restype = ctypes.c_int
        lib.attn_jvp_fwd_groups.argtypes = [ctypes.POINTER(Shape), vp, vp, vp, vp, vp, vp,
                                            ctypes.POINTER(Group), ctypes.c_int32, vp, vp, vp, vp]
        lib.attn_jvp_fwd_groups.restype = ctypes.c_int
        lib.attn_jvp_schedule_tiles_groups.argtypes = [
            ctypes.POINTER(Group), ctypes.c_int32, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32,
            ctypes.c_int32, ctypes.POINTER(ctypes.c_int32), ctypes.POINTER(ctypes.c_uint8),
            ctypes.c_int32]
        lib.attn_jvp_schedule_tiles_groups.restype = ctypes.c_int32
        lib.attn_jvp_bwd.argtypes = [ctypes.POINTER(Shape), vp, vp, vp, vp, vp, vp, vp, Mask,
                                     vp, vp, vp, vp]
        lib.attn_jvp_bwd.restype = ctypes.c_int
        lib.attn_jvp_bwd_groups.argtypes = [ctypes.POINTER(Shape), vp, vp, vp, vp, vp, vp, vp,
                                            ctypes.POINTER(Group), ctypes.c_int32, vp, vp, vp,
                                            vp]
        lib.attn_jvp_bwd_groups.restype = ctypes.c_int
        lib.attn_jvp_rope.argtypes = [ctypes.POINTER(Shape), vp, vp, vp, vp, vp, vp, vp, vp,
                                      vp, vp, vp]
        lib.attn_jvp_rope.restype = ctypes.c_int
        lib.attn_jvp_fwd_rope.argtypes = [ctypes.POINTER(Shape), vp, vp, vp, vp, vp, vp, vp, vp,
                                          Mask, vp, vp, vp, vp, vp, vp, vp, vp]
        lib.attn_jvp_fwd_rope.restype = ctypes.c_int
        lib.attn_jvp_debug_wait.argtypes = [ctypes.c_int64, ctypes.c_int32]
        lib.attn_jvp_debug_wait.restype = ctypes.c_int
        lib.attn_jvp_version.argtypes = []
        lib.attn_jvp_version.restype = ctypes.c_int32
        _lib = lib
        return lib


def status_string(code: int) -> str:
    return load().attn_jvp_status_string(code).decode()


class AttnJvpError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: status {code} ({status_string(code)})")


def check(code: int, where: str) -> None:
    if code != OK:
        raise AttnJvpError(code, where)
