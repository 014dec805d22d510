"""ctypes loader for libgdn.so and the raw C-ABI signatures of include/gdn.h.

The library is built in-tree (``build.py``).  Loading never falls back to
anything: if the shared library is missing and cannot be built, or a symbol
is absent, the import fails with an error that says so.
"""
from __future__ import annotations

import ctypes
import os
import threading

from . import build as _build

GDN_OK = 0
GDN_ERR_INVALID_ARG = 1
GDN_ERR_UNSUPPORTED = 2
GDN_ERR_ALIAS = 3
GDN_ERR_CUDA = 4
GDN_ERR_TIMEOUT = 5
GDN_ERR_SCRATCH_LIMIT = 6

GDN_F32 = 0
GDN_BF16 = 1

# name -> (restype, argtypes), mirroring include/gdn.h
_vp, _fp, _i, _ll = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong
_SCAN_ARGS = [_vp, _vp, _vp, _fp, _fp, _fp, _fp, _vp] + [_i] * 5 + [_i, _i, _vp]
_BWD_ARGS = [_vp] * 6 + [_vp, _vp] + [_vp] * 6 + [_i] * 5 + [_i, _vp]
SIGNATURES = {
    "gdn_chunk_fwd_backward": (ctypes.c_int, _BWD_ARGS),
    "gdn_chunk_bidir_backward": (ctypes.c_int, _BWD_ARGS),
    "gdn_chunk_fwd": (ctypes.c_int, _SCAN_ARGS),
    "gdn_chunk_bidir": (ctypes.c_int, _SCAN_ARGS),
    "gdn_chunk_fwd_noalloc": (ctypes.c_int, _SCAN_ARGS),
    "gdn_chunk_fwd_logits": (ctypes.c_int, _SCAN_ARGS),
    "gdn_chunk_bidir_logits": (ctypes.c_int, _SCAN_ARGS),
    "gdn_sink_window_attention": (ctypes.c_int, [_vp] * 6 + [_i] * 8 + [_vp]),
    "gdn_sink_window_slot": (ctypes.c_int, [_i, _i, _i]),
    "gdn_state_reset": (ctypes.c_int, [_fp, _i, _i, _i, _i, _vp]),
    "gdn_device_error": (ctypes.c_int, [_vp]),
    "gdn_workspace_release": (ctypes.c_int, []),
    "gdn_set_wait_limit": (ctypes.c_longlong, [_ll]),
    "gdn_set_time_segments": (ctypes.c_int, [_i]),
    "gdn_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "gdn_version": (ctypes.c_int, []),
    "gdn_launch_count": (ctypes.c_ulonglong, []),
    "gdn_profile_begin": (ctypes.c_int, [ctypes.c_int]),
    "gdn_profile_end": (ctypes.c_int, [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int]),
    "gdn_kernel_name": (ctypes.c_char_p, [ctypes.c_int]),
}

_lock = threading.Lock()
_lib = None


class GDNError(RuntimeError):
    """A non-OK gdn_status returned by the library."""

    def __init__(self, status: int, where: str):
        self.status = int(status)
        name = status_string(status)
        super().__init__(f"{where}: {name} ({status})")


def library_path() -> str:
    return _build.LIB_PATH


def load() -> ctypes.CDLL:
    """Load libgdn.so (building it first if it is missing or stale)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if _build.is_stale():
            try:
                _build.build()
            except Exception as e:  # no silent fallback: the CUDA path is the product
                if not os.path.exists(_build.LIB_PATH):
                    raise RuntimeError(
                        "libgdn.so is missing and could not be built (nvcc for sm_100a "
                        f"is required): {e}") from e
        lib = ctypes.CDLL(_build.LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)  # AttributeError if the symbol is missing
            fn.restype = res
            fn.argtypes = args
        _lib = lib
        return lib


def status_string(status: int) -> str:
    return load().gdn_status_string(int(status)).decode()


def check(status: int, where: str) -> None:
    if status != GDN_OK:
        raise GDNError(status, where)
