"""ctypes view of libsdpa_b200.so (the C ABI in include/sdpa_b200.h).

Argument marshalling only.  The library is loaded from this package's
directory; if it is missing, every call raises -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsdpa_b200.so")

ATTN_OK = 0
STATUS_NAMES = {
    0: "ATTN_OK", 1: "ATTN_ERR_NULL", 2: "ATTN_ERR_SHAPE", 3: "ATTN_ERR_GQA", 4: "ATTN_ERR_HEADDIM",
    5: "ATTN_ERR_ALIGN", 6: "ATTN_ERR_CAUSAL", 7: "ATTN_ERR_WORKSPACE", 8: "ATTN_ERR_CUDA",
    9: "ATTN_ERR_DEVICE_TIMEOUT", 10: "ATTN_ERR_ARCH", 11: "ATTN_ERR_SCALE", 12: "ATTN_ERR_SCRATCH_LIMIT",
    13: "ATTN_ERR_SEQLEN",
}
STATIC_SCRATCH_BYTES = 16 << 20
EXPORTS = ("attn_fwd", "attn_fwd_ex", "attn_fwd_varlen", "attn_decode_num_splits", "attn_decode_workspace_size", "attn_decode_splitkv",
           "attn_decode_splitkv_varlen", "attn_decode_splitkv_ex", "attn_decode_splitkv_static", "attn_rope_append", "attn_bwd", "attn_bwd_workspace_size",
           "attn_selftest_decode_wait_timeout", "attn_status_string",
           "attn_check_device_error", "attn_version")

class Extras(ctypes.Structure):
    """attn_extras_t of the C ABI."""
    _fields_ = [("seqlens_q", ctypes.c_void_p), ("seqlens_k", ctypes.c_void_p), ("bias", ctypes.c_void_p),
                ("bias_b", ctypes.c_int), ("bias_h", ctypes.c_int), ("layout", ctypes.c_int)]


_lock = threading.Lock()
_lib = None


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        name = STATUS_NAMES.get(status, str(status))
        try:
            msg = get().attn_status_string(status).decode()
        except Exception:  # pragma: no cover - message only
            msg = ""
        super().__init__(f"{where}: {name} ({msg})")


def _declare(lib):
    P, I, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.attn_fwd.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, P]
    lib.attn_fwd.restype = I
    EP = ctypes.POINTER(Extras)
    lib.attn_fwd_ex.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, EP, P]
    lib.attn_fwd_ex.restype = I
    lib.attn_decode_splitkv_ex.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, I, P, SZ, EP, P]
    lib.attn_decode_splitkv_ex.restype = I
    lib.attn_fwd_varlen.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P]
    lib.attn_fwd_varlen.restype = I
    lib.attn_decode_num_splits.argtypes = [I, I, I, I, I, I]
    lib.attn_decode_num_splits.restype = I
    lib.attn_decode_workspace_size.argtypes = [I, I, I, I, I, I, I]
    lib.attn_decode_workspace_size.restype = SZ
    lib.attn_decode_splitkv.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, I, P, SZ, P]
    lib.attn_decode_splitkv.restype = I
    lib.attn_decode_splitkv_varlen.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, F, I, I, P, SZ, P]
    lib.attn_decode_splitkv_varlen.restype = I
    lib.attn_decode_splitkv_static.argtypes = [P, P, P, P, P, I, I, I, I, I, I, F, I, I, P]
    lib.attn_decode_splitkv_static.restype = I
    lib.attn_rope_append.argtypes = [P, P, P, I, P, P, P, P, P, I, I, I, I, I, I, I, P]
    lib.attn_rope_append.restype = I
    lib.attn_bwd.argtypes = [P, P, P, P, P, P, P, P, P, I, I, I, I, I, I, F, I, P, SZ, P]
    lib.attn_bwd.restype = I
    lib.attn_bwd_workspace_size.argtypes = [I, I, I]
    lib.attn_bwd_workspace_size.restype = SZ
    lib.attn_selftest_decode_wait_timeout.argtypes = [P, P, P, P, P, I, I, I, I, I, I, P, SZ, P]
    lib.attn_selftest_decode_wait_timeout.restype = I
    lib.attn_status_string.argtypes = [I]
    lib.attn_status_string.restype = ctypes.c_char_p
    lib.attn_check_device_error.argtypes = [P]
    lib.attn_check_device_error.restype = I
    lib.attn_version.argtypes = []
    lib.attn_version.restype = I
    return lib


def get():
    """The loaded library; raises if the CUDA extension has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with `python -m scaled_dot_product_fa2_b200.build` "
                    "(there is no CPU fallback)")
            _lib = _declare(ctypes.CDLL(LIB_PATH))
    return _lib


def check(status: int, where: str) -> None:
    if status != ATTN_OK:
        raise AttnError(status, where)
