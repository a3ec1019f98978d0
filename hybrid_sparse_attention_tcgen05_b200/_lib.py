"""ctypes loader for libhysparse.so (the C ABI declared in include/hysparse.h).

No fallback: if the library is missing or cannot be loaded, every call raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhysparse.so")

# hs_status
HS_OK = 0
HS_ERR_INVALID_ARG = 1
HS_ERR_UNSUPPORTED = 2
HS_ERR_WORKSPACE = 3
HS_ERR_CUDA = 4
HS_ERR_INVALID_INDEX = 5
HS_ERR_TIMEOUT = 6

# hs_dtype
HS_F32 = 0
HS_BF16 = 1

EXPORTS = (
    "hysparse_workspace_size",
    "hysparse_full_attn_scores",
    "hysparse_topk",
    "hysparse_sparse_attn",
    "hysparse_sparse_attn_own_window",
    "hysparse_block_own_window",
    "hysparse_block",
    "hysparse_block_varlen",
    "hysparse_block_paged",
    "hysparse_full_attn_scores_noalloc",
    "hysparse_workspace_status",
    "hysparse_probe_l2_read",
    "hysparse_launch_count",
    "hysparse_status_string",
    "hysparse_version",
)


class HsShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("Lq", ctypes.c_int), ("Lkv", ctypes.c_int),
                ("Hq", ctypes.c_int), ("Hkv", ctypes.c_int), ("d", ctypes.c_int),
                ("dtype", ctypes.c_int), ("scale", ctypes.c_float)]


class HysparseError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} (status {status})")


_lib = None


def lib():
    """Load libhysparse.so once; raise if it is not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m hybrid_sparse_attention_tcgen05_b200.build` (there is no fallback path)")
    L = ctypes.CDLL(LIB_PATH)
    P, I, LL, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t
    SP = ctypes.POINTER(HsShape)
    L.hysparse_workspace_size.argtypes = [SP, I, I, I, I]
    L.hysparse_workspace_size.restype = SZ
    L.hysparse_full_attn_scores.argtypes = [SP, P, P, P, P, P, P, LL, I, I, P, SZ, P]
    L.hysparse_full_attn_scores.restype = I
    L.hysparse_topk.argtypes = [SP, P, LL, I, I, I, P, P]
    L.hysparse_topk.restype = I
    L.hysparse_sparse_attn.argtypes = [SP, P, P, P, P, I, P, I, P, P, P, P, SZ, P]
    L.hysparse_sparse_attn.restype = I
    L.hysparse_sparse_attn_own_window.argtypes = [SP, P, P, P, P, P, I, P, I, P, I, P, P, P, P, SZ, P]
    L.hysparse_sparse_attn_own_window.restype = I
    L.hysparse_block.argtypes = [SP, P, P, P, P, P, I, P, P, P, I, I, P, I, P, SZ, P]
    L.hysparse_block.restype = I
    L.hysparse_block_own_window.argtypes = [SP, P, P, P, P, P, I, P, P, P, P, I, P, I, I, P, I, P, SZ, P]
    L.hysparse_block_own_window.restype = I
    L.hysparse_block_varlen.argtypes = [SP, P, P, P, P, P, P, I, P, P, P, I, I, P, P, SZ, P]
    L.hysparse_block_varlen.restype = I
    L.hysparse_block_paged.argtypes = [SP, P, P, I, I, I, P, P, P, P, P, I, P, P, P, I, I, P, P, SZ, P]
    L.hysparse_block_paged.restype = I
    L.hysparse_full_attn_scores_noalloc.argtypes = [SP, P, P, P, P, P, P, LL, I, I, P]
    L.hysparse_full_attn_scores_noalloc.restype = I
    L.hysparse_probe_l2_read.argtypes = [P, SZ, I, I, I, P, P]
    L.hysparse_probe_l2_read.restype = I
    L.hysparse_launch_count.argtypes = []
    L.hysparse_launch_count.restype = ctypes.c_ulonglong
    L.hysparse_workspace_status.argtypes = [P, P]
    L.hysparse_workspace_status.restype = I
    L.hysparse_status_string.argtypes = [I]
    L.hysparse_status_string.restype = ctypes.c_char_p
    L.hysparse_version.argtypes = []
    L.hysparse_version.restype = ctypes.c_char_p
    _lib = L
    return L


def status_string(status: int) -> str:
    try:
        return lib().hysparse_status_string(int(status)).decode()
    except Exception:  # library missing: still say something useful
        return f"status {status}"


def check(status: int, what: str) -> None:
    if status != HS_OK:
        raise HysparseError(status, what)
