"""ctypes mirror of include/gdn.h and the loader of libgdn.so.

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  There is no CPU fallback; if libgdn.so is missing or cannot be loaded
the import of the binding's entry points raises.
"""
from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")

GDN_ABI_VERSION = 1
GDN_CHUNK = 64
GDN_F32, GDN_BF16 = 0, 1
GDN_FLAG_SPLIT_OFF = 1 << 0
GDN_FLAG_SPLIT_FORCE = 1 << 1
GDN_FLAG_PORTABLE = 1 << 2
GDN_FLAG_GATE_LOGITS = 1 << 3
GDN_FLAG_QK_L2NORM = 1 << 4

STATUS = {
    0: "GDN_OK",
    1: "GDN_ERR_INVALID_ARG",
    2: "GDN_ERR_UNSUPPORTED",
    3: "GDN_ERR_WORKSPACE",
    4: "GDN_ERR_CUDA",
    5: "GDN_ERR_TIMEOUT",
    6: "GDN_ERR_DEVICE",
    7: "GDN_ERR_TOO_LARGE",
}

_u32, _i32, _p = ctypes.c_uint32, ctypes.c_int32, ctypes.c_void_p

_COMMON = [
    ("struct_size", _u32), ("abi_version", _u32), ("dtype", _i32),
    ("B", _i32), ("T", _i32), ("Hk", _i32), ("Hv", _i32), ("dk", _i32), ("dv", _i32),
    ("num_seqs", _i32), ("flags", _u32),
    ("q", _p), ("k", _p), ("v", _p), ("beta", _p), ("g", _p),
    ("cu_seqlens", _p), ("cu_seqlens_host", _p), ("S0", _p),
]


class GdnFwdArgs(ctypes.Structure):
    _fields_ = _COMMON + [("o", _p), ("ST", _p), ("dev_status", _p)]


class GdnBwdArgs(ctypes.Structure):
    _fields_ = _COMMON + [
        ("dout", _p), ("dST", _p), ("dq", _p), ("dk_out", _p), ("dv_out", _p),
        ("dbeta", _p), ("dg", _p), ("dS0", _p), ("dev_status", _p),
    ]


class GdnDecodeArgs(ctypes.Structure):
    _fields_ = [
        ("struct_size", _u32), ("abi_version", _u32), ("dtype", _i32), ("N", _i32),
        ("Hk", _i32), ("Hv", _i32), ("dk", _i32), ("dv", _i32), ("num_slots", _i32),
        ("flags", _u32), ("q", _p), ("k", _p), ("v", _p), ("beta", _p), ("g", _p), ("S", _p),
        ("state_indices", _p), ("o", _p), ("dev_status", _p),
    ]


class GdnCombineArgs(ctypes.Structure):
    _fields_ = [
        ("struct_size", _u32), ("abi_version", _u32), ("N", _i32), ("Hv", _i32), ("dk", _i32),
        ("dv", _i32), ("M", _p), ("B", _p), ("X", _p),
    ]


class GdnHaloArgs(ctypes.Structure):
    _fields_ = [
        ("struct_size", _u32), ("abi_version", _u32), ("dtype", _i32), ("T", _i32), ("Hk", _i32),
        ("Hv", _i32), ("dk", _i32), ("flags", _u32), ("log_eps", ctypes.c_float), ("k", _p),
        ("beta", _p), ("g", _p), ("ok", _p), ("log_decay", _p),
    ]


EXPORTS = [
    "gdn_chunk_fwd_workspace_size", "gdn_chunk_fwd", "gdn_chunk_fwd_launch_count",
    "gdn_chunk_bwd_workspace_size", "gdn_chunk_bwd", "gdn_chunk_bwd_launch_count",
    "gdn_status_string", "gdn_chunk_fwd_noalloc", "gdn_decode_step", "gdn_affine_combine",
    "gdn_halo_check",
]

_lib = None


class GdnError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS.get(status, status)} ({status_string(status)})")


def lib() -> ctypes.CDLL:
    """Load libgdn.so (raises if it was not built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"libgdn.so not built at {LIB_PATH}; run "
                              "`python -m gated_deltanet_chunked_fwd_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        sz = ctypes.POINTER(ctypes.c_size_t)
        F, Bw = ctypes.POINTER(GdnFwdArgs), ctypes.POINTER(GdnBwdArgs)
        L.gdn_chunk_fwd_workspace_size.argtypes = [F, sz]
        L.gdn_chunk_fwd.argtypes = [F, _p, ctypes.c_size_t, _p]
        L.gdn_chunk_fwd_launch_count.argtypes = [F]
        L.gdn_chunk_bwd_workspace_size.argtypes = [Bw, sz]
        L.gdn_chunk_bwd.argtypes = [Bw, _p, ctypes.c_size_t, _p]
        L.gdn_chunk_bwd_launch_count.argtypes = [Bw]
        for fn in ("gdn_chunk_fwd_workspace_size", "gdn_chunk_fwd", "gdn_chunk_bwd_workspace_size",
                   "gdn_chunk_bwd", "gdn_chunk_fwd_launch_count", "gdn_chunk_bwd_launch_count"):
            getattr(L, fn).restype = ctypes.c_int
        L.gdn_decode_step.argtypes = [ctypes.POINTER(GdnDecodeArgs), _p]
        L.gdn_decode_step.restype = ctypes.c_int
        L.gdn_affine_combine.argtypes = [ctypes.POINTER(GdnCombineArgs), _p]
        L.gdn_affine_combine.restype = ctypes.c_int
        L.gdn_halo_check.argtypes = [ctypes.POINTER(GdnHaloArgs), _p]
        L.gdn_halo_check.restype = ctypes.c_int
        L.gdn_chunk_fwd_noalloc.argtypes = [F, _p]
        L.gdn_chunk_fwd_noalloc.restype = ctypes.c_int
        L.gdn_status_string.argtypes = [ctypes.c_int]
        L.gdn_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().gdn_status_string(int(status)).decode()
