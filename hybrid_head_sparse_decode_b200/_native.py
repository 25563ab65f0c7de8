"""ctypes binding to liblychee.so (the C ABI in include/lychee.h).

Argument marshalling only: every step of the decode-attention path runs in the
library's CUDA kernels.  PyTorch is used for device memory and streams; tensors
are passed as raw pointers.  There is no CPU fallback: if the library cannot be
loaded, or a tensor is not on a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch  # noqa: F401  (loads libcudart.so.12 into the process first)

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblychee.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_WORKSPACE = 3
ERR_CUDA = 4
ERR_BAD_INDEX = 5
ERR_TIMEOUT = 6

BF16 = 0
FP32 = 1
ROLE_SPARSE = 0
ROLE_RETRIEVAL = 1

# LYCHEE_NOALLOC_SCRATCH_BYTES of include/lychee.h
NOALLOC_SCRATCH_BYTES = 64 << 20

EXPORTED = ("lychee_workspace_size", "lychee_layer_workspace_size", "lychee_workspace_offsets", "lychee_hybrid_decode_attn",
            "lychee_hybrid_decode_attn_noalloc", "lychee_decode_stack",
            "lychee_check_device_error", "lychee_status_string", "lychee_version",
            "lychee_profile_begin", "lychee_profile_spans_begin", "lychee_profile_end",
            "lychee_append_kv",
            "lychee_hardkuma_roles", "lychee_hybrid_decode_attn_swa", "lychee_decode_stack_swa")


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("d", ctypes.c_int32), ("N_max", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("k", ctypes.c_int32), ("block", ctypes.c_int32)]


class LycheeError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} (status {status})")
        self.status = status


_lock = threading.Lock()
_lib = None


def load(path: str | None = None):
    """Load liblychee.so (built in-tree by hybrid_head_sparse_decode_b200.build)."""
    global _lib
    with _lock:
        if _lib is not None and path is None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"liblychee.so not found at {p}; build it with "
                               "`python -m hybrid_head_sparse_decode_b200.build`")
        lib = ctypes.CDLL(p)
        vp, i32, u32p = ctypes.c_void_p, ctypes.c_int32, ctypes.POINTER(ctypes.c_uint32)
        sp = ctypes.POINTER(Shape)
        lib.lychee_workspace_size.argtypes = [sp]
        lib.lychee_workspace_size.restype = ctypes.c_size_t
        lib.lychee_layer_workspace_size.argtypes = [sp]
        lib.lychee_layer_workspace_size.restype = ctypes.c_size_t
        lib.lychee_workspace_offsets.argtypes = [sp, ctypes.POINTER(ctypes.c_size_t),
                                                 ctypes.POINTER(ctypes.c_size_t),
                                                 ctypes.POINTER(i32)]
        lib.lychee_workspace_offsets.restype = ctypes.c_int
        lib.lychee_hybrid_decode_attn.argtypes = [sp] + [vp] * 10 + [ctypes.c_size_t, vp]
        lib.lychee_hybrid_decode_attn.restype = ctypes.c_int
        lib.lychee_hybrid_decode_attn_noalloc.argtypes = [sp] + [vp] * 11
        lib.lychee_hybrid_decode_attn_noalloc.restype = ctypes.c_int
        lib.lychee_decode_stack.argtypes = [sp, i32] + [vp] * 10 + [ctypes.c_size_t, vp]
        lib.lychee_decode_stack.restype = ctypes.c_int
        lib.lychee_hybrid_decode_attn_swa.argtypes = [sp] + [vp] * 9 + [i32] + [vp] * 4 + [
            ctypes.c_size_t, vp]
        lib.lychee_hybrid_decode_attn_swa.restype = ctypes.c_int
        lib.lychee_decode_stack_swa.argtypes = [sp, i32] + [vp] * 8 + [i32] + [vp] * 5 + [
            ctypes.c_size_t, vp]
        lib.lychee_decode_stack_swa.restype = ctypes.c_int
        lib.lychee_append_kv.argtypes = [sp] + [vp] * 6
        lib.lychee_append_kv.restype = ctypes.c_int
        lib.lychee_hardkuma_roles.argtypes = [vp, vp, i32, i32, ctypes.c_double, ctypes.c_double,
                                              i32, vp, vp, vp, vp]
        lib.lychee_hardkuma_roles.restype = ctypes.c_int
        lib.lychee_check_device_error.argtypes = [vp, vp, u32p]
        lib.lychee_check_device_error.restype = ctypes.c_int
        lib.lychee_status_string.argtypes = [ctypes.c_int]
        lib.lychee_status_string.restype = ctypes.c_char_p
        lib.lychee_version.argtypes = []
        lib.lychee_version.restype = i32
        lib.lychee_profile_begin.argtypes = [i32]
        lib.lychee_profile_begin.restype = ctypes.c_int
        lib.lychee_profile_spans_begin.argtypes = [i32]
        lib.lychee_profile_spans_begin.restype = ctypes.c_int
        lib.lychee_profile_end.argtypes = [i32, vp, vp, ctypes.POINTER(i32)]
        lib.lychee_profile_end.restype = ctypes.c_int
        if path is None:
            _lib = lib
        return lib


def status_string(status: int) -> str:
    try:
        return load().lychee_status_string(int(status)).decode()
    except Exception:  # the library itself failed to load
        return f"status {status}"
