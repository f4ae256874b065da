"""ctypes binding of libs3r.so (include/s3r.h). Argument marshalling only.

The library is loaded from this package directory; there is no fallback of any kind. If it is
missing, or a compute call is made without a CUDA device, the call raises.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libs3r.so")

S3R_OK = 0
S3R_ERR_INVALID_ARG = 1
S3R_ERR_UNSUPPORTED = 2
S3R_ERR_WORKSPACE = 3
S3R_ERR_CUDA = 4
S3R_ERR_TIMEOUT = 5

S3R_DEV_TIMEOUT = 0x1
S3R_DEV_BAD_INDEX = 0x2
S3R_FLAG_DEBUG_CHECKS = 0x1
S3R_FLAG_TEST_TIMEOUT = 0x2
S3R_FLAG_SINGLE_KERNEL = 0x4
S3R_FLAG_SAVE_FOR_BWD = 0x8
S3R_FLAG_NVTX = 0x10
S3R_MAX_BLOCKS = 49152
S3R_STATIC_WORKSPACE_BYTES = 32 << 20
STAGES = ("pool", "cmp", "topk", "sel_combine")  # S3R_STAGE_* order
BWD_STAGES = ("recompute", "prep", "dq", "dkv_cmp", "dkv_sel")  # S3R_BWD_STAGE_* order

# every function the header declares, with its ctypes signature
_P = ctypes.c_void_p
EXPORTS = {
    "s3r_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "s3r_version": (ctypes.c_int, []),
    "s3r_kernel_launches": (ctypes.c_uint64, []),
    "s3r_workspace_bytes": (ctypes.c_size_t, [_P]),
    "s3r_num_key_blocks": (ctypes.c_int64, [_P]),
    "s3r_read_device_status": (ctypes.c_int, [_P, _P, _P]),
    "s3r_workspace_status_word": (_P, [_P]),
    "s3r_last_device_error": (ctypes.c_int, [_P, _P]),
    "s3r_compress_kv": (ctypes.c_int, [_P, _P, _P, _P, _P, _P]),
    "s3r_cmp_attn_and_score": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "s3r_topk_blocks": (ctypes.c_int, [_P, _P, _P, _P]),
    "s3r_sel_attn": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P]),
    "s3r_gate_combine": (ctypes.c_int, [_P, _P, _P, _P, _P, _P]),
    "s3r_sparse_attn_fwd": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "s3r_sparse_attn_fwd_static": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "s3r_bwd_workspace_bytes": (ctypes.c_size_t, [_P]),
    "s3r_sparse_attn_bwd": (ctypes.c_int, [_P] * 12 + [ctypes.c_size_t, _P]),
}


class Params(ctypes.Structure):
    """Mirror of s3r_params."""

    _fields_ = [
        ("L", ctypes.c_int64),
        ("H", ctypes.c_int32),
        ("d", ctypes.c_int32),
        ("block", ctypes.c_int32),
        ("qblock", ctypes.c_int32),
        ("topk", ctypes.c_int32),
        ("scale", ctypes.c_float),
        ("flags", ctypes.c_uint32),
        ("forced", ctypes.c_int32),
        ("grid_h", ctypes.c_int32),
        ("grid_w", ctypes.c_int32),
        ("special", ctypes.c_int32),
        ("win_h", ctypes.c_int32),
        ("dev_status", ctypes.c_void_p),
        ("stage_events", ctypes.c_void_p),
    ]


class S3RError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} returned {status_string(status)}")


_lib = None


def load():
    """Load libs3r.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libs3r.so not found at {LIB_PATH}; build it with "
                "`python -m sparse_global_attention_s3r_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in EXPORTS.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def status_string(status: int) -> str:
    return load().s3r_status_string(int(status)).decode()


def check(fn: str, status: int) -> None:
    if status != S3R_OK:
        raise S3RError(fn, status)


def call(name: str, *args) -> None:
    """Call an entry point that returns s3r_status; raise on any error."""
    check(name, getattr(load(), name)(*args))


def kernel_launches() -> int:
    return int(load().s3r_kernel_launches())
