"""ctypes declarations of the cskv C ABI (include/cskv.h).

Loads ``libcskv.so`` from this package directory.  There is no fallback: if the
library is missing or does not load, every call raises.
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libcskv.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_WORKSPACE, ERR_LAUNCH = 0, 1, 2, 3, 4
F32, BF16, FP8E4M3 = 0, 1, 2
OVERLAP_PREVIOUS = 1  # csa_compress flags (CSKV_OVERLAP_PREVIOUS)
ATTN_PAIRS = 0x100  # OR-ed into hybrid_decode_attn's mode (CSKV_ATTN_PAIRS)
ATTN_KV_FP8 = 0x200  # OR-ed into hybrid_decode_attn's mode (CSKV_ATTN_KV_FP8)
KV8_ROW_BYTES = 336  # CSKV_KV8_ROW_BYTES
CSA, HCA = 0, 1
DEV_BAD_INDEX, DEV_TAIL_MISSING, DEV_CAPACITY, DEV_TIMEOUT = 1, 2, 4, 8
NOALLOC_SCRATCH_BYTES = 16 << 20

_p = ctypes.c_void_p
_i32 = ctypes.c_int
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t
_f = ctypes.c_float

SIGNATURES = {
    "cskv_status_string": (ctypes.c_char_p, [_i32]),
    "cskv_last_cuda_error": (ctypes.c_char_p, []),
    "cskv_version": (_i32, []),
    "cskv_launch_count": (ctypes.c_ulonglong, []),
    "cskv_copy_segments": (_i32, [_p, _p, _p, _p, _i32, _p]),
    "cskv_mapped_pointer": (_i32, [_p, _p]),
    "csa_compress": (_i32, [_p, _p, _p, _p, _p, _p, _p, _p, _i32, _p, _p, _p, _i64, _i32, _i32, _p,
                            _i32, _p, _f, _p, _i32, _i32, _p, _p, _i32, _p, _p]),
    "hca_compress": (_i32, [_p, _p, _p, _p, _p, _i32, _p, _p, _p, _i64, _i32, _i32, _p, _i32, _p, _f, _p, _p]),
    "rmsnorm_heads": (_i32, [_p, _i32, _i64, _i32, _p, _f, _p, _p]),
    "kv_quantize_fp8": (_i32, [_p, _i32, _i64, _p, _p]),
    "lindex_pool_keys": (_i32, [_p, _i32, _i32, _p, _p, _i32, _p, _p, _p, _i64, _p, _p, _p, _p]),
    "lindex_score_topk": (_i32, [_p, _p, _p, _p, _p, _p, _p, _p, _i32, _i32, _i32, _i32, _i32, _i32, _i64,
                                 _p, _p, _p, _i64, _p, _sz, _p, _p]),
    "lindex_score_topk_mxfp4": (_i32, [_p, _p, _p, _p, _p, _p, _p, _p, _p, _i32, _i32, _i32, _i32, _i32, _i64,
                                       _p, _p, _p, _i64, _p, _sz, _p, _p]),
    "lindex_topk_from_scores": (_i32, [_p, _i64, _p, _i32, _i32, _i64, _p, _p, _p, _sz, _p, _p]),
    "lindex_workspace_size": (_sz, [_i32, _i32, _i64]),
    "lindex_workspace_size_scan": (_sz, [_i32, _i64]),
    "hybrid_decode_attn": (_i32, [_i32, _p, _p, _p, _p, _i32, _p, _p, _p, _i32, _p, _f, _p, _p, _i32, _i32,
                                  _i32, _i32, _i32, _i64, _p, _p, _p, _sz, _p, _p]),
    "hybrid_attn_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32, _i64]),
    "hybrid_decode_attn_noalloc": (_i32, [_i32, _p, _p, _p, _p, _i32, _p, _p, _p, _i32, _p, _f, _p, _p, _i32,
                                          _i32, _i32, _i32, _i32, _i64, _p, _p, _p, _p]),
}

_lib = None


def load() -> ctypes.CDLL:
    """The loaded library (raises if it is not built or does not load)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m compressed_sparse_kv_compress_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class CskvError(RuntimeError):
    def __init__(self, fn: str, status: int):
        lib = load()
        msg = lib.cskv_status_string(status).decode()
        if status == ERR_LAUNCH:
            msg += f" ({lib.cskv_last_cuda_error().decode()})"
        super().__init__(f"{fn}: {msg}")
        self.status = status


def check(fn: str, status: int) -> None:
    if status != OK:
        raise CskvError(fn, status)
