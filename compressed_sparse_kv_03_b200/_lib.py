"""ctypes binding of the C ABI in include/csa.h (argument marshalling only).

Every step of the hot path runs in the CUDA library; this module only checks
tensor dtypes / devices / shapes, passes data pointers and the current
stream, and turns non-zero status codes into exceptions.  There is no CPU
fallback: if the library is missing, loading fails loudly.
"""
from __future__ import annotations

import ctypes as C
import os

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "_csa_b200.so")

CSA_OK = 0
STATUS_NAMES = {0: "CSA_OK", 1: "CSA_ERR_INVALID_ARG", 2: "CSA_ERR_UNSUPPORTED", 3: "CSA_ERR_CUDA",
                4: "CSA_ERR_DEVICE_CHECK", 5: "CSA_ERR_WORKSPACE"}

# kernel ids of csa_set_timing_events
KERNEL_INDEXER_SCORE = 0
KERNEL_TOPK_SELECT = 1
KERNEL_ATTENTION = 2
KERNEL_MERGE = 3
KERNEL_COMPRESS = 4
KERNEL_QUANTIZE = 5
KERNEL_TOPK_SAMPLE = 6


class CsaError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


class CacheT(C.Structure):
    """Mirror of csa_cache_t."""
    _fields_ = [("data", C.c_void_p), ("n_rows", C.c_int64), ("seq_stride", C.c_int64),
                ("page_table", C.c_void_p), ("page_size", C.c_int32), ("max_pages", C.c_int32)]


class QRopeT(C.Structure):
    """Mirror of csa_qrope_t."""
    _fields_ = [("q_gain", C.c_void_p), ("q_eps", C.c_float), ("rope_dims", C.c_int32),
                ("rope_base", C.c_float), ("derotate", C.c_int32), ("pos", C.c_void_p)]


_vp, _i32, _i64, _f32, _sz = C.c_void_p, C.c_int32, C.c_int64, C.c_float, C.c_size_t
_qr = C.POINTER(QRopeT)

# name -> (restype, argtypes); the exact list of functions include/csa.h declares
SIGNATURES = {
    "csa_version": (C.c_char_p, []),
    "csa_last_error": (C.c_char_p, []),
    "csa_launch_count": (C.c_uint64, []),
    "csa_set_timing_events": (C.c_int, [_i32, _vp, _vp]),
    "csa_set_attention_kernel": (C.c_int, [_i32]),
    "csa_set_batch_invariant": (C.c_int, [_i32]),
    "csa_test_attention_timeout": (C.c_int, [_i32]),
    "csa_indexer_topk_workspace_size": (_sz, [_i64, _i64, _i32]),
    "csa_sparse_attn_decode_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32]),
    "csa_sparse_attn_prefill_workspace_size": (_sz, [_i64, _i32, _i32]),
    "hca_attn_workspace_size": (_sz, [_i64, _i32, _i32, _i64, _i32]),
    "csa_workspace_init": (C.c_int, [_vp, _sz, _vp]),
    "csa_workspace_check": (C.c_int, [_vp, _vp]),
    "csa_compress_kv": (C.c_int, [_vp, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _vp, _vp]),
    "csa_norm_rope": (C.c_int, [_vp, _vp, _i64, _i32, _i32, _vp, _f32, _vp, _i64, _i32, _f32, _i32,
                                _vp]),
    "csa_cache_append": (C.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp,
                                   _vp, _vp, _vp, _i32, C.POINTER(CacheT), _i64, _vp, _sz, _vp]),
    "csa_indexer_topk": (C.c_int, [_vp, _vp, C.POINTER(CacheT), _vp, _vp, _i64, _i32, _i32, _i32,
                                   _i64, _i32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "csa_quantize_mxfp4": (C.c_int, [_vp, _i64, _i32, _vp, _vp, _vp]),
    "csa_indexer_topk_mxfp4": (C.c_int, [_vp, _vp, C.POINTER(CacheT), _vp, _vp, _vp, _i64, _i32,
                                         _i32, _i32, _i64, _i32, _vp, _vp, _vp, _vp, _sz, _vp]),
    "csa_sparse_attn_prefill": (C.c_int, [_vp, _vp, _i64, _vp, _vp, _vp, _i64, _i32, _i32, _i32,
                                          _i32, _f32, _vp, _vp, _vp, _vp, _sz, _vp, _qr]),
    "csa_sparse_attn_decode": (C.c_int, [_vp, C.POINTER(CacheT), _vp, _vp, _vp, _vp, _i32, _i32,
                                         _i32, _i32, _i32, _f32, _vp, _vp, _vp, _vp, _sz, _vp, _qr]),
    "csa_quantize_entries_fp8": (C.c_int, [_vp, _i64, _i32, _i32, _vp, _vp, _vp, _vp]),
    "csa_sparse_attn_decode_fp8": (C.c_int, [_vp, C.POINTER(CacheT), _vp, _vp, _i32, _vp, _vp, _vp,
                                             _vp, _i32, _i32, _i32, _i32, _i32, _f32, _vp, _vp,
                                             _vp, _vp, _sz, _vp]),
    "hca_attn": (C.c_int, [_vp, C.POINTER(CacheT), _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _i64,
                           _i32, _f32, _vp, _vp, _vp, _vp, _sz, _vp, _qr]),
    "csa_sparse_attn_decode_noalloc": (C.c_int, [_vp, C.POINTER(CacheT), _vp, _vp, _vp, _vp, _i32,
                                                 _i32, _i32, _i32, _i32, _f32, _vp, _vp, _vp,
                                                 _vp]),
}

_lib = None


def load(path=LIB_PATH):
    """Load the library (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(
            f"CUDA library {path} not found; build it with "
            "`python -m compressed_sparse_kv_03_b200.build` (there is no CPU fallback)")
    lib = C.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check(status):
    if status != CSA_OK:
        msg = load().csa_last_error().decode(errors="replace")
        raise CsaError(status, msg)
