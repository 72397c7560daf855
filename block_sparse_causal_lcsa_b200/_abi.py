"""ctypes view of include/lcsa.h: structs, prototypes and status codes.

Argument marshalling only; every step of the attention path runs in the
CUDA kernels of liblcsa.so. Importing this module loads the library and fails
loudly if it is missing or does not export every declared entry point.
"""
from __future__ import annotations

import ctypes as C
import os

from .build import LIB_PATH

MAX_STREAMS = 64

OK = 0
ERR_INVALID_ARG = -1
ERR_SHAPE = -2
ERR_ALIGN = -3
ERR_CAPACITY = -4
ERR_WORKSPACE = -5
ERR_CUDA = -6
ERR_TIMEOUT = -7
ERR_DEVICE_BOUNDS = -8
ERR_SCRATCH_LIMIT = -9
WINDOW_TRUNCATE_TOKENS = 2
WINDOW_PRESERVE_TOKENS = 3
SELECT_STATIC_SCRATCH_BYTES = 8 << 20

WINDOW_TRUNCATE = 0
WINDOW_PRESERVE = 1


class Tensor(C.Structure):
    _fields_ = [
        ("data", C.c_void_p),
        ("B", C.c_int32), ("H", C.c_int32), ("T", C.c_int32),
        ("Y", C.c_int32), ("X", C.c_int32), ("D", C.c_int32),
        ("stride_b", C.c_int64), ("stride_h", C.c_int64), ("stride_t", C.c_int64),
        ("stride_y", C.c_int64), ("stride_x", C.c_int64),
    ]


class KVCacheStruct(C.Structure):
    _fields_ = [
        ("k", C.c_void_p), ("v", C.c_void_p), ("k_pool", C.c_void_p),
        ("B", C.c_int32), ("H", C.c_int32), ("cap_frames", C.c_int32),
        ("Y", C.c_int32), ("X", C.c_int32), ("D", C.c_int32),
        ("begin", C.c_int64 * MAX_STREAMS),
        ("end", C.c_int64 * MAX_STREAMS),
    ]


class SelectParamsStruct(C.Structure):
    _fields_ = [
        ("top_k", C.c_int32), ("window", C.c_int32), ("window_mode", C.c_int32),
        ("kmax", C.c_int32), ("density", C.c_double), ("tie_eps", C.c_double),
    ]


# name -> (restype, argtypes), mirroring include/lcsa.h
PROTOTYPES = {
    "lcsa_abi_version": (C.c_int32, []),
    "lcsa_status_string": (C.c_char_p, [C.c_int]),
    "lcsa_pool_qk": (C.c_int, [C.POINTER(Tensor), C.POINTER(Tensor), C.c_void_p, C.c_void_p,
                               C.c_void_p]),
    "lcsa_kv_append": (C.c_int, [C.POINTER(KVCacheStruct), C.POINTER(Tensor), C.POINTER(Tensor),
                                 C.c_void_p, C.c_int32, C.c_void_p]),
    "lcsa_ingest_chunk": (C.c_int, [C.POINTER(Tensor), C.c_void_p, C.POINTER(KVCacheStruct), C.POINTER(Tensor),
                                    C.POINTER(Tensor), C.c_int32, C.c_void_p]),
    "lcsa_kv_advance": (C.c_int, [C.POINTER(KVCacheStruct), C.c_int32, C.c_int32, C.c_int32]),
    "lcsa_select_kmax": (C.c_int32, [C.POINTER(KVCacheStruct), C.c_int32,
                                     C.POINTER(SelectParamsStruct)]),
    "lcsa_select_workspace_bytes": (C.c_size_t, [C.POINTER(KVCacheStruct), C.c_int32]),
    "lcsa_select_blocks": (C.c_int, [C.c_void_p, C.c_int32, C.POINTER(KVCacheStruct),
                                     C.POINTER(SelectParamsStruct), C.c_void_p, C.c_void_p,
                                     C.c_void_p, C.c_size_t, C.c_void_p]),
    "lcsa_select_blocks_noalloc": (C.c_int, [C.c_void_p, C.c_int32, C.POINTER(KVCacheStruct),
                                             C.POINTER(SelectParamsStruct), C.c_void_p, C.c_void_p,
                                             C.c_void_p]),
    "lcsa_sparse_attn_fwd": (C.c_int, [C.POINTER(Tensor), C.POINTER(KVCacheStruct), C.c_void_p,
                                       C.c_void_p, C.c_int32, C.POINTER(Tensor), C.c_void_p,
                                       C.c_void_p]),
    "lcsa_sparse_attn_fwd_window": (C.c_int, [C.POINTER(Tensor), C.POINTER(KVCacheStruct), C.c_void_p, C.c_void_p,
                                              C.c_int32, C.c_int32, C.c_int32, C.POINTER(Tensor), C.c_void_p,
                                              C.c_void_p]),
    "lcsa_sparse_attn_fwd_workspace_bytes": (C.c_size_t, [C.c_int32]),
    "lcsa_sparse_attn_fwd_ex": (C.c_int, [C.POINTER(Tensor), C.POINTER(KVCacheStruct), C.c_void_p, C.c_void_p,
                                          C.c_int32, C.c_int32, C.c_int32, C.POINTER(Tensor), C.c_void_p,
                                          C.c_void_p, C.c_size_t, C.c_void_p]),
    "lcsa_segment_kmax": (C.c_int32, [C.POINTER(KVCacheStruct)]),
    "lcsa_segment_blocks": (C.c_int, [C.c_int32, C.POINTER(KVCacheStruct), C.c_int32, C.c_void_p, C.c_void_p,
                                      C.c_void_p]),
    "lcsa_sparse_attn_bwd_workspace_bytes": (C.c_size_t, [C.POINTER(KVCacheStruct), C.c_int32]),
    "lcsa_sparse_attn_bwd": (C.c_int, [C.POINTER(Tensor), C.POINTER(KVCacheStruct), C.c_void_p, C.c_void_p,
                                       C.c_int32, C.POINTER(Tensor), C.c_void_p, C.POINTER(Tensor),
                                       C.POINTER(Tensor), C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t,
                                       C.c_void_p]),
    "lcsa_last_device_error": (C.c_int, [C.c_void_p]),
    "lcsa_debug_set_wait_limit_ns": (C.c_int, [C.c_uint64]),
    "lcsa_debug_stalled_wait": (C.c_int, [C.c_uint64, C.c_void_p]),
    "lcsa_debug_exp2_poly": (C.c_int, [C.c_void_p, C.c_void_p, C.c_int64, C.c_void_p]),
    "lcsa_pipeline_create": (C.c_int, [C.POINTER(KVCacheStruct), C.c_int32, C.POINTER(SelectParamsStruct),
                                       C.POINTER(C.c_void_p)]),
    "lcsa_pipeline_submit": (C.c_int, [C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "lcsa_pipeline_sync": (C.c_int, [C.c_void_p]),
    "lcsa_pipeline_start_timer": (C.c_int, [C.c_void_p]),
    "lcsa_pipeline_elapsed_ms": (C.c_int, [C.c_void_p, C.POINTER(C.c_float)]),
    "lcsa_pipeline_destroy": (None, [C.c_void_p]),
}


def load(path: str = LIB_PATH) -> C.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            "liblcsa.so is not built (%s); run `python block_sparse_causal_lcsa_b200/build.py` "
            "or __graft_entry__.build()" % path)
    lib = C.CDLL(path)
    for name, (res, args) in PROTOTYPES.items():
        try:
            fn = getattr(lib, name)
        except AttributeError:
            raise ImportError("%s lacks the entry point %s (stale or foreign build)" % (path, name)) from None
        fn.restype = res
        fn.argtypes = args
    if lib.lcsa_abi_version() != 1:
        raise ImportError("liblcsa.so ABI version mismatch")
    return lib
