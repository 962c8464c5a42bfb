"""ctypes declarations of the C ABI in include/sparse_attn.h.

Loads the in-tree libsparse_attn.so.  There is no fallback: if the library is
missing or fails to load, importing the package raises.
"""
from __future__ import annotations

import ctypes as C
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libsparse_attn.so")

SA_OK = 0
SA_ERR_INVALID = 1
SA_ERR_UNSUPPORTED = 2
SA_ERR_WORKSPACE = 3
SA_ERR_CUDA = 4
SA_ERR_TIMEOUT = 5
SA_ERR_DEVICE_CHECK = 6

SA_SCORE_ENVELOPE = 0
SA_SCORE_CENTROID = 1

SA_OUT_F32 = 0
SA_OUT_BF16 = 1

SA_BUDGET_TOPK = 0
SA_BUDGET_RATIO = 1
SA_BUDGET_TOKENS = 2


class sa_kv_desc(C.Structure):
    _fields_ = [
        ("batch", C.c_int32),
        ("n_kv_heads", C.c_int32),
        ("head_dim", C.c_int32),
        ("page_size", C.c_int32),
        ("cap_tokens", C.c_int64),
        ("k", C.c_void_p),
        ("v", C.c_void_p),
        ("seq_len", C.c_void_p),
        ("chunk_off", C.c_void_p),
        ("n_chunks", C.c_void_p),
        ("max_pages", C.c_int32),
    ]


class sa_budget(C.Structure):
    _fields_ = [
        ("kind", C.c_int),
        ("top_k", C.c_int32),
        ("topk_ratio", C.c_double),
        ("topk_val", C.c_int32),
        ("bos", C.c_int32),
        ("eos", C.c_int32),
        ("token_budget", C.c_int32),
    ]


# name -> (restype, argtypes); mirrors include/sparse_attn.h
PROTOTYPES = {
    "sparse_attn_workspace_size": (C.c_size_t, [C.POINTER(sa_kv_desc), C.c_int32, C.c_int32, C.c_int32]),
    "sparse_attn_workspace_init": (C.c_int, [C.c_void_p, C.c_size_t, C.c_void_p]),
    "sparse_attn_build_meta": (C.c_int, [C.POINTER(sa_kv_desc), C.c_int, C.c_int32, C.c_void_p, C.c_void_p]),
    "sparse_attn_select": (C.c_int, [C.POINTER(sa_kv_desc), C.c_void_p, C.c_int, C.c_void_p, C.c_int32,
                                     C.POINTER(sa_budget), C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p,
                                     C.c_void_p, C.c_size_t, C.c_void_p]),
    "sparse_attn_decode": (C.c_int, [C.POINTER(sa_kv_desc), C.c_void_p, C.c_int32, C.c_int32, C.c_int32,
                                     C.c_int32, C.c_float, C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p,
                                     C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "sparse_attn_decode_step": (C.c_int, [C.POINTER(sa_kv_desc), C.c_void_p, C.c_int, C.c_void_p, C.c_int32,
                                          C.POINTER(sa_budget), C.c_int32, C.c_float, C.c_void_p,
                                          C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_size_t,
                                          C.c_void_p]),
    "sparse_attn_decode_step_wait_test": (C.c_int, [C.POINTER(sa_kv_desc), C.c_void_p, C.c_int, C.c_void_p,
                                                    C.c_int32, C.POINTER(sa_budget), C.c_int32, C.c_float,
                                                    C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                                    C.c_int32, C.c_uint32, C.c_void_p, C.c_size_t,
                                                    C.c_void_p]),
    "sparse_attn_decode_step_per_head": (C.c_int, [C.POINTER(sa_kv_desc), C.c_void_p, C.c_int, C.c_void_p,
                                                   C.c_int32, C.POINTER(sa_budget), C.c_int32, C.c_float,
                                                   C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                                   C.c_void_p, C.c_size_t, C.c_void_p]),
    "sparse_attn_decode_step_append": (C.c_int, [C.POINTER(sa_kv_desc), C.c_void_p, C.c_int, C.c_void_p,
                                                 C.c_int32, C.c_void_p, C.c_void_p, C.POINTER(sa_budget),
                                                 C.c_int32, C.c_float, C.c_void_p, C.c_void_p, C.c_void_p,
                                                 C.c_int, C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "sparse_attn_workspace_size_per_head": (C.c_size_t, [C.POINTER(sa_kv_desc), C.c_int32, C.c_int32]),
    "sparse_attn_select_per_head": (C.c_int, [C.POINTER(sa_kv_desc), C.c_void_p, C.c_int, C.c_void_p, C.c_int32,
                                              C.POINTER(sa_budget), C.c_int32, C.c_void_p, C.c_void_p,
                                              C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "sparse_attn_decode_per_head": (C.c_int, [C.POINTER(sa_kv_desc), C.c_void_p, C.c_int32, C.c_float,
                                              C.c_void_p, C.c_void_p, C.c_int32, C.c_void_p, C.c_void_p,
                                              C.c_void_p, C.c_size_t, C.c_void_p]),
    "sparse_attn_route_decode": (C.c_int, [C.POINTER(sa_kv_desc), C.c_void_p, C.c_int, C.c_void_p, C.c_int32,
                                           C.c_int32, C.c_int32, C.c_float, C.c_void_p, C.c_void_p, C.c_void_p,
                                           C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                           C.c_size_t, C.c_void_p]),
    "sparse_attn_route_decode_step": (C.c_int, [C.POINTER(sa_kv_desc), C.c_void_p, C.c_int, C.c_void_p,
                                                C.c_int32, C.c_int32, C.c_int32, C.c_float, C.c_void_p,
                                                C.c_float, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                                C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                                C.c_size_t, C.c_void_p]),
    "sparse_attn_route": (C.c_int, [C.POINTER(sa_kv_desc), C.c_void_p, C.c_int, C.c_void_p, C.c_int32,
                                    C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_int32, C.c_float,
                                    C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p,
                                    C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]),
    "sparse_attn_decode_static": (C.c_int, [C.POINTER(sa_kv_desc), C.c_void_p, C.c_int32, C.c_int32,
                                            C.c_int32, C.c_int32, C.c_float, C.c_void_p, C.c_void_p,
                                            C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]),
    "sparse_attn_get_device_status": (C.c_int, [C.c_void_p, C.POINTER(C.c_int), C.c_void_p]),
    "sparse_attn_status_string": (C.c_char_p, [C.c_int]),
}


def load(path: str = LIB_PATH) -> C.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"libsparse_attn.so not found at {path}; build it with "
            "`python block_sparse_kv_page_b200/build.py` (there is no CPU fallback)")
    lib = C.CDLL(path)
    for name, (res, args) in PROTOTYPES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib
