"""ctypes declarations of liblsa.so (include/lsa.h).  Loading fails loudly: there is no
fallback implementation of any call."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblsa.so")

c_int, c_size_t, c_void_p, c_float, c_char_p = (ctypes.c_int, ctypes.c_size_t, ctypes.c_void_p,
                                                ctypes.c_float, ctypes.c_char_p)

# name -> (restype, argtypes), in the order of include/lsa.h
SIGNATURES = {
    "lsa_status_string": (c_char_p, [c_int]),
    "lsa_last_error": (c_char_p, []),
    "lsa_abi_version": (c_int, []),
    "lsa_kernel_launches": (ctypes.c_ulonglong, []),
    "lsa_index_project_workspace_bytes": (c_size_t, [c_int] * 7),
    "lsa_index_project": (c_int, [c_int] * 7 + [c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_void_p,
                                               c_void_p, c_void_p, c_size_t, c_void_p]),
    "lsa_index_score_workspace_bytes": (c_size_t, [c_int] * 9),
    "lsa_index_score": (c_int, [c_int] * 7 + [c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                              c_int, c_void_p, c_void_p, c_int, c_void_p, c_void_p,
                                              c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                              c_void_p, c_void_p, c_size_t, c_void_p]),
    "lsa_select_union": (c_int, [c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p]),
    "lsa_compact": (c_int, [c_int, c_int, c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p]),
    "lsa_select_fetch_workspace_bytes": (c_size_t, [c_int, c_int]),
    "lsa_select_fetch": (c_int, [c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_void_p,
                                 c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "lsa_topk_keyed": (c_int, [c_int, c_int, c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "lsa_topk_workspace_bytes": (c_size_t, [c_int, c_int]),
    "lsa_topk": (c_int, [c_int, c_int, c_int, c_int, c_void_p, c_int, c_void_p, c_void_p, c_void_p,
                         c_void_p, c_void_p, c_size_t, c_void_p]),
    "lsa_fine_score_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int]),
    "lsa_fine_score": (c_int, [c_int, c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_int, c_void_p, c_void_p,
                               c_void_p, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "lsa_topk_noalloc": (c_int, [c_int, c_int, c_int, c_int, c_void_p, c_int, c_void_p, c_void_p, c_void_p,
                                 c_void_p, c_void_p]),
    "lsa_gather_cold": (c_int, [c_int, c_int, c_size_t, c_void_p, c_void_p, c_void_p, c_int, c_void_p,
                                c_void_p, c_void_p]),
    "lsa_hot_pool_state_bytes": (c_size_t, [c_int, c_int, c_int]),
    "lsa_hot_pool_workspace_bytes": (c_size_t, [c_int, c_int, c_int]),
    "lsa_hot_pool_layout": (c_int, [c_int, c_int, c_int, ctypes.POINTER(c_size_t)]),
    "lsa_hot_pool_reset": (c_int, [c_int, c_int, c_int, c_void_p, c_void_p]),
    "lsa_hot_pool_update": (c_int, [c_int, c_int, c_int, c_size_t, ctypes.c_uint32, c_void_p, c_void_p, c_void_p,
                                    c_void_p, c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
    "lsa_check_bounded_wait": (c_int, [ctypes.c_uint32, c_void_p, c_void_p]),
    "lsa_index_train_step_workspace_bytes": (c_size_t, [c_int] * 6),
    "lsa_index_train_step": (c_int, [c_int] * 7 + [c_void_p, c_void_p, c_void_p, c_void_p, c_float, c_int,
                                                    c_void_p, c_void_p, c_void_p, c_float, c_void_p, c_void_p,
                                                    c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                                    c_void_p, c_void_p, c_size_t, c_void_p]),
    "lsa_vote_labels_workspace_bytes": (c_size_t, [c_int, c_int, c_int]),
    "lsa_vote_labels": (c_int, [c_int, c_int, c_int, c_void_p, c_float, c_int, c_void_p, c_void_p,
                                c_void_p, c_float, c_void_p, c_void_p, c_size_t, c_void_p]),
}

_lib = None


def load() -> ctypes.CDLL:
    """The loaded library with argument types set.  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python -m lookahead_sparse_kv_score_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib
