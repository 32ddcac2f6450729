"""ctypes loader of the PBSA C-ABI library (``libpbsa.so``, built in-tree).

There is no fallback: if the library is missing this module raises, so a
caller can never silently run anything but the CUDA kernels.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpbsa.so")

c_int, c_float, c_void_p, c_size_t, c_int64 = (ctypes.c_int, ctypes.c_float, ctypes.c_void_p,
                                                ctypes.c_size_t, ctypes.c_int64)


class PbsaDims(ctypes.Structure):
    _fields_ = [("B", c_int), ("H", c_int), ("D", c_int), ("bs", c_int), ("scale", c_float),
                ("dtype", c_int), ("q_chunk", c_int)]


P = ctypes.POINTER(PbsaDims)

# field order and types of pbsa_route_args (include/pbsa.h)
ROUTE_FIELDS = [
    ("q", c_void_p), ("Tq", c_int), ("kpool", c_void_p), ("vpool", c_void_p), ("NB", c_int),
    ("blk_len", c_void_p), ("blk_pos", c_void_p), ("pool_ids", c_void_p), ("n_pool", c_int),
    ("q_bar", c_void_p), ("k_bar", c_void_p), ("scores", c_void_p), ("mem_score", c_void_p),
    ("P", c_int), ("n_sink", c_int), ("slot_src", c_void_p), ("slot_w", c_void_p),
    ("cand_ids", c_void_p), ("cand_src", c_void_p), ("n_cand", c_int), ("policy", c_int),
    ("win_ids", c_void_p), ("n_win", c_int), ("k", c_int), ("mem_ids", c_void_p),
    ("n_mem", c_int), ("mask", c_int), ("q_pos0", c_int), ("idx", c_void_p), ("cnt", c_void_p),
    ("Amax", c_int),
]


class PbsaRouteArgs(ctypes.Structure):
    _fields_ = ROUTE_FIELDS

# name -> (restype, argtypes); mirrors include/pbsa.h
SIGNATURES = {
    "pbsa_score_blocks": (c_int, [P, c_void_p, c_int, c_void_p, c_int, c_void_p, c_void_p, c_int,
                                  c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "pbsa_append_chunk": (c_int, [P, c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p, c_int,
                                  c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]),
    "pbsa_update_memory_workspace": (c_size_t, [P, c_int, c_int]),
    "pbsa_update_memory": (c_int, [P, c_void_p, c_void_p, c_int, c_void_p, c_void_p, c_void_p,
                                   c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p, c_int,
                                   c_void_p, c_int, c_void_p, c_size_t, c_void_p]),
    "pbsa_update_plan_bytes": (c_size_t, [P, c_int, c_int]),
    "pbsa_update_memory_bwd_workspace": (c_size_t, [P, c_int]),
    "pbsa_update_memory_bwd": (c_int, [P, c_int, c_int, c_int, c_void_p, c_void_p, c_void_p,
                                       c_void_p, c_size_t, c_void_p]),
    "pbsa_select_local": (c_int, [P, c_void_p, c_int, c_int, c_void_p, c_int, c_int, c_void_p,
                                  c_int, c_int, c_void_p, c_int, c_int, c_void_p, c_int, c_void_p,
                                  c_void_p, c_int, c_int, c_int, c_void_p]),
    "pbsa_select_hier": (c_int, [P, c_void_p, c_int, c_int, c_void_p, c_void_p, c_int, c_int,
                                 c_int, c_int, c_void_p, c_int, c_int, c_void_p, c_int, c_int,
                                 c_void_p, c_int, c_void_p, c_void_p, c_int, c_int, c_int,
                                 c_void_p]),
    "pbsa_route_workspace": (c_size_t, [P, c_int, c_int]),
    "pbsa_route_step": (c_int, [P, ctypes.POINTER(PbsaRouteArgs), c_void_p, c_size_t, c_void_p]),
    "pbsa_attn_fwd": (c_int, [P, c_void_p, c_int, c_int, c_void_p, c_void_p, c_int, c_void_p,
                              c_void_p, c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p,
                              c_void_p]),
    "pbsa_attn_bwd_workspace": (c_size_t, [P, c_int, c_int, c_int]),
    "pbsa_attn_bwd": (c_int, [P, c_void_p, c_int, c_int, c_void_p, c_void_p, c_int, c_void_p,
                              c_void_p, c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p,
                              c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                              c_void_p]),
    "pbsa_attn_bwd_noalloc": (c_int, [P, c_void_p, c_int, c_int, c_void_p, c_void_p, c_int,
                                      c_void_p, c_void_p, c_void_p, c_void_p, c_int, c_int,
                                      c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                      c_void_p]),
    "pbsa_attn_bwd_noalloc_max_scratch": (c_size_t, []),
    "pbsa_check_exp2": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_void_p]),
    "pbsa_get_status": (c_int, [c_void_p]),
    "pbsa_last_error": (ctypes.c_char_p, []),
    "pbsa_version": (ctypes.c_char_p, []),
    "pbsa_set_debug": (None, [c_int, c_int64]),
}

_lib = None


def lib() -> ctypes.CDLL:
    """Load libpbsa.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with `python -m block_sparse_attention_39_b200.build`"
                " (there is no CPU fallback)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib
