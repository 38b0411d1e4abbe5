"""ctypes declarations for libpa.so (include/pa.h).  Loading fails loudly: there is
no fallback implementation of any call."""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpa.so")

c_i32, c_i64, c_u64, c_f32, c_sz, c_vp = (ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64,
                                          ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p)
P_i32 = ctypes.POINTER(c_i32)


class PoolConfig(ctypes.Structure):
    _fields_ = [("num_layers", c_i32), ("num_blocks", c_i32), ("block_size", c_i32),
                ("num_kv_heads", c_i32), ("head_dim", c_i32), ("dtype", ctypes.c_int),
                ("act_dtype", ctypes.c_int)]


class PoolStats(ctypes.Structure):
    _fields_ = [("num_blocks", c_i32), ("num_free", c_i32), ("num_shared", c_i32),
                ("num_seqs", c_i32), ("num_tokens", c_i64), ("cow_copies", c_i64),
                ("peak_used", c_i32), ("num_cached", c_i32), ("num_evictable", c_i32),
                ("cache_hits", c_i64), ("cache_evictions", c_i64)]


# name -> (restype, argtypes); every function declared in include/pa.h
SIGNATURES = {
    "pa_last_error": (ctypes.c_char_p, []),
    "pa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "pa_pool_create": (ctypes.c_int, [ctypes.POINTER(PoolConfig), c_vp, c_vp, c_vp, ctypes.POINTER(c_vp)]),
    "pa_pool_destroy": (ctypes.c_int, [c_vp]),
    "pa_pool_stats": (ctypes.c_int, [c_vp, ctypes.POINTER(PoolStats)]),
    "pa_pool_set_scales": (ctypes.c_int, [c_vp, c_vp]),
    "pa_alloc_block": (ctypes.c_int, [c_vp, P_i32]),
    "pa_free_block": (ctypes.c_int, [c_vp, c_i32]),
    "pa_incref_block": (ctypes.c_int, [c_vp, c_i32]),
    "pa_block_refcount": (ctypes.c_int, [c_vp, c_i32, P_i32]),
    "pa_num_free_blocks": (ctypes.c_int, [c_vp, P_i32]),
    "pa_free_list": (ctypes.c_int, [c_vp, c_vp, c_i32, P_i32]),
    "pa_debug_fail_alloc_after": (ctypes.c_int, [c_vp, c_i64]),
    "pa_seq_add": (ctypes.c_int, [c_vp, P_i32]),
    "pa_seq_fork": (ctypes.c_int, [c_vp, c_i32, P_i32]),
    "pa_seq_free": (ctypes.c_int, [c_vp, c_i32]),
    "pa_seq_info": (ctypes.c_int, [c_vp, c_i32, P_i32, c_vp, c_i32, P_i32]),
    "pa_reserve_slots": (ctypes.c_int, [c_vp, c_vp, c_vp, c_i32, c_vp, c_vp, P_i32]),
    "pa_build_block_tables": (ctypes.c_int, [c_vp, c_vp, c_i32, c_i32, c_vp, c_vp]),
    "pa_prefix_register": (ctypes.c_int, [c_vp, c_i32, c_vp, c_i32, P_i32]),
    "pa_seq_add_cached": (ctypes.c_int, [c_vp, c_vp, c_i32, P_i32, P_i32]),
    "pa_prefix_evictable": (ctypes.c_int, [c_vp, c_vp, c_i32, P_i32]),
    "pa_swap_bytes": (ctypes.c_int, [c_vp, c_i32, ctypes.POINTER(c_sz)]),
    "pa_swap_out": (ctypes.c_int, [c_vp, c_i32, c_vp, c_sz, c_vp]),
    "pa_swap_in": (ctypes.c_int, [c_vp, c_i32, c_vp, c_sz, c_vp]),
    "pa_copy_blocks": (ctypes.c_int, [c_vp, c_vp, c_i32, c_vp]),
    "pa_append_kv": (ctypes.c_int, [c_vp, c_i32, c_vp, c_vp, c_vp, c_i32, c_vp]),
    "pa_decode_max_splits": (c_i32, [c_i32, c_i32, c_i32]),
    "pa_decode_workspace_bytes": (c_sz, [c_i32, c_i32, c_i32, c_i32]),
    "pa_decode_attention": (ctypes.c_int, [c_vp, c_i32, c_vp, c_vp, ctypes.c_int, c_vp, c_i32, c_vp,
                                           c_i32, c_i32, c_f32, c_i32, c_vp, c_sz, c_vp]),
    "pa_decode_attention_static": (ctypes.c_int, [c_vp, c_i32, c_vp, c_vp, ctypes.c_int, c_vp, c_i32, c_vp,
                                                  c_i32, c_i32, c_f32, c_i32, c_vp]),
    "pa_prefill_attention": (ctypes.c_int, [c_vp, c_i32, c_vp, c_vp, ctypes.c_int, c_vp, c_i32, c_vp, c_vp,
                                            c_i32, c_i32, c_i32, c_f32, c_vp]),
    "pa_device_error": (ctypes.c_int, [P_i32, c_i32]),
    "pa_debug_wait_test": (ctypes.c_int, [c_i64, c_i32]),
    "pa_launch_count": (c_u64, []),
}

_lib = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing; build it with `python -c 'import __graft_entry__ as g; "
                              "g.build()'` (nvcc, sm_100a). There is no non-native fallback.")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib
