"""Loads libpa_b200.so and declares the C signatures of include/pa.h.

There is no fallback: if the library is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpa_b200.so")

PA_OK, PA_ERR_INVALID, PA_ERR_OOM, PA_ERR_CUDA, PA_ERR_NOT_FOUND, PA_ERR_UNSUPPORTED = 0, -1, -2, -3, -4, -5
PA_F32, PA_BF16, PA_F16 = 0, 1, 2
PA_DEV_BAD_SLOT, PA_DEV_BAD_PAGE, PA_DEV_BAD_CTX, PA_DEV_BAD_PAIR, PA_DEV_BAD_PLAN = 1, 2, 4, 8, 16
PA_PREFIX_QUERIES_PER_CTA = 128
PA_DEV_TIMEOUT = 32
PA_DEV_BAD_UPDATE = 64
PA_DECODE_AUTO, PA_DECODE_CUDA_CORES, PA_DECODE_TENSOR_CORES = 0, 1, 2
PA_SHARED_PREFIX_AUTO, PA_SHARED_PREFIX_TCGEN05, PA_SHARED_PREFIX_MMA_SYNC, PA_SHARED_PREFIX_TCGEN05_SERIAL = 0, 1, 2, 3
PA_SHARED_PREFIX_TCGEN05_2CTA = 4
PA_SHARED_PREFIX_TCGEN05_ITEMS = 5
PA_LOW_FREE_FRACTION = 0.10


class PoolStats(ctypes.Structure):
    """pa_pool_stats of include/pa.h."""
    _fields_ = [("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32), ("free_pages", ctypes.c_int32),
                ("used_pages", ctypes.c_int32), ("shared_pages", ctypes.c_int32),
                ("num_sequences", ctypes.c_int32), ("logical_tokens", ctypes.c_int64),
                ("physical_tokens", ctypes.c_int64), ("waste_slots", ctypes.c_int64),
                ("waste_fraction", ctypes.c_double), ("free_fraction", ctypes.c_double),
                ("low_free_alarm", ctypes.c_int32), ("reserved0", ctypes.c_int32)]

PA_VERIFY_AUTO, PA_VERIFY_PER_SEQUENCE, PA_VERIFY_JOINT = 0, 1, 2
PA_FAULT_NONE, PA_FAULT_WITHHOLD_FIRST_ITEM = 0, 1
PA_PARTITION_TOKENS = 512
PA_FIXED_SCRATCH_BYTES = 32 * 1024 * 1024

_c = ctypes
_vp, _i32, _i64, _f32, _sz = _c.c_void_p, _c.c_int32, _c.c_int64, _c.c_float, _c.c_size_t
_pi32, _pi64 = _c.POINTER(_c.c_int32), _c.POINTER(_c.c_int64)

# name -> (restype, argtypes); mirrors include/pa.h
SIGNATURES = {
    "pa_last_error": (_c.c_char_p, []),
    "pa_version": (_c.c_char_p, []),
    "pa_reshape_and_cache": (_i32, [_vp, _vp, _i64, _i64, _vp, _i64, _vp, _vp, _i32, _i32, _i32, _i32, _i32,
                                    _vp, _vp]),
    "pa_copy_blocks": (_i32, [_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp]),
    "pa_block_tables_apply": (_i32, [_vp, _i32, _i32, _vp, _i32, _vp, _vp]),
    "pa_decode_workspace_size": (_sz, [_i32, _i32, _i32, _i64]),
    "pa_decode": (_i32, [_vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _vp, _i32,
                         _vp, _sz, _vp, _vp]),
    "pa_decode_verify_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i64]),
    "pa_set_verify_path": (_i32, [_i32]),
    "pa_set_verify_tiling": (_i32, [_i32]),
    "pa_decode_verify": (_i32, [_vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _f32,
                                _vp, _i32, _vp, _sz, _vp, _vp]),
    "pa_decode_partitions": (_i32, [_vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _vp,
                                    _i32, _vp, _sz, _vp, _vp]),
    "pa_decode_reduce": (_i32, [_vp, _i32, _i32, _i32, _i64, _vp, _i32, _vp, _sz, _vp]),
    "pa_decode_fixed_scratch": (_i32, [_vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32,
                                       _vp, _i32, _vp, _vp]),
    "pa_decode_shared_prefix": (_i32, [_vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _f32,
                                       _vp, _i32, _vp, _sz, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _vp, _vp]),
    "pa_set_decode_kernel": (_i32, [_i32]),
    "pa_set_shared_prefix_kernel": (_i32, [_i32]),
    "pa_set_fault_injection": (_i32, [_i32]),
    "pa_eval_exp2": (_i32, [_vp, _vp, _i64, _i32, _vp]),
    "pa_set_decode_tiling": (_i32, [_i32, _i32]),
    "pa_block_alloc_create": (_i32, [_i32, _i32, _pi32, _c.POINTER(_vp)]),
    "pa_block_alloc_destroy": (None, [_vp]),
    "pa_block_alloc_allocate_sequence": (_i32, [_vp, _i64, _i64]),
    "pa_block_alloc_append_token": (_i32, [_vp, _i64, _pi64, _pi32, _pi32]),
    "pa_block_alloc_fork": (_i32, [_vp, _i64, _i64]),
    "pa_block_alloc_free_sequence": (_i32, [_vp, _i64]),
    "pa_block_alloc_slot_mapping": (_i32, [_vp, _i64, _i64, _i64, _pi64]),
    "pa_block_alloc_block_table": (_i32, [_vp, _i64, _pi32, _i32, _pi32]),
    "pa_block_alloc_block_tables": (_i32, [_vp, _pi64, _i32, _pi32, _i32, _i32, _pi32]),
    "pa_block_alloc_table_updates": (_i32, [_vp, _pi64, _i32, _i32, _i32, _pi32, _i32, _pi32, _pi32]),
    "pa_block_alloc_num_tokens": (_i64, [_vp, _i64]),
    "pa_block_alloc_num_free": (_i32, [_vp]),
    "pa_block_alloc_num_sequences": (_i32, [_vp]),
    "pa_block_alloc_ref_count": (_i32, [_vp, _i32]),
    "pa_block_alloc_free_pool": (_i32, [_vp, _pi32, _i32, _pi32]),
    "pa_block_alloc_append_tokens": (_i32, [_vp, _pi64, _i32, _pi64, _pi32, _pi32, _pi32]),
    "pa_block_alloc_stats": (_i32, [_vp, ctypes.c_double, ctypes.c_void_p]),
    "pa_block_alloc_prefix_plan": (_i32, [_vp, _pi64, _i32, _i32, _pi32, _pi32, _pi32, _pi32, _pi32, _pi32,
                                          _pi32]),
}

_lock = threading.Lock()
_lib = None


def load() -> ctypes.CDLL:
    """The loaded library with every signature declared (raises if absent)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError(f"{LIB_PATH} is missing: build it with "
                                  "`python -m paged_kv_cache_356_b200.build` (needs nvcc)")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def last_error() -> str:
    msg = load().pa_last_error()
    return msg.decode() if msg else ""
