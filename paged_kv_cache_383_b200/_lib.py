"""ctypes loader for libpagedkv.so and the signatures of its C ABI.

Argument marshalling only: every step of the computation runs inside the
library.  If the shared library is missing this module raises at load time;
there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpagedkv.so")

# pa_status
PA_OK = 0
PA_ERR_INVALID_ARG = 1
PA_ERR_UNSUPPORTED = 2
PA_ERR_NO_FREE_BLOCKS = 3
PA_ERR_CUDA = 4
PA_ERR_DEVICE_OOB = 5
PA_ERR_WORKSPACE = 6
PA_ERR_DEVICE_TIMEOUT = 7

# bytes of the built-in scratch area behind pa_decode_noalloc
PA_NOALLOC_SCRATCH_BYTES = 32 << 20

# pa_dtype
PA_F16 = 0
PA_BF16 = 1

# pa_reduce
PA_REDUCE_AUTO = 0
PA_REDUCE_KERNEL = 1

# pa_kernel
PA_KERNEL_AUTO = 0
PA_KERNEL_SIMT = 1
PA_KERNEL_MMA = 2


class pa_decode_desc(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int),
        ("num_q_heads", ctypes.c_int),
        ("num_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("block_size", ctypes.c_int),
        ("max_blocks_per_seq", ctypes.c_int),
        ("num_blocks", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("partition_size", ctypes.c_int),
        ("max_context_len", ctypes.c_int),
        ("kernel", ctypes.c_int),
        ("reduce", ctypes.c_int),
        ("out_fp32", ctypes.c_int),
    ]


class pa_prefill_desc(ctypes.Structure):
    _fields_ = [
        ("num_seqs", ctypes.c_int),
        ("num_q_heads", ctypes.c_int),
        ("num_kv_heads", ctypes.c_int),
        ("head_dim", ctypes.c_int),
        ("block_size", ctypes.c_int),
        ("max_blocks_per_seq", ctypes.c_int),
        ("num_blocks", ctypes.c_int),
        ("dtype", ctypes.c_int),
        ("total_q", ctypes.c_int),
        ("max_q_len", ctypes.c_int),
        ("max_context_len", ctypes.c_int),
        ("kernel", ctypes.c_int),
        ("out_fp32", ctypes.c_int),
        ("pv", ctypes.c_int),
    ]


PA_PREFILL_AUTO, PA_PREFILL_TILE = 0, 1
# pa_prefill_pv
PA_PV_AUTO, PA_PV_SPLIT, PA_PV_SINGLE = 0, 1, 2

_vp = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_int = ctypes.c_int
_pi32 = ctypes.POINTER(ctypes.c_int32)
_pi64 = ctypes.POINTER(ctypes.c_int64)
_st = ctypes.c_int  # pa_status

# name -> (restype, argtypes); the same set include/pagedkv.h declares.
SIGNATURES = {
    "pa_version": (ctypes.c_char_p, []),
    "pa_status_string": (ctypes.c_char_p, [_st]),
    "pa_last_error": (ctypes.c_char_p, []),
    "pa_decode_workspace_bytes": (ctypes.c_size_t,
                                  [ctypes.POINTER(pa_decode_desc)]),
    "pa_decode_partition_size": (_int, [ctypes.POINTER(pa_decode_desc)]),
    "pa_decode": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float,
                        ctypes.POINTER(pa_decode_desc), _vp, ctypes.c_size_t,
                        _vp, _vp]),
    "pa_decode_noalloc": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float,
                                ctypes.POINTER(pa_decode_desc), _vp, _vp]),
    "pa_prefill": (_st, [_vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.c_float,
                         ctypes.POINTER(pa_prefill_desc), _vp, ctypes.c_size_t,
                         _vp, _vp]),
    "pa_prefill_workspace_bytes": (ctypes.c_size_t,
                                   [ctypes.POINTER(pa_prefill_desc)]),
    "pa_cache_write": (_st, [_vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int,
                             _int, _int, _vp, _vp]),
    "pa_copy_blocks": (_st, [_vp, _vp, _vp, _int, _int, _int, _int, _int, _int,
                             _vp, _vp]),
    "pa_swap_blocks": (_st, [_vp, _vp, _vp, _vp, _vp, _int, _int, _int, _int,
                             _int, _int, _int, _vp, _vp]),
    "pa_bm_create": (_st, [_int, _int, _pi32, ctypes.POINTER(_vp)]),
    "pa_bm_destroy": (None, [_vp]),
    "pa_bm_add_seq": (_st, [_vp, _i64]),
    "pa_bm_fork": (_st, [_vp, _i64, _i64]),
    "pa_bm_append": (_st, [_vp, _i64, _int, _pi64, _pi32, _int,
                           ctypes.POINTER(_int)]),
    "pa_bm_append_batch": (_st, [_vp, _pi64, _pi32, _int, _pi64, _pi32, _int,
                                 ctypes.POINTER(_int), ctypes.POINTER(_int)]),
    "pa_bm_free_seq": (_st, [_vp, _i64]),
    "pa_bm_truncate": (_st, [_vp, _i64, _i64]),
    "pa_bm_block_table": (_st, [_vp, _pi64, _int, _int, _pi32, _pi32]),
    "pa_launch_count": (_i64, []),
    "pa_read_probe": (_st, [_vp, ctypes.c_size_t, _vp, _vp]),
    "pa_wait_probe": (_st, [_vp, _vp]),
    "pa_bm_num_free": (_int, [_vp]),
    "pa_bm_refcount": (_int, [_vp, _int]),
    "pa_bm_seq_len": (_i64, [_vp, _i64]),
    "pa_bm_num_seq_blocks": (_int, [_vp, _i64]),
    "pa_bm_num_used": (_int, [_vp]),
    "pa_pool_blocks": (_i64, [ctypes.c_uint64, _int, _int, _int, _int,
                              _int]),
    "pa_bm_match_prefix": (_st, [_vp, _i64, _pi32, _i64, _pi64]),
    "pa_bm_cache_insert": (_st, [_vp, _i64, _pi32, _i64]),
    "pa_bm_cache_evict": (_st, [_vp, _int, ctypes.POINTER(_int)]),
    "pa_bm_num_cached": (_int, [_vp]),
    "pa_bm_cache_nodes": (_st, [_vp, _int, _pi32, _pi32, _pi32,
                                ctypes.POINTER(_int)]),
    "pa_bm_set_host_blocks": (_st, [_vp, _int]),
    "pa_bm_swap_out": (_st, [_vp, _pi64, _int, _pi32, _int,
                             ctypes.POINTER(_int)]),
    "pa_bm_swap_in": (_st, [_vp, _pi64, _int, _pi32, _int,
                            ctypes.POINTER(_int)]),
    "pa_bm_num_free_host": (_int, [_vp]),
    "pa_bm_host_refcount": (_int, [_vp, _int]),
    "pa_bm_is_swapped": (_int, [_vp, _i64]),
    "pa_bm_seq_blocks": (_st, [_vp, _i64, _pi32, _int, ctypes.POINTER(_int)]),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load libpagedkv.so (once) and declare every entry point's signature."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python -m paged_kv_cache_383_b200.build_lib` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


class PagedKVError(RuntimeError):
    """A non-OK pa_status, with the library's description."""

    def __init__(self, status: int, where: str):
        lib = load()
        text = lib.pa_status_string(status).decode()
        detail = lib.pa_last_error().decode()
        super().__init__(f"{where}: {text} ({status}): {detail}")
        self.status = status


class NoFreeBlocksError(PagedKVError):
    """The block pool cannot supply the blocks an append needs."""


def check(status: int, where: str) -> None:
    if status == PA_OK:
        return
    if status == PA_ERR_NO_FREE_BLOCKS:
        raise NoFreeBlocksError(status, where)
    raise PagedKVError(status, where)
