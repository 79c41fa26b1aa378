"""ctypes declarations of libpa.so (see include/pa.h for the contract).

Loading fails loudly when the library has not been built: there is no
fallback implementation.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpa.so")

PA_OK = 0
STATUS_NAMES = {
    0: "PA_OK", 1: "PA_ERR_INVALID_ARG", 2: "PA_ERR_UNSUPPORTED",
    3: "PA_ERR_WORKSPACE", 4: "PA_ERR_CUDA", 5: "PA_ERR_OUT_OF_BLOCKS",
    6: "PA_ERR_NOT_FOUND", 7: "PA_ERR_DEVICE",
}

# Every function the header declares, with (restype, argtypes).
_i32, _i64, _u64 = ctypes.c_int, ctypes.c_int64, ctypes.c_uint64
_f32, _vp, _sz = ctypes.c_float, ctypes.c_void_p, ctypes.c_size_t
SIGNATURES = {
    "pa_status_string": (ctypes.c_char_p, [_i32]),
    "pa_decode_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32]),
    "pa_decode": (_i32, [_vp, _vp, _vp, _vp, _i32, _f32, _f32, _vp, _i32, _vp,
                         _i32, _i32, _i32, _i32, _i32, _i32, _i32, _f32, _i32,
                         _vp, _sz, _vp]),
    "pa_decode_append": (_i32, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _f32, _f32, _vp, _i32,
                                _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                                _f32, _i32, _vp, _sz, _vp]),
    "pa_decode_no_alloc": (_i32, [_vp, _vp, _vp, _vp, _i32, _f32, _f32, _vp, _i32,
                                  _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                                  _f32, _i32, _vp]),
    "pa_prefill": (_i32, [_vp, _vp, _vp, _vp, _i32, _vp, _i32, _vp, _vp, _i32, _i32, _i32,
                          _i32, _i32, _i32, _i32, _i32, _i32, _f32, _vp]),
    "pa_reshape_and_cache": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32,
                                    _i32, _i32, _i32, _f32, _f32, _vp]),
    "pa_copy_blocks": (_i32, [_vp, _vp, _vp, _i32, _sz, _i32, _vp]),
    "pa_swap_blocks": (_i32, [_vp, _vp, _vp, _vp, _vp, _i32, _sz, _i32, _i32, _vp]),
    "pa_get_device_error": (_i32, [ctypes.POINTER(ctypes.c_uint32)]),
    "pa_pool_create": (_vp, [_i32, _i32]),
    "pa_pool_destroy": (None, [_vp]),
    "pa_pool_shuffle_free": (_i32, [_vp, _u64]),
    "pa_pool_add_seq": (_i32, [_vp, _i64]),
    "pa_pool_fork": (_i32, [_vp, _i64, _i64]),
    "pa_pool_append": (_i32, [_vp, _i64, _i32, _vp, _vp, ctypes.POINTER(_i32)]),
    "pa_pool_append_decode": (_i32, [_vp, _vp, _i32, _vp, _vp, ctypes.POINTER(_i32)]),
    "pa_pool_free_seq": (_i32, [_vp, _i64]),
    "pa_pool_block_tables": (_i32, [_vp, _vp, _i32, _vp, _i32, _vp]),
    "pa_pool_enable_prefix_caching": (_i32, [_vp, _i32]),
    "pa_pool_append_tokens": (_i32, [_vp, _i64, _vp, _i32, _vp, _vp, ctypes.POINTER(_i32),
                                     ctypes.POINTER(_i32)]),
    "pa_pool_num_cached": (_i32, [_vp]),
    "pa_pool_swap_out": (_i32, [_vp, _vp, _i64, _vp, _i32, ctypes.POINTER(_i32)]),
    "pa_pool_swap_in": (_i32, [_vp, _vp, _i64, _vp, _i32, ctypes.POINTER(_i32)]),
    "pa_pool_num_free": (_i32, [_vp]),
    "pa_pool_refcount": (_i32, [_vp, _i32]),
    "pa_pool_seq_len": (_i64, [_vp, _i64]),
    "pa_pool_seq_lens": (_i32, [_vp, _vp, _i32, _vp]),
    "pa_pool_seq_num_blocks": (_i32, [_vp, _i64]),
}

_lib = None


class LibraryNotBuilt(RuntimeError):
    pass


def lib() -> ctypes.CDLL:
    """The loaded libpa.so with argument types set."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise LibraryNotBuilt(
            f"{LIB_PATH} is missing: build it with "
            "`python -m paged_kv_cache_429_b200.build` (no fallback exists)")
    handle = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(handle, name)
        fn.restype = res
        fn.argtypes = args
    _lib = handle
    return handle
