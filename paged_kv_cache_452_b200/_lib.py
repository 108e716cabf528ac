"""Loads libpa.so and declares the C signatures of include/pa.h."""
import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpa.so")

# Every exported symbol of include/pa.h, with (restype, argtypes).
_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_F = ctypes.c_float
_SZ = ctypes.c_size_t
SIGNATURES = {
    "pa_last_error": (ctypes.c_char_p, []),
    "pa_version": (ctypes.c_char_p, []),
    "pa_block_bytes": (_SZ, [_P]),
    "pa_cache_write": (ctypes.c_int, [_P, _P, _P, _P, _I32, _P, _P, _P]),
    "pa_copy_blocks": (ctypes.c_int, [_P, _P, _P, _I32, _P, _P, _P]),
    "pa_decode_workspace_size": (_SZ, [_P, _I32]),
    "pa_decode": (ctypes.c_int, [_P, _P, _P, _P, _P, _I32, _P, _I32, _F, _P, _P, _SZ, _P]),
    "pa_decode_static": (ctypes.c_int, [_P, _P, _P, _P, _P, _I32, _P, _I32, _F, _P, _P]),
    "pa_decode_fused": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _I32, _P, _I32, _F, _P, _P, _SZ, _P]),
    "pa_prefill_workspace_size": (_SZ, [_P, _I32, _I32]),
    "pa_prefix_groups": (ctypes.c_int, [_P, _I32, _P, _I32, _I32, _P, _P, _P, _P, _P, _P, _P]),
    "pa_decode_prefix_workspace_size": (_SZ, [_P, _I32, _I32, _I32]),
    "pa_decode_prefix": (ctypes.c_int, [_P, _P, _P, _P, _P, _I32, _P, _I32, _P, _P, _P, _P, _P, _I32, _I32, _I32,
                                        _F, _P, _P, _SZ, _P]),
    "pa_decode_chunked_prefill": (ctypes.c_int,
                                  [_P, _P, _P, _P, _P, _I32, _P, _P, _I32, _I32, _I32, _F, _P, _P, _SZ, _P]),
    "pa_pool_create": (ctypes.c_int, [_I32, _I32, _P, _P]),
    "pa_pool_destroy": (None, [_P]),
    "pa_pool_add_seq": (ctypes.c_int, [_P, _I64, _P, _I32, _P]),
    "pa_pool_append": (ctypes.c_int, [_P, _I64, _I32, _P]),
    "pa_pool_fork": (ctypes.c_int, [_P, _I64, _I64]),
    "pa_pool_take_copies": (ctypes.c_int, [_P, _P, _P, _I32, _P]),
    "pa_pool_slots": (ctypes.c_int, [_P, _I64, _I32, _I32, _P]),
    "pa_pool_free_seq": (ctypes.c_int, [_P, _I64]),
    "pa_pool_block_table": (ctypes.c_int, [_P, _I64, _P, _I32, _P]),
    "pa_pool_block_tables": (ctypes.c_int, [_P, _P, _I32, _I32, _P]),
    "pa_pool_num_tokens": (ctypes.c_int, [_P, _I64, _P]),
    "pa_pool_ref_cnt": (_I32, [_P, _I32]),
    "pa_pool_num_free": (_I32, [_P]),
    "pa_pool_free_order": (ctypes.c_int, [_P, _P, _I32, _P]),
}


class PaError(RuntimeError):
    def __init__(self, code, msg):
        super().__init__(msg)
        self.code = code


_lib = None


def lib():
    """The loaded library; raises (no fallback) if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with "
                              "`python paged_kv_cache_452_b200/build.py`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


lib()
