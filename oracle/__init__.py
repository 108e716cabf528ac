"""Plain CPU oracle for paged decode attention -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s cpu_baseline /
reference leg may import this package.  It shares no code with the product
package ``paged_kv_cache_452_b200`` and neither imports the other.

Contents
--------
* ``cache_write`` / ``attention`` / ``e4m3_decode`` / ``e4m3_encode``: numpy
  front ends of the fp64 C oracle in ``pa_oracle.c`` (built with gcc).
* ``copy_blocks``: whole-block copies inside the pools (copy-on-write).
* ``pool_model.BlockPoolModel``: a dict/list restatement of the block pool
  (free_block_queue, ref_cnt, hash-keyed prefix sharing).
* ``admission``: the pages' memory arithmetic (blocks per sequence, bytes per
  block, contiguous vs paged admission).

Pins (tests/test_oracle.py) tie every function here to something other than
itself: torch's fp64 scaled_dot_product_attention, torch's float8_e4m3fn cast,
closed forms, brute force on tiny inputs, and the pages' worked example.
"""
import ctypes
import os

import numpy as np

from . import admission  # noqa: F401
from .build import build as _build
from .pool_model import BlockPoolModel, PoolModelError  # noqa: F401

# this module's own dtype codes (see pa_oracle.c)
_DT = {"f32": 0, "bf16": 1, "e4m3": 2}
_ELEM = {"f32": 4, "bf16": 2, "e4m3": 1}
_NPDT = {"f32": np.float32, "bf16": np.uint16, "e4m3": np.uint8}

_lib = None


def lib():
    global _lib
    if _lib is None:
        path = _build()
        L = ctypes.CDLL(path)
        c_p = ctypes.c_void_p
        c_i = ctypes.c_int
        L.oracle_e4m3_decode.restype = ctypes.c_double
        L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
        L.oracle_e4m3_encode.restype = ctypes.c_uint8
        L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
        L.oracle_cache_write.restype = c_i
        L.oracle_cache_write.argtypes = [c_i, c_i, c_p, c_p, c_p, c_i, c_i, c_i, c_i, c_i,
                                         ctypes.c_float, ctypes.c_float, c_p, c_p, c_p, c_p]
        L.oracle_attention.restype = None
        L.oracle_attention.argtypes = [c_p, c_i, c_p, c_p, c_p, c_i, c_i, c_p, c_p,
                                       ctypes.c_double, ctypes.c_double, c_p, c_p, c_i, c_i, c_i, c_i,
                                       ctypes.c_double, c_p, c_i]
        L.oracle_max_threads.restype = c_i
        _lib = L
    return _lib


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def _ptr(a: np.ndarray):
    return a.ctypes.data_as(ctypes.c_void_p)


def e4m3_decode(codes) -> np.ndarray:
    """fp64 value of each e4m3 code (OCP E4M3 definition)."""
    codes = np.asarray(codes, dtype=np.uint8)
    f = lib().oracle_e4m3_decode
    return np.array([f(int(c)) for c in codes.ravel()], dtype=np.float64).reshape(codes.shape)


def e4m3_encode(x) -> np.ndarray:
    """e4m3 code of each fp32 value: round to nearest even, saturate to +-448."""
    x = np.asarray(x, dtype=np.float32)
    f = lib().oracle_e4m3_encode
    return np.array([f(float(v)) for v in x.ravel()], dtype=np.uint8).reshape(x.shape)


def _scale_args(scale, num_kv_heads):
    """(fp32 scalar, per-head fp32 array or None) for a scale given as one
    number for the pool or as one number per kv head; the array is kept
    alive by the caller while the C call runs."""
    a = np.asarray(scale, dtype=np.float32)
    if a.ndim == 0:
        return float(a), None
    assert a.shape == (num_kv_heads,), a.shape
    return 1.0, np.ascontiguousarray(a)


def new_cache(num_blocks, num_kv_heads, block_size, head_dim, kv_dtype, d_major=False):
    """A K or V pool in the storage format, filled with a sentinel (NaN for
    fp32/bf16, the e4m3 NaN code for fp8) so that any read of an unwritten
    slot shows up.  Token-major [NB][Hkv][bs][D]; d_major=True gives
    [NB][Hkv][D][bs], the layout of an e4m3 V pool."""
    shape = (num_blocks, num_kv_heads, head_dim, block_size) if d_major else \
        (num_blocks, num_kv_heads, block_size, head_dim)
    if kv_dtype == "f32":
        return np.full(shape, np.nan, dtype=np.float32)
    if kv_dtype == "bf16":
        return np.full(shape, 0x7FC0, dtype=np.uint16)
    return np.full(shape, 0x7F, dtype=np.uint8)


def new_caches(num_blocks, num_kv_heads, block_size, head_dim, kv_dtype):
    """(K pool, V pool) in the layouts the cache write uses for kv_dtype."""
    return (new_cache(num_blocks, num_kv_heads, block_size, head_dim, kv_dtype),
            new_cache(num_blocks, num_kv_heads, block_size, head_dim, kv_dtype,
                      d_major=(kv_dtype == "e4m3")))


def cache_write(k_new, v_new, slot_mapping, k_cache, v_cache, in_dtype, kv_dtype,
                k_scale=1.0, v_scale=1.0):
    """Scatter new K/V rows into the pools through slot_mapping (in place).

    k_new, v_new: [T][Hkv][D] raw storage (float32 array for fp32, uint16 bits
    for bf16).  slot_mapping: int64 [T]; a negative slot is skipped.
    k_cache is [NB][Hkv][bs][D]; v_cache is too, except for e4m3 where it is
    d-major [NB][Hkv][D][bs].  k_scale / v_scale: one fp32 number for the
    pool, or one per kv head.
    """
    k_new = np.ascontiguousarray(k_new)
    v_new = np.ascontiguousarray(v_new)
    slots = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    nb, hkv, bs, d = k_cache.shape
    assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
    assert v_cache.shape == ((nb, hkv, d, bs) if kv_dtype == "e4m3" else (nb, hkv, bs, d))
    assert k_new.shape == (slots.shape[0], hkv, d), k_new.shape
    assert k_new.dtype == _NPDT[in_dtype] and k_cache.dtype == _NPDT[kv_dtype]
    ks, kh = _scale_args(k_scale, hkv)
    vs, vh = _scale_args(v_scale, hkv)
    rc = lib().oracle_cache_write(_DT[in_dtype], _DT[kv_dtype], _ptr(k_new), _ptr(v_new),
                                  _ptr(slots), slots.shape[0], nb, bs, hkv, d, ks, vs,
                                  None if kh is None else _ptr(kh), None if vh is None else _ptr(vh),
                                  _ptr(k_cache), _ptr(v_cache))
    if rc != 0:
        raise ValueError("slot past the end of the pool")


def copy_blocks(k_cache, v_cache, pairs):
    """Copy-on-write's device half ("PagedAttention：KV cache 即虚拟内存
    (block manager & 碎片)", 深入原理, 共享 → prefix caching: a fork that
    diverges inside a shared block triggers a copy): for each (src, dst)
    pair, block dst of each pool becomes block src, every kv head and slot
    in the storage format.  In place."""
    for src, dst in pairs:
        k_cache[dst] = k_cache[src]
        v_cache[dst] = v_cache[src]


def attention(q, row_seq, row_pos, block_tables, k_cache, v_cache, kv_dtype, num_q_heads,
              scale, k_scale=1.0, v_scale=1.0, num_threads=0) -> np.ndarray:
    """fp64 softmax attention for each query row over the keys its sequence's
    block table points at.

    q: [R][Hq][D] (any float dtype; upcast to fp64 exactly).
    row_seq[r], row_pos[r]: sequence and position of row r; it attends keys
    0..row_pos[r].  block_tables: int32 [S][max_blocks].
    k_scale / v_scale are the cache's fp32 scales, one number for the pool or
    one per kv head (an e4m3 code dequantises to its value times its head's
    fp32 scale, in fp64).
    Returns out [R][Hq][D] fp64.
    """
    q = np.ascontiguousarray(q, dtype=np.float64)
    row_seq = np.ascontiguousarray(row_seq, dtype=np.int32)
    row_pos = np.ascontiguousarray(row_pos, dtype=np.int32)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    nb, hkv, bs, d = k_cache.shape
    assert v_cache.shape == ((nb, hkv, d, bs) if kv_dtype == "e4m3" else (nb, hkv, bs, d))
    r = q.shape[0]
    assert q.shape == (r, num_q_heads, d)
    out = np.empty((r, num_q_heads, d), dtype=np.float64)
    ks, kh = _scale_args(k_scale, hkv)
    vs, vh = _scale_args(v_scale, hkv)
    lib().oracle_attention(_ptr(q), r, _ptr(row_seq), _ptr(row_pos), _ptr(bt), bt.shape[1],
                           _DT[kv_dtype], _ptr(k_cache), _ptr(v_cache), ks, vs,
                           None if kh is None else _ptr(kh), None if vh is None else _ptr(vh),
                           bs, num_q_heads, hkv, d, float(scale), _ptr(out), int(num_threads))
    return out
