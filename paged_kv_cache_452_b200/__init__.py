"""Paged KV-cache decode attention for B200 (sm_100a): a thin Python binding
over the C ABI of libpa.so (include/pa.h).

Every function here only marshals arguments (torch tensors -> device
pointers, the current CUDA stream) and calls the library function of the
same name; all work runs in the library's CUDA kernels or its C++ block pool.
Importing fails loudly if libpa.so has not been built
(``python paged_kv_cache_452_b200/build.py``); there is no fallback.
"""
import ctypes
import math
import os

import torch

from ._lib import LIB_PATH, PaError, lib  # noqa: F401

PA_F32, PA_BF16, PA_FP8_E4M3 = 0, 1, 2
_CODES = {"f32": PA_F32, "bf16": PA_BF16, "e4m3": PA_FP8_E4M3}
_TORCH = {PA_F32: torch.float32, PA_BF16: torch.bfloat16, PA_FP8_E4M3: torch.uint8}
_NAMES = {v: k for k, v in _CODES.items()}


class CacheDesc(ctypes.Structure):
    """pa_cache_desc: shape and storage of one layer's paged cache."""
    _fields_ = [("num_blocks", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("kv_dtype", ctypes.c_int32),
                ("q_dtype", ctypes.c_int32), ("k_scale", ctypes.c_float),
                ("v_scale", ctypes.c_float), ("k_head_scales", ctypes.c_void_p),
                ("v_head_scales", ctypes.c_void_p)]

    @classmethod
    def make(cls, num_blocks, block_size, num_kv_heads, num_q_heads, head_dim, kv_dtype="bf16",
             q_dtype="bf16", k_scale=1.0, v_scale=1.0, k_head_scales=None, v_head_scales=None):
        """k_head_scales / v_head_scales: optional device fp32 tensors
        [num_kv_heads] (an e4m3 pool's per-kv-head scales); the desc keeps a
        reference so they stay alive as long as it does."""
        kv = _CODES.get(kv_dtype, kv_dtype)
        q = _CODES.get(q_dtype, q_dtype)
        d = cls(num_blocks, block_size, num_kv_heads, num_q_heads, head_dim, kv, q,
                float(k_scale), float(v_scale), _ptr(k_head_scales), _ptr(v_head_scales))
        d._keep = (k_head_scales, v_head_scales)
        return d

    @property
    def group(self):
        return self.num_q_heads // self.num_kv_heads

    @property
    def kv_torch_dtype(self):
        return _TORCH[self.kv_dtype]

    @property
    def q_torch_dtype(self):
        return _TORCH[self.q_dtype]


def _check(rc, what):
    if rc != 0:
        raise PaError(rc, f"{what}: {lib().pa_last_error().decode()}")


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def pa_block_bytes(desc: CacheDesc) -> int:
    return int(lib().pa_block_bytes(ctypes.byref(desc)))


def alloc_cache(desc: CacheDesc, device, fill=None):
    """Allocate (K pool, V pool) as torch tensors in the library's layout:
    K [NB][Hkv][bs][D]; V the same, or [NB][Hkv][D][bs] for an e4m3 pool.
    fill: optional element value (a raw byte for e4m3)."""
    nb, bs, h, d = desc.num_blocks, desc.block_size, desc.num_kv_heads, desc.head_dim
    dt = desc.kv_torch_dtype
    k = torch.empty((nb, h, bs, d), dtype=dt, device=device)
    v = torch.empty((nb, h, d, bs) if desc.kv_dtype == PA_FP8_E4M3 else (nb, h, bs, d), dtype=dt,
                    device=device)
    if fill is not None:
        k.fill_(fill)
        v.fill_(fill)
    return k, v


def pa_cache_write(desc, k_new, v_new, slot_mapping, k_cache, v_cache, stream=None):
    """Scatter new K/V rows [T][Hkv][D] into the pools through int64 slots."""
    n = int(slot_mapping.shape[0])
    _check(lib().pa_cache_write(ctypes.byref(desc), _ptr(k_new), _ptr(v_new), _ptr(slot_mapping), n,
                                _ptr(k_cache), _ptr(v_cache), _stream(stream)), "pa_cache_write")


def pa_copy_blocks(desc, src, dst, k_cache, v_cache, stream=None):
    """Copy-on-write's device half: K/V block dst[i] := block src[i] (int32 device tensors)."""
    n = int(src.shape[0])
    if int(dst.shape[0]) != n:
        raise PaError(1, "pa_copy_blocks: src and dst differ in length")
    _check(lib().pa_copy_blocks(ctypes.byref(desc), _ptr(src), _ptr(dst), n, _ptr(k_cache), _ptr(v_cache),
                                _stream(stream)), "pa_copy_blocks")


def pa_decode_workspace_size(desc, num_seqs) -> int:
    n = int(lib().pa_decode_workspace_size(ctypes.byref(desc), int(num_seqs)))
    if n == 0:
        raise PaError(1, "pa_decode_workspace_size: " + lib().pa_last_error().decode())
    return n


def pa_prefill_workspace_size(desc, num_seqs, num_tokens) -> int:
    n = int(lib().pa_prefill_workspace_size(ctypes.byref(desc), int(num_seqs), int(num_tokens)))
    if n == 0:
        raise PaError(1, "pa_prefill_workspace_size: " + lib().pa_last_error().decode())
    return n


def alloc_workspace(nbytes, device):
    """Caller-owned scratch; the error word in its first bytes starts at zero."""
    return torch.zeros(int(nbytes), dtype=torch.uint8, device=device)


def workspace_error(workspace) -> int:
    """The error word a kernel sets when a bounded wait times out (1) or a
    block table entry is outside the pool (2).  Synchronises."""
    return int(workspace[:4].view(torch.int32).item())


def pa_decode(desc, q, k_cache, v_cache, block_tables, seq_lens, scale, out, workspace, stream=None):
    """One decode step: q [S][Hq][D] attends seq_lens[s] keys via block_tables [S][max_blocks]."""
    s = int(seq_lens.shape[0])
    _check(lib().pa_decode(ctypes.byref(desc), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                           int(block_tables.shape[1]), _ptr(seq_lens), s, float(scale), _ptr(out),
                           _ptr(workspace), int(workspace.numel() * workspace.element_size()),
                           _stream(stream)), "pa_decode")


def pa_decode_fused(desc, q, k_new, v_new, k_cache, v_cache, block_tables, seq_lens, scale, out, workspace,
                    stream=None):
    """pa_cache_write of each sequence's new token (rows k_new[s], v_new[s],
    at position seq_lens[s] - 1 through its block table) and pa_decode, in
    one launch."""
    s = int(seq_lens.shape[0])
    _check(lib().pa_decode_fused(ctypes.byref(desc), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                 _ptr(v_cache), _ptr(block_tables), int(block_tables.shape[1]), _ptr(seq_lens), s,
                                 float(scale), _ptr(out), _ptr(workspace),
                                 int(workspace.numel() * workspace.element_size()), _stream(stream)),
           "pa_decode_fused")


def pa_decode_static(desc, q, k_cache, v_cache, block_tables, seq_lens, scale, out, stream=None):
    """pa_decode without a workspace: the scratch is a fixed 8 MiB area built
    into the library, for callers that cannot allocate device memory."""
    s = int(seq_lens.shape[0])
    _check(lib().pa_decode_static(ctypes.byref(desc), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
                                  int(block_tables.shape[1]), _ptr(seq_lens), s, float(scale), _ptr(out),
                                  _stream(stream)), "pa_decode_static")


def pa_decode_chunked_prefill(desc, q, k_cache, v_cache, block_tables, query_start_loc, seq_lens,
                              max_q_len, scale, out, workspace, stream=None):
    """A mixed step: sequence s owns rows query_start_loc[s]..query_start_loc[s+1]-1 (causal)."""
    s = int(seq_lens.shape[0])
    _check(lib().pa_decode_chunked_prefill(
        ctypes.byref(desc), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables),
        int(block_tables.shape[1]), _ptr(query_start_loc), _ptr(seq_lens), s, int(q.shape[0]),
        int(max_q_len), float(scale), _ptr(out), _ptr(workspace),
        int(workspace.numel() * workspace.element_size()), _stream(stream)),
        "pa_decode_chunked_prefill")


class PrefixGroups:
    """Shared prefixes of a decode batch (pa_prefix_groups): CSR prefix_start
    / prefix_members, prefix_blocks, and per sequence seq_prefix / seq_slot
    (-1 outside any prefix), as int32 tensors on the host."""

    def __init__(self, block_tables, seq_lens, block_size):
        bt = block_tables.detach().cpu().contiguous().to(torch.int32)
        sl = seq_lens.detach().cpu().contiguous().to(torch.int32)
        n = int(sl.shape[0])
        self.prefix_start = torch.zeros(n + 1, dtype=torch.int32)
        self.prefix_members = torch.zeros(max(1, n), dtype=torch.int32)
        self.prefix_blocks = torch.zeros(max(1, n), dtype=torch.int32)
        self.seq_prefix = torch.zeros(max(1, n), dtype=torch.int32)
        self.seq_slot = torch.zeros(max(1, n), dtype=torch.int32)
        np_, nm = ctypes.c_int32(), ctypes.c_int32()
        _check(lib().pa_prefix_groups(_ptr(bt), int(bt.shape[1]), _ptr(sl), n, int(block_size),
                                      _ptr(self.prefix_start), _ptr(self.prefix_members), _ptr(self.prefix_blocks),
                                      _ptr(self.seq_prefix), _ptr(self.seq_slot), ctypes.byref(np_),
                                      ctypes.byref(nm)), "pa_prefix_groups")
        self.num_prefixes, self.num_members = np_.value, nm.value
        self.max_prefix_blocks = int(self.prefix_blocks[:self.num_prefixes].max()) if self.num_prefixes else 0

    def to(self, device):
        """The arrays pa_decode_prefix reads, on `device` (a dict)."""
        return {k: getattr(self, k).to(device) for k in
                ("prefix_start", "prefix_members", "prefix_blocks", "seq_prefix", "seq_slot")}


def pa_decode_prefix_workspace_size(desc, num_seqs, num_members, max_prefix_blocks) -> int:
    n = int(lib().pa_decode_prefix_workspace_size(ctypes.byref(desc), int(num_seqs), int(num_members),
                                                  int(max_prefix_blocks)))
    if n == 0:
        raise PaError(1, "pa_decode_prefix_workspace_size: " + lib().pa_last_error().decode())
    return n


def pa_decode_prefix(desc, q, k_cache, v_cache, block_tables, seq_lens, groups, dev_groups, scale, out,
                     workspace, stream=None):
    """pa_decode with each shared prefix attended once for all its sequences
    (groups: a PrefixGroups; dev_groups: its arrays on the device)."""
    s = int(seq_lens.shape[0])
    g = dev_groups
    _check(lib().pa_decode_prefix(
        ctypes.byref(desc), _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), int(block_tables.shape[1]),
        _ptr(seq_lens), s, _ptr(g["prefix_start"]), _ptr(g["prefix_members"]), _ptr(g["prefix_blocks"]),
        _ptr(g["seq_prefix"]), _ptr(g["seq_slot"]), int(groups.num_prefixes), int(groups.num_members),
        int(groups.max_prefix_blocks), float(scale), _ptr(out), _ptr(workspace),
        int(workspace.numel() * workspace.element_size()), _stream(stream)), "pa_decode_prefix")


def default_scale(head_dim):
    return 1.0 / math.sqrt(head_dim)


class BlockPool:
    """Host block pool (pa_pool_*): free_block_queue, ref_cnt, prefix sharing,
    fork with copy-on-write."""

    def __init__(self, num_blocks, block_size, initial_free_order=None):
        self._lib = lib()
        h = ctypes.c_void_p()
        arr = None
        if initial_free_order is not None:
            order = [int(b) for b in initial_free_order]
            if len(order) != num_blocks:
                raise PaError(1, "initial_free_order must have num_blocks entries")
            arr = (ctypes.c_int32 * num_blocks)(*order)
        _check(self._lib.pa_pool_create(int(num_blocks), int(block_size), arr, ctypes.byref(h)),
               "pa_pool_create")
        self._h = h
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self):
        if self._h:
            self._lib.pa_pool_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add_seq(self, seq_id, num_tokens, token_ids=None) -> int:
        arr = None
        if token_ids is not None:
            ids = [int(t) for t in token_ids]
            arr = (ctypes.c_int32 * len(ids))(*ids)
        cached = ctypes.c_int32(0)
        _check(self._lib.pa_pool_add_seq(self._h, int(seq_id), arr, int(num_tokens), ctypes.byref(cached)),
               "pa_pool_add_seq")
        return cached.value

    def append(self, seq_id, n_new):
        out = (ctypes.c_int64 * max(1, n_new))()
        _check(self._lib.pa_pool_append(self._h, int(seq_id), int(n_new), out), "pa_pool_append")
        return list(out[:n_new])

    def fork(self, parent_id, child_id):
        """child_id shares every block of parent_id (copy on write)."""
        _check(self._lib.pa_pool_fork(self._h, int(parent_id), int(child_id)), "pa_pool_fork")

    def take_copies(self):
        """The (src, dst) block copies queued by copy-on-write, oldest first."""
        n = ctypes.c_int32()
        self._lib.pa_pool_take_copies(self._h, None, None, 0, ctypes.byref(n))
        src = (ctypes.c_int32 * max(1, n.value))()
        dst = (ctypes.c_int32 * max(1, n.value))()
        _check(self._lib.pa_pool_take_copies(self._h, src, dst, n.value, ctypes.byref(n)), "pa_pool_take_copies")
        return [(src[i], dst[i]) for i in range(n.value)]

    def slots(self, seq_id, start, n):
        out = (ctypes.c_int64 * max(1, n))()
        _check(self._lib.pa_pool_slots(self._h, int(seq_id), int(start), int(n), out), "pa_pool_slots")
        return list(out[:n])

    def free_seq(self, seq_id):
        _check(self._lib.pa_pool_free_seq(self._h, int(seq_id)), "pa_pool_free_seq")

    def num_tokens(self, seq_id):
        n = ctypes.c_int32()
        _check(self._lib.pa_pool_num_tokens(self._h, int(seq_id), ctypes.byref(n)), "pa_pool_num_tokens")
        return n.value

    def block_table(self, seq_id):
        n = ctypes.c_int32()
        self._lib.pa_pool_block_table(self._h, int(seq_id), None, 0, ctypes.byref(n))
        out = (ctypes.c_int32 * max(1, n.value))()
        _check(self._lib.pa_pool_block_table(self._h, int(seq_id), out, n.value, ctypes.byref(n)),
               "pa_pool_block_table")
        return list(out[:n.value])

    def block_tables(self, seq_ids, max_blocks):
        """Padded int32 table [len(seq_ids)][max_blocks] as a CPU torch tensor."""
        ids = (ctypes.c_int64 * max(1, len(seq_ids)))(*[int(s) for s in seq_ids])
        out = torch.empty((len(seq_ids), max_blocks), dtype=torch.int32)
        _check(self._lib.pa_pool_block_tables(self._h, ids, len(seq_ids), int(max_blocks),
                                              ctypes.c_void_p(out.data_ptr())), "pa_pool_block_tables")
        return out

    def ref_cnt(self, block):
        return int(self._lib.pa_pool_ref_cnt(self._h, int(block)))

    def num_free(self):
        return int(self._lib.pa_pool_num_free(self._h))

    def free_order(self):
        n = ctypes.c_int32()
        cap = self.num_blocks
        out = (ctypes.c_int32 * max(1, cap))()
        _check(self._lib.pa_pool_free_order(self._h, out, cap, ctypes.byref(n)), "pa_pool_free_order")
        return list(out[:n.value])
