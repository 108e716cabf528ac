"""Host-side checks of the C ABI library (no GPU needed): every declared
symbol is exported, the byte accounting matches the pages' formula, and bad
arguments are rejected before anything is launched."""
import ctypes
import os
import re

import pytest

import paged_kv_cache_452_b200 as pa
from oracle import admission

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "include", "pa.h")


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_symbol_is_exported_and_bound():
    names = declared_functions()
    assert len(names) >= 20
    L = ctypes.CDLL(pa.LIB_PATH)
    for n in names:
        assert hasattr(L, n), n
    from paged_kv_cache_452_b200._lib import SIGNATURES
    assert set(SIGNATURES) == set(names)


def test_version_and_error_string():
    assert b"sm_100a" in pa.lib().pa_version()
    assert pa.lib().pa_last_error() == b""


@pytest.mark.parametrize("bs,hkv,d,kv,eb", [(16, 8, 128, "bf16", 2), (16, 8, 128, "e4m3", 1),
                                             (32, 8, 128, "bf16", 2), (16, 2, 64, "f32", 4)])
def test_block_bytes_matches_formula(bs, hkv, d, kv, eb):
    desc = pa.CacheDesc.make(100, bs, hkv, hkv * 4, d, kv, "bf16" if kv != "f32" else "f32", 0.5, 0.5)
    assert pa.pa_block_bytes(desc) == admission.block_bytes(bs, hkv, d, eb)


def _call_write(desc, n=1, ptr=16):
    slots = ctypes.c_void_p(ptr)
    return pa.lib().pa_cache_write(ctypes.byref(desc) if desc is not None else None, ptr, ptr, slots, n,
                                   ptr, ptr, None)


def test_cache_write_rejects_bad_arguments_on_host():
    good = pa.CacheDesc.make(16, 16, 2, 4, 64, "bf16", "bf16")
    assert _call_write(None) == 1
    assert b"desc is NULL" in pa.lib().pa_last_error()
    assert _call_write(good, n=0) == 0  # nothing to do, nothing launched
    assert _call_write(good, n=-1) == 1
    assert _call_write(good, ptr=18) == 1  # misaligned
    bad_bs = pa.CacheDesc.make(16, 8, 2, 4, 64, "bf16", "bf16")
    assert _call_write(bad_bs) == 2  # block size 8 not built
    bad_d = pa.CacheDesc.make(16, 16, 2, 4, 96, "bf16", "bf16")
    assert _call_write(bad_d) == 2
    bad_g = pa.CacheDesc.make(16, 16, 3, 4, 64, "bf16", "bf16")
    assert _call_write(bad_g) == 1  # 4 query heads over 3 KV heads
    mixed = pa.CacheDesc.make(16, 16, 2, 4, 64, "f32", "bf16")
    assert _call_write(mixed) == 2  # bf16 rows into an fp32 pool
    no_scale = pa.CacheDesc.make(16, 16, 2, 4, 128, "e4m3", "bf16", 0.0, 1.0)
    assert _call_write(no_scale) == 1


def test_copy_blocks_rejects_bad_arguments_on_host():
    desc = pa.CacheDesc.make(16, 16, 2, 8, 128, "bf16", "bf16")
    L = pa.lib()
    p = 256
    assert L.pa_copy_blocks(None, p, p, 1, p, p, None) == 1
    assert L.pa_copy_blocks(ctypes.byref(desc), p, p, -1, p, p, None) == 1
    assert L.pa_copy_blocks(ctypes.byref(desc), p, p, 0, p, p, None) == 0  # nothing to copy, nothing launched
    assert L.pa_copy_blocks(ctypes.byref(desc), None, p, 2, p, p, None) == 1
    assert b"NULL" in L.pa_last_error()
    assert L.pa_copy_blocks(ctypes.byref(desc), p + 2, p, 2, p, p, None) == 1  # int32 ids misaligned
    assert L.pa_copy_blocks(ctypes.byref(desc), p, p, 2, p, p + 8, None) == 1  # pool not 16-byte aligned
    assert b"misaligned" in L.pa_last_error()


def test_pool_fork_and_copy_queue_errors():
    pool = pa.BlockPool(4, 4)
    with pytest.raises(pa.PaError) as e:
        pool.fork(1, 2)  # no parent
    assert e.value.code == 1
    pool.add_seq(1, 3)
    pool.fork(1, 2)
    with pytest.raises(pa.PaError):
        pool.fork(1, 2)  # the child exists
    pool.append(2, 1)  # copy-on-write of the shared, partly filled block
    L = pa.lib()
    n = ctypes.c_int32()
    assert L.pa_pool_take_copies(pool._h, None, None, 0, ctypes.byref(n)) == 1 and n.value == 1
    assert pool.take_copies() == [(0, 1)]  # kept after the refusal; block 1 is next in the queue
    assert pool.take_copies() == []


def test_decode_rejects_bad_arguments_on_host():
    desc = pa.CacheDesc.make(16, 16, 2, 8, 128, "bf16", "bf16")
    L = pa.lib()
    p = 256
    rc = L.pa_decode(ctypes.byref(desc), p, p, p, p, 4, p, -1, 1.0, p, p, 1 << 20, None)
    assert rc == 1
    rc = L.pa_decode(ctypes.byref(desc), p, p, p, p, 4, p, 0, 1.0, p, p, 1 << 20, None)
    assert rc == 0  # empty batch
    rc = L.pa_decode(ctypes.byref(desc), p, p, p, p, 4, p, 3, 1.0, p, p + 16, 1 << 20, None)
    assert rc == 1 and b"misaligned" in L.pa_last_error()
    rc = L.pa_decode(ctypes.byref(desc), None, p, p, p, 4, p, 3, 1.0, p, p, 1 << 20, None)
    assert rc == 1


def test_static_decode_checks_arguments_before_touching_its_scratch():
    """pa_decode_static refuses what pa_decode refuses, on the host, before
    it clears any scratch: a batch past 16384 sequences (whatever its
    scratch size: a CUDA-core desc needs only the 256-byte error word),
    NULL or misaligned pointers."""
    L = pa.lib()
    p = 256
    simt = pa.CacheDesc.make(16, 16, 128, 128, 64, "f32", "f32")  # group 1: the CUDA-core path
    rc = L.pa_decode_static(ctypes.byref(simt), p, p, p, p, 1, p, 16385, 1.0, p, None)
    assert rc == 2 and b"16384" in L.pa_last_error()
    tc = pa.CacheDesc.make(16, 16, 2, 8, 128, "bf16", "bf16")
    assert L.pa_decode_static(ctypes.byref(tc), p, p, p, p, 1, p, 20000, 1.0, p, None) == 2
    assert L.pa_decode_static(ctypes.byref(tc), None, p, p, p, 1, p, 3, 1.0, p, None) == 1
    assert L.pa_decode_static(ctypes.byref(tc), p + 2, p, p, p, 1, p, 3, 1.0, p, None) == 1
    assert b"misaligned" in L.pa_last_error()
    assert L.pa_decode_static(ctypes.byref(tc), p, p, p, p, 1, p, 0, 1.0, p, None) == 0  # empty batch
    assert L.pa_decode_static(None, p, p, p, p, 1, p, 3, 1.0, p, None) == 1


def _groups_model(tables, lens, bs):
    """Plain restatement of the grouping rule: sequences whose rows start
    with the same block, two or more; the prefix is the longest leading run
    every member shares, cut to keep each member's last token outside."""
    cap = [0 if n <= 0 else min((n - 1) // bs, len(r)) for r, n in zip(tables, lens)]
    by_first = {}
    for s, r in enumerate(tables):
        if cap[s] >= 1:
            by_first.setdefault(r[0], []).append(s)
    out = []
    for mem in sorted(by_first.values(), key=lambda m: m[0]):
        if len(mem) < 2:
            continue
        k = min(cap[s] for s in mem)
        while k > 0 and any(tables[s][:k] != tables[mem[0]][:k] for s in mem):
            k -= 1
        if k >= 1:
            out.append((mem, k))
    return out


def test_prefix_groups_match_a_plain_model():
    import numpy as np
    import torch
    g = np.random.default_rng(7)
    for trial in range(200):
        bs = int(g.choice([16, 32]))
        n = int(g.integers(0, 12))
        width = 8
        base = [list(g.permutation(100)[:width]) for _ in range(3)]
        tables, lens = [], []
        for _ in range(n):
            r = list(base[int(g.integers(0, 3))]) if g.random() < 0.7 else list(g.permutation(100)[:width] + 100)
            cut = int(g.integers(0, width + 1))
            r[cut:] = list(g.permutation(100)[:width - cut] + 200)
            tables.append(r)
            lens.append(int(g.integers(0, width * bs + 1)))
        bt = torch.tensor(tables, dtype=torch.int32).reshape(n, width)
        grp = pa.PrefixGroups(bt, torch.tensor(lens, dtype=torch.int32), bs)
        want = _groups_model([list(map(int, r)) for r in tables], lens, bs)
        got = []
        for p in range(grp.num_prefixes):
            mem = grp.prefix_members[int(grp.prefix_start[p]):int(grp.prefix_start[p + 1])].tolist()
            got.append((mem, int(grp.prefix_blocks[p])))
        assert got == want, (trial, got, want)
        for p, (mem, _) in enumerate(got):
            for j, s in enumerate(mem):
                assert int(grp.seq_prefix[s]) == p and int(grp.prefix_members[int(grp.seq_slot[s])]) == s
        members = {s for mem, _ in got for s in mem}
        assert all(int(grp.seq_prefix[s]) == -1 for s in range(n) if s not in members)
