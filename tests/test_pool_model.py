"""Pins for the oracle's memory arithmetic and block-pool model: the pages'
worked example, closed forms, and hand-derived traces."""
import json
import os

import pytest

from oracle import admission as adm
from oracle.pool_model import BlockPoolModel, PoolModelError, block_hash, fnv1a64

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fragmentation_example.json")


def test_worked_example_4_vs_13():
    ex = json.load(open(GOLDEN))
    bs, pool, max_len, lens = ex["block"], ex["pool"], ex["max_len"], ex["lens"]
    assert adm.contiguous_capacity(pool, max_len, bs) == ex["printed_contiguous"] == 4
    assert adm.paged_admission_fcfs(lens, pool, bs) == ex["printed_paged"] == 13
    # the listing's own loop (skip a request that does not fit, keep going)
    assert adm.paged_admission_skip(lens, pool, bs) == 14
    assert [adm.blocks_for(n, bs) for n in lens] == [3, 8, 19, 4, 14, 6, 12, 3, 10, 5, 4, 27, 3, 16, 6, 7]


def test_worked_example_through_the_pool_model():
    ex = json.load(open(GOLDEN))
    pool = BlockPoolModel(ex["pool"], ex["block"])
    admitted = 0
    for i, n in enumerate(ex["lens"]):
        try:
            pool.add_seq(i, n)
        except PoolModelError as e:
            assert e.code == "NO_BLOCKS"
            break
        admitted += 1
    assert admitted == 13
    assert pool.num_free() == 128 - 118


def test_blocks_for_closed_form_and_waste_bound():
    for bs in (1, 16, 32):
        for n in range(0, 1001):
            m = adm.blocks_for(n, bs)
            assert m == -(-n // bs)
            if n > 0:
                assert 0 <= m * bs - n < bs  # at most one partially filled block
        pool = BlockPoolModel(1001 * 1001, bs) if bs == 1 else BlockPoolModel(40000, bs)
        for n in range(0, 1001, 7):
            pool.add_seq(n, n)
            assert len(pool.block_table(n)) == adm.blocks_for(n, bs)


def test_block_bytes_formula():
    assert adm.block_bytes(16, 8, 128, 2) == 65536  # bf16, 8 KV heads, d128
    assert adm.block_bytes(16, 8, 128, 1) == 32768  # fp8 halves it
    assert adm.block_bytes(32, 8, 128, 2) == 2 * adm.block_bytes(16, 8, 128, 2)
    assert adm.block_bytes(16, 2, 64, 4) == 2 * 16 * 2 * 64 * 4
    # one request's cache, per layer, equals its blocks' bytes when full
    assert adm.request_kv_bytes(1, 8, 128, 64, 2) == 4 * adm.block_bytes(16, 8, 128, 2)


def test_append_takes_a_block_exactly_when_the_last_is_full():
    pool = BlockPoolModel(10, 4, initial_free_order=[3, 1, 4, 0, 5, 9, 2, 6, 8, 7])
    pool.add_seq("a", 0)
    assert pool.block_table("a") == []
    slots = pool.append("a", 9)
    # positions 0..3 -> block 3, 4..7 -> block 1, 8 -> block 4
    assert slots == [12, 13, 14, 15, 4, 5, 6, 7, 16]
    assert pool.block_table("a") == [3, 1, 4]
    assert pool.append("a", 3) == [17, 18, 19]
    assert pool.num_free() == 7
    assert pool.append("a", 1) == [0]  # block 0 is next in the queue
    assert pool.slots("a", 4, 2) == [4, 5]


def test_lifecycle_ref_cnt_and_free_order():
    pool = BlockPoolModel(6, 2)
    pool.add_seq(1, 5)  # blocks 0,1,2
    pool.add_seq(2, 2)  # block 3
    assert pool.free_order() == [4, 5]
    pool.free_seq(1)  # released in reverse logical order to the tail
    assert pool.free_order() == [4, 5, 2, 1, 0]
    assert pool.ref_cnt[:4] == [0, 0, 0, 1]
    with pytest.raises(PoolModelError) as e:
        pool.free_seq(1)
    assert e.value.code == "INVALID_ARG"
    pool.add_seq(3, 7)  # pops 4,5,2,1
    assert pool.block_table(3) == [4, 5, 2, 1]
    with pytest.raises(PoolModelError) as e:
        pool.add_seq(4, 3)  # needs 2, only block 0 free: nothing changes
    assert e.value.code == "NO_BLOCKS"
    assert pool.free_order() == [0] and 4 not in pool.seqs


def test_prefix_sharing_touch_and_eviction():
    bs = 4
    pool = BlockPoolModel(8, bs)
    prefix = [7, 7, 1, 2, 9, 9, 3, 4]  # two full blocks
    a = prefix + [5, 5, 5]
    b = prefix + [6]
    assert pool.add_seq("a", len(a), a) == 0
    ta = pool.block_table("a")  # [0, 1, 2]
    assert pool.add_seq("b", len(b), b) == 8  # both prefix blocks hit
    tb = pool.block_table("b")
    assert tb[:2] == ta[:2] and tb[2] not in ta
    assert pool.ref_cnt[ta[0]] == 2 and pool.ref_cnt[ta[1]] == 2
    pool.free_seq("a")
    assert pool.ref_cnt[ta[0]] == 1 and pool.ref_cnt[ta[2]] == 0
    pool.free_seq("b")
    # parked with their hashes: a third request still hits, and touch()
    # unlinks them from the free queue
    order_before = pool.free_order()
    assert pool.add_seq("c", 8, prefix) == 8
    assert pool.block_table("c") == ta[:2]
    assert pool.free_order() == [x for x in order_before if x not in ta[:2]]
    # a different prefix misses
    assert pool.add_seq("d", 4, [1, 2, 3, 4]) == 0


def test_reused_block_loses_its_hash():
    pool = BlockPoolModel(2, 2)
    pool.add_seq("a", 2, [1, 2])
    blk = pool.block_table("a")[0]
    pool.free_seq("a")
    pool.add_seq("b", 3)  # pops both blocks; the cached one is evicted
    assert blk in pool.block_table("b")
    pool.free_seq("b")
    assert pool.add_seq("c", 2, [1, 2]) == 0


def test_hash_depends_on_parent_and_tokens():
    h1 = block_hash(0, [1, 2, 3])
    assert h1 != block_hash(0, [1, 2, 4])
    assert h1 != block_hash(1, [1, 2, 3])
    assert h1 == block_hash(0, (1, 2, 3))
    # published FNV-1a 64 test vectors
    assert fnv1a64(b"") == 0xCBF29CE484222325
    assert fnv1a64(b"a") == 0xAF63DC4C8601EC8C
    assert fnv1a64(b"foobar") == 0x85944171F73967E8
    # parent (8 bytes LE) then int32 LE token ids
    assert block_hash(5, [1]) == fnv1a64(bytes([5, 0, 0, 0, 0, 0, 0, 0, 1, 0, 0, 0]))


def test_fork_shares_blocks_and_copies_on_write_when_a_sequence_diverges():
    # hand-derived trace, block size 4, free queue 6 2 5 0 7 1 3 4
    pool = BlockPoolModel(8, 4, initial_free_order=[6, 2, 5, 0, 7, 1, 3, 4])
    pool.add_seq("p", 6)  # positions 0..3 in block 6, 4..5 in block 2 (half full)
    pool.fork("p", "c")
    assert pool.block_table("c") == [6, 2] and pool.num_tokens("c") == 6
    assert pool.ref_cnt[6] == 2 and pool.ref_cnt[2] == 2
    assert pool.take_copies() == []
    # the child writes position 6 into the shared, half-full block 2: it
    # moves to a copy in block 5 (head of the queue) and writes slot 5*4+2
    assert pool.append("c", 1) == [22]
    assert pool.block_table("c") == [6, 5] and pool.block_table("p") == [6, 2]
    assert (pool.ref_cnt[2], pool.ref_cnt[5], pool.ref_cnt[6]) == (1, 1, 2)
    assert pool.take_copies() == [(2, 5)]
    assert pool.take_copies() == []  # taken once
    # the parent is now block 2's only owner: it writes in place
    assert pool.append("p", 2) == [10, 11]
    assert pool.take_copies() == []
    # a full shared block is never copied: the next token opens block 0
    pool.fork("p", "d")
    assert pool.append("d", 1) == [0]
    assert pool.block_table("d") == [6, 2, 0] and pool.take_copies() == []
    assert (pool.ref_cnt[6], pool.ref_cnt[2]) == (3, 2)
    # release walks blocks in reverse: c's block 5 goes to the tail, 6 stays
    pool.free_seq("c")
    assert pool.free_order() == [7, 1, 3, 4, 5] and pool.ref_cnt[6] == 2


def test_copy_on_write_is_all_or_nothing():
    pool = BlockPoolModel(2, 4)
    pool.add_seq("a", 5)  # blocks 0 (full) and 1 (one token)
    pool.fork("a", "b")
    with pytest.raises(PoolModelError) as e:
        pool.append("b", 1)  # the copy needs a block and none is free
    assert e.value.code == "NO_BLOCKS"
    assert pool.block_table("b") == [0, 1] and pool.ref_cnt == [2, 2]
    assert pool.num_tokens("b") == 5 and pool.take_copies() == []
    with pytest.raises(PoolModelError):
        pool.fork("a", "b")  # the child exists
    with pytest.raises(PoolModelError):
        pool.fork("zz", "e")  # no such parent
    pool.append("b", 0)  # nothing to write: no copy, no block
    assert pool.take_copies() == []


def test_fork_of_an_empty_sequence_and_release_of_both():
    pool = BlockPoolModel(3, 4)
    pool.add_seq("a", 0)
    pool.fork("a", "b")
    assert pool.block_table("b") == [] and pool.append("b", 2) == [0, 1]
    assert pool.take_copies() == []  # no shared block to copy
    pool.free_seq("a")
    pool.free_seq("b")
    assert pool.free_order() == [1, 2, 0] and pool.ref_cnt == [0, 0, 0]
