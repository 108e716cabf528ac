"""The C++ block pool (product) against the oracle's pool model: identical
block tables, slots, ref_cnts and free-queue order, bit for bit, on scripted
and random traces and on every workload's admission."""
import numpy as np
import pytest

import pa_workloads as W
from oracle.pool_model import BlockPoolModel, PoolModelError
from oracle.workload import pool_tables
from paged_kv_cache_452_b200 import BlockPool, PaError

CODES = {"INVALID_ARG": 1, "NO_BLOCKS": 3, "STATE": 5}


def same_state(c: BlockPool, m: BlockPoolModel):
    assert c.free_order() == m.free_order()
    assert c.num_free() == m.num_free()
    assert [c.ref_cnt(b) for b in range(m.num_blocks)] == m.ref_cnt
    for sid in m.seqs:
        assert c.block_table(sid) == m.block_table(sid)
        assert c.num_tokens(sid) == m.num_tokens(sid)


def both(c, m, op, *args):
    """Run one operation on both pools; they must agree on result or error."""
    try:
        r_m = getattr(m, op)(*args)
        err_m = None
    except PoolModelError as e:
        r_m, err_m = None, CODES[e.code]
    try:
        r_c = getattr(c, op)(*args)
        err_c = None
    except PaError as e:
        r_c, err_c = None, e.code
    assert err_c == err_m, (op, args, err_c, err_m)
    if err_m is None and op != "free_seq":
        assert r_c == r_m, (op, args)
    return err_m


def test_scripted_trace_matches_model():
    order = [5, 2, 7, 0, 1, 6, 3, 4]
    c, m = BlockPool(8, 4, order), BlockPoolModel(8, 4, order)
    both(c, m, "add_seq", 1, 6, None)
    both(c, m, "append", 1, 3)
    both(c, m, "add_seq", 2, 8, [1, 2, 3, 4, 5, 6, 7, 8])
    both(c, m, "add_seq", 3, 9, [1, 2, 3, 4, 5, 6, 7, 8, 9])  # shares two blocks
    same_state(c, m)
    assert both(c, m, "add_seq", 4, 20, None) == 3  # no room
    both(c, m, "free_seq", 2)
    both(c, m, "free_seq", 1)
    same_state(c, m)
    assert both(c, m, "free_seq", 1) == 1
    both(c, m, "add_seq", 5, 8, [1, 2, 3, 4, 5, 6, 7, 8])
    both(c, m, "slots", 5, 2, 5)
    assert both(c, m, "slots", 5, 6, 5) == 1
    same_state(c, m)


def test_fork_and_copy_on_write_trace_matches_model():
    order = [6, 2, 5, 0, 7, 1, 3, 4]
    c, m = BlockPool(8, 4, order), BlockPoolModel(8, 4, order)
    both(c, m, "add_seq", 1, 6, None)
    both(c, m, "fork", 1, 2)
    same_state(c, m)
    both(c, m, "append", 2, 1)  # copy-on-write of the half-full shared block
    assert both(c, m, "take_copies") is None
    both(c, m, "append", 1, 2)
    both(c, m, "fork", 1, 3)
    both(c, m, "append", 3, 1)  # the shared block is full: no copy
    both(c, m, "take_copies")
    same_state(c, m)
    assert both(c, m, "fork", 1, 3) == 1  # the child exists
    assert both(c, m, "fork", 99, 5) == 1  # no such parent
    both(c, m, "free_seq", 2)
    both(c, m, "free_seq", 1)
    same_state(c, m)
    # no free block left for the copy: all-or-nothing
    c2, m2 = BlockPool(2, 4), BlockPoolModel(2, 4)
    both(c2, m2, "add_seq", 1, 5, None)
    both(c2, m2, "fork", 1, 2)
    assert both(c2, m2, "append", 2, 1) == 3
    assert both(c2, m2, "take_copies") is None
    same_state(c2, m2)


@pytest.mark.parametrize("seed", range(6))
def test_random_traces_match_model(seed):
    g = np.random.default_rng(seed)
    nb, bs = int(g.integers(8, 64)), int(g.choice([1, 4, 16]))
    order = g.permutation(nb).tolist()
    c, m = BlockPool(nb, bs, order), BlockPoolModel(nb, bs, order)
    prefixes = [g.integers(0, 5, size=3 * bs).tolist() for _ in range(3)]
    live, next_id = [], 0
    for _ in range(400):
        op = g.integers(0, 6)
        if op == 0 or not live:
            n = int(g.integers(0, 4 * bs))
            toks = None
            if g.random() < 0.6:
                pre = prefixes[int(g.integers(0, 3))]
                toks = (pre + g.integers(0, 5, size=max(0, n)).tolist())[:n]
            if both(c, m, "add_seq", next_id, n, toks) is None:
                live.append(next_id)
            next_id += 1
        elif op == 1:
            sid = live[int(g.integers(0, len(live)))]
            both(c, m, "append", sid, int(g.integers(0, 2 * bs)))
        elif op == 2:
            sid = live.pop(int(g.integers(0, len(live))))
            both(c, m, "free_seq", sid)
        elif op == 3:
            sid = live[int(g.integers(0, len(live)))]
            n = m.num_tokens(sid)
            if n:
                a = int(g.integers(0, n))
                both(c, m, "slots", sid, a, int(g.integers(0, n - a + 1)))
        elif op == 4:  # fork; appends to either side then copy on write
            if both(c, m, "fork", live[int(g.integers(0, len(live)))], next_id) is None:
                live.append(next_id)
            next_id += 1
        else:
            both(c, m, "take_copies")
        same_state(c, m)


@pytest.mark.parametrize("name", ["tiny_fp32", "gqa_bf16", "prefix_bf16", "fp8_long", "mixed_prefill_bs16",
                                  "mixed_prefill_bs32", "long_prefix_bf16"])
@pytest.mark.parametrize("size", ["small", "full"])
def test_workload_admission_matches_model(name, size):
    wl = W.make(name, size)
    tables, step_slots, num_cached, model = pool_tables(wl)
    c = BlockPool(wl.num_blocks, wl.block_size, wl.free_order)
    cached = [c.add_seq(s, int(wl.context_lens[s]), wl.token_ids(s)) for s in range(wl.num_seqs)]
    slots = []
    for s in range(wl.num_seqs):
        slots.extend(c.append(s, int(wl.q_lens[s])))
    assert cached == num_cached
    assert np.array_equal(np.asarray(slots), step_slots)
    assert np.array_equal(c.block_tables(list(range(wl.num_seqs)), tables.shape[1]).numpy(), tables)
    assert c.free_order() == model.free_order()
    if name == "prefix_bf16":
        shared = tables[0, : wl.prefix_len // wl.block_size]
        assert all(c.ref_cnt(int(b)) == int(wl.sharing.sum()) for b in shared)
        # the first sharing sequence fills the prefix blocks, the others hit them
        hits = [n for n, sh in zip(cached, wl.sharing) if sh]
        assert hits[0] == 0 and all(n == wl.prefix_len for n in hits[1:])
        assert all(n == 0 for n, sh in zip(cached, wl.sharing) if not sh)
    if name == "tiny_fp32":
        # the fully specified configuration: 3 + 8 + 19 + 4 blocks in
        # admission order, then the decode token of each full sequence (128
        # and 64 tokens) starts a new block: the 35th and 36th of the
        # permutation
        perm = wl.free_order.tolist()
        assert [len(r[r >= 0]) for r in tables] == [3, 9, 19, 5]
        assert tables[0, :3].tolist() == perm[:3]
        assert tables[1, 8] == perm[34] and tables[3, 4] == perm[35]
