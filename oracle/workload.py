"""Expected results of one layer-step of a workload, from the oracle alone.
TEST INFRASTRUCTURE ONLY.

Given a ``pa_workloads`` workload (seeded draws only), this runs the pool
model to get block tables and slots, the C oracle's cache write for the
context and the step's new tokens, and the oracle's attention for the step's
query rows.  ``seqs`` restricts the K/V work to some sequences (sampled
checks at full size): their physical blocks are renumbered into a compact
pool, which changes no result because the output does not depend on where the
blocks sit.
"""
import numpy as np
import torch

from . import attention, cache_write, new_caches
from .pool_model import BlockPoolModel


def _raw(t: torch.Tensor) -> np.ndarray:
    """Storage bits of a CPU tensor: float32 values or bf16 bit patterns."""
    if t.dtype == torch.float32:
        return t.contiguous().numpy()
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def pool_tables(wl):
    """Pool model replay: admit every sequence in order, then append this
    step's tokens; returns tables [S][max_blocks] (-1 padded), step slots,
    per-sequence cached-token counts and the final model."""
    S = wl.num_seqs
    m = BlockPoolModel(wl.num_blocks, wl.block_size, [int(b) for b in wl.free_order])
    num_cached = []
    for s in range(S):
        tok = wl.token_ids(s)
        num_cached.append(m.add_seq(s, int(wl.context_lens[s]), None if tok is None else tok.tolist()))
    step_slots = []
    for s in range(S):
        step_slots.extend(m.append(s, int(wl.q_lens[s])))
    nblk = [len(m.block_table(s)) for s in range(S)]
    tables = np.full((S, max(1, max(nblk) if nblk else 1)), -1, dtype=np.int32)
    for s in range(S):
        tables[s, :nblk[s]] = m.block_table(s)
    return tables, np.asarray(step_slots, dtype=np.int64), num_cached, m


def prepare(wl, seqs=None):
    """Pool replay and input draws for `seqs` (everything but the oracle's
    own arithmetic): tables, compact renumbering, raw K/V/q arrays, slots."""
    tables, step_slots, num_cached, model = pool_tables(wl)
    S, bs = wl.num_seqs, wl.block_size
    seqs = list(range(S)) if seqs is None else sorted(int(s) for s in seqs)
    qsl = np.concatenate([[0], np.cumsum(wl.q_lens)]).astype(np.int64)
    used = sorted({int(b) for s in seqs for b in tables[s] if b >= 0})
    remap = {b: i for i, b in enumerate(used)}
    ctab = np.full((S, tables.shape[1]), 0, dtype=np.int32)
    for s in seqs:
        for i, b in enumerate(tables[s]):
            if b >= 0:
                ctab[s, i] = remap[int(b)]

    def slots_of(s, positions):
        return np.array([ctab[s, p // bs] * bs + p % bs for p in positions], dtype=np.int64)

    writes = []  # (k raw, v raw, compact slots)
    for s in seqs:
        n = int(wl.context_lens[s])
        if n:
            k, v = wl.prior_kv(s)
            writes.append((_raw(k), _raw(v), slots_of(s, range(n))))
    k_new, v_new = wl.new_kv()
    kn, vn = _raw(k_new), _raw(v_new)
    rows, row_seq, row_pos = [], [], []
    for s in seqs:
        c = int(wl.context_lens[s])
        r0, r1 = int(qsl[s]), int(qsl[s + 1])
        if r1 > r0:
            writes.append((kn[r0:r1], vn[r0:r1], slots_of(s, range(c, c + r1 - r0))))
        for r in range(r0, r1):
            rows.append(r)
            row_seq.append(s)
            row_pos.append(c + r - r0)
    q = wl.queries().to(torch.float64).numpy()[rows] if rows else np.zeros((0, wl.num_q_heads, wl.head_dim))
    return {
        "wl": wl, "tables": tables, "step_slots": step_slots, "num_cached": num_cached, "model": model,
        "seqs": seqs, "remap": remap, "compact_tables": ctab, "num_compact": max(1, len(used)),
        "writes": writes, "rows": np.asarray(rows, dtype=np.int64), "row_seq": row_seq, "row_pos": row_pos,
        "q": q,
    }


def compute(prep, num_threads=0):
    """The oracle's arithmetic for a prepared step: cache writes into a fresh
    compact pool, then attention for every prepared row."""
    wl = prep["wl"]
    kc, vc = new_caches(prep["num_compact"], wl.num_kv_heads, wl.block_size, wl.head_dim, wl.kv_dtype)
    for k, v, sl in prep["writes"]:
        cache_write(k, v, sl, kc, vc, wl.q_dtype, wl.kv_dtype, wl.k_scale, wl.v_scale)
    if len(prep["rows"]):
        out = attention(prep["q"], prep["row_seq"], prep["row_pos"], prep["compact_tables"], kc, vc, wl.kv_dtype,
                        wl.num_q_heads, 1.0 / np.sqrt(wl.head_dim), wl.k_scale, wl.v_scale, num_threads)
    else:
        out = prep["q"]
    return kc, vc, out


def expected(wl, seqs=None, num_threads=0):
    prep = prepare(wl, seqs)
    kc, vc, out = compute(prep, num_threads)
    res = dict(prep)
    res.update({"k_cache": kc, "v_cache": vc, "out": out})
    return res
