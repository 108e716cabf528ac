"""Drive one attention layer-step through the library: admit sequences into
the C++ block pool, write their cached context with pa_cache_write, append
this step's tokens, then write and attend.

``setup(workload, device)`` accepts any object with the attributes of
``pa_workloads.Workload`` (lengths, free-list order, per-sequence draws); it
only moves data and calls the library.
"""
from dataclasses import dataclass
from typing import List, Optional

import numpy as np
import torch

from . import (PA_FP8_E4M3, BlockPool, CacheDesc, PrefixGroups, alloc_cache, alloc_workspace, default_scale,
               pa_cache_write, pa_decode, pa_decode_chunked_prefill, pa_decode_fused, pa_decode_prefix,
               pa_decode_prefix_workspace_size, pa_decode_workspace_size, pa_prefill_workspace_size)

# sentinel stored in unwritten cache elements so a stray read shows up
_SENTINEL = {0: float("nan"), 1: float("nan"), 2: 0x7F}


@dataclass
class DeviceBatch:
    desc: CacheDesc
    pool: BlockPool
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    tables: torch.Tensor  # device int32 [S][max_blocks]
    seq_lens: torch.Tensor  # device int32 [S], tokens attended after the step
    qsl: Optional[torch.Tensor]  # device int32 [S+1], None for a pure decode step
    q: torch.Tensor  # device [rows][Hq][D]
    k_new: torch.Tensor  # device [rows][Hkv][D]
    v_new: torch.Tensor
    slots: torch.Tensor  # device int64 [rows]
    out: torch.Tensor  # device [rows][Hq][D]
    workspace: torch.Tensor
    max_q_len: int
    scale: float
    tables_host: torch.Tensor
    slots_host: torch.Tensor
    prior_slots: List[np.ndarray]  # per sequence, slots of the context tokens written at setup
    num_cached: List[int]  # per sequence, tokens covered by shared blocks

    @property
    def decode_only(self):
        return self.qsl is None


def _desc_for(wl, device=None):
    """The pool's desc; per-kv-head e4m3 scales (an array in the workload)
    go to the device as fp32 tensors that the desc keeps alive."""
    ks, vs = wl.k_scale, wl.v_scale
    kh = vh = None
    if np.ndim(ks) == 1:
        kh, ks = torch.from_numpy(np.asarray(ks, dtype=np.float32)).to(device), 1.0
    if np.ndim(vs) == 1:
        vh, vs = torch.from_numpy(np.asarray(vs, dtype=np.float32)).to(device), 1.0
    return CacheDesc.make(wl.num_blocks, wl.block_size, wl.num_kv_heads, wl.num_q_heads, wl.head_dim,
                          wl.kv_dtype, wl.q_dtype, ks, vs, kh, vh)


def setup(wl, device, write_chunk_tokens: int = 1 << 18) -> DeviceBatch:
    S = wl.num_seqs
    pool = BlockPool(wl.num_blocks, wl.block_size, wl.free_order)
    fp8 = wl.kv_dtype == "e4m3"
    num_cached, prior_slots = [], []
    for s in range(S):
        c = pool.add_seq(s, int(wl.context_lens[s]), wl.token_ids(s))
        num_cached.append(c)
        prior_slots.append(np.asarray(pool.slots(s, c, int(wl.context_lens[s]) - c), dtype=np.int64))
    step_slots = []
    for s in range(S):
        step_slots.extend(pool.append(s, int(wl.q_lens[s])))
    k_new, v_new = wl.new_kv()
    q = wl.queries()

    # K/V pools first; the context is written in chunks as it is drawn.  An
    # e4m3 pool needs its per-tensor scales (the drawn values' amax) before
    # anything is quantised, so its context is staged on the device and
    # written once every draw is in.
    desc = _desc_for(wl, device)
    k_cache, v_cache = alloc_cache(desc, device, fill=_SENTINEL[desc.kv_dtype])
    staged, staged_tokens = [], 0
    for s, (k, v) in enumerate(_draws_in_order(wl, S)):
        c = num_cached[s]
        if k.shape[0] - c > 0:
            staged.append((k[c:].to(device), v[c:].to(device), torch.from_numpy(prior_slots[s]).to(device)))
            staged_tokens += k.shape[0] - c
        if not fp8 and staged_tokens >= write_chunk_tokens:
            _write_staged(desc, staged, k_cache, v_cache)
            staged, staged_tokens = [], 0
    if fp8:
        wl.fp8_scales_from_draws()
        desc = _desc_for(wl, device)
    _write_staged(desc, staged, k_cache, v_cache)

    max_blocks = max(1, max(-(-(int(wl.context_lens[s]) + int(wl.q_lens[s])) // wl.block_size)
                            for s in range(S)) if S else 1)
    tables_host = pool.block_tables(list(range(S)), max_blocks)
    seq_lens = torch.from_numpy((wl.context_lens + wl.q_lens).astype(np.int32))
    decode_only = bool(np.all(wl.q_lens == 1))
    qsl = None
    if not decode_only:
        qsl = torch.from_numpy(np.concatenate([[0], np.cumsum(wl.q_lens)]).astype(np.int32)).to(device)
    rows = wl.num_new_tokens
    if decode_only:
        ws_bytes = pa_decode_workspace_size(desc, S)
    else:
        ws_bytes = pa_prefill_workspace_size(desc, S, rows)
    slots_host = torch.tensor(step_slots, dtype=torch.int64)
    batch = DeviceBatch(
        desc=desc, pool=pool, k_cache=k_cache, v_cache=v_cache, tables=tables_host.to(device),
        seq_lens=seq_lens.to(device), qsl=qsl, q=q.to(device), k_new=k_new.to(device),
        v_new=v_new.to(device), slots=slots_host.to(device),
        out=torch.empty((rows, wl.num_q_heads, wl.head_dim), dtype=desc.q_torch_dtype, device=device),
        workspace=alloc_workspace(ws_bytes, device), max_q_len=int(wl.q_lens.max()) if S else 0,
        scale=default_scale(wl.head_dim), tables_host=tables_host, slots_host=slots_host,
        prior_slots=prior_slots, num_cached=num_cached)
    torch.cuda.synchronize(device)
    return batch


def clone(b: DeviceBatch) -> DeviceBatch:
    """A second copy of a batch on the same device: its own K/V pools (device
    copies of b's), output and zeroed workspace; the step inputs and the host
    pool are shared.  Cheaper than drawing the workload again."""
    import copy
    c = copy.copy(b)
    c.k_cache = b.k_cache.clone()
    c.v_cache = b.v_cache.clone()
    c.out = torch.empty_like(b.out)
    c.workspace = torch.zeros_like(b.workspace)
    return c


def _draws_in_order(wl, S, window=None):
    """wl.prior_kv(s) for s = 0..S-1, drawn on a few host threads ahead of
    use (the draws are independent per sequence), yielded in order."""
    import concurrent.futures as cf
    import os
    window = window or max(2, min(32, (os.cpu_count() or 4)))
    with cf.ThreadPoolExecutor(max_workers=window) as ex:
        futs = {}
        for s in range(min(window, S)):
            futs[s] = ex.submit(wl.prior_kv, s)
        for s in range(S):
            r = futs.pop(s).result()
            if s + window < S:
                futs[s + window] = ex.submit(wl.prior_kv, s + window)
            yield r


def _write_staged(desc, staged, k_cache, v_cache):
    if staged:
        pa_cache_write(desc, torch.cat([x[0] for x in staged]), torch.cat([x[1] for x in staged]),
                       torch.cat([x[2] for x in staged]), k_cache, v_cache)


def write_step(b: DeviceBatch, stream=None):
    """pa_cache_write of this step's new K/V rows."""
    pa_cache_write(b.desc, b.k_new, b.v_new, b.slots, b.k_cache, b.v_cache, stream)


def attend(b: DeviceBatch, stream=None):
    """pa_decode (pure decode) or pa_decode_chunked_prefill (mixed step)."""
    if b.decode_only:
        pa_decode(b.desc, b.q, b.k_cache, b.v_cache, b.tables, b.seq_lens, b.scale, b.out, b.workspace, stream)
    else:
        pa_decode_chunked_prefill(b.desc, b.q, b.k_cache, b.v_cache, b.tables, b.qsl, b.seq_lens, b.max_q_len,
                                  b.scale, b.out, b.workspace, stream)


def step(b: DeviceBatch, stream=None):
    write_step(b, stream)
    attend(b, stream)


@dataclass
class PrefixPlan:
    groups: PrefixGroups
    dev: dict
    workspace: torch.Tensor


def prefix_plan(b: DeviceBatch) -> PrefixPlan:
    """The batch's shared prefixes (from its block tables) and the workspace
    pa_decode_prefix needs, on b's device."""
    dev = b.tables.device
    groups = PrefixGroups(b.tables_host, b.seq_lens, b.desc.block_size)
    ws = pa_decode_prefix_workspace_size(b.desc, b.seq_lens.shape[0], groups.num_members, groups.max_prefix_blocks)
    return PrefixPlan(groups, groups.to(dev), alloc_workspace(ws, dev))


def attend_prefix(b: DeviceBatch, plan: PrefixPlan, stream=None):
    """pa_decode_prefix: each shared prefix attended once for its sequences."""
    pa_decode_prefix(b.desc, b.q, b.k_cache, b.v_cache, b.tables, b.seq_lens, plan.groups, plan.dev, b.scale, b.out,
                     plan.workspace, stream)


def step_prefix(b: DeviceBatch, plan: PrefixPlan, stream=None):
    write_step(b, stream)
    attend_prefix(b, plan, stream)


def step_fused(b: DeviceBatch, stream=None):
    """The same step as one launch: pa_decode_fused writes each sequence's
    new token and attends (pure decode steps on the tensor-core path)."""
    pa_decode_fused(b.desc, b.q, b.k_new, b.v_new, b.k_cache, b.v_cache, b.tables, b.seq_lens, b.scale, b.out,
                    b.workspace, stream)
