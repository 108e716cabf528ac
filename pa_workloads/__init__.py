"""Seeded synthetic inputs for the paged decode attention workloads.

This module draws numbers and nothing else: sequence lengths, the pool's
initial free-list order, token ids for prefix hashing, N(0,1) query/key/value
values cast to the input dtype, and FP8 scales (per tensor or per kv head)
from the drawn values' absolute maximum.  It holds none of the method's arithmetic (no block
tables, slots, cache writes or attention); the oracle and the CUDA path each
derive those from these same arrays.

Workloads (sizes as named by the paged-attention benchmark plan):

* ``tiny_fp32``: 4 sequences, context [40,128,300,64], block 16, a pool of
  128 blocks handed out in a seeded random permutation, 2 query = 2 KV heads,
  head_dim 64, fp32 N(0,1) seed 0; one decode step.
* ``gqa_bf16``: 64 sequences, context uniform in [32, 2048], 32 query / 8 KV
  heads, head_dim 128, block 16, pool 1.25x the blocks needed, shuffled.
* ``prefix_bf16``: 256 sequences; half share one 1024-token prefix (64
  blocks); suffix lengths lognormal (median 512, sigma 1) clipped to
  [16, 8192]; 32/8 heads, head_dim 128, block 16.
* ``fp8_long``: 128 sequences, context uniform in [4096, 32768], 64/8 heads,
  head_dim 128, block 16, FP8-e4m3 cache with per-tensor K and V scales,
  bf16 queries and bf16 new K/V.
* ``mixed_prefill``: 8 prefill chunks of 512 query tokens over 0..4096 prior
  tokens each, plus 248 decode rows over contexts uniform in [64, 4096];
  32/8 heads, head_dim 128, block 16 or 32.
* ``long_prefix_bf16`` (a case of our own for the shared-prefix path, not
  one of the plan's five): 64 sequences that all share one 32768-token
  prefix (2048 blocks, 134 MB of K/V, more than the L2 cache holds), suffix
  lengths lognormal (median 512, sigma 1) clipped to [16, 2048]; 32/8 heads,
  head_dim 128, block 16.

Each has a ``small`` variant with the same structure at sizes a plain CPU
oracle finishes in seconds.  Randomness: ``tiny_fp32`` draws everything from
``np.random.default_rng(0)`` in a fixed order (permutation, then per sequence
K then V, then new K, new V, q); the others use one independent stream per
(workload, sequence, purpose) via ``np.random.SeedSequence``.
"""
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

GLOBAL = 2**31 - 1  # sequence index used by per-workload streams

S_LENGTHS, S_PERM, S_K, S_V, S_KNEW, S_VNEW, S_Q, S_TOKENS, S_SUFFIX = range(9)

DTYPE_TORCH = {"f32": torch.float32, "bf16": torch.bfloat16}
FP8_MAX = 448.0


def rng(seed_key: int, seq: int, stream: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([0, int(seed_key), int(seq), int(stream)]))


def _cast(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t if dtype == "f32" else t.to(DTYPE_TORCH[dtype])


@dataclass
class Workload:
    name: str
    seed_key: int
    kv_dtype: str  # storage of the cache: "f32" | "bf16" | "e4m3"
    q_dtype: str  # queries and new K/V: "f32" | "bf16"
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    context_lens: np.ndarray  # int64 [S]: tokens cached before the step
    q_lens: np.ndarray  # int64 [S]: tokens added this step (1 = decode row)
    free_order: np.ndarray  # int32 [num_blocks]: initial free-list order
    prefix_len: int = 0
    sharing: Optional[np.ndarray] = None  # bool [S]: sequences sharing the one prefix
    # several prefixes (tests): int [S], the prefix group of each sequence or
    # -1; group g's prefix_len tokens are drawn from their own streams
    prefix_group: Optional[np.ndarray] = None
    vocab: int = 32000
    k_scale: float = 1.0  # e4m3 pools: one fp32 scale, or an array of one per kv head
    v_scale: float = 1.0
    # how an e4m3 pool's scales are set: "tensor" (amax / 448 over every
    # drawn value), "head" (amax / 448 per kv head) or "fixed" (as given)
    scale_mode: str = "tensor"
    _fixed: Optional[dict] = field(default=None, repr=False)
    _amax: Optional[dict] = field(default=None, repr=False)

    # ---- shape helpers (no method arithmetic) --------------------------------
    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def num_new_tokens(self) -> int:
        return int(self.q_lens.sum())

    @property
    def max_q_len(self) -> int:
        return int(self.q_lens.max()) if self.num_seqs else 0

    # ---- draws ---------------------------------------------------------------
    def token_ids(self, s: int) -> Optional[np.ndarray]:
        """Token ids of the cached context of sequence s (None: no hashing)."""
        if self.sharing is None and self.prefix_group is None:
            return None
        n = int(self.context_lens[s])
        own = rng(self.seed_key, s, S_TOKENS).integers(0, self.vocab, size=n, dtype=np.int64)
        src = self._prefix_stream(s)
        if src is not None:
            pre = rng(self.seed_key, src, S_TOKENS).integers(0, self.vocab, size=self.prefix_len,
                                                             dtype=np.int64)
            own[: self.prefix_len] = pre
        return own.astype(np.int32)

    def _prefix_stream(self, s: int) -> Optional[int]:
        """Sequence index of the streams sequence s's shared prefix is drawn
        from (None: no shared prefix)."""
        if self.sharing is not None and self.sharing[s]:
            return GLOBAL
        if self.prefix_group is not None and self.prefix_group[s] >= 0:
            return GLOBAL - 1 - int(self.prefix_group[s])
        return None

    def _normal(self, seq: int, stream: int, rows: int, heads: int) -> np.ndarray:
        return rng(self.seed_key, seq, stream).standard_normal((rows, heads, self.head_dim),
                                                               dtype=np.float32)

    def prior_kv_f32(self, s: int):
        """fp32 draws of K and V for the cached context of sequence s:
        [context_len][kv_heads][head_dim] each."""
        if self._fixed is not None:
            return self._fixed["k"][s], self._fixed["v"][s]
        n = int(self.context_lens[s])
        k = self._normal(s, S_K, n, self.num_kv_heads)
        v = self._normal(s, S_V, n, self.num_kv_heads)
        src = self._prefix_stream(s)
        if src is not None:
            p = self.prefix_len
            k[:p] = self._normal(src, S_K, p, self.num_kv_heads)
            v[:p] = self._normal(src, S_V, p, self.num_kv_heads)
        return k, v

    def prior_kv(self, s: int):
        """K, V of sequence s's cached context in the input dtype (torch, CPU).
        Records the draws' absolute maxima for fp8_scales_from_draws."""
        k, v = self.prior_kv_f32(s)
        k, v = _cast(k, self.q_dtype), _cast(v, self.q_dtype)
        if self._amax is None:
            self._amax = {}
        self._amax[s] = (_head_amax(k, self.num_kv_heads), _head_amax(v, self.num_kv_heads))
        return k, v

    def new_kv(self):
        """K, V of this step's new tokens: [num_new_tokens][kv_heads][head_dim]."""
        if self._fixed is not None:
            return _cast(self._fixed["k_new"], self.q_dtype), _cast(self._fixed["v_new"], self.q_dtype)
        t = self.num_new_tokens
        k = self._normal(GLOBAL, S_KNEW, t, self.num_kv_heads)
        v = self._normal(GLOBAL, S_VNEW, t, self.num_kv_heads)
        return _cast(k, self.q_dtype), _cast(v, self.q_dtype)

    def queries(self):
        """Queries of this step's new tokens: [num_new_tokens][q_heads][head_dim]."""
        if self._fixed is not None:
            return _cast(self._fixed["q"], self.q_dtype)
        return _cast(self._normal(GLOBAL, S_Q, self.num_new_tokens, self.num_q_heads), self.q_dtype)

    def set_fp8_scales(self, amax_k, amax_v):
        """Scales = amax / 448 (fp32), so the largest drawn value maps onto
        the largest finite e4m3 value: one number each, or (arrays of amax)
        one per kv head."""
        def sc(a):
            a = np.asarray(a, dtype=np.float32)
            q = (a / np.float32(FP8_MAX)).astype(np.float32)
            return float(q) if q.ndim == 0 else q
        self.k_scale = sc(amax_k)
        self.v_scale = sc(amax_v)

    def fp8_scales_from_draws(self):
        """amax over every K (V) value this workload draws, prior and new, in
        the input dtype (per kv head when scale_mode is "head"); sets and
        returns (k_scale, v_scale).  scale_mode "fixed" keeps the given ones."""
        if self.scale_mode == "fixed":
            return self.k_scale, self.v_scale
        ak = np.zeros(self.num_kv_heads, dtype=np.float32)
        av = np.zeros(self.num_kv_heads, dtype=np.float32)
        for s in range(self.num_seqs):
            if self._amax is None or s not in self._amax:
                self.prior_kv(s)
            ak = np.maximum(ak, self._amax[s][0])
            av = np.maximum(av, self._amax[s][1])
        k, v = self.new_kv()
        ak = np.maximum(ak, _head_amax(k, self.num_kv_heads))
        av = np.maximum(av, _head_amax(v, self.num_kv_heads))
        if self.scale_mode == "head":
            self.set_fp8_scales(ak, av)
        else:
            self.set_fp8_scales(ak.max(), av.max())
        return self.k_scale, self.v_scale


def _head_amax(x: torch.Tensor, heads: int) -> np.ndarray:
    """Largest |value| per kv head of a [rows][heads][head_dim] tensor."""
    if x.numel() == 0:
        return np.zeros(heads, dtype=np.float32)
    return x.abs().amax(dim=(0, 2)).float().numpy().astype(np.float32)


def _pool_size(need_blocks: int) -> int:
    return int(np.ceil(1.25 * need_blocks))


def _blocks_needed(context_lens, q_lens, bs, shared_blocks=0, n_sharing=0):
    # capacity bookkeeping for sizing the pool only: whole blocks per sequence
    tot = sum(-(-(int(c) + int(q)) // bs) for c, q in zip(context_lens, q_lens))
    return tot - shared_blocks * max(0, n_sharing - 1)


def _finish(name, seed_key, kv_dtype, q_dtype, hq, hkv, d, bs, ctx, qlen, nb=None,
            prefix_len=0, sharing=None) -> Workload:
    ctx = np.asarray(ctx, dtype=np.int64)
    qlen = np.asarray(qlen, dtype=np.int64)
    if nb is None:
        shared_blocks = prefix_len // bs
        n_sharing = int(sharing.sum()) if sharing is not None else 0
        nb = _pool_size(_blocks_needed(ctx, qlen, bs, shared_blocks, n_sharing))
        nb = max(nb, 1)
    order = rng(seed_key, GLOBAL, S_PERM).permutation(nb).astype(np.int32)
    return Workload(name, seed_key, kv_dtype, q_dtype, hq, hkv, d, bs, nb, ctx, qlen, order,
                    prefix_len, sharing)


def tiny_fp32() -> Workload:
    lens = [40, 128, 300, 64]
    hq = hkv = 2
    d = 64
    g = np.random.default_rng(0)
    perm = g.permutation(128).astype(np.int32)
    ks, vs = [], []
    for n in lens:
        ks.append(g.standard_normal((n, hkv, d), dtype=np.float32))
        vs.append(g.standard_normal((n, hkv, d), dtype=np.float32))
    k_new = g.standard_normal((4, hkv, d), dtype=np.float32)
    v_new = g.standard_normal((4, hkv, d), dtype=np.float32)
    q = g.standard_normal((4, hq, d), dtype=np.float32)
    return Workload("tiny_fp32", 0, "f32", "f32", hq, hkv, d, 16, 128,
                    np.array(lens, dtype=np.int64), np.ones(4, dtype=np.int64), perm,
                    _fixed={"k": ks, "v": vs, "k_new": k_new, "v_new": v_new, "q": q})


def gqa_bf16(size: str = "full") -> Workload:
    key = 1 if size == "full" else 101
    n, lo, hi = (64, 32, 2048) if size == "full" else (6, 0, 300)
    ctx = rng(key, GLOBAL, S_LENGTHS).integers(lo, hi, size=n, endpoint=True)
    return _finish("gqa_bf16" + ("" if size == "full" else "_small"), key, "bf16", "bf16",
                   32, 8, 128, 16, ctx, np.ones(n))


def prefix_bf16(size: str = "full") -> Workload:
    key = 2 if size == "full" else 102
    if size == "full":
        n, prefix, median, lo, hi = 256, 1024, 512, 16, 8192
    else:
        n, prefix, median, lo, hi = 8, 64, 40, 16, 200
    suf = rng(key, GLOBAL, S_SUFFIX).lognormal(mean=np.log(median), sigma=1.0, size=n)
    suf = np.clip(np.rint(suf), lo, hi).astype(np.int64)
    sharing = np.zeros(n, dtype=bool)
    sharing[: n // 2] = True
    ctx = suf + np.where(sharing, prefix, 0)
    return _finish("prefix_bf16" + ("" if size == "full" else "_small"), key, "bf16", "bf16",
                   32, 8, 128, 16, ctx, np.ones(n), prefix_len=prefix, sharing=sharing)


def long_prefix_bf16(size: str = "full") -> Workload:
    key = 5 if size == "full" else 105
    if size == "full":
        n, prefix, median, lo, hi = 64, 32768, 512, 16, 2048
    else:
        n, prefix, median, lo, hi = 6, 320, 40, 16, 120
    suf = rng(key, GLOBAL, S_SUFFIX).lognormal(mean=np.log(median), sigma=1.0, size=n)
    suf = np.clip(np.rint(suf), lo, hi).astype(np.int64)
    return _finish("long_prefix_bf16" + ("" if size == "full" else "_small"), key, "bf16", "bf16",
                   32, 8, 128, 16, suf + prefix, np.ones(n), prefix_len=prefix, sharing=np.ones(n, dtype=bool))


def fp8_long(size: str = "full") -> Workload:
    key = 3 if size == "full" else 103
    n, lo, hi = (128, 4096, 32768) if size == "full" else (4, 100, 700)
    ctx = rng(key, GLOBAL, S_LENGTHS).integers(lo, hi, size=n, endpoint=True)
    return _finish("fp8_long" + ("" if size == "full" else "_small"), key, "e4m3", "bf16",
                   64, 8, 128, 16, ctx, np.ones(n))


def mixed_prefill(block_size: int = 16, size: str = "full") -> Workload:
    key = 4 if size == "full" else 104
    if size == "full":
        nchunk, chunk, plo, phi, ndec, dlo, dhi = 8, 512, 0, 4096, 248, 64, 4096
    else:
        nchunk, chunk, plo, phi, ndec, dlo, dhi = 2, 40, 0, 100, 5, 10, 200
    g = rng(key, GLOBAL, S_LENGTHS)
    pre = g.integers(plo, phi, size=nchunk, endpoint=True)
    dec = g.integers(dlo, dhi, size=ndec, endpoint=True)
    ctx = np.concatenate([pre, dec])
    qlen = np.concatenate([np.full(nchunk, chunk), np.ones(ndec)])
    return _finish(f"mixed_prefill_bs{block_size}" + ("" if size == "full" else "_small"), key,
                   "bf16", "bf16", 32, 8, 128, block_size, ctx, qlen)


def custom(name, context_lens, q_lens=None, kv_dtype="bf16", q_dtype="bf16", num_q_heads=8,
           num_kv_heads=2, head_dim=128, block_size=16, seed_key=900, num_blocks=None,
           scale_mode="tensor", k_scale=1.0, v_scale=1.0, prefix_len=0, prefix_group=None) -> Workload:
    """Explicit shapes for edge-case tests.  e4m3 scales: scale_mode
    "tensor" / "head" derive them from the draws; "fixed" takes k_scale and
    v_scale as given (a number, or one per kv head).  prefix_group (one int
    per sequence, -1 for none): sequences of group g begin with the same
    prefix_len tokens (token ids and K/V), which the pool's prefix hashing
    then shares."""
    ctx = np.asarray(context_lens, dtype=np.int64)
    ql = np.ones_like(ctx) if q_lens is None else np.asarray(q_lens, dtype=np.int64)
    wl = _finish(name, seed_key, kv_dtype, q_dtype, num_q_heads, num_kv_heads, head_dim,
                 block_size, ctx, ql, nb=num_blocks)
    wl.scale_mode = scale_mode
    if prefix_group is not None:
        wl.prefix_group = np.asarray(prefix_group, dtype=np.int64)
        wl.prefix_len = int(prefix_len)
        assert all(int(c) >= prefix_len for c, g in zip(ctx, wl.prefix_group) if g >= 0)
    if scale_mode == "fixed":
        wl.k_scale = k_scale if np.ndim(k_scale) == 0 else np.asarray(k_scale, dtype=np.float32)
        wl.v_scale = v_scale if np.ndim(v_scale) == 0 else np.asarray(v_scale, dtype=np.float32)
    return wl


def first_seqs(wl: Workload, n: int) -> Workload:
    """The first n sequences of a workload, with the same draws per sequence
    and a pool sized (1.25x) and shuffled for them alone."""
    n = min(n, wl.num_seqs)
    sharing = None if wl.sharing is None else wl.sharing[:n].copy()
    out = _finish(f"{wl.name}_first{n}", wl.seed_key, wl.kv_dtype, wl.q_dtype, wl.num_q_heads, wl.num_kv_heads,
                  wl.head_dim, wl.block_size, wl.context_lens[:n], wl.q_lens[:n], prefix_len=wl.prefix_len,
                  sharing=sharing)
    out.scale_mode = wl.scale_mode
    return out


WORKLOADS = {
    "tiny_fp32": lambda size="full": tiny_fp32(),
    "gqa_bf16": gqa_bf16,
    "prefix_bf16": prefix_bf16,
    "fp8_long": fp8_long,
    "mixed_prefill_bs16": lambda size="full": mixed_prefill(16, size),
    "mixed_prefill_bs32": lambda size="full": mixed_prefill(32, size),
    "long_prefix_bf16": long_prefix_bf16,
}


def make(name: str, size: str = "full") -> Workload:
    return WORKLOADS[name](size)
