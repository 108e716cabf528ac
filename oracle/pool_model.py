"""Block pool model: a plain dict/list restatement of the paged KV-cache
block manager.  TEST INFRASTRUCTURE ONLY (see oracle/__init__.py).

Follows
-------
* "vLLM innenfra: slik gjør paged attention GPU-minnet til blokker på 16
  tokens", paragraph 2: a pool of free blocks kept in ``free_block_queue``;
  a finished request hands its blocks back to that queue (the step() list,
  item 3).
* "49 vLLM / PagedAttention", block-table snippet: a new block is taken when
  ``len(blocks) * block_size <= req.len``, i.e. when the token being
  appended is the first slot of a new block; blocks need not be contiguous.
* "PagedAttention：KV cache 即虚拟内存（block manager & 碎片）", 深入原理:
  - V1 结构: ``free_block_queue`` is a doubly linked list in eviction order;
    allocation pops the head, release pushes the tail (both O(1)); every
    block has a ``ref_cnt``; ``cached_block_hash_to_block`` maps a block's
    token hash to the block.
  - 生命周期: admission pops blocks for the prompt; decode pops one more
    when the last block is full; finishing decrements ``ref_cnt`` and
    releases the block at 0.
  - 共享 → prefix caching: a block is keyed by the hash of its tokens and
    its parent's hash; equal prefixes give equal hashes, so a second request
    points at the existing block and ``touch()`` raises its ``ref_cnt``;
    only whole blocks are shared; a fork that diverges inside a shared block
    triggers copy-on-write.
* "49 vLLM / PagedAttention", Почему это важно and, under Вопросы пытливого
  ума, the prefix-sharing answer: blocks shared between requests are
  copy-on-write, like pages shared between processes.

Readings where the pages are silent
-----------------------------------
* Hash: FNV-1a 64 over the parent hash (8 bytes, little endian; 0 for the
  first block) followed by the block's token ids (int32, little endian).  A
  hit also compares the stored token ids, so a collision cannot alias.
* Hits are the longest run of leading full blocks found in the map; the
  first miss ends sharing for the rest of the sequence.  A newly allocated
  full block is entered in the map unless its hash is already there.
* A released block keeps its hash while it sits in the free queue and stays
  shareable; popping it for reuse evicts the hash.  ``touch()`` of such a
  parked block unlinks it from the queue.
* Releasing a sequence walks its blocks in reverse logical order, so the
  tail of a sequence is evicted before its (possibly shared) prefix.
* Allocation is all-or-nothing: on shortage nothing changes.
* ``append`` takes no token ids, so blocks filled by decoding are never hashed.
* Fork (copy-on-write): ``fork(parent, child)`` gives the child the parent's
  length and block table and raises every block's ``ref_cnt`` by one.  When
  ``append`` is about to write into a sequence's last block while that block
  is partly filled and shared (``ref_cnt`` > 1), the sequence first moves to
  a new block popped from the head: the pair (shared block, new block) is
  queued for the caller to copy on the device, the shared block's
  ``ref_cnt`` drops by one, and the new block (never hashed) replaces it in
  the table.  A full shared block is never copied: the next token opens a
  new block anyway.  The copy's block counts toward the all-or-nothing
  check.  ``take_copies`` returns the queued pairs, oldest first, and
  empties the queue.
"""
from collections import OrderedDict

FNV_OFFSET = 0xCBF29CE484222325
FNV_PRIME = 0x100000001B3
MASK64 = (1 << 64) - 1


class PoolModelError(Exception):
    def __init__(self, code, msg):
        super().__init__(f"{code}: {msg}")
        self.code = code  # "INVALID_ARG" | "NO_BLOCKS" | "STATE"


def fnv1a64(data: bytes) -> int:
    h = FNV_OFFSET
    for byte in data:
        h ^= byte
        h = (h * FNV_PRIME) & MASK64
    return h


def block_hash(parent: int, tokens) -> int:
    return fnv1a64(parent.to_bytes(8, "little") + b"".join(
        int(t).to_bytes(4, "little", signed=True) for t in tokens))


class BlockPoolModel:
    def __init__(self, num_blocks, block_size, initial_free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise PoolModelError("INVALID_ARG", "num_blocks and block_size must be positive")
        order = list(range(num_blocks)) if initial_free_order is None else [int(b) for b in initial_free_order]
        if sorted(order) != list(range(num_blocks)):
            raise PoolModelError("INVALID_ARG", "initial free order is not a permutation")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free_queue = OrderedDict((b, None) for b in order)  # head = first
        self.ref_cnt = [0] * num_blocks
        self.block_key = [None] * num_blocks  # (hash, tokens) while cached
        self.hash_to_block = {}
        self.seqs = {}  # seq_id -> {"blocks": [...], "num_tokens": n}
        self.copies = []  # (src, dst) block pairs queued by copy-on-write

    # -- queries -------------------------------------------------------------
    def num_free(self):
        return len(self.free_queue)

    def free_order(self):
        return list(self.free_queue.keys())

    def block_table(self, seq_id):
        return list(self._seq(seq_id)["blocks"])

    def num_tokens(self, seq_id):
        return self._seq(seq_id)["num_tokens"]

    def _seq(self, seq_id):
        if seq_id not in self.seqs:
            raise PoolModelError("INVALID_ARG", f"unknown sequence {seq_id}")
        return self.seqs[seq_id]

    # -- primitives ----------------------------------------------------------
    def _pop_head(self):
        b, _ = self.free_queue.popitem(last=False)
        key = self.block_key[b]
        if key is not None:  # evict the cached hash
            if self.hash_to_block.get(key[0]) == b:
                del self.hash_to_block[key[0]]
            self.block_key[b] = None
        self.ref_cnt[b] = 1
        return b

    def _touch(self, b):
        if self.ref_cnt[b] == 0:
            del self.free_queue[b]
        self.ref_cnt[b] += 1

    # -- operations ----------------------------------------------------------
    def add_seq(self, seq_id, num_tokens, token_ids=None):
        """Admit a prompt of num_tokens; returns the number of tokens whose
        blocks were found in the prefix cache."""
        if seq_id in self.seqs:
            raise PoolModelError("INVALID_ARG", f"sequence {seq_id} exists")
        if num_tokens < 0:
            raise PoolModelError("INVALID_ARG", "negative length")
        if token_ids is not None and len(token_ids) != num_tokens:
            raise PoolModelError("INVALID_ARG", "token_ids length mismatch")
        bs = self.block_size
        nblk = (num_tokens + bs - 1) // bs
        keys = []
        if token_ids is not None:
            parent = 0
            for i in range(num_tokens // bs):
                toks = tuple(int(t) for t in token_ids[i * bs:(i + 1) * bs])
                parent = block_hash(parent, toks)
                keys.append((parent, toks))
        hits = []
        for key in keys:
            b = self.hash_to_block.get(key[0])
            if b is None or self.block_key[b] != key:
                break
            hits.append(b)
        parked = sum(1 for b in hits if self.ref_cnt[b] == 0)
        need = nblk - len(hits)
        if need > len(self.free_queue) - parked:
            raise PoolModelError("NO_BLOCKS", f"need {need} blocks")
        for b in hits:
            self._touch(b)
        blocks = list(hits)
        for i in range(len(hits), nblk):
            b = self._pop_head()
            if i < len(keys) and keys[i][0] not in self.hash_to_block:
                self.block_key[b] = keys[i]
                self.hash_to_block[keys[i][0]] = b
            blocks.append(b)
        self.seqs[seq_id] = {"blocks": blocks, "num_tokens": num_tokens}
        return len(hits) * bs

    def append(self, seq_id, n_new):
        """Grow a sequence by n_new tokens; returns their flat slots."""
        seq = self._seq(seq_id)
        if n_new < 0:
            raise PoolModelError("INVALID_ARG", "negative count")
        bs = self.block_size
        blocks = seq["blocks"]
        start = seq["num_tokens"]
        cow = n_new > 0 and start % bs != 0 and self.ref_cnt[blocks[-1]] > 1
        need = max(0, (start + n_new + bs - 1) // bs - len(blocks)) + (1 if cow else 0)
        if need > len(self.free_queue):
            raise PoolModelError("NO_BLOCKS", f"need {need} blocks")
        if cow:  # the shared, partly filled last block: copy it first
            src = blocks[-1]
            dst = self._pop_head()
            self.ref_cnt[src] -= 1
            blocks[-1] = dst
            self.copies.append((src, dst))
        slots = []
        for p in range(start, start + n_new):
            if len(blocks) * bs <= p:  # the block-table snippet's test
                blocks.append(self._pop_head())
            slots.append(blocks[p // bs] * bs + p % bs)
        seq["num_tokens"] = start + n_new
        return slots

    def fork(self, parent_id, child_id):
        """A new sequence with the parent's length and blocks, all shared."""
        parent = self._seq(parent_id)
        if child_id in self.seqs:
            raise PoolModelError("INVALID_ARG", f"sequence {child_id} exists")
        for b in parent["blocks"]:
            self.ref_cnt[b] += 1
        self.seqs[child_id] = {"blocks": list(parent["blocks"]), "num_tokens": parent["num_tokens"]}

    def take_copies(self):
        """The (src, dst) pairs queued by copy-on-write, oldest first."""
        out, self.copies = self.copies, []
        return out

    def slots(self, seq_id, start, n):
        """Flat slots of positions [start, start + n) of a sequence."""
        seq = self._seq(seq_id)
        if start < 0 or n < 0 or start + n > seq["num_tokens"]:
            raise PoolModelError("INVALID_ARG", "positions out of range")
        bs = self.block_size
        return [seq["blocks"][p // bs] * bs + p % bs for p in range(start, start + n)]

    def free_seq(self, seq_id):
        seq = self._seq(seq_id)
        for b in seq["blocks"]:
            if self.ref_cnt[b] <= 0:
                raise PoolModelError("STATE", f"ref_cnt underflow on block {b}")
        for b in reversed(seq["blocks"]):
            self.ref_cnt[b] -= 1
            if self.ref_cnt[b] == 0:
                self.free_queue[b] = None  # push tail
        del self.seqs[seq_id]
