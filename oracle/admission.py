"""The pages' KV memory arithmetic.  TEST INFRASTRUCTURE ONLY.

* ``blocks_for``: a sequence of n tokens occupies ceil(n / block_size) blocks
  (block-table snippet on "49 vLLM / PagedAttention"; the 分页 branch of the
  代码 listing on "PagedAttention：KV cache 即虚拟内存（block manager & 碎片）").
* ``block_bytes``: 2 (K and V) x block_size x kv_heads x head_dim x dtype
  bytes ("vLLM innenfra: slik gjør paged attention GPU-minnet til blokker på
  16 tokens", paragraph 2).
* ``request_kv_bytes``: one request's cache = 2 x layers x heads x head_dim x
  tokens, times the element size ("49 vLLM / PagedAttention", section
  "Пейджинг для KV-кэша: откуда берётся ×2–4"; the page omits the element
  size, which is restored here).
* ``contiguous_capacity`` / ``paged_admission_*``: the same block pool
  filled under the two strategies of the 代码 section's worked example.  A
  contiguous engine reserves ceil(max_len / block) blocks for every request;
  a paged one takes ceil(len / block).  The page's listing skips a request
  that does not fit and keeps scanning (``paged_admission_skip``); its
  printed answer, 13, is what first-come-first-served admission gives when
  it stops at the first request that does not fit (``paged_admission_fcfs``).
"""


def blocks_for(num_tokens: int, block_size: int) -> int:
    if num_tokens < 0 or block_size <= 0:
        raise ValueError("bad size")
    return (num_tokens + block_size - 1) // block_size


def block_bytes(block_size: int, num_kv_heads: int, head_dim: int, dtype_bytes: int) -> int:
    return 2 * block_size * num_kv_heads * head_dim * dtype_bytes


def request_kv_bytes(num_layers: int, num_heads: int, head_dim: int, num_tokens: int,
                     dtype_bytes: int) -> int:
    return 2 * num_layers * num_heads * head_dim * num_tokens * dtype_bytes


def contiguous_capacity(pool_blocks: int, max_len: int, block_size: int) -> int:
    return pool_blocks // blocks_for(max_len, block_size)


def paged_admission_fcfs(lengths, pool_blocks: int, block_size: int) -> int:
    used = admitted = 0
    for n in lengths:
        need = blocks_for(n, block_size)
        if used + need > pool_blocks:
            break
        used += need
        admitted += 1
    return admitted


def paged_admission_skip(lengths, pool_blocks: int, block_size: int) -> int:
    used = admitted = 0
    for n in lengths:
        need = blocks_for(n, block_size)
        if used + need <= pool_blocks:
            used += need
            admitted += 1
    return admitted
