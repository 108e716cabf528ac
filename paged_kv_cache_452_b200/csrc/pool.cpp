// Host block pool: free_block_queue, ref_cnt and hash-keyed prefix sharing.
//
// The block manager described on "PagedAttention：KV cache 即虚拟内存（block
// manager & 碎片）", section 深入原理 (V1 结构, 生命周期, 共享 → prefix caching),
// with the allocation rule of the block-table snippet on "49 vLLM /
// PagedAttention" (a new block when the token being appended starts one),
// and copy-on-write for forked sequences (the same sharing bullet: a fork
// that diverges inside a shared block triggers a copy; "49 vLLM /
// PagedAttention", Почему это важно).  It only produces block tables, slots
// and the list of block copies; it never touches KV bytes.
//
// free_block_queue is an intrusive doubly linked list over block ids (prev/
// next arrays), so pop-head, push-tail and unlinking a parked block that a
// prefix hit touches are all O(1).  A block is in the queue exactly when its
// ref_cnt is 0.
#include <cstdint>
#include <cstring>
#include <string>
#include <unordered_map>
#include <vector>

#include "pa.h"
#include "pa_error.h"

namespace {

constexpr uint64_t kFnvOffset = 0xCBF29CE484222325ull;
constexpr uint64_t kFnvPrime = 0x100000001B3ull;

uint64_t fnv1a_bytes(uint64_t h, const uint8_t* p, size_t n) {
  for (size_t i = 0; i < n; ++i) {
    h ^= p[i];
    h *= kFnvPrime;
  }
  return h;
}

// Hash of a full block: FNV-1a 64 over parent (8 bytes LE) then token ids
// (int32 LE).  x86-64 and aarch64 hosts are little endian.
uint64_t block_key(uint64_t parent, const int32_t* tokens, int n) {
  uint8_t pb[8];
  std::memcpy(pb, &parent, 8);
  uint64_t h = fnv1a_bytes(kFnvOffset, pb, 8);
  return fnv1a_bytes(h, reinterpret_cast<const uint8_t*>(tokens), sizeof(int32_t) * (size_t)n);
}

struct Seq {
  std::vector<int32_t> blocks;
  int32_t num_tokens = 0;
};

}  // namespace

struct pa_pool {
  int32_t num_blocks = 0;
  int32_t block_size = 0;
  // free_block_queue: head/tail and links; -1 terminates
  std::vector<int32_t> prev, next;
  int32_t head = -1, tail = -1, nfree = 0;
  std::vector<int32_t> ref_cnt;
  // prefix cache
  std::vector<uint8_t> cached;          // block holds a hash
  std::vector<uint64_t> hash;           // its hash
  std::vector<std::vector<int32_t>> toks;  // its token ids (for collision checks)
  std::unordered_map<uint64_t, int32_t> hash_to_block;
  std::unordered_map<int64_t, Seq> seqs;
  // copy-on-write pairs (shared block, its new copy) for the caller to run
  std::vector<int32_t> copy_src, copy_dst;

  void push_tail(int32_t b) {
    prev[b] = tail;
    next[b] = -1;
    if (tail >= 0) next[tail] = b; else head = b;
    tail = b;
    ++nfree;
  }
  void unlink(int32_t b) {
    if (prev[b] >= 0) next[prev[b]] = next[b]; else head = next[b];
    if (next[b] >= 0) prev[next[b]] = prev[b]; else tail = prev[b];
    prev[b] = next[b] = -1;
    --nfree;
  }
  int32_t pop_head() {
    int32_t b = head;
    unlink(b);
    if (cached[b]) {  // reuse evicts the cached hash
      auto it = hash_to_block.find(hash[b]);
      if (it != hash_to_block.end() && it->second == b) hash_to_block.erase(it);
      cached[b] = 0;
      toks[b].clear();
    }
    ref_cnt[b] = 1;
    return b;
  }
  void touch(int32_t b) {
    if (ref_cnt[b] == 0) unlink(b);
    ++ref_cnt[b];
  }
};

extern "C" {

int pa_pool_create(int32_t num_blocks, int32_t block_size, const int32_t* initial_free_order,
                   pa_pool** out) {
  pa::clear_error();
  if (!out) return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_create: out is NULL");
  *out = nullptr;
  if (num_blocks <= 0 || block_size <= 0)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_create: num_blocks=%d block_size=%d", num_blocks,
                    block_size);
  pa_pool* p = new pa_pool();
  p->num_blocks = num_blocks;
  p->block_size = block_size;
  p->prev.assign(num_blocks, -1);
  p->next.assign(num_blocks, -1);
  p->ref_cnt.assign(num_blocks, 0);
  p->cached.assign(num_blocks, 0);
  p->hash.assign(num_blocks, 0);
  p->toks.resize(num_blocks);
  std::vector<uint8_t> seen(num_blocks, 0);
  for (int32_t i = 0; i < num_blocks; ++i) {
    int32_t b = initial_free_order ? initial_free_order[i] : i;
    if (b < 0 || b >= num_blocks || seen[b]) {
      delete p;
      return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_create: initial order is not a permutation");
    }
    seen[b] = 1;
    p->push_tail(b);
  }
  *out = p;
  return PA_OK;
}

void pa_pool_destroy(pa_pool* pool) { delete pool; }

int pa_pool_add_seq(pa_pool* pool, int64_t seq_id, const int32_t* token_ids, int32_t num_tokens,
                    int32_t* num_cached_tokens) {
  pa::clear_error();
  if (!pool) return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_add_seq: pool is NULL");
  if (num_tokens < 0) return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_add_seq: num_tokens < 0");
  if (pool->seqs.count(seq_id))
    return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_add_seq: sequence %lld exists", (long long)seq_id);
  const int32_t bs = pool->block_size;
  const int32_t nblk = (int32_t)(((int64_t)num_tokens + bs - 1) / bs);
  const int32_t nfull = token_ids ? num_tokens / bs : 0;

  std::vector<uint64_t> keys(nfull);
  uint64_t parent = 0;
  for (int32_t i = 0; i < nfull; ++i) {
    parent = block_key(parent, token_ids + (size_t)i * bs, bs);
    keys[i] = parent;
  }
  // longest run of leading full blocks present in the prefix cache
  std::vector<int32_t> hits;
  for (int32_t i = 0; i < nfull; ++i) {
    auto it = pool->hash_to_block.find(keys[i]);
    if (it == pool->hash_to_block.end()) break;
    int32_t b = it->second;
    const std::vector<int32_t>& t = pool->toks[b];
    if (!pool->cached[b] || t.size() != (size_t)bs ||
        std::memcmp(t.data(), token_ids + (size_t)i * bs, sizeof(int32_t) * bs) != 0)
      break;
    hits.push_back(b);
  }
  int32_t parked = 0;
  for (int32_t b : hits) parked += pool->ref_cnt[b] == 0;
  const int32_t need = nblk - (int32_t)hits.size();
  if (need > pool->nfree - parked)
    return pa::fail(PA_ERR_NO_BLOCKS, "pa_pool_add_seq: need %d blocks, %d free", need,
                    pool->nfree - parked);

  Seq seq;
  seq.num_tokens = num_tokens;
  seq.blocks.reserve(nblk);
  for (int32_t b : hits) {
    pool->touch(b);
    seq.blocks.push_back(b);
  }
  for (int32_t i = (int32_t)hits.size(); i < nblk; ++i) {
    int32_t b = pool->pop_head();
    if (i < nfull && !pool->hash_to_block.count(keys[i])) {
      pool->cached[b] = 1;
      pool->hash[b] = keys[i];
      pool->toks[b].assign(token_ids + (size_t)i * bs, token_ids + (size_t)(i + 1) * bs);
      pool->hash_to_block[keys[i]] = b;
    }
    seq.blocks.push_back(b);
  }
  pool->seqs.emplace(seq_id, std::move(seq));
  if (num_cached_tokens) *num_cached_tokens = (int32_t)hits.size() * bs;
  return PA_OK;
}

int pa_pool_append(pa_pool* pool, int64_t seq_id, int32_t n_new, int64_t* slots_out) {
  pa::clear_error();
  if (!pool) return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_append: pool is NULL");
  auto it = pool->seqs.find(seq_id);
  if (it == pool->seqs.end())
    return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_append: unknown sequence %lld", (long long)seq_id);
  if (n_new < 0 || (n_new > 0 && !slots_out))
    return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_append: bad n_new/slots_out");
  Seq& seq = it->second;
  const int64_t bs = pool->block_size;
  const int64_t start = seq.num_tokens;
  const int64_t end = start + n_new;
  if (end > INT32_MAX) return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_append: length overflow");
  // writing into a partly filled last block that another sequence shares:
  // move to a copy of it first
  const bool cow = n_new > 0 && start % bs != 0 && pool->ref_cnt[seq.blocks.back()] > 1;
  const int64_t need = (end + bs - 1) / bs - (int64_t)seq.blocks.size() + (cow ? 1 : 0);
  if (need > pool->nfree)
    return pa::fail(PA_ERR_NO_BLOCKS, "pa_pool_append: need %lld blocks, %d free", (long long)need,
                    pool->nfree);
  if (cow) {
    const int32_t src = seq.blocks.back();
    const int32_t dst = pool->pop_head();
    --pool->ref_cnt[src];
    seq.blocks.back() = dst;
    pool->copy_src.push_back(src);
    pool->copy_dst.push_back(dst);
  }
  for (int64_t p = start; p < end; ++p) {
    if ((int64_t)seq.blocks.size() * bs <= p) seq.blocks.push_back(pool->pop_head());
    slots_out[p - start] = (int64_t)seq.blocks[p / bs] * bs + p % bs;
  }
  seq.num_tokens = (int32_t)end;
  return PA_OK;
}

int pa_pool_fork(pa_pool* pool, int64_t parent_id, int64_t child_id) {
  pa::clear_error();
  if (!pool) return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_fork: pool is NULL");
  auto it = pool->seqs.find(parent_id);
  if (it == pool->seqs.end())
    return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_fork: unknown sequence %lld", (long long)parent_id);
  if (pool->seqs.count(child_id))
    return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_fork: sequence %lld exists", (long long)child_id);
  Seq child = it->second;  // same length and blocks
  for (int32_t b : child.blocks) ++pool->ref_cnt[b];
  pool->seqs.emplace(child_id, std::move(child));
  return PA_OK;
}

int pa_pool_take_copies(pa_pool* pool, int32_t* src, int32_t* dst, int32_t cap, int32_t* n) {
  pa::clear_error();
  if (!pool || !n) return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_take_copies: NULL argument");
  const size_t k = pool->copy_src.size();
  *n = (int32_t)k;
  if ((int64_t)k > cap || (k > 0 && (!src || !dst)))
    return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_take_copies: capacity %d < %zu", cap, k);
  if (k > 0) {
    std::memcpy(src, pool->copy_src.data(), sizeof(int32_t) * k);
    std::memcpy(dst, pool->copy_dst.data(), sizeof(int32_t) * k);
  }
  pool->copy_src.clear();
  pool->copy_dst.clear();
  return PA_OK;
}

int pa_pool_slots(const pa_pool* pool, int64_t seq_id, int32_t start, int32_t n, int64_t* slots_out) {
  pa::clear_error();
  if (!pool) return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_slots: pool is NULL");
  auto it = pool->seqs.find(seq_id);
  if (it == pool->seqs.end())
    return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_slots: unknown sequence %lld", (long long)seq_id);
  const Seq& seq = it->second;
  if (start < 0 || n < 0 || (int64_t)start + n > seq.num_tokens || (n > 0 && !slots_out))
    return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_slots: positions [%d, %d) outside [0, %d)", start,
                    start + n, seq.num_tokens);
  const int64_t bs = pool->block_size;
  for (int32_t i = 0; i < n; ++i) {
    int64_t p = (int64_t)start + i;
    slots_out[i] = (int64_t)seq.blocks[p / bs] * bs + p % bs;
  }
  return PA_OK;
}

int pa_pool_free_seq(pa_pool* pool, int64_t seq_id) {
  pa::clear_error();
  if (!pool) return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_free_seq: pool is NULL");
  auto it = pool->seqs.find(seq_id);
  if (it == pool->seqs.end())
    return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_free_seq: unknown sequence %lld", (long long)seq_id);
  const std::vector<int32_t>& blocks = it->second.blocks;
  for (int32_t b : blocks)
    if (pool->ref_cnt[b] <= 0)
      return pa::fail(PA_ERR_STATE, "pa_pool_free_seq: ref_cnt underflow on block %d", b);
  for (auto r = blocks.rbegin(); r != blocks.rend(); ++r) {
    if (--pool->ref_cnt[*r] == 0) pool->push_tail(*r);
  }
  pool->seqs.erase(it);
  return PA_OK;
}

int pa_pool_block_table(const pa_pool* pool, int64_t seq_id, int32_t* out, int32_t cap, int32_t* n) {
  pa::clear_error();
  if (!pool || !n) return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_block_table: NULL argument");
  auto it = pool->seqs.find(seq_id);
  if (it == pool->seqs.end())
    return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_block_table: unknown sequence %lld", (long long)seq_id);
  const std::vector<int32_t>& blocks = it->second.blocks;
  *n = (int32_t)blocks.size();
  if ((int32_t)blocks.size() > cap || (!out && !blocks.empty()))
    return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_block_table: capacity %d < %d", cap, *n);
  if (!blocks.empty()) std::memcpy(out, blocks.data(), sizeof(int32_t) * blocks.size());
  return PA_OK;
}

int pa_pool_block_tables(const pa_pool* pool, const int64_t* seq_ids, int32_t num_seqs,
                         int32_t max_blocks, int32_t* out) {
  pa::clear_error();
  if (!pool || (num_seqs > 0 && (!seq_ids || !out)) || num_seqs < 0 || max_blocks < 0)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_block_tables: bad arguments");
  for (int32_t s = 0; s < num_seqs; ++s) {
    auto it = pool->seqs.find(seq_ids[s]);
    if (it == pool->seqs.end())
      return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_block_tables: unknown sequence %lld",
                      (long long)seq_ids[s]);
    const std::vector<int32_t>& blocks = it->second.blocks;
    if ((int32_t)blocks.size() > max_blocks)
      return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_block_tables: sequence %lld has %zu > %d blocks",
                      (long long)seq_ids[s], blocks.size(), max_blocks);
    int32_t* row = out + (size_t)s * max_blocks;
    for (int32_t i = 0; i < max_blocks; ++i) row[i] = i < (int32_t)blocks.size() ? blocks[i] : -1;
  }
  return PA_OK;
}

int pa_pool_num_tokens(const pa_pool* pool, int64_t seq_id, int32_t* n) {
  pa::clear_error();
  if (!pool || !n) return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_num_tokens: NULL argument");
  auto it = pool->seqs.find(seq_id);
  if (it == pool->seqs.end())
    return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_num_tokens: unknown sequence %lld", (long long)seq_id);
  *n = it->second.num_tokens;
  return PA_OK;
}

int32_t pa_pool_ref_cnt(const pa_pool* pool, int32_t block) {
  if (!pool || block < 0 || block >= pool->num_blocks) return -1;
  return pool->ref_cnt[block];
}

int32_t pa_pool_num_free(const pa_pool* pool) { return pool ? pool->nfree : -1; }

int pa_pool_free_order(const pa_pool* pool, int32_t* out, int32_t cap, int32_t* n) {
  pa::clear_error();
  if (!pool || !n) return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_free_order: NULL argument");
  *n = pool->nfree;
  if (pool->nfree > cap || (!out && pool->nfree > 0))
    return pa::fail(PA_ERR_INVALID_ARG, "pa_pool_free_order: capacity %d < %d", cap, pool->nfree);
  int32_t i = 0;
  for (int32_t b = pool->head; b >= 0; b = pool->next[b]) out[i++] = b;
  return PA_OK;
}

int pa_prefix_groups(const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                     int32_t num_seqs, int32_t block_size, int32_t* prefix_start, int32_t* prefix_members,
                     int32_t* prefix_blocks, int32_t* seq_prefix, int32_t* seq_slot, int32_t* num_prefixes,
                     int32_t* num_members) {
  pa::clear_error();
  if (num_seqs < 0 || max_blocks_per_seq < 0 || block_size <= 0)
    return pa::fail(PA_ERR_INVALID_ARG, "pa_prefix_groups: bad sizes");
  if (!num_prefixes || !num_members || (num_seqs > 0 && (!block_tables || !seq_lens || !prefix_start ||
                                                         !prefix_members || !prefix_blocks || !seq_prefix ||
                                                         !seq_slot)))
    return pa::fail(PA_ERR_INVALID_ARG, "pa_prefix_groups: NULL pointer");
  // blocks sequence s could share: whole blocks before the one holding its
  // last token, within its table row
  auto cap = [&](int s) {
    const int32_t len = seq_lens[s];
    if (len <= 0) return 0;
    const int32_t c = (len - 1) / block_size;
    return c < max_blocks_per_seq ? c : max_blocks_per_seq;
  };
  const int32_t* row0 = block_tables;
  auto row = [&](int s) { return row0 + (int64_t)s * max_blocks_per_seq; };
  // candidates grouped by their first physical block, in order of first appearance
  std::unordered_map<int32_t, int32_t> group_of_block;
  std::vector<std::vector<int32_t>> groups;
  for (int s = 0; s < num_seqs; ++s) {
    seq_prefix[s] = -1;
    seq_slot[s] = -1;
    if (cap(s) < 1) continue;
    auto it = group_of_block.find(row(s)[0]);
    if (it == group_of_block.end()) {
      group_of_block.emplace(row(s)[0], (int32_t)groups.size());
      groups.push_back({s});
    } else {
      groups[it->second].push_back(s);
    }
  }
  int32_t np = 0, nm = 0;
  prefix_start[0] = 0;
  for (const auto& g : groups) {
    if (g.size() < 2) continue;
    // the longest leading run of blocks every member has in common
    int32_t common = cap(g[0]);
    for (size_t k = 1; k < g.size(); ++k) {
      const int32_t c = cap(g[k]);
      if (c < common) common = c;
      int32_t i = 0;
      while (i < common && row(g[k])[i] == row(g[0])[i]) ++i;
      common = i;
    }
    if (common < 1) continue;
    prefix_blocks[np] = common;
    for (size_t k = 0; k < g.size(); ++k) {
      prefix_members[nm] = g[k];
      seq_prefix[g[k]] = np;
      seq_slot[g[k]] = nm;
      ++nm;
    }
    ++np;
    prefix_start[np] = nm;
  }
  *num_prefixes = np;
  *num_members = nm;
  return PA_OK;
}

}  // extern "C"
