/*
 * pa.h -- C ABI of the paged KV-cache decode-attention library (libpa.so).
 *
 * The operation.  A sequence's keys and values live in fixed-size physical
 * blocks of block_size tokens (16 by default) drawn from one pool; the blocks
 * of a sequence need not be contiguous, and a per-sequence block table maps
 * its logical block i to a physical block ("vLLM innenfra: slik gjør paged
 * attention GPU-minnet til blokker på 16 tokens", paragraph 2; "49 vLLM /
 * PagedAttention", section "Идея и механизм"; "PagedAttention：KV cache 即虚拟
 * 内存（block manager & 碎片）", section 直接答案).  Paging changes neither
 * the attention output nor the amount of compute (same page, follow-up
 * "分页改变输出或加速 kernel 吗？"): the kernels here compute ordinary softmax
 * attention, gathering K/V through the table.
 *
 * Conventions for every call
 *  - Return value: PA_OK (0) or a pa_status error code; pa_last_error()
 *    returns a message for the last failure on the calling thread.
 *  - Device pointers are owned by the caller.  The library never allocates
 *    device memory: scratch space comes from a caller buffer sized by the
 *    matching *_workspace_size call.
 *  - Device calls are asynchronous on `stream` (a cudaStream_t; NULL = the
 *    legacy default stream).  Launch failures come back as PA_ERR_CUDA;
 *    argument checks are done on the host before anything is enqueued, so an
 *    error return means nothing was launched.
 *  - Pool calls are host-only, single-threaded per pool, and never touch KV
 *    bytes.
 *
 * Data layout in device memory
 *  - K pool: [num_blocks][num_kv_heads][block_size][head_dim].
 *  - V pool: the same for PA_F32 / PA_BF16 caches; d-major
 *    [num_blocks][num_kv_heads][head_dim][block_size] for PA_FP8_E4M3 caches.
 *  - Flat slot of the token at position p of a sequence with block table T:
 *    T[p / block_size] * block_size + p % block_size.
 *  - Queries, new K/V rows and outputs are row-major [rows][heads][head_dim]
 *    in the query dtype.  Query head h reads KV head h / (num_q_heads /
 *    num_kv_heads).
 *  - Block tables: int32 [num_seqs][max_blocks_per_seq], row s padded past
 *    its last block with any value (never read).
 *  - All base pointers 16-byte aligned.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID_ARG = 1, /* bad pointer, size, alignment or id */
  PA_ERR_UNSUPPORTED = 2, /* valid but not built: dtype/head_dim/block_size/group combination */
  PA_ERR_NO_BLOCKS = 3,   /* pool exhausted; the pool is left unchanged */
  PA_ERR_CUDA = 4,        /* a CUDA runtime/driver call failed */
  PA_ERR_STATE = 5        /* inconsistent pool state (e.g. ref_cnt underflow) */
} pa_status;

typedef enum { PA_F32 = 0, PA_BF16 = 1, PA_FP8_E4M3 = 2 } pa_dtype;

/* Shape and storage of one layer's paged cache. */
typedef struct {
  int32_t num_blocks;   /* physical blocks in the pool */
  int32_t block_size;   /* tokens per block: 16 or 32 */
  int32_t num_kv_heads;
  int32_t num_q_heads;  /* a multiple of num_kv_heads */
  int32_t head_dim;     /* 64 or 128 */
  int32_t kv_dtype;     /* pa_dtype of the pool */
  int32_t q_dtype;      /* pa_dtype of queries, new K/V and outputs: PA_F32 or PA_BF16 */
  float k_scale;        /* per-tensor scales of an e4m3 pool (stored = e4m3(x / scale)); */
  float v_scale;        /* ignored for fp32/bf16 pools */
  /* Per-kv-head scales of an e4m3 pool: NULL, or a device array of
   * num_kv_heads positive finite fp32 values (4-byte aligned, owned by the
   * caller, read by the kernels): kv head h stores e4m3(x / scale[h]) and
   * its codes dequantise to code * scale[h]; k_scale (v_scale) is then
   * unused for K (V).  Ignored for fp32/bf16 pools.  The pages leave the
   * granularity of an FP8 cache's scale open ("PagedAttention：KV cache
   * 即虚拟内存（block manager & 碎片）", the num_gpu_blocks formula and the
   * follow-up on a KV-bound step). */
  const float* k_head_scales;
  const float* v_head_scales;
} pa_cache_desc;

/* Message for the last failing call on this thread ("" if none). */
const char* pa_last_error(void);

/* Library version string. */
const char* pa_version(void);

/* Bytes one physical block holds for K and V together:
 * 2 * block_size * num_kv_heads * head_dim * sizeof(kv element)
 * ("vLLM innenfra ...", paragraph 2).  Returns 0 for an invalid desc. */
size_t pa_block_bytes(const pa_cache_desc* desc);

/* ---- device calls --------------------------------------------------------- */

/* pa_cache_write: scatter this step's new K and V rows into their blocks.
 * Follows the "write(blocks[-1], kv)" step of the block-table snippet on "49
 * vLLM / PagedAttention"; slot_mapping carries each new token's flat slot.
 *   k_new, v_new   device, [num_tokens][num_kv_heads][head_dim], q_dtype
 *   slot_mapping   device, int64 [num_tokens]; a negative slot is skipped, and
 *                  so is a slot >= num_blocks * block_size
 *   k_cache/v_cache device pools (layout above), written in place
 * fp32 -> fp32 and bf16 -> bf16 are bit copies; fp32/bf16 -> e4m3 stores
 * e4m3(fp32(x) / fp32(scale)) rounded to nearest-even with saturation to
 * +-448.  bf16 -> fp32 and fp32 -> bf16 are PA_ERR_UNSUPPORTED.  Two new
 * tokens with the same slot race (last writer unspecified). */
int pa_cache_write(const pa_cache_desc* desc, const void* k_new, const void* v_new,
                   const int64_t* slot_mapping, int32_t num_tokens, void* k_cache, void* v_cache,
                   void* stream);

/* pa_decode_fused: pa_cache_write of each sequence's new token and
 * pa_decode, in one launch (the write of "write(blocks[-1], kv)" in the
 * block-table snippet on "49 vLLM / PagedAttention", followed by the step's
 * attention).  Sequence s's new token sits at position p = seq_lens[s] - 1
 * (seq_lens counts it, as for pa_decode); its rows k_new[s], v_new[s] are
 * stored at p's slot, block_tables[s][p / block_size] * block_size +
 * p % block_size, as exactly the bytes pa_cache_write stores (e4m3
 * quantisation included), and the attention over keys 0 .. p uses them.
 * The result (pool bytes and out) equals pa_cache_write followed by
 * pa_decode; only the tensor-core decode path is fused (bf16 queries, a bf16
 * or e4m3 pool, GQA group 2..8; head_dim 64/128 for bf16, 128 for e4m3):
 * other descs give PA_ERR_UNSUPPORTED.
 *   k_new, v_new   device, [num_seqs][num_kv_heads][head_dim], bf16
 *   k_cache, v_cache  device pools, written at each new token's slot
 *   other arguments and the workspace as for pa_decode (a sequence with
 *   seq_lens[s] == 0 writes nothing and gives a zero row). */
int pa_decode_fused(const pa_cache_desc* desc, const void* q, const void* k_new, const void* v_new, void* k_cache,
                    void* v_cache, const int32_t* block_tables, int32_t max_blocks_per_seq,
                    const int32_t* seq_lens, int32_t num_seqs, float scale, void* out, void* workspace,
                    size_t workspace_bytes, void* stream);

/* pa_copy_blocks: the device half of copy-on-write ("PagedAttention：KV
 * cache 即虚拟内存（block manager & 碎片）", 深入原理, 共享 → prefix caching: a
 * fork that diverges inside a shared block triggers a copy).  For i < n, K
 * block dst[i] and V block dst[i] become byte copies of blocks src[i]
 * (every kv head and slot, in the pool's storage format).
 *   src, dst   device, int32 [n] block ids (from pa_pool_take_copies); a
 *              pair with an id outside [0, num_blocks), or src == dst, is
 *              skipped
 *   k_cache, v_cache  device pools as for pa_cache_write, 16-byte aligned
 * The pairs run concurrently: no block may be a destination twice, or both
 * a destination and a source, in one call.  Asynchronous on `stream`; run
 * it before the pa_cache_write that writes into the new blocks. */
int pa_copy_blocks(const pa_cache_desc* desc, const int32_t* src, const int32_t* dst, int32_t n,
                   void* k_cache, void* v_cache, void* stream);

/* Scratch bytes pa_decode needs for num_seqs sequences on the current device. */
size_t pa_decode_workspace_size(const pa_cache_desc* desc, int32_t num_seqs);

/* pa_decode: one decode step of paged attention.  Sequence s has one query
 * row (row s of q) at position seq_lens[s] - 1 and attends its keys
 * 0 .. seq_lens[s] - 1, gathered through block_tables[s]; seq_lens counts
 * the token written this step.  out[s][h][:] = softmax(scale * q K^T) V.
 * The block table plays the page table's part ("49 vLLM / PagedAttention",
 * «Идея и механизм»); the result is the one dense attention gives over the
 * same keys ("PagedAttention：KV cache 即虚拟内存（block manager & 碎片）",
 * the follow-up "分页改变输出或加速 kernel 吗？").
 *   q           device, [num_seqs][num_q_heads][head_dim], q_dtype
 *   block_tables device, int32 [num_seqs][max_blocks_per_seq]
 *   seq_lens    device, int32 [num_seqs]; 0 gives a zero output row
 *   out         device, [num_seqs][num_q_heads][head_dim], q_dtype
 *   workspace   device, >= pa_decode_workspace_size bytes, 256-byte aligned,
 *               zero-filled once before its first use; every call leaves it
 *               ready for the next (also when replayed from a CUDA graph).
 *               Its first 4 bytes are an error word the kernels set (never
 *               clear): 1 = a bounded internal wait timed out, 2 = a block
 *               table entry outside [0, num_blocks) (read as block 0),
 *               3 = a sequence longer than its table row (clamped),
 *               5 = an internal consistency check failed (a library bug;
 *               the affected rows are not written).  Read it
 *               after the stream synchronises; after any error, zero the
 *               whole workspace again.  Calls sharing a workspace must not
 *               overlap on the GPU.  Bytes 4..7 are a fault-injection word
 *               for tests, zero in normal use: set to 1, the later pieces of
 *               a context split over several warps do not report in, so the
 *               merging warp's bounded wait runs out (after 1 ms) and sets
 *               error word 1 without any fault; that call's output is wrong.
 * Forward progress: the split-K merge waits for pieces held by other CTAs
 * of the same launch, so the launch is sized to be resident all at once
 * (the CTAs per SM the runtime reports, times the SMs).  Do not run two
 * pa_decode calls at the same time on one GPU (separate streams without an
 * ordering between them): each could hold SMs the other's waiting pieces
 * need, and both would end at the 2 s bound with error word 1.
 * Long contexts are split over many CTAs (split-K over blocks) and merged
 * with a log-sum-exp combine; the split points depend only on seq_lens and
 * the device, so a result does not depend on where the blocks sit. */
int pa_decode(const pa_cache_desc* desc, const void* q, const void* k_cache, const void* v_cache,
              const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
              int32_t num_seqs, float scale, void* out, void* workspace, size_t workspace_bytes,
              void* stream);

/* pa_decode_static: pa_decode without a caller workspace, for callers that
 * cannot allocate device memory (inside a captured CUDA graph where
 * allocation is not allowed, under another owner's allocator, or on a path
 * that must not allocate after start-up).  The paper has no counterpart;
 * this is a convenience of this library.
 * Same arguments and result as pa_decode, minus the workspace: the scratch
 * is an 8 MiB area compiled into the library, held by every GPU that loads
 * it until the process exits.  Batches whose pa_decode_workspace_size
 * exceeds 8 MiB are rejected with PA_ERR_UNSUPPORTED (use pa_decode).
 * The first call on a device looks up the area's device address (with that
 * device current); make that first call before any stream capture.  Every
 * call clears the area's error word and arrival counters on `stream` first,
 * so the in-kernel reports that pa_decode leaves in its workspace's error
 * word are neither kept between calls nor readable by the caller: a call
 * whose kernel met an out-of-pool table entry or a timed-out wait still
 * returns PA_OK (use pa_decode where those reports are needed).  Argument
 * checks are pa_decode's, made before anything is enqueued.  All calls share
 * the one area: calls that overlap on the GPU race.  Allocates nothing. */
int pa_decode_static(const pa_cache_desc* desc, const void* q, const void* k_cache, const void* v_cache,
                     const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                     int32_t num_seqs, float scale, void* out, void* stream);

/* ---- shared prefixes ------------------------------------------------------
 * Sequences admitted with prefix caching share the physical blocks of a
 * common prefix (ref_cnt > 1; "49 vLLM / PagedAttention", Почему это важно;
 * "PagedAttention：KV cache 即虚拟内存（block manager & 碎片）", 深入原理,
 * 共享 → prefix caching).  pa_decode reads those blocks once per sequence;
 * pa_decode_prefix attends each shared prefix once for all its sequences,
 * as one dense contraction (every member's query rows against the prefix's
 * keys) on the tensor cores, and merges that partial result with each
 * sequence's own suffix by a log-sum-exp combine. */

/* pa_prefix_groups (host): the shared prefixes of a decode batch, from its
 * block tables.  Sequences whose rows start with the same physical block form
 * a group when there are two or more; the group's prefix is the longest run
 * of leading table entries all members have in common, cut so that every
 * member keeps at least its last token (position seq_lens[s] - 1) outside
 * it.  Groups with an empty prefix are dropped.
 *   block_tables  host int32 [num_seqs][max_blocks_per_seq]; seq_lens host
 *                 int32 [num_seqs] (as for pa_decode)
 *   outputs (host, caller-allocated): prefix_start [num_seqs + 1] and
 *   prefix_members [num_seqs] (CSR: prefix p's sequences are
 *   prefix_members[prefix_start[p] .. prefix_start[p+1] - 1], increasing),
 *   prefix_blocks [num_seqs] (blocks in prefix p), seq_prefix / seq_slot
 *   [num_seqs] (sequence s's prefix and its index in prefix_members, or -1),
 *   *num_prefixes, *num_members. */
int pa_prefix_groups(const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                     int32_t num_seqs, int32_t block_size, int32_t* prefix_start, int32_t* prefix_members,
                     int32_t* prefix_blocks, int32_t* seq_prefix, int32_t* seq_slot, int32_t* num_prefixes,
                     int32_t* num_members);

/* Scratch bytes pa_decode_prefix needs: pa_decode's plus the prefixes'
 * partial results (num_members sequences, prefixes of up to
 * max_prefix_blocks blocks).  The partials are kept per chunk of a prefix's
 * keys: whole 128-key tiles, at least 256 keys, as few chunks as give about
 * 128 prefix-kernel units (a unit = prefix x kv head x 128/G members x
 * chunk), each chunk holding (reference, sum) and head_dim fp32 values per
 * member row and query head. */
size_t pa_decode_prefix_workspace_size(const pa_cache_desc* desc, int32_t num_seqs, int32_t num_members,
                                       int32_t max_prefix_blocks);

/* pa_decode_prefix: pa_decode's result for a batch with shared prefixes
 * described as pa_prefix_groups gives them (device copies of its outputs):
 *   prefix_start [num_prefixes + 1], prefix_members [num_members],
 *   prefix_blocks [num_prefixes], seq_prefix [num_seqs], seq_slot [num_seqs]
 *   device int32; max_prefix_blocks (host) >= every prefix_blocks[p].
 * Every member's table row must hold the prefix's blocks in its first
 * prefix_blocks[p] entries and its context must extend past them.  A bf16
 * pool with bf16 queries, a GQA group of 2..8 and head_dim 64/128 runs the
 * prefixes on a tcgen05 kernel, then the suffixes on the decode kernel,
 * which folds each prefix partial in; other descs (and num_prefixes == 0)
 * run pa_decode.  The workspace is as for pa_decode, sized by
 * pa_decode_prefix_workspace_size; error word 4 = a context that does not
 * extend past its prefix (that row is zero).  When it pays: pa_decode
 * re-reads a shared prefix once per sharing sequence, from L2 when the
 * prefix's K/V fit there (then pa_decode is the faster of the two: measured
 * on B200, a 4 MB prefix shared by 128 sequences took 204 us this way
 * against 163 us) and from HBM when they do not (a 134 MB prefix shared by
 * 64 sequences: 142 us this way against 869 us). */
int pa_decode_prefix(const pa_cache_desc* desc, const void* q, const void* k_cache, const void* v_cache,
                     const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                     int32_t num_seqs, const int32_t* prefix_start, const int32_t* prefix_members,
                     const int32_t* prefix_blocks, const int32_t* seq_prefix, const int32_t* seq_slot,
                     int32_t num_prefixes, int32_t num_members, int32_t max_prefix_blocks, float scale, void* out,
                     void* workspace, size_t workspace_bytes, void* stream);

/* Scratch bytes pa_decode_chunked_prefill needs. */
size_t pa_prefill_workspace_size(const pa_cache_desc* desc, int32_t num_seqs, int32_t num_tokens);

/* pa_decode_chunked_prefill: one mixed step where some sequences add a chunk
 * of prompt tokens and others decode one token ("vLLM innenfra ...", the
 * step() list, item 1, and the paragraph on continuous batching: prefill and
 * decode share a step).  Sequence s owns query rows
 * query_start_loc[s] .. query_start_loc[s+1]-1 (q_len_s rows); its row i sits
 * at position seq_lens[s] - q_len_s + i and attends keys 0 .. that position
 * (causal).  seq_lens counts every token including this step's.  The new
 * tokens' K/V must already be in the pool (pa_cache_write).
 *   q, out          device, [num_tokens][num_q_heads][head_dim], q_dtype
 *   query_start_loc device, int32 [num_seqs + 1], query_start_loc[0] = 0,
 *                   non-decreasing, query_start_loc[num_seqs] = num_tokens
 *   seq_lens        device, int32 [num_seqs], seq_lens[s] >= q_len_s
 *   max_q_len       host, >= every q_len_s
 *   workspace       as for pa_decode, sized by pa_prefill_workspace_size.
 * Decode rows (q_len_s = 1) run on pa_decode's kernels.  Prompt rows of a
 * bf16 pool with bf16 queries run on a tcgen05 kernel (TMEM accumulators)
 * when the GQA group divides 128 and the batch's unit table fits in shared
 * memory, else on an mma.sync kernel when the group divides 64, else on the
 * CUDA-core kernel; every dtype and group is served.  Errors and the
 * workspace error word are as for pa_decode. */
int pa_decode_chunked_prefill(const pa_cache_desc* desc, const void* q, const void* k_cache,
                              const void* v_cache, const int32_t* block_tables,
                              int32_t max_blocks_per_seq, const int32_t* query_start_loc,
                              const int32_t* seq_lens, int32_t num_seqs, int32_t num_tokens,
                              int32_t max_q_len, float scale, void* out, void* workspace,
                              size_t workspace_bytes, void* stream);

/* ---- host block pool --------------------------------------------------------
 * The block manager of "PagedAttention：KV cache 即虚拟内存（block manager &
 * 碎片）", section 深入原理: free_block_queue is a doubly linked list in
 * eviction order (pop head to allocate, push tail to release, both O(1));
 * every block has a ref_cnt; full blocks are keyed by a hash of their tokens
 * and their parent's hash so that equal prefixes share blocks (touch()
 * raises ref_cnt); a finished sequence decrements ref_cnt and releases a
 * block at 0.  Decoding takes a new block exactly when the token being
 * appended starts one (block-table snippet on "49 vLLM / PagedAttention").
 *
 * Details the pages leave open, as implemented:
 *  - block hash: FNV-1a 64 over the parent hash (8 bytes little endian, 0
 *    for the first block) then the block's token ids (int32 little endian);
 *    a hit also compares the stored token ids;
 *  - sharing covers the longest run of leading full blocks found in the
 *    map; a newly allocated full block enters the map unless its hash is
 *    already there;
 *  - a released block keeps its hash while parked in the free queue and can
 *    still be shared (touch() unlinks it); popping it for reuse evicts it;
 *  - release walks a sequence's blocks in reverse logical order;
 *  - every allocation is all-or-nothing (PA_ERR_NO_BLOCKS changes nothing);
 *  - blocks filled by pa_pool_append are never hashed;
 *  - copy-on-write ("分叉触发 copy-on-write" in the same bullet) copies a
 *    shared block only when a sequence writes into it while it is partly
 *    filled; a full shared block is never copied (see pa_pool_append). */

typedef struct pa_pool pa_pool;

/* initial_free_order: NULL for 0..num_blocks-1, else a permutation of it
 * (head first).  *out receives a handle owned by the library. */
int pa_pool_create(int32_t num_blocks, int32_t block_size, const int32_t* initial_free_order,
                   pa_pool** out);
void pa_pool_destroy(pa_pool* pool);

/* Admit a prompt of num_tokens (token_ids NULL: no prefix sharing).
 * num_cached_tokens (nullable) receives the tokens covered by shared blocks. */
int pa_pool_add_seq(pa_pool* pool, int64_t seq_id, const int32_t* token_ids, int32_t num_tokens,
                    int32_t* num_cached_tokens);

/* Grow a sequence by n_new tokens; slots_out[n_new] receives their flat slots.
 * Copy-on-write: if n_new > 0 and the sequence's last block is partly filled
 * and shared (ref_cnt > 1, after pa_pool_fork), the sequence first moves to
 * a block popped from the head of the free queue; the pair (shared block,
 * new block) is queued for pa_pool_take_copies, the shared block's ref_cnt
 * drops by one, and the new tokens go to the new block.  That block counts
 * toward the all-or-nothing check. */
int pa_pool_append(pa_pool* pool, int64_t seq_id, int32_t n_new, int64_t* slots_out);

/* Fork: child_id becomes a sequence with parent_id's length and block
 * table; every block's ref_cnt rises by one (the blocks are shared, copy on
 * write).  PA_ERR_INVALID_ARG if the parent is unknown or the child exists. */
int pa_pool_fork(pa_pool* pool, int64_t parent_id, int64_t child_id);

/* The block copies that copy-on-write queued, oldest first: src[i] is the
 * shared block, dst[i] its new copy.  *n receives the count and the queue is
 * emptied; PA_ERR_INVALID_ARG if cap < count (*n is still set, the queue
 * kept).  Run them on the device with pa_copy_blocks before the
 * pa_cache_write of the tokens that pa_pool_append placed in the copies. */
int pa_pool_take_copies(pa_pool* pool, int32_t* src, int32_t* dst, int32_t cap, int32_t* n);

/* Flat slots of positions [start, start + n) of a sequence (all < its length). */
int pa_pool_slots(const pa_pool* pool, int64_t seq_id, int32_t start, int32_t n, int64_t* slots_out);

/* Release a sequence: ref_cnt-- per block, blocks reaching 0 go to the tail. */
int pa_pool_free_seq(pa_pool* pool, int64_t seq_id);

/* Copy a sequence's block table into out[cap]; *n receives its length
 * (PA_ERR_INVALID_ARG if cap is too small; *n is still set). */
int pa_pool_block_table(const pa_pool* pool, int64_t seq_id, int32_t* out, int32_t cap, int32_t* n);

/* Fill out[num_seqs][max_blocks] with the tables of seq_ids, padding with -1. */
int pa_pool_block_tables(const pa_pool* pool, const int64_t* seq_ids, int32_t num_seqs,
                         int32_t max_blocks, int32_t* out);

/* Tokens a sequence holds. */
int pa_pool_num_tokens(const pa_pool* pool, int64_t seq_id, int32_t* n);

/* ref_cnt of a block (-1 if out of range). */
int32_t pa_pool_ref_cnt(const pa_pool* pool, int32_t block);

/* Blocks in the free queue. */
int32_t pa_pool_num_free(const pa_pool* pool);

/* The free queue head to tail into out[cap]; *n receives its length. */
int pa_pool_free_order(const pa_pool* pool, int32_t* out, int32_t cap, int32_t* n);

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
