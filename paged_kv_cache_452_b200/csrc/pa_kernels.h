// Internal: kernel parameter blocks and launchers (host <-> device contract).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace pa {

// dtype codes match pa_dtype in pa.h
enum : int { kF32 = 0, kBF16 = 1, kFP8 = 2 };

struct CacheWriteParams {
  const uint8_t* k_new;
  const uint8_t* v_new;
  const int64_t* slots;
  uint8_t* k_cache;
  uint8_t* v_cache;
  int32_t num_tokens, num_kv_heads, head_dim, block_size;
  int64_t num_slots;  // num_blocks * block_size
  float k_scale, v_scale;
  const float* k_head;  // per-kv-head scales (device) or nullptr: k_scale / v_scale
  const float* v_head;
};
cudaError_t launch_cache_write(const CacheWriteParams& p, int in_dtype, int kv_dtype, cudaStream_t stream);

// Whole-block copies inside both pools (copy-on-write): K and V block dst[i]
// become copies of block src[i]; pairs with an id outside [0, num_blocks)
// or src == dst are skipped.
struct CopyBlocksParams {
  const int32_t* src;
  const int32_t* dst;
  int32_t n;
  int32_t num_blocks;
  int64_t block_bytes;  // bytes of one block of one pool
  uint8_t* k_cache;
  uint8_t* v_cache;
};
cudaError_t launch_copy_blocks(const CopyBlocksParams& p, int num_sms, cudaStream_t stream);

// Rows of a decode or mixed step.  Sequence s owns query rows
// qsl[s] .. qsl[s+1]-1 (qsl == nullptr: exactly row s), the last of which
// sits at position seq_lens[s] - 1.
struct AttnRows {
  const int32_t* seq_lens;
  const int32_t* qsl;
  int32_t num_seqs;
  int32_t num_rows;
};

// Workspace carve-up of the split-K decode kernel.
struct DecodeWorkspace {
  int32_t* err;             // error word (first 4 bytes of the caller's buffer)
  unsigned int* cnt;        // [num_seqs * num_kv_heads] arrival counters: zero between calls
  float* ml;                // [workers][G][2] partial (max, sum), one cut piece per warp
  float* o;                 // [workers][G][D] partial unnormalised outputs
};

struct DecodeParams {
  const uint8_t* q;  // bf16 [rows][Hq][D]
  uint8_t* out;      // bf16 [rows][Hq][D]
  const uint8_t* v_cache;
  const int32_t* block_tables;
  int32_t max_blocks;
  AttnRows rows;
  int32_t num_q_heads, num_kv_heads, group;
  int32_t num_blocks;  // table entries outside [0, num_blocks) are flagged and read as block 0
  int32_t nstages;
  int32_t grid;
  float scale_log2;  // softmax scale * log2(e), times the per-tensor K dequant factor for fp8
  float out_scale;   // 1, or the per-tensor V dequant factor for fp8
  const float* k_head;  // fp8 per-kv-head scales (device; they multiply scale_log2 / out_scale) or nullptr
  const float* v_head;
  // fused cache write (pa_decode_fused): the new token's rows [rows][Hkv][D]
  // (bf16) and the pools to store them in; k_new == nullptr: no write
  const uint8_t* k_new;
  const uint8_t* v_new;
  uint8_t* k_pool;
  uint8_t* v_pool;
  float k_scale_w, v_scale_w;  // per-tensor quantisation scales of the write (fp8)
  // shared prefixes (pa_decode_prefix; pfx_of == nullptr: none): sequence s
  // with pfx_of[s] = p >= 0 skips the first pfx_blocks[p] blocks of its row
  // and folds the chunk partials of member slot pfx_slot[s] into its result
  const int32_t* pfx_of;
  const int32_t* pfx_slot;
  const int32_t* pfx_blocks;
  const float* pfx_ml;  // [chunks][num_members][Hq][2]
  const float* pfx_o;   // [chunks][num_members][Hq][D]
  int32_t pfx_members;
  int32_t pfx_chunk_blocks;  // blocks per prefix chunk (prefix_chunk_keys / block_size)
  DecodeWorkspace ws;
};

// kv: kBF16 or kFP8; returns cudaErrorNotSupported for unsupported shapes.
cudaError_t launch_decode_tc(const DecodeParams& p, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                             int kv, int head_dim, int block_size, int num_sms, cudaStream_t stream);
size_t decode_tc_smem_bytes(int kv, int head_dim, int block_size, int group, int num_seqs, int nstages);
int decode_tc_workers(int num_sms);  // the most worker warps a launch can have (workspace sizing)
size_t decode_tc_workspace_bytes(int num_seqs, int num_kv_heads, int group, int head_dim, int num_sms);

// Prompt rows (q_len > 1) of a mixed step on the tensor-core path.
struct PrefillParams {
  const uint8_t* q;  // bf16 [rows][Hq][D]
  uint8_t* out;      // bf16 [rows][Hq][D]
  const int32_t* block_tables;
  int32_t max_blocks;
  AttnRows rows;  // qsl required
  int32_t num_q_heads, num_kv_heads, group, num_blocks;
  int32_t nstages;    // ring stages (the tcgen05 kernel: K stages)
  int32_t nstages_v;  // the tcgen05 kernel's V stages
  float scale_log2;
  int32_t* err;  // workspace error word
  // the tcgen05 kernel's unit queue: a claim counter and a count of CTAs
  // done, both zero between launches (workspace header words 2 and 3)
  int32_t* unit_ctr;
  int32_t* unit_exit;
  int32_t after_decode;  // 1: launched right behind this step's decode kernel
  // Shared-prefix mode of the tcgen05 kernel (pa_decode_prefix): units are
  // (prefix, kv head, tile of members, chunk of prefix keys) and each writes
  // partial (max reference, sum, unnormalised O) rows instead of outputs.
  // rows.num_seqs then counts prefixes; the other rows fields are unused.
  const int32_t* pfx_start;    // [P + 1] CSR into pfx_members
  const int32_t* pfx_members;  // [M] sequence of each member slot (= its decode row)
  const int32_t* pfx_blocks;   // [P] blocks in each prefix
  int32_t num_members;         // M
  int32_t chunk_keys;          // prefix keys per unit, a multiple of 128
  float* pfx_ml;               // [chunks][M][Hq][2] (max reference, sum), log2 domain
  float* pfx_o;                // [chunks][M][Hq][D]
};

// The split of a prefix into chunks of keys that pa_decode_prefix uses: a
// unit of the prefix kernel is (prefix, kv head, 128 / G members, chunk).
// Chunks are whole 128-key tiles, at least two, and as few as give about
// kPrefixUnits units in all: every chunk adds a partial per member row that
// the prefix kernel writes and the decode folds in one after the other, and
// measured on B200 that fold outweighs spreading the prefix over more SMs
// (a 32768-token prefix shared by 64 sequences: 91 us at about 128 units,
// 131 us at 512; a 1024-token prefix: 194 us with 256-key chunks, 237 us
// with 128).  A function of the batch's sizes alone, so the workspace size
// does not depend on the device.
constexpr int kPrefixUnits = 128;
inline int prefix_chunk_keys(int max_prefix_blocks, int block_size, int num_members, int group, int num_kv_heads) {
  const long long keys = (long long)max_prefix_blocks * block_size;
  const int per_tile = 128 / group;  // members per unit
  const long long member_tiles = num_members > per_tile ? (num_members + per_tile - 1) / per_tile : 1;
  const long long per_chunk = member_tiles * (num_kv_heads > 0 ? num_kv_heads : 1);
  const long long chunks = per_chunk >= kPrefixUnits ? 1 : (kPrefixUnits + per_chunk - 1) / per_chunk;
  const long long ck = ((keys + chunks - 1) / chunks + 127) / 128 * 128;
  return (int)(ck < 256 ? 256 : ck);
}
cudaError_t launch_prefix_umma(const PrefillParams& p, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                               int head_dim, int block_size, int num_sms, cudaStream_t stream);
bool prefill_tc_supported(int kv, int q, int head_dim, int block_size, int group);
// The same rows on tcgen05 (TMEM accumulators); cudaErrorNotSupported when
// the shape or the batch's unit table does not fit (the caller falls back).
bool prefill_umma_supported(int kv, int q, int head_dim, int block_size, int group);
// tm_q: the queries as [tokens][Hq][D] bf16, boxes of [128 / G tokens][G
// heads][64 elements] with 128-byte swizzle (one box per 64-column chunk of
// a unit's Q tile).
cudaError_t launch_prefill_umma(const PrefillParams& p, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                const CUtensorMap& tm_q, int head_dim, int block_size, int num_tokens, int num_sms,
                                cudaStream_t stream);
cudaError_t launch_prefill_tc(const PrefillParams& p, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                              int head_dim, int block_size, int num_tokens, cudaStream_t stream);

struct SimtParams {
  const uint8_t* q;  // [rows][Hq][D] in q dtype
  uint8_t* out;
  const uint8_t* k_cache;
  const uint8_t* v_cache;
  const int32_t* block_tables;
  int32_t max_blocks;
  AttnRows rows;
  int32_t num_q_heads, num_kv_heads, head_dim, block_size;
  float scale;
  float k_scale, v_scale;
  const float* k_head;  // fp8 per-kv-head scales (device) or nullptr: k_scale / v_scale
  const float* v_head;
  int32_t only_multi_row;  // 1: skip sequences with exactly one query row
  int32_t num_blocks;      // table entries outside [0, num_blocks) are flagged and read as block 0
  int32_t* err;            // error word of the caller's workspace
};
cudaError_t launch_attn_simt(const SimtParams& p, int q_dtype, int kv_dtype, cudaStream_t stream);

}  // namespace pa
