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
  float scale_log2;  // softmax scale * log2(e), times the K dequant factor for fp8
  float out_scale;   // 1, or the V dequant factor for fp8
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
};
bool prefill_tc_supported(int kv, int q, int head_dim, int block_size, int group);
// The same rows on tcgen05 (TMEM accumulators); cudaErrorNotSupported when
// the shape or the batch's unit table does not fit (the caller falls back).
bool prefill_umma_supported(int kv, int q, int head_dim, int block_size, int group);
cudaError_t launch_prefill_umma(const PrefillParams& p, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                int head_dim, int block_size, int num_tokens, int num_sms, cudaStream_t stream);
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
  int32_t only_multi_row;  // 1: skip sequences with exactly one query row
  int32_t num_blocks;      // table entries outside [0, num_blocks) are flagged and read as block 0
  int32_t* err;            // error word of the caller's workspace
};
cudaError_t launch_attn_simt(const SimtParams& p, int q_dtype, int kv_dtype, cudaStream_t stream);

}  // namespace pa
