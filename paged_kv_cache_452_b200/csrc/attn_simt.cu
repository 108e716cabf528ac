// Paged attention on CUDA cores: fp32 caches (where a 1e-4 tolerance rules
// out reduced-precision tensor-core inputs), GQA group 1 or > 8 (a
// matrix-vector product, not a dense contraction), and the prompt rows of a
// mixed chunked-prefill step.
//
// One warp per (query row, query head); lanes split head_dim; keys are
// visited one at a time through the block table with an online softmax
// (running max, running sum, rescaled accumulator).  Query row r of sequence
// s sits at position seq_lens[s] - q_len_s + (r - first row of s) and attends
// keys 0 .. that position.
#include <cuda_runtime.h>

#include "pa_device.cuh"
#include "pa_kernels.h"

namespace pa {
namespace {

template <int KV>
__device__ __forceinline__ float load_kv(const uint8_t* base, int64_t idx) {
  if constexpr (KV == kF32) {
    return reinterpret_cast<const float*>(base)[idx];
  } else if constexpr (KV == kBF16) {
    return dev::bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(base)[idx]);
  } else {
    return dev::e4m3_to_f32(base[idx]);  // exact
  }
}

template <int QT>
__device__ __forceinline__ float load_q(const uint8_t* base, int64_t idx) {
  if constexpr (QT == kF32) return reinterpret_cast<const float*>(base)[idx];
  else return dev::bf16_bits_to_f32(reinterpret_cast<const uint16_t*>(base)[idx]);
}

template <int QT>
__device__ __forceinline__ void store_out(uint8_t* base, int64_t idx, float v) {
  if constexpr (QT == kF32) reinterpret_cast<float*>(base)[idx] = v;
  else reinterpret_cast<__nv_bfloat16*>(base)[idx] = __float2bfloat16_rn(v);
}

template <int QT, int KV, int D>
__global__ void __launch_bounds__(128) attn_simt_kernel(const SimtParams p) {
  dev::grid_dep_wait();
  constexpr int E = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t wid = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int hq = p.num_q_heads;
  if (wid >= (int64_t)p.rows.num_rows * hq) return;
  const int r = (int)(wid / hq), h = (int)(wid % hq);
  int s = r, first = r, qlen = 1;
  if (p.rows.qsl) {  // last s with qsl[s] <= r
    int lo = 0, hi = p.rows.num_seqs - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (p.rows.qsl[mid] <= r) lo = mid; else hi = mid - 1;
    }
    s = lo;
    first = p.rows.qsl[s];
    qlen = p.rows.qsl[s + 1] - first;
  }
  if (p.only_multi_row && qlen == 1) return;
  int pos = p.rows.seq_lens[s] - qlen + (r - first);
  if (pos >= p.max_blocks * p.block_size) {  // context longer than its table row: flag, clamp
    if (lane == 0) atomicCAS(p.err, 0, 3);
    pos = p.max_blocks * p.block_size - 1;
  }
  const int kvh = h / (hq / p.num_kv_heads);
  const float ks = p.k_head ? __ldg(p.k_head + kvh) : p.k_scale;  // e4m3 dequantisation scales
  const float vs = p.v_head ? __ldg(p.v_head + kvh) : p.v_scale;
  const int hkv = p.num_kv_heads, bs = p.block_size;
  const int64_t qo = ((int64_t)r * hq + h) * D;
  float qv[E], acc[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    qv[e] = load_q<QT>(p.q, qo + lane + 32 * e) * p.scale;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const int32_t* table = p.block_tables + (int64_t)s * p.max_blocks;
  for (int j = 0; j <= pos; ++j) {
    int64_t blk = table[j / bs];
    if (blk < 0 || blk >= p.num_blocks) {  // bad table entry: flag it, read block 0
      if (lane == 0) atomicCAS(p.err, 0, 2);
      blk = 0;
    }
    const int off = j % bs;
    const int64_t kb = ((blk * hkv + kvh) * bs + off) * D;
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < E; ++e) dot += qv[e] * load_kv<KV>(p.k_cache, kb + lane + 32 * e);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
    if (KV == kFP8) dot *= ks;
    const float mn = fmaxf(m, dot);
    const float corr = expf(m - mn), pj = expf(dot - mn);
    l = l * corr + pj;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const int d = lane + 32 * e;
      const int64_t vi = KV == kFP8 ? ((blk * hkv + kvh) * D + d) * bs + off : kb + d;
      acc[e] = acc[e] * corr + pj * load_kv<KV>(p.v_cache, vi);
    }
    m = mn;
  }
  const float inv = (pos >= 0 ? 1.f / l : 0.f) * (KV == kFP8 ? vs : 1.f);
#pragma unroll
  for (int e = 0; e < E; ++e) store_out<QT>(p.out, qo + lane + 32 * e, pos >= 0 ? acc[e] * inv : 0.f);
}

template <int QT, int KV>
cudaError_t launch_d(const SimtParams& p, cudaStream_t stream) {
  const int64_t warps = (int64_t)p.rows.num_rows * p.num_q_heads;
  if (warps == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((warps + 3) / 4);
  if (p.head_dim == 64) attn_simt_kernel<QT, KV, 64><<<grid, 128, 0, stream>>>(p);
  else if (p.head_dim == 128) attn_simt_kernel<QT, KV, 128><<<grid, 128, 0, stream>>>(p);
  else return cudaErrorNotSupported;
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_simt(const SimtParams& p, int q_dtype, int kv_dtype, cudaStream_t stream) {
  if (q_dtype == kF32) {
    if (kv_dtype == kF32) return launch_d<kF32, kF32>(p, stream);
    if (kv_dtype == kFP8) return launch_d<kF32, kFP8>(p, stream);
  } else if (q_dtype == kBF16) {
    if (kv_dtype == kBF16) return launch_d<kBF16, kBF16>(p, stream);
    if (kv_dtype == kFP8) return launch_d<kBF16, kFP8>(p, stream);
  }
  return cudaErrorNotSupported;
}

}  // namespace pa
