// pa_cache_write: the slot_mapping scatter of this step's new K/V rows.
//
// Follows the "write(blocks[-1], kv)" step of the block-table snippet on "49
// vLLM / PagedAttention": token t's row goes to offset slot % block_size of
// physical block slot / block_size.  HBM-bound and tiny per decode step; every
// thread moves one 16-byte vector of a new row (coalesced reads; the writes
// of one row land in one contiguous span of the block, except e4m3 V, whose
// block is d-major).
#include <cuda_runtime.h>

#include "pa_device.cuh"
#include "pa_kernels.h"

namespace pa {
namespace {

// IN: element type of k_new/v_new (float or __nv_bfloat16); TO_FP8: quantise.
template <typename IN, bool TO_FP8>
__global__ void __launch_bounds__(256) cache_write_kernel(CacheWriteParams p) {
  dev::grid_dep_wait();
  dev::grid_dep_launch();
  constexpr int VEC = 16 / sizeof(IN);  // elements per 16-byte vector
  const int chunks = p.head_dim / VEC;
  const int64_t per_side = (int64_t)p.num_tokens * p.num_kv_heads * chunks;
  const int64_t total = 2 * per_side;
  for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
       idx += (int64_t)gridDim.x * blockDim.x) {
    const int side = idx >= per_side;  // 0: K, 1: V
    int64_t r = side ? idx - per_side : idx;
    const int c = (int)(r % chunks);
    r /= chunks;
    const int h = (int)(r % p.num_kv_heads);
    const int64_t t = r / p.num_kv_heads;
    const int64_t slot = __ldg(p.slots + t);
    if (slot < 0 || slot >= p.num_slots) continue;
    const int64_t blk = slot / p.block_size;
    const int off = (int)(slot % p.block_size);
    const IN* src = reinterpret_cast<const IN*>(side ? p.v_new : p.k_new) +
                    ((t * p.num_kv_heads + h) * p.head_dim + (int64_t)c * VEC);
    const uint4 raw = __ldg(reinterpret_cast<const uint4*>(src));
    uint8_t* cache = side ? p.v_cache : p.k_cache;
    if constexpr (!TO_FP8) {
      IN* dst = reinterpret_cast<IN*>(cache) +
                (((blk * p.num_kv_heads + h) * p.block_size + off) * p.head_dim + (int64_t)c * VEC);
      *reinterpret_cast<uint4*>(dst) = raw;
    } else {
      const float* head = side ? p.v_head : p.k_head;
      const float scale = head ? __ldg(head + h) : (side ? p.v_scale : p.k_scale);
      float x[VEC];
      if constexpr (sizeof(IN) == 4) {
        x[0] = __uint_as_float(raw.x);
        x[1] = __uint_as_float(raw.y);
        x[2] = __uint_as_float(raw.z);
        x[3] = __uint_as_float(raw.w);
      } else {
        const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          x[2 * i] = dev::bf16_bits_to_f32(w[i] & 0xFFFFu);
          x[2 * i + 1] = dev::bf16_bits_to_f32(w[i] >> 16);
        }
      }
      uint8_t q[VEC];
#pragma unroll
      for (int i = 0; i < VEC; i += 2) {
        const uint16_t pair = dev::e4m3x2_from_f32(__fdiv_rn(x[i], scale), __fdiv_rn(x[i + 1], scale));
        q[i] = (uint8_t)(pair & 0xFF);
        q[i + 1] = (uint8_t)(pair >> 8);
      }
      if (!side) {  // K: token-major, VEC contiguous bytes
        uint8_t* dst = cache + ((blk * p.num_kv_heads + h) * p.block_size + off) * p.head_dim +
                       (int64_t)c * VEC;
        if constexpr (VEC == 8) {
          uint2 v;
          v.x = q[0] | (q[1] << 8) | (q[2] << 16) | ((uint32_t)q[3] << 24);
          v.y = q[4] | (q[5] << 8) | (q[6] << 16) | ((uint32_t)q[7] << 24);
          *reinterpret_cast<uint2*>(dst) = v;
        } else {
          *reinterpret_cast<uint32_t*>(dst) = q[0] | (q[1] << 8) | (q[2] << 16) | ((uint32_t)q[3] << 24);
        }
      } else {  // V: d-major, one byte per d at stride block_size
        uint8_t* dst = cache + ((blk * p.num_kv_heads + h) * p.head_dim + (int64_t)c * VEC) * p.block_size + off;
#pragma unroll
        for (int i = 0; i < VEC; ++i) dst[(int64_t)i * p.block_size] = q[i];
      }
    }
  }
}

}  // namespace

cudaError_t launch_cache_write(const CacheWriteParams& p, int in_dtype, int kv_dtype, cudaStream_t stream) {
  const int elem = in_dtype == 0 ? 4 : 2;
  const int64_t total = 2LL * p.num_tokens * p.num_kv_heads * (p.head_dim * elem / 16);
  if (total == 0) return cudaSuccess;
  const int threads = 256;
  int64_t blocks = (total + threads - 1) / threads;
  if (blocks > 148 * 64) blocks = 148 * 64;
  const bool fp8 = kv_dtype == 2;
  if (in_dtype == 0) {
    if (fp8) cache_write_kernel<float, true><<<(unsigned)blocks, threads, 0, stream>>>(p);
    else cache_write_kernel<float, false><<<(unsigned)blocks, threads, 0, stream>>>(p);
  } else {
    if (fp8) cache_write_kernel<__nv_bfloat16, true><<<(unsigned)blocks, threads, 0, stream>>>(p);
    else cache_write_kernel<__nv_bfloat16, false><<<(unsigned)blocks, threads, 0, stream>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace pa
