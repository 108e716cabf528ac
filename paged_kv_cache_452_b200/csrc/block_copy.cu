// pa_copy_blocks: whole-block copies inside the K and V pools, the device
// half of copy-on-write.  "PagedAttention：KV cache 即虚拟内存（block manager &
// 碎片）", section 深入原理, 共享 → prefix caching: blocks shared by several
// sequences are copied when a fork diverges inside one; "49 vLLM /
// PagedAttention", Почему это важно: shared blocks are copy-on-write, like
// pages shared between processes.  The host pool decides which blocks to
// copy (pa_pool_append, pa_pool_take_copies); this kernel moves the bytes.
//
// A block of one pool is one contiguous span of Hkv * bs * D elements in
// every layout ([NB][Hkv][bs][D], and [NB][Hkv][D][bs] for an e4m3 V pool),
// so a pair is two flat copies.  The work is HBM-bound: a CTA takes one
// block of one pool at a time and its threads stream it in 16-byte vectors,
// four loads in flight per thread before the stores, with streaming cache
// hints (the bytes are not read again soon); the grid is a multiple of the
// SM count and strides over all pairs and both pools.
#include <cuda_runtime.h>

#include "pa_device.cuh"
#include "pa_kernels.h"

namespace pa {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;
constexpr int kCtasPerSM = 8;  // 2 048 threads per SM

// Work item 2i copies K block src[i] to dst[i], item 2i + 1 the V block.
template <typename V>
__global__ void __launch_bounds__(kThreads) copy_blocks_kernel(const CopyBlocksParams p) {
  const int64_t vecs = p.block_bytes / (int64_t)sizeof(V);
  for (int item = blockIdx.x; item < 2 * p.n; item += gridDim.x) {
    const int i = item >> 1;
    const int32_t s = __ldg(p.src + i), d = __ldg(p.dst + i);
    if (s < 0 || s >= p.num_blocks || d < 0 || d >= p.num_blocks || s == d) continue;
    uint8_t* pool = (item & 1) ? p.v_cache : p.k_cache;
    const V* from = reinterpret_cast<const V*>(pool + (int64_t)s * p.block_bytes);
    V* to = reinterpret_cast<V*>(pool + (int64_t)d * p.block_bytes);
    for (int64_t j = threadIdx.x; j < vecs; j += (int64_t)kThreads * kUnroll) {
      V r[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t k = j + (int64_t)u * kThreads;
        if (k < vecs) r[u] = __ldcs(from + k);
      }
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) {
        const int64_t k = j + (int64_t)u * kThreads;
        if (k < vecs) __stcs(to + k, r[u]);
      }
    }
  }
}

template <typename V>
cudaError_t launch(const CopyBlocksParams& p, int num_sms, cudaStream_t stream) {
  const int items = 2 * p.n;
  const int grid = items < kCtasPerSM * num_sms ? items : kCtasPerSM * num_sms;
  copy_blocks_kernel<V><<<grid, kThreads, 0, stream>>>(p);
  return cudaPeekAtLastError();
}

}  // namespace

cudaError_t launch_copy_blocks(const CopyBlocksParams& p, int num_sms, cudaStream_t stream) {
  if (p.n <= 0) return cudaSuccess;
  // the widest access that divides a block (the pools are 16-byte aligned)
  if (p.block_bytes % 16 == 0) return launch<uint4>(p, num_sms, stream);
  if (p.block_bytes % 4 == 0) return launch<unsigned int>(p, num_sms, stream);
  return launch<unsigned char>(p, num_sms, stream);
}

}  // namespace pa
