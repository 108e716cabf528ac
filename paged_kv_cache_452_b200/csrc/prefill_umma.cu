// Prompt rows of a mixed chunked-prefill + decode step on the 5th-generation
// tensor cores (tcgen05, TMEM accumulators): bf16 queries over a bf16 pool.
//
// What it computes: every query row of a sequence that adds a chunk of
// prompt tokens this step attends, causally, the sequence's keys up to its
// own position, gathered block by block through the block table ("vLLM
// innenfra: slik gjør paged attention GPU-minnet til blokker på 16 tokens",
// the step() list: a step schedules decode and chunked prefill together; the
// chunk's K/V are already in the pool).
//
// How: one CTA per unit = (sequence, kv head, 128 / G query positions).  The
// GQA group's heads of each position fill the MMA's M = 128 rows, so every
// K/V tile serves all of them.
//  * warp 0 walks the block table and brings 128-key K/V tiles into a ring of
//    shared-memory stages with TMA (2-D boxes of [block][128 B], 128-byte
//    swizzle, boxes of consecutive blocks stacked into one swizzled tile);
//    blocks past the keys the unit needs are read out of range, which TMA
//    fills with zeros;
//  * warp 1 holds the TMEM allocation and, from one thread, issues
//    S = Q K^T (M 128, N 128, K 16 steps; double-buffered S in TMEM) and
//    O += P V (N = head_dim; O stays in TMEM across tiles), committing each
//    to an mbarrier;
//  * warps 2..5 own one query row per thread: they read the row of S from
//    TMEM, mask (causal, context length), keep a running max reference that
//    moves only when the row's max grows by more than 2^8 (then the row of
//    O in TMEM and the running sum are rescaled: the result is unchanged,
//    the rescale is rare), write P = 2^(s - ref) as bf16 into a swizzled
//    shared tile for the PV MMA, and at the end divide O by the sum.
// Every wait is bounded (2 s, then the error word is set); TMEM is freed on
// every path.
#include <cuda_runtime.h>

#include "pa_device.cuh"
#include "pa_kernels.h"

namespace pa {
namespace {

constexpr int kRows = 128;    // query rows per unit (positions x group): the MMA's M
constexpr int kKeys = 128;    // keys per K/V tile: N of S = Q K^T, K of O = P V
constexpr int kThreads = 192;  // warp 0 loads, warp 1 issues MMAs, warps 2..5 one row per thread
constexpr uint32_t kTmemCols = 512;
constexpr int kSmemOptIn = 232448;  // 227 KB per block
constexpr int kChunk = 128 * 128;   // one 128-byte-wide chunk of a 128-row tile
constexpr float kRefSlack = 8.f;    // log2 growth of a row max before its reference moves

template <int D, int BS>
struct U {
  static constexpr int NCH = D / 64;               // 128-byte chunks of a row
  static constexpr int QBYTES = NCH * kChunk;      // Q tile
  static constexpr int KVT = NCH * kChunk;         // K (or V) tile
  static constexpr int STAGE = 2 * KVT;
  static constexpr int BPT = kKeys / BS;           // blocks per tile
  static constexpr int BOXES = 2 * NCH * BPT;      // TMA boxes per stage
  static constexpr int KSTEPS_S = D / 16;
  static constexpr int KSTEPS_O = kKeys / 16;
  static_assert(BOXES <= 32, "one box per producer lane");
};

struct Bars {
  // ring: full[i], empty[i]; then s_full[2], s_free[2], p_full, o_full, q_full, done
  uint64_t* full;
  uint64_t* empty;
  uint64_t* s_full;
  uint64_t* s_free;
  uint64_t* p_full;
  uint64_t* o_full;
  uint64_t* q_full;
  uint64_t* done;
};

struct ULayout {
  uint32_t q, p, ring, bars, tmem, prefix, total;
};
__host__ __device__ inline ULayout u_layout(int qbytes, int stage, int nst, int num_seqs) {
  ULayout L;
  uint32_t off = 0;
  L.q = off;
  off += qbytes;
  L.p = off;
  off += 2 * kChunk;
  L.ring = off;
  off += (uint32_t)stage * nst;
  L.bars = off;
  off += (uint32_t)(2 * nst + 8) * 8;
  L.tmem = off;
  off += 16;
  L.prefix = off;
  off += (uint32_t)(num_seqs + 1) * 4;
  L.total = off + 1024;  // slack for aligning the base to 1024 bytes
  return L;
}

// Byte offset of 16-byte unit u of row r in a 128-byte-swizzled chunk.
__device__ __forceinline__ uint32_t swz(int r, int u) { return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4)); }

template <int D, int BS>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_umma_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const PrefillParams p) {
  using C = U<D, BS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int NST = p.nstages;
  const int S = p.rows.num_seqs;
  const ULayout L = u_layout(C::QBYTES, C::STAGE, NST, S);
  uint8_t* qs = smem + L.q;
  uint8_t* ps = smem + L.p;
  uint8_t* ring = smem + L.ring;
  uint64_t* bar0 = reinterpret_cast<uint64_t*>(smem + L.bars);
  Bars B{bar0, bar0 + NST, bar0 + 2 * NST, bar0 + 2 * NST + 2, bar0 + 2 * NST + 4, bar0 + 2 * NST + 5,
         bar0 + 2 * NST + 6, bar0 + 2 * NST + 7};
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.tmem);
  int32_t* prefix = reinterpret_cast<int32_t*>(smem + L.prefix);  // units before sequence s
  __shared__ int32_t warp_tot[kThreads / 32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.group, hq = p.num_q_heads, hkv = p.num_kv_heads;
  const int QB = kRows / G;  // query positions per unit

  dev::grid_dep_wait();
  // ---- query blocks per prompt sequence, exclusive prefix ---------------------
  for (int s = tid; s < S; s += kThreads) {
    const int qlen = p.rows.qsl[s + 1] - p.rows.qsl[s];
    prefix[s] = qlen > 1 ? (qlen + QB - 1) / QB : 0;
  }
  __syncthreads();
  {
    const int ipt = (S + kThreads - 1) / kThreads;
    const int lo = min(S, tid * ipt), hi = min(S, lo + ipt);
    int sum = 0;
    for (int i = lo; i < hi; ++i) sum += prefix[i];
    int x = sum;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, x, off);
      if (lane >= off) x += y;
    }
    if (lane == 31) warp_tot[warp] = x;
    __syncthreads();
    int run = x - sum;
    for (int w = 0; w < warp; ++w) run += warp_tot[w];
    for (int i = lo; i < hi; ++i) {
      const int v = prefix[i];
      prefix[i] = run;
      run += v;
    }
    if (tid == kThreads - 1) prefix[S] = run;
  }
  __syncthreads();
  dev::grid_dep_launch();
  const int nunits = prefix[S] * hkv;
  if ((int)blockIdx.x >= nunits) return;  // surplus CTA: nothing allocated yet

  // ---- this CTA's unit: ordinal i / Hkv (a sequence's last query blocks
  // first), kv head i % Hkv ------------------------------------------------------
  int s = 0;
  {
    const int ub = blockIdx.x / hkv;
    int lo = 0, hi = S - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= ub) lo = mid; else hi = mid - 1;
    }
    s = lo;
  }
  const int h = blockIdx.x % hkv;
  const int nqb = prefix[s + 1] - prefix[s];
  const int qb = nqb - 1 - (blockIdx.x / hkv - prefix[s]);
  const int first = p.rows.qsl[s];
  const int qlen = p.rows.qsl[s + 1] - first;
  const int seq_len = p.rows.seq_lens[s];
  const int pos0 = seq_len - qlen;  // position of the sequence's first query row
  const int q0 = qb * QB;           // first query (local index) of the unit
  const int qn = min(QB, qlen - q0);
  const int kend = min(seq_len, pos0 + q0 + qn);  // keys the unit needs: [0, kend)
  int nbneed = (kend + BS - 1) / BS;
  if (nbneed > p.max_blocks) {
    if (tid == 0) atomicCAS(p.err, 0, 3);
    nbneed = p.max_blocks;
  }
  const int ntiles = (nbneed * BS + kKeys - 1) / kKeys;

  if (tid == 0) {
    // one arrival (a TMA transaction or an MMA commit), or one per row warp
    for (int i = 0; i < 2 * NST; ++i) dev::mbar_init(&bar0[i], 1);
    for (int i = 0; i < 2; ++i) {
      dev::mbar_init(&B.s_full[i], 1);
      dev::mbar_init(&B.s_free[i], 4);
    }
    dev::mbar_init(B.p_full, 4);
    dev::mbar_init(B.o_full, 1);
    dev::mbar_init(B.q_full, 4);
    dev::mbar_init(B.done, 1);
    dev::fence_barrier_init();
  }
  if (warp == 1) {
    dev::tmem_alloc(tmem_slot, kTmemCols);
    dev::tmem_relinquish();
  }
  dev::tc_fence_before();
  __syncthreads();
  dev::tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  const uint32_t t_s0 = tbase, t_o = tbase + 2 * kKeys;  // S buffers at columns 0 and 128, O at 256

  if (warp == 0) {
    // ======================= loads: K/V tiles through the block table ========
    const uint64_t pol = dev::policy_evict_last();  // the sequence's other units read the same tiles
    const int32_t oob_row = p.num_blocks * hkv * BS;  // past the pool: TMA fills zeros
    bool ok = true;
    int k = 0;
    for (; k < ntiles && ok; ++k) {
      const int st = k % NST;
      if (k >= NST) ok = __all_sync(0xffffffffu, dev::mbar_wait(&B.empty[st], ((k / NST) - 1) & 1, p.err));
      if (!ok) break;
      int32_t y = oob_row;
      int kv = 0, c = 0, j = 0;
      if (lane < C::BOXES) {
        kv = lane / (C::NCH * C::BPT);
        c = (lane / C::BPT) % C::NCH;
        j = lane % C::BPT;
        const int b = k * C::BPT + j;
        if (b < nbneed) {
          int blk = __ldg(p.block_tables + (int64_t)s * p.max_blocks + b);
          if (blk < 0 || blk >= p.num_blocks) {  // bad table entry: flag, read block 0
            atomicCAS(p.err, 0, 2);
            blk = 0;
          }
          y = (blk * hkv + h) * BS;
        }
      }
      if (lane == 0) dev::mbar_arrive_expect_tx(&B.full[st], (uint32_t)C::STAGE);
      __syncwarp();
      if (lane < C::BOXES) {
        uint8_t* dst = ring + (size_t)st * C::STAGE + kv * C::KVT + c * kChunk + j * BS * 128;
        dev::tma_load_2d(dst, kv ? &tm_v : &tm_k, c * 64, y, &B.full[st], pol);
      }
    }
    // drain: the last stages issued must land before this CTA may exit
    if (lane == 0) {
      for (int d = max(0, k - NST); d < k; ++d)
        dev::mbar_wait(&B.full[d % NST], (uint32_t)((d / NST) & 1), nullptr, 100000000ull);
    }
  } else if (warp == 1) {
    // ======================= MMA issue (one thread) ===========================
    if (lane == 0) {
      const uint32_t idesc_s = dev::umma_idesc_bf16(kKeys, false);
      const uint32_t idesc_o = dev::umma_idesc_bf16(D, true);
      const uint32_t q_u32 = dev::smem_u32(qs), p_u32 = dev::smem_u32(ps), ring_u32 = dev::smem_u32(ring);
      auto issue_s = [&](int k) {  // S[k & 1] = Q K_k^T
        const uint32_t kb = ring_u32 + (uint32_t)((k % NST) * C::STAGE);
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS_S; ++ks) {
          const uint32_t off = (uint32_t)((ks >> 2) * kChunk + (ks & 3) * 32);
          dev::umma_ss(t_s0 + (uint32_t)((k & 1) * kKeys), dev::umma_desc_sw128(q_u32 + off, 16, 1024),
                       dev::umma_desc_sw128(kb + off, 16, 1024), idesc_s, ks > 0 ? 1u : 0u);
        }
        dev::umma_commit(&B.s_full[k & 1]);
      };
      bool ok = dev::mbar_wait(B.q_full, 0, p.err);
      if (ok && ntiles > 0) {
        ok = dev::mbar_wait(&B.full[0], 0, p.err);
        if (ok) {
          dev::tc_fence_after();
          issue_s(0);
        }
      }
      for (int k = 0; k < ntiles && ok; ++k) {
        if (k + 1 < ntiles) {
          ok = dev::mbar_wait(&B.full[(k + 1) % NST], (uint32_t)(((k + 1) / NST) & 1), p.err);
          if (ok && k + 1 >= 2) ok = dev::mbar_wait(&B.s_free[(k + 1) & 1], (uint32_t)((((k + 1) >> 1) - 1) & 1), p.err);
          if (!ok) break;
          dev::tc_fence_after();
          issue_s(k + 1);
        }
        ok = dev::mbar_wait(B.p_full, (uint32_t)(k & 1), p.err);
        if (!ok) break;
        dev::tc_fence_after();
        const uint32_t vb = ring_u32 + (uint32_t)((k % NST) * C::STAGE + C::KVT);
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS_O; ++ks) {
          // A = P (K-major, 16 keys per step); B = V (MN-major: d contiguous,
          // 64-wide chunks kChunk apart, 8-key row groups 1024 bytes apart)
          const uint32_t aoff = (uint32_t)((ks >> 2) * kChunk + (ks & 3) * 32);
          dev::umma_ss(t_o, dev::umma_desc_sw128(p_u32 + aoff, 16, 1024),
                       dev::umma_desc_sw128(vb + (uint32_t)(ks * 16 * 128), kChunk, 1024), idesc_o,
                       (k > 0 || ks > 0) ? 1u : 0u);
        }
        dev::umma_commit(B.o_full);
        dev::umma_commit(&B.empty[k % NST]);
      }
      // every MMA issued above has completed before TMEM may be freed
      dev::umma_commit(B.done);
      dev::mbar_wait(B.done, 0, nullptr, 100000000ull);
    }
    __syncwarp();
  } else {
    // ======================= rows: softmax, P, output =========================
    const int quarter = warp & 3;
    const int r = 32 * quarter + lane;  // this thread's row (its TMEM lane)
    const uint32_t lane_addr = (uint32_t)(32 * quarter) << 16;
    const bool valid = r < qn * G;
    const int pos = pos0 + q0 + r / G;  // the row's position: keys <= pos
    const int64_t grow = ((int64_t)(first + q0 + r / G) * hq + (int64_t)h * G + r % G) * D;
    // ---- Q row into the swizzled Q tile (zero for rows past the unit) ----
    {
      const uint4* src = reinterpret_cast<const uint4*>(p.q + grow * 2);
#pragma unroll
      for (int c = 0; c < C::NCH; ++c) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const uint4 v = valid ? __ldg(src + c * 8 + u) : make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(qs + c * kChunk + swz(r, u)) = v;
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(B.q_full);
    }
    float ref = -1e30f, lsum = 0.f;
    bool ok = true;
    for (int k = 0; k < ntiles && ok; ++k) {
      ok = __all_sync(0xffffffffu, dev::mbar_wait(&B.s_full[k & 1], (uint32_t)((k >> 1) & 1), p.err));
      if (!ok) break;
      dev::tc_fence_after();
      float sv[kKeys];
#pragma unroll
      for (int c = 0; c < kKeys / 32; ++c) {
        uint32_t w[32];
        dev::tmem_ld32(t_s0 + (uint32_t)((k & 1) * kKeys + 32 * c) + lane_addr, w);
#pragma unroll
        for (int i = 0; i < 32; ++i) sv[32 * c + i] = __uint_as_float(w[i]);
      }
      dev::tc_fence_before();
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&B.s_free[k & 1]);
      // mask and scale; the row's max over this tile
      const int key0 = k * kKeys;
      const int lim = min(pos + 1, seq_len) - key0;  // keys [key0, key0 + lim) are visible
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < kKeys; ++i) {
        sv[i] = (valid && i < lim) ? sv[i] * p.scale_log2 : -INFINITY;
        mx = fmaxf(mx, sv[i]);
      }
      // the previous PV MMA has finished: P may be rewritten, O is stable
      if (k > 0) {
        ok = __all_sync(0xffffffffu, dev::mbar_wait(B.o_full, (uint32_t)((k - 1) & 1), p.err));
        if (!ok) break;
        dev::tc_fence_after();
      }
      const bool move = mx > ref + kRefSlack;
      const float alpha = move ? dev::ex2(ref - mx) : 1.f;
      if (k > 0 && __any_sync(0xffffffffu, move)) {
        // rescale this row of O in TMEM (rows that keep their reference use 1)
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t w[32];
          const uint32_t ta = t_o + (uint32_t)(32 * c) + lane_addr;
          dev::tmem_ld32(ta, w);
#pragma unroll
          for (int i = 0; i < 32; ++i) w[i] = __float_as_uint(__uint_as_float(w[i]) * alpha);
          dev::tmem_st32(ta, w);
        }
      }
      if (move) {
        lsum *= alpha;
        ref = mx;
      }
      // P = 2^(s - ref) as bf16 into the swizzled P tile; the running sum
      float ps_row = 0.f;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          uint32_t pk[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float a = dev::ex2(sv[64 * c + 8 * u + 2 * e] - ref);
            const float b = dev::ex2(sv[64 * c + 8 * u + 2 * e + 1] - ref);
            ps_row += a + b;
            pk[e] = dev::pack_bf16(a, b);
          }
          *reinterpret_cast<uint4*>(ps + c * kChunk + swz(r, u)) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
      lsum += ps_row;
      // the tile holding the context's end: slots past it hold stale pool
      // bytes (masked scores, but 0 * NaN would poison P V): zero their V rows
      const int stale0 = seq_len - key0, stale1 = min(kKeys, nbneed * BS - key0);
      if (stale0 < stale1) {
        uint8_t* vt = ring + (size_t)(k % NST) * C::STAGE + C::KVT;
        const int units = (stale1 - stale0) * C::NCH * 8;
        for (int i = tid - 64; i < units; i += 128) {
          const int key = stale0 + i / (C::NCH * 8), rest = i % (C::NCH * 8);
          *reinterpret_cast<uint4*>(vt + (rest >> 3) * kChunk + key * 128 + (rest & 7) * 16) = make_uint4(0, 0, 0, 0);
        }
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      dev::tc_fence_before();
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(B.p_full);
    }
    // ---- O / sum -> output row ----
    if (ok && ntiles > 0) {
      ok = __all_sync(0xffffffffu, dev::mbar_wait(B.o_full, (uint32_t)((ntiles - 1) & 1), p.err));
      if (ok) {
        dev::tc_fence_after();
        const float inv = valid ? 1.f / lsum : 0.f;
        uint4* dst = reinterpret_cast<uint4*>(p.out + grow * 2);
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t w[32];
          dev::tmem_ld32(t_o + (uint32_t)(32 * c) + lane_addr, w);
          if (valid) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint32_t pk[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                pk[e] = dev::pack_bf16(__uint_as_float(w[8 * u + 2 * e]) * inv,
                                       __uint_as_float(w[8 * u + 2 * e + 1]) * inv);
              dst[4 * c + u] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
          }
        }
      }
    }
  }

  // ---- free TMEM once every warp is past its last tcgen05 access ----
  dev::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    dev::tc_fence_after();
    dev::tmem_dealloc(tbase, kTmemCols);
  }
}

template <int D, int BS>
cudaError_t launch_u(const PrefillParams& p, const CUtensorMap& tm_k, const CUtensorMap& tm_v, int grid,
                     cudaStream_t stream) {
  using C = U<D, BS>;
  const ULayout L = u_layout(C::QBYTES, C::STAGE, p.nstages, p.rows.num_seqs);
  auto kern = prefill_umma_kernel<D, BS>;
  static int set_for[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || set_for[dev] < (int)L.total) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
    if (e != cudaSuccess) return e;
    if (dev < 64) set_for[dev] = (int)L.total;
  }
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tm_k, tm_v, p);
}

}  // namespace

bool prefill_umma_supported(int kv, int q, int head_dim, int block_size, int group) {
  return kv == kBF16 && q == kBF16 && (head_dim == 64 || head_dim == 128) && (block_size == 16 || block_size == 32) &&
         group >= 1 && group <= 32 && (kRows % group) == 0;
}

cudaError_t launch_prefill_umma(const PrefillParams& p_in, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                int head_dim, int block_size, int num_tokens, cudaStream_t stream) {
  PrefillParams p = p_in;
  const int nch = head_dim / 64;
  const int qbytes = nch * kChunk, stage = 2 * nch * kChunk;
  const int fixed = (int)u_layout(qbytes, stage, 0, p.rows.num_seqs).total;
  int nst = (kSmemOptIn - fixed) / (stage + 16);
  if (nst > 4) nst = 4;
  if (nst < 2) return cudaErrorNotSupported;  // too many sequences for the unit table: caller falls back
  p.nstages = nst;
  const int qb = kRows / p.group;
  const int64_t grid = ((int64_t)num_tokens / qb + p.rows.num_seqs) * p.num_kv_heads;
  if (grid <= 0) return cudaSuccess;
  if (grid > INT32_MAX) return cudaErrorNotSupported;
  if (head_dim == 128 && block_size == 16) return launch_u<128, 16>(p, tm_k, tm_v, (int)grid, stream);
  if (head_dim == 128 && block_size == 32) return launch_u<128, 32>(p, tm_k, tm_v, (int)grid, stream);
  if (head_dim == 64 && block_size == 16) return launch_u<64, 16>(p, tm_k, tm_v, (int)grid, stream);
  if (head_dim == 64 && block_size == 32) return launch_u<64, 32>(p, tm_k, tm_v, (int)grid, stream);
  return cudaErrorNotSupported;
}

}  // namespace pa
