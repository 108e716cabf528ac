// Prompt rows of a mixed chunked-prefill + decode step, tensor-core path
// (bf16 queries over a bf16 pool).
//
// What it computes: every query row of a sequence that adds a chunk of prompt
// tokens this step attends, causally, the sequence's keys up to its own
// position, gathered block by block through the block table ("vLLM innenfra:
// slik gjør paged attention GPU-minnet til blokker på 16 tokens", the step()
// list: a step schedules decode and chunked prefill together; the chunk's K/V
// are already in the pool).
//
// How: the work unit is (sequence, kv head, block of query positions).  The
// GQA group's query heads of each position are packed into the MMA's M rows
// (rows = positions x group), so the unit's 64 rows share every K/V tile: a
// dense contraction.  One producer warp streams the unit's K/V tiles with TMA
// (2-D tensor-map boxes of [block][128 B], 128-byte swizzle) into a ring of
// shared-memory stages; four warps each own 16 rows and, per tile, compute
// S = Q K^T (mma.sync m16n8k16, bf16 in, fp32 out), apply the causal and
// length mask, update an online softmax per row, and accumulate O += P V with
// P taken straight from the S registers.  Within a sequence, its last query
// blocks (the ones with the most keys) take the lowest CTA indices.
#include <cuda_runtime.h>

#include "pa_device.cuh"
#include "pa_kernels.h"

namespace pa {
namespace {

constexpr int kComputeWarps = 4;
constexpr int kThreads = (kComputeWarps + 1) * 32;
constexpr int kRows = kComputeWarps * 16;  // query rows (positions x group) per unit
constexpr int kMaxStages = 16;
constexpr int kSmemPerSM = 233472;
constexpr int kCtasPerSM = 2;

template <int D, int BS>
struct PCfg {
  static constexpr int ROW = D * 2;
  static constexpr int TILE = BS * ROW;
  static constexpr int STAGE = 2 * TILE;
  static constexpr int NCH = ROW / 128;
  static constexpr int KSTEPS = D / 16;  // k-steps of S = Q K^T
  static constexpr int NK = BS / 8;      // 8-key n-tiles of S per tile
  static constexpr int ND = D / 8;       // 8-wide d n-tiles of O
  static_assert(ROW % 128 == 0 && BS % 16 == 0, "shape");
};

struct PLayout {
  uint32_t ring, bars, prefix, total;
};
__host__ __device__ inline PLayout p_layout(int stage, int nst, int num_seqs) {
  PLayout L;
  uint32_t off = 0;
  L.ring = off;
  off += (uint32_t)stage * nst;
  L.bars = off;
  off += (uint32_t)nst * 16;
  L.prefix = off;
  off += (uint32_t)(num_seqs + 1) * 4;
  L.total = off + 1024;
  return L;
}

template <int D, int BS>
__global__ void __launch_bounds__(kThreads, kCtasPerSM)
    prefill_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                      const PrefillParams p) {
  using C = PCfg<D, BS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int NST = p.nstages;
  const int S = p.rows.num_seqs;
  const PLayout L = p_layout(C::STAGE, NST, S);
  uint8_t* ring = smem + L.ring;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + NST;
  int32_t* prefix = reinterpret_cast<int32_t*>(smem + L.prefix);  // query blocks before sequence s
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
  if (tid == 0) {
    for (int i = 0; i < NST; ++i) {
      dev::mbar_init(&full[i], 1);
      dev::mbar_init(&empty[i], kComputeWarps);
    }
    dev::fence_barrier_init();
  }
  __syncthreads();
  dev::grid_dep_launch();

  // ---- this CTA's unit: CTA i takes query-block ordinal i / Hkv, kv head i % Hkv
  const int nunits = prefix[S] * hkv;
  if ((int)blockIdx.x >= nunits) return;
  int s = 0;
  {
    // the ordinal's sequence: the last s with prefix[s] <= ordinal (a
    // sequence's blocks are contiguous; sequences with none are skipped)
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
  const int qb = nqb - 1 - (blockIdx.x / hkv - prefix[s]);  // last blocks of each sequence first
  const int first = p.rows.qsl[s];
  const int qlen = p.rows.qsl[s + 1] - first;
  const int seq_len = p.rows.seq_lens[s];
  const int pos0 = seq_len - qlen;  // position of the sequence's first query row
  const int q0 = qb * QB;           // first query (local index) of the unit
  const int qn = min(QB, qlen - q0);
  // keys needed: 0 .. pos0 + q0 + qn - 1
  const int kend = min(seq_len, pos0 + q0 + qn);
  int ntiles = (kend + BS - 1) / BS;
  if (ntiles > p.max_blocks) {
    if (tid == 0) atomicCAS(p.err, 0, 3);
    ntiles = p.max_blocks;
  }

  if (warp == kComputeWarps) {
    // ======================= producer: K/V tiles through the table ===========
    const uint64_t pol = dev::policy_evict_first();
    bool ok = true;
    int stage = 0;
    uint32_t phase = 0;
    for (int base = 0; base < ntiles && ok; base += 32) {
      int blk = 0;
      if (base + lane < ntiles) {
        blk = __ldg(p.block_tables + (int64_t)s * p.max_blocks + base + lane);
        if (blk < 0 || blk >= p.num_blocks) {
          atomicCAS(p.err, 0, 2);
          blk = 0;
        }
      }
      const int cnt = min(32, ntiles - base);
      for (int j = 0; j < cnt && ok; ++j) {
        const int blkj = __shfl_sync(0xffffffffu, blk, j);
        const int k = base + j;
        if (k >= NST) ok = __all_sync(0xffffffffu, dev::mbar_wait(&empty[stage], (phase - 1) & 1, p.err));
        if (!ok) break;
        uint8_t* st = ring + (size_t)stage * C::STAGE;
        if (lane == 0) dev::mbar_arrive_expect_tx(&full[stage], (uint32_t)C::STAGE);
        __syncwarp();
        const int32_t krow = (blkj * hkv + h) * BS;
        if (lane < C::NCH)
          dev::tma_load_2d(st + lane * BS * 128, &tm_k, lane * 64, krow, &full[stage], pol);
        else if (lane < 2 * C::NCH)
          dev::tma_load_2d(st + C::TILE + (lane - C::NCH) * BS * 128, &tm_v, (lane - C::NCH) * 64, krow,
                           &full[stage], pol);
        if (++stage == NST) {
          stage = 0;
          ++phase;
        }
      }
    }
    return;
  }

  // ======================= compute warps: 16 rows each ===========================
  const int g = lane >> 2, tq = lane & 3;
  const int lr = lane & 7, li = lane >> 3;
  const uint32_t ring_u32 = dev::smem_u32(ring);
  // rows of this thread: r0 = 16 * warp + g, r1 = r0 + 8; row r is query
  // (local) q0 + r / G, head h * G + r % G
  const int r0 = 16 * warp + g, r1 = r0 + 8;
  const int qa = q0 + r0 / G, qc = q0 + r1 / G;  // local query indices
  const bool va = (r0 / G) < qn, vc = (r1 / G) < qn;
  const int pa_ = pos0 + qa, pc = pos0 + qc;  // positions (keys allowed up to and including)
  const uint16_t* qbase = reinterpret_cast<const uint16_t*>(p.q);
  const int64_t rowa = ((int64_t)(first + qa) * hq + (int64_t)h * G + r0 % G) * D;
  const int64_t rowc = ((int64_t)(first + qc) * hq + (int64_t)h * G + r1 % G) * D;
  // ---- Q A-fragments: a0a1 (row g, k 2t..), a2a3 (row g+8), a4a5 (row g, k 2t+8..), a6a7 ----
  uint32_t qf[C::KSTEPS][4];
#pragma unroll
  for (int kk = 0; kk < C::KSTEPS; ++kk) {
    const int d = 16 * kk + 2 * tq;
    qf[kk][0] = va ? __ldg(reinterpret_cast<const uint32_t*>(qbase + rowa + d)) : 0u;
    qf[kk][1] = vc ? __ldg(reinterpret_cast<const uint32_t*>(qbase + rowc + d)) : 0u;
    qf[kk][2] = va ? __ldg(reinterpret_cast<const uint32_t*>(qbase + rowa + d + 8)) : 0u;
    qf[kk][3] = vc ? __ldg(reinterpret_cast<const uint32_t*>(qbase + rowc + d + 8)) : 0u;
  }
  float ma = -1e30f, mc = -1e30f, la = 0.f, lc = 0.f;
  float o[C::ND][4];
#pragma unroll
  for (int i = 0; i < C::ND; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
  // the last key any row of this warp may see
  const int wlast = min(kend - 1, pos0 + q0 + min(qn, (16 * warp + 15) / G + 1) - 1);

  bool ok = true;
  int stage = 0;
  uint32_t phase = 0;
  for (int k = 0; k < ntiles && ok; ++k) {
    ok = __all_sync(0xffffffffu, dev::mbar_wait(&full[stage], phase & 1, p.err));
    if (!ok) break;
    const int key0 = k * BS;
    if (key0 <= wlast) {  // tiles wholly past this warp's rows are skipped
      const uint32_t kbase = ring_u32 + stage * C::STAGE;
      const uint32_t vbase = kbase + C::TILE;
      if (seq_len - key0 < BS) {
        // stale bytes past the context: zero their V rows (masked scores
        // would still give 0 * NaN); every warp reads this tile, so the
        // first warp to get here is not enough -- each zeroes, idempotently
        const int valid = seq_len - key0;
        uint8_t* vt = ring + (size_t)stage * C::STAGE + C::TILE;
        for (int i = lane; i < (BS - valid) * C::NCH * 8; i += 32) {
          const int key = valid + i / (C::NCH * 8), rest = i % (C::NCH * 8);
          *reinterpret_cast<uint4*>(vt + (rest >> 3) * (BS * 128) + key * 128 + (rest & 7) * 16) =
              make_uint4(0, 0, 0, 0);
        }
        // order these generic-proxy writes before the TMA refill of the stage
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
      }
      // ---- S = Q K^T: 16 rows x BS keys ----
      float sc[C::NK][4];
#pragma unroll
      for (int n = 0; n < C::NK; ++n) sc[n][0] = sc[n][1] = sc[n][2] = sc[n][3] = 0.f;
#pragma unroll
      for (int kk = 0; kk < C::KSTEPS; ++kk) {
#pragma unroll
        for (int n2 = 0; n2 < C::NK / 2; ++n2) {
          // matrices: (keys 16n2+0..7, chunk 2kk), (keys 16n2+0..7, chunk
          // 2kk+1), (keys 16n2+8..15, chunk 2kk), (keys 16n2+8..15, chunk 2kk+1)
          const int key = 16 * n2 + (li >> 1) * 8 + lr;
          const int gu = 2 * kk + (li & 1);
          const uint32_t addr = kbase + (gu >> 3) * (BS * 128) + key * 128 + (((gu & 7) ^ (key & 7)) << 4);
          uint32_t b0, b1, b2, b3;
          dev::ldsm_x4(addr, b0, b1, b2, b3);
          dev::mma_bf16(sc[2 * n2], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
          dev::mma_bf16(sc[2 * n2 + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
        }
      }
      // ---- mask (causal and context length), online softmax per row ----
      float mxa = -INFINITY, mxc = -INFINITY;
#pragma unroll
      for (int n = 0; n < C::NK; ++n) {
        const int kc = key0 + 8 * n + 2 * tq;
        sc[n][0] = (va && kc <= pa_ && kc < seq_len) ? sc[n][0] * p.scale_log2 : -INFINITY;
        sc[n][1] = (va && kc + 1 <= pa_ && kc + 1 < seq_len) ? sc[n][1] * p.scale_log2 : -INFINITY;
        sc[n][2] = (vc && kc <= pc && kc < seq_len) ? sc[n][2] * p.scale_log2 : -INFINITY;
        sc[n][3] = (vc && kc + 1 <= pc && kc + 1 < seq_len) ? sc[n][3] * p.scale_log2 : -INFINITY;
        mxa = fmaxf(mxa, fmaxf(sc[n][0], sc[n][1]));
        mxc = fmaxf(mxc, fmaxf(sc[n][2], sc[n][3]));
      }
#pragma unroll
      for (int off = 1; off < 4; off <<= 1) {
        mxa = fmaxf(mxa, __shfl_xor_sync(0xffffffffu, mxa, off));
        mxc = fmaxf(mxc, __shfl_xor_sync(0xffffffffu, mxc, off));
      }
      const float mna = fmaxf(ma, mxa), mnc = fmaxf(mc, mxc);
      const float ala = dev::ex2(ma - mna), alc = dev::ex2(mc - mnc);
      ma = mna;
      mc = mnc;
      float psa = 0.f, psc = 0.f;
      uint32_t pf[C::NK][2];  // P as bf16 pairs: [n][0] row g, [n][1] row g+8
#pragma unroll
      for (int n = 0; n < C::NK; ++n) {
        const float p0 = dev::ex2(sc[n][0] - mna), p1 = dev::ex2(sc[n][1] - mna);
        const float p2 = dev::ex2(sc[n][2] - mnc), p3 = dev::ex2(sc[n][3] - mnc);
        psa += p0 + p1;
        psc += p2 + p3;
        pf[n][0] = dev::pack_bf16(p0, p1);
        pf[n][1] = dev::pack_bf16(p2, p3);
      }
      la = la * ala + psa;
      lc = lc * alc + psc;
#pragma unroll
      for (int i = 0; i < C::ND; ++i) {
        o[i][0] *= ala;
        o[i][1] *= ala;
        o[i][2] *= alc;
        o[i][3] *= alc;
      }
      // ---- O += P V: P is the A operand (keys 16j..16j+15 per k-step) ----
#pragma unroll
      for (int j = 0; j < C::NK / 2; ++j) {
        const uint32_t a0 = pf[2 * j][0], a1 = pf[2 * j][1], a2 = pf[2 * j + 1][0], a3 = pf[2 * j + 1][1];
#pragma unroll
        for (int nd = 0; nd < C::ND; nd += 2) {
          // matrices: (keys 16j+0..7, d chunk nd), (keys 16j+8..15, chunk nd),
          // (keys 16j+0..7, chunk nd+1), (keys 16j+8..15, chunk nd+1); .trans
          const int key = 16 * j + (li & 1) * 8 + lr;
          const int gu = nd + (li >> 1);
          const uint32_t addr = vbase + (gu >> 3) * (BS * 128) + key * 128 + (((gu & 7) ^ (key & 7)) << 4);
          uint32_t b0, b1, b2, b3;
          dev::ldsm_x4_t(addr, b0, b1, b2, b3);
          dev::mma_bf16(o[nd], a0, a1, a2, a3, b0, b1);
          dev::mma_bf16(o[nd + 1], a0, a1, a2, a3, b2, b3);
        }
      }
    }
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(&empty[stage]);
    if (++stage == NST) {
      stage = 0;
      ++phase;
    }
  }
  if (!ok) return;
  // ---- normalise and write: thread holds rows g, g+8, d = 8 nd + 2t, +1 ----
#pragma unroll
  for (int off = 1; off < 4; off <<= 1) {
    la += __shfl_xor_sync(0xffffffffu, la, off);
    lc += __shfl_xor_sync(0xffffffffu, lc, off);
  }
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
  const float ia = 1.f / la, ic = 1.f / lc;
#pragma unroll
  for (int nd = 0; nd < C::ND; ++nd) {
    const int d = 8 * nd + 2 * tq;
    if (va)
      *reinterpret_cast<__nv_bfloat162*>(out + rowa + d) = __floats2bfloat162_rn(o[nd][0] * ia, o[nd][1] * ia);
    if (vc)
      *reinterpret_cast<__nv_bfloat162*>(out + rowc + d) = __floats2bfloat162_rn(o[nd][2] * ic, o[nd][3] * ic);
  }
}

template <int D, int BS>
cudaError_t launch_p(const PrefillParams& p, const CUtensorMap& tm_k, const CUtensorMap& tm_v, int grid,
                     cudaStream_t stream) {
  using C = PCfg<D, BS>;
  const PLayout L = p_layout(C::STAGE, p.nstages, p.rows.num_seqs);
  auto kern = prefill_tc_kernel<D, BS>;
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

bool prefill_tc_supported(int kv, int q, int head_dim, int block_size, int group) {
  return kv == kBF16 && q == kBF16 && (head_dim == 64 || head_dim == 128) && (block_size == 16 || block_size == 32) &&
         group >= 1 && group <= 16 && (kRows % group) == 0;
}

cudaError_t launch_prefill_tc(const PrefillParams& p_in, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                              int head_dim, int block_size, int num_tokens, cudaStream_t stream) {
  PrefillParams p = p_in;
  const int stage = 2 * block_size * head_dim * 2;
  const int budget = kSmemPerSM / kCtasPerSM - 1024 - 64;
  const int fixed = (int)p_layout(stage, 0, p.rows.num_seqs).total;
  int nst = (budget - fixed) / (stage + 16);
  if (nst > kMaxStages) nst = kMaxStages;
  if (nst < 2) return cudaErrorNotSupported;
  p.nstages = nst;
  const int qb = kRows / p.group;
  // units are at most one per (query block, kv head): an upper bound the
  // kernel trims (surplus CTAs exit at once)
  const int64_t grid = ((int64_t)num_tokens / qb + p.rows.num_seqs) * p.num_kv_heads;
  if (grid <= 0) return cudaSuccess;
  if (grid > INT32_MAX) return cudaErrorNotSupported;
  if (head_dim == 128 && block_size == 16) return launch_p<128, 16>(p, tm_k, tm_v, (int)grid, stream);
  if (head_dim == 128 && block_size == 32) return launch_p<128, 32>(p, tm_k, tm_v, (int)grid, stream);
  if (head_dim == 64 && block_size == 16) return launch_p<64, 16>(p, tm_k, tm_v, (int)grid, stream);
  if (head_dim == 64 && block_size == 32) return launch_p<64, 32>(p, tm_k, tm_v, (int)grid, stream);
  return cudaErrorNotSupported;
}

}  // namespace pa
