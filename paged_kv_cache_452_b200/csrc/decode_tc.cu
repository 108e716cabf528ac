// pa_decode, tensor-core path (bf16 or e4m3 cache, bf16 queries, GQA group
// 2..8): paged attention for one decode step.
//
// What it computes: for every decode sequence and query head, softmax
// attention of its one query row over the sequence's keys, gathered block by
// block through the block table ("PagedAttention：KV cache 即虚拟内存（block
// manager & 碎片）", 直接答案: paging only changes where the keys live, not the
// result).
//
// How, on sm_100a:
//  * Work = (sequence, kv head, block) tiles.  The tiles of the whole batch
//    are laid end to end and cut into one equal, contiguous range per CTA
//    (persistent grid, 2 CTAs per SM), so a long context is split over
//    several CTAs (split-K over blocks) and every SM streams the same number
//    of bytes whatever the length mix.  A range cut inside a sequence leaves
//    a partial (max, sum, unnormalised output) that a second kernel merges
//    with a log-sum-exp combine; uncut sequences are finished in place.
//  * One producer warp gathers tiles through the block table with TMA: the
//    K tile (and the bf16 V tile) as 2-D tensor-map boxes of [block][128 B]
//    with 128-byte swizzle, the e4m3 V tile (d-major, contiguous) as one bulk
//    copy, into a ring of shared-memory stages guarded by mbarriers.  The
//    query rows of each (sequence, kv head) come in by bulk copy too.
//  * Four consumer warps take tiles round-robin.  GQA groups are packed with
//    keys on the MMA's M side and the group's query rows on N (8, padded):
//    S^T = K Q^T and O^T += V^T P^T with mma.sync m16n8k16 (fp32 accumulate),
//    an online softmax per query column, and P^T moved into the B operand
//    with movmatrix.  e4m3 K/V become f16 exactly (bit placement, see
//    pa_device.cuh), and the 2^8 factor plus the per-tensor scales are folded
//    into the softmax scale and the output scale.
//  * At the end of a sequence's range the four warps' states are merged in
//    shared memory.
#include <cuda_runtime.h>

#include "pa_device.cuh"
#include "pa_kernels.h"

namespace pa {
namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kGPad = 8;          // query rows per MMA N tile
constexpr int kMergeStride = 4;   // padding of the merge buffer rows (floats)
constexpr int kMaxStages = 32;
constexpr int kSmemPerSM = 233472;  // B200: 228 KB per SM
constexpr int kCtasPerSM = 2;

template <int KV, int D, int BS>
struct Cfg {
  static constexpr bool FP8 = KV == kFP8;
  static constexpr int ELEM = FP8 ? 1 : 2;
  static constexpr int ROW = D * ELEM;   // bytes per token row
  static constexpr int TILE = BS * ROW;  // bytes of one K (or V) tile
  static constexpr int STAGE = 2 * TILE;
  static constexpr int NCH = ROW / 128;  // 128-byte chunks per K/V row
  static constexpr int KM = BS / 16;     // 16-key m-tiles per tile
  static constexpr int DM = D / 16;      // 16-d m-tiles of O^T
  static constexpr int QROW = D * 2;     // bytes per bf16 query row
  static constexpr int KSTEPS = D / 16;  // k-steps of S^T = K Q^T
  static_assert(ROW % 128 == 0, "rows must be whole 128-byte swizzle rows");
  static_assert(BS % 16 == 0, "block size must be a multiple of 16");
};

struct SmemLayout {
  uint32_t ring, qbuf, merge_o, merge_ml, bars, prefix, total;
};

__host__ __device__ inline SmemLayout smem_layout(int stage_bytes, int qrow_bytes, int d, int nstages,
                                                  int num_seqs) {
  SmemLayout L;
  uint32_t off = 0;
  L.ring = off;
  off += (uint32_t)stage_bytes * nstages;
  L.qbuf = off;
  off += 2u * kGPad * qrow_bytes;
  L.merge_o = off;
  off += (uint32_t)kConsumerWarps * kGPad * (d + kMergeStride) * 4;
  L.merge_ml = off;
  off += (uint32_t)kConsumerWarps * kGPad * 2 * 4;
  L.bars = off;
  off += (uint32_t)(2 * nstages + 4) * 8;
  L.prefix = off;
  off += (uint32_t)(num_seqs + 1) * 4;
  L.total = off + 1024;  // slack for aligning the base to 1024 bytes
  return L;
}

// Largest s in [0, S) with hkv * prefix[s] <= t (that sequence has tiles).
__device__ __forceinline__ int find_seq(const int32_t* prefix, int S, int hkv, int64_t t) {
  int lo = 0, hi = S - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if ((int64_t)hkv * prefix[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ int64_t range_start(int64_t c, int64_t T, int64_t P) { return c * T / P; }
__device__ __forceinline__ int64_t cta_of(int64_t x, int64_t T, int64_t P) { return ((x + 1) * P - 1) / T; }

template <int KV, int D, int BS>
__global__ void __launch_bounds__(kThreads, kCtasPerSM)
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const DecodeParams p) {
  using C = Cfg<KV, D, BS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int NST = p.nstages;
  const int S = p.rows.num_seqs;
  const SmemLayout L = smem_layout(C::STAGE, C::QROW, D, NST, S);
  uint8_t* ring = smem + L.ring;
  uint8_t* qbuf = smem + L.qbuf;
  float* merge_o = reinterpret_cast<float*>(smem + L.merge_o);
  float* merge_ml = reinterpret_cast<float*>(smem + L.merge_ml);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* empty = full + NST;
  uint64_t* qfull = empty + NST;
  uint64_t* qempty = qfull + 2;
  int32_t* prefix = reinterpret_cast<int32_t*>(smem + L.prefix);
  __shared__ int32_t warp_tot[kThreads / 32];
  __shared__ int abort_flag;

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int hkv = p.num_kv_heads, G = p.group, hq = p.num_q_heads;

  // Everything read below may have been produced by the previous kernel in
  // the stream (programmatic dependent launch lets this grid start early).
  dev::grid_dep_wait();

  // ---- blocks per sequence, exclusive prefix over the batch ----------------
  for (int s = tid; s < S; s += kThreads) {
    const int len = p.rows.seq_lens[s];
    const int qlen = p.rows.qsl ? p.rows.qsl[s + 1] - p.rows.qsl[s] : 1;
    int nb = (qlen == 1 && len > 0) ? (len + BS - 1) / BS : 0;
    if (nb > p.max_blocks) {  // context longer than its table row: flag, clamp
      atomicCAS(p.ws.err, 0, 3);
      nb = p.max_blocks;
    }
    prefix[s] = nb;
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
    abort_flag = 0;
    for (int i = 0; i < NST; ++i) {
      dev::mbar_init(&full[i], 1);
      dev::mbar_init(&empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      dev::mbar_init(&qfull[i], 1);
      dev::mbar_init(&qempty[i], kConsumerWarps);
    }
    dev::fence_barrier_init();
  }
  // query rows >= G stay zero (the bulk copy fills rows 0..G-1 only)
  for (int i = tid; i < 2 * kGPad * C::QROW / 16; i += kThreads) {
    const int row = (i * 16 / C::QROW) % kGPad;
    if (row >= G) reinterpret_cast<uint4*>(qbuf)[i] = make_uint4(0, 0, 0, 0);
  }
  __syncthreads();

  const int64_t T = (int64_t)hkv * prefix[S];
  const int64_t P = gridDim.x;
  const int64_t cta = blockIdx.x;
  const int64_t t0 = range_start(cta, T, P), t1 = range_start(cta + 1, T, P);
  if (cta == 0)
    for (int i = tid; i <= S; i += kThreads) p.ws.prefix[i] = prefix[i];
  dev::grid_dep_launch();
  if (t0 >= t1) return;

  if (warp == kConsumerWarps) {
    // ===================== producer warp: gather through the table ==========
    if (lane == 0) {
      dev::prefetch_tmap(&tm_k);
      if (!C::FP8) dev::prefetch_tmap(&tm_v);
    }
    const uint64_t pol = dev::policy_evict_first();
    const int nblocks = p.max_blocks;
    int seg_count = 0;
    bool ok = true;
    int64_t issued = 0;
    for (int64_t base = t0; base < t1 && ok; base += 32) {
      const int64_t t = base + lane;
      int s = 0, h = 0, blk = 0, row = 0, seg_start = 0;
      if (t < t1) {
        s = find_seq(prefix, S, hkv, t);
        const int nb = prefix[s + 1] - prefix[s];
        const int64_t local = t - (int64_t)hkv * prefix[s];
        h = (int)(local / nb);
        const int i = (int)(local - (int64_t)h * nb);
        blk = __ldg(p.block_tables + (int64_t)s * nblocks + i);
        seg_start = (i == 0) || (t == t0);
        if (seg_start) row = p.rows.qsl ? __ldg(p.rows.qsl + s) : s;
      }
      const int cnt = (int)(t1 - base < 32 ? t1 - base : 32);
      for (int j = 0; j < cnt; ++j) {
        const int hj = __shfl_sync(0xffffffffu, h, j);
        int blkj = __shfl_sync(0xffffffffu, blk, j);
        const int rowj = __shfl_sync(0xffffffffu, row, j);
        const int ssj = __shfl_sync(0xffffffffu, seg_start, j);
        if (lane == 0 && ok) {
          if (blkj < 0 || blkj >= p.num_blocks) {  // bad table entry: flag, read block 0
            atomicCAS(p.ws.err, 0, 2);
            blkj = 0;
          }
          if (ssj) {
            const int qb = seg_count & 1;
            if (seg_count >= 2) ok = dev::mbar_wait(&qempty[qb], ((seg_count >> 1) - 1) & 1, p.ws.err);
            if (ok) {
              dev::mbar_arrive_expect_tx(&qfull[qb], (uint32_t)(G * C::QROW));
              dev::bulk_load(qbuf + qb * kGPad * C::QROW,
                             p.q + ((int64_t)rowj * hq + (int64_t)hj * G) * C::QROW, (uint32_t)(G * C::QROW),
                             &qfull[qb], pol);
            }
            ++seg_count;
          }
          const int64_t k = base + j - t0;
          const int stage = (int)(k % NST);
          const uint32_t n = (uint32_t)(k / NST);
          if (ok && n > 0) ok = dev::mbar_wait(&empty[stage], (n - 1) & 1, p.ws.err);
          if (ok) {
            uint8_t* st = ring + (size_t)stage * C::STAGE;
            dev::mbar_arrive_expect_tx(&full[stage], (uint32_t)C::STAGE);
            const int32_t krow = (blkj * hkv + hj) * BS;
#pragma unroll
            for (int c = 0; c < C::NCH; ++c)
              dev::tma_load_2d(st + c * BS * 128, &tm_k, c * (128 / C::ELEM), krow, &full[stage], pol);
            if constexpr (C::FP8) {
              dev::bulk_load(st + C::TILE, p.v_cache + ((int64_t)blkj * hkv + hj) * C::TILE, (uint32_t)C::TILE,
                             &full[stage], pol);
            } else {
#pragma unroll
              for (int c = 0; c < C::NCH; ++c)
                dev::tma_load_2d(st + C::TILE + c * BS * 128, &tm_v, c * 64, krow, &full[stage], pol);
            }
            ++issued;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    }
    if (!ok && lane == 0) {
      // drain: let copies already issued land before the CTA can exit
      for (int64_t k = (issued > NST ? issued - NST : 0); k < issued; ++k)
        dev::mbar_wait(&full[k % NST], (uint32_t)((k / NST) & 1), nullptr, 100000000ull);
    }
    return;
  }

  // ======================= consumer warps ===================================
  const int g = lane >> 2, tq = lane & 3;
  const uint32_t ring_u32 = dev::smem_u32(ring);
  const uint32_t qbuf_u32 = dev::smem_u32(qbuf);
  const int lr = lane & 7, li = lane >> 3;  // ldmatrix: row within matrix, matrix index
  // A timed-out wait sets `ok` false: the warp stops waiting and computing,
  // but still reaches every merge barrier, and all consumer warps leave
  // together after the barrier that follows (abort_flag), so none is left
  // waiting on a barrier the others never reach.
  int64_t t = t0;
  int seg_count = 0;
  bool ok = true;
  while (t < t1) {
    const int s = find_seq(prefix, S, hkv, t);
    const int nb = prefix[s + 1] - prefix[s];
    const int64_t seg0 = (int64_t)hkv * prefix[s];
    const int h = (int)((t - seg0) / nb);
    const int64_t a = seg0 + (int64_t)h * nb, b = a + nb;
    const int64_t pe = min(b, t1);
    const int len = min(__ldg(p.rows.seq_lens + s), nb * BS);
    const int row = p.rows.qsl ? __ldg(p.rows.qsl + s) : s;

    // ---- query fragments (B operand of S^T = K Q^T) ----
    const int qb = seg_count & 1;
    if (ok) ok = dev::mbar_wait(&qfull[qb], (seg_count >> 1) & 1, p.ws.err);
    uint32_t qf[C::KSTEPS][2];
    const uint32_t qrow_u32 = qbuf_u32 + qb * kGPad * C::QROW;
    if constexpr (!C::FP8) {
#pragma unroll
      for (int j = 0; j < C::KSTEPS / 2; ++j)
        dev::ldsm_x4(qrow_u32 + lr * C::QROW + (4 * j + li) * 16, qf[2 * j][0], qf[2 * j][1], qf[2 * j + 1][0],
                     qf[2 * j + 1][1]);
    } else {
      // d order inside a 16-wide k-step follows the e4m3 byte split: logical
      // k (2t, 2t+1 | 2t+8, 2t+9) <-> d (4t, 4t+2 | 4t+1, 4t+3)
      const uint8_t* qr = qbuf + qb * kGPad * C::QROW + g * C::QROW;
#pragma unroll
      for (int u = 0; u < C::KSTEPS; ++u) {
        const uint2 w = *reinterpret_cast<const uint2*>(qr + (16 * u + 4 * tq) * 2);
        const float q0 = dev::bf16_bits_to_f32(w.x & 0xFFFFu), q1 = dev::bf16_bits_to_f32(w.x >> 16);
        const float q2 = dev::bf16_bits_to_f32(w.y & 0xFFFFu), q3 = dev::bf16_bits_to_f32(w.y >> 16);
        qf[u][0] = dev::pack_f16(q0, q2);
        qf[u][1] = dev::pack_f16(q1, q3);
      }
    }
    __syncwarp();
    if (lane == 0) dev::mbar_arrive(&qempty[qb]);

    float m0 = -1e30f, m1 = -1e30f, l0 = 0.f, l1 = 0.f;
    float o[C::DM][4];
#pragma unroll
    for (int i = 0; i < C::DM; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

    for (int64_t tile = t + warp; tile < pe && ok; tile += kConsumerWarps) {
      const int64_t k = tile - t0;
      const int stage = (int)(k % NST);
      ok = dev::mbar_wait(&full[stage], (uint32_t)((k / NST) & 1), p.ws.err);
      if (!ok) break;
      const uint32_t kbase = ring_u32 + stage * C::STAGE;
      const uint32_t vbase = kbase + C::TILE;
      const int key0 = (int)(tile - a) * BS;
      if (len - key0 < BS) {
        // Slots past the context hold whatever the pool last stored there
        // (possibly NaN/Inf bit patterns): their scores are masked to -inf,
        // but 0 * NaN would still poison P*V, so their V rows are zeroed.
        const int valid = len - key0;
        uint8_t* vt = ring + (size_t)stage * C::STAGE + C::TILE;
        if constexpr (!C::FP8) {
          for (int i = lane; i < (BS - valid) * C::NCH * 8; i += 32) {
            const int key = valid + i / (C::NCH * 8), rest = i % (C::NCH * 8);
            *reinterpret_cast<uint4*>(vt + (rest >> 3) * (BS * 128) + key * 128 + (rest & 7) * 16) =
                make_uint4(0, 0, 0, 0);
          }
        } else {
          for (int i = lane; i < D * (BS - valid); i += 32) vt[(i / (BS - valid)) * BS + valid + i % (BS - valid)] = 0;
        }
        // order these generic-proxy writes before the async-proxy (TMA)
        // writes that refill this stage later
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
      }

      // ---- S^T = K Q^T ----
      float sc[C::KM][4];
#pragma unroll
      for (int km = 0; km < C::KM; ++km) {
        float acc0[4] = {0.f, 0.f, 0.f, 0.f}, acc1[4] = {0.f, 0.f, 0.f, 0.f};
        if constexpr (!C::FP8) {
          const int key = 16 * km + (li & 1) * 8 + lr;
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk) {
            const int gu = 2 * kk + (li >> 1);
            const uint32_t addr = kbase + (gu >> 3) * (BS * 128) + key * 128 + (((gu & 7) ^ (key & 7)) << 4);
            uint32_t a0, a1, a2, a3;
            dev::ldsm_x4(addr, a0, a1, a2, a3);
            if (kk & 1) dev::mma_bf16(acc1, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
            else dev::mma_bf16(acc0, a0, a1, a2, a3, qf[kk][0], qf[kk][1]);
          }
        } else {
          // A-row r holds key 2r (r < 8) or 2(r-8)+1, matching the key order
          // of the d-major V operand after the byte split
          const int ar = (li & 1) * 8 + lr;
          const int key = 16 * km + (ar < 8 ? 2 * ar : 2 * (ar - 8) + 1);
#pragma unroll
          for (int uu = 0; uu < C::KSTEPS / 2; ++uu) {
            const int unit = 2 * uu + (li >> 1);
            const uint32_t addr = kbase + key * 128 + ((unit ^ (key & 7)) << 4);
            uint32_t w0, w1, w2, w3;
            dev::ldsm_x4(addr, w0, w1, w2, w3);
            uint32_t l0w, h0w, l1w, h1w, l2w, h2w, l3w, h3w;
            dev::e4m3x4_to_f16x2x2(w0, l0w, h0w);
            dev::e4m3x4_to_f16x2x2(w1, l1w, h1w);
            dev::e4m3x4_to_f16x2x2(w2, l2w, h2w);
            dev::e4m3x4_to_f16x2x2(w3, l3w, h3w);
            dev::mma_f16(acc0, l0w, l1w, h0w, h1w, qf[2 * uu][0], qf[2 * uu][1]);
            dev::mma_f16(acc1, l2w, l3w, h2w, h3w, qf[2 * uu + 1][0], qf[2 * uu + 1][1]);
          }
        }
        // rows of this thread: keys r0 (row g) and r1 (row g+8)
        const int r0 = key0 + 16 * km + (C::FP8 ? 2 * g : g);
        const int r1 = key0 + 16 * km + (C::FP8 ? 2 * g + 1 : g + 8);
        sc[km][0] = r0 < len ? (acc0[0] + acc1[0]) * p.scale_log2 : -INFINITY;
        sc[km][1] = r0 < len ? (acc0[1] + acc1[1]) * p.scale_log2 : -INFINITY;
        sc[km][2] = r1 < len ? (acc0[2] + acc1[2]) * p.scale_log2 : -INFINITY;
        sc[km][3] = r1 < len ? (acc0[3] + acc1[3]) * p.scale_log2 : -INFINITY;
      }

      // ---- online softmax per query column (columns 2tq, 2tq+1) ----
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int km = 0; km < C::KM; ++km) {
        mx0 = fmaxf(mx0, fmaxf(sc[km][0], sc[km][2]));
        mx1 = fmaxf(mx1, fmaxf(sc[km][1], sc[km][3]));
      }
#pragma unroll
      for (int off = 4; off < 32; off <<= 1) {
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
      }
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float al0 = dev::ex2(m0 - mn0), al1 = dev::ex2(m1 - mn1);
      m0 = mn0;
      m1 = mn1;
      uint32_t pb0[C::KM], pb1[C::KM];
      float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
      for (int km = 0; km < C::KM; ++km) {
        const float p00 = dev::ex2(sc[km][0] - mn0), p01 = dev::ex2(sc[km][1] - mn1);
        const float p10 = dev::ex2(sc[km][2] - mn0), p11 = dev::ex2(sc[km][3] - mn1);
        ps0 += p00 + p10;
        ps1 += p01 + p11;
        if constexpr (C::FP8) {
          pb0[km] = dev::movmatrix_t(dev::pack_f16(p00, p01));
          pb1[km] = dev::movmatrix_t(dev::pack_f16(p10, p11));
        } else {
          pb0[km] = dev::movmatrix_t(dev::pack_bf16(p00, p01));
          pb1[km] = dev::movmatrix_t(dev::pack_bf16(p10, p11));
        }
      }
      l0 = l0 * al0 + ps0;
      l1 = l1 * al1 + ps1;
#pragma unroll
      for (int i = 0; i < C::DM; ++i) {
        o[i][0] *= al0;
        o[i][1] *= al1;
        o[i][2] *= al0;
        o[i][3] *= al1;
      }

      // ---- O^T += V^T P^T ----
      if constexpr (!C::FP8) {
#pragma unroll
        for (int mt = 0; mt < C::DM; ++mt) {
#pragma unroll
          for (int km = 0; km < C::KM; ++km) {
            const int key = 16 * km + (li >> 1) * 8 + lr;
            const int gu = 2 * mt + (li & 1);
            const uint32_t addr = vbase + (gu >> 3) * (BS * 128) + key * 128 + (((gu & 7) ^ (key & 7)) << 4);
            uint32_t a0, a1, a2, a3;
            dev::ldsm_x4_t(addr, a0, a1, a2, a3);
            dev::mma_bf16(o[mt], a0, a1, a2, a3, pb0[km], pb1[km]);
          }
        }
      } else {
#pragma unroll
        for (int mt2 = 0; mt2 < C::DM / 2; ++mt2) {
#pragma unroll
          for (int km = 0; km < C::KM; ++km) {
            const int d = 16 * (2 * mt2 + (li >> 1)) + (li & 1) * 8 + lr;
            uint32_t w0, w1, w2, w3;
            dev::ldsm_x4(vbase + d * BS + km * 16, w0, w1, w2, w3);
            uint32_t l0w, h0w, l1w, h1w, l2w, h2w, l3w, h3w;
            dev::e4m3x4_to_f16x2x2(w0, l0w, h0w);
            dev::e4m3x4_to_f16x2x2(w1, l1w, h1w);
            dev::e4m3x4_to_f16x2x2(w2, l2w, h2w);
            dev::e4m3x4_to_f16x2x2(w3, l3w, h3w);
            dev::mma_f16(o[2 * mt2], l0w, l1w, h0w, h1w, pb0[km], pb1[km]);
            dev::mma_f16(o[2 * mt2 + 1], l2w, l3w, h2w, h3w, pb0[km], pb1[km]);
          }
        }
      }
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(&empty[stage]);
    }
    if (!ok && lane == 0) abort_flag = 1;

    // ---- merge the four warps' states for this (sequence, kv head) ----
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    constexpr int MS = D + kMergeStride;
    float* mo = merge_o + warp * kGPad * MS;
    float* mml = merge_ml + warp * kGPad * 2;
    if (g == 0) {
      mml[(2 * tq) * 2] = m0;
      mml[(2 * tq) * 2 + 1] = l0;
      mml[(2 * tq + 1) * 2] = m1;
      mml[(2 * tq + 1) * 2 + 1] = l1;
    }
#pragma unroll
    for (int mt = 0; mt < C::DM; ++mt) {
      const int d0 = 16 * mt + g;
      mo[(2 * tq) * MS + d0] = o[mt][0];
      mo[(2 * tq + 1) * MS + d0] = o[mt][1];
      mo[(2 * tq) * MS + d0 + 8] = o[mt][2];
      mo[(2 * tq + 1) * MS + d0 + 8] = o[mt][3];
    }
    dev::named_bar_sync(1, kConsumerWarps * 32);
    const bool aborted = *reinterpret_cast<volatile int*>(&abort_flag) != 0;
    const bool complete = (t == a) && (pe == b);
    const int64_t slot = 2 * cta + (t == t0 ? 0 : 1);
    for (int idx = tid; idx < (aborted ? 0 : G * D); idx += kConsumerWarps * 32) {
      const int jq = idx / D, d = idx - jq * D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, merge_ml[(w * kGPad + jq) * 2]);
      float lsum = 0.f, acc = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float e = dev::ex2(merge_ml[(w * kGPad + jq) * 2] - M);
        lsum += merge_ml[(w * kGPad + jq) * 2 + 1] * e;
        acc += merge_o[(w * kGPad + jq) * MS + d] * e;
      }
      if (complete) {
        const int64_t oi = ((int64_t)row * hq + (int64_t)h * G + jq) * D + d;
        reinterpret_cast<__nv_bfloat16*>(p.out)[oi] = __float2bfloat16_rn(acc / lsum * p.out_scale);
      } else {
        p.ws.o[(slot * G + jq) * D + d] = acc;
        if (d == 0) {
          p.ws.ml[(slot * G + jq) * 2] = M;
          p.ws.ml[(slot * G + jq) * 2 + 1] = lsum;
        }
      }
    }
    dev::named_bar_sync(1, kConsumerWarps * 32);
    if (aborted) return;
    t = pe;
    ++seg_count;
  }
}

// Merges the partials of every (sequence, kv head) whose tiles were split
// over several CTAs: a log-sum-exp combine, one warp per (sequence, kv head),
// contributors spread over lanes and reduced with warp shuffles.
template <int D>
__global__ void __launch_bounds__(128) decode_combine_kernel(const DecodeParams p) {
  dev::grid_dep_wait();
  const int lane = threadIdx.x & 31;
  const int64_t wid = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int S = p.rows.num_seqs, hkv = p.num_kv_heads, G = p.group, hq = p.num_q_heads;
  if (wid >= (int64_t)S * hkv) return;
  const int s = (int)(wid / hkv), h = (int)(wid % hkv);
  const int32_t* prefix = p.ws.prefix;
  const int nb = prefix[s + 1] - prefix[s];
  const int row = p.rows.qsl ? p.rows.qsl[s] : s;
  __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out);
  if (nb == 0) {
    const int qlen = p.rows.qsl ? p.rows.qsl[s + 1] - p.rows.qsl[s] : 1;
    if (qlen == 1)  // an empty context attends nothing: zero output
      for (int jq = 0; jq < G; ++jq)
        for (int d = lane; d < D; d += 32)
          out[((int64_t)row * hq + (int64_t)h * G + jq) * D + d] = __float2bfloat16_rn(0.f);
    return;
  }
  const int64_t T = (int64_t)hkv * prefix[S];
  const int64_t P = p.grid;
  const int64_t a = (int64_t)hkv * prefix[s] + (int64_t)h * nb, b = a + nb;
  const int64_t cf = cta_of(a, T, P), cl = cta_of(b - 1, T, P);
  if (cf == cl) return;  // finished in place by its only CTA
  constexpr int E = D / 32;
  for (int jq = 0; jq < G; ++jq) {
    float M = -INFINITY;
    for (int64_t c = cf + lane; c <= cl; c += 32) {
      const int64_t slot = 2 * c + (range_start(c, T, P) < a ? 1 : 0);
      M = fmaxf(M, p.ws.ml[(slot * G + jq) * 2]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, off));
    float lsum = 0.f, acc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) acc[e] = 0.f;
    for (int64_t cb = cf; cb <= cl; cb += 32) {
      const int64_t c = cb + lane;
      float w = 0.f;
      int64_t slot = 0;
      if (c <= cl) {
        slot = 2 * c + (range_start(c, T, P) < a ? 1 : 0);
        w = dev::ex2(p.ws.ml[(slot * G + jq) * 2] - M);
        lsum += p.ws.ml[(slot * G + jq) * 2 + 1] * w;
      }
      const int n = (int)(cl - cb + 1 < 32 ? cl - cb + 1 : 32);
      for (int k = 0; k < n; ++k) {
        const float wk = __shfl_sync(0xffffffffu, w, k);
        const int64_t sk = __shfl_sync(0xffffffffu, slot, k);
        const float* po = p.ws.o + (sk * G + jq) * D;
#pragma unroll
        for (int e = 0; e < E; ++e) acc[e] += wk * po[lane + 32 * e];
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) lsum += __shfl_xor_sync(0xffffffffu, lsum, off);
    const float inv = p.out_scale / lsum;
#pragma unroll
    for (int e = 0; e < E; ++e)
      out[((int64_t)row * hq + (int64_t)h * G + jq) * D + lane + 32 * e] = __float2bfloat16_rn(acc[e] * inv);
  }
}

template <int KV, int D, int BS>
cudaError_t launch_instance(const DecodeParams& p, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                            cudaStream_t stream) {
  using C = Cfg<KV, D, BS>;
  const SmemLayout L = smem_layout(C::STAGE, C::QROW, D, p.nstages, p.rows.num_seqs);
  auto kern = decode_tc_kernel<KV, D, BS>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = L.total;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, kern, tm_k, tm_v, p);
  if (e != cudaSuccess) return e;
  const int64_t warps = (int64_t)p.rows.num_seqs * p.num_kv_heads;
  cudaLaunchConfig_t cc = {};
  cc.gridDim = dim3((unsigned)((warps + 3) / 4));
  cc.blockDim = dim3(128);
  cc.dynamicSmemBytes = 0;
  cc.stream = stream;
  cc.attrs = attr;
  cc.numAttrs = 1;
  return cudaLaunchKernelEx(&cc, decode_combine_kernel<D>, p);
}

}  // namespace

int decode_tc_grid(int num_sms) { return kCtasPerSM * num_sms; }

size_t decode_tc_smem_bytes(int kv, int head_dim, int block_size, int num_seqs, int nstages) {
  const int elem = kv == kFP8 ? 1 : 2;
  const int stage = 2 * block_size * head_dim * elem;
  return smem_layout(stage, head_dim * 2, head_dim, nstages, num_seqs).total;
}

// Stages that fit two CTAs per SM.
static int pick_stages(int kv, int head_dim, int block_size, int num_seqs) {
  const int elem = kv == kFP8 ? 1 : 2;
  const int stage = 2 * block_size * head_dim * elem;
  const int budget = kSmemPerSM / kCtasPerSM - 1024;  // 1 KB per CTA is reserved
  const int fixed = (int)smem_layout(stage, head_dim * 2, head_dim, 0, num_seqs).total;
  int n = (budget - fixed) / (stage + 16);
  if (n > kMaxStages) n = kMaxStages;
  return n;
}

size_t decode_tc_workspace_bytes(int num_seqs, int group, int head_dim, int num_sms) {
  const size_t P = (size_t)decode_tc_grid(num_sms);
  size_t off = 256;                                      // error word
  off += ((size_t)(num_seqs + 1) * 4 + 255) / 256 * 256;  // prefix
  off += (2 * P * group * 2 * 4 + 255) / 256 * 256;      // (max, sum)
  off += 2 * P * group * head_dim * 4;                   // partial outputs
  return off;
}

cudaError_t launch_decode_tc(const DecodeParams& p_in, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                             int kv, int head_dim, int block_size, int num_sms, cudaStream_t stream) {
  DecodeParams p = p_in;
  p.nstages = pick_stages(kv, head_dim, block_size, p.rows.num_seqs);
  if (p.nstages < 2) return cudaErrorNotSupported;
  p.grid = decode_tc_grid(num_sms);
  if (kv == kBF16) {
    if (head_dim == 128 && block_size == 16) return launch_instance<kBF16, 128, 16>(p, tm_k, tm_v, stream);
    if (head_dim == 128 && block_size == 32) return launch_instance<kBF16, 128, 32>(p, tm_k, tm_v, stream);
    if (head_dim == 64 && block_size == 16) return launch_instance<kBF16, 64, 16>(p, tm_k, tm_v, stream);
    if (head_dim == 64 && block_size == 32) return launch_instance<kBF16, 64, 32>(p, tm_k, tm_v, stream);
  } else if (kv == kFP8) {
    if (head_dim == 128 && block_size == 16) return launch_instance<kFP8, 128, 16>(p, tm_k, tm_v, stream);
    if (head_dim == 128 && block_size == 32) return launch_instance<kFP8, 128, 32>(p, tm_k, tm_v, stream);
  }
  return cudaErrorNotSupported;
}

}  // namespace pa
