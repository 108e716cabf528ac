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
//    are laid end to end and cut into one equal, contiguous range per warp
//    (persistent grid, 3 CTAs of 4 warps per SM), so a long context is split
//    over several warps (split-K over blocks) and every warp streams the
//    same number of bytes whatever the length mix.  Each warp works alone:
//    a (sequence, kv head) that lies wholly in its range is finished in
//    registers and written out.  One cut by warp ranges is merged by the
//    warp holding its first piece: that piece sits at the end of the warp's
//    range, so it finishes after the later pieces, which sit at the starts
//    of later warps' ranges.  Those store a partial (max, sum, unnormalised
//    output) and count themselves in with a release reduction; the merging
//    warp acquires the count (a bounded wait that normally ends at once) and
//    folds the partials into its own state with a log-sum-exp combine in the
//    MMA fragment layout.
//  * Each warp gathers its tiles through the block table with TMA: the K
//    tile (and the bf16 V tile) as 2-D tensor-map boxes of [block][128 B]
//    with 128-byte swizzle, the e4m3 V tile (d-major, contiguous) as one bulk
//    copy, into the warp's own ring of shared-memory stages, each guarded by
//    an mbarrier.  A warp refills a stage as soon as it has consumed it, so
//    every warp keeps its next tiles in flight and the load issue work is
//    spread over all warps of the SM.
//  * GQA groups are packed with
//    keys on the MMA's M side and the group's query rows on N (8, padded):
//    S^T = K Q^T and O^T += V^T P^T with mma.sync m16n8k16 (fp32 accumulate),
//    an online softmax per query column, and P^T moved into the B operand
//    with movmatrix.  e4m3 K/V become f16 exactly (the hardware's paired
//    e4m3 -> f16x2 conversion, two per four bytes), and the per-tensor
//    scales are folded into the softmax scale and the output scale.
#include <cuda_runtime.h>

#include "pa_device.cuh"
#include "pa_kernels.h"

namespace pa {
namespace {

constexpr int kWarps = 4;  // compute warps per CTA; each also issues its own loads
constexpr int kThreads = kWarps * 32;
constexpr int kGPad = 8;         // query rows per MMA N tile
constexpr int kMaxStagesPerWarp = 8;
constexpr int kSmemPerSM = 233472;  // B200: 228 KB per SM
constexpr float kRefSlack = 8.f;    // log2 growth of a column max before its softmax reference moves
// CTAs per SM: three (12 warps), as long as each warp's ring keeps two
// stages; more warps hide the latency of the per-tile work (the e4m3
// unpacking above all) and cut the tile space finer.  Measured against two
// CTAs: e4m3 -12% time, bf16 with long shared prefixes -11%, bf16 GQA the
// same.  The workspace is sized for this count.
template <int KV>
constexpr int ctas_per_sm() { return 3; }
constexpr int kMaxCtasPerSM = 3;

template <int KV, int D, int BS>
struct Cfg {
  static constexpr bool FP8 = KV == kFP8;
  static constexpr int ELEM = FP8 ? 1 : 2;
  static constexpr int ROW = D * ELEM;   // bytes per token row
  static constexpr int TILE = BS * ROW;  // bytes of one K (or V) tile
  static constexpr int KVB = 2 * TILE;   // K and V tiles of a stage
  static constexpr int NCH = ROW / 128;  // 128-byte chunks per K/V row
  static constexpr int KM = BS / 16;     // 16-key m-tiles per tile
  static constexpr int DM = D / 16;      // 16-d m-tiles of O^T
  static constexpr int KSTEPS = D / 16;  // k-steps of S^T = K Q^T
  static_assert(ROW % 128 == 0, "rows must be whole 128-byte swizzle rows");
  static_assert(BS % 16 == 0, "block size must be a multiple of 16");
};

struct SmemLayout {
  uint32_t ring, bars, info, prefix, total;
};

// A stage holds one tile's K and V and, when the tile opens a (sequence, kv
// head) piece, that piece's query rows (`q_area` bytes, a multiple of 1 KB so
// the next stage's tiles stay 1 KB aligned for the 128-byte swizzle).
__host__ __device__ inline int q_area_bytes(int group, int d) { return (group * d * 2 + 1023) / 1024 * 1024; }

__host__ __device__ inline SmemLayout smem_layout(int stage_bytes, int nsw, int num_seqs) {
  SmemLayout L;
  uint32_t off = 0;
  L.ring = off;
  off += (uint32_t)stage_bytes * nsw * kWarps;
  L.bars = off;
  off += (uint32_t)kWarps * nsw * 8;
  L.info = off;
  off += (uint32_t)kWarps * nsw * 16;
  L.prefix = off;
  off += (uint32_t)(num_seqs + 1) * 4;
  L.total = off + 1024;  // slack for aligning the base to 1024 bytes
  return L;
}

// Tile indices fit in 32 bits (the host rejects batches whose tile count
// could reach 2^31), so all per-tile arithmetic is 32-bit.

// Largest s in [0, S) with hkv * prefix[s] <= t (that sequence has tiles).
__device__ __forceinline__ int find_seq(const int32_t* prefix, int S, int hkv, int t) {
  int lo = 0, hi = S - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (hkv * prefix[mid] <= t) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// CTA c owns tiles [range_start(c), range_start(c + 1)); cta_of(x) is the
// CTA owning tile x.
__device__ __forceinline__ int range_start(int c, int T, int P) { return (int)((int64_t)c * T / P); }
__device__ __forceinline__ int cta_of(int x, int T, int P) { return (int)((((int64_t)x + 1) * P - 1) / T); }

// e4m3 tiles: thread (g, t) of an ldmatrix holds bytes 4t..4t+3 of a row,
// converted as the pairs (4t, 4t+1) -> A columns 2t, 2t+1 and (4t+2, 4t+3)
// -> A columns 2t+8, 2t+9.  For P V, whose A rows are d and whose columns
// are keys, logical k j therefore reads key kperm(j); S^T = K Q^T puts key
// kperm(r) on its A row r so that P^T, moved into the B operand, follows the
// same order.
__device__ __forceinline__ int kperm(int r) {
  return r < 8 ? 4 * (r >> 1) + (r & 1) : 4 * ((r - 8) >> 1) + 2 + (r & 1);
}

// Blocks of sequence s's row that its shared prefix covers (pa_decode_prefix;
// 0 otherwise): the prefix kernel attends them, the decode skips them.  A
// prefix that reaches the sequence's last token was refused in the
// prologue (error 4), and such a sequence has no tiles.
__device__ __forceinline__ int seq_skip(const DecodeParams& p, bool pfx, int s) {
  if (!pfx) return 0;
  const int pf = __ldg(p.pfx_of + s);
  return pf >= 0 ? __ldg(p.pfx_blocks + pf) : 0;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Arrival counters of cut pieces.  A contributor stores its partial, then
// lane 0 adds one with release semantics (no result, so no round trip); the
// merger acquires the count.  Counters start at zero (the workspace contract)
// and the merger puts its counter back to zero once it has merged.
__device__ __forceinline__ void count_in_release(unsigned int* cnt) {
  asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(cnt) : "memory");
}
__device__ __forceinline__ unsigned int load_acquire(const unsigned int* cnt) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(cnt) : "memory");
  return v;
}

// pa_decode_fused's write, by the warp that owns sequence s's last tile
// (its stage `st` has landed): the new token's K and V rows for kv head h
// (row `row` of k_new / v_new) go to offset `key` of the sequence's last
// block (entry nb - 1 of its table row) in the pools, as the bytes
// pa_cache_write stores, and into the stage.  A context clamped to its table row (error 3) or a last block
// outside the pool (error 2, already flagged) writes nothing to the pool.
template <class C>
__device__ __forceinline__ void fused_write(const DecodeParams& p, uint8_t* st, int s, int h, int row, int len,
                                            int key, int nb, int lane) {
  constexpr int BS = C::KM * 16, D = C::DM * 16;
  if (__ldg(p.rows.seq_lens + s) != len) return;  // clamped context: the token is not in the table row
  const int hkv = p.num_kv_heads;
  const int blk = __ldg(p.block_tables + (int64_t)s * p.max_blocks + (nb - 1));
  const bool to_pool = blk >= 0 && blk < p.num_blocks;
  const int64_t nrow = ((int64_t)row * hkv + h) * D * 2;  // bf16 new rows
  if constexpr (!C::FP8) {
    // lanes 0..15: 16-byte units of the K row, lanes 16..31: of the V row
    const int side = lane >> 4, u = lane & 15;
    if (u < C::NCH * 8) {
      const uint4 x = __ldg(reinterpret_cast<const uint4*>((side ? p.v_new : p.k_new) + nrow + u * 16));
      const int c = u >> 3, uu = u & 7;
      *reinterpret_cast<uint4*>(st + side * C::TILE + c * BS * 128 + key * 128 + ((uu ^ (key & 7)) << 4)) = x;
      if (to_pool)
        *reinterpret_cast<uint4*>((side ? p.v_pool : p.k_pool) + (((int64_t)blk * hkv + h) * BS + key) * C::ROW +
                                  u * 16) = x;
    }
  } else {
    // lane l quantises d = 4l .. 4l+3 of the K row and of the V row
    const float ks = p.k_head ? __ldg(p.k_head + h) : p.k_scale_w;
    const float vs = p.v_head ? __ldg(p.v_head + h) : p.v_scale_w;
    const uint2 kx = __ldg(reinterpret_cast<const uint2*>(p.k_new + nrow + 8 * lane));
    const uint2 vx = __ldg(reinterpret_cast<const uint2*>(p.v_new + nrow + 8 * lane));
    const uint32_t k01 = dev::e4m3x2_from_f32(__fdiv_rn(dev::bf16_bits_to_f32(kx.x & 0xFFFFu), ks),
                                              __fdiv_rn(dev::bf16_bits_to_f32(kx.x >> 16), ks));
    const uint32_t k23 = dev::e4m3x2_from_f32(__fdiv_rn(dev::bf16_bits_to_f32(kx.y & 0xFFFFu), ks),
                                              __fdiv_rn(dev::bf16_bits_to_f32(kx.y >> 16), ks));
    const uint32_t v01 = dev::e4m3x2_from_f32(__fdiv_rn(dev::bf16_bits_to_f32(vx.x & 0xFFFFu), vs),
                                              __fdiv_rn(dev::bf16_bits_to_f32(vx.x >> 16), vs));
    const uint32_t v23 = dev::e4m3x2_from_f32(__fdiv_rn(dev::bf16_bits_to_f32(vx.y & 0xFFFFu), vs),
                                              __fdiv_rn(dev::bf16_bits_to_f32(vx.y >> 16), vs));
    const uint32_t kw = k01 | (k23 << 16);
    // K: token-major 128-byte row, 128-byte swizzle in the stage
    *reinterpret_cast<uint32_t*>(st + key * 128 + (((lane >> 2) ^ (key & 7)) << 4) + 4 * (lane & 3)) = kw;
    // V: d-major [D][BS], one byte per d
    const uint8_t vb[4] = {(uint8_t)(v01 & 0xFF), (uint8_t)(v01 >> 8), (uint8_t)(v23 & 0xFF), (uint8_t)(v23 >> 8)};
#pragma unroll
    for (int i = 0; i < 4; ++i) st[C::TILE + (4 * lane + i) * BS + key] = vb[i];
    if (to_pool) {
      *reinterpret_cast<uint32_t*>(p.k_pool + (((int64_t)blk * hkv + h) * BS + key) * C::ROW + 4 * lane) = kw;
#pragma unroll
      for (int i = 0; i < 4; ++i) p.v_pool[(((int64_t)blk * hkv + h) * D + 4 * lane + i) * BS + key] = vb[i];
    }
  }
}

template <int KV, int D, int BS>
__global__ void __launch_bounds__(kThreads, ctas_per_sm<KV>())
    decode_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                     const DecodeParams p) {
  using C = Cfg<KV, D, BS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int NSW = p.nstages;  // ring stages per warp
  const int S = p.rows.num_seqs;
  const int hkv = p.num_kv_heads, G = p.group, hq = p.num_q_heads;
  const int QA = q_area_bytes(G, D);
  const int STAGE = C::KVB + QA;  // bytes per ring stage
  const bool pfx = p.pfx_of != nullptr;
  const SmemLayout L = smem_layout(STAGE, NSW, S);
  int32_t* prefix = reinterpret_cast<int32_t*>(smem + L.prefix);
  __shared__ int32_t warp_tot[kWarps];

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;

  // Programmatic dependent launch lets this grid start while the previous
  // kernel in the stream (normally the step's cache write) still runs.  The
  // prologue below reads only the step's inputs (lengths, query offsets,
  // block tables) and this call's workspace, which no kernel of the step
  // writes; the K/V pool and the queries are touched only after the wait
  // placed before the first copy is issued.

  // ---- blocks per sequence, exclusive prefix over the batch ----------------
  for (int s = tid; s < S; s += kThreads) {
    const int len = p.rows.seq_lens[s];
    const int qlen = p.rows.qsl ? p.rows.qsl[s + 1] - p.rows.qsl[s] : 1;
    int nb = (qlen == 1 && len > 0) ? (len + BS - 1) / BS : 0;
    if (nb > p.max_blocks) {  // context longer than its table row: flag, clamp
      atomicCAS(p.ws.err, 0, 3);
      nb = p.max_blocks;
    }
    if (pfx) {
      // a shared prefix's blocks are attended by the prefix kernel: only the
      // suffix is tiled here; its last token must lie past the prefix
      int skip = 0;
      const int pf = nb > 0 ? p.pfx_of[s] : -1;
      if (pf >= 0) {
        skip = p.pfx_blocks[pf];
        if ((int64_t)skip * BS > (int64_t)len - 1 || skip >= nb) {
          atomicCAS(p.ws.err, 0, 4);  // flag; the row stays zero
          skip = 0;
          nb = 0;
        } else {
          nb -= skip;
        }
      }
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
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L.bars) + warp * NSW;  // this warp's ring
  if (lane == 0) {
    for (int i = 0; i < NSW; ++i) dev::mbar_init(&full[i], 1);
    dev::fence_barrier_init();
  }
  __syncthreads();

  const int T = hkv * prefix[S];
  const int W = gridDim.x * kWarps;  // warps of the grid: the workers
  const int wk = blockIdx.x * kWarps + warp;
  // a decode row with an empty context attends nothing: zero output
  for (int s = blockIdx.x; s < S; s += gridDim.x) {
    const int qlen = p.rows.qsl ? p.rows.qsl[s + 1] - p.rows.qsl[s] : 1;
    if (qlen == 1 && prefix[s + 1] == prefix[s]) {
      const int row = p.rows.qsl ? p.rows.qsl[s] : s;
      for (int i = tid; i < hq * D; i += kThreads)
        reinterpret_cast<__nv_bfloat16*>(p.out)[(int64_t)row * hq * D + i] = __float2bfloat16_rn(0.f);
    }
  }
  const int wbeg = range_start(wk, T, W), wend = range_start(wk + 1, T, W);
  if (wbeg >= wend) {
    // no tiles: leave once the step's cache write is complete, so that a
    // kernel launched behind this one (the step's prompt rows) can rely on
    // every CTA of this grid having waited for it
    dev::grid_dep_wait();
    return;  // no CTA-wide synchronisation follows
  }

  // ---- this warp's tiles: [wbeg, wend); warp-tile u is tile wbeg + u --------
  const int nmine = wend - wbeg;
  uint8_t* ring = smem + L.ring + (size_t)warp * NSW * STAGE;
  const uint32_t ring_u32 = dev::smem_u32(ring);
  int4* info = reinterpret_cast<int4*>(smem + L.info) + warp * NSW;  // per stage: query row, length
  const uint64_t pol = dev::policy_evict_first();
  if (lane == 0) {
    dev::prefetch_tmap(&tm_k);
    if (!C::FP8) dev::prefetch_tmap(&tm_v);
  }

  // Lane l of a batch describes warp-tile ub + l: its kv head, physical block
  // and, if the tile opens a piece, the piece's query row and context length
  // (row -1 otherwise).  Two batches are kept: the one being issued and the
  // next one, whose global loads are in flight meanwhile.
  struct Desc {
    int h, blk, row, len;
  };
  auto describe = [&](int ub) {
    Desc d{0, 0, -1, 0};
    const int u = ub + lane;
    if (u < nmine) {
      const int t = wbeg + u;
      const int s = find_seq(prefix, S, hkv, t);
      const int nb = prefix[s + 1] - prefix[s];
      const int local = t - hkv * prefix[s];
      d.h = local / nb;
      const int skip = seq_skip(p, pfx, s);
      const int i = local - d.h * nb + skip;
      d.blk = __ldg(p.block_tables + (int64_t)s * p.max_blocks + i);
      if (d.blk < 0 || d.blk >= p.num_blocks) {  // bad table entry: flag, read block 0
        atomicCAS(p.ws.err, 0, 2);
        d.blk = 0;
      }
      if (i == skip || t == wbeg) {  // the tile opens a piece
        d.row = p.rows.qsl ? __ldg(p.rows.qsl + s) : s;
        d.len = min(__ldg(p.rows.seq_lens + s), (nb + skip) * BS);
      }
    }
    return d;
  };
  int cb = 0;
  Desc cur = describe(0), nxt{0, 0, -1, 0};
  // Issue warp-tile u into stage u % NSW (warp-uniform call, u increasing).
  // A tile that opens a piece also brings the piece's query rows into the
  // stage's query area, and its row and length into the stage's info slot.
  auto issue = [&](int u) {
    if (u >= cb + 32) {
      cb += 32;
      cur = nxt;
      nxt = describe(cb + 32);
    }
    const int hj = __shfl_sync(0xffffffffu, cur.h, u - cb);
    const int blkj = __shfl_sync(0xffffffffu, cur.blk, u - cb);
    const int rowj = __shfl_sync(0xffffffffu, cur.row, u - cb);
    const int lenj = __shfl_sync(0xffffffffu, cur.len, u - cb);
    const int st_i = u % NSW;
    uint8_t* st = ring + (size_t)st_i * STAGE;
    const uint32_t qbytes = (uint32_t)(G * D * 2);
    if (lane == 0) {
      if (rowj >= 0) info[st_i] = make_int4(rowj, lenj, 0, 0);
      dev::mbar_arrive_expect_tx(&full[st_i], (uint32_t)C::KVB + (rowj >= 0 ? qbytes : 0u));
    }
    __syncwarp();
    // one copy per lane, all in the same instructions: lanes 0..NCH-1 take
    // the K tile's 128-byte column boxes, the next lanes the V tile, the
    // next one the query rows
    const int32_t krow = (blkj * hkv + hj) * BS;
    if (lane < C::NCH) {
      dev::tma_load_2d(st + lane * BS * 128, &tm_k, lane * (128 / C::ELEM), krow, &full[st_i], pol);
    } else if (lane < 2 * C::NCH) {
      const int c = lane - C::NCH;
      if constexpr (C::FP8) {
        dev::bulk_load(st + C::TILE, p.v_cache + ((int64_t)blkj * hkv + hj) * C::TILE, (uint32_t)C::TILE,
                       &full[st_i], pol);
      } else {
        dev::tma_load_2d(st + C::TILE + c * BS * 128, &tm_v, c * 64, krow, &full[st_i], pol);
      }
    } else if (lane == 2 * C::NCH && rowj >= 0) {
      dev::bulk_load(st + C::KVB, p.q + ((int64_t)rowj * hq + (int64_t)hj * G) * D * 2, qbytes, &full[st_i], pol);
    }
  };
  int issued = 0;
  dev::grid_dep_wait();  // the pool rows this step wrote are visible from here on
  // only now may a dependent launch start (it relies on this wait, above)
  dev::grid_dep_launch();
  // Fault injection for tests (the workspace's second word, zero in normal
  // use): the later pieces of a cut context skip their count-in, so the
  // merging warp's wait runs out, after 1 ms instead of 2 s, and reports it.
  const bool inject = *reinterpret_cast<volatile const int32_t*>(p.ws.err + 1) == 1;
  for (; issued < NSW && issued < nmine; ++issued) issue(issued);
  nxt = describe(32);  // the next batch, needed from warp-tile 32 on

  const int g = lane >> 2, tq = lane & 3;
  const int lr = lane & 7, li = lane >> 3;  // ldmatrix: row within matrix, matrix index
  const int c0 = 2 * tq, c1 = 2 * tq + 1;   // this thread's query columns
  // A timed-out wait sets `ok` false: the warp stops waiting and computing
  // and leaves after draining its copies; every wait is bounded.
  int t = wbeg;
  int stage = 0;
  uint32_t phase = 0;
  int done = 0;  // warp-tiles consumed
  bool ok = true;
  while (t < wend && ok) {
    const int s = find_seq(prefix, S, hkv, t);
    const int nb = prefix[s + 1] - prefix[s];
    const int seg0 = hkv * prefix[s];
    const int h = (t - seg0) / nb;
    const int a = seg0 + h * nb, b = a + nb;
    const int pe = min(b, wend);
    const int skip = seq_skip(p, pfx, s);  // tile a holds block `skip` of the row
    int row = 0, len = 0;
    // this kv head's softmax and output scales (e4m3 per-head dequantisation)
    const float sl2 = p.k_head ? p.scale_log2 * __ldg(p.k_head + h) : p.scale_log2;
    const float osc = p.v_head ? p.out_scale * __ldg(p.v_head + h) : p.out_scale;
    uint32_t qf[C::KSTEPS][2];

    float m0 = -1e30f, m1 = -1e30f, l0 = 0.f, l1 = 0.f;
    float o[C::DM][4];
#pragma unroll
    for (int i = 0; i < C::DM; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;

    for (int tile = t; ok && tile < pe; ++tile) {
      ok = __all_sync(0xffffffffu, dev::mbar_wait(&full[stage], phase & 1, p.ws.err));
      if (!ok) break;
      if (tile == t) {
        // the piece's first tile: its stage carries the query rows and info
        const int4 inf = info[stage];
        row = inf.x;
        len = inf.y;
        // the row comes from this warp's own bookkeeping; a value outside
        // the batch is an internal inconsistency: flag it, write nothing
        if ((unsigned)row >= (unsigned)p.rows.num_rows || len <= 0) {
          if (lane == 0) atomicCAS(p.ws.err, 0, 5);
          ok = false;
          break;
        }
        if (p.k_new != nullptr && pe == b && lane < 2 * (D * 2 / 128)) {
          // pa_decode_fused: this piece ends the sequence, whose new K/V rows
          // its last tile stores; pull them into L2 now so that the write
          // does not wait on a cold load
          const uint8_t* src = ((lane & 1) ? p.v_new : p.k_new) + ((int64_t)row * hkv + h) * D * 2 + (lane >> 1) * 128;
          asm volatile("prefetch.global.L2 [%0];" ::"l"(src));
        }
        // ---- query fragments (B operand of S^T = K Q^T), rows >= G are zero ----
        const uint8_t* qs = ring + (size_t)stage * STAGE + C::KVB + g * D * 2;
        if constexpr (!C::FP8) {
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk) {
            qf[kk][0] = g < G ? *reinterpret_cast<const uint32_t*>(qs + (16 * kk + 2 * tq) * 2) : 0u;
            qf[kk][1] = g < G ? *reinterpret_cast<const uint32_t*>(qs + (16 * kk + 2 * tq + 8) * 2) : 0u;
          }
        } else {
          // d order inside a 16-wide k-step follows the e4m3 byte pairs
          // (a thread's four bytes of a K row are d 4t..4t+3):
          // logical k (2t, 2t+1 | 2t+8, 2t+9) <-> d (4t, 4t+1 | 4t+2, 4t+3)
#pragma unroll
          for (int kk = 0; kk < C::KSTEPS; ++kk) {
            uint2 w = make_uint2(0u, 0u);
            if (g < G) w = *reinterpret_cast<const uint2*>(qs + (16 * kk + 4 * tq) * 2);
            const float q0 = dev::bf16_bits_to_f32(w.x & 0xFFFFu), q1 = dev::bf16_bits_to_f32(w.x >> 16);
            const float q2 = dev::bf16_bits_to_f32(w.y & 0xFFFFu), q3 = dev::bf16_bits_to_f32(w.y >> 16);
            qf[kk][0] = dev::pack_f16(q0, q1);
            qf[kk][1] = dev::pack_f16(q2, q3);
          }
        }
      }
      const uint32_t kbase = ring_u32 + stage * STAGE;
      const uint32_t vbase = kbase + C::TILE;
      const int key0 = (tile - a + skip) * BS;
      if (p.k_new != nullptr && tile == b - 1) {
        // pa_decode_fused: the sequence's last tile holds its new token at
        // position len - 1; store the token's K/V rows into the pool and
        // over the landed tile, so the attention below uses them
        fused_write<C>(p, ring + (size_t)stage * STAGE, s, h, row, len, len - 1 - key0, skip + nb, lane);
        __syncwarp();
      }
      if (len - key0 < BS) {
        // Slots past the context hold whatever the pool last stored there
        // (possibly NaN/Inf bit patterns): their scores are masked to -inf,
        // but 0 * NaN would still poison P*V, so their V rows are zeroed.
        const int valid = len - key0;
        uint8_t* vt = ring + (size_t)stage * STAGE + C::TILE;
        if constexpr (!C::FP8) {
          for (int i = lane; i < (BS - valid) * C::NCH * 8; i += 32) {
            const int key = valid + i / (C::NCH * 8), rest = i % (C::NCH * 8);
            *reinterpret_cast<uint4*>(vt + (rest >> 3) * (BS * 128) + key * 128 + (rest & 7) * 16) =
                make_uint4(0, 0, 0, 0);
          }
        } else {
          for (int i = lane; i < D * (BS - valid); i += 32)
            vt[(i / (BS - valid)) * BS + valid + i % (BS - valid)] = 0;
        }
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
          // A-row r holds key kperm(r), the key order of the d-major V
          // operand after the byte pairing (logical k j <-> key kperm(j))
          const int ar = (li & 1) * 8 + lr;
          const int key = 16 * km + kperm(ar);
#pragma unroll
          for (int uu = 0; uu < C::KSTEPS / 2; ++uu) {
            const int unit = 2 * uu + (li >> 1);
            const uint32_t addr = kbase + key * 128 + ((unit ^ (key & 7)) << 4);
            uint32_t w0, w1, w2, w3;
            dev::ldsm_x4(addr, w0, w1, w2, w3);
            uint32_t l0w, h0w, l1w, h1w, l2w, h2w, l3w, h3w;
            dev::e4m3x4_to_f16x2(w0, l0w, h0w);
            dev::e4m3x4_to_f16x2(w1, l1w, h1w);
            dev::e4m3x4_to_f16x2(w2, l2w, h2w);
            dev::e4m3x4_to_f16x2(w3, l3w, h3w);
            dev::mma_f16(acc0, l0w, l1w, h0w, h1w, qf[2 * uu][0], qf[2 * uu][1]);
            dev::mma_f16(acc1, l2w, l3w, h2w, h3w, qf[2 * uu + 1][0], qf[2 * uu + 1][1]);
          }
        }
        // rows of this thread: keys r0 (row g) and r1 (row g+8)
        const int r0 = key0 + 16 * km + (C::FP8 ? kperm(g) : g);
        const int r1 = key0 + 16 * km + (C::FP8 ? kperm(g + 8) : g + 8);
        sc[km][0] = r0 < len ? (acc0[0] + acc1[0]) * sl2 : -INFINITY;
        sc[km][1] = r0 < len ? (acc0[1] + acc1[1]) * sl2 : -INFINITY;
        sc[km][2] = r1 < len ? (acc0[2] + acc1[2]) * sl2 : -INFINITY;
        sc[km][3] = r1 < len ? (acc0[3] + acc1[3]) * sl2 : -INFINITY;
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
      // Each column's exponentials use a reference that moves only when the
      // column's max exceeds it by more than 2^8 (log2 units): then the
      // running output and sum are rescaled; otherwise P = 2^(s - ref) stays
      // at most 2^8 and nothing is rescaled.  Any reference gives the same
      // result, and partials carry theirs as their max.
      const bool mv0 = mx0 > m0 + kRefSlack, mv1 = mx1 > m1 + kRefSlack;
      if (__any_sync(0xffffffffu, mv0 || mv1)) {
        const float mn0 = mv0 ? mx0 : m0, mn1 = mv1 ? mx1 : m1;
        const float al0 = dev::ex2(m0 - mn0), al1 = dev::ex2(m1 - mn1);
        m0 = mn0;
        m1 = mn1;
        l0 *= al0;
        l1 *= al1;
#pragma unroll
        for (int i = 0; i < C::DM; ++i) {
          o[i][0] *= al0;
          o[i][1] *= al1;
          o[i][2] *= al0;
          o[i][3] *= al1;
        }
      }
      uint32_t pb0[C::KM], pb1[C::KM];
      float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
      for (int km = 0; km < C::KM; ++km) {
        const float p00 = dev::ex2(sc[km][0] - m0), p01 = dev::ex2(sc[km][1] - m1);
        const float p10 = dev::ex2(sc[km][2] - m0), p11 = dev::ex2(sc[km][3] - m1);
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
      l0 += ps0;
      l1 += ps1;

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
            dev::e4m3x4_to_f16x2(w0, l0w, h0w);
            dev::e4m3x4_to_f16x2(w1, l1w, h1w);
            dev::e4m3x4_to_f16x2(w2, l2w, h2w);
            dev::e4m3x4_to_f16x2(w3, l3w, h3w);
            dev::mma_f16(o[2 * mt2], l0w, l1w, h0w, h1w, pb0[km], pb1[km]);
            dev::mma_f16(o[2 * mt2 + 1], l2w, l3w, h2w, h3w, pb0[km], pb1[km]);
          }
        }
      }
      // this stage is consumed: refill it with warp-tile u + NSW.  The
      // proxy fence orders this warp's generic-proxy accesses to the stage
      // before the TMA (async proxy) writes into it again.
      __syncwarp();
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      if (issued < nmine) issue(issued++);
      ++done;
      if (++stage == NSW) {
        stage = 0;
        ++phase;
      }
    }
    if (!ok) break;

    // ---- finish this (sequence, kv head) piece ----
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, off);
      l1 += __shfl_xor_sync(0xffffffffu, l1, off);
    }
    const int64_t obase = ((int64_t)row * hq + (int64_t)h * G) * D;
    if (t != a) {
      // a later piece of a sequence cut by warp ranges (it starts this
      // warp's range, so each warp has at most one): store the partial in
      // the warp's slot and count it in
      float* po = p.ws.o + (int64_t)wk * G * D;
      float* pml = p.ws.ml + (int64_t)wk * G * 2;
#pragma unroll
      for (int mt = 0; mt < C::DM; ++mt) {
        const int d0 = 16 * mt + g;
        if (c0 < G) {
          po[c0 * D + d0] = o[mt][0];
          po[c0 * D + d0 + 8] = o[mt][2];
        }
        if (c1 < G) {
          po[c1 * D + d0] = o[mt][1];
          po[c1 * D + d0 + 8] = o[mt][3];
        }
      }
      if (g == 0) {
        if (c0 < G) {
          pml[c0 * 2] = m0;
          pml[c0 * 2 + 1] = l0;
        }
        if (c1 < G) {
          pml[c1 * 2] = m1;
          pml[c1 * 2 + 1] = l1;
        }
      }
      __syncwarp();
      if (lane == 0 && !inject) count_in_release(p.ws.cnt + (int64_t)s * hkv + h);
    } else {
      // the sequence's first piece: this warp finishes the (sequence, kv
      // head).  If the context was cut by the end of this warp's range, the
      // other pieces sit at the starts of later warps' ranges and finish
      // first: wait for their count and fold their partials into this
      // warp's state in the MMA fragment layout (a log-sum-exp combine).  A
      // shared prefix's chunk partials (pa_decode_prefix) are folded the
      // same way.  Then the output.
      float M0 = m0, M1 = m1, L0 = l0, L1 = l1;
      // fold one partial: (max, sum) pairs and O rows of the group's query
      // heads, column c at pml + 2c and po + c * D; its (max, sum) and its
      // outputs are loaded together, so a partial costs one round trip to L2
      auto fold = [&](const float* pml, const float* po) {
        const float mc0 = c0 < G ? __ldcg(pml + c0 * 2) : -INFINITY;
        const float mc1 = c1 < G ? __ldcg(pml + c1 * 2) : -INFINITY;
        const float lc0 = c0 < G ? __ldcg(pml + c0 * 2 + 1) : 0.f;
        const float lc1 = c1 < G ? __ldcg(pml + c1 * 2 + 1) : 0.f;
        float oc[C::DM][4];
#pragma unroll
        for (int mt = 0; mt < C::DM; ++mt) {
          const int d0 = 16 * mt + g;
          oc[mt][0] = c0 < G ? __ldcg(po + c0 * D + d0) : 0.f;
          oc[mt][2] = c0 < G ? __ldcg(po + c0 * D + d0 + 8) : 0.f;
          oc[mt][1] = c1 < G ? __ldcg(po + c1 * D + d0) : 0.f;
          oc[mt][3] = c1 < G ? __ldcg(po + c1 * D + d0 + 8) : 0.f;
        }
        const float n0 = fmaxf(M0, mc0), n1 = fmaxf(M1, mc1);
        const float a0 = dev::ex2(M0 - n0), a1 = dev::ex2(M1 - n1);
        const float w0 = dev::ex2(mc0 - n0), w1 = dev::ex2(mc1 - n1);
        L0 = L0 * a0 + lc0 * w0;
        L1 = L1 * a1 + lc1 * w1;
#pragma unroll
        for (int mt = 0; mt < C::DM; ++mt) {
          o[mt][0] = o[mt][0] * a0 + oc[mt][0] * w0;
          o[mt][2] = o[mt][2] * a0 + oc[mt][2] * w0;
          o[mt][1] = o[mt][1] * a1 + oc[mt][1] * w1;
          o[mt][3] = o[mt][3] * a1 + oc[mt][3] * w1;
        }
        M0 = n0;
        M1 = n1;
      };
      unsigned int* cnt = p.ws.cnt + (int64_t)s * hkv + h;
      bool ready = true;
      if (pe != b) {
        const int cf = wk, cl = cta_of(b - 1, T, W);
        int others = 0;
        for (int c = cf + 1; c <= cl; ++c) others += range_start(c, T, W) < range_start(c + 1, T, W);
        if (lane == 0) {
          const uint64_t t_start = dev::globaltimer_ns();
          const uint64_t limit = inject ? 1000000ull : 2000000000ull;
          while (load_acquire(cnt) < (unsigned)others) {
            if (dev::globaltimer_ns() - t_start > limit) {  // bounded: flag and give up
              atomicCAS(p.ws.err, 0, 1);
              ready = false;
              break;
            }
          }
        }
        ready = __shfl_sync(0xffffffffu, ready, 0);
        __syncwarp();
        for (int c = cf + 1; c <= cl && ready; ++c) {
          if (range_start(c, T, W) >= range_start(c + 1, T, W)) continue;
          fold(p.ws.ml + (int64_t)c * G * 2, p.ws.o + (int64_t)c * G * D);
        }
      }
      if (skip > 0) {
        // the shared prefix's chunks, computed for member slot j
        const int j = __ldg(p.pfx_slot + s);
        const int nch = (__ldg(p.pfx_blocks + __ldg(p.pfx_of + s)) + p.pfx_chunk_blocks - 1) / p.pfx_chunk_blocks;
        for (int c = 0; c < nch; ++c) {
          const int64_t prow = ((int64_t)c * p.pfx_members + j) * hq + (int64_t)h * G;
          fold(p.pfx_ml + prow * 2, p.pfx_o + prow * D);
        }
      }
      // L0/L1 are whole-column sums: l0/l1 were reduced over the warp above
      // and a partial's sum is per column
      __nv_bfloat16* out = reinterpret_cast<__nv_bfloat16*>(p.out) + obase;
      const float i0 = osc / L0, i1 = osc / L1;
#pragma unroll
      for (int mt = 0; mt < C::DM; ++mt) {
        const int d0 = 16 * mt + g;
        if (c0 < G) {
          out[c0 * D + d0] = __float2bfloat16_rn(o[mt][0] * i0);
          out[c0 * D + d0 + 8] = __float2bfloat16_rn(o[mt][2] * i0);
        }
        if (c1 < G) {
          out[c1 * D + d0] = __float2bfloat16_rn(o[mt][1] * i1);
          out[c1 * D + d0 + 8] = __float2bfloat16_rn(o[mt][3] * i1);
        }
      }
      if (pe != b) {
        // ready for the next call (or a replay of this one)
        __syncwarp();
        if (lane == 0 && ready) *cnt = 0u;
      }
    }
    t = pe;
  }
  if (!ok && lane == 0) {
    // drain: let this warp's copies still in flight land before exiting
    for (int k = done; k < issued; ++k) dev::mbar_wait(&full[k % NSW], (uint32_t)((k / NSW) & 1), nullptr, 100000000ull);
  }
}

// Forward progress: a merging warp waits for pieces held by later CTAs, so
// every CTA of the grid must be resident at once.  The grid is therefore
// capped at the CTAs per SM that the runtime reports for this instance's
// shared memory and registers, times the SMs.  (Two decode grids must not
// run at the same time on one GPU: each could hold the SMs the other's later
// CTAs wait for; the bounded wait would then end both with error word 1.)
template <int KV, int D, int BS>
cudaError_t launch_instance(DecodeParams p, const CUtensorMap& tm_k, const CUtensorMap& tm_v, int num_sms,
                            cudaStream_t stream) {
  using C = Cfg<KV, D, BS>;
  const SmemLayout L = smem_layout(C::KVB + q_area_bytes(p.group, D), p.nstages, p.rows.num_seqs);
  auto kern = decode_tc_kernel<KV, D, BS>;
  // raise the kernel's dynamic shared memory limit once per device
  static int set_for[64] = {0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev >= 64 || set_for[dev] < (int)L.total) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L.total);
    if (e != cudaSuccess) return e;
    if (dev < 64) set_for[dev] = (int)L.total;
  }
  // resident CTAs per SM for this shared-memory size, queried once per
  // device and size (host arithmetic only: allowed while a stream captures)
  static int occ_smem[64] = {0}, occ_ctas[64] = {0};
  int resident = dev < 64 && occ_smem[dev] == (int)L.total ? occ_ctas[dev] : 0;
  if (resident == 0) {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&resident, kern, kThreads, L.total);
    if (e != cudaSuccess) return e;
    if (dev < 64) {
      occ_smem[dev] = (int)L.total;
      occ_ctas[dev] = resident;
    }
  }
  if (resident < 1) return cudaErrorNotSupported;
  if (p.grid > resident * num_sms) p.grid = resident * num_sms;
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
  return cudaLaunchKernelEx(&cfg, kern, tm_k, tm_v, p);
}

}  // namespace

int decode_tc_workers(int num_sms) { return kMaxCtasPerSM * num_sms * kWarps; }

size_t decode_tc_smem_bytes(int kv, int head_dim, int block_size, int group, int num_seqs, int nstages) {
  const int elem = kv == kFP8 ? 1 : 2;
  const int stage = 2 * block_size * head_dim * elem + q_area_bytes(group, head_dim);
  return smem_layout(stage, nstages, num_seqs).total;
}

// Ring stages per warp that fit `ctas` CTAs per SM.
static int pick_stages(int kv, int head_dim, int block_size, int group, int num_seqs, int ctas) {
  const int elem = kv == kFP8 ? 1 : 2;
  const int stage = 2 * block_size * head_dim * elem + q_area_bytes(group, head_dim);
  // 1 KB per CTA is reserved, plus a little static shared memory
  const int budget = kSmemPerSM / ctas - 1024 - 64;
  const int fixed = (int)smem_layout(stage, 0, num_seqs).total;
  int n = (budget - fixed) / (kWarps * (stage + 8 + 16));
  if (n > kMaxStagesPerWarp) n = kMaxStagesPerWarp;
  return n;
}

size_t decode_tc_workspace_bytes(int num_seqs, int num_kv_heads, int group, int head_dim, int num_sms) {
  const size_t P = (size_t)decode_tc_workers(num_sms);  // one partial slot per warp
  size_t off = 256;                                                  // error word
  off += ((size_t)num_seqs * num_kv_heads * 4 + 255) / 256 * 256;  // arrival counters
  off += (P * group * 2 * 4 + 255) / 256 * 256;                      // (max, sum)
  off += P * group * head_dim * 4;                                   // partial outputs
  return off;
}

cudaError_t launch_decode_tc(const DecodeParams& p_in, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                             int kv, int head_dim, int block_size, int num_sms, cudaStream_t stream) {
  DecodeParams p = p_in;
  // the dtype's CTAs per SM while each warp still gets a double-buffered
  // ring, else fewer CTAs with deeper rings (large blocks)
  int ctas = kv == kFP8 ? ctas_per_sm<kFP8>() : ctas_per_sm<kBF16>();
  for (;; --ctas) {
    p.nstages = pick_stages(kv, head_dim, block_size, p.group, p.rows.num_seqs, ctas);
    if (p.nstages >= 2 || ctas == 1) break;
  }
  if (p.nstages < 2) return cudaErrorNotSupported;
  p.grid = ctas * num_sms;
  if (kv == kBF16) {
    if (head_dim == 128 && block_size == 16) return launch_instance<kBF16, 128, 16>(p, tm_k, tm_v, num_sms, stream);
    if (head_dim == 128 && block_size == 32) return launch_instance<kBF16, 128, 32>(p, tm_k, tm_v, num_sms, stream);
    if (head_dim == 64 && block_size == 16) return launch_instance<kBF16, 64, 16>(p, tm_k, tm_v, num_sms, stream);
    if (head_dim == 64 && block_size == 32) return launch_instance<kBF16, 64, 32>(p, tm_k, tm_v, num_sms, stream);
  } else if (kv == kFP8) {
    if (head_dim == 128 && block_size == 16) return launch_instance<kFP8, 128, 16>(p, tm_k, tm_v, num_sms, stream);
    if (head_dim == 128 && block_size == 32) return launch_instance<kFP8, 128, 32>(p, tm_k, tm_v, num_sms, stream);
  }
  return cudaErrorNotSupported;
}

}  // namespace pa
