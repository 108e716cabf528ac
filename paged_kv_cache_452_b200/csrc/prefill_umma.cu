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
// How: a unit = (sequence, kv head, 128 / G query positions); the GQA
// group's heads of each position fill the MMA's M = 128 rows, so every K/V
// tile serves all of them.  One persistent CTA per SM walks its share of the
// units; the rings, the S buffers and the barriers run on across units, so
// the next unit's first tiles load while the current one finishes.
//  * warps 0 and 6 walk the block table and bring the K and the V halves of
//    128-key tiles into two rings of shared-memory stages with TMA (2-D
//    boxes of [block][128 B], 128-byte swizzle, boxes of consecutive blocks
//    stacked into one swizzled tile); a K stage is free again as soon as its
//    S MMA has run, a V stage once its PV MMA has; blocks past the keys the
//    unit needs are read out of range, which TMA fills with zeros; table
//    entries are read one tile ahead; the V loader also brings each unit's
//    query rows into the Q tile with TMA (3-D boxes of [positions][group
//    heads][128 B], which land in the MMA's row order) as soon as the
//    previous unit's last S MMA has run, so the next unit's first S does not
//    wait for a load issued after the previous unit's output;
//  * warp 1 holds the TMEM allocation and, from one thread, issues
//    S = Q K^T (M 128, N 128, K 16 steps; double-buffered S in TMEM), each
//    as soon as its K tile has landed and the row warps have read the S two
//    tiles back; warp 7, from one thread, issues O += P V (N = head_dim; O
//    stays in TMEM across tiles; P read from TMEM) once a tile's P is
//    written; each thread commits its MMAs to mbarriers.  The two streams
//    share no TMEM and wait for different things, so neither thread's waits
//    hold up the other's MMAs;
//  * warps 2..5 own one query row per thread (a warp per TMEM lane
//    quarter, so one per SM sub-partition): they read the row's 128 scores
//    of a tile from TMEM into registers, mask (causal, context length; only
//    the tiles at a row's end), write P = 2^(s - ref) as bf16 into one of
//    two P buffers in TMEM (so a tile's softmax need not wait for the
//    previous tile's PV to finish reading its P), and at the end divide O by
//    the sum.  The exponent reference ref is the row max of the unit's first
//    tile; later tiles skip the max unless their weights would grow past
//    2^64 (then ref moves and O and the running sum are rescaled: rare, and
//    the result is the same softmax up to rounding).  No row warp waits
//    for another; their softmax sets the tile period.
// Every wait is bounded (2 s, then the error word is set); TMEM is freed on
// every path.
#include <cuda_runtime.h>

#include "pa_device.cuh"
#include "pa_kernels.h"

namespace pa {
namespace {

constexpr int kRows = 128;    // query rows per unit (positions x group): the MMA's M
constexpr int kKeys = 128;    // keys per K/V tile: N of S = Q K^T, K of O = P V
// One softmax warp per TMEM lane quarter, a thread per query row: the row's
// 128 scores of a tile sit in registers and no row warp waits for another
// (splitting a row over two or four warps that exchange row maxima through
// shared memory measured slower).
constexpr int kRowWarps = 4;
// warp 0 loads K, warp 1 issues the S MMAs, then the row warps, then the V
// loader and the warp that issues the PV MMAs
constexpr int kThreads = 32 * (kRowWarps + 4);
constexpr int kVWarp = kRowWarps + 2;
constexpr int kPvWarp = kRowWarps + 3;
constexpr uint32_t kTmemCols = 512;
constexpr int kSmemOptIn = 232448;  // 227 KB per block: dynamic plus static shared memory
constexpr int kStaticSmem = 64;     // the kernel's static shared memory (warp_tot), at most
static_assert(4 * (kThreads / 32) <= kStaticSmem, "static shared memory reserve");
constexpr int kChunk = 128 * 128;   // one 128-byte-wide chunk of a 128-row tile
constexpr float kBig = 18446744073709551616.f;  // 2^64: the most a tile's weights may sum to on the fast path
constexpr int kUQ = 4;              // unit queue entries (the K loader claims, the other roles follow)
// roles that read each queue entry: the V loader, the two MMA threads and
// the four row warps
constexpr int kUQReaders = 7;

template <int D, int BS>
struct U {
  static constexpr int NCH = D / 64;               // 128-byte chunks of a row
  static constexpr int QBYTES = NCH * kChunk;      // Q tile
  static constexpr int KVT = NCH * kChunk;         // K (or V) tile: one ring stage
  static constexpr int BPT = kKeys / BS;           // blocks per tile
  static constexpr int BOXES = NCH * BPT;          // TMA boxes per stage
  static constexpr int KSTEPS_S = D / 16;
  static constexpr int KSTEPS_O = kKeys / 16;
  static_assert(BOXES <= 32, "one box per loader lane");
};

struct Bars {
  // kfull[NSK], kempty[NSK], vfull[NSV], vempty[NSV], then s_full[2],
  // s_free[2], p_full[2], o_full[2], q_full, o_free, done, uq_full[kUQ],
  // uq_empty[kUQ], q_free
  uint64_t* kfull;
  uint64_t* kempty;
  uint64_t* vfull;
  uint64_t* vempty;
  uint64_t* s_full;
  uint64_t* s_free;
  uint64_t* p_full;
  uint64_t* o_full;
  uint64_t* q_full;
  uint64_t* o_free;
  uint64_t* done;
  uint64_t* uq_full;
  uint64_t* uq_empty;
  uint64_t* q_free;
};

struct ULayout {
  uint32_t q, kring, vring, bars, tmem, uq, prefix, total;
};
__host__ __device__ inline ULayout u_layout(int qbytes, int kvt, int nsk, int nsv, int num_seqs) {
  ULayout L;
  uint32_t off = 0;
  L.q = off;
  off += qbytes;
  L.kring = off;
  off += (uint32_t)kvt * nsk;
  L.vring = off;
  off += (uint32_t)kvt * nsv;
  L.bars = off;
  off += (uint32_t)(2 * nsk + 2 * nsv + 12 + 2 * kUQ) * 8;
  L.tmem = off;
  off += 16;
  L.uq = off;  // unit queue [kUQ]
  off += kUQ * 4;
  L.prefix = off;
  off += (uint32_t)(num_seqs + 1) * 4;
  L.total = off + 1024;  // slack for aligning the base to 1024 bytes
  return L;
}

// Byte offset of 16-byte unit u of row r in a 128-byte-swizzled chunk.
__device__ __forceinline__ uint32_t swz(int r, int u) { return (uint32_t)(r * 128 + ((u ^ (r & 7)) << 4)); }

// PFX: the shared-prefix mode (pa_decode_prefix): a unit is (prefix, kv
// head, 128 / G member sequences, one chunk of the prefix's keys); its rows
// are the members' decode queries, every prefix key is visible to every row,
// and it writes partial (max reference, sum, unnormalised O) rows.
template <int D, int BS, bool PFX>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_umma_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_q, const PrefillParams p) {
  using C = U<D, BS>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int NSK = p.nstages, NSV = p.nstages_v;
  const int S = p.rows.num_seqs;
  const ULayout L = u_layout(C::QBYTES, C::KVT, NSK, NSV, S);
  uint8_t* qs = smem + L.q;
  uint8_t* kring = smem + L.kring;
  uint8_t* vring = smem + L.vring;
  uint64_t* bar0 = reinterpret_cast<uint64_t*>(smem + L.bars);
  uint64_t* bx = bar0 + 2 * NSK + 2 * NSV;
  Bars B{bar0,   bar0 + NSK, bar0 + 2 * NSK, bar0 + 2 * NSK + NSV, bx, bx + 2, bx + 4, bx + 6, bx + 8, bx + 9,
         bx + 10, bx + 11,   bx + 11 + kUQ,  bx + 11 + 2 * kUQ};
  int32_t* uq = reinterpret_cast<int32_t*>(smem + L.uq);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L.tmem);
  int32_t* prefix = reinterpret_cast<int32_t*>(smem + L.prefix);  // units before sequence s
  __shared__ int32_t warp_tot[kThreads / 32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = p.group, hq = p.num_q_heads, hkv = p.num_kv_heads;
  const int QB = kRows / G;  // query positions per unit

  // Launched right behind the decode kernel of the same step, this grid starts
  // only once every decode CTA has passed its own wait for the step's cache
  // write (it triggers its dependents after that wait), and its CTAs take SMs
  // as the decode's CTAs leave them; it does not wait for the decode grid to
  // finish, which it does not depend on.
  if (!p.after_decode) dev::grid_dep_wait();
  // ---- units per prompt sequence (per prefix), exclusive prefix ---------------
  for (int s = tid; s < S; s += kThreads) {
    if constexpr (PFX) {
      const int nm = p.pfx_start[s + 1] - p.pfx_start[s];
      const int nc = (p.pfx_blocks[s] * BS + p.chunk_keys - 1) / p.chunk_keys;
      prefix[s] = ((nm + QB - 1) / QB) * nc;
    } else {
      const int qlen = p.rows.qsl[s + 1] - p.rows.qsl[s];
      prefix[s] = qlen > 1 ? (qlen + QB - 1) / QB : 0;
    }
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
  // Units are claimed from a counter in the workspace, in ordinal order, so a
  // CTA that starts late or has short units simply takes fewer.  The last CTA
  // to finish puts the counter back to zero for the next launch.
  auto finish_queue = [&]() {
    if (tid == 0) {
      __threadfence();
      if (atomicAdd(p.unit_exit, 1) == (int)gridDim.x - 1) {
        atomicExch(p.unit_ctr, 0);
        atomicExch(p.unit_exit, 0);
      }
    }
  };
  if ((int)blockIdx.x >= nunits) {  // nothing allocated yet
    finish_queue();
    return;
  }

  // Ordinal i is query block i / Hkv (a sequence's last query blocks first,
  // the longest units of a sequence first) of kv head i % Hkv.
  // A unit's rows are query rows first + q0 .. first + q0 + qn - 1 (in PFX
  // mode: member slots first .. first + qn - 1); its keys are blocks
  // blk0 .. blk0 + nbneed - 1 of sequence s's table row.
  struct Unit {
    int s, h, first, q0, qn, pos0, seq_len, nbneed, ntiles, blk0, chunk;
  };
  auto unit_of = [&](int idx) {
    Unit u;
    const int ub = idx / hkv;
    int lo = 0, hi = S - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= ub) lo = mid; else hi = mid - 1;
    }
    u.h = idx % hkv;
    if constexpr (PFX) {
      // prefix lo: member tile mt, key chunk c
      const int nkeys = p.pfx_blocks[lo] * BS;
      const int nc = (nkeys + p.chunk_keys - 1) / p.chunk_keys;
      const int local = ub - prefix[lo];
      const int mt = local / nc;
      u.chunk = local - mt * nc;
      const int m0 = p.pfx_start[lo], nm = p.pfx_start[lo + 1] - m0;
      u.s = p.pfx_members[m0];  // every member's row holds the prefix's blocks
      u.first = m0 + mt * QB;
      u.q0 = 0;
      u.qn = min(QB, nm - mt * QB);
      u.pos0 = 1 << 30;  // no causal limit: every prefix key is visible
      const int kbeg = u.chunk * p.chunk_keys;
      u.seq_len = min(p.chunk_keys, nkeys - kbeg);  // keys of this chunk
      u.blk0 = kbeg / BS;
      u.nbneed = u.seq_len / BS;
      if (u.blk0 + u.nbneed > p.max_blocks) {
        if (warp == 2 && lane == 0) atomicCAS(p.err, 0, 3);
        u.nbneed = max(0, p.max_blocks - u.blk0);
      }
      u.ntiles = (u.seq_len + kKeys - 1) / kKeys;
      return u;
    }
    u.s = lo;
    u.blk0 = 0;
    u.chunk = 0;
    const int qb = prefix[lo + 1] - prefix[lo] - 1 - (ub - prefix[lo]);
    u.first = p.rows.qsl[lo];
    const int qlen = p.rows.qsl[lo + 1] - u.first;
    u.seq_len = p.rows.seq_lens[lo];
    u.pos0 = u.seq_len - qlen;  // position of the sequence's first query row
    u.q0 = qb * QB;             // first query (local index) of the unit
    u.qn = min(QB, qlen - u.q0);
    const int kend = min(u.seq_len, u.pos0 + u.q0 + u.qn);  // keys the unit needs: [0, kend)
    u.nbneed = (kend + BS - 1) / BS;
    if (u.nbneed > p.max_blocks) {
      if (warp == 2 && lane == 0) atomicCAS(p.err, 0, 3);  // (one reporter)
      u.nbneed = p.max_blocks;
    }
    u.ntiles = (u.nbneed * BS + kKeys - 1) / kKeys;
    return u;
  };

  if (tid == 0) {
    // one arrival (a TMA transaction or an MMA commit), or one per row warp
    for (int i = 0; i < 2 * NSK + 2 * NSV; ++i) dev::mbar_init(&bar0[i], 1);
    for (int i = 0; i < 2; ++i) {
      dev::mbar_init(&B.s_full[i], 1);
      dev::mbar_init(&B.s_free[i], kRowWarps);
    }
    for (int i = 0; i < 2; ++i) {
      dev::mbar_init(&B.p_full[i], kRowWarps);
      dev::mbar_init(&B.o_full[i], 1);
    }
    // the Q tile: one TMA transaction (the V loader), or in the shared-prefix
    // mode, whose rows are gathered member by member, one arrival per row warp
    dev::mbar_init(B.q_full, PFX ? kRowWarps : 1);
    dev::mbar_init(B.q_free, 1);
    dev::mbar_init(B.o_free, kRowWarps);
    dev::mbar_init(B.done, 2);
    for (int i = 0; i < kUQ; ++i) {
      dev::mbar_init(&B.uq_full[i], 1);
      dev::mbar_init(&B.uq_empty[i], kUQReaders);
    }
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
  // S buffers at columns 0 and 128, O at 256 (D columns), then the two P
  // buffers (64 columns each: 128 bf16 keys per row)
  const uint32_t t_s0 = tbase, t_o = tbase + 2 * kKeys, t_p = t_o + D;
  static_assert(2 * kKeys + D + 2 * (kKeys / 2) <= (int)kTmemCols, "TMEM columns");
  // Tiles are counted over all of this CTA's units ("g"): ring stages,
  // S buffers and the per-tile barriers' phases follow that count.

  if (warp == 0 || warp == kVWarp) {
    // ======================= loads: the K (warp 0) or V (last warp) ring ======
    const bool is_v = warp == kVWarp;
    const int nsr = is_v ? NSV : NSK;
    uint64_t* fullb = is_v ? B.vfull : B.kfull;
    uint64_t* emptyb = is_v ? B.vempty : B.kempty;
    uint8_t* ringb = is_v ? vring : kring;
    const CUtensorMap* tm = is_v ? &tm_v : &tm_k;
    const uint64_t pol = dev::policy_evict_last();  // the sequence's other units read the same tiles
    const int32_t oob_row = p.num_blocks * hkv * BS;  // past the pool: TMA fills zeros
    const int c = lane / C::BPT, j = lane % C::BPT;   // this lane's box: 128-byte chunk, block in tile
    // this lane's table entry for tile k of unit u (-2: past the needed
    // blocks); the check waits until the entry is used, so the load overlaps
    // a tile
    auto entry = [&](const Unit& u, int k) -> int32_t {
      const int b = k * C::BPT + j;
      return (lane < C::BOXES && b < u.nbneed) ? __ldg(p.block_tables + (int64_t)u.s * p.max_blocks + u.blk0 + b)
                                                : -2;
    };
    bool ok = true;
    int g = 0;
    int st = 0;        // g % nsr
    uint32_t lph = 0;  // (g / nsr) & 1
    int qlast = -1;    // the last unit whose Q rows this warp loaded
    const uint64_t qpol = dev::policy_evict_first();
    for (int n = 0;; ++n) {
      // queue entry n: the K loader claims the unit and publishes it, the V
      // loader reads it (a timed-out wait ends the walk, -1 for the others)
      const int slot = n % kUQ;
      int idx = -1;
      if (!is_v) {
        if (ok && lane == 0) idx = atomicAdd(p.unit_ctr, 1);
        idx = __shfl_sync(0xffffffffu, idx, 0);
        if (idx >= nunits) idx = -1;
        if (n >= kUQ && ok)
          ok = __all_sync(0xffffffffu, dev::mbar_wait(&B.uq_empty[slot], (uint32_t)(((n / kUQ) - 1) & 1), p.err));
        if (!ok) idx = -1;
        if (lane == 0) {
          uq[slot] = idx;
          dev::mbar_arrive(&B.uq_full[slot]);
        }
      } else {
        if (ok) ok = __all_sync(0xffffffffu, dev::mbar_wait(&B.uq_full[slot], (uint32_t)((n / kUQ) & 1), p.err));
        if (ok) idx = uq[slot];
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(&B.uq_empty[slot]);
      }
      __syncwarp();
      if (idx < 0) break;
      const Unit u = unit_of(idx);
      if constexpr (!PFX) {
        if (is_v) {
          // this unit's query rows, once the previous unit's S MMAs are done
          // with the Q tile: rows first + q0 .. + QB - 1 (positions past the
          // unit are other rows or zeros, masked by the row warps)
          if (n > 0 && ok) ok = __all_sync(0xffffffffu, dev::mbar_wait(B.q_free, (uint32_t)((n - 1) & 1), p.err));
          if (ok && lane == 0) {
            dev::mbar_arrive_expect_tx(B.q_full, (uint32_t)C::QBYTES);
#pragma unroll
            for (int cq = 0; cq < C::NCH; ++cq)
              dev::tma_load_3d(qs + cq * kChunk, &tm_q, cq * 64, u.h * G, u.first + u.q0, B.q_full, qpol);
            qlast = n;
          }
          __syncwarp();
          if (!ok) break;
        }
      }
      int32_t enext = entry(u, 0);
      for (int k = 0; k < u.ntiles && ok; ++k, ++g) {
        if (g >= nsr) ok = __all_sync(0xffffffffu, dev::mbar_wait(&emptyb[st], lph ^ 1u, p.err));
        if (!ok) break;
        int32_t blk = enext;
        if (k + 1 < u.ntiles) enext = entry(u, k + 1);
        int32_t y = oob_row;
        if (blk != -2) {
          if (blk < 0 || blk >= p.num_blocks) {  // bad table entry: flag, read block 0
            atomicCAS(p.err, 0, 2);
            blk = 0;
          }
          y = (blk * hkv + u.h) * BS;
        }
        if (lane == 0) dev::mbar_arrive_expect_tx(&fullb[st], (uint32_t)C::KVT);
        __syncwarp();
        if (lane < C::BOXES)
          dev::tma_load_2d(ringb + (size_t)st * C::KVT + c * kChunk + j * BS * 128, tm, c * 64, y, &fullb[st], pol);
        if (++st == nsr) {
          st = 0;
          lph ^= 1u;
        }
      }
    }
    // drain: the last stages (and Q tile) issued must land before this CTA
    // may exit
    if (lane == 0) {
      for (int d = max(0, g - nsr); d < g; ++d)
        dev::mbar_wait(&fullb[d % nsr], (uint32_t)((d / nsr) & 1), nullptr, 100000000ull);
      if (qlast >= 0) dev::mbar_wait(B.q_full, (uint32_t)(qlast & 1), nullptr, 100000000ull);
    }
    __syncwarp();
  } else if (warp == 1 || warp == kPvWarp) {
    // ============ MMA issue: S (warp 1) or PV (warp 7), one thread each =========
    const bool is_pv = warp == kPvWarp;
    if (lane == 0) {
      const uint32_t idesc_s = dev::umma_idesc_bf16(kKeys, false);
      const uint32_t idesc_o = dev::umma_idesc_bf16(D, true);
      // descriptors built once; an MMA adds its byte offset / 16 to the
      // start-address field (addresses stay below 256 KB: no carry out)
      const uint64_t dq = dev::umma_desc_sw128(dev::smem_u32(qs), 16, 1024);
      const uint64_t dk = dev::umma_desc_sw128(dev::smem_u32(kring), 16, 1024);
      const uint64_t dv = dev::umma_desc_sw128(dev::smem_u32(vring), kChunk, 1024);
      // Ring stage and phase of the next S (K ring) or the next PV (V ring),
      // advanced tile by tile: the issuing path between MMAs is kept short and
      // free of divisions, since every instruction on it delays the tensor
      // pipe's next tile.
      int ks_st = 0, vs_st = 0;
      uint32_t ks_ph = 0, vs_ph = 0;
      // S[g & 1] = Q K_g^T once K_g has landed and S[g & 1]'s last reader is done
      // `last`: the unit's last S, after which the Q tile may be reloaded
      auto issue_s = [&](int g, bool last) -> bool {
        if (!dev::mbar_wait(&B.kfull[ks_st], ks_ph, p.err)) return false;
        if (g >= 2 && !dev::mbar_wait(&B.s_free[g & 1], (uint32_t)(((g >> 1) - 1) & 1), p.err)) return false;
        dev::tc_fence_after();
        const uint64_t kb = dk + (uint64_t)ks_st * (uint64_t)(C::KVT >> 4);
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS_S; ++ks) {
          const uint64_t off = (uint64_t)(((ks >> 2) * kChunk + (ks & 3) * 32) >> 4);
          dev::umma_ss(t_s0 + (uint32_t)((g & 1) * kKeys), dq + off, kb + off, idesc_s, ks > 0 ? 1u : 0u);
        }
        dev::umma_commit(&B.s_full[g & 1]);
        dev::umma_commit(&B.kempty[ks_st]);
        if (last) dev::umma_commit(B.q_free);
        if (++ks_st == NSK) {
          ks_st = 0;
          ks_ph ^= 1u;
        }
        return true;
      };
      bool ok = true;
      int g0 = 0, nu = 0;  // first tile of the current unit; units done
      for (;; ++nu) {
        const int slot = nu % kUQ;
        int idx = -1;
        if (ok) ok = dev::mbar_wait(&B.uq_full[slot], (uint32_t)((nu / kUQ) & 1), p.err);
        if (ok) idx = uq[slot];
        dev::mbar_arrive(&B.uq_empty[slot]);
        if (idx < 0) break;
        const Unit u = unit_of(idx);
        if (!is_pv) {
          // S of every tile of the unit, each as early as its inputs allow
          // (two tiles ahead of the row warps at most: the S buffers)
          ok = dev::mbar_wait(B.q_full, (uint32_t)(nu & 1), p.err);  // this unit's Q rows are in place
          if (ok && u.ntiles == 0) dev::umma_commit(B.q_free);
          for (int k = 0; k < u.ntiles && ok; ++k) ok = issue_s(g0 + k, k + 1 == u.ntiles);
          g0 += u.ntiles;
          continue;
        }
        for (int k = 0; k < u.ntiles && ok; ++k) {
          const int g = g0 + k;
          // p_full[g & 1] and o_full[g & 1] complete once per tile of that
          // parity: tile g is their phase g >> 1
          ok = dev::mbar_wait(&B.p_full[g & 1], (uint32_t)((g >> 1) & 1), p.err) &&
               dev::mbar_wait(&B.vfull[vs_st], vs_ph, p.err);
          // the previous unit's O has been read out before this unit overwrites it
          if (ok && k == 0 && nu > 0) ok = dev::mbar_wait(B.o_free, (uint32_t)((nu - 1) & 1), p.err);
          if (!ok) break;
          dev::tc_fence_after();
          const uint64_t vb = dv + (uint64_t)vs_st * (uint64_t)(C::KVT >> 4);
#pragma unroll
          for (int ks = 0; ks < C::KSTEPS_O; ++ks) {
            // A = P from TMEM buffer g & 1 (16 keys = 8 columns per step); B =
            // V (MN-major: d contiguous, 64-wide chunks kChunk apart, 8-key row
            // groups 1024 bytes apart)
            dev::umma_ts(t_o, t_p + (uint32_t)((g & 1) * (kKeys / 2) + 8 * ks),
                         vb + (uint64_t)((ks * 16 * 128) >> 4), idesc_o, (k > 0 || ks > 0) ? 1u : 0u);
          }
          dev::umma_commit(&B.o_full[g & 1]);
          dev::umma_commit(&B.vempty[vs_st]);
          if (++vs_st == NSV) {
            vs_st = 0;
            vs_ph ^= 1u;
          }
        }
        g0 += u.ntiles;
      }
      // every MMA this thread issued has completed before TMEM may be freed
      // (the barrier takes one commit from each of the two threads)
      dev::umma_commit(B.done);
      dev::mbar_wait(B.done, 0, nullptr, 100000000ull);
    }
    __syncwarp();
  } else {
    // ======================= rows: softmax, P, output =========================
    // Thread = row r (its TMEM lane): the row's 128 keys of each tile and its
    // D columns of O.  The exponent reference of a row is taken from the
    // unit's first tile (its row max); later tiles keep it and skip the max,
    // since 2^(s * scale - ref) only has to stay finite: fp32 and bf16 share
    // an exponent range up to 2^127, so a tile whose sum of weights stays at
    // most kBig (2^64) is exact to rounding.  A tile above that (or not
    // finite) takes the slow path: its row max, a new reference, the running
    // sum and O rescaled, and the tile's weights recomputed.
    const int quarter = warp & 3;
    const int r = 32 * quarter + lane;  // this thread's row (its TMEM lane)
    const uint32_t lane_addr = (uint32_t)(32 * quarter) << 16;
    bool ok = true;
    auto wait_ok = [&](uint64_t* bar, uint32_t parity) {
      if (ok) ok = __all_sync(0xffffffffu, dev::mbar_wait(bar, parity, p.err));
    };
    // the row's scores of a tile, keys past `lim` (or all, for a row past the
    // unit) set to -inf
    auto load_s = [&](uint32_t ts, float (&sv)[kKeys], bool whole, int lim, bool valid) {
      uint32_t w[kKeys];
      dev::tmem_ld(ts, w);
#pragma unroll
      for (int i = 0; i < kKeys; ++i) sv[i] = __uint_as_float(w[i]);
      if (!whole) {  // only the tiles at a row's causal or context end
#pragma unroll
        for (int i = 0; i < kKeys; ++i) sv[i] = (valid && i < lim) ? sv[i] : -INFINITY;
      }
    };
    // the row's max score times the scale (the scale is positive)
    auto row_max = [&](const float (&sv)[kKeys]) {
      float mp[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mp[i] = sv[i];
#pragma unroll
      for (int i = 8; i < kKeys; i += 2) mp[(i >> 1) & 7] = dev::max3(mp[(i >> 1) & 7], sv[i], sv[i + 1]);
      return dev::max3(dev::max3(mp[0], mp[1], mp[2]), dev::max3(mp[3], mp[4], mp[5]), fmaxf(mp[6], mp[7])) *
             p.scale_log2;
    };
    // P = 2^(s * scale - ref) as bf16 pairs, and the tile's fp32 sum of them
    auto weights = [&](const float (&sv)[kKeys], float ref, uint32_t (&pk)[kKeys / 2]) {
      float sp[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) sp[i] = 0.f;
#pragma unroll
      for (int i = 0; i < kKeys / 2; ++i) {
        const float a = dev::ex2(fmaf(sv[2 * i], p.scale_log2, -ref));
        const float b = dev::ex2(fmaf(sv[2 * i + 1], p.scale_log2, -ref));
        sp[i & 7] += a + b;
        pk[i] = dev::pack_bf16(a, b);
      }
      return ((sp[0] + sp[1]) + (sp[2] + sp[3])) + ((sp[4] + sp[5]) + (sp[6] + sp[7]));
    };
    int g0 = 0;
    for (int n = 0;; ++n) {
      // each row warp reads queue entry n itself
      int idx = -1;
      {
        const int slot = n % kUQ;
        wait_ok(&B.uq_full[slot], (uint32_t)((n / kUQ) & 1));
        if (ok) idx = uq[slot];
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(&B.uq_empty[slot]);
      }
      if (idx < 0) break;
      const Unit u = unit_of(idx);
      const bool valid = r < u.qn * G;
      const int pos = u.pos0 + u.q0 + r / G;  // the row's position: keys <= pos
      // the row's query: row first + q0 + r / G, or (PFX) the decode row of
      // member slot first + r / G
      const int qrow = !PFX ? u.first + u.q0 + r / G : (valid ? __ldg(p.pfx_members + u.first + r / G) : 0);
      const int64_t grow = ((int64_t)qrow * hq + (int64_t)u.h * G + r % G) * D;
      // ---- shared-prefix mode: the member's Q row into the swizzled Q tile
      // (zero for rows past the unit); the previous unit's MMAs have all
      // completed (its output was read after them)
      if constexpr (PFX) {
        const uint4* src = reinterpret_cast<const uint4*>(p.q + grow * 2);
#pragma unroll
        for (int v = 0; v < C::NCH * 8; ++v) {
          const uint4 x = valid ? __ldg(src + v) : make_uint4(0, 0, 0, 0);
          *reinterpret_cast<uint4*>(qs + (v >> 3) * kChunk + swz(r, v & 7)) = x;
        }
        asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(B.q_full);
      }
      float ref = -1e30f, lsum = 0.f;  // a row with nothing visible keeps -1e30: its weights are 0
      for (int k = 0; k < u.ntiles; ++k) {
        const int g = g0 + k;
        wait_ok(&B.s_full[g & 1], (uint32_t)((g >> 1) & 1));
        dev::tc_fence_after();
        const uint32_t ts = t_s0 + (uint32_t)((g & 1) * kKeys) + lane_addr;
        const int lim = min(pos + 1, u.seq_len) - k * kKeys;  // keys [0, lim) of the tile are visible
        const bool whole = valid && lim >= kKeys;
        float sv[kKeys];
        load_s(ts, sv, whole, lim, valid);
        if (k == 0) ref = fmaxf(ref, row_max(sv));
        uint32_t pk[kKeys / 2];
        float tsum = weights(sv, ref, pk);
        if (k > 0 && __any_sync(0xffffffffu, !(tsum <= kBig))) {
          // slow path (the S buffer is still this tile's: it is released below)
          load_s(ts, sv, whole, lim, valid);
          const float mx = row_max(sv);
          const bool move = mx > ref;
          const float alpha = move ? dev::ex2(ref - mx) : 1.f;
          if (move) {
            lsum *= alpha;
            ref = mx;
          }
          tsum = weights(sv, ref, pk);
          // O rescaled once the previous tile's PV has finished (rows that keep
          // their reference use 1)
          wait_ok(&B.o_full[(g - 1) & 1], (uint32_t)(((g - 1) >> 1) & 1));
          dev::tc_fence_after();
          uint32_t w[D];
          dev::tmem_ld(t_o + lane_addr, w);
#pragma unroll
          for (int i = 0; i < D; ++i) w[i] = __float_as_uint(__uint_as_float(w[i]) * alpha);
          dev::tmem_st(t_o + lane_addr, w);
        }
        lsum += tsum;
        // S buffer g & 1 is free for the S two tiles on
        dev::tc_fence_before();
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(&B.s_free[g & 1]);
        // P buffer g & 1 was last read by the PV of tile g - 2 (an earlier
        // unit's PVs are all done: its epilogue waited for them)
        if (k >= 2) {
          wait_ok(&B.o_full[g & 1], (uint32_t)(((g >> 1) - 1) & 1));
          dev::tc_fence_after();
        }
        // the row's 128 keys, two per column, into P buffer g & 1
        dev::tmem_st(t_p + (uint32_t)((g & 1) * (kKeys / 2)) + lane_addr, pk);
        // the tile holding the context's end: slots past it hold stale pool
        // bytes (masked scores, but 0 * NaN would poison P V): zero their V rows
        const int key0 = k * kKeys;
        const int stale0 = u.seq_len - key0, stale1 = min(kKeys, u.nbneed * BS - key0);
        if (stale0 < stale1) {
          wait_ok(&B.vfull[g % NSV], (uint32_t)((g / NSV) & 1));
          uint8_t* vt = vring + (size_t)(g % NSV) * C::KVT;
          const int units = (stale1 - stale0) * C::NCH * 8;
          for (int i = tid - 64; i < units; i += 32 * kRowWarps) {
            const int key = stale0 + i / (C::NCH * 8), rest = i % (C::NCH * 8);
            *reinterpret_cast<uint4*>(vt + (rest >> 3) * kChunk + key * 128 + (rest & 7) * 16) =
                make_uint4(0, 0, 0, 0);
          }
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        dev::tc_fence_before();
        __syncwarp();
        if (lane == 0) dev::mbar_arrive(&B.p_full[g & 1]);
      }
      // ---- O / sum -> the output row; then O is free ----
      if (u.ntiles > 0) {
        wait_ok(&B.o_full[(g0 + u.ntiles - 1) & 1], (uint32_t)(((g0 + u.ntiles - 1) >> 1) & 1));
        dev::tc_fence_after();
        uint32_t w[D];
        dev::tmem_ld(t_o + lane_addr, w);
        if constexpr (PFX) {
          // partial row of member slot first + r / G, q head h * G + r % G:
          // (reference, sum) and the unnormalised O
          const int64_t prow =
              ((int64_t)u.chunk * p.num_members + u.first + r / G) * hq + (int64_t)u.h * G + r % G;
          if (valid && ok) *reinterpret_cast<float2*>(p.pfx_ml + prow * 2) = make_float2(ref, lsum);
          float4* dst = reinterpret_cast<float4*>(p.pfx_o + prow * D);
          if (valid && ok) {
#pragma unroll
            for (int uu = 0; uu < D / 4; ++uu)
              dst[uu] = make_float4(__uint_as_float(w[4 * uu]), __uint_as_float(w[4 * uu + 1]),
                                    __uint_as_float(w[4 * uu + 2]), __uint_as_float(w[4 * uu + 3]));
          }
        } else {
          const float inv = valid ? 1.f / lsum : 0.f;
          uint4* dst = reinterpret_cast<uint4*>(p.out + grow * 2);
          if (valid && ok) {
#pragma unroll
            for (int uu = 0; uu < D / 8; ++uu) {
              uint32_t pq[4];
#pragma unroll
              for (int e = 0; e < 4; ++e)
                pq[e] = dev::pack_bf16(__uint_as_float(w[8 * uu + 2 * e]) * inv,
                                       __uint_as_float(w[8 * uu + 2 * e + 1]) * inv);
              dst[uu] = make_uint4(pq[0], pq[1], pq[2], pq[3]);
            }
          }
        }
      }
      dev::tc_fence_before();
      __syncwarp();
      if (lane == 0) dev::mbar_arrive(B.o_free);
      g0 += u.ntiles;
    }
  }

  // ---- free TMEM once every warp is past its last tcgen05 access ----
  dev::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    dev::tc_fence_after();
    dev::tmem_dealloc(tbase, kTmemCols);
  }
  finish_queue();
}

template <int D, int BS, bool PFX = false>
cudaError_t launch_u(const PrefillParams& p, const CUtensorMap& tm_k, const CUtensorMap& tm_v, const CUtensorMap& tm_q,
                     int grid,
                     cudaStream_t stream) {
  using C = U<D, BS>;
  const ULayout L = u_layout(C::QBYTES, C::KVT, p.nstages, p.nstages_v, p.rows.num_seqs);
  auto kern = prefill_umma_kernel<D, BS, PFX>;
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
  return cudaLaunchKernelEx(&cfg, kern, tm_k, tm_v, tm_q, p);
}

}  // namespace

bool prefill_umma_supported(int kv, int q, int head_dim, int block_size, int group) {
  return kv == kBF16 && q == kBF16 && (head_dim == 64 || head_dim == 128) && (block_size == 16 || block_size == 32) &&
         group >= 1 && group <= 32 && (kRows % group) == 0;
}

cudaError_t launch_prefill_umma(const PrefillParams& p_in, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                                const CUtensorMap& tm_q, int head_dim, int block_size, int num_tokens, int num_sms, cudaStream_t stream) {
  PrefillParams p = p_in;
  const int nch = head_dim / 64;
  const int qbytes = nch * kChunk, kvt = nch * kChunk;
  const int fixed = (int)u_layout(qbytes, kvt, 0, 0, p.rows.num_seqs).total;
  const int nbuf = (kSmemOptIn - kStaticSmem - fixed) / (kvt + 16);  // K and V stages that fit
  const int nsk = min(4, nbuf / 2), nsv = min(4, nbuf - nbuf / 2);
  if (nsk < 2 || nsv < 2) return cudaErrorNotSupported;  // too many sequences for the unit table: caller falls back
  p.nstages = nsk;
  p.nstages_v = nsv;
  const int qb = kRows / p.group;
  const int64_t bound = ((int64_t)num_tokens / qb + p.rows.num_seqs) * p.num_kv_heads;  // units, at most
  if (bound <= 0) return cudaSuccess;
  const int64_t grid = bound < num_sms ? bound : num_sms;  // one persistent CTA per SM
  if (head_dim == 128 && block_size == 16) return launch_u<128, 16>(p, tm_k, tm_v, tm_q, (int)grid, stream);
  if (head_dim == 128 && block_size == 32) return launch_u<128, 32>(p, tm_k, tm_v, tm_q, (int)grid, stream);
  if (head_dim == 64 && block_size == 16) return launch_u<64, 16>(p, tm_k, tm_v, tm_q, (int)grid, stream);
  if (head_dim == 64 && block_size == 32) return launch_u<64, 32>(p, tm_k, tm_v, tm_q, (int)grid, stream);
  return cudaErrorNotSupported;
}

cudaError_t launch_prefix_umma(const PrefillParams& p_in, const CUtensorMap& tm_k, const CUtensorMap& tm_v,
                               int head_dim, int block_size, int num_sms, cudaStream_t stream) {
  PrefillParams p = p_in;
  const int nch = head_dim / 64;
  const int qbytes = nch * kChunk, kvt = nch * kChunk;
  const int fixed = (int)u_layout(qbytes, kvt, 0, 0, p.rows.num_seqs).total;
  const int nbuf = (kSmemOptIn - kStaticSmem - fixed) / (kvt + 16);
  const int nsk = min(4, nbuf / 2), nsv = min(4, nbuf - nbuf / 2);
  if (nsk < 2 || nsv < 2) return cudaErrorNotSupported;
  p.nstages = nsk;
  p.nstages_v = nsv;
  // units: at most (member tiles) x (chunks) x kv heads; the exact count is
  // the kernel's, CTAs past it return at once
  const int qb = kRows / p.group;
  const int64_t chunks = ((int64_t)p.max_blocks * block_size + p.chunk_keys - 1) / p.chunk_keys;
  const int64_t bound = ((int64_t)p.num_members / qb + p.rows.num_seqs) * chunks * p.num_kv_heads;
  if (bound <= 0) return cudaSuccess;
  const int64_t grid = bound < num_sms ? bound : num_sms;
  if (head_dim == 128 && block_size == 16) return launch_u<128, 16, true>(p, tm_k, tm_v, tm_k, (int)grid, stream);
  if (head_dim == 128 && block_size == 32) return launch_u<128, 32, true>(p, tm_k, tm_v, tm_k, (int)grid, stream);
  if (head_dim == 64 && block_size == 16) return launch_u<64, 16, true>(p, tm_k, tm_v, tm_k, (int)grid, stream);
  if (head_dim == 64 && block_size == 32) return launch_u<64, 32, true>(p, tm_k, tm_v, tm_k, (int)grid, stream);
  return cudaErrorNotSupported;
}

}  // namespace pa
