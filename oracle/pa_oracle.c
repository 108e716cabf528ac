/*
 * pa_oracle.c -- plain, slow, obviously-correct CPU oracle for paged decode
 * attention (fp64).
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product (paged_kv_cache_452_b200/)
 * loads, links or calls this file; only tests/, __graft_entry__.smoke() and
 * bench.py's cpu_baseline leg do.  It shares no header, helper, table or
 * constant with the CUDA path.
 *
 * What it computes, and the passages it follows:
 *
 *  - oracle_cache_write: the "write(blocks[-1], kv)" step of the block-table
 *    snippet on "49 vLLM / PagedAttention" (section "Таблица блоков (идея
 *    пейджинга)"), with the new token's flat slot split into (physical block,
 *    offset) = (slot / block_size, slot % block_size).  fp32/bf16 caches get a
 *    byte copy; an FP8 cache gets e4m3(fp32(x) / fp32(scale)), rounded to
 *    nearest-even and saturated to +-448.  The scale is one fp32 per pool,
 *    or one per kv head (this build's reading: the pages motivate FP8 KV,
 *    "PagedAttention：KV cache 即虚拟内存…", num_gpu_blocks and the KV-bound
 *    question, halving the bytes per block, and leave the scale open).
 *
 *  - oracle_attention: attention over the keys a block table points at.  The
 *    page "PagedAttention：KV cache 即虚拟内存（block manager & 碎片）" states
 *    (section 直接答案, and the follow-up "分页改变输出或加速 kernel 吗？")
 *    that paging changes neither the output nor the compute, so the oracle is
 *    the plain definition of softmax attention, evaluated over K/V fetched one
 *    token at a time through the table: logical position j lives in physical
 *    block table[j / bs] at offset j % bs.  Straight loops, fp64 throughout,
 *    no online softmax, no blocking.
 *
 *  - Cache layout (the pages leave it open; this is the build's reading):
 *    K is [num_blocks][kv_heads][block_size][head_dim] for every dtype; V is
 *    the same for fp32/bf16 caches, and d-major [num_blocks][kv_heads]
 *    [head_dim][block_size] for e4m3 caches.  The index of element d of the
 *    token at offset o of block b, head h, is written out at each use.
 *
 *  - e4m3 encode/decode from the OCP 8-bit floating point definition (E4M3:
 *    sign, 4 exponent bits with bias 7, 3 mantissa bits, exponent field 0 is
 *    subnormal, S.1111.111 is NaN, no infinities, largest finite 448).
 *
 * The dtype codes below are this file's own: 0 = fp32, 1 = bf16, 2 = e4m3.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define ORC_F32 0
#define ORC_BF16 1
#define ORC_E4M3 2

static size_t orc_elem_bytes(int dt) { return dt == ORC_F32 ? 4 : (dt == ORC_BF16 ? 2 : 1); }

/* ---- e4m3 (OCP FP8 E4M3) ---------------------------------------------- */

double oracle_e4m3_decode(uint8_t code) {
  int s = (code >> 7) & 1;
  int e = (code >> 3) & 15;
  int m = code & 7;
  double mag;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    mag = ldexp((double)m / 8.0, -6); /* subnormal: 0.mmm * 2^(1-7) */
  else
    mag = ldexp(1.0 + (double)m / 8.0, e - 7); /* normal: 1.mmm * 2^(e-7) */
  return s ? -mag : mag;
}

/* Round to nearest representable e4m3 value, ties to the even code (mantissa
 * LSB 0); magnitudes at or above 448 saturate to 448; NaN -> S.1111.111.
 * Done by scanning the finite non-negative codes in increasing order. */
uint8_t oracle_e4m3_encode(float x) {
  uint8_t sign;
  double a;
  int c;
  if (isnan(x)) return 0x7F;
  sign = signbit(x) ? 0x80 : 0x00;
  a = fabs((double)x);
  if (a >= 448.0) return (uint8_t)(sign | 0x7E);
  for (c = 0; c < 0x7E; ++c) {
    double lo = oracle_e4m3_decode((uint8_t)c);
    double hi = oracle_e4m3_decode((uint8_t)(c + 1));
    if (a <= hi) {
      double dlo = a - lo, dhi = hi - a;
      int pick;
      if (dlo < dhi)
        pick = c;
      else if (dhi < dlo)
        pick = c + 1;
      else
        pick = (c & 1) ? c + 1 : c;
      return (uint8_t)(sign | pick);
    }
  }
  return (uint8_t)(sign | 0x7E);
}

/* ---- element load as a real number ------------------------------------- */

static float orc_load_f32(const void* p, int dt, size_t i) {
  if (dt == ORC_F32) {
    float v;
    memcpy(&v, (const char*)p + 4 * i, 4);
    return v;
  } else { /* bf16: the upper half of an fp32 */
    uint16_t b;
    uint32_t w;
    float v;
    memcpy(&b, (const char*)p + 2 * i, 2);
    w = (uint32_t)b << 16;
    memcpy(&v, &w, 4);
    return v;
  }
}

static double orc_load_cache(const void* p, int dt, size_t i, double scale) {
  if (dt == ORC_E4M3) return oracle_e4m3_decode(((const uint8_t*)p)[i]) * scale;
  return (double)orc_load_f32(p, dt, i);
}

/* ---- cache write -------------------------------------------------------- */

/* Offset of element d of the token at (block b, head h, offset o): token-major
 * [b][h][o][d], or d-major [b][h][d][o] (e4m3 V). */
static size_t orc_index(int d_major, size_t b, size_t h, size_t o, size_t d, int num_kv_heads,
                        int block_size, int head_dim) {
  if (d_major) return ((b * num_kv_heads + h) * head_dim + d) * block_size + o;
  return ((b * num_kv_heads + h) * block_size + o) * head_dim + d;
}

/* k_new, v_new: [num_tokens][num_kv_heads][head_dim] in in_dtype (fp32 or bf16).
 * k_cache, v_cache: the pools, laid out as described at the top of this file.
 * k_head_scales, v_head_scales: NULL (k_scale / v_scale for every head) or
 * one fp32 scale per kv head.
 * A negative slot is skipped.  Returns 0, or -1 if a slot is past the pool. */
int oracle_cache_write(int in_dtype, int kv_dtype, const void* k_new, const void* v_new,
                       const int64_t* slots, int num_tokens, int num_blocks, int block_size,
                       int num_kv_heads, int head_dim, float k_scale, float v_scale,
                       const float* k_head_scales, const float* v_head_scales,
                       void* k_cache, void* v_cache) {
  int t, h, d, side;
  for (t = 0; t < num_tokens; ++t) {
    int64_t slot = slots[t];
    int64_t blk, off;
    if (slot < 0) continue;
    if (slot >= (int64_t)num_blocks * block_size) return -1;
    blk = slot / block_size;
    off = slot % block_size;
    for (side = 0; side < 2; ++side) {
      const void* src = side == 0 ? k_new : v_new;
      void* dst = side == 0 ? k_cache : v_cache;
      const float* head_scales = side == 0 ? k_head_scales : v_head_scales;
      for (h = 0; h < num_kv_heads; ++h) {
        float scale = head_scales ? head_scales[h] : (side == 0 ? k_scale : v_scale);
        for (d = 0; d < head_dim; ++d) {
          size_t si = ((size_t)t * num_kv_heads + h) * head_dim + d;
          int d_major = (side == 1 && kv_dtype == ORC_E4M3);
          size_t di = orc_index(d_major, (size_t)blk, (size_t)h, (size_t)off, (size_t)d, num_kv_heads,
                                block_size, head_dim);
          if (kv_dtype == ORC_E4M3) {
            float x = orc_load_f32(src, in_dtype, si);
            float y = x / scale; /* one IEEE fp32 division */
            ((uint8_t*)dst)[di] = oracle_e4m3_encode(y);
          } else {
            size_t eb = orc_elem_bytes(kv_dtype);
            memcpy((char*)dst + eb * di, (const char*)src + eb * si, eb);
          }
        }
      }
    }
  }
  return 0;
}

/* ---- attention ---------------------------------------------------------- */

/* q:   [num_rows][num_q_heads][head_dim] fp64.
 * Row r belongs to sequence row_seq[r] and sits at position row_pos[r]; it
 * attends the keys at positions 0..row_pos[r] of that sequence (causal; a
 * decode row sits at the last position, so it attends the whole context).
 * Query head h reads KV head h / (num_q_heads / num_kv_heads).
 * block_tables: [num_seqs][max_blocks] int32.
 * An e4m3 code of kv head h dequantises to its value times k_head_scales[h]
 * (v_head_scales[h] for V), or times k_scale (v_scale) when those are NULL.
 * out: [num_rows][num_q_heads][head_dim] fp64. */
void oracle_attention(const double* q, int num_rows, const int32_t* row_seq, const int32_t* row_pos,
                      const int32_t* block_tables, int max_blocks, int kv_dtype, const void* k_cache,
                      const void* v_cache, double k_scale, double v_scale, const float* k_head_scales,
                      const float* v_head_scales, int block_size, int num_q_heads, int num_kv_heads,
                      int head_dim, double scale, double* out, int num_threads) {
  int group = num_q_heads / num_kv_heads;
  long task, ntasks = (long)num_rows * num_q_heads;
#ifdef _OPENMP
  if (num_threads > 0) omp_set_num_threads(num_threads);
#pragma omp parallel for schedule(dynamic, 1)
#endif
  for (task = 0; task < ntasks; ++task) {
    int r = (int)(task / num_q_heads);
    int h = (int)(task % num_q_heads);
    int kvh = h / group;
    double ks = k_head_scales ? (double)k_head_scales[kvh] : k_scale;
    double vs = v_head_scales ? (double)v_head_scales[kvh] : v_scale;
    int s = row_seq[r];
    int n = row_pos[r] + 1;
    const double* qv = q + ((size_t)r * num_q_heads + h) * head_dim;
    double* o = out + ((size_t)r * num_q_heads + h) * head_dim;
    double* logit = (double*)malloc(sizeof(double) * (size_t)n);
    double mx = -INFINITY, z = 0.0;
    int j, d;
    for (j = 0; j < n; ++j) {
      int32_t blk = block_tables[(size_t)s * max_blocks + j / block_size];
      int off = j % block_size;
      double dot = 0.0;
      for (d = 0; d < head_dim; ++d)
        dot += qv[d] * orc_load_cache(k_cache, kv_dtype,
                                      orc_index(0, blk, kvh, off, d, num_kv_heads, block_size, head_dim),
                                      ks);
      logit[j] = scale * dot;
      if (logit[j] > mx) mx = logit[j];
    }
    for (j = 0; j < n; ++j) z += exp(logit[j] - mx);
    for (d = 0; d < head_dim; ++d) o[d] = 0.0;
    for (j = 0; j < n; ++j) {
      int32_t blk = block_tables[(size_t)s * max_blocks + j / block_size];
      int off = j % block_size;
      double w = exp(logit[j] - mx) / z;
      for (d = 0; d < head_dim; ++d)
        o[d] += w * orc_load_cache(v_cache, kv_dtype,
                                   orc_index(kv_dtype == ORC_E4M3, blk, kvh, off, d, num_kv_heads,
                                             block_size, head_dim),
                                   vs);
    }
    free(logit);
  }
}

#ifdef _OPENMP
int oracle_max_threads(void) { return omp_get_max_threads(); }
#else
int oracle_max_threads(void) { return 1; }
#endif
