// Public entry points of libpa.so (declared in include/pa.h): argument
// checks, path selection, tensor-map encoding, launches.  Host code only.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "pa.h"
#include "pa_error.h"
#include "pa_kernels.h"

namespace pa {

static thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

void clear_error() { g_err.clear(); }

namespace {

int elem_bytes(int dt) { return dt == kF32 ? 4 : dt == kBF16 ? 2 : dt == kFP8 ? 1 : 0; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_desc(const pa_cache_desc* d, const char* who) {
  if (!d) return fail(PA_ERR_INVALID_ARG, "%s: desc is NULL", who);
  if (d->num_blocks <= 0 || d->num_kv_heads <= 0 || d->num_q_heads <= 0 || d->head_dim <= 0 ||
      d->block_size <= 0)
    return fail(PA_ERR_INVALID_ARG, "%s: non-positive size in desc", who);
  if (d->num_q_heads % d->num_kv_heads)
    return fail(PA_ERR_INVALID_ARG, "%s: num_q_heads %d not a multiple of num_kv_heads %d", who,
                d->num_q_heads, d->num_kv_heads);
  if (elem_bytes(d->kv_dtype) == 0 || (d->q_dtype != kF32 && d->q_dtype != kBF16))
    return fail(PA_ERR_INVALID_ARG, "%s: bad dtype (kv %d, q %d)", who, d->kv_dtype, d->q_dtype);
  if (d->block_size != 16 && d->block_size != 32)
    return fail(PA_ERR_UNSUPPORTED, "%s: block_size %d (built: 16, 32)", who, d->block_size);
  if (d->head_dim != 64 && d->head_dim != 128)
    return fail(PA_ERR_UNSUPPORTED, "%s: head_dim %d (built: 64, 128)", who, d->head_dim);
  if (d->kv_dtype == kFP8) {
    // per-tensor scales must be usable wherever per-head ones are not given
    if (!d->k_head_scales && !(std::isfinite(d->k_scale) && d->k_scale > 0.f))
      return fail(PA_ERR_INVALID_ARG, "%s: e4m3 cache needs a positive finite k_scale or k_head_scales", who);
    if (!d->v_head_scales && !(std::isfinite(d->v_scale) && d->v_scale > 0.f))
      return fail(PA_ERR_INVALID_ARG, "%s: e4m3 cache needs a positive finite v_scale or v_head_scales", who);
    if (!aligned(d->k_head_scales, 4) || !aligned(d->v_head_scales, 4))
      return fail(PA_ERR_INVALID_ARG, "%s: misaligned head scales", who);
  }
  if ((int64_t)d->num_blocks * d->num_kv_heads * d->block_size >= (int64_t)INT32_MAX)
    return fail(PA_ERR_UNSUPPORTED, "%s: pool rows exceed 2^31", who);
  return PA_OK;
}

int num_sms(int* out) {
  static std::atomic<int> cached[64];  // per device, 0 = not yet queried
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess && dev < 64 && (*out = cached[dev].load(std::memory_order_relaxed)) > 0) return PA_OK;
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(out, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return fail(PA_ERR_CUDA, "cannot query the device: %s", cudaGetErrorString(e));
  if (dev < 64) cached[dev].store(*out, std::memory_order_relaxed);
  return PA_OK;
}

// The tensor-core decode covers bf16 queries over a bf16 or e4m3 pool with a
// GQA group of 2..8 (a dense group x keys contraction), head_dim 64/128 for
// bf16 and 128 for e4m3.
bool use_tc(const pa_cache_desc* d) {
  const int g = d->num_q_heads / d->num_kv_heads;
  if (d->q_dtype != kBF16 || g < 2 || g > 8) return false;
  if (d->kv_dtype == kBF16) return d->head_dim == 64 || d->head_dim == 128;
  if (d->kv_dtype == kFP8) return d->head_dim == 128;
  return false;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// 2-D map over a token-major pool viewed as rows of head_dim elements; one
// box is [block_size rows][128 bytes] with 128-byte swizzle.
int encode_kv_map(CUtensorMap* m, const void* base, int dt, const pa_cache_desc* d);

// Encoded maps of recently used pools (a pool is normally reused every step):
// a small table keyed by everything the encoding depends on.
int make_kv_map(CUtensorMap* m, const void* base, int dt, const pa_cache_desc* d) {
  struct Entry {
    const void* base;
    int dt, nb, hkv, bs, hd;
    CUtensorMap map;
  };
  static Entry cache[16];
  static int used = 0, next = 0;
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    for (int i = 0; i < used; ++i) {
      const Entry& e = cache[i];
      if (e.base == base && e.dt == dt && e.nb == d->num_blocks && e.hkv == d->num_kv_heads &&
          e.bs == d->block_size && e.hd == d->head_dim) {
        *m = e.map;
        return PA_OK;
      }
    }
  }
  int rc = encode_kv_map(m, base, dt, d);
  if (rc) return rc;
  std::lock_guard<std::mutex> lock(mu);
  Entry& e = cache[next];
  e = Entry{base, dt, d->num_blocks, d->num_kv_heads, d->block_size, d->head_dim, *m};
  next = (next + 1) % 16;
  if (used < 16) ++used;
  return PA_OK;
}

int encode_kv_map(CUtensorMap* m, const void* base, int dt, const pa_cache_desc* d) {
  auto enc = encode_fn();
  if (!enc) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const int eb = elem_bytes(dt);
  cuuint64_t dims[2] = {(cuuint64_t)d->head_dim, (cuuint64_t)d->num_blocks * d->num_kv_heads * d->block_size};
  cuuint64_t strides[1] = {(cuuint64_t)d->head_dim * eb};
  cuuint32_t box[2] = {(cuuint32_t)(128 / eb), (cuuint32_t)d->block_size};
  cuuint32_t estr[2] = {1, 1};
  // the row stride must step over a whole row and stay a multiple of 16
  // bytes: a map whose strides overlap or shrink is refused before encoding
  if (strides[0] < dims[0] * eb || strides[0] % 16 != 0)
    return fail(PA_ERR_INVALID_ARG, "tensor map: row stride %llu bytes for %llu-byte rows",
                (unsigned long long)strides[0], (unsigned long long)(dims[0] * eb));
  CUresult r = enc(m, dt == kBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return PA_OK;
}

// 3-D map over the queries [tokens][Hq][D] (bf16) for the tcgen05 prompt-row
// kernel: a box is [128 / G tokens][G heads][64 elements], 128-byte swizzle,
// so one box fills one 64-column chunk of a unit's Q tile in row order
// (position-major, group head minor).
int encode_q_map(CUtensorMap* m, const void* q, int num_tokens, const pa_cache_desc* d) {
  auto enc = encode_fn();
  if (!enc) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable");
  const int group = d->num_q_heads / d->num_kv_heads;
  cuuint64_t dims[3] = {(cuuint64_t)d->head_dim, (cuuint64_t)d->num_q_heads, (cuuint64_t)num_tokens};
  // each stride steps over the whole previous dimension: rows do not overlap
  cuuint64_t strides[2] = {(cuuint64_t)d->head_dim * 2, (cuuint64_t)d->num_q_heads * d->head_dim * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)group, (cuuint32_t)(128 / group)};
  cuuint32_t estr[3] = {1, 1, 1};
  if (!aligned(q, 16)) return fail(PA_ERR_INVALID_ARG, "q must be 16-byte aligned");
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(PA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return PA_OK;
}

int cuda_status(cudaError_t e, const char* who) {
  if (e == cudaSuccess) return PA_OK;
  return fail(PA_ERR_CUDA, "%s: %s", who, cudaGetErrorString(e));
}

struct WsCarve {
  DecodeWorkspace ws;
  size_t bytes;
};

WsCarve carve(void* base, int num_seqs, int num_kv_heads, int group, int head_dim, int sms) {
  WsCarve c;
  uint8_t* b = static_cast<uint8_t*>(base);
  const size_t P = (size_t)decode_tc_workers(sms);
  size_t off = 0;
  c.ws.err = reinterpret_cast<int32_t*>(b + off);
  off += 256;
  c.ws.cnt = reinterpret_cast<unsigned int*>(b + off);
  off += ((size_t)num_seqs * num_kv_heads * 4 + 255) / 256 * 256;
  c.ws.ml = reinterpret_cast<float*>(b + off);
  off += (P * group * 2 * 4 + 255) / 256 * 256;
  c.ws.o = reinterpret_cast<float*>(b + off);
  off += P * group * head_dim * 4;
  c.bytes = off;
  return c;
}

// pa_decode_prefix runs the shared prefixes on the tcgen05 kernel: a bf16
// pool and queries, a GQA group that the tensor-core decode takes and that
// divides the kernel's 128 rows.
bool prefix_path(const pa_cache_desc* d) {
  return use_tc(d) && d->kv_dtype == kBF16 &&
         prefill_umma_supported(d->kv_dtype, d->q_dtype, d->head_dim, d->block_size, d->num_q_heads / d->num_kv_heads);
}

// Bytes of the prefix partials after pa_decode's own scratch.
int prefix_chunk_keys_for(const pa_cache_desc* d, int32_t num_members, int32_t max_prefix_blocks) {
  return prefix_chunk_keys(max_prefix_blocks, d->block_size, num_members, d->num_q_heads / d->num_kv_heads,
                           d->num_kv_heads);
}

size_t prefix_partial_bytes(const pa_cache_desc* d, int32_t num_members, int32_t max_prefix_blocks, size_t* ml_bytes) {
  const size_t ck = (size_t)prefix_chunk_keys_for(d, num_members, max_prefix_blocks);
  const size_t chunks = ((size_t)max_prefix_blocks * d->block_size + ck - 1) / ck;
  const size_t rows = chunks * (size_t)num_members * d->num_q_heads;
  *ml_bytes = (rows * 2 * 4 + 255) / 256 * 256;
  return *ml_bytes + rows * d->head_dim * 4;
}

// Shared prefixes of a pa_decode_prefix call, for the decode kernel.
struct PrefixArgs {
  const int32_t* seq_prefix;
  const int32_t* seq_slot;
  const int32_t* prefix_blocks;
  const float* ml;
  const float* o;
  int32_t num_members;
  int32_t chunk_keys;
};

// The new tokens' rows that pa_decode_fused writes in the decode launch.
struct FusedWrite {
  const void* k_new;
  const void* v_new;
  void* k_pool;
  void* v_pool;
};

// Decode rows (q_len == 1) of a batch on the tensor-core path; qsl may be null.
int run_decode_tc(const pa_cache_desc* d, const void* q, const void* k_cache, const void* v_cache,
                  const int32_t* block_tables, int32_t max_blocks, const int32_t* seq_lens, const int32_t* qsl,
                  int32_t num_seqs, int32_t num_rows, float scale, void* out, void* workspace,
                  size_t workspace_bytes, cudaStream_t stream, const char* who, const FusedWrite* fw = nullptr,
                  const PrefixArgs* pa = nullptr) {
  int sms = 0;
  int rc = num_sms(&sms);
  if (rc) return rc;
  const int group = d->num_q_heads / d->num_kv_heads;
  WsCarve c = carve(workspace, num_seqs, d->num_kv_heads, group, d->head_dim, sms);
  if (workspace_bytes < c.bytes)
    return fail(PA_ERR_INVALID_ARG, "%s: workspace %zu < %zu bytes", who, workspace_bytes, c.bytes);
  CUtensorMap tm_k, tm_v;
  if ((rc = make_kv_map(&tm_k, k_cache, d->kv_dtype, d))) return rc;
  if (d->kv_dtype == kBF16) {
    if ((rc = make_kv_map(&tm_v, v_cache, d->kv_dtype, d))) return rc;
  } else {
    tm_v = tm_k;  // e4m3 V tiles are contiguous and come by bulk copy
  }
  DecodeParams p = {};
  p.q = static_cast<const uint8_t*>(q);
  p.out = static_cast<uint8_t*>(out);
  p.v_cache = static_cast<const uint8_t*>(v_cache);
  p.block_tables = block_tables;
  p.max_blocks = max_blocks;
  p.rows.seq_lens = seq_lens;
  p.rows.qsl = qsl;
  p.rows.num_seqs = num_seqs;
  p.rows.num_rows = num_rows;
  p.num_q_heads = d->num_q_heads;
  p.num_kv_heads = d->num_kv_heads;
  p.num_blocks = d->num_blocks;
  p.group = group;
  const float log2e = 1.4426950408889634f;
  if (d->kv_dtype == kFP8) {
    // f16 operands hold the stored e4m3 values; the dequantisation scales
    // fold into the softmax scale and the output scale (per piece, when
    // they are per kv head)
    p.k_head = d->k_head_scales;
    p.v_head = d->v_head_scales;
    p.scale_log2 = scale * log2e * (p.k_head ? 1.f : d->k_scale);
    p.out_scale = p.v_head ? 1.f : d->v_scale;
    p.k_scale_w = d->k_scale;
    p.v_scale_w = d->v_scale;
  } else {
    p.scale_log2 = scale * log2e;
    p.out_scale = 1.f;
  }
  p.ws = c.ws;
  if (pa) {
    p.pfx_of = pa->seq_prefix;
    p.pfx_slot = pa->seq_slot;
    p.pfx_blocks = pa->prefix_blocks;
    p.pfx_ml = pa->ml;
    p.pfx_o = pa->o;
    p.pfx_members = pa->num_members;
    p.pfx_chunk_blocks = pa->chunk_keys / d->block_size;
  }
  if (fw) {
    p.k_new = static_cast<const uint8_t*>(fw->k_new);
    p.v_new = static_cast<const uint8_t*>(fw->v_new);
    p.k_pool = static_cast<uint8_t*>(fw->k_pool);
    p.v_pool = static_cast<uint8_t*>(fw->v_pool);
  }
  cudaError_t e = launch_decode_tc(p, tm_k, tm_v, d->kv_dtype, d->head_dim, d->block_size, sms, stream);
  if (e == cudaErrorNotSupported) return fail(PA_ERR_UNSUPPORTED, "%s: shape not built for the tensor-core path", who);
  return cuda_status(e, who);
}

int run_simt(const pa_cache_desc* d, const void* q, const void* k_cache, const void* v_cache,
             const int32_t* block_tables, int32_t max_blocks, const int32_t* seq_lens, const int32_t* qsl,
             int32_t num_seqs, int32_t num_rows, int only_multi_row, float scale, void* out, void* workspace,
             cudaStream_t stream, const char* who) {
  SimtParams p = {};
  p.num_blocks = d->num_blocks;
  p.err = static_cast<int32_t*>(workspace);
  p.q = static_cast<const uint8_t*>(q);
  p.out = static_cast<uint8_t*>(out);
  p.k_cache = static_cast<const uint8_t*>(k_cache);
  p.v_cache = static_cast<const uint8_t*>(v_cache);
  p.block_tables = block_tables;
  p.max_blocks = max_blocks;
  p.rows.seq_lens = seq_lens;
  p.rows.qsl = qsl;
  p.rows.num_seqs = num_seqs;
  p.rows.num_rows = num_rows;
  p.num_q_heads = d->num_q_heads;
  p.num_kv_heads = d->num_kv_heads;
  p.head_dim = d->head_dim;
  p.block_size = d->block_size;
  p.scale = scale;
  p.k_scale = d->k_scale;
  p.v_scale = d->v_scale;
  if (d->kv_dtype == kFP8) {
    p.k_head = d->k_head_scales;
    p.v_head = d->v_head_scales;
  }
  p.only_multi_row = only_multi_row;
  cudaError_t e = launch_attn_simt(p, d->q_dtype, d->kv_dtype, stream);
  if (e == cudaErrorNotSupported)
    return fail(PA_ERR_UNSUPPORTED, "%s: q dtype %d with kv dtype %d", who, d->q_dtype, d->kv_dtype);
  return cuda_status(e, who);
}

}  // namespace

int check_attn_args(const pa_cache_desc* d, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int32_t max_blocks, const int32_t* seq_lens, int32_t num_seqs,
                    void* out, void* workspace, const char* who) {
  int rc = check_desc(d, who);
  if (rc) return rc;
  if (num_seqs < 0 || max_blocks < 0) return fail(PA_ERR_INVALID_ARG, "%s: negative size", who);
  if (num_seqs == 0) return PA_OK;
  if (!q || !k_cache || !v_cache || !block_tables || !seq_lens || !out || !workspace)
    return fail(PA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(block_tables, 4) || !aligned(seq_lens, 4) || !aligned(workspace, 256))
    return fail(PA_ERR_INVALID_ARG, "%s: misaligned pointer", who);
  if (num_seqs > 16384) return fail(PA_ERR_UNSUPPORTED, "%s: more than 16384 sequences per call", who);
  // (sequence, kv head, block) tiles are indexed with 32-bit integers
  if ((int64_t)num_seqs * max_blocks * d->num_kv_heads >= (int64_t)INT32_MAX)
    return fail(PA_ERR_UNSUPPORTED, "%s: num_seqs * max_blocks_per_seq * num_kv_heads reaches 2^31", who);
  return PA_OK;
}

}  // namespace pa

using namespace pa;

extern "C" {

const char* pa_last_error(void) { return g_err.c_str(); }

const char* pa_version(void) { return "pa 0.1.0 (sm_100a)"; }

size_t pa_block_bytes(const pa_cache_desc* d) {
  if (!d || elem_bytes(d->kv_dtype) == 0 || d->block_size <= 0 || d->num_kv_heads <= 0 || d->head_dim <= 0)
    return 0;
  return 2ull * d->block_size * d->num_kv_heads * d->head_dim * elem_bytes(d->kv_dtype);
}

int pa_cache_write(const pa_cache_desc* d, const void* k_new, const void* v_new, const int64_t* slot_mapping,
                   int32_t num_tokens, void* k_cache, void* v_cache, void* stream) {
  clear_error();
  int rc = check_desc(d, "pa_cache_write");
  if (rc) return rc;
  if (num_tokens < 0) return fail(PA_ERR_INVALID_ARG, "pa_cache_write: num_tokens < 0");
  if (num_tokens == 0) return PA_OK;
  if (!k_new || !v_new || !slot_mapping || !k_cache || !v_cache)
    return fail(PA_ERR_INVALID_ARG, "pa_cache_write: NULL pointer");
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(k_cache, 16) || !aligned(v_cache, 16) ||
      !aligned(slot_mapping, 8))
    return fail(PA_ERR_INVALID_ARG, "pa_cache_write: misaligned pointer");
  if (d->kv_dtype != kFP8 && d->kv_dtype != d->q_dtype)
    return fail(PA_ERR_UNSUPPORTED, "pa_cache_write: q dtype %d into kv dtype %d", d->q_dtype, d->kv_dtype);
  CacheWriteParams p = {};
  p.k_new = static_cast<const uint8_t*>(k_new);
  p.v_new = static_cast<const uint8_t*>(v_new);
  p.slots = slot_mapping;
  p.k_cache = static_cast<uint8_t*>(k_cache);
  p.v_cache = static_cast<uint8_t*>(v_cache);
  p.num_tokens = num_tokens;
  p.num_kv_heads = d->num_kv_heads;
  p.head_dim = d->head_dim;
  p.block_size = d->block_size;
  p.num_slots = (int64_t)d->num_blocks * d->block_size;
  p.k_scale = d->k_scale;
  p.v_scale = d->v_scale;
  if (d->kv_dtype == kFP8) {
    p.k_head = d->k_head_scales;
    p.v_head = d->v_head_scales;
  }
  return cuda_status(launch_cache_write(p, d->q_dtype, d->kv_dtype, static_cast<cudaStream_t>(stream)),
                     "pa_cache_write");
}

int pa_copy_blocks(const pa_cache_desc* d, const int32_t* src, const int32_t* dst, int32_t n, void* k_cache,
                   void* v_cache, void* stream) {
  clear_error();
  int rc = check_desc(d, "pa_copy_blocks");
  if (rc) return rc;
  if (n < 0) return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: n < 0");
  if (n == 0) return PA_OK;
  if (!src || !dst || !k_cache || !v_cache) return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: NULL pointer");
  if (!aligned(src, 4) || !aligned(dst, 4) || !aligned(k_cache, 16) || !aligned(v_cache, 16))
    return fail(PA_ERR_INVALID_ARG, "pa_copy_blocks: misaligned pointer");
  int sms = 0;
  if ((rc = num_sms(&sms))) return rc;
  CopyBlocksParams p = {};
  p.src = src;
  p.dst = dst;
  p.n = n;
  p.num_blocks = d->num_blocks;
  p.block_bytes = (int64_t)(pa_block_bytes(d) / 2);
  p.k_cache = static_cast<uint8_t*>(k_cache);
  p.v_cache = static_cast<uint8_t*>(v_cache);
  return cuda_status(launch_copy_blocks(p, sms, static_cast<cudaStream_t>(stream)), "pa_copy_blocks");
}

size_t pa_decode_workspace_size(const pa_cache_desc* d, int32_t num_seqs) {
  clear_error();
  if (check_desc(d, "pa_decode_workspace_size") || num_seqs < 0) return 0;
  if (!use_tc(d)) return 256;
  int sms = 0;
  if (num_sms(&sms)) return 0;
  return decode_tc_workspace_bytes(num_seqs, d->num_kv_heads, d->num_q_heads / d->num_kv_heads, d->head_dim, sms);
}

int pa_decode(const pa_cache_desc* d, const void* q, const void* k_cache, const void* v_cache,
              const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens, int32_t num_seqs,
              float scale, void* out, void* workspace, size_t workspace_bytes, void* stream) {
  clear_error();
  int rc = check_attn_args(d, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, num_seqs, out,
                           workspace, "pa_decode");
  if (rc || num_seqs == 0) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (use_tc(d))
    return run_decode_tc(d, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, nullptr, num_seqs,
                         num_seqs, scale, out, workspace, workspace_bytes, st, "pa_decode");
  if (workspace_bytes < 256) return fail(PA_ERR_INVALID_ARG, "pa_decode: workspace < 256 bytes");
  return run_simt(d, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, nullptr, num_seqs, num_seqs,
                  0, scale, out, workspace, st, "pa_decode");
}

int pa_decode_fused(const pa_cache_desc* d, const void* q, const void* k_new, const void* v_new, void* k_cache,
                    void* v_cache, const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                    int32_t num_seqs, float scale, void* out, void* workspace, size_t workspace_bytes,
                    void* stream) {
  clear_error();
  const char* who = "pa_decode_fused";
  int rc = check_attn_args(d, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, num_seqs, out,
                           workspace, who);
  if (rc || num_seqs == 0) return rc;
  if (!k_new || !v_new) return fail(PA_ERR_INVALID_ARG, "%s: NULL pointer", who);
  if (!aligned(k_new, 16) || !aligned(v_new, 16)) return fail(PA_ERR_INVALID_ARG, "%s: misaligned pointer", who);
  if (!use_tc(d))
    return fail(PA_ERR_UNSUPPORTED, "%s: the write is fused only into the tensor-core decode (bf16 queries, "
                "GQA group 2..8); use pa_cache_write + pa_decode", who);
  const FusedWrite fw{k_new, v_new, k_cache, v_cache};
  return run_decode_tc(d, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, nullptr, num_seqs, num_seqs,
                       scale, out, workspace, workspace_bytes, static_cast<cudaStream_t>(stream), who, &fw);
}

size_t pa_decode_prefix_workspace_size(const pa_cache_desc* d, int32_t num_seqs, int32_t num_members,
                                       int32_t max_prefix_blocks) {
  const size_t base = pa_decode_workspace_size(d, num_seqs);
  if (base == 0 || num_members < 0 || max_prefix_blocks < 0) return 0;
  if (!prefix_path(d)) return base;
  size_t ml_bytes = 0;
  return base + prefix_partial_bytes(d, num_members, max_prefix_blocks, &ml_bytes);
}

int pa_decode_prefix(const pa_cache_desc* d, const void* q, const void* k_cache, const void* v_cache,
                     const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                     int32_t num_seqs, const int32_t* prefix_start, const int32_t* prefix_members,
                     const int32_t* prefix_blocks, const int32_t* seq_prefix, const int32_t* seq_slot,
                     int32_t num_prefixes, int32_t num_members, int32_t max_prefix_blocks, float scale, void* out,
                     void* workspace, size_t workspace_bytes, void* stream) {
  clear_error();
  const char* who = "pa_decode_prefix";
  int rc = check_attn_args(d, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, num_seqs, out,
                           workspace, who);
  if (rc || num_seqs == 0) return rc;
  if (num_prefixes < 0 || num_members < 0 || max_prefix_blocks < 0 || num_members > num_seqs ||
      max_prefix_blocks > max_blocks_per_seq)
    return fail(PA_ERR_INVALID_ARG, "%s: bad prefix sizes", who);
  if (num_prefixes == 0 || !prefix_path(d))
    return pa_decode(d, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, num_seqs, scale, out,
                     workspace, workspace_bytes, stream);
  if (!prefix_start || !prefix_members || !prefix_blocks || !seq_prefix || !seq_slot)
    return fail(PA_ERR_INVALID_ARG, "%s: NULL prefix array", who);
  if (!aligned(prefix_start, 4) || !aligned(prefix_members, 4) || !aligned(prefix_blocks, 4) ||
      !aligned(seq_prefix, 4) || !aligned(seq_slot, 4))
    return fail(PA_ERR_INVALID_ARG, "%s: misaligned prefix array", who);
  const size_t base = pa_decode_workspace_size(d, num_seqs);
  size_t ml_bytes = 0;
  const size_t need = base + prefix_partial_bytes(d, num_members, max_prefix_blocks, &ml_bytes);
  if (base == 0 || workspace_bytes < need)
    return fail(PA_ERR_INVALID_ARG, "%s: workspace %zu < %zu bytes", who, workspace_bytes, need);
  int sms = 0;
  if ((rc = num_sms(&sms))) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* pml = reinterpret_cast<float*>(ws + base);
  float* po = reinterpret_cast<float*>(ws + base + ml_bytes);
  // 1. every shared prefix once for all its members: chunk partials
  CUtensorMap tm_k, tm_v;
  if ((rc = make_kv_map(&tm_k, k_cache, d->kv_dtype, d))) return rc;
  if ((rc = make_kv_map(&tm_v, v_cache, d->kv_dtype, d))) return rc;
  PrefillParams pp = {};
  pp.q = static_cast<const uint8_t*>(q);
  pp.block_tables = block_tables;
  pp.max_blocks = max_blocks_per_seq;
  pp.rows.num_seqs = num_prefixes;
  pp.num_q_heads = d->num_q_heads;
  pp.num_kv_heads = d->num_kv_heads;
  pp.group = d->num_q_heads / d->num_kv_heads;
  pp.num_blocks = d->num_blocks;
  pp.scale_log2 = scale * 1.4426950408889634f;
  pp.err = static_cast<int32_t*>(workspace);
  pp.unit_ctr = static_cast<int32_t*>(workspace) + 2;
  pp.unit_exit = static_cast<int32_t*>(workspace) + 3;
  pp.pfx_start = prefix_start;
  pp.pfx_members = prefix_members;
  pp.pfx_blocks = prefix_blocks;
  pp.num_members = num_members;
  pp.chunk_keys = prefix_chunk_keys_for(d, num_members, max_prefix_blocks);
  pp.pfx_ml = pml;
  pp.pfx_o = po;
  cudaError_t e = launch_prefix_umma(pp, tm_k, tm_v, d->head_dim, d->block_size, sms, st);
  if (e == cudaErrorNotSupported)
    return pa_decode(d, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, num_seqs, scale, out,
                     workspace, workspace_bytes, stream);
  if ((rc = cuda_status(e, who))) return rc;
  // 2. the suffixes on the decode kernel, folding each member's chunk partials
  const PrefixArgs pa{seq_prefix, seq_slot, prefix_blocks, pml, po, num_members, pp.chunk_keys};
  return run_decode_tc(d, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, nullptr, num_seqs,
                       num_seqs, scale, out, workspace, base, st, who, nullptr, &pa);
}

size_t pa_prefill_workspace_size(const pa_cache_desc* d, int32_t num_seqs, int32_t num_tokens) {
  (void)num_tokens;
  return pa_decode_workspace_size(d, num_seqs);
}

int pa_decode_chunked_prefill(const pa_cache_desc* d, const void* q, const void* k_cache, const void* v_cache,
                              const int32_t* block_tables, int32_t max_blocks_per_seq,
                              const int32_t* query_start_loc, const int32_t* seq_lens, int32_t num_seqs,
                              int32_t num_tokens, int32_t max_q_len, float scale, void* out, void* workspace,
                              size_t workspace_bytes, void* stream) {
  clear_error();
  const char* who = "pa_decode_chunked_prefill";
  int rc = check_attn_args(d, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, num_seqs, out,
                           workspace, who);
  if (rc || num_seqs == 0) return rc;
  if (!query_start_loc || !aligned(query_start_loc, 4)) return fail(PA_ERR_INVALID_ARG, "%s: bad query_start_loc", who);
  if (num_tokens < 0 || max_q_len < 0) return fail(PA_ERR_INVALID_ARG, "%s: negative size", who);
  if (num_tokens == 0) return PA_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (use_tc(d)) {
    // decode rows on the decode kernel, prompt rows on the prefill kernel
    rc = run_decode_tc(d, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, query_start_loc,
                       num_seqs, num_tokens, scale, out, workspace, workspace_bytes, st, who);
    if (rc) return rc;
    if (max_q_len <= 1) return PA_OK;
    const int group = d->num_q_heads / d->num_kv_heads;
    const bool umma = prefill_umma_supported(d->kv_dtype, d->q_dtype, d->head_dim, d->block_size, group);
    if (umma || prefill_tc_supported(d->kv_dtype, d->q_dtype, d->head_dim, d->block_size, group)) {
      CUtensorMap tm_k, tm_v;
      if ((rc = make_kv_map(&tm_k, k_cache, d->kv_dtype, d))) return rc;
      if ((rc = make_kv_map(&tm_v, v_cache, d->kv_dtype, d))) return rc;
      PrefillParams pp = {};
      pp.q = static_cast<const uint8_t*>(q);
      pp.out = static_cast<uint8_t*>(out);
      pp.block_tables = block_tables;
      pp.max_blocks = max_blocks_per_seq;
      pp.rows.seq_lens = seq_lens;
      pp.rows.qsl = query_start_loc;
      pp.rows.num_seqs = num_seqs;
      pp.rows.num_rows = num_tokens;
      pp.num_q_heads = d->num_q_heads;
      pp.num_kv_heads = d->num_kv_heads;
      pp.group = group;
      pp.num_blocks = d->num_blocks;
      pp.scale_log2 = scale * 1.4426950408889634f;
      pp.err = static_cast<int32_t*>(workspace);
      pp.unit_ctr = static_cast<int32_t*>(workspace) + 2;
      pp.unit_exit = static_cast<int32_t*>(workspace) + 3;
      pp.after_decode = 1;  // run_decode_tc launched this step's decode just before
      cudaError_t e = cudaErrorNotSupported;
      int sms = 0;
      if ((rc = num_sms(&sms))) return rc;
      if (umma) {
        CUtensorMap tm_q;
        if ((rc = encode_q_map(&tm_q, q, num_tokens, d))) return rc;
        e = launch_prefill_umma(pp, tm_k, tm_v, tm_q, d->head_dim, d->block_size, num_tokens, sms, st);
      }
      if (e == cudaErrorNotSupported && prefill_tc_supported(d->kv_dtype, d->q_dtype, d->head_dim, d->block_size, group))
        e = launch_prefill_tc(pp, tm_k, tm_v, d->head_dim, d->block_size, num_tokens, st);
      if (e != cudaErrorNotSupported) return cuda_status(e, who);
    }
    return run_simt(d, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, query_start_loc, num_seqs,
                    num_tokens, 1, scale, out, workspace, st, who);
  }
  if (workspace_bytes < 256) return fail(PA_ERR_INVALID_ARG, "%s: workspace < 256 bytes", who);
  return run_simt(d, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, query_start_loc, num_seqs,
                  num_tokens, 0, scale, out, workspace, st, who);
}

}  // extern "C"
