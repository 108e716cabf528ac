// pa_decode_static: pa_decode for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc: code that runs inside a captured
// CUDA graph where allocation is not allowed, an embedding whose memory
// belongs to someone else's allocator, or a hard real-time path that must
// not allocate after start-up.  For them this entry point takes the same
// inputs and outputs as pa_decode but uses a scratch area compiled into the
// library instead of a caller workspace.
//
// The scratch is one file-scope __device__ array of kStaticScratchBytes
// (8 MiB).  Every GPU that loads the library holds it until the process
// exits.  Host code cannot use the array's name as a device address (on the
// host it names a stand-in), so the first call on each device, with that
// device current, asks the runtime for the device address with
// cudaGetSymbolAddress and keeps it; that first call should therefore come
// before any stream capture.  All calls share the array and it keeps the
// previous call's contents: each call clears the parts that must start at
// zero (the error word and the arrival counters), and calls that overlap on
// the GPU race on it.  Because the error word lives in that array and the
// next call clears it, the in-kernel reports pa_decode leaves in its
// workspace (a bounded wait that ran out, a table entry outside the pool, a
// context longer than its table row) cannot be read by a caller of this
// entry point; callers that need them use pa_decode.  Nothing here
// allocates.
#include <cuda_runtime.h>

#include <mutex>

#include "pa.h"
#include "pa_error.h"

namespace {

constexpr size_t kStaticScratchBytes = 8u << 20;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of the scratch on the current device (looked up once per device).
int scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "pa_decode_static: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return pa::fail(PA_ERR_UNSUPPORTED, "pa_decode_static: device %d", dev);
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p)
      return pa::fail(PA_ERR_CUDA, "pa_decode_static: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return PA_OK;
}

}  // namespace

extern "C" int pa_decode_static(const pa_cache_desc* desc, const void* q, const void* k_cache, const void* v_cache,
                                const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* seq_lens,
                                int32_t num_seqs, float scale, void* out, void* stream) {
  pa::clear_error();
  const char* who = "pa_decode_static";
  // every check pa_decode makes on its arguments, before anything is
  // enqueued; the workspace pointer it checks is a host stand-in (the
  // scratch's device address is looked up only once the call is accepted)
  alignas(256) static unsigned char workspace_stand_in[1];
  int rc = pa::check_attn_args(desc, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, num_seqs,
                               out, workspace_stand_in, who);
  if (rc || num_seqs == 0) return rc;
  const size_t need = pa_decode_workspace_size(desc, num_seqs);
  if (need == 0) return PA_ERR_INVALID_ARG;  // the size query already recorded why
  if (need > kStaticScratchBytes)
    return pa::fail(PA_ERR_UNSUPPORTED,
                    "%s: this batch needs %zu bytes of scratch, the static area holds %zu; "
                    "use pa_decode with a workspace",
                    who, need, kStaticScratchBytes);
  void* ws = nullptr;
  if ((rc = scratch_address(&ws))) return rc;
  // what must start at zero: the error word (256 bytes) and, on the
  // tensor-core path, the arrival counters (4 bytes per sequence and kv head,
  // padded to 256); the CUDA-core path's scratch is the error word alone.
  // Never more than the batch's own scratch, which fits in the area.
  size_t zeroed = 256 + ((size_t)num_seqs * desc->num_kv_heads * 4 + 255) / 256 * 256;
  if (zeroed > need) zeroed = need;
  cudaError_t e = cudaMemsetAsync(ws, 0, zeroed, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return pa::fail(PA_ERR_CUDA, "%s: %s", who, cudaGetErrorString(e));
  return pa_decode(desc, q, k_cache, v_cache, block_tables, max_blocks_per_seq, seq_lens, num_seqs, scale, out, ws,
                   kStaticScratchBytes, stream);
}
