// Internal: last-error bookkeeping shared by the pool and the device calls,
// and the host-side argument check shared by the attention entry points.
#pragma once

#include <cstdarg>

#include "pa.h"

namespace pa {

// Records a printf-style message for pa_last_error() on this thread and
// returns `code`, so call sites can write `return fail(PA_ERR_..., "...")`.
int fail(int code, const char* fmt, ...);

// Clears the message (called at the start of every public entry point).
void clear_error();

// Host-side checks of an attention call (desc, pointers, alignment, batch
// limits) done before anything is enqueued; PA_OK or the recorded error.
int check_attn_args(const pa_cache_desc* d, const void* q, const void* k_cache, const void* v_cache,
                    const int32_t* block_tables, int32_t max_blocks, const int32_t* seq_lens, int32_t num_seqs,
                    void* out, void* workspace, const char* who);

}  // namespace pa
