// Internal: last-error bookkeeping shared by the pool and the device calls.
#pragma once

#include <cstdarg>

#include "pa.h"

namespace pa {

// Records a printf-style message for pa_last_error() on this thread and
// returns `code`, so call sites can write `return fail(PA_ERR_..., "...")`.
int fail(int code, const char* fmt, ...);

// Clears the message (called at the start of every public entry point).
void clear_error();

}  // namespace pa
