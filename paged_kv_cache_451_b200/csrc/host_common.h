// Host-side helpers shared by the library's translation units.
#pragma once

#include <cstdarg>
#include <cstdio>

#include "../../include/pagedkv.h"

namespace pagedkv {

// Record a message for kv_last_error() and return `code`.
int fail(int code, const char* fmt, ...);
// Clear the calling thread's message and return KV_OK.
int ok();

}  // namespace pagedkv
