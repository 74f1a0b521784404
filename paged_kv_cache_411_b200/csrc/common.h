// Shared host-side helpers of libpagedkv: status plumbing and the per-thread
// last-error message.  No CUDA types here so the allocator stays host-only.
#pragma once

#include <cstdarg>
#include <cstdio>
#include <string>

#include "pagedkv.h"

namespace pagedkv {

// Records a formatted message as the calling thread's last error and returns `s`.
pa_status fail(pa_status s, const char* fmt, ...);
// Clears the calling thread's last error.
void clear_error();

}  // namespace pagedkv
