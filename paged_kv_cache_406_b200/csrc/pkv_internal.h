// Internal helpers shared by the library's translation units (not installed).
#pragma once

#include <cstdarg>
#include <cstdio>
#include <string>

#include "paged_kv.h"

namespace pkv {

// Records `code` and a printf-style message as the calling thread's last error
// and returns `code`, so call sites can `return fail(...)`.
int fail(int code, const char* fmt, ...);

// Clears the calling thread's last error and returns PKV_OK.
int ok();

}  // namespace pkv
