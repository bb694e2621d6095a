// Host-side error reporting shared by the C-ABI entry points: each entry point clears the calling
// thread's last-error text on entry and, when it refuses a call, stores a one-line reason there
// (read back with iskv_last_error()).
#pragma once

#include <cuda_runtime.h>

#include "iskv.h"

namespace iskv {

void clear_last_error();
iskv_status fail(iskv_status st, const char *fmt, ...);
iskv_status cuda_fail(cudaError_t e, const char *where);

}  // namespace iskv
