// Device-side error word shared by every kernel of the library.
#pragma once

#include <cuda_runtime.h>

#include "../../include/pagedkv.h"

namespace pagedkv {

// First error any kernel recorded since the host last read it (0 = none).
// One copy per device; read and cleared by kv_get_device_error.
__device__ int g_device_error;

__device__ __forceinline__ void record_error(int code) { atomicCAS(&g_device_error, 0, code); }

}  // namespace pagedkv
