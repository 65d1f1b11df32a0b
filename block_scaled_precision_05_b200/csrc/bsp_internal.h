// bsp_internal.h -- host-side helpers shared by the library's translation units.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "bsp.h"

namespace bsp {

struct DeviceInfo {
  int id = -1;
  int sm_count = 0;
  uint32_t* err_word = nullptr;  // device address of this device's error word
};

// Checks the current device is sm_100 and returns its cached properties.
int current_device(DeviceInfo* out);

// The driver's cuTensorMapEncodeTiled, looked up once through the runtime.
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn encode_tiled_fn();

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline int64_t round_up(int64_t a, int64_t b) { return ceil_div(a, b) * b; }

// Maps the result of a launch to a status (and clears a sticky-free error).
inline int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? BSP_OK : BSP_ERR_CUDA;
}

}  // namespace bsp
