// host.h -- host-side plumbing shared by the libbi translation units:
// error reporting, the device status word, TMA descriptor encoding.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/bi.h"

namespace bi {

// Records a one-line reason for the calling host thread and returns `st`.
bi_status fail(bi_status st, const char* fmt, ...);

// Maps a CUDA runtime error to BI_ERR_CUDA with its message.
bi_status cuda_fail(cudaError_t e, const char* where);

// Checks that the current device is an sm_100 part; cached per device.
bi_status require_sm100();

// Device address of the library's status word on the current device.
int32_t* status_word();

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda
// link). rank 2 or 3, dims/strides in elements/bytes as the driver wants them
// (strides for dims 1..rank-1 only).
bi_status encode_tmap(CUtensorMap* map, CUtensorMapDataType dtype, uint32_t rank,
                      void* base, const uint64_t* dims, const uint64_t* strides_bytes,
                      const uint32_t* box, CUtensorMapSwizzle swizzle);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

inline int num_sms() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

}  // namespace bi

#define BI_CHECK_LAUNCH(where)                         \
  do {                                                 \
    cudaError_t e_ = cudaGetLastError();               \
    if (e_ != cudaSuccess) return bi::cuda_fail(e_, where); \
  } while (0)
