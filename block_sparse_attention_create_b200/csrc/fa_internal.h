// Host-side helpers shared by the library's translation units (not part of the ABI).
#pragma once

#include <cuda_runtime.h>

#include "fa.h"

namespace fa {

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// SM count of the current device (cached per device); 0 when no device.
int num_sms_current_device();

// Device error flags kept in word 0 of the forward workspace.
constexpr int kDevErrTimeout = 1;

// Per-device state (kernel attributes, SM counts) is kept for this many devices.
constexpr int kMaxDevices = 64;

}  // namespace fa

#define FA_CUDA_CHECK(expr)                           \
  do {                                                \
    cudaError_t fa_err__ = (expr);                    \
    if (fa_err__ != cudaSuccess) return FA_ERR_CUDA;  \
  } while (0)
