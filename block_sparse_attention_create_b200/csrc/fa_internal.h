// Host-side helpers shared by the library's translation units (not part of the ABI).
#pragma once

#include <cuda.h>
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

// 3-D TMA map over a contiguous (bh, rows, D) 16-bit tensor: box = 64 elements x
// box_rows rows x 1, 128-byte swizzle; rows past `rows` read as zeros.  False if the
// driver's encoder is unavailable or rejects the arguments.
bool make_tile_map(CUtensorMap* map, const void* ptr, bool bf16, int D, int rows, int bh,
                   int box_rows);

}  // namespace fa

#define FA_CUDA_CHECK(expr)                           \
  do {                                                \
    cudaError_t fa_err__ = (expr);                    \
    if (fa_err__ != cudaSuccess) return FA_ERR_CUDA;  \
  } while (0)
