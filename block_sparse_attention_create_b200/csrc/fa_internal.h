// Host-side helpers shared by the library's translation units (not part of the ABI).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include "fa.h"

namespace fa {

inline cudaStream_t as_stream(void* s) { return reinterpret_cast<cudaStream_t>(s); }

// SM count of the current device (cached per device); 0 when no device.
int num_sms_current_device();

// Testing hook (fa_debug_set_mma_stall): true while it is on, with the wait limit
// the kernels then use.
bool debug_stall(unsigned long long* wait_limit_ns);

// Device error flags kept in word 0 of the forward workspace.
constexpr int kDevErrTimeout = 1;

// Per-device state (kernel attributes, SM counts) is kept for this many devices.
constexpr int kMaxDevices = 64;

// 3-D TMA map over a contiguous (bh, rows, D) 16-bit tensor: box = 64 elements x
// box_rows rows x 1, 128-byte swizzle; rows past `rows` read as zeros.  False if the
// driver's encoder is unavailable or rejects the arguments.
bool make_tile_map(CUtensorMap* map, const void* ptr, bool bf16, int D, int rows, int bh,
                   int box_rows);

// Launch with programmatic dependent launch: the kernel may be scheduled while the
// previous kernel on the stream is still running and must execute grid_dep_wait()
// before it touches memory that an earlier kernel writes or reads.
template <class... KArgs, class... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

}  // namespace fa

// Device side of programmatic dependent launch (PTX griddepcontrol): wait until the
// grids this one depends on have completed and their writes are visible; let the
// next grid on the stream be scheduled (it still waits for this one to complete
// before it reads anything).
#if defined(__CUDACC__)
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
#endif

#define FA_CUDA_CHECK(expr)                           \
  do {                                                \
    cudaError_t fa_err__ = (expr);                    \
    if (fa_err__ != cudaSuccess) return FA_ERR_CUDA;  \
  } while (0)
