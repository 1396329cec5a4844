// Host-side entry points shared by the operations: status strings, device
// queries, the device error word of the workspaces and the testing hook that
// makes the kernels' bounded waits run out.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <mutex>

#include "fa_internal.h"

namespace fa {

int num_sms_current_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  static std::mutex mu;
  static int cache[kMaxDevices] = {};
  std::lock_guard<std::mutex> lock(mu);
  if (cache[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
}

namespace {
// Testing hook for the bounded-wait failure path (fa_debug_set_mma_stall).
std::atomic<int> g_stall{0};
std::atomic<unsigned long long> g_stall_wait_limit_ns{2000000000ull};
}  // namespace

bool debug_stall(unsigned long long* wait_limit_ns) {
  if (!g_stall.load()) return false;
  *wait_limit_ns = g_stall_wait_limit_ns.load();
  return true;
}

}  // namespace fa

extern "C" void fa_debug_set_mma_stall(int32_t on, uint64_t wait_limit_ns) {
  fa::g_stall_wait_limit_ns.store(wait_limit_ns > 0 ? wait_limit_ns : 2000000000ull);
  fa::g_stall.store(on ? 1 : 0);
}

extern "C" const char* fa_status_string(int32_t status) {
  switch (status) {
    case FA_OK: return "FA_OK";
    case FA_ERR_INVALID_ARG: return "FA_ERR_INVALID_ARG";
    case FA_ERR_UNSUPPORTED: return "FA_ERR_UNSUPPORTED";
    case FA_ERR_CUDA: return "FA_ERR_CUDA";
    case FA_ERR_TIMEOUT: return "FA_ERR_TIMEOUT";
    case FA_ERR_SCRATCH_TOO_SMALL: return "FA_ERR_SCRATCH_TOO_SMALL";
    default: return "FA_ERR_UNKNOWN";
  }
}

extern "C" int32_t fa_num_sms(void) { return fa::num_sms_current_device(); }

extern "C" fa_status fa_get_last_device_error(void* workspace, void* stream) {
  if (workspace == nullptr) return FA_ERR_INVALID_ARG;
  cudaStream_t s = fa::as_stream(stream);
  FA_CUDA_CHECK(cudaStreamSynchronize(s));
  int32_t word = 0;
  FA_CUDA_CHECK(cudaMemcpyAsync(&word, workspace, sizeof(word), cudaMemcpyDeviceToHost, s));
  FA_CUDA_CHECK(cudaStreamSynchronize(s));
  if (word != 0) {
    FA_CUDA_CHECK(cudaMemsetAsync(workspace, 0, sizeof(word), s));
    FA_CUDA_CHECK(cudaStreamSynchronize(s));
    if (word & fa::kDevErrTimeout) return FA_ERR_TIMEOUT;
  }
  return FA_OK;
}
