// fa_flex_attention_fwd_noalloc: block-mask build + forward with every piece of
// scratch (the block tables and the device error word) in one file-scope device
// array, so that a call needs no device memory from its caller beyond Q, K, V and
// the outputs.
//
// For callers that cannot allocate device memory at the call site: an operator or
// plugin host that hands the op only its input and output tensors has no
// allocator to ask for the block tables and the workspace that
// fa_create_block_mask and fa_flex_attention_fwd take from their caller; a serving
// loop that reserved its device memory up front may have nothing left for
// cudaMalloc, and cudaMalloc / cudaFree synchronise the whole device.
//
// The array is fixed at FA_NOALLOC_SCRATCH_BYTES per device; problems whose tables
// do not fit are rejected before anything is launched.  Every call on a device
// uses the same array, so calls whose GPU work overlaps race on it.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "fa_internal.h"

// The scratch: block tables + error word of the allocation-free forward.
static __device__ __align__(256) unsigned char g_noalloc_scratch[FA_NOALLOC_SCRATCH_BYTES];

namespace fa {
namespace {

constexpr size_t kScratchBytes = FA_NOALLOC_SCRATCH_BYTES;
constexpr size_t kAlign = 256;

constexpr size_t align_up(size_t n) { return (n + kAlign - 1) / kAlign * kAlign; }

// Byte offsets of the pieces inside the scratch for an nq x nkv mask.  The error
// word comes first, in a slot of its own.
struct ScratchLayout {
  size_t err, kv_num, full_num, order, kv_idx, full_idx, total;
};

ScratchLayout scratch_layout(int32_t nq, int32_t nkv) {
  const size_t nq_s = static_cast<size_t>(nq), nkv_s = static_cast<size_t>(nkv);
  ScratchLayout l{};
  l.err = 0;
  l.kv_num = kAlign;
  l.full_num = l.kv_num + align_up(nq_s * sizeof(int32_t));
  l.order = l.full_num + align_up(nq_s * sizeof(int32_t));
  l.kv_idx = l.order + align_up(2 * nq_s * sizeof(int32_t));
  l.full_idx = l.kv_idx + align_up(nq_s * nkv_s * sizeof(int32_t));
  l.total = l.full_idx + align_up(nq_s * nkv_s * sizeof(int32_t));
  return l;
}

// Identity of the CUDA context current on this thread (0 if none or if the driver
// entry points are unavailable): a cudaDeviceReset replaces the device's primary
// context, and the module -- with the scratch array -- is loaded again in the new
// one, possibly at another address.
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long*);

unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* a = nullptr;
    void* b = nullptr;
    cudaDriverEntryPointQueryResult qa, qb;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &a, cudaEnableDefault, &qa) == cudaSuccess &&
        qa == cudaDriverEntryPointSuccess &&
        cudaGetDriverEntryPoint("cuCtxGetId", &b, cudaEnableDefault, &qb) == cudaSuccess &&
        qb == cudaDriverEntryPointSuccess) {
      get_current = reinterpret_cast<CtxGetCurrentFn>(a);
      get_id = reinterpret_cast<CtxGetIdFn>(b);
    }
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of the scratch on the current device.  The set-up -- the
// cudaGetSymbolAddress lookup, which on the first call in a context also loads
// this file's device module and so reserves the array -- runs once per device and
// context, with that device current; later calls read the cached address.
// nullptr if the lookup fails.
unsigned char* scratch_on_current_device() {
  static std::mutex mu;
  static unsigned char* addr[kMaxDevices] = {};
  static unsigned long long ctx_of[kMaxDevices] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  const unsigned long long ctx = current_context_id();
  if (addr[dev] == nullptr || ctx == 0 || ctx != ctx_of[dev]) {
    void* ptr = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
    if (e != cudaSuccess || ptr == nullptr) return nullptr;
    addr[dev] = static_cast<unsigned char*>(ptr);
    ctx_of[dev] = current_context_id();  // the lookup made the context current if none was
  }
  return addr[dev];
}

}  // namespace
}  // namespace fa

extern "C" fa_status fa_flex_attention_fwd_noalloc(
    const void* q, const void* k, const void* v, int32_t dtype, int32_t B, int32_t H,
    int32_t L, int32_t S, int32_t D, int32_t mask_kind, int32_t window,
    const int32_t* doc_id, int32_t score_kind, float softcap, float scale, void* out,
    float* lse, int32_t* device_error, void* stream) {
  using namespace fa;
  // Argument checks of both calls, up front, so that nothing is launched on an error.
  int32_t nq = 0, nkv = 0;
  const fa_status dims = fa_block_mask_dims(L, S, FA_BLOCK, &nq, &nkv);
  if (dims != FA_OK) return dims;
  if (mask_kind < FA_MASK_CAUSAL || mask_kind > FA_MASK_DOCUMENT_CAUSAL) return FA_ERR_INVALID_ARG;
  if (mask_kind == FA_MASK_SLIDING_WINDOW_CAUSAL && window < 1) return FA_ERR_INVALID_ARG;
  if (mask_kind == FA_MASK_DOCUMENT_CAUSAL && doc_id == nullptr && (L > 0 || S > 0))
    return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_INVALID_ARG;
  if (B < 0 || H < 0) return FA_ERR_INVALID_ARG;
  if (score_kind != FA_SCORE_NONE && score_kind != FA_SCORE_TANH_SOFTCAP) return FA_ERR_INVALID_ARG;
  if (score_kind == FA_SCORE_TANH_SOFTCAP && !(softcap > 0.f && std::isfinite(softcap)))
    return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  const ScratchLayout sl = scratch_layout(nq, nkv);
  if (sl.total > kScratchBytes) return FA_ERR_SCRATCH_TOO_SMALL;
  if (static_cast<int64_t>(B) * H == 0 || L == 0) return FA_OK;
  if (q == nullptr || out == nullptr || (S > 0 && (k == nullptr || v == nullptr)))
    return FA_ERR_INVALID_ARG;
  auto misaligned = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) != 0; };
  if (misaligned(q) || misaligned(out) || (S > 0 && (misaligned(k) || misaligned(v))))
    return FA_ERR_INVALID_ARG;
  if (static_cast<int64_t>(B) * H * nq > INT32_MAX) return FA_ERR_UNSUPPORTED;

  unsigned char* base = scratch_on_current_device();
  if (base == nullptr) return FA_ERR_CUDA;
  const cudaStream_t s = as_stream(stream);
  // The forward kernel only ORs flags into the error word: it must start at zero.
  int32_t* err = reinterpret_cast<int32_t*>(base + sl.err);
  FA_CUDA_CHECK(cudaMemsetAsync(err, 0, sizeof(int32_t), s));

  fa_block_mask bm{};
  bm.kv_num_blocks = reinterpret_cast<int32_t*>(base + sl.kv_num);
  bm.full_kv_num_blocks = reinterpret_cast<int32_t*>(base + sl.full_num);
  bm.q_order = reinterpret_cast<int32_t*>(base + sl.order);
  bm.kv_indices = reinterpret_cast<int32_t*>(base + sl.kv_idx);
  bm.full_kv_indices = reinterpret_cast<int32_t*>(base + sl.full_idx);
  const fa_status ms = fa_create_block_mask(mask_kind, window, doc_id, L, S, FA_BLOCK, &bm, stream);
  if (ms != FA_OK) return ms;
  const fa_status fs = fa_flex_attention_fwd(q, k, v, dtype, B, H, L, S, D, &bm, score_kind,
                                             softcap, scale, out, lse, err, stream);
  if (fs != FA_OK) return fs;
  if (device_error != nullptr)
    FA_CUDA_CHECK(cudaMemcpyAsync(device_error, err, sizeof(int32_t), cudaMemcpyDefault, s));
  return FA_OK;
}
