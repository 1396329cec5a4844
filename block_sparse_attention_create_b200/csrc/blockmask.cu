// BlockMask builder: classifies every 128x128 block of the (Q_LEN x KV_LEN)
// score grid under one of the three mask rules of the FlexAttention how-to
// (dreaming.press, "Mask 1: causal", "Mask 2: sliding-window causal",
// "Mask 3: document-packed") and writes the per-row partial / full block lists
// (FlexAttention vs SDPA on M1 Max, qiita kiarina, "役割とデータの流れ":
// BlockMask = the computed range grouped into 128x128 token blocks).
//
// Block (i, j) covers q in [128 i, 128 i + 127] and kv in [128 j, 128 j + 127].
// It is EMPTY if no pair is allowed, FULL if all 128 x 128 pairs are in range and
// allowed, PARTIAL otherwise.  Causal and sliding-window blocks are classified in
// closed form (the allowed keys of row q are the interval (q - W, q]); document
// blocks are classified exactly for arbitrary ids: a value-range test settles the
// common cases and a warp visits every pair otherwise.  A tabulated mask (one bit
// per pair) is classified by OR / AND over the block's 128 x 4 words.
#include <cstdint>

#include "fa_internal.h"

namespace fa {
namespace {

constexpr int kBlock = FA_BLOCK;
constexpr int kClassifyThreads = 256;
constexpr int kOrderThreads = 1024;

__device__ __forceinline__ void warp_minmax(int& mn, int& mx) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    mn = min(mn, __shfl_xor_sync(0xffffffffu, mn, o));
    mx = max(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  }
}

// One CTA per q-block row i (blockIdx.x) of mask instance blockIdx.y.  cls[j]: 0
// empty, 1 partial, 2 full.
__global__ void __launch_bounds__(kClassifyThreads)
classify_rows_kernel(int kind, int window, const int32_t* __restrict__ doc_all,
                     const uint32_t* __restrict__ bitmap_all, int q_len, int kv_len, int n_kv,
                     int32_t* __restrict__ kv_num, int32_t* __restrict__ kv_idx,
                     int32_t* __restrict__ full_num, int32_t* __restrict__ full_idx) {
  extern __shared__ uint8_t cls[];
  __shared__ int q_doc_min, q_doc_max;
  const int i = blockIdx.x;
  const int64_t inst = blockIdx.y;
  const int n_q = gridDim.x;
  // this instance's mask data and tables
  const int32_t* doc = doc_all ? doc_all + inst * max(q_len, kv_len) : nullptr;
  const uint32_t* bitmap =
      bitmap_all ? bitmap_all + inst * static_cast<int64_t>(q_len) * n_kv * 4 : nullptr;
  kv_num += inst * n_q;
  full_num += inst * n_q;
  kv_idx += inst * n_q * static_cast<int64_t>(n_kv);
  full_idx += inst * n_q * static_cast<int64_t>(n_kv);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t q0 = static_cast<int64_t>(i) * kBlock;
  const int64_t q1 = min(static_cast<int64_t>(q_len), q0 + kBlock) - 1;
  const bool q_whole = q0 + kBlock <= q_len;

  if (kind == FA_MASK_BITMAP) {
    // a warp per kv block: lane l reads rows q0 + l + 32 r (r < 4), all four words;
    // bits past kv_len do not count, rows past q_len neither
    const int nwarps = blockDim.x >> 5;
    const size_t wpr = static_cast<size_t>(n_kv) * 4;  // words per bitmap row
    for (int j = warp; j < n_kv; j += nwarps) {
      const int64_t k0 = static_cast<int64_t>(j) * kBlock;
      uint32_t valid[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int64_t nk = kv_len - (k0 + 32 * w);  // keys of word w that exist
        valid[w] = nk >= 32 ? 0xFFFFFFFFu : (nk <= 0 ? 0u : ((1u << nk) - 1u));
      }
      bool any = false, all = q_whole && k0 + kBlock <= kv_len;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int64_t q = q0 + lane + 32 * r;
        if (q >= q_len) continue;
        const uint4 v4 = __ldg(reinterpret_cast<const uint4*>(bitmap + q * wpr + 4 * j));
        const uint32_t wv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          any |= (wv[w] & valid[w]) != 0u;
          all &= (wv[w] & valid[w]) == valid[w];
        }
      }
      any = __any_sync(0xffffffffu, any);
      all = __all_sync(0xffffffffu, all);
      if (lane == 0) cls[j] = any ? (all ? 2 : 1) : 0;
    }
  } else if (kind != FA_MASK_DOCUMENT_CAUSAL) {
    for (int j = threadIdx.x; j < n_kv; j += blockDim.x) {
      const int64_t k0 = static_cast<int64_t>(j) * kBlock;
      const int64_t k1 = min(static_cast<int64_t>(kv_len), k0 + kBlock) - 1;
      const bool whole = q_whole && (k0 + kBlock <= kv_len);
      bool live, full;
      if (kind == FA_MASK_CAUSAL) {
        live = k0 <= q1;
        full = whole && k1 <= q0;
      } else {  // sliding window: row q sees kv in [q - W + 1, q]
        live = (k0 <= q1) && (k1 >= q0 - window + 1);
        full = whole && (k1 <= q0) && (q1 - k0 < window);
      }
      cls[j] = live ? (full ? 2 : 1) : 0;
    }
  } else {
    // value range of the ids of this q-block
    if (warp == 0) {
      int mn = INT32_MAX, mx = INT32_MIN;
      for (int64_t q = q0 + lane; q <= q1; q += 32) {
        const int d = __ldg(doc + q);
        mn = min(mn, d);
        mx = max(mx, d);
      }
      warp_minmax(mn, mx);
      if (lane == 0) {
        q_doc_min = mn;
        q_doc_max = mx;
      }
    }
    __syncthreads();
    const int qmn = q_doc_min, qmx = q_doc_max;
    const int nwarps = blockDim.x >> 5;
    for (int j = warp; j < n_kv; j += nwarps) {
      const int64_t k0 = static_cast<int64_t>(j) * kBlock;
      const int64_t k1 = min(static_cast<int64_t>(kv_len), k0 + kBlock) - 1;
      if (k0 > q1) {  // strictly above the causal diagonal
        if (lane == 0) cls[j] = 0;
        continue;
      }
      int kmn = INT32_MAX, kmx = INT32_MIN;
      for (int64_t kv = k0 + lane; kv <= k1; kv += 32) {
        const int d = __ldg(doc + kv);
        kmn = min(kmn, d);
        kmx = max(kmx, d);
      }
      warp_minmax(kmn, kmx);
      uint8_t c;
      if (kmx < qmn || kmn > qmx) {
        c = 0;  // no id in common: no pair can match
      } else if (k1 <= q0 && qmn == qmx && kmn == kmx) {
        // below the diagonal, one id on both sides (and they overlap, so equal)
        c = (q_whole && k0 + kBlock <= kv_len) ? 2 : 1;
      } else {
        // visit every pair: lane owns 4 query rows
        bool any = false, all = true;
        for (int r = 0; r < 4; ++r) {
          const int64_t q = q0 + lane * 4 + r;
          if (q >= q_len) {
            all = false;
            continue;
          }
          const int dq = __ldg(doc + q);
          for (int cc = 0; cc < kBlock; ++cc) {
            const int64_t kv = k0 + cc;
            const bool ok = kv < kv_len && kv <= q && __ldg(doc + kv) == dq;
            any |= ok;
            all &= ok;
          }
        }
        any = __any_sync(0xffffffffu, any);
        all = __all_sync(0xffffffffu, all);
        c = any ? (all ? 2 : 1) : 0;
      }
      if (lane == 0) cls[j] = c;
    }
  }
  __syncthreads();

  // Compaction, ascending j: warp 0 turns the classes into the two lists.
  if (warp == 0) {
    const int64_t base_row = static_cast<int64_t>(i) * n_kv;
    int np = 0, nf = 0;
    const unsigned lt = (1u << lane) - 1u;
    for (int base = 0; base < n_kv; base += 32) {
      const int j = base + lane;
      const uint8_t c = j < n_kv ? cls[j] : 0;
      const unsigned pm = __ballot_sync(0xffffffffu, c == 1);
      const unsigned fm = __ballot_sync(0xffffffffu, c == 2);
      if (c == 1) kv_idx[base_row + np + __popc(pm & lt)] = j;
      if (c == 2) full_idx[base_row + nf + __popc(fm & lt)] = j;
      np += __popc(pm);
      nf += __popc(fm);
    }
    for (int t = np + lane; t < n_kv; t += 32) kv_idx[base_row + t] = 0;
    for (int t = nf + lane; t < n_kv; t += 32) full_idx[base_row + t] = 0;
    if (lane == 0) {
      kv_num[i] = np;
      full_num[i] = nf;
    }
  }
}

// Schedule table q_order[2 * n_q]: rank k (rows by descending live count, ties by
// ascending row) -> [2k] = row, [2k+1] = partial count | full count << 16.  Keys
// (n_kv - count) << 13 | row are unique, so every sort of them gives the same
// order: up to 2048 rows each thread ranks its rows by counting smaller keys;
// above that a bitonic sort in shared memory.
__global__ void __launch_bounds__(kOrderThreads)
order_rows_kernel(int n_q, int n_kv, int n_pow2, const int32_t* __restrict__ kv_num,
                  const int32_t* __restrict__ full_num, int32_t* __restrict__ sched) {
  extern __shared__ uint32_t keys[];
  // one CTA per mask instance
  kv_num += static_cast<int64_t>(blockIdx.x) * n_q;
  full_num += static_cast<int64_t>(blockIdx.x) * n_q;
  sched += static_cast<int64_t>(blockIdx.x) * 2 * n_q;
  const bool rank_sort = n_q <= 2048;
  const int n_keys = rank_sort ? n_q : n_pow2;
  for (int t = threadIdx.x; t < n_keys; t += blockDim.x) {
    if (t < n_q) {
      const int cnt = kv_num[t] + full_num[t];
      keys[t] = (static_cast<uint32_t>(n_kv - cnt) << 13) | static_cast<uint32_t>(t);
    } else {
      keys[t] = 0xFFFFFFFFu;
    }
  }
  __syncthreads();
  if (rank_sort) {
    for (int t = threadIdx.x; t < n_q; t += blockDim.x) {
      const uint32_t key = keys[t];
      int rank = 0;
      for (int j = 0; j < n_q; ++j) rank += keys[j] < key ? 1 : 0;
      sched[2 * rank] = t;
      sched[2 * rank + 1] = kv_num[t] | (full_num[t] << 16);
    }
    return;
  }
  for (int k = 2; k <= n_pow2; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int t = threadIdx.x; t < n_pow2; t += blockDim.x) {
        const int p = t ^ j;
        if (p > t) {
          const uint32_t a = keys[t], b = keys[p];
          const bool ascending = (t & k) == 0;
          if ((a > b) == ascending) {
            keys[t] = b;
            keys[p] = a;
          }
        }
      }
      __syncthreads();
    }
  }
  for (int t = threadIdx.x; t < n_q; t += blockDim.x) {
    const int row = static_cast<int>(keys[t] & 0x1FFFu);
    sched[2 * t] = row;
    sched[2 * t + 1] = kv_num[row] | (full_num[row] << 16);
  }
}

// Column lists: one CTA per kv block j.  Every warp classifies q-block rows
// (i, j) by binary search in row i's ascending partial and full lists; warp 0 then
// compacts the classes in ascending i.
__global__ void __launch_bounds__(kClassifyThreads)
transpose_kernel(int n_q, int n_kv, const int32_t* __restrict__ kv_num,
                 const int32_t* __restrict__ kv_idx, const int32_t* __restrict__ full_num,
                 const int32_t* __restrict__ full_idx, int32_t* __restrict__ q_num,
                 int32_t* __restrict__ q_idx, int32_t* __restrict__ full_q_num,
                 int32_t* __restrict__ full_q_idx) {
  extern __shared__ uint8_t cls[];
  const int j = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  {  // this instance's tables and column lists
    const int64_t inst = blockIdx.y;
    kv_num += inst * n_q;
    full_num += inst * n_q;
    kv_idx += inst * n_q * static_cast<int64_t>(n_kv);
    full_idx += inst * n_q * static_cast<int64_t>(n_kv);
    q_num += inst * n_kv;
    full_q_num += inst * n_kv;
    q_idx += inst * n_kv * static_cast<int64_t>(n_q);
    full_q_idx += inst * n_kv * static_cast<int64_t>(n_q);
  }
  auto contains = [j](const int32_t* list, int n) {
    int lo = 0, hi = n;  // first position with list[pos] >= j
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (__ldg(list + mid) < j) lo = mid + 1; else hi = mid;
    }
    return lo < n && __ldg(list + lo) == j;
  };
  for (int i = threadIdx.x; i < n_q; i += blockDim.x) {
    const size_t row = static_cast<size_t>(i) * n_kv;
    uint8_t c = 0;
    if (contains(full_idx + row, __ldg(full_num + i))) c = 2;
    else if (contains(kv_idx + row, __ldg(kv_num + i))) c = 1;
    cls[i] = c;
  }
  __syncthreads();
  if (warp == 0) {
    const size_t base_col = static_cast<size_t>(j) * n_q;
    int np = 0, nf = 0;
    const unsigned lt = (1u << lane) - 1u;
    for (int base = 0; base < n_q; base += 32) {
      const int i = base + lane;
      const uint8_t c = i < n_q ? cls[i] : 0;
      const unsigned pm = __ballot_sync(0xffffffffu, c == 1);
      const unsigned fm = __ballot_sync(0xffffffffu, c == 2);
      if (c == 1) q_idx[base_col + np + __popc(pm & lt)] = i;
      if (c == 2) full_q_idx[base_col + nf + __popc(fm & lt)] = i;
      np += __popc(pm);
      nf += __popc(fm);
    }
    for (int t = np + lane; t < n_q; t += 32) q_idx[base_col + t] = 0;
    for (int t = nf + lane; t < n_q; t += 32) full_q_idx[base_col + t] = 0;
    if (lane == 0) {
      q_num[j] = np;
      full_q_num[j] = nf;
    }
  }
}

}  // namespace
}  // namespace fa

extern "C" fa_status fa_block_mask_dims(int32_t q_len, int32_t kv_len, int32_t block,
                                        int32_t* n_q_blocks, int32_t* n_kv_blocks) {
  if (n_q_blocks == nullptr || n_kv_blocks == nullptr) return FA_ERR_INVALID_ARG;
  if (block != FA_BLOCK || q_len < 0 || kv_len < 0 || q_len > FA_MAX_LEN || kv_len > FA_MAX_LEN)
    return FA_ERR_INVALID_ARG;
  *n_q_blocks = (q_len + FA_BLOCK - 1) / FA_BLOCK;
  *n_kv_blocks = (kv_len + FA_BLOCK - 1) / FA_BLOCK;
  return FA_OK;
}

namespace fa {
namespace {

// Shared tail of the two builders: fill the scalar fields, classify, order.
fa_status build_tables(int32_t kind, int32_t window, const int32_t* doc_id, const uint32_t* bitmap,
                       int32_t mask_batch, int32_t mask_heads, int32_t q_len, int32_t kv_len,
                       int32_t block, int32_t nq, int32_t nkv, fa_block_mask* bm, void* stream) {
  bm->q_len = q_len;
  bm->kv_len = kv_len;
  bm->block = block;
  bm->n_q_blocks = nq;
  bm->n_kv_blocks = nkv;
  bm->kind = kind;
  bm->window = kind == FA_MASK_SLIDING_WINDOW_CAUSAL ? window : 0;
  bm->doc_id = kind == FA_MASK_DOCUMENT_CAUSAL ? doc_id : nullptr;
  bm->bitmap = kind == FA_MASK_BITMAP ? bitmap : nullptr;
  bm->mask_batch = mask_batch;
  bm->mask_heads = mask_heads;
  if (nq == 0) return FA_OK;

  const int inst = mask_batch * mask_heads;
  cudaStream_t s = as_stream(stream);
  classify_rows_kernel<<<dim3(nq, inst), kClassifyThreads, nkv > 0 ? nkv : 1, s>>>(
      kind, bm->window, bm->doc_id, bm->bitmap, q_len, kv_len, nkv, bm->kv_num_blocks,
      bm->kv_indices, bm->full_kv_num_blocks, bm->full_kv_indices);
  FA_CUDA_CHECK(cudaGetLastError());
  int n_pow2 = 1;
  while (n_pow2 < nq) n_pow2 <<= 1;
  const size_t order_smem = (nq <= 2048 ? nq : n_pow2) * sizeof(uint32_t);
  order_rows_kernel<<<inst, kOrderThreads, order_smem, s>>>(
      nq, nkv, n_pow2, bm->kv_num_blocks, bm->full_kv_num_blocks, bm->q_order);
  FA_CUDA_CHECK(cudaGetLastError());
  return FA_OK;
}

bool tables_present(const fa_block_mask* bm, int32_t nq, int32_t nkv) {
  if (nq > 0 && (bm->kv_num_blocks == nullptr || bm->full_kv_num_blocks == nullptr ||
                 bm->q_order == nullptr))
    return false;
  if (nq > 0 && nkv > 0 && (bm->kv_indices == nullptr || bm->full_kv_indices == nullptr))
    return false;
  return true;
}

}  // namespace
}  // namespace fa

extern "C" fa_status fa_create_block_mask(int32_t kind, int32_t window, const int32_t* doc_id,
                                          int32_t q_len, int32_t kv_len, int32_t block,
                                          fa_block_mask* bm, void* stream) {
  using namespace fa;
  if (bm == nullptr) return FA_ERR_INVALID_ARG;
  if (kind < FA_MASK_CAUSAL || kind > FA_MASK_DOCUMENT_CAUSAL) return FA_ERR_INVALID_ARG;
  int32_t nq = 0, nkv = 0;
  const fa_status st = fa_block_mask_dims(q_len, kv_len, block, &nq, &nkv);
  if (st != FA_OK) return st;
  if (kind == FA_MASK_SLIDING_WINDOW_CAUSAL && window < 1) return FA_ERR_INVALID_ARG;
  if (kind == FA_MASK_DOCUMENT_CAUSAL && doc_id == nullptr && (q_len > 0 || kv_len > 0))
    return FA_ERR_INVALID_ARG;
  if (!tables_present(bm, nq, nkv)) return FA_ERR_INVALID_ARG;
  return build_tables(kind, window, doc_id, nullptr, 1, 1, q_len, kv_len, block, nq, nkv, bm,
                      stream);
}

extern "C" fa_status fa_create_block_mask_bitmap(const uint32_t* bitmap, int32_t q_len,
                                                 int32_t kv_len, int32_t block, fa_block_mask* bm,
                                                 void* stream) {
  using namespace fa;
  if (bm == nullptr) return FA_ERR_INVALID_ARG;
  int32_t nq = 0, nkv = 0;
  const fa_status st = fa_block_mask_dims(q_len, kv_len, block, &nq, &nkv);
  if (st != FA_OK) return st;
  if (q_len > 0 && kv_len > 0 &&
      (bitmap == nullptr || (reinterpret_cast<uintptr_t>(bitmap) & 15u) != 0))
    return FA_ERR_INVALID_ARG;
  if (!tables_present(bm, nq, nkv)) return FA_ERR_INVALID_ARG;
  return build_tables(FA_MASK_BITMAP, 0, nullptr, bitmap, 1, 1, q_len, kv_len, block, nq, nkv, bm,
                      stream);
}

extern "C" fa_status fa_create_block_mask_bh(int32_t kind, int32_t window, const int32_t* doc_id,
                                             const uint32_t* bitmap, int32_t mask_batch,
                                             int32_t mask_heads, int32_t q_len, int32_t kv_len,
                                             int32_t block, fa_block_mask* bm, void* stream) {
  using namespace fa;
  if (bm == nullptr) return FA_ERR_INVALID_ARG;
  if (kind < FA_MASK_CAUSAL || kind > FA_MASK_BITMAP) return FA_ERR_INVALID_ARG;
  if (mask_batch < 1 || mask_heads < 1 || static_cast<int64_t>(mask_batch) * mask_heads > 65535)
    return FA_ERR_INVALID_ARG;
  int32_t nq = 0, nkv = 0;
  const fa_status st = fa_block_mask_dims(q_len, kv_len, block, &nq, &nkv);
  if (st != FA_OK) return st;
  if (kind == FA_MASK_SLIDING_WINDOW_CAUSAL && window < 1) return FA_ERR_INVALID_ARG;
  if (kind == FA_MASK_DOCUMENT_CAUSAL && doc_id == nullptr && (q_len > 0 || kv_len > 0))
    return FA_ERR_INVALID_ARG;
  if (kind == FA_MASK_BITMAP && q_len > 0 && kv_len > 0 &&
      (bitmap == nullptr || (reinterpret_cast<uintptr_t>(bitmap) & 15u) != 0))
    return FA_ERR_INVALID_ARG;
  if (!tables_present(bm, nq, nkv)) return FA_ERR_INVALID_ARG;
  return build_tables(kind, window, doc_id, bitmap, mask_batch, mask_heads, q_len, kv_len, block,
                      nq, nkv, bm, stream);
}

extern "C" fa_status fa_block_mask_transpose(const fa_block_mask* bm, int32_t* q_num_blocks,
                                             int32_t* q_indices, int32_t* full_q_num_blocks,
                                             int32_t* full_q_indices, void* stream) {
  using namespace fa;
  if (bm == nullptr || bm->block != FA_BLOCK || bm->n_q_blocks < 0 || bm->n_kv_blocks < 0)
    return FA_ERR_INVALID_ARG;
  const int32_t nq = bm->n_q_blocks, nkv = bm->n_kv_blocks;
  if (nq == 0 || nkv == 0) return FA_OK;
  if (!tables_present(bm, nq, nkv) || q_num_blocks == nullptr || q_indices == nullptr ||
      full_q_num_blocks == nullptr || full_q_indices == nullptr)
    return FA_ERR_INVALID_ARG;
  const int inst = (bm->mask_batch > 1 ? bm->mask_batch : 1) * (bm->mask_heads > 1 ? bm->mask_heads : 1);
  transpose_kernel<<<dim3(nkv, inst), kClassifyThreads, nq, as_stream(stream)>>>(
      nq, nkv, bm->kv_num_blocks, bm->kv_indices, bm->full_kv_num_blocks, bm->full_kv_indices,
      q_num_blocks, q_indices, full_q_num_blocks, full_q_indices);
  FA_CUDA_CHECK(cudaGetLastError());
  return FA_OK;
}
