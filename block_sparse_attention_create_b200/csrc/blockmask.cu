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
  __shared__ int q_ids[kBlock];  // document masks: the ids of this q-block's rows
  grid_dep_launch_dependents();  // programmatic dependent launch, see interval_tables_kernel
  grid_dep_wait();
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
    // Rows are read whole, coalesced: lane l of a warp takes kv blocks l, l + 32, ...
    // (each block's 4 words of a row are one 16-byte load), the warps take the
    // block's rows in turn.  Per group of 32 blocks a warp folds its rows into an
    // "any bit set" and an "all bits set" flag per block, ballots them into two
    // words and merges those into the CTA's words in shared memory (OR / AND).
    // Bits past kv_len do not count, rows past q_len are not read.
    const int nwarps = blockDim.x >> 5;
    const int nwords = (n_kv + 31) / 32;
    uint32_t* any_bits = reinterpret_cast<uint32_t*>(cls + ((n_kv + 15) & ~15));
    uint32_t* all_bits = any_bits + nwords;
    for (int t = threadIdx.x; t < nwords; t += blockDim.x) {
      any_bits[t] = 0u;
      all_bits[t] = 0xFFFFFFFFu;
    }
    __syncthreads();
    const size_t wpr = static_cast<size_t>(n_kv) * 4;  // words per bitmap row
    for (int m = 0; m < nwords; ++m) {
      const int j = 32 * m + lane;
      const int64_t k0 = static_cast<int64_t>(j) * kBlock;
      uint32_t valid[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const int64_t nk = kv_len - (k0 + 32 * w);  // keys of word w that exist
        valid[w] = nk >= 32 ? 0xFFFFFFFFu : (nk <= 0 ? 0u : ((1u << nk) - 1u));
      }
      bool any = false, all = true;
      if (j < n_kv) {
#pragma unroll 4
        for (int64_t q = q0 + warp; q <= q1; q += nwarps) {
          const uint4 v4 = __ldg(reinterpret_cast<const uint4*>(bitmap + q * wpr + 4 * j));
          const uint32_t wv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
          for (int w = 0; w < 4; ++w) {
            any |= (wv[w] & valid[w]) != 0u;
            all &= (wv[w] & valid[w]) == valid[w];
          }
        }
      }
      const uint32_t any_w = __ballot_sync(0xffffffffu, any);
      const uint32_t all_w = __ballot_sync(0xffffffffu, all);
      if (lane == 0) {
        atomicOr(&any_bits[m], any_w);
        atomicAnd(&all_bits[m], all_w);
      }
    }
    __syncthreads();
    for (int j = threadIdx.x; j < n_kv; j += blockDim.x) {
      const bool whole = q_whole && static_cast<int64_t>(j + 1) * kBlock <= kv_len;
      const bool any = (any_bits[j >> 5] >> (j & 31)) & 1u;
      const bool all = (all_bits[j >> 5] >> (j & 31)) & 1u;
      cls[j] = any ? (all && whole ? 2 : 1) : 0;
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
    // the ids of this q-block, and their value range
    for (int64_t q = q0 + threadIdx.x; q <= q1; q += blockDim.x) q_ids[q - q0] = __ldg(doc + q);
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
        // Not FULL: that needs one id on both sides.  Live iff some key k has a query
        // q >= k of its document.  One pass per distinct id among the block's keys,
        // lowest key first: that key k_v is the first of its id v, so the block is
        // live iff some query q >= k_v has id v (the warp tests the block's query
        // ids, staged in shared memory, 4 per lane); then every key of id v is done.
        // Keys past k1 take no pass.  Control flow is warp-uniform (ballots).
        int kid[4];
        uint32_t todo[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int64_t kv = k0 + lane + 32 * r;
          kid[r] = kv <= k1 ? __ldg(doc + kv) : 0;
          todo[r] = __ballot_sync(0xffffffffu, kv <= k1);
        }
        bool live = false;
        while (!live && (todo[0] | todo[1] | todo[2] | todo[3]) != 0u) {
          const int r0 = todo[0] ? 0 : (todo[1] ? 1 : (todo[2] ? 2 : 3));
          const int src_lane = __ffs(todo[r0]) - 1;
          const int kidr = r0 == 0 ? kid[0] : (r0 == 1 ? kid[1] : (r0 == 2 ? kid[2] : kid[3]));
          const int v = __shfl_sync(0xffffffffu, kidr, src_lane);
          const int64_t kmin = k0 + src_lane + 32 * r0;
          bool hit = false;
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int64_t q = q0 + lane + 32 * r;
            hit |= q <= q1 && q >= kmin && q_ids[q - q0] == v;
          }
          live = __any_sync(0xffffffffu, hit);
#pragma unroll
          for (int r = 0; r < 4; ++r) todo[r] &= ~__ballot_sync(0xffffffffu, kid[r] == v);
        }
        c = live ? 1 : 0;
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
  grid_dep_launch_dependents();
  grid_dep_wait();  // the counts come from classify_rows_kernel
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

// Causal and sliding-window masks in one launch.  Their live kv blocks of row i form
// one interval [lo, hi] and the FULL ones a sub-interval [flo, fhi]; so each row's
// lists, counts and the schedule follow from closed forms with no classification
// pass.  Row q-block i covers q in [q0, q1], kv block j covers [k0, k1] with
// k0 = 128 j, k1 = min(128 j + 127, kv_len - 1):
//   live  iff k0 <= q1 (causal) and k1 >= q0 - W + 1 (window);
//   full  iff both blocks are whole, k1 <= q0 (all pairs causal) and q1 - k0 < W.
struct RowRanges {
  int lo, hi, flo, fhi;  // live [lo, hi], full [flo, fhi]; empty when lo > hi / flo > fhi
};

__device__ __forceinline__ RowRanges interval_row(int kind, int window, int q_len, int kv_len,
                                                  int n_kv, int i) {
  RowRanges r{1, 0, 1, 0};
  if (n_kv == 0) return r;
  const int q0 = i * kBlock;
  const int q1 = min(q_len, q0 + kBlock) - 1;
  r.hi = min(q1 / kBlock, n_kv - 1);
  r.lo = 0;
  if (kind == FA_MASK_SLIDING_WINDOW_CAUSAL) {
    const int64_t t = static_cast<int64_t>(q0) - window + 1;  // smallest key any row sees
    if (t > kv_len - 1) return RowRanges{1, 0, 1, 0};
    r.lo = t <= 0 ? 0 : static_cast<int>(t / kBlock);
  }
  if (q0 + kBlock <= q_len && q0 >= kBlock - 1) {
    r.fhi = min((q0 - (kBlock - 1)) / kBlock, kv_len / kBlock - 1);
    if (kind == FA_MASK_SLIDING_WINDOW_CAUSAL) {
      const int64_t d = static_cast<int64_t>(q1) - window;
      r.flo = d < 0 ? 0 : static_cast<int>(d / kBlock) + 1;
    } else {
      r.flo = 0;
    }
  }
  return r;
}

__device__ __forceinline__ int live_count(const RowRanges& r) { return max(0, r.hi - r.lo + 1); }
__device__ __forceinline__ int full_count(const RowRanges& r) { return max(0, r.fhi - r.flo + 1); }

// CTA b builds rows b, b + gridDim.x, ...; every CTA first tabulates the live
// count of all rows in shared memory, from which a row's rank in the schedule
// (descending live count, ties by ascending row) is a count.  Mask instance
// blockIdx.y gets its own copy (the rule does not depend on batch or head).
__global__ void __launch_bounds__(kClassifyThreads)
interval_tables_kernel(int kind, int window, int q_len, int kv_len, int n_q, int n_kv,
                       int32_t* __restrict__ kv_num, int32_t* __restrict__ kv_idx,
                       int32_t* __restrict__ full_num, int32_t* __restrict__ full_idx,
                       int32_t* __restrict__ sched) {
  extern __shared__ int32_t live_cnt[];
  __shared__ int warp_sum[kClassifyThreads / 32];
  // launched as a programmatic dependent: a kernel still running before this one may
  // read the tables (a forward of the previous step)
  grid_dep_launch_dependents();
  grid_dep_wait();
  {
    const int64_t inst = blockIdx.y;
    kv_num += inst * n_q;
    full_num += inst * n_q;
    kv_idx += inst * n_q * static_cast<int64_t>(n_kv);
    full_idx += inst * n_q * static_cast<int64_t>(n_kv);
    sched += inst * 2 * n_q;
  }
  for (int r = threadIdx.x; r < n_q; r += blockDim.x)
    live_cnt[r] = live_count(interval_row(kind, window, q_len, kv_len, n_kv, r));
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int i = blockIdx.x; i < n_q; i += gridDim.x) {
    const RowRanges rr = interval_row(kind, window, q_len, kv_len, n_kv, i);
    const int nf = full_count(rr);
    const int np = live_count(rr) - nf;
    // partial blocks: [lo, flo) then (fhi, hi] around the full ones (or all of [lo, hi])
    const int part_a = nf > 0 ? rr.flo - rr.lo : np;
    const size_t row = static_cast<size_t>(i) * n_kv;
    for (int e = threadIdx.x; e < n_kv; e += blockDim.x) {
      kv_idx[row + e] = e < np ? (e < part_a ? rr.lo + e : rr.fhi + 1 + (e - part_a)) : 0;
      full_idx[row + e] = e < nf ? rr.flo + e : 0;
    }
    // rank = rows with a larger live count + earlier rows with the same count
    const int c = live_cnt[i];
    int rank = 0;
    for (int r = threadIdx.x; r < n_q; r += blockDim.x) {
      const int cr = live_cnt[r];
      rank += (cr > c || (cr == c && r < i)) ? 1 : 0;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) rank += __shfl_xor_sync(0xffffffffu, rank, o);
    if (lane == 0) warp_sum[warp] = rank;
    __syncthreads();
    if (threadIdx.x == 0) {
      int total = 0;
      for (int w = 0; w < kClassifyThreads / 32; ++w) total += warp_sum[w];
      kv_num[i] = np;
      full_num[i] = nf;
      sched[2 * total] = i;
      sched[2 * total + 1] = np | (nf << 16);
    }
    __syncthreads();
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
  // programmatic dependent launch: the tables are complete before they are read
  grid_dep_wait();
  grid_dep_launch_dependents();
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
  if (kind == FA_MASK_CAUSAL || kind == FA_MASK_SLIDING_WINDOW_CAUSAL) {
    // closed forms: lists, counts and schedule in one launch
    const int sms = num_sms_current_device();
    if (sms <= 0) return FA_ERR_CUDA;
    const int grid = nq < 2 * sms ? nq : 2 * sms;
    FA_CUDA_CHECK(launch_pdl(interval_tables_kernel, dim3(grid, inst), dim3(kClassifyThreads),
                             nq * sizeof(int32_t), s, kind, bm->window, q_len, kv_len, nq, nkv,
                             bm->kv_num_blocks, bm->kv_indices, bm->full_kv_num_blocks,
                             bm->full_kv_indices, bm->q_order));
    return FA_OK;
  }
  // shared memory: a class byte per kv block, and for tabulated masks two bit words
  // per 32 blocks (any / all bits set)
  const size_t cls_smem = static_cast<size_t>((nkv + 15) & ~15) + 16 +
                          (kind == FA_MASK_BITMAP ? 8 * static_cast<size_t>((nkv + 31) / 32) : 0);
  FA_CUDA_CHECK(launch_pdl(classify_rows_kernel, dim3(nq, inst), dim3(kClassifyThreads),
                           cls_smem, s, kind, bm->window, bm->doc_id,
                           bm->bitmap, q_len, kv_len, nkv, bm->kv_num_blocks, bm->kv_indices,
                           bm->full_kv_num_blocks, bm->full_kv_indices));
  int n_pow2 = 1;
  while (n_pow2 < nq) n_pow2 <<= 1;
  const size_t order_smem = (nq <= 2048 ? nq : n_pow2) * sizeof(uint32_t);
  FA_CUDA_CHECK(launch_pdl(order_rows_kernel, dim3(inst), dim3(kOrderThreads), order_smem, s, nq,
                           nkv, n_pow2, bm->kv_num_blocks, bm->full_kv_num_blocks, bm->q_order));
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
  FA_CUDA_CHECK(launch_pdl(transpose_kernel, dim3(nkv, inst), dim3(kClassifyThreads),
                           static_cast<size_t>(nq), as_stream(stream), nq, nkv, bm->kv_num_blocks,
                           bm->kv_indices, bm->full_kv_num_blocks, bm->full_kv_indices,
                           q_num_blocks, q_indices, full_q_num_blocks, full_q_indices));
  return FA_OK;
}
