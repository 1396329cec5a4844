// Host-side validation of BlockMask tables (no CUDA call).  The forward kernel
// trusts the tables it is given: a partial count above nKV, an index out of range
// or a schedule entry pointing at a wrong row would make it read outside the
// tables or K / V.  Tables built by this library's builders are correct by
// construction; tables from elsewhere (built by the caller, deserialised, edited)
// can be checked here first, on host copies.
//
// The conditions restate the table layout of the FlexAttention BlockMask
// (FlexAttention vs SDPA on M1 Max, qiita kiarina, "役割とデータの流れ"; FlexAttention
// how-to, dreaming.press, "The two mistakes..."): per q-block row, the PARTIAL and
// the FULL kv blocks, each list ascending, disjoint, padded with zeros.
#include <cstdint>
#include <vector>

#include "fa.h"

namespace {

bool check_list(const int32_t* idx, int32_t num, int32_t n_kv, std::vector<uint8_t>& seen) {
  int32_t prev = -1;
  for (int32_t j = 0; j < num; ++j) {
    const int32_t b = idx[j];
    if (b < 0 || b >= n_kv || b <= prev || seen[b]) return false;
    seen[b] = 1;
    prev = b;
  }
  for (int32_t j = num; j < n_kv; ++j)
    if (idx[j] != 0) return false;
  return true;
}

}  // namespace

extern "C" FA_API fa_status fa_block_mask_validate(
    const int32_t* kv_num_blocks, const int32_t* kv_indices, const int32_t* full_kv_num_blocks,
    const int32_t* full_kv_indices, const int32_t* q_order, int32_t n_q_blocks,
    int32_t n_kv_blocks, int32_t instances, int64_t* first_bad) {
  if (first_bad != nullptr) *first_bad = -1;
  if (n_q_blocks < 0 || n_kv_blocks < 0 || instances < 1 || n_q_blocks > FA_MAX_LEN / FA_BLOCK ||
      n_kv_blocks > FA_MAX_LEN / FA_BLOCK)
    return FA_ERR_INVALID_ARG;
  if (n_q_blocks == 0) return FA_OK;
  if (kv_num_blocks == nullptr || full_kv_num_blocks == nullptr || q_order == nullptr ||
      (n_kv_blocks > 0 && (kv_indices == nullptr || full_kv_indices == nullptr)))
    return FA_ERR_INVALID_ARG;
  const int64_t nq = n_q_blocks, nkv = n_kv_blocks;
  std::vector<uint8_t> seen(static_cast<size_t>(nkv > 0 ? nkv : 1));
  std::vector<uint8_t> ranked(static_cast<size_t>(nq));
  for (int64_t inst = 0; inst < instances; ++inst) {
    const int32_t* np = kv_num_blocks + inst * nq;
    const int32_t* nf = full_kv_num_blocks + inst * nq;
    // rows: counts, ranges, order, disjointness, zero padding
    for (int64_t i = 0; i < nq; ++i) {
      const int64_t where = inst * nq + i;
      if (np[i] < 0 || nf[i] < 0 || static_cast<int64_t>(np[i]) + nf[i] > nkv || np[i] > 0xFFFF ||
          nf[i] > 0xFFFF) {
        if (first_bad != nullptr) *first_bad = where;
        return FA_ERR_INVALID_ARG;
      }
      if (nkv == 0) continue;
      std::fill(seen.begin(), seen.end(), 0);
      const int64_t row = (inst * nq + i) * nkv;
      if (!check_list(kv_indices + row, np[i], n_kv_blocks, seen) ||
          !check_list(full_kv_indices + row, nf[i], n_kv_blocks, seen)) {
        if (first_bad != nullptr) *first_bad = where;
        return FA_ERR_INVALID_ARG;
      }
    }
    // schedule: every row once, with its counts, by descending live count, then row
    const int32_t* ord = q_order + inst * 2 * nq;
    std::fill(ranked.begin(), ranked.end(), 0);
    int64_t prev_n = -1, prev_row = -1;
    for (int64_t k = 0; k < nq; ++k) {
      const int32_t r = ord[2 * k];
      const uint32_t packed = static_cast<uint32_t>(ord[2 * k + 1]);
      const int64_t where = inst * nq + (r >= 0 && r < nq ? r : 0);
      bool ok = r >= 0 && r < nq && !ranked[r];
      if (ok) {
        ranked[r] = 1;
        ok = static_cast<int32_t>(packed & 0xFFFFu) == np[r] &&
             static_cast<int32_t>(packed >> 16) == nf[r];
        const int64_t n = static_cast<int64_t>(np[r]) + nf[r];
        ok = ok && (k == 0 || n < prev_n || (n == prev_n && r > prev_row));
        prev_n = n;
        prev_row = r;
      }
      if (!ok) {
        if (first_bad != nullptr) *first_bad = where;
        return FA_ERR_INVALID_ARG;
      }
    }
  }
  return FA_OK;
}
