// Backward pass of the block-sparse attention forward (FlashAttention-2 article,
// "あえて再計算して転送を減らす": recompute the attention matrix on chip from the
// saved inputs and the row statistics instead of storing it).  With the forward's
// LSE, P = exp(s - LSE) is recomputed block by block over the same BlockMask:
//
//   delta_i = rowsum(dO_i * O_i)
//   dS_ij  = P_ij (dO_i . v_j - delta_i)     (times 1 - tanh^2 under the softcap)
//   dQ_i   = scale * sum_j dS_ij k_j          (q-block rows: the kv lists)
//   dK_j   = scale * sum_i dS_ij q_i,  dV_j = sum_i P_ij dO_i
//                                            (kv-block columns: the column lists)
//
// Three kernels: delta (a warp per row); dK and dV, one CTA per 128-key tile over
// its column lists and the query heads that share its K/V head; dQ, one CTA per
// 128-query tile over its row lists, in the forward's schedule order.  Every
// output tile is owned by one CTA (no atomics, deterministic; dQ recomputes S and
// dP instead of accumulating into global memory).
//
// Both gradient kernels have one shape: a stationary 128-row tile pair (dK/dV: K
// and V; dQ: Q and dO) and 64-row sub-tiles of the other pair streamed through a
// two-stage shared-memory ring by TMA.  Per sub-tile the products run on the 5th-
// generation tensor cores with fp32 accumulators in Tensor Memory:
//   X = A0 B0^T, Y = A1 B1^T     (SS MMAs, M = 128, N = 64, K = D)
//     dK/dV: X = S^T = K Q^T, Y = dP^T = V dO^T;   dQ: X = S = Q K^T, Y = dP = dO V^T
//   thread t of the compute warpgroup owns TMEM lane t (row t of the stationary
//   tile): it turns its row of X and Y into P and dS, rounded to 16 bits and
//   written back over X and Y, as the A operands of
//   dK/dV: dV += P^T dO, dK += dS^T Q;   dQ: dQ += dS K
//     (TS MMAs: A from TMEM, B the streamed tile read MN-major, accumulators in TMEM).
// Warps 0-3 compute, warp 4 loads (TMA, and the row statistics the sub-tile needs),
// warp 5 issues the MMAs and owns TMEM.  The next sub-tile's X and Y are issued
// right after the current one's accumulating products by the same thread, so they
// overwrite P and dS only after those products have read them (tcgen05 operations
// of one thread run in issue order).  At D = 64 a CTA takes 256 TMEM columns and two
// CTAs share an SM, so one CTA's MMAs overlap the other's elementwise work.
//
// Every mbarrier wait is bounded (2 s): on expiry the kernel sets the error word
// (word 0 of the workspace), stops every role, drains its copies and MMAs, frees
// TMEM and returns; fa_get_last_device_error reports FA_ERR_TIMEOUT.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kBwdWarps = 8;  // delta kernel
constexpr float kBwdLog2e = 1.4426950408889634f;
constexpr int kSub = 64;                    // rows of a streamed sub-tile
constexpr int kTcThreads = 192;             // warps 0-3 compute, 4 loads, 5 MMA
constexpr int kLoadWarp = 4;
constexpr int kIssueWarp = 5;
constexpr int kModeDkdv = 0;
constexpr int kModeDq = 1;
constexpr int kBwdWorkspaceHeader = 256;  // word 0: device error flags, then delta

struct BwdParams {
  const uint16_t *q, *k, *v, *out, *dout;
  const float* lse;
  float* delta;
  int32_t* err;
  uint16_t *dq, *dk, *dv;
  const int32_t *kv_num, *kv_idx, *full_num, *full_idx;      // row lists
  const int32_t *q_num, *q_idx, *full_q_num, *full_q_idx;   // column lists
  const int32_t* sched;                                      // forward's q-block order
  const int32_t* doc_id;
  const uint32_t* bitmap;
  int B, H, Hkv, G, L, S, n_q, n_kv, kind, window, softcap_on, is_bf16;
  // per-(batch, head) masks: instance of (b, h) = (mask_b ? b : 0) * mask_heads +
  // (mask_h ? h : 0), with its own lists, schedule, ids or bitmap rows
  int mask_b, mask_h, mask_heads, doc_len;
  float scale, scale_log2, cap_c, cap_k;
  unsigned long long timeout_ns;
  int stall;  // testing hook: nothing is loaded, the waits run out
  int dkdv_overlaps_dq;  // dK/dV launched right after dQ (see bwd_tc_kernel)
};

// delta_i = rowsum(dO_i * O_i) over the B * H * L rows: D / 8 lanes per row, each
// reading 16 bytes of O and of dO (so a warp covers 32 * 8 / D rows per pass), the
// partial sums combined by shuffles within the row's lanes; grid-stride over rows.
template <int D>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_delta_kernel(const BwdParams p) {
  // programmatic dependent launch: O and dO are complete; dQ may start its prologue
  grid_dep_wait();
  grid_dep_launch_dependents();
  constexpr int kLanes = D / 8;                // lanes per row
  constexpr int kRowsPerBlock = kBwdWarps * 32 / kLanes;
  const int64_t rows = static_cast<int64_t>(p.B) * p.H * p.L;
  const bool bf16 = p.is_bf16 != 0;
  const int sub = threadIdx.x % kLanes;
  // the loop runs while the block's first row is in range (uniform over the block),
  // so every lane reaches the shuffles; rows past the end load and store nothing
  for (int64_t first = static_cast<int64_t>(blockIdx.x) * kRowsPerBlock; first < rows;
       first += static_cast<int64_t>(gridDim.x) * kRowsPerBlock) {
    const int64_t row = first + threadIdx.x / kLanes;
    const bool in = row < rows;
    const int64_t off = (in ? row : 0) * D + sub * 8;
    const uint4 o4 = __ldg(reinterpret_cast<const uint4*>(p.out + off));
    const uint4 g4 = __ldg(reinterpret_cast<const uint4*>(p.dout + off));
    const uint32_t ow[4] = {o4.x, o4.y, o4.z, o4.w}, gw[4] = {g4.x, g4.y, g4.z, g4.w};
    float acc = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 o, g;
      if (bf16) {
        o = make_float2(__uint_as_float(ow[i] << 16), __uint_as_float(ow[i] & 0xFFFF0000u));
        g = make_float2(__uint_as_float(gw[i] << 16), __uint_as_float(gw[i] & 0xFFFF0000u));
      } else {
        o = __half22float2(*reinterpret_cast<const __half2*>(&ow[i]));
        g = __half22float2(*reinterpret_cast<const __half2*>(&gw[i]));
      }
      acc = fmaf(o.x, g.x, fmaf(o.y, g.y, acc));
    }
#pragma unroll
    for (int s = kLanes / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s, kLanes);
    if (in && sub == 0) p.delta[row] = acc;
  }
}

// ---------------------------------------------------------------- tcgen05 kernels
template <int D>
struct TcCfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kStatBytes = 128 * D * 2;    // a stationary 128-row tile
  static constexpr int kSubBytes = kSub * D * 2;    // a streamed 64-row tile
  static constexpr int kStatChunk = 128 * 128;      // one 64-column box of 128 rows
  static constexpr int kSubChunk = kSub * 128;      // one 64-column box of 64 rows
  // TMEM: X [0, 64), Y [64, 128), accumulators from 128 (D columns each)
  __host__ __device__ static constexpr uint32_t tmem_cols(int mode) {
    return (128 + (mode == kModeDkdv ? 2 : 1) * D) <= 256 ? 256u : 512u;
  }
  static constexpr int kCtasPerSm = D == 64 ? 2 : 1;
};

template <int D>
struct __align__(1024) TcSmem {
  uint8_t stat[2][TcCfg<D>::kStatBytes];            // dK/dV: K, V;  dQ: Q, dO
  uint8_t sub[2][2][TcCfg<D>::kSubBytes];           // [stage][operand] dK/dV: Q, dO; dQ: K, V
  float lse2[2][kSub];                              // dK/dV: per streamed query row
  float delta[2][kSub];
  int32_t aux[2][kSub * 4];                         // partial blocks: ids or bitmap words
  uint64_t stat_full;
  uint64_t full[2], empty[2];
  uint64_t x_full, comp_done, acc_full, drain;
  uint32_t tmem_base;
  volatile int abort_flag;
};

// Mask instance of (batch, head).
__device__ __forceinline__ int bwd_instance(const BwdParams& p, int64_t bh) {
  const int64_t b = bh / p.H, h = bh - b * p.H;
  return static_cast<int>((p.mask_b ? b : 0) * p.mask_heads + (p.mask_h ? h : 0));
}

// The sequence of 64-row sub-tiles one CTA streams.  dK/dV (CTA = key tile jb of K/V
// head kvbh): for each query head of the group, each block of column jb's lists,
// both halves of the q block.  dQ (CTA = query tile qb of head bh): each block of
// row qb's lists, both halves of the kv block.  Every role walks the same sequence.
template <int MODE>
struct StepIter {
  // fixed per CTA
  int64_t tile_bh;  // dK/dV: kvbh; dQ: bh
  int tile_blk;     // dK/dV: jb; dQ: qb
  // current list
  int g, np, nf, t, half;
  int64_t list_base;
  int inst;
  // current step
  int64_t bh;     // query head of the step (dK/dV) / of the tile (dQ)
  int blk;        // dK/dV: q block; dQ: kv block
  bool full;

  __device__ __forceinline__ void open_list(const BwdParams& p) {
    if constexpr (MODE == kModeDkdv) {
      const int64_t b = tile_bh / p.Hkv, kvh = tile_bh - b * p.Hkv;
      bh = b * p.H + kvh * p.G + g;
      inst = bwd_instance(p, bh);
      const int64_t col = static_cast<int64_t>(inst) * p.n_kv + tile_blk;
      np = p.n_q > 0 ? __ldg(p.q_num + col) : 0;
      nf = p.n_q > 0 ? __ldg(p.full_q_num + col) : 0;
      list_base = col * p.n_q;
    } else {
      bh = tile_bh;
      inst = bwd_instance(p, bh);
      const int64_t row = static_cast<int64_t>(inst) * p.n_q + tile_blk;
      np = p.n_kv > 0 ? __ldg(p.kv_num + row) : 0;
      nf = p.n_kv > 0 ? __ldg(p.full_num + row) : 0;
      list_base = row * p.n_kv;
    }
    t = 0;
    half = 0;
  }
  __device__ __forceinline__ void init(const BwdParams& p, int64_t tbh, int tblk) {
    tile_bh = tbh;
    tile_blk = tblk;
    g = 0;
    open_list(p);
  }
  // Advance to the next step; false when the sequence is exhausted.
  __device__ __forceinline__ bool next(const BwdParams& p) {
    while (t >= np + nf) {
      if (MODE == kModeDq || ++g >= p.G) return false;
      open_list(p);
    }
    full = t >= np;
    const int32_t* idx = MODE == kModeDkdv ? (full ? p.full_q_idx : p.q_idx)
                                           : (full ? p.full_idx : p.kv_idx);
    blk = __ldg(idx + list_base + (full ? t - np : t));
    return true;
  }
  __device__ __forceinline__ int row0() const { return blk * 128 + half * kSub; }
  __device__ __forceinline__ void step() {
    if (++half == 2) {
      half = 0;
      ++t;
    }
  }
};

template <int D>
__device__ __noinline__ bool tc_wait_slow(TcSmem<D>& sm, uint64_t* bar, uint32_t parity,
                                          const BwdParams& p) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (sm.abort_flag) return false;
    if (globaltimer_ns() - t0 > p.timeout_ns) {
      sm.abort_flag = 1;
      atomicOr(p.err, kDevErrTimeout);
      return false;
    }
  }
}
template <int D>
__device__ __forceinline__ bool tc_wait(TcSmem<D>& sm, uint64_t* bar, uint32_t parity,
                                        const BwdParams& p) {
  if (mbar_try_wait(bar, parity)) return true;
  return tc_wait_slow(sm, bar, parity, p);
}
// whole warp waits; the warp agrees on the outcome
template <int D>
__device__ __forceinline__ bool tc_wait_warp(TcSmem<D>& sm, uint64_t* bar, uint32_t parity,
                                             const BwdParams& p) {
  return __all_sync(0xffffffffu, tc_wait(sm, bar, parity, p));
}
// lane 0 waits, the warp gets the outcome
template <int D>
__device__ __forceinline__ bool tc_wait_lane0(TcSmem<D>& sm, uint64_t* bar, uint32_t parity,
                                              const BwdParams& p) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = tc_wait(sm, bar, parity, p);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

template <int D>
__device__ __forceinline__ void tma_tile(const CUtensorMap* map, int row0, int64_t z, uint8_t* dst,
                                         int chunk_bytes, uint64_t* bar, uint64_t pol) {
#pragma unroll
  for (int c = 0; c < TcCfg<D>::kChunks; ++c)
    tma_load_3d(dst + c * chunk_bytes, map, bar, c * 64, row0, static_cast<int32_t>(z), pol);
}

// Warp 4: the stationary tiles once, then per step the two streamed sub-tiles (TMA)
// and what the compute warps need per streamed row: dK/dV the query rows' log2-scale
// LSE and delta; PARTIAL blocks of document / tabulated masks the ids / words.
template <int MODE, int D>
__device__ void tc_load_role(TcSmem<D>& sm, const BwdParams& p, const CUtensorMap* ts0,
                             const CUtensorMap* ts1, const CUtensorMap* tb0, const CUtensorMap* tb1,
                             int64_t tile_bh, int tile_blk, int64_t stat_z) {
  using C = TcCfg<D>;
  const int lane = threadIdx.x & 31;
  const uint64_t pol = policy_evict_last();
  if (p.stall) return;  // testing hook: nothing is loaded
  if (lane == 0) {
    mbar_arrive_expect_tx(&sm.stat_full, 2 * C::kStatBytes);
    tma_tile<D>(ts0, tile_blk * 128, stat_z, sm.stat[0], C::kStatChunk, &sm.stat_full, pol);
    tma_tile<D>(ts1, tile_blk * 128, stat_z, sm.stat[1], C::kStatChunk, &sm.stat_full, pol);
  }
  StepIter<MODE> it;
  it.init(p, tile_bh, tile_blk);
  int s = 0;
  bool ok = true;
  for (; it.next(p); it.step(), ++s) {
    const int st = s & 1;
    if (!tc_wait_lane0(sm, &sm.empty[st], ((s >> 1) & 1) ^ 1, p)) {
      ok = false;
      break;
    }
    const int r0 = it.row0();
    // the streamed rows: dK/dV query rows of head it.bh; dQ key rows of its K/V head
    const int64_t kvbh = MODE == kModeDkdv ? tile_bh
                                           : (it.bh / p.H) * p.Hkv + (it.bh % p.H) / p.G;
    if constexpr (MODE == kModeDkdv) {
      for (int r = lane; r < kSub; r += 32) {
        const int i = r0 + r;
        float l2 = INFINITY, dl = 0.f;  // rows past L, or with no live key: P = 0
        if (i < p.L) {
          const float l = __ldg(p.lse + it.bh * p.L + i);
          if (l != -INFINITY) {
            l2 = l * kBwdLog2e;
            dl = p.delta[it.bh * p.L + i];
          }
        }
        sm.lse2[st][r] = l2;
        sm.delta[st][r] = dl;
      }
    }
    if (!it.full && p.kind == FA_MASK_DOCUMENT_CAUSAL) {
      // ids of the streamed rows (queries for dK/dV, keys for dQ) of this instance
      const int32_t* docs = p.doc_id + static_cast<int64_t>(it.inst) * p.doc_len;
      const int n = MODE == kModeDkdv ? p.L : p.S;
      for (int r = lane; r < kSub; r += 32) sm.aux[st][r] = __ldg(docs + min(r0 + r, n - 1));
    } else if (MODE == kModeDkdv && !it.full && p.kind == FA_MASK_BITMAP) {
      // the 4 words of key tile tile_blk in each of the 64 query rows
      const uint32_t* rows = p.bitmap + static_cast<int64_t>(it.inst) * p.L * 4 * p.n_kv;
      for (int e = lane; e < kSub * 4; e += 32) {
        const int i = min(r0 + e / 4, p.L - 1);
        sm.aux[st][e] = static_cast<int32_t>(
            __ldg(rows + static_cast<int64_t>(i) * 4 * p.n_kv + 4 * tile_blk + (e & 3)));
      }
    }
    __syncwarp();
    if (lane == 0) {
      mbar_arrive_expect_tx(&sm.full[st], 2 * C::kSubBytes);
      const int64_t z = MODE == kModeDkdv ? it.bh : kvbh;
      tma_tile<D>(tb0, r0, z, sm.sub[st][0], C::kSubChunk, &sm.full[st], pol);
      tma_tile<D>(tb1, r0, z, sm.sub[st][1], C::kSubChunk, &sm.full[st], pol);
    }
    __syncwarp();
  }
  if (!ok && lane == 0) {
    // let the copies in flight land (bounded) before the CTA exits
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&sm.stat_full, 0) && globaltimer_ns() - t0 < p.timeout_ns) {
    }
    for (int u = s - 2; u < s; ++u) {
      if (u < 0) continue;
      while (!mbar_try_wait(&sm.full[u & 1], (u >> 1) & 1) && globaltimer_ns() - t0 < p.timeout_ns) {
      }
    }
  }
}

// Warp 5: per step s, the accumulating products of step s - 1 (once its P / dS are
// written), then X and Y of step s.
template <int MODE, int D>
__device__ void tc_issue_role(TcSmem<D>& sm, const BwdParams& p, uint32_t tmem, int64_t tile_bh,
                              int tile_blk) {
  using C = TcCfg<D>;
  const bool bf16 = p.is_bf16 != 0;
  const uint32_t id_x = idesc_f16_f32(bf16, 128, kSub, false);
  const uint32_t id_acc = idesc_f16_f32(bf16, 128, D, true);
  const uint32_t t_x = tmem, t_y = tmem + 64, t_acc0 = tmem + 128, t_acc1 = tmem + 128 + D;
  StepIter<MODE> it;
  it.init(p, tile_bh, tile_blk);
  bool ok = tc_wait_lane0(sm, &sm.stat_full, 0, p);
  int s = 0;
  bool acc_started = false;
  // the accumulating products of the step whose operands sit in stage st
  auto issue_acc = [&](int st) {
    if (elect_one_sync()) {
#pragma unroll
      for (int kk = 0; kk < kSub / 16; ++kk) {
        const uint32_t acc = (acc_started || kk > 0) ? 1u : 0u;
        if constexpr (MODE == kModeDkdv) {
          // dV += P^T dO (B = dO sub-tile, MN-major), dK += dS^T Q (B = Q sub-tile)
          const uint64_t bdo = sdesc_sw128(smem_u32(sm.sub[st][1]), C::kSubChunk, 1024);
          const uint64_t bq = sdesc_sw128(smem_u32(sm.sub[st][0]), C::kSubChunk, 1024);
          umma_ts(t_acc0, t_x + kk * 8, bdo + static_cast<uint64_t>(kk * 128), id_acc, acc);
          umma_ts(t_acc1, t_y + kk * 8, bq + static_cast<uint64_t>(kk * 128), id_acc, acc);
        } else {
          // dQ += dS K (B = K sub-tile, MN-major)
          const uint64_t bk = sdesc_sw128(smem_u32(sm.sub[st][0]), C::kSubChunk, 1024);
          umma_ts(t_acc0, t_y + kk * 8, bk + static_cast<uint64_t>(kk * 128), id_acc, acc);
        }
      }
      umma_commit(&sm.empty[st]);
    }
    __syncwarp();
    acc_started = true;
  };
  for (; ok && it.next(p); it.step(), ++s) {
    const int st = s & 1;
    if (s > 0) {
      ok = tc_wait_lane0(sm, &sm.comp_done, (s - 1) & 1, p);
      if (!ok) break;
      tc_fence_after();
      issue_acc(st ^ 1);
    }
    ok = tc_wait_lane0(sm, &sm.full[st], (s >> 1) & 1, p);
    if (!ok) break;
    tc_fence_after();
    if (elect_one_sync()) {
      const uint64_t a0 = sdesc_sw128(smem_u32(sm.stat[0]), 16, 1024);
      const uint64_t a1 = sdesc_sw128(smem_u32(sm.stat[1]), 16, 1024);
      const uint64_t b0 = sdesc_sw128(smem_u32(sm.sub[st][0]), 16, 1024);
      const uint64_t b1 = sdesc_sw128(smem_u32(sm.sub[st][1]), 16, 1024);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        // K step kk: 32 bytes into the 128-byte swizzled rows, 64-column box kk / 4
        const uint64_t oa = static_cast<uint64_t>(((kk >> 2) * C::kStatChunk + (kk & 3) * 32) >> 4);
        const uint64_t ob = static_cast<uint64_t>(((kk >> 2) * C::kSubChunk + (kk & 3) * 32) >> 4);
        umma_ss(t_x, a0 + oa, b0 + ob, id_x, kk > 0 ? 1u : 0u);
        umma_ss(t_y, a1 + oa, b1 + ob, id_x, kk > 0 ? 1u : 0u);
      }
      umma_commit(&sm.x_full);
    }
    __syncwarp();
  }
  if (ok && s > 0) {
    ok = tc_wait_lane0(sm, &sm.comp_done, (s - 1) & 1, p);
    if (ok) {
      tc_fence_after();
      issue_acc((s - 1) & 1);
    }
  }
  if (ok) {
    if (elect_one_sync()) umma_commit(&sm.acc_full);  // with no step: arrives at once
    __syncwarp();
  } else {
    // drain every MMA this warp issued before TMEM is released
    if (elect_one_sync()) umma_commit(&sm.drain);
    __syncwarp();
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&sm.drain, 0) && globaltimer_ns() - t0 < p.timeout_ns) {
    }
  }
}

__device__ __forceinline__ uint32_t pack16(float lo, float hi, bool bf16) {
  if (bf16) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// What one 32-column group of a step needs besides X and Y.
struct GroupArgs {
  const float* lse2;   // dK/dV: the columns' log2-scale LSE and delta (shared memory)
  const float* delta;
  const int32_t* aux;  // PARTIAL blocks: the columns' document ids / tabulated words
  float my_l2, my_dl;  // dQ: this row's
  int my, r0, c0;      // this thread's row index; first streamed row; first column
  int my_id;           // documents: this row's id
  uint32_t word;       // dQ tabulated masks: this row's word for the group's 32 keys
};

// P and dS for 32 columns of this thread's row, packed to 16-bit pairs.  FULL,
// SOFTCAP and the mask KIND are compile-time, so a step runs one short variant.
template <int MODE, bool FULL, bool SOFTCAP, int KIND>
__device__ __forceinline__ void group_grads(const BwdParams& p, const uint32_t (&xr)[32],
                                            const uint32_t (&yr)[32], const GroupArgs& a,
                                            bool bf16, uint32_t (&pk_p)[16], uint32_t (&pk_d)[16]) {
#pragma unroll
  for (int c2 = 0; c2 < 16; ++c2) {
    float pv[2], dv[2];
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int cc = 2 * c2 + e;  // column a.c0 + cc: streamed row a.r0 + a.c0 + cc
      const float x = __uint_as_float(xr[cc]);
      const float y = __uint_as_float(yr[cc]);
      const float l2 = MODE == kModeDkdv ? a.lse2[a.c0 + cc] : a.my_l2;
      const float dl = MODE == kModeDkdv ? a.delta[a.c0 + cc] : a.my_dl;
      // s (log2 units) and the softcap's derivative, tanh y = 1 - 2 / (e^{2y} + 1)
      float sl2, dcap = 1.f;
      if constexpr (SOFTCAP) {
        const float th = 1.f - 2.f * rcp_approx(ex2_approx(x * p.cap_k) + 1.f);
        sl2 = p.cap_c * kBwdLog2e * th;
        dcap = 1.f - th * th;
      } else {
        sl2 = x * p.scale_log2;
      }
      const float pij = ex2_approx(sl2 - l2);
      float dsij = pij * (y - dl);
      if constexpr (SOFTCAP) dsij *= dcap;
      bool keep = true;
      if constexpr (!FULL) {
        const int other = a.r0 + a.c0 + cc;
        const int i = MODE == kModeDkdv ? other : a.my;
        const int j = MODE == kModeDkdv ? a.my : other;
        keep = i < p.L && j < p.S;
        if constexpr (KIND == FA_MASK_CAUSAL) {
          keep = keep && j <= i;
        } else if constexpr (KIND == FA_MASK_SLIDING_WINDOW_CAUSAL) {
          keep = keep && j <= i && i - j < p.window;
        } else if constexpr (KIND == FA_MASK_DOCUMENT_CAUSAL) {
          keep = keep && j <= i && a.aux[a.c0 + cc] == a.my_id;
        } else {
          const uint32_t w = MODE == kModeDkdv
                                 ? static_cast<uint32_t>(a.aux[(a.c0 + cc) * 4 + ((a.my >> 5) & 3)])
                                 : a.word;
          keep = keep && ((w >> (j & 31)) & 1u) != 0u;
        }
      }
      pv[e] = keep ? pij : 0.f;
      dv[e] = keep ? dsij : 0.f;
    }
    pk_p[c2] = pack16(pv[0], pv[1], bf16);
    pk_d[c2] = pack16(dv[0], dv[1], bf16);
  }
}

template <int MODE, bool SOFTCAP>
__device__ __forceinline__ void group_dispatch(const BwdParams& p, bool full,
                                               const uint32_t (&xr)[32], const uint32_t (&yr)[32],
                                               const GroupArgs& a, bool bf16, uint32_t (&pk_p)[16],
                                               uint32_t (&pk_d)[16]) {
  if (full) {
    group_grads<MODE, true, SOFTCAP, 0>(p, xr, yr, a, bf16, pk_p, pk_d);
  } else {
    switch (p.kind) {
      case FA_MASK_CAUSAL:
        group_grads<MODE, false, SOFTCAP, FA_MASK_CAUSAL>(p, xr, yr, a, bf16, pk_p, pk_d);
        break;
      case FA_MASK_SLIDING_WINDOW_CAUSAL:
        group_grads<MODE, false, SOFTCAP, FA_MASK_SLIDING_WINDOW_CAUSAL>(p, xr, yr, a, bf16, pk_p, pk_d);
        break;
      case FA_MASK_DOCUMENT_CAUSAL:
        group_grads<MODE, false, SOFTCAP, FA_MASK_DOCUMENT_CAUSAL>(p, xr, yr, a, bf16, pk_p, pk_d);
        break;
      default:
        group_grads<MODE, false, SOFTCAP, FA_MASK_BITMAP>(p, xr, yr, a, bf16, pk_p, pk_d);
        break;
    }
  }
}

// Warps 0-3: thread t owns row t of the stationary tile (TMEM lane t).
template <int MODE, int D>
__device__ void tc_compute_role(TcSmem<D>& sm, const BwdParams& p, uint32_t tmem, int64_t tile_bh,
                                int tile_blk) {
  const int t = threadIdx.x;
  const uint32_t lane_off = static_cast<uint32_t>((t >> 5) * 32) << 16;
  const uint32_t t_x = tmem + lane_off, t_y = tmem + 64 + lane_off;
  const uint32_t t_acc0 = tmem + 128 + lane_off, t_acc1 = tmem + 128 + D + lane_off;
  const bool bf16 = p.is_bf16 != 0;
  // this thread's row: dK/dV key j of K/V head tile_bh; dQ query i of head tile_bh
  GroupArgs a;
  a.my = tile_blk * 128 + t;
  a.my_l2 = INFINITY;
  a.my_dl = 0.f;
  if (MODE == kModeDq && a.my < p.L) {
    const float l = __ldg(p.lse + tile_bh * p.L + a.my);
    if (l != -INFINITY) {
      a.my_l2 = l * kBwdLog2e;
      a.my_dl = p.delta[tile_bh * p.L + a.my];
    }
  }
  StepIter<MODE> it;
  it.init(p, tile_bh, tile_blk);
  int s = 0;
  for (; it.next(p); it.step(), ++s) {
    const int st = s & 1;
    if (!tc_wait_warp(sm, &sm.x_full, s & 1, p)) return;
    tc_fence_after();
    a.r0 = it.row0();
    a.lse2 = sm.lse2[st];
    a.delta = sm.delta[st];
    a.aux = sm.aux[st];
    a.my_id = 0;
    uint32_t w_lo = 0, w_hi = 0;
    // the thread's own id / words for PARTIAL blocks of document / tabulated masks
    if (!it.full && p.kind == FA_MASK_DOCUMENT_CAUSAL) {
      const int n = MODE == kModeDkdv ? p.S : p.L;
      a.my_id = __ldg(p.doc_id + static_cast<int64_t>(it.inst) * p.doc_len + min(a.my, n - 1));
    } else if (MODE == kModeDq && !it.full && p.kind == FA_MASK_BITMAP) {
      const uint32_t* row = p.bitmap + (static_cast<int64_t>(it.inst) * p.L + min(a.my, p.L - 1)) *
                                           4 * p.n_kv;
      w_lo = __ldg(row + (a.r0 >> 5));
      w_hi = __ldg(row + (a.r0 >> 5) + 1);
    }
#pragma unroll 1
    for (int h = 0; h < 2; ++h) {
      uint32_t xr[32], yr[32];
      tmem_ld32(t_x + 32 * h, xr);
      tmem_ld32(t_y + 32 * h, yr);
      tmem_wait_ld();
      reg_fence32(xr);
      reg_fence32(yr);
      a.c0 = 32 * h;
      a.word = h == 0 ? w_lo : w_hi;
      uint32_t pk_p[16], pk_d[16];
      if (p.softcap_on)
        group_dispatch<MODE, true>(p, it.full, xr, yr, a, bf16, pk_p, pk_d);
      else
        group_dispatch<MODE, false>(p, it.full, xr, yr, a, bf16, pk_p, pk_d);
      // 16-bit results over the columns just read: P (dK/dV) at X [16h, 16h + 16),
      // dS at Y [16h, 16h + 16)
      if constexpr (MODE == kModeDkdv) tmem_st16(t_x + 16 * h, pk_p);
      tmem_st16(t_y + 16 * h, pk_d);
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if ((t & 31) == 0) mbar_arrive(&sm.comp_done);
  }
  // epilogue: the accumulators of this thread's row -> dK, dV or dQ
  const int my = a.my;
  const bool valid = MODE == kModeDkdv ? my < p.S : my < p.L;
  uint16_t* out0 = MODE == kModeDkdv ? p.dv : p.dq;   // dV (unscaled) / dQ (scaled)
  const size_t orow = static_cast<size_t>(tile_bh) * (MODE == kModeDkdv ? p.S : p.L) + my;
  if (s > 0) {
    if (!tc_wait_warp(sm, &sm.acc_full, 0, p)) return;
    tc_fence_after();
  }
#pragma unroll
  for (int ai = 0; ai < (MODE == kModeDkdv ? 2 : 1); ++ai) {
    uint16_t* dst = ai == 0 ? out0 : p.dk;
    const float f = (MODE == kModeDq || ai == 1) ? p.scale : 1.f;
    const uint32_t t_acc = ai == 0 ? t_acc0 : t_acc1;
#pragma unroll
    for (int c0 = 0; c0 < D / 32; ++c0) {
      uint32_t r[32];
      if (s > 0) {
        tmem_ld32(t_acc + 32 * c0, r);
        tmem_wait_ld();
        reg_fence32(r);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) r[e] = 0u;  // no live block: zero gradient
      }
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e)
        pk[e] = pack16(__uint_as_float(r[2 * e]) * f, __uint_as_float(r[2 * e + 1]) * f, bf16);
      if (valid) {
        uint4* o = reinterpret_cast<uint4*>(dst + orow * D + 32 * c0);
#pragma unroll
        for (int e = 0; e < 4; ++e) o[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
      }
    }
  }
}

template <int MODE, int D>
__global__ void __launch_bounds__(kTcThreads, TcCfg<D>::kCtasPerSm)
bwd_tc_kernel(const __grid_constant__ CUtensorMap ts0, const __grid_constant__ CUtensorMap ts1,
              const __grid_constant__ CUtensorMap tb0, const __grid_constant__ CUtensorMap tb1,
              const __grid_constant__ BwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  TcSmem<D>& sm = *reinterpret_cast<TcSmem<D>*>(smem_raw + ((1024u - (base & 1023u)) & 1023u));
  const int warp = threadIdx.x >> 5;
  constexpr uint32_t kCols = TcCfg<D>::tmem_cols(MODE);

  // the CTA's tile.  dK/dV: key tile jb of K/V head kvbh, columns in ascending jb
  // (the longest causal columns first).  dQ: query tile of head bh at rank `rank` of
  // its instance's schedule (longest rows first).
  int64_t tile_bh, stat_z;
  int tile_blk;
  if constexpr (MODE == kModeDkdv) {
    const int64_t n_kvbh = static_cast<int64_t>(p.B) * p.Hkv;
    tile_blk = static_cast<int>(blockIdx.x / n_kvbh);
    tile_bh = blockIdx.x - static_cast<int64_t>(tile_blk) * n_kvbh;
    stat_z = tile_bh;
  } else {
    const int64_t n_bh = static_cast<int64_t>(p.B) * p.H;
    const int rank = static_cast<int>(blockIdx.x / n_bh);
    tile_bh = blockIdx.x - static_cast<int64_t>(rank) * n_bh;
    const int64_t inst = bwd_instance(p, tile_bh);
    tile_blk = __ldg(p.sched + 2 * (inst * p.n_q + rank));
    stat_z = tile_bh;
  }

  if (threadIdx.x == 0) {
    mbar_init(&sm.stat_full, 1);
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.x_full, 1);
    mbar_init(&sm.comp_done, 4);  // one arrival per compute warp
    mbar_init(&sm.acc_full, 1);
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kLoadWarp && (threadIdx.x & 31) == 0) {
    prefetch_tensormap(&ts0);
    prefetch_tensormap(&ts1);
    prefetch_tensormap(&tb0);
    prefetch_tensormap(&tb1);
  }
  if (warp == kIssueWarp) {
    tmem_alloc(&sm.tmem_base, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  // Programmatic dependent launch.  dQ waits here for the row sums.  dK/dV launched
  // right after dQ reads nothing dQ writes, and its inputs (row sums, column lists)
  // were complete before any dQ CTA could let it launch, so it runs beside dQ's
  // last CTAs and waits for dQ only before it exits, which keeps the stream's
  // order; launched after anything else, it waits here.
  const bool overlap = MODE == kModeDkdv && p.dkdv_overlaps_dq != 0;
  if (!overlap) grid_dep_wait();
  grid_dep_launch_dependents();

  if (warp < 4) {
    tc_compute_role<MODE, D>(sm, p, tmem, tile_bh, tile_blk);
  } else if (warp == kLoadWarp) {
    tc_load_role<MODE, D>(sm, p, &ts0, &ts1, &tb0, &tb1, tile_bh, tile_blk, stat_z);
  } else {
    tc_issue_role<MODE, D>(sm, p, tmem, tile_bh, tile_blk);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kIssueWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
  if (overlap) grid_dep_wait();  // dQ has finished before this grid does
}

template <int MODE, int D>
fa_status tc_launch(const BwdParams& prm, bool bf16, cudaStream_t s) {
  CUtensorMap ts0, ts1, tb0, tb1;
  const int64_t BH = static_cast<int64_t>(prm.B) * prm.H, BHkv = static_cast<int64_t>(prm.B) * prm.Hkv;
  if (MODE == kModeDkdv) {
    if (!make_tile_map(&ts0, prm.k, bf16, D, prm.S, static_cast<int>(BHkv), 128)) return FA_ERR_CUDA;
    if (!make_tile_map(&ts1, prm.v, bf16, D, prm.S, static_cast<int>(BHkv), 128)) return FA_ERR_CUDA;
    if (!make_tile_map(&tb0, prm.q, bf16, D, prm.L, static_cast<int>(BH), kSub)) return FA_ERR_CUDA;
    if (!make_tile_map(&tb1, prm.dout, bf16, D, prm.L, static_cast<int>(BH), kSub)) return FA_ERR_CUDA;
  } else {
    if (!make_tile_map(&ts0, prm.q, bf16, D, prm.L, static_cast<int>(BH), 128)) return FA_ERR_CUDA;
    if (!make_tile_map(&ts1, prm.dout, bf16, D, prm.L, static_cast<int>(BH), 128)) return FA_ERR_CUDA;
    if (!make_tile_map(&tb0, prm.k, bf16, D, prm.S, static_cast<int>(BHkv), kSub)) return FA_ERR_CUDA;
    if (!make_tile_map(&tb1, prm.v, bf16, D, prm.S, static_cast<int>(BHkv), kSub)) return FA_ERR_CUDA;
  }
  const size_t smem = sizeof(TcSmem<D>) + 1024;
  int dev = 0;
  FA_CUDA_CHECK(cudaGetDevice(&dev));
  {
    static std::mutex mu;
    static bool done[kMaxDevices] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
    if (!done[dev]) {
      FA_CUDA_CHECK(cudaFuncSetAttribute(bwd_tc_kernel<MODE, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem)));
      done[dev] = true;
    }
  }
  const int64_t grid = MODE == kModeDkdv ? static_cast<int64_t>(prm.n_kv) * BHkv
                                         : static_cast<int64_t>(prm.n_q) * BH;
  if (grid == 0) return FA_OK;
  FA_CUDA_CHECK(launch_pdl(bwd_tc_kernel<MODE, D>, dim3(static_cast<unsigned>(grid)), dim3(kTcThreads),
                           smem, s, ts0, ts1, tb0, tb1, prm));
  return FA_OK;
}

template <int D>
fa_status bwd_launch(const BwdParams& prm_in, bool bf16, cudaStream_t s) {
  BwdParams prm = prm_in;
  const int64_t rows = static_cast<int64_t>(prm.B) * prm.H * prm.L;
  const int64_t krows = static_cast<int64_t>(prm.B) * prm.Hkv * prm.S;
  if (rows > 0) {
    // grid-stride: a few blocks per SM cover any row count
    const int64_t per_block = kBwdWarps * 32 / (D / 8);
    const int64_t want = (rows + per_block - 1) / per_block;
    const int sms = num_sms_current_device();
    const int64_t cap = static_cast<int64_t>(sms > 0 ? sms : 148) * 8;
    const unsigned qgrid = static_cast<unsigned>(want < cap ? want : cap);
    FA_CUDA_CHECK(launch_pdl(bwd_delta_kernel<D>, dim3(qgrid), dim3(kBwdWarps * 32), 0, s, prm));
  }
  if (rows > 0) {
    const fa_status st = tc_launch<kModeDq, D>(prm, bf16, s);
    if (st != FA_OK) return st;
  }
  if (krows > 0) {
    prm.dkdv_overlaps_dq = rows > 0 ? 1 : 0;  // dQ was launched just before
    const fa_status st = tc_launch<kModeDkdv, D>(prm, bf16, s);
    if (st != FA_OK) return st;
  }
  return FA_OK;
}

}  // namespace
}  // namespace fa

extern "C" size_t fa_bwd_workspace_bytes(int32_t B, int32_t H, int32_t L) {
  if (B < 0 || H < 0 || L < 0) return 0;
  return fa::kBwdWorkspaceHeader + static_cast<size_t>(B) * H * L * sizeof(float);
}

extern "C" fa_status fa_flex_attention_bwd(
    const void* q, const void* k, const void* v, const void* out, const void* dout,
    const float* lse, int32_t dtype, int32_t B, int32_t H, int32_t H_kv, int32_t L, int32_t S,
    int32_t D, const fa_block_mask* bm, const int32_t* q_num_blocks, const int32_t* q_indices,
    const int32_t* full_q_num_blocks, const int32_t* full_q_indices, int32_t score_kind,
    float softcap, float scale, void* dq, void* dk, void* dv, void* workspace,
    size_t workspace_bytes, void* stream) {
  using namespace fa;
  if (bm == nullptr) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_INVALID_ARG;
  if (B < 0 || H < 0 || L < 0 || S < 0 || H_kv < 1 || (H > 0 && H % H_kv != 0))
    return FA_ERR_INVALID_ARG;
  if (score_kind != FA_SCORE_NONE && score_kind != FA_SCORE_TANH_SOFTCAP) return FA_ERR_INVALID_ARG;
  if (score_kind == FA_SCORE_TANH_SOFTCAP && !(softcap > 0.f && std::isfinite(softcap)))
    return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (bm->block != FA_BLOCK || bm->q_len != L || bm->kv_len != S) return FA_ERR_INVALID_ARG;
  // per-(batch, head) masks: one instance per batch element and / or head (0 reads as 1)
  const int mb = bm->mask_batch > 1 ? bm->mask_batch : 1;
  const int mh = bm->mask_heads > 1 ? bm->mask_heads : 1;
  if ((mb != 1 && mb != B) || (mh != 1 && mh != H)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H * L == 0 && static_cast<int64_t>(B) * H_kv * S == 0) return FA_OK;
  if (static_cast<int64_t>(B) * H * L > (int64_t{1} << 33) ||
      static_cast<int64_t>(B) * H_kv * S > (int64_t{1} << 33) ||
      static_cast<int64_t>(B) * H > INT32_MAX)
    return FA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(bm->n_kv_blocks) * B * H_kv > INT32_MAX ||
      static_cast<int64_t>(bm->n_q_blocks) * B * H > INT32_MAX)
    return FA_ERR_UNSUPPORTED;
  if (workspace == nullptr || workspace_bytes < fa_bwd_workspace_bytes(B, H, L))
    return FA_ERR_INVALID_ARG;
  const bool any_q = static_cast<int64_t>(B) * H * L > 0, any_k = static_cast<int64_t>(B) * H_kv * S > 0;
  if (any_q && (q == nullptr || out == nullptr || dout == nullptr || lse == nullptr || dq == nullptr))
    return FA_ERR_INVALID_ARG;
  if (any_k && (k == nullptr || v == nullptr || dk == nullptr || dv == nullptr))
    return FA_ERR_INVALID_ARG;
  if (bm->n_q_blocks > 0 && (bm->kv_num_blocks == nullptr || bm->full_kv_num_blocks == nullptr ||
                             bm->q_order == nullptr))
    return FA_ERR_INVALID_ARG;
  if (bm->n_q_blocks > 0 && bm->n_kv_blocks > 0 &&
      (bm->kv_indices == nullptr || bm->full_kv_indices == nullptr || q_num_blocks == nullptr ||
       q_indices == nullptr || full_q_num_blocks == nullptr || full_q_indices == nullptr))
    return FA_ERR_INVALID_ARG;
  if (bm->kind == FA_MASK_DOCUMENT_CAUSAL && bm->doc_id == nullptr) return FA_ERR_INVALID_ARG;
  if (bm->kind == FA_MASK_BITMAP && S > 0 && bm->bitmap == nullptr) return FA_ERR_INVALID_ARG;
  // q, k, v, dout are TMA tiles, out and dout are read in 16-byte pieces and the
  // gradients written in 16-byte pieces: 16 bytes; the workspace holds the error word
  // and the row sums: 16 bytes; the rest is read as 4-byte values
  auto off16 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) != 0; };
  auto off4 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 3u) != 0; };
  if (off16(q) || off16(k) || off16(v) || off16(out) || off16(dout) || off16(dq) || off16(dk) ||
      off16(dv) || off16(workspace) || off4(lse))
    return FA_ERR_INVALID_ARG;
  if (off4(bm->kv_num_blocks) || off4(bm->full_kv_num_blocks) || off4(bm->kv_indices) ||
      off4(bm->full_kv_indices) || off4(bm->q_order) || off4(bm->doc_id) || off4(bm->bitmap) ||
      off4(q_num_blocks) || off4(q_indices) || off4(full_q_num_blocks) || off4(full_q_indices))
    return FA_ERR_INVALID_ARG;

  BwdParams prm{};
  prm.q = static_cast<const uint16_t*>(q);
  prm.k = static_cast<const uint16_t*>(k);
  prm.v = static_cast<const uint16_t*>(v);
  prm.out = static_cast<const uint16_t*>(out);
  prm.dout = static_cast<const uint16_t*>(dout);
  prm.lse = lse;
  prm.err = static_cast<int32_t*>(workspace);
  prm.delta = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kBwdWorkspaceHeader);
  prm.dq = static_cast<uint16_t*>(dq);
  prm.dk = static_cast<uint16_t*>(dk);
  prm.dv = static_cast<uint16_t*>(dv);
  prm.kv_num = bm->kv_num_blocks;
  prm.kv_idx = bm->kv_indices;
  prm.full_num = bm->full_kv_num_blocks;
  prm.full_idx = bm->full_kv_indices;
  prm.q_num = q_num_blocks;
  prm.q_idx = q_indices;
  prm.full_q_num = full_q_num_blocks;
  prm.full_q_idx = full_q_indices;
  prm.sched = bm->q_order;
  prm.doc_id = bm->doc_id;
  prm.bitmap = bm->bitmap;
  prm.B = B;
  prm.H = H;
  prm.Hkv = H_kv;
  prm.G = H > 0 ? H / H_kv : 1;
  prm.L = L;
  prm.S = S;
  prm.n_q = bm->n_q_blocks;
  prm.n_kv = bm->n_kv_blocks;
  prm.kind = bm->kind;
  prm.window = bm->window;
  prm.mask_b = mb > 1 ? 1 : 0;
  prm.mask_h = mh > 1 ? 1 : 0;
  prm.mask_heads = mh;
  prm.doc_len = L > S ? L : S;
  prm.softcap_on = score_kind == FA_SCORE_TANH_SOFTCAP ? 1 : 0;
  prm.is_bf16 = dtype == FA_BF16 ? 1 : 0;
  prm.scale = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(D));
  prm.scale_log2 = prm.scale * kBwdLog2e;
  prm.cap_c = prm.softcap_on ? softcap : 1.f;
  prm.cap_k = prm.softcap_on ? 2.f * prm.scale * kBwdLog2e / softcap : 0.f;
  prm.timeout_ns = 2000000000ull;
  if (debug_stall(&prm.timeout_ns)) prm.stall = 1;
  const cudaStream_t s = as_stream(stream);
  const bool b16 = dtype == FA_BF16;
  return D == 64 ? bwd_launch<64>(prm, b16, s) : bwd_launch<128>(prm, b16, s);
}
