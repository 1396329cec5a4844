// Block-sparse attention forward for B200 (sm_100a).
//
// Computes out = softmax(Q K^T * scale + mask / score_mod) V
// (attention definition: SDPA tutorial, qiita GeneLab_999, section 1; mask and
// score_mod rules: FlexAttention how-to, dreaming.press, "Mask 1..3" and "Bonus: a
// score_mod for soft-capping") one 128 x 128 block at a time with an online
// softmax (running max and running sum, reconciled at the end: FlashAttention
// explainer, service-dock.com, third section; FlashAttention-2 article,
// media.tcdigital.jp, "分割統治法（Tiling）によるSRAM活用"), so the L x S score
// matrix never reaches HBM, and EMPTY blocks of the BlockMask are never touched.
//
// Kernel organisation (one persistent CTA per SM, 320 threads):
//   warps 0-3   softmax warpgroup of slot 0     warps 4-7   softmax warpgroup of slot 1
//   warp 8      TMA producer (one lane)         warp 9      tcgen05.mma issuer + TMEM owner
// A "slot" owns one 128-row Q tile, an S/P region (128 TMEM columns) and an O
// accumulator (D TMEM columns).  The two slots work on independent work units
// (batch*head, q-block) so that the tensor core computes one slot's S = Q K^T and
// O += P V while the other slot's softmax runs.  K and V tiles stream through a
// shared ring of shared-memory stages filled by TMA (128-byte swizzle, no multicast).
//
// Per block j of a unit, in the order the MMA warp issues them:
//   S_j  = Q K_j^T        (SS MMA, M=128 N=128 K=D, fp32 in TMEM)    -> s_full
//   softmax warpgroup: S -> registers, scale (+ softcap), mask on PARTIAL blocks only,
//   running max with deferred rescaling of O, P = exp2(x - m) as bf16/fp16 written
//   back into the S columns                                           -> p_full
//   O   += P V_j          (TS MMA: A = P from TMEM, B = V MN-major)   -> (next S_j+1)
// Because tcgen05 operations of one thread complete in issue order and S_{j+1} is
// issued after PV_j, the commit that signals S_{j+1} also guarantees PV_j is done:
// the softmax may rescale O in TMEM right after it sees S_{j+1}.
//
// Every mbarrier wait is bounded: after `timeout_ns` the waiting warp sets an abort
// flag and the device error word, all roles stop, in-flight copies and MMAs are
// drained (again with a bound), TMEM is freed and the CTA returns.
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

constexpr int kNumSlots = 2;
constexpr int kSoftmaxWarps = 4 * kNumSlots;
constexpr int kProducerWarp = kSoftmaxWarps;
constexpr int kMmaWarp = kSoftmaxWarps + 1;
constexpr int kThreads = (kSoftmaxWarps + 4) * 32;  // + one warpgroup: producer, MMA, 2 spare
// Register split (per thread) after launch: 384 threads x 168 = 64512 registers at
// launch; softmax warpgroups take 208, the control warpgroup 88:
// 256 x 208 + 128 x 88 = 64512, and per SM sub-partition 208 + 208 + 88 <= 512.
constexpr int kRegsSoftmax = 208;
constexpr int kRegsControl = 88;
constexpr int kBlockN = 128;                 // rows of a Q tile / K,V tile
constexpr int kChunkBytes = 128 * 128;       // one TMA box: 128 rows x 64 elems x 2 B
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;    // log2 units: O is rescaled only when max grows > 2^8

template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kBlockN * D * 2;
  static constexpr int kStages = (D == 64) ? 8 : 4;
  static constexpr uint32_t kTmemCols = 512;
  __host__ __device__ static constexpr uint32_t s_col(int slot) { return 128u * slot; }
  __host__ __device__ static constexpr uint32_t o_col(int slot) { return 256u + static_cast<uint32_t>(D) * slot; }
};

template <int D>
struct __align__(1024) Smem {
  uint8_t q[kNumSlots][Cfg<D>::kTileBytes];
  uint8_t kv[Cfg<D>::kStages][Cfg<D>::kTileBytes];
  uint64_t q_full[kNumSlots];
  uint64_t q_empty[kNumSlots];
  uint64_t s_full[kNumSlots];
  uint64_t p_full[kNumSlots];
  uint64_t o_full[kNumSlots];
  uint64_t o_empty[kNumSlots];
  uint64_t kv_full[Cfg<D>::kStages];
  uint64_t kv_empty[Cfg<D>::kStages];
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
};

struct Params {
  const int32_t* kv_num;
  const int32_t* kv_idx;
  const int32_t* full_num;
  const int32_t* full_idx;
  const int32_t* q_order;
  const int32_t* doc_id;
  void* out;
  float* lse;
  int32_t* err;
  int BH, L, S, n_kv, num_units;
  int mask_kind, window, softcap_on, is_bf16;
  float scale_log2;  // scale * log2(e)
  float cap_k;       // 2 * scale * log2(e) / c : exp2(s * cap_k) = e^(2 s scale / c)
  float cap_a;       // c * log2(e)
  unsigned long long timeout_ns;
};

// ---------------------------------------------------------------- scheduling
// Work unit u -> (q-block rank u / BH in q_order, batch*head u % BH).  Units are
// dealt to the grid's (CTA, slot) workers in rounds, alternating direction
// ("snake"), so the heaviest rows of the LPT order spread over all workers.
struct Unit {
  int bh, qblk, np, n;
};

__device__ __forceinline__ Unit decode_unit(const Params& p, int u) {
  const int k = u / p.BH;
  Unit x;
  x.bh = u - k * p.BH;
  x.qblk = __ldg(p.q_order + k);
  x.np = __ldg(p.kv_num + x.qblk);
  x.n = x.np + __ldg(p.full_num + x.qblk);
  return x;
}

// kv-block index of the j-th block of the unit: partial blocks first, then full ones.
__device__ __forceinline__ int block_index(const Params& p, const Unit& x, int j, bool& full) {
  const size_t row = static_cast<size_t>(x.qblk) * p.n_kv;
  if (j < x.np) {
    full = false;
    return __ldg(p.kv_idx + row + j);
  }
  full = true;
  return __ldg(p.full_idx + row + (j - x.np));
}

struct Sched {
  int worker, workers, round;
  __device__ __forceinline__ int next(int num_units) {
    const int u = round * workers + ((round & 1) ? (workers - 1 - worker) : worker);
    ++round;
    return u < num_units ? u : -1;
  }
};

struct SlotState {
  Sched sched;
  Unit unit;
  int j;      // current block within the unit
  int units;  // non-empty units finished on this slot
  bool active;
};

__device__ __forceinline__ bool next_nonempty(SlotState& st, const Params& p) {
  while (true) {
    const int u = st.sched.next(p.num_units);
    if (u < 0) {
      st.active = false;
      return false;
    }
    st.unit = decode_unit(p, u);
    if (st.unit.n > 0) {
      st.j = 0;
      st.active = true;
      return true;
    }
  }
}

// ---------------------------------------------------------------- bounded wait
template <int D>
__device__ __forceinline__ bool wait_slow(Smem<D>& sm, uint64_t* bar, uint32_t parity, const Params& p) {
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
__device__ __forceinline__ bool wait_bar(Smem<D>& sm, uint64_t* bar, uint32_t parity, const Params& p) {
  if (mbar_try_wait(bar, parity)) return true;
  return wait_slow(sm, bar, parity, p);
}

// Whole-warp wait: every lane waits, and the warp agrees on the outcome so that
// warp-collective tcgen05 instructions after it are executed by all lanes or none.
template <int D>
__device__ __forceinline__ bool wait_warp(Smem<D>& sm, uint64_t* bar, uint32_t parity, const Params& p) {
  return __all_sync(0xffffffffu, wait_bar(sm, bar, parity, p));
}

// ---------------------------------------------------------------- roles
template <int D>
__device__ void producer_role(Smem<D>& sm, const Params& p, const CUtensorMap* tq,
                              const CUtensorMap* tk, const CUtensorMap* tv) {
  using C = Cfg<D>;
  const uint64_t pol_kv = policy_evict_last();
  const uint64_t pol_q = policy_evict_first();
  SlotState st[kNumSlots];
  int kv_cnt = 0;
  int q_armed[kNumSlots] = {};
  bool ok = true;

  auto load_tile = [&](const CUtensorMap* map, int row0, int bh, uint8_t* dst, uint64_t* bar,
                       uint64_t pol) {
#pragma unroll
    for (int c = 0; c < C::kChunks; ++c) tma_load_3d(dst + c * kChunkBytes, map, bar, c * 64, row0, bh, pol);
  };
  auto load_kv = [&](const CUtensorMap* map, SlotState& s) -> bool {
    const int stage = kv_cnt % C::kStages;
    const uint32_t phase = (kv_cnt / C::kStages) & 1;
    if (!wait_bar(sm, &sm.kv_empty[stage], phase ^ 1, p)) return false;
    mbar_arrive_expect_tx(&sm.kv_full[stage], C::kTileBytes);
    bool full;
    const int kvb = block_index(p, s.unit, s.j, full);
    load_tile(map, kvb * kBlockN, s.unit.bh, sm.kv[stage], &sm.kv_full[stage], pol_kv);
    ++kv_cnt;
    return true;
  };
  auto load_q = [&](int slot) -> bool {
    SlotState& s = st[slot];
    if (!wait_bar(sm, &sm.q_empty[slot], (s.units & 1) ^ 1, p)) return false;
    mbar_arrive_expect_tx(&sm.q_full[slot], C::kTileBytes);
    load_tile(tq, s.unit.qblk * kBlockN, s.unit.bh, sm.q[slot], &sm.q_full[slot], pol_q);
    ++q_armed[slot];
    return true;
  };

  for (int s = 0; s < kNumSlots; ++s) {
    st[s].sched = Sched{static_cast<int>(blockIdx.x) * kNumSlots + s,
                        static_cast<int>(gridDim.x) * kNumSlots, 0};
    st[s].units = 0;
    q_armed[s] = 0;
    if (ok && next_nonempty(st[s], p)) ok = load_q(s) && load_kv(tk, st[s]);
  }
  bool any = true;
  while (ok && any) {
    any = false;
#pragma unroll
    for (int s = 0; s < kNumSlots; ++s) {
      if (!ok) break;
      if (!st[s].active) continue;
      any = true;
      ok = load_kv(tv, st[s]);
      if (!ok) break;
      ++st[s].j;
      if (st[s].j < st[s].unit.n) {
        ok = load_kv(tk, st[s]);
      } else {
        ++st[s].units;
        if (next_nonempty(st[s], p)) ok = load_q(s) && load_kv(tk, st[s]);
      }
    }
  }
  if (!ok) {
    // Drain: wait (bounded) for every TMA copy this warp armed, so that no copy
    // lands in shared memory after the CTA has exited.
    const uint64_t t0 = globaltimer_ns();
    for (int stage = 0; stage < C::kStages; ++stage) {
      const int fills = kv_cnt / C::kStages + (stage < kv_cnt % C::kStages ? 1 : 0);
      if (fills == 0) continue;
      while (!mbar_try_wait(&sm.kv_full[stage], (fills - 1) & 1) &&
             globaltimer_ns() - t0 < p.timeout_ns) {
      }
    }
    for (int s = 0; s < kNumSlots; ++s) {
      if (q_armed[s] == 0) continue;
      while (!mbar_try_wait(&sm.q_full[s], (q_armed[s] - 1) & 1) &&
             globaltimer_ns() - t0 < p.timeout_ns) {
      }
    }
  }
}

template <int D>
__device__ void mma_role(Smem<D>& sm, const Params& p, uint32_t tmem) {
  using C = Cfg<D>;
  const int lane = threadIdx.x & 31;
  const uint32_t idesc_s = idesc_f16_f32(p.is_bf16 != 0, 128, 128, false);
  const uint32_t idesc_pv = idesc_f16_f32(p.is_bf16 != 0, 128, D, true);
  SlotState st[kNumSlots];
  int blk[kNumSlots] = {};
  int kv_cnt = 0;
  bool ok = true;

  auto issue_s = [&](int slot) -> bool {
    SlotState& s = st[slot];
    if (s.j == 0 && !wait_warp(sm, &sm.q_full[slot], s.units & 1, p)) return false;
    const int stage = kv_cnt % C::kStages;
    if (!wait_warp(sm, &sm.kv_full[stage], (kv_cnt / C::kStages) & 1, p)) return false;
    tc_fence_after();
    if (lane == 0) {
      const uint32_t qa = smem_u32(sm.q[slot]);
      const uint32_t ka = smem_u32(sm.kv[stage]);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
        umma_ss(tmem + C::s_col(slot), sdesc_sw128(qa + off, 16, 1024),
                sdesc_sw128(ka + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
      }
      umma_commit(&sm.kv_empty[stage]);
      umma_commit(&sm.s_full[slot]);
      if (s.j == s.unit.n - 1) umma_commit(&sm.q_empty[slot]);
    }
    __syncwarp();
    ++kv_cnt;
    return true;
  };
  auto issue_pv = [&](int slot) -> bool {
    SlotState& s = st[slot];
    if (!wait_warp(sm, &sm.p_full[slot], blk[slot] & 1, p)) return false;
    if (s.j == 0 && !wait_warp(sm, &sm.o_empty[slot], (s.units & 1) ^ 1, p)) return false;
    const int stage = kv_cnt % C::kStages;
    if (!wait_warp(sm, &sm.kv_full[stage], (kv_cnt / C::kStages) & 1, p)) return false;
    tc_fence_after();
    if (lane == 0) {
      const uint32_t va = smem_u32(sm.kv[stage]);
#pragma unroll
      for (int kk = 0; kk < kBlockN / 16; ++kk) {
        umma_ts(tmem + C::o_col(slot), tmem + C::s_col(slot) + kk * 8,
                sdesc_sw128(va + kk * 2048, kChunkBytes, 1024), idesc_pv,
                (s.j > 0 || kk > 0) ? 1u : 0u);
      }
      umma_commit(&sm.kv_empty[stage]);
      if (s.j == s.unit.n - 1) umma_commit(&sm.o_full[slot]);
    }
    __syncwarp();
    ++kv_cnt;
    ++blk[slot];
    return true;
  };

  for (int s = 0; s < kNumSlots; ++s) {
    st[s].sched = Sched{static_cast<int>(blockIdx.x) * kNumSlots + s,
                        static_cast<int>(gridDim.x) * kNumSlots, 0};
    st[s].units = 0;
    blk[s] = 0;
    if (ok && next_nonempty(st[s], p)) ok = issue_s(s);
  }
  bool any = true;
  while (ok && any) {
    any = false;
#pragma unroll
    for (int s = 0; s < kNumSlots; ++s) {
      if (!ok) break;
      if (!st[s].active) continue;
      any = true;
      ok = issue_pv(s);
      if (!ok) break;
      ++st[s].j;
      if (st[s].j < st[s].unit.n) {
        ok = issue_s(s);
      } else {
        ++st[s].units;
        if (next_nonempty(st[s], p)) ok = issue_s(s);
      }
    }
  }
  if (!ok) {
    // Drain every MMA this thread issued before TMEM is released.
    if (lane == 0) umma_commit(&sm.drain);
    __syncwarp();
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&sm.drain, 0) && globaltimer_ns() - t0 < p.timeout_ns) {
    }
  }
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi, bool bf16) {
  if (bf16) {
    __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&h);
  }
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

template <int D>
__device__ void softmax_role(Smem<D>& sm, const Params& p, uint32_t tmem, int slot) {
  using C = Cfg<D>;
  const int t = threadIdx.x - slot * 128;   // row of the tile this thread owns
  const int wq = t >> 5;                    // TMEM lane quarter of this warp
  const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
  const uint32_t t_s = tmem + C::s_col(slot) + lane_off;
  const uint32_t t_o = tmem + C::o_col(slot) + lane_off;
  const bool bf16 = p.is_bf16 != 0;
  Sched sched{static_cast<int>(blockIdx.x) * kNumSlots + slot,
              static_cast<int>(gridDim.x) * kNumSlots, 0};
  int blk = 0, units = 0;

  while (true) {
    const int u = sched.next(p.num_units);
    if (u < 0) break;
    const Unit un = decode_unit(p, u);
    const int row = un.qblk * kBlockN + t;
    const bool valid = row < p.L;
    const size_t orow = static_cast<size_t>(un.bh) * p.L + row;
    uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + orow * D);
    if (un.n == 0) {
      if (valid) {
#pragma unroll
        for (int i = 0; i < D / 8; ++i) dst[i] = make_uint4(0, 0, 0, 0);
        if (p.lse) p.lse[orow] = -INFINITY;
      }
      continue;
    }
    const int dq = (p.mask_kind == FA_MASK_DOCUMENT_CAUSAL && valid) ? __ldg(p.doc_id + row) : 0;
    // live keys of this row: kv in [lo, hi] (and, for documents, doc_id[kv] == dq)
    const int hi = min(row, p.S - 1);
    const int lo = p.mask_kind == FA_MASK_SLIDING_WINDOW_CAUSAL ? max(row - p.window + 1, 0) : 0;
    float m = -INFINITY, l = 0.f;

    for (int j = 0; j < un.n; ++j) {
      bool full;
      const int kvb = block_index(p, un, j, full);
      if (!wait_warp(sm, &sm.s_full[slot], blk & 1, p)) return;
      tc_fence_after();
      float x[128];
      {
        uint32_t xr[128];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld32(t_s + c * 32, *reinterpret_cast<uint32_t(*)[32]>(xr + c * 32));
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 128; ++i) x[i] = __uint_as_float(xr[i]);
      }
      // scores in log2 units: x = log2(e) * score_mod(s * scale)
      if (p.softcap_on) {
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          const float e = ex2_approx(x[i] * p.cap_k);            // e^(2y), y = s * scale / c
          x[i] = p.cap_a - 2.f * p.cap_a * rcp_approx(e + 1.f);  // c * log2(e) * tanh(y)
        }
      } else {
#pragma unroll
        for (int i = 0; i < 128; ++i) x[i] *= p.scale_log2;
      }
      if (!full) {  // PARTIAL block: evaluate the mask rule per element
        const int a = lo - kvb * kBlockN;  // live columns: a <= i <= b
        const int b = hi - kvb * kBlockN;
        if (p.mask_kind == FA_MASK_DOCUMENT_CAUSAL) {
          const int kv0 = kvb * kBlockN;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            uint32_t same = 0;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int kv = kv0 + c * 32 + i;
              const int d = kv < p.S ? __ldg(p.doc_id + kv) : dq + 1;
              same |= (d == dq ? 1u : 0u) << i;
            }
            asm volatile("" ::: "memory");  // keep one chunk of id loads in flight at a time
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const int ii = c * 32 + i;
              if (ii < a || ii > b || !((same >> i) & 1u)) x[ii] = -INFINITY;
            }
          }
        } else {
#pragma unroll
          for (int i = 0; i < 128; ++i)
            if (i < a || i > b) x[i] = -INFINITY;
        }
      }
      float mb = x[0];
#pragma unroll
      for (int i = 1; i < 128; ++i) mb = fmaxf(mb, x[i]);
      const float m_new = fmaxf(m, mb);
      // Deferred rescale: keep the stale max unless the new one exceeds it by more
      // than 2^8; exact, because l and O always use the same max.
      float alpha = 1.f;
      bool rescale_o = false;
      if (m_new > m + kRescaleThreshold) {
        if (m != -INFINITY) {
          alpha = ex2_approx(m - m_new);
          l *= alpha;
          rescale_o = true;  // O already holds contributions of this row
        }
        m = m_new;
      }
      const float mu = (m == -INFINITY) ? 0.f : m;
      float sum = 0.f;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float p0 = ex2_approx(x[c * 64 + 2 * i] - mu);
          const float p1 = ex2_approx(x[c * 64 + 2 * i + 1] - mu);
          sum += p0 + p1;
          pk[i] = pack2(p0, p1, bf16);
        }
        tmem_st32(t_s + c * 32, pk);  // P (16-bit pairs) over the first 64 S columns
      }
      l += sum;
      if (__any_sync(0xffffffffu, rescale_o)) {
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(t_o + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
          tmem_st32(t_o + c * 32, r);
        }
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&sm.p_full[slot]);
      ++blk;
    }

    // epilogue: O / l -> out, LSE
    if (!wait_warp(sm, &sm.o_full[slot], units & 1, p)) return;
    tc_fence_after();
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int c = 0; c < D / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(t_o + c * 32, r);
      tmem_wait_ld();
      uint32_t pk[16];
#pragma unroll
      for (int i = 0; i < 16; ++i)
        pk[i] = pack2(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv, bf16);
      if (valid) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          dst[c * 4 + i] = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
      }
    }
    tc_fence_before();
    mbar_arrive(&sm.o_empty[slot]);
    if (valid && p.lse) p.lse[orow] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
    ++units;
  }
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
fwd_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
           const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  Smem<D>& sm = *reinterpret_cast<Smem<D>*>(smem_raw + ((1024u - (base & 1023u)) & 1023u));
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNumSlots; ++s) {
      mbar_init(&sm.q_full[s], 1);
      mbar_init(&sm.q_empty[s], 1);
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], 128);
      mbar_init(&sm.o_full[s], 1);
      mbar_init(&sm.o_empty[s], 128);
    }
    for (int i = 0; i < Cfg<D>::kStages; ++i) {
      mbar_init(&sm.kv_full[i], 1);
      mbar_init(&sm.kv_empty[i], 1);
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kProducerWarp && (threadIdx.x & 31) == 0) {
    prefetch_tensormap(&tmap_q);
    prefetch_tensormap(&tmap_k);
    prefetch_tensormap(&tmap_v);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sm.tmem_base, Cfg<D>::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // Role dispatch.  Each register configuration has its own code path to the end
  // of the kernel; the final rendezvous is a named barrier over all threads.
  if (warp < kSoftmaxWarps) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsSoftmax));
    softmax_role<D>(sm, p, tmem, warp / 4);
    tc_fence_before();
    named_barrier_sync(1, kThreads);
    return;
  }
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsControl));
  if (warp == kProducerWarp) {
    if ((threadIdx.x & 31) == 0) producer_role<D>(sm, p, &tmap_q, &tmap_k, &tmap_v);
  } else if (warp == kMmaWarp) {
    mma_role<D>(sm, p, tmem);
  }
  tc_fence_before();
  named_barrier_sync(1, kThreads);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg<D>::kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 3-D map over a (BH, rows, D) tensor: box = 64 elements x 128 rows x 1, 128-byte
// swizzle; rows past `rows` read as zeros.
bool make_map(CUtensorMap* map, const void* ptr, bool bf16, int D, int rows, int bh) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(bh)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                                 static_cast<cuuint64_t>(D) * 2 * static_cast<cuuint64_t>(rows)};
  const cuuint32_t box[3] = {64, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
                        const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

template <int D>
fa_status launch(const void* q, const void* k, const void* v, bool bf16, int BH, int L, int S,
                 const Params& prm, cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, bf16, D, L, BH)) return FA_ERR_CUDA;
  // With S == 0 no K/V tile is ever loaded; the maps only need to be well formed.
  if (!make_map(&tk, S > 0 ? k : q, bf16, D, S > 0 ? S : L, BH)) return FA_ERR_CUDA;
  if (!make_map(&tv, S > 0 ? v : q, bf16, D, S > 0 ? S : L, BH)) return FA_ERR_CUDA;
  const size_t smem = sizeof(Smem<D>) + 1024;
  int dev = 0;
  FA_CUDA_CHECK(cudaGetDevice(&dev));
  {
    static std::mutex mu;
    static bool done[kMaxDevices] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
    if (!done[dev]) {
      FA_CUDA_CHECK(cudaFuncSetAttribute(fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem)));
      done[dev] = true;
    }
  }
  const int sms = num_sms_current_device();
  if (sms <= 0) return FA_ERR_CUDA;
  const int want = (prm.num_units + kNumSlots - 1) / kNumSlots;
  const int grid = want < sms ? want : sms;
  fwd_kernel<D><<<grid, kThreads, smem, stream>>>(tq, tk, tv, prm);
  FA_CUDA_CHECK(cudaGetLastError());
  return FA_OK;
}

}  // namespace
}  // namespace fa

extern "C" size_t fa_fwd_workspace_bytes(void) { return 256; }

extern "C" fa_status fa_flex_attention_fwd(const void* q, const void* k, const void* v,
                                           int32_t dtype, int32_t B, int32_t H, int32_t L,
                                           int32_t S, int32_t D, const fa_block_mask* bm,
                                           int32_t score_kind, float softcap, float scale,
                                           void* out, float* lse, void* workspace,
                                           void* stream) {
  using namespace fa;
  if (bm == nullptr || workspace == nullptr) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_INVALID_ARG;
  if (B < 0 || H < 0 || L < 0 || S < 0) return FA_ERR_INVALID_ARG;
  if (score_kind != FA_SCORE_NONE && score_kind != FA_SCORE_TANH_SOFTCAP) return FA_ERR_INVALID_ARG;
  if (score_kind == FA_SCORE_TANH_SOFTCAP && !(softcap > 0.f && std::isfinite(softcap)))
    return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (bm->block != FA_BLOCK || bm->q_len != L || bm->kv_len != S) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  const int64_t BH64 = static_cast<int64_t>(B) * H;
  if (BH64 == 0 || L == 0) return FA_OK;
  if (BH64 * bm->n_q_blocks > INT32_MAX) return FA_ERR_UNSUPPORTED;
  if (q == nullptr || out == nullptr || (S > 0 && (k == nullptr || v == nullptr)))
    return FA_ERR_INVALID_ARG;
  auto misaligned = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) != 0; };
  if (misaligned(q) || misaligned(out) || (S > 0 && (misaligned(k) || misaligned(v))))
    return FA_ERR_INVALID_ARG;
  if (bm->kv_num_blocks == nullptr || bm->full_kv_num_blocks == nullptr || bm->q_order == nullptr)
    return FA_ERR_INVALID_ARG;
  if (bm->kind == FA_MASK_DOCUMENT_CAUSAL && bm->doc_id == nullptr) return FA_ERR_INVALID_ARG;

  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(D));
  Params prm{};
  prm.kv_num = bm->kv_num_blocks;
  prm.kv_idx = bm->kv_indices;
  prm.full_num = bm->full_kv_num_blocks;
  prm.full_idx = bm->full_kv_indices;
  prm.q_order = bm->q_order;
  prm.doc_id = bm->doc_id;
  prm.out = out;
  prm.lse = lse;
  prm.err = static_cast<int32_t*>(workspace);
  prm.BH = static_cast<int>(BH64);
  prm.L = L;
  prm.S = S;
  prm.n_kv = bm->n_kv_blocks;
  prm.num_units = static_cast<int>(BH64 * bm->n_q_blocks);
  prm.mask_kind = bm->kind;
  prm.window = bm->window;
  prm.softcap_on = score_kind == FA_SCORE_TANH_SOFTCAP ? 1 : 0;
  prm.is_bf16 = dtype == FA_BF16 ? 1 : 0;
  prm.scale_log2 = sc * kLog2e;
  prm.cap_k = prm.softcap_on ? 2.f * sc * kLog2e / softcap : 0.f;
  prm.cap_a = prm.softcap_on ? softcap * kLog2e : 0.f;
  prm.timeout_ns = 2000000000ull;
  const cudaStream_t s = as_stream(stream);
  if (D == 64) return launch<64>(q, k, v, dtype == FA_BF16, prm.BH, L, S, prm, s);
  return launch<128>(q, k, v, dtype == FA_BF16, prm.BH, L, S, prm, s);
}
