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
  // Q tiles per slot: two at D=64, so the next unit's Q loads while this one runs.
  static constexpr int kQBuf = (D == 64) ? 2 : 1;
  static constexpr uint32_t kTmemCols = 512;
  __host__ __device__ static constexpr uint32_t s_col(int slot) { return 128u * slot; }
  __host__ __device__ static constexpr uint32_t o_col(int slot) { return 256u + static_cast<uint32_t>(D) * slot; }
};

template <int D>
struct __align__(1024) Smem {
  uint8_t q[kNumSlots][Cfg<D>::kQBuf][Cfg<D>::kTileBytes];
  uint8_t kv[Cfg<D>::kStages][Cfg<D>::kTileBytes];
  uint64_t q_full[kNumSlots][Cfg<D>::kQBuf];
  uint64_t q_empty[kNumSlots][Cfg<D>::kQBuf];
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
  const int32_t* kv_idx;
  const int32_t* full_idx;
  const int32_t* sched;  // per rank k: [2k] = q-block row, [2k+1] = partial | full << 16
  const int32_t* doc_id;
  void* out;
  float* lse;
  int32_t* err;
  int BH, L, S, n_kv, num_units;
  int mask_kind, window, softcap_on, is_bf16;
  int split_p;       // P fed to the PV product as two 16-bit terms (hi + lo)
  float scale_log2;  // scale * log2(e)
  float cap_k;       // 2 * scale * log2(e) / c : exp2(s * cap_k) = e^(2 s scale / c)
  float cap_a;       // c * log2(e)
  unsigned long long timeout_ns;
};

// ---------------------------------------------------------------- scheduling
// Work unit u -> (rank u / BH of the LPT-ordered schedule table, batch*head u % BH).
// Units are dealt to the grid's (CTA, slot) workers in rounds, alternating
// direction ("snake"), so the heaviest rows of the LPT order spread over all
// workers.  Every role of a CTA walks the same sequence.
struct Unit {
  int bh, qblk, np, n;
};

__device__ __forceinline__ int2 ldg_nc_v2(const int32_t* ptr) {
  int2 v;
  asm volatile("ld.global.nc.v2.s32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(ptr));
  return v;
}
__device__ __forceinline__ int ldg_nc(const int32_t* ptr) {
  int v;
  asm volatile("ld.global.nc.s32 %0, [%1];" : "=r"(v) : "l"(ptr));
  return v;
}

// Unit sequence of one worker with a one-unit lookahead: the schedule entry of
// the next unit is requested when the current one is handed out, so its global
// load latency overlaps a whole unit of work.
struct UnitIter {
  int worker, workers, round, num_units, BH;
  const int32_t* sched;
  int nu;   // next unit id, -1 when exhausted
  int2 nx;  // its schedule entry (load in flight)

  __device__ __forceinline__ void init(const Params& p, int slot) {
    worker = static_cast<int>(blockIdx.x) * kNumSlots + slot;
    workers = static_cast<int>(gridDim.x) * kNumSlots;
    round = 0;
    num_units = p.num_units;
    BH = p.BH;
    sched = p.sched;
    fetch();
  }
  __device__ __forceinline__ void fetch() {
    const int u = round * workers + ((round & 1) ? (workers - 1 - worker) : worker);
    ++round;
    nu = u < num_units ? u : -1;
    if (nu >= 0) nx = ldg_nc_v2(sched + 2 * (nu / BH));
  }
  __device__ __forceinline__ bool pop(Unit& x) {
    if (nu < 0) return false;
    const int k = nu / BH;
    x.bh = nu - k * BH;
    x.qblk = nx.x;
    x.np = nx.y & 0xFFFF;
    x.n = x.np + (nx.y >> 16);
    fetch();
    return true;
  }
  __device__ __forceinline__ bool pop_nonempty(Unit& x) {
    while (pop(x))
      if (x.n > 0) return true;
    return false;
  }
};

// kv-block index of the j-th block of the unit: partial blocks first, then full ones.
__device__ __forceinline__ int block_index(const Params& p, const Unit& x, int j) {
  const size_t row = static_cast<size_t>(x.qblk) * p.n_kv;
  return j < x.np ? ldg_nc(p.kv_idx + row + j) : ldg_nc(p.full_idx + row + (j - x.np));
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
// TMA producer: the whole warp walks the MMA warp's consumption order (per slot:
// Q, K_0, then V_j, K_{j+1} ...; slots interleaved the way the MMA warp visits
// them) and lane 0 issues the copies.  Block indices are fetched 32 at a time,
// one per lane, and the first chunk of the slot's next unit is requested when
// its current unit starts.
struct ProdSlot {
  UnitIter it;
  Unit cur, nxt;
  bool has_cur, has_nxt;
  int j;           // block of `cur` whose V is loaded next
  int units;       // non-empty units started on this slot
  int chunk;       // 32-block chunk of cur's list held in `idx`
  int idx, nxt_idx;
};

__device__ __forceinline__ int chunk_index(const Params& p, const Unit& x, int chunk, int lane) {
  const int jj = chunk * 32 + lane;
  return jj < x.n ? block_index(p, x, jj) : 0;
}

template <int D>
__device__ void producer_role(Smem<D>& sm, const Params& p, const CUtensorMap* tq,
                              const CUtensorMap* tk, const CUtensorMap* tv) {
  using C = Cfg<D>;
  const int lane = threadIdx.x & 31;
  const uint64_t pol_kv = policy_evict_last();
  const uint64_t pol_q = policy_evict_first();
  ProdSlot st[kNumSlots];
  int kv_cnt = 0;
  int q_armed[kNumSlots][C::kQBuf] = {};
  bool ok = true;

  auto load_tile = [&](const CUtensorMap* map, int row0, int bh, uint8_t* dst, uint64_t* bar,
                       uint64_t pol) {
#pragma unroll
    for (int c = 0; c < C::kChunks; ++c) tma_load_3d(dst + c * kChunkBytes, map, bar, c * 64, row0, bh, pol);
  };
  auto kv_block = [&](ProdSlot& s, int j) -> int {
    const int chunk = j >> 5;
    if (chunk != s.chunk) {
      s.idx = chunk_index(p, s.cur, chunk, lane);
      s.chunk = chunk;
    }
    return __shfl_sync(0xffffffffu, s.idx, j & 31);
  };
  auto load_kv = [&](const CUtensorMap* map, ProdSlot& s, int j) -> bool {
    const int stage = kv_cnt % C::kStages;
    const uint32_t phase = (kv_cnt / C::kStages) & 1;
    const int kvb = kv_block(s, j);
    if (!wait_warp(sm, &sm.kv_empty[stage], phase ^ 1, p)) return false;
    if (lane == 0) {
      mbar_arrive_expect_tx(&sm.kv_full[stage], C::kTileBytes);
      load_tile(map, kvb * kBlockN, s.cur.bh, sm.kv[stage], &sm.kv_full[stage], pol_kv);
    }
    __syncwarp();
    ++kv_cnt;
    return true;
  };
  // Make `nxt` current (its first index chunk is already in flight) and look one unit ahead.
  auto advance = [&](ProdSlot& s) {
    s.has_cur = s.has_nxt;
    s.cur = s.nxt;
    s.idx = s.nxt_idx;
    s.chunk = 0;
    s.j = 0;
    s.has_nxt = s.it.pop_nonempty(s.nxt);
    if (s.has_nxt) s.nxt_idx = chunk_index(p, s.nxt, 0, lane);
  };
  auto start_unit = [&](int slot) -> bool {  // Q and K_0 of the current unit
    ProdSlot& s = st[slot];
    const int b = s.units % C::kQBuf;
    const uint32_t phase = (s.units / C::kQBuf) & 1;
    if (!wait_warp(sm, &sm.q_empty[slot][b], phase ^ 1, p)) return false;
    if (lane == 0) {
      mbar_arrive_expect_tx(&sm.q_full[slot][b], C::kTileBytes);
      load_tile(tq, s.cur.qblk * kBlockN, s.cur.bh, sm.q[slot][b], &sm.q_full[slot][b], pol_q);
    }
    __syncwarp();
    ++q_armed[slot][b];
    ++s.units;
    return load_kv(tk, s, 0);
  };

#pragma unroll
  for (int s = 0; s < kNumSlots; ++s) {
    st[s].it.init(p, s);
    st[s].units = 0;
    st[s].has_nxt = st[s].it.pop_nonempty(st[s].nxt);
    if (st[s].has_nxt) st[s].nxt_idx = chunk_index(p, st[s].nxt, 0, lane);
    advance(st[s]);
    if (ok && st[s].has_cur) ok = start_unit(s);
  }
  bool any = true;
  while (ok && any) {
    any = false;
#pragma unroll
    for (int s = 0; s < kNumSlots; ++s) {
      if (!ok) break;
      if (!st[s].has_cur) continue;
      any = true;
      ok = load_kv(tv, st[s], st[s].j);
      if (!ok) break;
      ++st[s].j;
      if (st[s].j < st[s].cur.n) {
        ok = load_kv(tk, st[s], st[s].j);
      } else {
        advance(st[s]);
        if (st[s].has_cur) ok = start_unit(s);
      }
    }
  }
  if (!ok && lane == 0) {
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
    for (int s = 0; s < kNumSlots; ++s)
      for (int b = 0; b < C::kQBuf; ++b) {
        if (q_armed[s][b] == 0) continue;
        while (!mbar_try_wait(&sm.q_full[s][b], (q_armed[s][b] - 1) & 1) &&
               globaltimer_ns() - t0 < p.timeout_ns) {
        }
      }
  }
  __syncwarp();
}

// MMA issuer: one thread issues every tcgen05.mma of the CTA.  Per slot and block
// j it issues PV_{j-1} then S_j, so each slot alternates between the tensor core
// and its softmax warpgroup while the other slot fills the gap.
struct MmaSlot {
  UnitIter it;
  Unit cur;
  bool active;
  int j;      // block whose PV is issued next
  int units;  // non-empty units started on this slot
  int blk;    // blocks finished on this slot (p_full phase)
};

template <int D>
__device__ void mma_role(Smem<D>& sm, const Params& p, uint32_t tmem) {
  using C = Cfg<D>;
  const int lane = threadIdx.x & 31;
  const uint32_t idesc_s = idesc_f16_f32(p.is_bf16 != 0, 128, 128, false);
  const uint32_t idesc_pv = idesc_f16_f32(p.is_bf16 != 0, 128, D, true);
  MmaSlot st[kNumSlots];
  int kv_cnt = 0;
  bool ok = true;

  auto issue_s = [&](int slot, int j) -> bool {
    MmaSlot& s = st[slot];
    const int b = (s.units - 1) % C::kQBuf;  // Q buffer of the current unit
    if (j == 0 && !wait_warp(sm, &sm.q_full[slot][b], ((s.units - 1) / C::kQBuf) & 1, p))
      return false;
    const int stage = kv_cnt % C::kStages;
    if (!wait_warp(sm, &sm.kv_full[stage], (kv_cnt / C::kStages) & 1, p)) return false;
    tc_fence_after();
    if (lane == 0) {
      const uint32_t qa = smem_u32(sm.q[slot][b]);
      const uint32_t ka = smem_u32(sm.kv[stage]);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = (kk >> 2) * kChunkBytes + (kk & 3) * 32;
        umma_ss(tmem + C::s_col(slot), sdesc_sw128(qa + off, 16, 1024),
                sdesc_sw128(ka + off, 16, 1024), idesc_s, kk > 0 ? 1u : 0u);
      }
      umma_commit(&sm.kv_empty[stage]);
      umma_commit(&sm.s_full[slot]);
      if (j == s.cur.n - 1) umma_commit(&sm.q_empty[slot][b]);
    }
    __syncwarp();
    ++kv_cnt;
    return true;
  };
  auto issue_pv = [&](int slot) -> bool {
    MmaSlot& s = st[slot];
    if (!wait_warp(sm, &sm.p_full[slot], s.blk & 1, p)) return false;
    // O of this slot is free once the epilogue of its previous unit has read it
    if (s.j == 0 && !wait_warp(sm, &sm.o_empty[slot], ((s.units - 1) & 1) ^ 1, p)) return false;
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
      if (p.split_p) {
#pragma unroll
        for (int kk = 0; kk < kBlockN / 16; ++kk)
          umma_ts(tmem + C::o_col(slot), tmem + C::s_col(slot) + 64 + kk * 8,
                  sdesc_sw128(va + kk * 2048, kChunkBytes, 1024), idesc_pv, 1u);
      }
      umma_commit(&sm.kv_empty[stage]);
      if (s.j == s.cur.n - 1) umma_commit(&sm.o_full[slot]);
    }
    __syncwarp();
    ++kv_cnt;
    ++s.blk;
    return true;
  };
  auto start_unit = [&](int slot) -> bool {
    MmaSlot& s = st[slot];
    s.active = s.it.pop_nonempty(s.cur);
    if (!s.active) return true;
    s.j = 0;
    ++s.units;
    return issue_s(slot, 0);
  };

#pragma unroll
  for (int s = 0; s < kNumSlots; ++s) {
    st[s].it.init(p, s);
    st[s].units = 0;
    st[s].blk = 0;
    if (ok) ok = start_unit(s);
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
      ok = st[s].j < st[s].cur.n ? issue_s(s, st[s].j) : start_unit(s);
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

__device__ __forceinline__ void unpack2(uint32_t v, bool bf16, float& lo, float& hi) {
  if (bf16) {
    lo = __uint_as_float(v << 16);
    hi = __uint_as_float(v & 0xFFFF0000u);
  } else {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&v));
    lo = f.x;
    hi = f.y;
  }
}

// Softmax warpgroup of one slot: thread t owns row t of the slot's 128-row tile
// (TMEM lane t), so row max and row sum need no shuffles.
template <int D>
__device__ void softmax_role(Smem<D>& sm, const Params& p, uint32_t tmem, int slot) {
  using C = Cfg<D>;
  const int t = threadIdx.x - slot * 128;   // row of the tile this thread owns
  const int wq = t >> 5;                    // TMEM lane quarter of this warp
  const uint32_t lane_off = static_cast<uint32_t>(wq * 32) << 16;
  const uint32_t t_s = tmem + C::s_col(slot) + lane_off;
  const uint32_t t_o = tmem + C::o_col(slot) + lane_off;
  const bool bf16 = p.is_bf16 != 0;
  // Factor that turns the value kept in x[] into log2 units: the raw score is
  // kept (and scaled inside the exponent's FFMA) unless a score_mod rewrote it.
  const float xs = p.softcap_on ? 1.f : p.scale_log2;
  UnitIter it;
  it.init(p, slot);
  int blk = 0, units = 0;
  Unit un;

  while (it.pop(un)) {
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
    float m = -INFINITY, l = 0.f;  // running max (log2 units) and running sum
    int kvb = block_index(p, un, 0);

    for (int j = 0; j < un.n; ++j) {
      const bool full = j >= un.np;
      const int kvb_next = j + 1 < un.n ? block_index(p, un, j + 1) : 0;
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
      if (p.softcap_on) {  // x = log2(e) * c * tanh(s * scale / c)
#pragma unroll
        for (int i = 0; i < 128; ++i) {
          const float e = ex2_approx(x[i] * p.cap_k);            // e^(2y), y = s * scale / c
          x[i] = p.cap_a - 2.f * p.cap_a * rcp_approx(e + 1.f);  // c * log2(e) * tanh(y)
        }
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
      // row max: 16 independent chains, then a tree
      float mx[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) mx[i] = x[i];
#pragma unroll
      for (int i = 16; i < 128; ++i) mx[i & 15] = fmaxf(mx[i & 15], x[i]);
#pragma unroll
      for (int w = 8; w > 0; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) mx[i] = fmaxf(mx[i], mx[i + w]);
      const float m_new = fmaxf(m, mx[0] * xs);
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
      const float neg_mu = (m == -INFINITY) ? 0.f : -m;
      // P = exp2(x * xs - m) as 16-bit pairs: P_hi = round(p) over S columns 0-63 and,
      // when split, P_lo = round(p - P_hi) over columns 64-127 (both PV products are
      // accumulated, so P carries ~16 significant bits instead of 8).
      float sums[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) sums[i] = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t ph[16], pl[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = ex2_approx(fmaf(x[c * 32 + 2 * i], xs, neg_mu));
          const float p1 = ex2_approx(fmaf(x[c * 32 + 2 * i + 1], xs, neg_mu));
          sums[i & 7] += p0 + p1;
          ph[i] = pack2(p0, p1, bf16);
          float h0, h1;
          unpack2(ph[i], bf16, h0, h1);
          pl[i] = pack2(p0 - h0, p1 - h1, bf16);
        }
        tmem_st16(t_s + c * 16, ph);
        if (p.split_p) tmem_st16(t_s + 64 + c * 16, pl);
      }
#pragma unroll
      for (int w = 4; w > 0; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) sums[i] += sums[i + w];
      l += sums[0];
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
      kvb = kvb_next;
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
      for (int b = 0; b < Cfg<D>::kQBuf; ++b) {
        mbar_init(&sm.q_full[s][b], 1);
        mbar_init(&sm.q_empty[s][b], 1);
      }
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
    producer_role<D>(sm, p, &tmap_q, &tmap_k, &tmap_v);
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
  prm.kv_idx = bm->kv_indices;
  prm.full_idx = bm->full_kv_indices;
  prm.sched = bm->q_order;
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
  prm.split_p = 1;
  prm.timeout_ns = 2000000000ull;
  const cudaStream_t s = as_stream(stream);
  if (D == 64) return launch<64>(q, k, v, dtype == FA_BF16, prm.BH, L, S, prm, s);
  return launch<128>(q, k, v, dtype == FA_BF16, prm.BH, L, S, prm, s);
}
