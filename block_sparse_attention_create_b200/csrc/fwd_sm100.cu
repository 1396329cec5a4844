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

// TMEM layouts (512 columns, lanes = the 128 rows of a tile):
//  D = 64  ("separate P"): S0 [0,128) S1 [128,256) P0 [256,320) P1 [320,384)
//          O0 [384,448) O1 [448,512).  The softmax frees S as soon as it has read
//          it, so S_{j+1} is computed on the tensor core while softmax j runs.
//  D = 128 ("aliased P"):  S0/P0 [0,128) S1/P1 [128,256) O0 [256,384) O1 [384,512).
//          P overwrites the S it came from (hi in columns 0-63, lo in 64-127), so
//          S_{j+1} waits for PV_j; the other slot covers that gap.
template <int D>
struct Cfg {
  static constexpr int kChunks = D / 64;
  static constexpr int kTileBytes = kBlockN * D * 2;
  static constexpr int kStages = (D == 64) ? 8 : 4;
  // Q tiles per slot: two at D=64, so the next unit's Q loads while this one runs.
  static constexpr int kQBuf = (D == 64) ? 2 : 1;
  static constexpr bool kSepP = (D == 64);
  static constexpr uint32_t kTmemCols = 512;
  __host__ __device__ static constexpr uint32_t s_col(int slot) { return 128u * slot; }
  __host__ __device__ static constexpr uint32_t p_col(int slot) {
    return kSepP ? 256u + 64u * slot : 128u * slot;
  }
  __host__ __device__ static constexpr uint32_t o_col(int slot) {
    return kSepP ? 384u + 64u * slot : 256u + static_cast<uint32_t>(D) * slot;
  }
};

template <int D>
struct __align__(1024) Smem {
  uint8_t q[kNumSlots][Cfg<D>::kQBuf][Cfg<D>::kTileBytes];
  uint8_t kv[Cfg<D>::kStages][Cfg<D>::kTileBytes];
  uint64_t q_full[kNumSlots][Cfg<D>::kQBuf];
  uint64_t q_empty[kNumSlots][Cfg<D>::kQBuf];
  uint64_t s_full[kNumSlots];
  uint64_t s_empty[kNumSlots];  // separate-P layout: softmax has read S
  uint64_t p_full[kNumSlots];
  uint64_t pv_done[kNumSlots];  // separate-P layout: PV_j finished (P buffer and O stable)
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

// Wait polled by lane 0 only (the lane elect_one_sync picks in a converged warp);
// the outcome is broadcast to the warp.  For the producer and MMA warps, whose
// dependent work is issued by that lane.
template <int D>
__device__ __forceinline__ bool wait_lane0(Smem<D>& sm, uint64_t* bar, uint32_t parity, const Params& p) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = wait_bar(sm, bar, parity, p);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

// ---------------------------------------------------------------- roles
// The producer and the MMA warp keep one state record per slot.  Every function
// that touches a slot's record takes the slot as a template parameter, so the
// records live in registers (a runtime slot index would put them in local memory).

// TMA producer: the whole warp walks the MMA warp's consumption order (per slot:
// Q, K_0, then V_j, K_{j+1} ...; slots interleaved the way the MMA warp visits
// them) and one elected lane issues the copies.  Block indices are fetched 32 at
// a time, one per lane, and the first chunk of the slot's next unit is requested
// when its current unit starts.
struct ProdSlot {
  UnitIter it;
  Unit cur, nxt;
  bool has_cur, has_nxt;
  int j;      // block of `cur` whose V is loaded next
  int units;  // non-empty units started on this slot
  int chunk;  // 32-block chunk of cur's list held in `idx`
  int idx, nxt_idx;
};

struct ProdShared {
  int kv_cnt;  // tiles issued into the K/V ring (both slots)
  uint64_t pol_kv, pol_q;
};

__device__ __forceinline__ int chunk_index(const Params& p, const Unit& x, int chunk, int lane) {
  const int jj = chunk * 32 + lane;
  return jj < x.n ? block_index(p, x, jj) : 0;
}

template <int D>
__device__ __forceinline__ void load_tile(const CUtensorMap* map, int row0, int bh, uint8_t* dst,
                                          uint64_t* bar, uint64_t pol) {
#pragma unroll
  for (int c = 0; c < Cfg<D>::kChunks; ++c)
    tma_load_3d(dst + c * kChunkBytes, map, bar, c * 64, row0, bh, pol);
}

template <int D>
__device__ __forceinline__ bool prod_load_kv(Smem<D>& sm, const Params& p, const CUtensorMap* map,
                                             ProdSlot& s, int j, ProdShared& ps, int lane) {
  using C = Cfg<D>;
  const int stage = ps.kv_cnt % C::kStages;
  const uint32_t phase = (ps.kv_cnt / C::kStages) & 1;
  const int chunk = j >> 5;
  if (chunk != s.chunk) {
    s.idx = chunk_index(p, s.cur, chunk, lane);
    s.chunk = chunk;
  }
  const int kvb = __shfl_sync(0xffffffffu, s.idx, j & 31);
  if (!wait_lane0(sm, &sm.kv_empty[stage], phase ^ 1, p)) return false;
  if (elect_one_sync()) {
    mbar_arrive_expect_tx(&sm.kv_full[stage], C::kTileBytes);
    load_tile<D>(map, kvb * kBlockN, s.cur.bh, sm.kv[stage], &sm.kv_full[stage], ps.pol_kv);
  }
  __syncwarp();
  ++ps.kv_cnt;
  return true;
}

// Make `nxt` current (its first index chunk is already in flight) and look one unit ahead.
__device__ __forceinline__ void prod_advance(ProdSlot& s, const Params& p, int lane) {
  s.has_cur = s.has_nxt;
  s.cur = s.nxt;
  s.idx = s.nxt_idx;
  s.chunk = 0;
  s.j = 0;
  s.has_nxt = s.it.pop_nonempty(s.nxt);
  if (s.has_nxt) s.nxt_idx = chunk_index(p, s.nxt, 0, lane);
}

// Q and K_0 of the slot's current unit.
template <int D, int SLOT>
__device__ __forceinline__ bool prod_start_unit(Smem<D>& sm, const Params& p, const CUtensorMap* tq,
                                                const CUtensorMap* tk, ProdSlot& s, ProdShared& ps,
                                                int lane) {
  using C = Cfg<D>;
  const int b = s.units % C::kQBuf;
  const uint32_t phase = (s.units / C::kQBuf) & 1;
  if (!wait_lane0(sm, &sm.q_empty[SLOT][b], phase ^ 1, p)) return false;
  if (elect_one_sync()) {
    mbar_arrive_expect_tx(&sm.q_full[SLOT][b], C::kTileBytes);
    load_tile<D>(tq, s.cur.qblk * kBlockN, s.cur.bh, sm.q[SLOT][b], &sm.q_full[SLOT][b], ps.pol_q);
  }
  __syncwarp();
  ++s.units;
  return prod_load_kv<D>(sm, p, tk, s, 0, ps, lane);
}

template <int D, int SLOT>
__device__ __forceinline__ bool prod_init(Smem<D>& sm, const Params& p, const CUtensorMap* tq,
                                          const CUtensorMap* tk, ProdSlot& s, ProdShared& ps, int lane) {
  s.it.init(p, SLOT);
  s.units = 0;
  s.has_nxt = s.it.pop_nonempty(s.nxt);
  if (s.has_nxt) s.nxt_idx = chunk_index(p, s.nxt, 0, lane);
  prod_advance(s, p, lane);
  return s.has_cur ? prod_start_unit<D, SLOT>(sm, p, tq, tk, s, ps, lane) : true;
}

// V_j of the current block, then K_{j+1} (or the next unit's Q and K_0).
template <int D, int SLOT>
__device__ __forceinline__ bool prod_step(Smem<D>& sm, const Params& p, const CUtensorMap* tq,
                                          const CUtensorMap* tk, const CUtensorMap* tv, ProdSlot& s,
                                          ProdShared& ps, int lane, bool& any) {
  if (!s.has_cur) return true;
  any = true;
  if (!prod_load_kv<D>(sm, p, tv, s, s.j, ps, lane)) return false;
  ++s.j;
  if (s.j < s.cur.n) return prod_load_kv<D>(sm, p, tk, s, s.j, ps, lane);
  prod_advance(s, p, lane);
  return s.has_cur ? prod_start_unit<D, SLOT>(sm, p, tq, tk, s, ps, lane) : true;
}

template <int D>
__device__ void producer_role(Smem<D>& sm, const Params& p, const CUtensorMap* tq,
                              const CUtensorMap* tk, const CUtensorMap* tv) {
  using C = Cfg<D>;
  static_assert(kNumSlots == 2, "the producer loop visits two slots");
  const int lane = threadIdx.x & 31;
  ProdShared ps;
  ps.kv_cnt = 0;
  ps.pol_kv = policy_evict_last();
  ps.pol_q = policy_evict_first();
  ProdSlot s0, s1;
  bool ok = prod_init<D, 0>(sm, p, tq, tk, s0, ps, lane);
  if (ok) ok = prod_init<D, 1>(sm, p, tq, tk, s1, ps, lane);
  bool any = true;
  while (ok && any) {
    any = false;
    ok = prod_step<D, 0>(sm, p, tq, tk, tv, s0, ps, lane, any);
    if (ok) ok = prod_step<D, 1>(sm, p, tq, tk, tv, s1, ps, lane, any);
  }
  if (!ok && elect_one_sync()) {
    // Drain: wait (bounded) for every TMA copy this warp armed, so that no copy
    // lands in shared memory after the CTA has exited.
    const uint64_t t0 = globaltimer_ns();
    for (int stage = 0; stage < C::kStages; ++stage) {
      const int fills = ps.kv_cnt / C::kStages + (stage < ps.kv_cnt % C::kStages ? 1 : 0);
      if (fills == 0) continue;
      while (!mbar_try_wait(&sm.kv_full[stage], (fills - 1) & 1) &&
             globaltimer_ns() - t0 < p.timeout_ns) {
      }
    }
    for (int slot = 0; slot < kNumSlots; ++slot) {
      const int units = slot == 0 ? s0.units : s1.units;
      for (int b = 0; b < C::kQBuf; ++b) {
        const int fills = units > b ? (units - 1 - b) / C::kQBuf + 1 : 0;
        if (fills == 0) continue;
        while (!mbar_try_wait(&sm.q_full[slot][b], (fills - 1) & 1) &&
               globaltimer_ns() - t0 < p.timeout_ns) {
        }
      }
    }
  }
  __syncwarp();
}

// MMA issuer: one elected thread issues every tcgen05.mma of the CTA.  Per slot and
// block j it issues PV_{j-1} then S_j, so each slot alternates between the tensor
// core and its softmax warpgroup while the other slot fills the gap.
struct MmaSlot {
  UnitIter it;
  Unit cur;
  bool active;
  int j;      // block whose PV is issued next
  int units;  // non-empty units started on this slot
  int blk;    // blocks finished on this slot (p_full phase)
};

struct MmaShared {
  int kv_cnt;
  uint32_t tmem, idesc_s, idesc_pv;
  bool split;
};

template <int D, int SLOT>
__device__ __forceinline__ bool mma_issue_s(Smem<D>& sm, const Params& p, MmaSlot& s, int j,
                                            MmaShared& ms) {
  using C = Cfg<D>;
  const int b = (s.units - 1) % C::kQBuf;  // Q buffer of the current unit
  if (j == 0 && !wait_lane0(sm, &sm.q_full[SLOT][b], ((s.units - 1) / C::kQBuf) & 1, p)) return false;
  const int stage = ms.kv_cnt % C::kStages;
  if (!wait_lane0(sm, &sm.kv_full[stage], (ms.kv_cnt / C::kStages) & 1, p)) return false;
  tc_fence_after();
  // descriptors are warp-uniform: computed by every lane, issued by one
  const uint64_t qd = sdesc_sw128(smem_u32(sm.q[SLOT][b]), 16, 1024);
  const uint64_t kd = sdesc_sw128(smem_u32(sm.kv[stage]), 16, 1024);
  const uint32_t d_s = ms.tmem + C::s_col(SLOT);
  const bool last = j == s.cur.n - 1;
  if (elect_one_sync()) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      // K step kk: 32 bytes into the 128-byte swizzled row, chunk kk / 4
      const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
      umma_ss(d_s, qd + off, kd + off, ms.idesc_s, kk > 0 ? 1u : 0u);
    }
    umma_commit(&sm.kv_empty[stage]);
    umma_commit(&sm.s_full[SLOT]);
    if (last) umma_commit(&sm.q_empty[SLOT][b]);
  }
  __syncwarp();
  ++ms.kv_cnt;
  return true;
}

template <int D, int SLOT>
__device__ __forceinline__ bool mma_issue_pv(Smem<D>& sm, const Params& p, MmaSlot& s, MmaShared& ms) {
  using C = Cfg<D>;
  if (!wait_lane0(sm, &sm.p_full[SLOT], s.blk & 1, p)) return false;
  // O of this slot is free once the epilogue of its previous unit has read it
  if (s.j == 0 && !wait_lane0(sm, &sm.o_empty[SLOT], ((s.units - 1) & 1) ^ 1, p)) return false;
  const int stage = ms.kv_cnt % C::kStages;
  if (!wait_lane0(sm, &sm.kv_full[stage], (ms.kv_cnt / C::kStages) & 1, p)) return false;
  tc_fence_after();
  const uint64_t vd = sdesc_sw128(smem_u32(sm.kv[stage]), kChunkBytes, 1024);
  const uint32_t d_o = ms.tmem + C::o_col(SLOT);
  const uint32_t a_p = ms.tmem + C::s_col(SLOT);
  const uint32_t acc0 = s.j > 0 ? 1u : 0u;
  const bool last = s.j == s.cur.n - 1;
  if (elect_one_sync()) {
    // K step kk covers 16 rows of V (2048 bytes, two 8-row swizzle atoms)
#pragma unroll
    for (int kk = 0; kk < kBlockN / 16; ++kk)
      umma_ts(d_o, a_p + kk * 8, vd + static_cast<uint64_t>(kk * 128), ms.idesc_pv,
              kk > 0 ? 1u : acc0);
    if (ms.split) {
#pragma unroll
      for (int kk = 0; kk < kBlockN / 16; ++kk)
        umma_ts(d_o, a_p + 64 + kk * 8, vd + static_cast<uint64_t>(kk * 128), ms.idesc_pv, 1u);
    }
    umma_commit(&sm.kv_empty[stage]);
    if (last) umma_commit(&sm.o_full[SLOT]);
  }
  __syncwarp();
  ++ms.kv_cnt;
  ++s.blk;
  return true;
}

template <int D, int SLOT>
__device__ __forceinline__ bool mma_start_unit(Smem<D>& sm, const Params& p, MmaSlot& s, MmaShared& ms) {
  s.active = s.it.pop_nonempty(s.cur);
  if (!s.active) return true;
  s.j = 0;
  ++s.units;
  return mma_issue_s<D, SLOT>(sm, p, s, 0, ms);
}

template <int D, int SLOT>
__device__ __forceinline__ bool mma_step(Smem<D>& sm, const Params& p, MmaSlot& s, MmaShared& ms,
                                         bool& any) {
  if (!s.active) return true;
  any = true;
  if (!mma_issue_pv<D, SLOT>(sm, p, s, ms)) return false;
  ++s.j;
  return s.j < s.cur.n ? mma_issue_s<D, SLOT>(sm, p, s, s.j, ms)
                       : mma_start_unit<D, SLOT>(sm, p, s, ms);
}

template <int D>
__device__ void mma_role(Smem<D>& sm, const Params& p, uint32_t tmem) {
  static_assert(kNumSlots == 2, "the MMA loop visits two slots");
  MmaShared ms;
  ms.kv_cnt = 0;
  ms.tmem = tmem;
  ms.idesc_s = idesc_f16_f32(p.is_bf16 != 0, 128, 128, false);
  ms.idesc_pv = idesc_f16_f32(p.is_bf16 != 0, 128, D, true);
  ms.split = p.split_p != 0;
  MmaSlot s0, s1;
  s0.it.init(p, 0);
  s1.it.init(p, 1);
  s0.units = s1.units = 0;
  s0.blk = s1.blk = 0;
  bool ok = mma_start_unit<D, 0>(sm, p, s0, ms);
  if (ok) ok = mma_start_unit<D, 1>(sm, p, s1, ms);
  bool any = true;
  while (ok && any) {
    any = false;
    ok = mma_step<D, 0>(sm, p, s0, ms, any);
    if (ok) ok = mma_step<D, 1>(sm, p, s1, ms, any);
  }
  if (!ok) {
    // Drain every MMA this warp issued before TMEM is released.
    if (elect_one_sync()) umma_commit(&sm.drain);
    __syncwarp();
    const uint64_t t0 = globaltimer_ns();
    while (!mbar_try_wait(&sm.drain, 0) && globaltimer_ns() - t0 < p.timeout_ns) {
    }
  }
}

// ---------------------------------------------------------------- separate-P roles
// With P in its own TMEM columns each slot runs a stream of S ops one block ahead
// of its stream of PV ops.  The MMA warp and the producer walk the same rounds:
//   start:   S(slot 0, block 0), S(slot 1, block 0)
//   round r: S(slot 0, r+1), S(slot 1, r+1), PV(slot 0, r), PV(slot 1, r)
// where a slot's blocks run over its non-empty units back to back.  S ops consume
// K tiles (and the unit's Q at block 0), PV ops consume V tiles, in that order.

// A position in a slot's block stream (producer side: with block indices).
struct ProdCursor {
  UnitIter it;
  Unit cur, nxt;
  bool has_cur, has_nxt;
  int j;      // block of `cur`
  int units;  // non-empty units entered
  int chunk;  // 32-block chunk of cur's list held in `idx`
  int idx, nxt_idx;
};

__device__ __forceinline__ void pc_enter_next(ProdCursor& c, const Params& p, int lane) {
  c.has_cur = c.has_nxt;
  c.cur = c.nxt;
  c.idx = c.nxt_idx;
  c.chunk = 0;
  c.j = 0;
  if (c.has_cur) ++c.units;
  c.has_nxt = c.it.pop_nonempty(c.nxt);
  if (c.has_nxt) c.nxt_idx = chunk_index(p, c.nxt, 0, lane);
}

__device__ __forceinline__ void pc_init(ProdCursor& c, const Params& p, int slot, int lane) {
  c.it.init(p, slot);
  c.units = 0;
  c.has_nxt = c.it.pop_nonempty(c.nxt);
  if (c.has_nxt) c.nxt_idx = chunk_index(p, c.nxt, 0, lane);
  pc_enter_next(c, p, lane);
}

// Move to the next block of the stream; true if that entered a new unit.
__device__ __forceinline__ bool pc_step(ProdCursor& c, const Params& p, int lane) {
  ++c.j;
  if (c.j < c.cur.n) return false;
  pc_enter_next(c, p, lane);
  return true;
}

__device__ __forceinline__ int pc_block(ProdCursor& c, const Params& p, int lane) {
  const int chunk = c.j >> 5;
  if (chunk != c.chunk) {
    c.idx = chunk_index(p, c.cur, chunk, lane);
    c.chunk = chunk;
  }
  return __shfl_sync(0xffffffffu, c.idx, c.j & 31);
}

template <int D>
__device__ __forceinline__ bool sep_load_tile(Smem<D>& sm, const Params& p, const CUtensorMap* map,
                                              int kvb, int bh, ProdShared& ps) {
  using C = Cfg<D>;
  const int stage = ps.kv_cnt % C::kStages;
  const uint32_t phase = (ps.kv_cnt / C::kStages) & 1;
  if (!wait_lane0(sm, &sm.kv_empty[stage], phase ^ 1, p)) return false;
  if (elect_one_sync()) {
    mbar_arrive_expect_tx(&sm.kv_full[stage], C::kTileBytes);
    load_tile<D>(map, kvb * kBlockN, bh, sm.kv[stage], &sm.kv_full[stage], ps.pol_kv);
  }
  __syncwarp();
  ++ps.kv_cnt;
  return true;
}

// Loads for one S op at the K cursor: the unit's Q when at block 0, then K.
template <int D, int SLOT>
__device__ __forceinline__ bool sep_prod_s(Smem<D>& sm, const Params& p, const CUtensorMap* tq,
                                           const CUtensorMap* tk, ProdCursor& c, ProdShared& ps,
                                           int lane) {
  using C = Cfg<D>;
  if (c.j == 0) {
    const int u = c.units - 1;
    const int b = u % C::kQBuf;
    if (!wait_lane0(sm, &sm.q_empty[SLOT][b], ((u / C::kQBuf) & 1) ^ 1, p)) return false;
    if (elect_one_sync()) {
      mbar_arrive_expect_tx(&sm.q_full[SLOT][b], C::kTileBytes);
      load_tile<D>(tq, c.cur.qblk * kBlockN, c.cur.bh, sm.q[SLOT][b], &sm.q_full[SLOT][b], ps.pol_q);
    }
    __syncwarp();
  }
  const int kvb = pc_block(c, p, lane);
  return sep_load_tile<D>(sm, p, tk, kvb, c.cur.bh, ps);
}

// The V load of a slot's PV op r reads the block its K load of round r - 1 read,
// so the K cursor leaves a one-entry record {bh, block} behind for it.
struct PendingV {
  int bh, kvb;
  bool valid;
};

template <int D, int SLOT>
__device__ __forceinline__ bool sep_prod_round_s(Smem<D>& sm, const Params& p, const CUtensorMap* tq,
                                                 const CUtensorMap* tk, ProdCursor& c, PendingV& pv,
                                                 ProdShared& ps, int lane) {
  if (!c.has_cur) {
    pv.valid = false;
    return true;
  }
  pv.bh = c.cur.bh;
  pv.kvb = pc_block(c, p, lane);
  pv.valid = true;
  pc_step(c, p, lane);
  return c.has_cur ? sep_prod_s<D, SLOT>(sm, p, tq, tk, c, ps, lane) : true;
}

template <int D>
__device__ void producer_role_sep(Smem<D>& sm, const Params& p, const CUtensorMap* tq,
                                  const CUtensorMap* tk, const CUtensorMap* tv) {
  using C = Cfg<D>;
  static_assert(kNumSlots == 2, "the producer loop visits two slots");
  const int lane = threadIdx.x & 31;
  ProdShared ps;
  ps.kv_cnt = 0;
  ps.pol_kv = policy_evict_last();
  ps.pol_q = policy_evict_first();
  ProdCursor k0, k1;
  PendingV v0, v1;
  pc_init(k0, p, 0, lane);
  pc_init(k1, p, 1, lane);
  bool ok = true;
  if (k0.has_cur) ok = sep_prod_s<D, 0>(sm, p, tq, tk, k0, ps, lane);
  if (ok && k1.has_cur) ok = sep_prod_s<D, 1>(sm, p, tq, tk, k1, ps, lane);
  while (ok && (k0.has_cur || k1.has_cur)) {
    ok = sep_prod_round_s<D, 0>(sm, p, tq, tk, k0, v0, ps, lane);
    if (ok) ok = sep_prod_round_s<D, 1>(sm, p, tq, tk, k1, v1, ps, lane);
    if (ok && v0.valid) ok = sep_load_tile<D>(sm, p, tv, v0.kvb, v0.bh, ps);
    if (ok && v1.valid) ok = sep_load_tile<D>(sm, p, tv, v1.kvb, v1.bh, ps);
  }
  if (!ok && elect_one_sync()) {
    const uint64_t t0 = globaltimer_ns();
    for (int stage = 0; stage < C::kStages; ++stage) {
      const int fills = ps.kv_cnt / C::kStages + (stage < ps.kv_cnt % C::kStages ? 1 : 0);
      if (fills == 0) continue;
      while (!mbar_try_wait(&sm.kv_full[stage], (fills - 1) & 1) &&
             globaltimer_ns() - t0 < p.timeout_ns) {
      }
    }
    for (int slot = 0; slot < kNumSlots; ++slot) {
      const int units = slot == 0 ? k0.units : k1.units;
      for (int b = 0; b < C::kQBuf; ++b) {
        const int fills = units > b ? (units - 1 - b) / C::kQBuf + 1 : 0;
        if (fills == 0) continue;
        while (!mbar_try_wait(&sm.q_full[slot][b], (fills - 1) & 1) &&
               globaltimer_ns() - t0 < p.timeout_ns) {
        }
      }
    }
  }
  __syncwarp();
}

// MMA-side position in a slot's block stream.
struct MmaCursor {
  UnitIter it;
  Unit cur;
  bool active;
  int j;      // block of `cur`
  int units;  // non-empty units entered
  int ops;    // ops issued on this stream (barrier phase)
};

__device__ __forceinline__ void mc_enter_next(MmaCursor& c) {
  c.active = c.it.pop_nonempty(c.cur);
  c.j = 0;
  if (c.active) ++c.units;
}
__device__ __forceinline__ void mc_init(MmaCursor& c, const Params& p, int slot) {
  c.it.init(p, slot);
  c.units = 0;
  c.ops = 0;
  mc_enter_next(c);
}
__device__ __forceinline__ void mc_step(MmaCursor& c) {
  ++c.ops;
  if (++c.j >= c.cur.n) mc_enter_next(c);
}

template <int D, int SLOT>
__device__ __forceinline__ bool sep_mma_s(Smem<D>& sm, const Params& p, MmaCursor& c, MmaShared& ms) {
  using C = Cfg<D>;
  const int u = c.units - 1;
  const int b = u % C::kQBuf;
  // the softmax must have read the previous S of this slot
  if (c.ops > 0 && !wait_lane0(sm, &sm.s_empty[SLOT], (c.ops - 1) & 1, p)) return false;
  if (c.j == 0 && !wait_lane0(sm, &sm.q_full[SLOT][b], (u / C::kQBuf) & 1, p)) return false;
  const int stage = ms.kv_cnt % C::kStages;
  if (!wait_lane0(sm, &sm.kv_full[stage], (ms.kv_cnt / C::kStages) & 1, p)) return false;
  tc_fence_after();
  const uint64_t qd = sdesc_sw128(smem_u32(sm.q[SLOT][b]), 16, 1024);
  const uint64_t kd = sdesc_sw128(smem_u32(sm.kv[stage]), 16, 1024);
  const uint32_t d_s = ms.tmem + C::s_col(SLOT);
  const bool last = c.j == c.cur.n - 1;
  if (elect_one_sync()) {
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
      umma_ss(d_s, qd + off, kd + off, ms.idesc_s, kk > 0 ? 1u : 0u);
    }
    umma_commit(&sm.kv_empty[stage]);
    umma_commit(&sm.s_full[SLOT]);
    if (last) umma_commit(&sm.q_empty[SLOT][b]);
  }
  __syncwarp();
  ++ms.kv_cnt;
  return true;
}

// The PV op of round r is the block the S op of round r - 1 covered: the S cursor
// leaves {first, last, unit number} behind for it.
struct PendingPV {
  bool valid, first, last;
  int units;  // non-empty units entered when that block was current
  int ops;    // PV ops issued on this slot
};

template <int D, int SLOT>
__device__ __forceinline__ bool sep_mma_pv(Smem<D>& sm, const Params& p, PendingPV& v, MmaShared& ms) {
  using C = Cfg<D>;
  if (!wait_lane0(sm, &sm.p_full[SLOT], v.ops & 1, p)) return false;
  // O of this slot is free once the epilogue of its previous unit has read it
  if (v.first && v.units > 1 && !wait_lane0(sm, &sm.o_empty[SLOT], (v.units - 2) & 1, p))
    return false;
  const int stage = ms.kv_cnt % C::kStages;
  if (!wait_lane0(sm, &sm.kv_full[stage], (ms.kv_cnt / C::kStages) & 1, p)) return false;
  tc_fence_after();
  const uint64_t vd = sdesc_sw128(smem_u32(sm.kv[stage]), kChunkBytes, 1024);
  const uint32_t d_o = ms.tmem + C::o_col(SLOT);
  const uint32_t a_p = ms.tmem + C::p_col(SLOT);
  const uint32_t acc0 = v.first ? 0u : 1u;
  const bool last = v.last;
  if (elect_one_sync()) {
#pragma unroll
    for (int kk = 0; kk < kBlockN / 16; ++kk)
      umma_ts(d_o, a_p + kk * 8, vd + static_cast<uint64_t>(kk * 128), ms.idesc_pv,
              kk > 0 ? 1u : acc0);
    umma_commit(&sm.kv_empty[stage]);
    umma_commit(&sm.pv_done[SLOT]);
    if (last) umma_commit(&sm.o_full[SLOT]);
  }
  __syncwarp();
  ++ms.kv_cnt;
  ++v.ops;
  return true;
}

template <int D, int SLOT>
__device__ __forceinline__ bool sep_mma_round_s(Smem<D>& sm, const Params& p, MmaCursor& c,
                                                PendingPV& v, MmaShared& ms) {
  if (!c.active) {
    v.valid = false;
    return true;
  }
  v.valid = true;
  v.first = c.j == 0;
  v.last = c.j == c.cur.n - 1;
  v.units = c.units;
  mc_step(c);
  return c.active ? sep_mma_s<D, SLOT>(sm, p, c, ms) : true;
}

template <int D>
__device__ void mma_role_sep(Smem<D>& sm, const Params& p, uint32_t tmem) {
  static_assert(kNumSlots == 2, "the MMA loop visits two slots");
  MmaShared ms;
  ms.kv_cnt = 0;
  ms.tmem = tmem;
  ms.idesc_s = idesc_f16_f32(p.is_bf16 != 0, 128, 128, false);
  ms.idesc_pv = idesc_f16_f32(p.is_bf16 != 0, 128, D, true);
  ms.split = false;
  MmaCursor s0, s1;  // S streams of the two slots
  PendingPV v0, v1;  // their PV streams, one block behind
  v0.ops = v1.ops = 0;
  mc_init(s0, p, 0);
  mc_init(s1, p, 1);
  bool ok = true;
  if (s0.active) ok = sep_mma_s<D, 0>(sm, p, s0, ms);
  if (ok && s1.active) ok = sep_mma_s<D, 1>(sm, p, s1, ms);
  while (ok && (s0.active || s1.active)) {
    ok = sep_mma_round_s<D, 0>(sm, p, s0, v0, ms);
    if (ok) ok = sep_mma_round_s<D, 1>(sm, p, s1, v1, ms);
    if (ok && v0.valid) ok = sep_mma_pv<D, 0>(sm, p, v0, ms);
    if (ok && v1.valid) ok = sep_mma_pv<D, 1>(sm, p, v1, ms);
  }
  if (!ok) {
    if (elect_one_sync()) umma_commit(&sm.drain);
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

// 64 consecutive S columns of this thread's row (TMEM lane) into registers.
__device__ __forceinline__ void load_s_half(uint32_t taddr, float (&x)[64]) {
  uint32_t xr[64];
  tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(xr));
  tmem_ld32(taddr + 32, *reinterpret_cast<uint32_t(*)[32]>(xr + 32));
  tmem_wait_ld();
#pragma unroll
  for (int i = 0; i < 64; ++i) x[i] = __uint_as_float(xr[i]);
}

// Mask rule on 64 columns of a PARTIAL block: column i (key kv0 + i) is live iff
// a <= i <= b (causal / window interval, clipped to the keys that exist) and, for
// documents, doc_id[kv0 + i] == dq.  Dead entries become -inf.
__device__ __forceinline__ void apply_mask(const Params& p, float (&x)[64], int a, int b, int kv0,
                                           int dq) {
  if (p.mask_kind == FA_MASK_DOCUMENT_CAUSAL) {
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      uint32_t same = 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int kv = kv0 + c * 32 + i;
        const int d = kv < p.S ? __ldg(p.doc_id + kv) : dq + 1;
        same |= (d == dq ? 1u : 0u) << i;
      }
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const int ii = c * 32 + i;
        if (ii < a || ii > b || !((same >> i) & 1u)) x[ii] = -INFINITY;
      }
    }
  } else {
#pragma unroll
    for (int i = 0; i < 64; ++i)
      if (i < a || i > b) x[i] = -INFINITY;
  }
}

// Max of 64 values: 8 chains of three-input maxima, then a tree.
__device__ __forceinline__ float row_max64(const float (&x)[64]) {
  float mx[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) mx[i] = fmaxf(x[i], x[i + 8]);
#pragma unroll
  for (int i = 16; i < 64; i += 16)
#pragma unroll
    for (int c = 0; c < 8; ++c) mx[c] = fmax3(mx[c], x[i + c], x[i + 8 + c]);
  mx[0] = fmax3(mx[0], mx[1], mx[2]);
  mx[3] = fmax3(mx[3], mx[4], mx[5]);
  mx[6] = fmaxf(mx[6], mx[7]);
  return fmax3(mx[0], mx[3], mx[6]);
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
  const uint32_t t_p = tmem + C::p_col(slot) + lane_off;
  const uint32_t t_o = tmem + C::o_col(slot) + lane_off;
  const bool bf16 = p.is_bf16 != 0;
  // Factor that turns the value kept in x[] into log2 units: the raw score is
  // kept (and scaled inside the exponent's FFMA) unless a score_mod rewrote it.
  const float xs = p.softcap_on ? 1.f : p.scale_log2;
  const bool split = p.split_p != 0 && !C::kSepP;
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
      // Pass 1: the block's row max from the raw scores (a PARTIAL block's masked
      // entries excluded).  The softcap is monotone, so the max of the capped scores
      // is the cap of the raw max.  Pass 2 then turns each half of 64 keys into P with
      // that one max: P_hi of half h goes to P columns [32h, 32h + 32); with the
      // split, P_lo goes to columns 64 + [32h, 32h + 32), held in registers until
      // half 1 has been read (in the aliased layout those columns are still S).
      const int a = lo - kvb * kBlockN;  // live columns of the block: a <= i <= b
      const int b = hi - kvb * kBlockN;
      float rmax = -INFINITY;
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        float x[64];
        load_s_half(t_s + h * 64, x);
        if (!full) apply_mask(p, x, a - h * 64, b - h * 64, kvb * kBlockN + h * 64, dq);
        rmax = fmaxf(rmax, row_max64(x));
      }
      float mb = rmax;
      if (rmax != -INFINITY) {
        if (p.softcap_on) {
          mb = p.cap_a - 2.f * p.cap_a * rcp_approx(ex2_approx(rmax * p.cap_k) + 1.f);
        } else {
          mb = rmax * xs;
        }
      }
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
      const float neg_mu = (m == -INFINITY) ? 0.f : -m;
      if constexpr (C::kSepP) {
        // the previous PV of this slot must be done before P is overwritten or O rescaled
        if (blk > 0 && !wait_warp(sm, &sm.pv_done[slot], (blk - 1) & 1, p)) return;
        tc_fence_after();
      }
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
      uint32_t pl_hold[32];
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        float x[64];
        load_s_half(t_s + h * 64, x);
        if (h == 1) {
          if constexpr (C::kSepP) {  // all of S is read: the MMA warp may refill it
            tc_fence_before();
            __syncwarp();
            if ((t & 31) == 0) mbar_arrive(&sm.s_empty[slot]);
          }
          if (split) tmem_st32(t_p + 64, pl_hold);
        }
        if (p.softcap_on) {  // x = log2(e) * c * tanh(s * scale / c)
#pragma unroll
          for (int i = 0; i < 64; i += 2) {
            const float2 e = make_float2(ex2_approx(x[i] * p.cap_k), ex2_approx(x[i + 1] * p.cap_k));
            const float2 r = make_float2(rcp_approx(e.x + 1.f), rcp_approx(e.y + 1.f));
            const float2 v = fma2(r, make_float2(-2.f * p.cap_a, -2.f * p.cap_a),
                                  make_float2(p.cap_a, p.cap_a));
            x[i] = v.x;
            x[i + 1] = v.y;
          }
        }
        if (!full) apply_mask(p, x, a - h * 64, b - h * 64, kvb * kBlockN + h * 64, dq);
        // P = exp2(x * xs - m) as 16-bit pairs; with the split, P_hi = p truncated to
        // bf16 and P_lo = round(p - P_hi), so P_hi + P_lo carries ~16 significant bits.
        float2 sums[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) sums[i] = make_float2(0.f, 0.f);
        const float2 xs2 = make_float2(xs, xs), nm2 = make_float2(neg_mu, neg_mu);
        uint32_t ph[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 a2 = fma2(make_float2(x[2 * i], x[2 * i + 1]), xs2, nm2);
          const float2 pp = make_float2(ex2_approx(a2.x), ex2_approx(a2.y));
          sums[i & 3] = add2(sums[i & 3], pp);
          if (!split) {
            ph[i] = pack2(pp.x, pp.y, bf16);
          } else if (bf16) {
            const uint32_t u0 = __float_as_uint(pp.x), u1 = __float_as_uint(pp.y);
            ph[i] = __byte_perm(u0, u1, 0x7632);
            const float2 lo2 = sub2(pp, make_float2(__uint_as_float(u0 & 0xFFFF0000u),
                                                    __uint_as_float(u1 & 0xFFFF0000u)));
            pl_hold[i] = pack2(lo2.x, lo2.y, true);
          } else {
            ph[i] = pack2(pp.x, pp.y, false);
            float h0, h1;
            unpack2(ph[i], false, h0, h1);
            pl_hold[i] = pack2(pp.x - h0, pp.y - h1, false);
          }
        }
        tmem_st32(t_p + h * 32, ph);
        sums[0] = add2(add2(sums[0], sums[1]), add2(sums[2], sums[3]));
        l += sums[0].x + sums[0].y;
      }
      if (split) tmem_st32(t_p + 96, pl_hold);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if ((t & 31) == 0) mbar_arrive(&sm.p_full[slot]);
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
    __syncwarp();
    if ((t & 31) == 0) mbar_arrive(&sm.o_empty[slot]);
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
      mbar_init(&sm.s_empty[s], 4);
      mbar_init(&sm.pv_done[s], 1);
      mbar_init(&sm.p_full[s], 4);   // one arrival per softmax warp
      mbar_init(&sm.o_full[s], 1);
      mbar_init(&sm.o_empty[s], 4);
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
    if constexpr (Cfg<D>::kSepP)
      producer_role_sep<D>(sm, p, &tmap_q, &tmap_k, &tmap_v);
    else
      producer_role<D>(sm, p, &tmap_q, &tmap_k, &tmap_v);
  } else if (warp == kMmaWarp) {
    if constexpr (Cfg<D>::kSepP)
      mma_role_sep<D>(sm, p, tmem);
    else
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
