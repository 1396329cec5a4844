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
// Kernel organisation (one persistent CTA per SM, 352 threads, 11 warps):
//   warps 0-3   softmax warpgroup of slot 0     warps 4-7   softmax warpgroup of slot 1
//   warp 8      TMA producer of slot 0          warp 9      TMA producer of slot 1
//   warp 10     tcgen05.mma issuer of both slots and TMEM owner
// A "slot" owns one 128-row Q tile at a time, an S region and a P region in TMEM and
// an O accumulator (D TMEM columns).  The two slots work on independent work units
// (batch*head, q-block) so that the tensor core computes one slot's products while
// the other slot's softmax runs.  Each slot streams its own K and V tiles through
// shared-memory rings filled by TMA (128-byte swizzle, no multicast).  The MMA warp
// polls both slots and issues whichever product is ready.
//
// Per block j of a unit:
//   S_j  = Q K_j^T        (SS MMA, M=128 N=128 K=D, fp32 in TMEM)    -> s_full
//   softmax warpgroup: S -> registers, scale (+ softcap), mask on PARTIAL blocks only,
//   running max with rescaling of O, P = exp2(x - m) as 16-bit values   -> p_full
//   O   += P V_j          (TS MMA: A = P from TMEM, B = V MN-major)
// D = 64: P has its own TMEM columns, so S_{j+1} is computed during softmax j and the
// softmax waits for PV_{j-1} (pv_done) only before it overwrites P.  D = 128: P
// overwrites the S it came from (TMEM holds no more), S_{j+1} is issued after PV_j
// (tcgen05 operations of one thread run in issue order), and the commit that
// signals S_{j+1} also means PV_j is done.
// Epilogue of a unit, O / l: at D = 64, for a unit of at most stage_max_blocks()
// blocks, each softmax warp writes its 32 rows into the unit's Q tile and one lane
// stores them with a TMA tensor store, so the LSU carries no output traffic; longer
// units and D = 128 store from registers.
//
// Every mbarrier wait is bounded: after `timeout_ns` the waiting warp sets an abort
// flag and the device error word, all roles stop, in-flight copies and MMAs are
// drained (again with a bound), TMEM is freed and the CTA returns.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdint>
#include <mutex>

#include "fa_internal.h"
#include "sm100_ptx.cuh"

namespace fa {
namespace {

constexpr int kNumSlots = 2;
constexpr int kSoftmaxWarps = 4 * kNumSlots;
constexpr int kProducerWarp = kSoftmaxWarps;      // + slot: one TMA producer warp per slot
constexpr int kMmaWarp = kSoftmaxWarps + kNumSlots;
constexpr int kThreads = (kSoftmaxWarps + kNumSlots + 1) * 32;  // + 2 producers, MMA
// Registers: 168 per thread.  Warps are spread over the SM's four sub-partitions,
// three per sub-partition here, and each sub-partition has a quarter of the
// register file (16384): 3 x 32 x 168 fits, 3 x 32 x 176 does not.
constexpr int kBlockN = 128;                 // rows of a Q tile / K,V tile
constexpr int kChunkBytes = 128 * 128;       // one TMA box: 128 rows x 64 elems x 2 B
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// Mask families, one kernel instantiation each (only its mask code is compiled in):
// causal and sliding-window (an interval of keys per row), document, tabulated.
constexpr int kMaskRange = 0;
constexpr int kMaskDoc = 1;
constexpr int kMaskBitmap = 2;
__host__ __device__ constexpr int mask_family(int kind) {
  return kind == FA_MASK_DOCUMENT_CAUSAL ? kMaskDoc : (kind == FA_MASK_BITMAP ? kMaskBitmap : kMaskRange);
}
// Units of at most this many blocks store O through the staging tile (TMA store);
// longer ones store it from registers.  Measured at D = 64: short units end every
// few blocks, and their direct stores queued behind one another in the load/store
// unit (window 256, 32k: 77 -> 74 us staged); a long unit's stores drain during
// its successor, and there the staging cost 3-11% (window 4096; causal 8192:
// 127 -> 142 us with every unit staged).  The tabulated-mask kernel stages every
// unit: with both epilogues compiled in, its register allocation spills in the
// block loop, and the bitmap loads there wait on the spilled values (8192, random
// block classes: 305 us mixed, 259 us all staged, 262 us all direct).
template <int MK>
__host__ __device__ constexpr int stage_max_blocks() {
  return MK == kMaskBitmap ? (1 << 30) : 4;
}

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
  // Per slot: a ring of K tiles and a ring of V tiles.  At D = 64 the K ring has
  // three stages (the shared memory left after two of everything takes one more
  // tile per slot; a third K stage lets the producer run a block further ahead and
  // gained 1-1.5% on windows and documents, a third V stage nothing).
  static constexpr int kKRing = (D == 64) ? 3 : 1;
  static constexpr int kVRing = (D == 64) ? 2 : 1;
  // Q tiles per slot: two at D=64, so the next unit's Q loads while this one runs.
  static constexpr int kQBuf = (D == 64) ? 2 : 1;
  static constexpr bool kSepP = (D == 64);
  // D = 64: O of a short unit leaves through shared memory, one TMA store per warp
  // (its 32 rows), so the epilogue issues no global stores of its own.  The staging
  // tile is the unit's own Q tile (same size and swizzle, no longer read once the
  // unit's MMAs are done), which the softmax warps then release together with the
  // MMA warp.  D = 128 (one Q buffer, reloaded at once for the next unit) stores
  // from registers.
  static constexpr bool kStageO = (D == 64);
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
  uint8_t k[kNumSlots][Cfg<D>::kKRing][Cfg<D>::kTileBytes];
  uint8_t v[kNumSlots][Cfg<D>::kVRing][Cfg<D>::kTileBytes];
  uint64_t q_full[kNumSlots][Cfg<D>::kQBuf];
  uint64_t q_empty[kNumSlots][Cfg<D>::kQBuf];
  uint64_t k_full[kNumSlots][Cfg<D>::kKRing];
  uint64_t k_empty[kNumSlots][Cfg<D>::kKRing];
  uint64_t v_full[kNumSlots][Cfg<D>::kVRing];
  uint64_t v_empty[kNumSlots][Cfg<D>::kVRing];
  uint64_t s_full[kNumSlots];
  uint64_t s_empty[kNumSlots];  // separate-P layout: softmax has read S
  uint64_t p_full[kNumSlots];
  uint64_t pv_done[kNumSlots];  // separate-P layout: PV_j finished (P buffer and O stable)
  uint64_t o_full[kNumSlots];
  uint64_t o_empty[kNumSlots];
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort_flag;
};

// Dynamic shared memory of a CTA (the struct plus 1024 bytes to align it) within the
// 227 KB a block may use.
static_assert(sizeof(Smem<64>) + 1024 <= 232448, "shared memory of the D = 64 forward");
static_assert(sizeof(Smem<128>) + 1024 <= 232448, "shared memory of the D = 128 forward");

struct Params {
  const int32_t* kv_idx;
  const int32_t* full_idx;
  const int32_t* sched;  // per rank k: [2k] = q-block row, [2k+1] = partial | full << 16
  const int32_t* doc_id;
  const uint32_t* bitmap;  // tabulated mask: row q's words at bitmap + q * bitmap_words
  void* out;
  float* lse;
  int32_t* err;
  int BH, L, S, n_kv, num_units, bitmap_words;
  int H, Hkv, kv_group;  // query heads, K/V heads, H / Hkv
  // per-(batch, head) masks: instance of (b, h) = (mask_b ? b : 0) * mask_heads +
  // (mask_h ? h : 0); each instance has its tables, schedule and mask data
  int n_q, mask_b, mask_h, mask_heads, doc_len;
  int mask_kind, window, softcap_on, is_bf16;
  int split_p;       // P fed to the PV product as two 16-bit terms (hi + lo)
  // Deferred rescale: the running max used for P (and O, l) moves only when the
  // block max exceeds it by more than this (log2 units).  0: P always uses the
  // exact running max, so each row's largest weight is exactly 1 in 16 bits.
  float rescale_thr;
  float scale_log2;  // scale * log2(e)
  float cap_k;       // 2 * scale * log2(e) / c : exp2(s * cap_k) = e^(2 s scale / c)
  float cap_a;       // c * log2(e)
  unsigned long long timeout_ns;
  int stall_mma;  // testing hook: the MMA warp issues nothing (see fa_debug_set_mma_stall)
};

// ---------------------------------------------------------------- scheduling
// Work unit u -> (rank u / BH of the LPT-ordered schedule table, batch*head u % BH).
// Units are dealt to the grid's (CTA, slot) workers in rounds, alternating
// direction ("snake"), so the heaviest rows of the LPT order spread over all
// workers.  Every role of a CTA walks the same sequence.
struct Unit {
  int bh, qblk, np, n;
  int kvbh;  // batch * Hkv + K/V head of this unit's query head
  int inst;  // mask instance of (b, h)
};

// BHM: the kernel serves per-(batch, head) masks; without it every unit reads
// instance 0 and the instance arithmetic is compiled out.
template <bool BHM>
__device__ __forceinline__ int mask_instance(const Params& p, int bh) {
  if constexpr (!BHM) return 0;
  const int b = bh / p.H;
  return (p.mask_b ? b : 0) * p.mask_heads + (p.mask_h ? bh - b * p.H : 0);
}

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
template <bool BHM>
struct UnitIter {
  int worker, round;
  int nu;   // next unit id, -1 when exhausted
  int2 nx;  // its schedule entry (load in flight)

  __device__ __forceinline__ void init(const Params& p, int slot) {
    worker = static_cast<int>(blockIdx.x) * kNumSlots + slot;
    round = 0;
    fetch(p);
  }
  __device__ __forceinline__ void fetch(const Params& p) {
    const int workers = static_cast<int>(gridDim.x) * kNumSlots;
    const int u = round * workers + ((round & 1) ? (workers - 1 - worker) : worker);
    ++round;
    nu = u < p.num_units ? u : -1;
    if (nu >= 0) {
      const int k = nu / p.BH;
      nx = ldg_nc_v2(p.sched + 2 * (static_cast<size_t>(mask_instance<BHM>(p, nu - k * p.BH)) * p.n_q + k));
    }
  }
  __device__ __forceinline__ bool pop(const Params& p, Unit& x) {
    if (nu < 0) return false;
    const int k = nu / p.BH;
    x.bh = nu - k * p.BH;
    // grouped-query attention: query head h reads K/V head h / kv_group
    x.kvbh = p.kv_group == 1 ? x.bh : (x.bh / p.H) * p.Hkv + (x.bh % p.H) / p.kv_group;
    x.inst = mask_instance<BHM>(p, x.bh);
    x.qblk = nx.x;
    x.np = nx.y & 0xFFFF;
    x.n = x.np + (nx.y >> 16);
    fetch(p);
    return true;
  }
  __device__ __forceinline__ bool pop_nonempty(const Params& p, Unit& x) {
    while (pop(p, x))
      if (x.n > 0) return true;
    return false;
  }
};

// kv-block index of the j-th block of the unit: partial blocks first, then full ones.
__device__ __forceinline__ int block_index(const Params& p, const Unit& x, int j) {
  const size_t row = (static_cast<size_t>(x.inst) * p.n_q + x.qblk) * p.n_kv;
  return j < x.np ? ldg_nc(p.kv_idx + row + j) : ldg_nc(p.full_idx + row + (j - x.np));
}

// ---------------------------------------------------------------- bounded wait
template <int D>
__device__ __forceinline__ bool wait_slow(Smem<D>& sm, uint64_t* bar, uint32_t parity, const Params& p) {
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    // (not unrolled: every wait site inlines this loop, and the kernel's code must
    // stay small enough for the instruction caches)
#pragma unroll 1
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
// Each slot has its own producer warp, its own ring of K tiles and its own ring of
// V tiles; the MMA warp serves both slots, issuing whichever slot's next MMA is
// ready.  A slot's blocks run over its non-empty units back to back (block i of
// the slot's stream); K_i goes to K-ring stage i % kKRing, V_i to V-ring stage
// i % kVRing, so producer and MMA warp agree on stages without a shared order.
// The MMA warp's per-slot functions take the slot as a template parameter, so that
// the state of both slots lives in registers; the producer code takes it as a
// runtime value, so that both producer warps run one copy of it (the kernel's code
// size is held down for the instruction caches: each instantiation holds only its
// own mask family and score_mod, and slow paths stay loops).

// Producer-side position in a slot's block stream, with block indices fetched 32
// at a time (one per lane) and the next unit's first chunk requested early.
template <bool BHM>
struct ProdCursor {
  UnitIter<BHM> it;
  Unit cur, nxt;
  bool has_cur, has_nxt;
  int j;      // block of `cur`
  int units;  // non-empty units entered
  int chunk;  // 32-block chunk of cur's list held in `idx`
  int idx, nxt_idx;
};

__device__ __forceinline__ int chunk_index(const Params& p, const Unit& x, int chunk, int lane) {
  const int jj = chunk * 32 + lane;
  return jj < x.n ? block_index(p, x, jj) : 0;
}

template <bool BHM>
__device__ __forceinline__ void pc_enter_next(ProdCursor<BHM>& c, const Params& p, int lane) {
  c.has_cur = c.has_nxt;
  c.cur = c.nxt;
  c.idx = c.nxt_idx;
  c.chunk = 0;
  c.j = 0;
  if (c.has_cur) ++c.units;
  c.has_nxt = c.it.pop_nonempty(p, c.nxt);
  if (c.has_nxt) c.nxt_idx = chunk_index(p, c.nxt, 0, lane);
}

template <bool BHM>
__device__ __forceinline__ void pc_init(ProdCursor<BHM>& c, const Params& p, int slot, int lane) {
  c.it.init(p, slot);
  c.units = 0;
  c.has_nxt = c.it.pop_nonempty(p, c.nxt);
  if (c.has_nxt) c.nxt_idx = chunk_index(p, c.nxt, 0, lane);
  pc_enter_next(c, p, lane);
}

template <bool BHM>
__device__ __forceinline__ void pc_step(ProdCursor<BHM>& c, const Params& p, int lane) {
  if (++c.j >= c.cur.n) pc_enter_next(c, p, lane);
}

template <bool BHM>
__device__ __forceinline__ int pc_block(ProdCursor<BHM>& c, const Params& p, int lane) {
  const int chunk = c.j >> 5;
  if (chunk != c.chunk) {
    c.idx = chunk_index(p, c.cur, chunk, lane);
    c.chunk = chunk;
  }
  return __shfl_sync(0xffffffffu, c.idx, c.j & 31);
}

template <int D>
__device__ __forceinline__ void load_tile(const CUtensorMap* map, int row0, int bh, uint8_t* dst,
                                          uint64_t* bar, uint64_t pol) {
#pragma unroll
  for (int c = 0; c < Cfg<D>::kChunks; ++c)
    tma_load_3d(dst + c * kChunkBytes, map, bar, c * 64, row0, bh, pol);
}

// Arm `full` for one tile and issue its TMA copy, after `empty` shows the stage free.
template <int D>
__device__ __forceinline__ bool produce(Smem<D>& sm, const Params& p, const CUtensorMap* map,
                                       int row0, int bh, uint8_t* dst, uint64_t* full,
                                       uint64_t* empty, int fill, uint64_t pol) {
  if (!wait_lane0(sm, empty, (fill & 1) ^ 1, p)) return false;
  if (elect_one_sync()) {
    mbar_arrive_expect_tx(full, Cfg<D>::kTileBytes);
    load_tile<D>(map, row0, bh, dst, full, pol);
  }
  __syncwarp();
  return true;
}

struct ProdCounts {
  int k, v;  // K / V tiles issued on this slot
};

template <int D, bool BHM>
__device__ __forceinline__ bool produce_k(int SLOT, Smem<D>& sm, const Params& p, const CUtensorMap* tq,
                                          const CUtensorMap* tk, ProdCursor<BHM>& c, ProdCounts& n,
                                          int kvb, uint64_t pol_q, uint64_t pol_kv) {
  using C = Cfg<D>;
  if (c.j == 0) {  // the unit's Q tile first
    const int u = c.units - 1;
    const int b = u % C::kQBuf;
    if (!produce<D>(sm, p, tq, c.cur.qblk * kBlockN, c.cur.bh, sm.q[SLOT][b], &sm.q_full[SLOT][b],
                    &sm.q_empty[SLOT][b], u / C::kQBuf, pol_q))
      return false;
  }
  const int st = n.k % C::kKRing;
  if (!produce<D>(sm, p, tk, kvb * kBlockN, c.cur.kvbh, sm.k[SLOT][st], &sm.k_full[SLOT][st],
                  &sm.k_empty[SLOT][st], n.k / C::kKRing, pol_kv))
    return false;
  ++n.k;
  return true;
}

template <int D>
__device__ __forceinline__ bool produce_v(int SLOT, Smem<D>& sm, const Params& p, const CUtensorMap* tv,
                                          ProdCounts& n, int kvb, int bh, uint64_t pol_kv) {
  using C = Cfg<D>;
  const int st = n.v % C::kVRing;
  if (!produce<D>(sm, p, tv, kvb * kBlockN, bh, sm.v[SLOT][st], &sm.v_full[SLOT][st],
                  &sm.v_empty[SLOT][st], n.v / C::kVRing, pol_kv))
    return false;
  ++n.v;
  return true;
}

// One producer warp per slot.  Separate-P layout: K runs one block ahead of V
// (K_0, K_1, V_0, K_2, V_1, ...), matching S_{i+1} being issued during softmax i.
// Aliased layout: K_i, V_i, K_{i+1}, ...
template <int D, bool BHM>
__device__ void producer_role(int SLOT, Smem<D>& sm, const Params& p, const CUtensorMap* tq,
                              const CUtensorMap* tk, const CUtensorMap* tv) {
  using C = Cfg<D>;
  const int lane = threadIdx.x & 31;
  const uint64_t pol_kv = policy_evict_last();
  const uint64_t pol_q = policy_evict_first();
  ProdCursor<BHM> c;
  ProdCounts n{0, 0};
  pc_init(c, p, SLOT, lane);
  bool ok = true;
  if constexpr (C::kSepP) {
    int pend_kvb = 0, pend_bh = 0;
    bool pend = false;
    if (c.has_cur) {
      pend_kvb = pc_block(c, p, lane);
      pend_bh = c.cur.kvbh;
      pend = true;
      ok = produce_k<D>(SLOT, sm, p, tq, tk, c, n, pend_kvb, pol_q, pol_kv);
    }
    while (ok && pend) {
      pc_step(c, p, lane);
      int next_kvb = 0, next_bh = 0;
      const bool next = c.has_cur;
      if (next) {
        next_kvb = pc_block(c, p, lane);
        next_bh = c.cur.kvbh;
        ok = produce_k<D>(SLOT, sm, p, tq, tk, c, n, next_kvb, pol_q, pol_kv);
      }
      if (ok) ok = produce_v<D>(SLOT, sm, p, tv, n, pend_kvb, pend_bh, pol_kv);
      pend = next;
      pend_kvb = next_kvb;
      pend_bh = next_bh;
    }
  } else {
    while (ok && c.has_cur) {
      const int kvb = pc_block(c, p, lane);
      ok = produce_k<D>(SLOT, sm, p, tq, tk, c, n, kvb, pol_q, pol_kv);
      if (ok) ok = produce_v<D>(SLOT, sm, p, tv, n, kvb, c.cur.kvbh, pol_kv);
      pc_step(c, p, lane);
    }
  }
  if (!ok && elect_one_sync()) {
    // Drain: wait (bounded) for every TMA copy this warp armed, so that no copy
    // lands in shared memory after the CTA has exited.
    const uint64_t t0 = globaltimer_ns();
    for (int st = 0; st < C::kKRing; ++st) {
      const int fills = n.k / C::kKRing + (st < n.k % C::kKRing ? 1 : 0);
      while (fills > 0 && !mbar_try_wait(&sm.k_full[SLOT][st], (fills - 1) & 1) &&
             globaltimer_ns() - t0 < p.timeout_ns) {
      }
    }
    for (int st = 0; st < C::kVRing; ++st) {
      const int fills = n.v / C::kVRing + (st < n.v % C::kVRing ? 1 : 0);
      while (fills > 0 && !mbar_try_wait(&sm.v_full[SLOT][st], (fills - 1) & 1) &&
             globaltimer_ns() - t0 < p.timeout_ns) {
      }
    }
    for (int b = 0; b < C::kQBuf; ++b) {
      const int fills = c.units > b ? (c.units - 1 - b) / C::kQBuf + 1 : 0;
      while (fills > 0 && !mbar_try_wait(&sm.q_full[SLOT][b], (fills - 1) & 1) &&
             globaltimer_ns() - t0 < p.timeout_ns) {
      }
    }
  }
  __syncwarp();
}

// MMA-side position in a slot's block stream (no block indices needed).
template <bool BHM>
struct MmaStream {
  UnitIter<BHM> it;
  Unit cur;
  bool active;
  int j;      // block of `cur`
  int units;  // non-empty units entered
  int i;      // position in the slot's block stream
};

template <bool BHM>
__device__ __forceinline__ void ms_enter_next(MmaStream<BHM>& c, const Params& p) {
  c.active = c.it.pop_nonempty(p, c.cur);
  c.j = 0;
  if (c.active) ++c.units;
}
template <bool BHM>
__device__ __forceinline__ void ms_init(MmaStream<BHM>& c, const Params& p, int slot) {
  c.it.init(p, slot);
  c.units = 0;
  c.i = 0;
  ms_enter_next(c, p);
}
template <bool BHM>
__device__ __forceinline__ void ms_step(MmaStream<BHM>& c, const Params& p) {
  ++c.i;
  if (++c.j >= c.cur.n) ms_enter_next(c, p);
}

struct MmaShared {
  uint32_t tmem, idesc_s, idesc_pv;
  bool split;
};

// Probe by the whole warp: every lane tests the phase (one shared-memory access for
// the warp) and the vote makes the answer warp-uniform; no shuffle from a leader lane.
__device__ __forceinline__ bool probe(uint64_t* bar, uint32_t parity) {
  return __all_sync(0xffffffffu, mbar_test_wait(bar, parity));
}

// S_i = Q K_i^T for the slot's stream position `c`, if its inputs are ready.
// `prev_done`: the S buffer may be overwritten (aliased layout: PV_{i-1} issued;
// separate-P layout: the softmax has read S_{i-1}).
template <int D, int SLOT, bool BHM>
__device__ __forceinline__ bool try_s(Smem<D>& sm, const Params& p, MmaStream<BHM>& c,
                                      MmaShared& ms) {
  using C = Cfg<D>;
  const int u = c.units - 1;
  const int b = u % C::kQBuf;
  const int st = c.i % C::kKRing;
  if constexpr (C::kSepP) {
    if (c.i > 0 && !probe(&sm.s_empty[SLOT], (c.i - 1) & 1)) return false;
  }
  if (c.j == 0 && !probe(&sm.q_full[SLOT][b], (u / C::kQBuf) & 1)) return false;
  if (!probe(&sm.k_full[SLOT][st], (c.i / C::kKRing) & 1)) return false;
  tc_fence_after();
  // descriptors are warp-uniform: computed by every lane, issued by one
  const uint64_t qd = sdesc_sw128(smem_u32(sm.q[SLOT][b]), 16, 1024);
  const uint64_t kd = sdesc_sw128(smem_u32(sm.k[SLOT][st]), 16, 1024);
  const uint32_t d_s = ms.tmem + C::s_col(SLOT);
  const bool last = c.j == c.cur.n - 1;
  if (elect_one_sync()) {
    // (fully unrolled at D=64, where the MMAs are short enough for issue cost to show)
#pragma unroll(D == 64 ? 4 : 1)
    for (int kk = 0; kk < D / 16; ++kk) {
      // K step kk: 32 bytes into the 128-byte swizzled row, chunk kk / 4
      const uint64_t off = static_cast<uint64_t>(((kk >> 2) * kChunkBytes + (kk & 3) * 32) >> 4);
      umma_ss(d_s, qd + off, kd + off, ms.idesc_s, kk > 0 ? 1u : 0u);
    }
    umma_commit(&sm.k_empty[SLOT][st]);
    umma_commit(&sm.s_full[SLOT]);
    if (last) umma_commit(&sm.q_empty[SLOT][b]);
  }
  __syncwarp();
  ms_step(c, p);
  return true;
}

// O += P_i V_i for the slot's stream position `c`, if its inputs are ready.
template <int D, int SLOT, bool BHM>
__device__ __forceinline__ bool try_pv(Smem<D>& sm, const Params& p, MmaStream<BHM>& c,
                                       MmaShared& ms) {
  using C = Cfg<D>;
  const int st = c.i % C::kVRing;
  if (!probe(&sm.p_full[SLOT], c.i & 1)) return false;
  // O of this slot is free once the epilogue of its previous unit has read it
  if (c.j == 0 && c.units > 1 && !probe(&sm.o_empty[SLOT], (c.units - 2) & 1)) return false;
  if (!probe(&sm.v_full[SLOT][st], (c.i / C::kVRing) & 1)) return false;
  tc_fence_after();
  const uint64_t vd = sdesc_sw128(smem_u32(sm.v[SLOT][st]), kChunkBytes, 1024);
  const uint32_t d_o = ms.tmem + C::o_col(SLOT);
  const uint32_t a_p = ms.tmem + C::p_col(SLOT);
  const uint32_t acc0 = c.j > 0 ? 1u : 0u;
  const bool last = c.j == c.cur.n - 1;
  if (elect_one_sync()) {
    // K step kk covers 16 rows of V (2048 bytes, two 8-row swizzle atoms)
#pragma unroll(D == 64 ? 8 : 1)
    for (int kk = 0; kk < kBlockN / 16; ++kk)
      umma_ts(d_o, a_p + kk * 8, vd + static_cast<uint64_t>(kk * 128), ms.idesc_pv,
              kk > 0 ? 1u : acc0);
    if (ms.split) {
#pragma unroll 1
      for (int kk = 0; kk < kBlockN / 16; ++kk)
        umma_ts(d_o, a_p + 64 + kk * 8, vd + static_cast<uint64_t>(kk * 128), ms.idesc_pv, 1u);
    }
    umma_commit(&sm.v_empty[SLOT][st]);
    if constexpr (C::kSepP) umma_commit(&sm.pv_done[SLOT]);
    if (last) umma_commit(&sm.o_full[SLOT]);
  }
  __syncwarp();
  ms_step(c, p);
  return true;
}

// Per slot: its S stream and its PV stream (the PV stream trails).  The PV is tried
// first.  In the aliased layout S_{i+1} may only follow PV_i (the MMAs of one thread
// run in issue order, so PV_i has read P before S_{i+1} overwrites it), and this
// lets S_{i+1} follow it in the same pass (a pass later cost the D = 128 softcap
// workload 15%).  In the separate-P layout a PV ahead of an S that is also ready
// lets the softmax, which waits for PV_{i-1} before it writes P_i, go on sooner
// (causal 8192: 131 -> 123 us; window 4096: 121 -> 116 us).
template <int D, int SLOT, bool BHM>
__device__ __forceinline__ bool mma_slot(Smem<D>& sm, const Params& p, MmaStream<BHM>& cs,
                                         MmaStream<BHM>& cp, MmaShared& ms) {
  bool progress = false;
  if (cp.active && (!cs.active || cp.i < cs.i)) progress |= try_pv<D, SLOT>(sm, p, cp, ms);
  if (cs.active && (Cfg<D>::kSepP || cs.i == cp.i)) progress |= try_s<D, SLOT>(sm, p, cs, ms);
  return progress;
}

template <int D, bool BHM>
__device__ void mma_role(Smem<D>& sm, const Params& p, uint32_t tmem) {
  static_assert(kNumSlots == 2, "the MMA loop serves two slots");
  MmaShared ms;
  ms.tmem = tmem;
  ms.idesc_s = idesc_f16_f32(p.is_bf16 != 0, 128, 128, false);
  ms.idesc_pv = idesc_f16_f32(p.is_bf16 != 0, 128, D, true);
  ms.split = p.split_p != 0 && !Cfg<D>::kSepP;
  MmaStream<BHM> s0, p0, s1, p1;
  ms_init(s0, p, 0);
  ms_init(p0, p, 0);
  ms_init(s1, p, 1);
  ms_init(p1, p, 1);
  bool ok = true;
  uint64_t last_progress = 0;  // 0: progress since the last idle check
  int idle = 0;
  while (p0.active || p1.active) {
    bool progress = false;
    if (!p.stall_mma) {
      progress = mma_slot<D, 0>(sm, p, s0, p0, ms);
      progress |= mma_slot<D, 1>(sm, p, s1, p1, ms);
    }
    if (progress) {
      idle = 0;
      last_progress = 0;
      continue;
    }
    // nothing ready: back off briefly, and give up after the timeout
    if (++idle >= 64) {
      idle = 0;
      const uint64_t now = globaltimer_ns();
      if (last_progress == 0) last_progress = now;
      if (sm.abort_flag) {
        ok = false;
        break;
      }
      if (now - last_progress > p.timeout_ns) {
        sm.abort_flag = 1;
        if ((threadIdx.x & 31) == 0) atomicOr(p.err, kDevErrTimeout);
        ok = false;
        break;
      }
    }
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
  reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(xr));
  reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(xr + 32));
#pragma unroll
  for (int i = 0; i < 64; ++i) x[i] = __uint_as_float(xr[i]);
}

// v if a <= I <= b (and, with bit I % 32 of `same` required, the key's document
// matches), else -inf: predicated selects, so rows with different bounds in one
// warp do not diverge.
template <int I>
__device__ __forceinline__ float keep_if_in(float v, int a, int b) {
  float r;
  asm("{\n\t.reg .pred p;\n\t"
      "setp.le.s32 p, %2, %3;\n\t"
      "setp.ge.and.s32 p, %4, %3, p;\n\t"
      "selp.f32 %0, %1, 0fFF800000, p;\n\t}"
      : "=f"(r) : "f"(v), "r"(a), "n"(I), "r"(b));
  return r;
}
template <int I>
__device__ __forceinline__ float keep_if_in_doc(float v, int a, int b, uint32_t same) {
  float r;
  asm("{\n\t.reg .pred p;\n\t.reg .b32 t;\n\t"
      "setp.le.s32 p, %2, %3;\n\t"
      "setp.ge.and.s32 p, %4, %3, p;\n\t"
      "and.b32 t, %5, %6;\n\t"
      "setp.ne.and.u32 p, t, 0, p;\n\t"
      "selp.f32 %0, %1, 0fFF800000, p;\n\t}"
      : "=f"(r) : "f"(v), "r"(a), "n"(I), "r"(b), "r"(same), "n"(1u << (I & 31)));
  return r;
}

// Columns I .. I|31 (one 32-column word) with a per-column document / bitmap bit.
template <int I>
struct MaskCols {
  static __device__ __forceinline__ void doc(float (&x)[64], int a, int b, uint32_t same) {
    x[I] = keep_if_in_doc<I>(x[I], a, b, same);
    if constexpr (I % 32 != 31) MaskCols<I + 1>::doc(x, a, b, same);
  }
};

// Columns I .. E-1 against the interval [a, b].
template <int I, int E>
struct RangeCols {
  static __device__ __forceinline__ void apply(float (&x)[64], int a, int b) {
    x[I] = keep_if_in<I>(x[I], a, b);
    if constexpr (I + 1 < E) RangeCols<I + 1, E>::apply(x, a, b);
  }
};

// Interval rule on the 32 columns C0 .. C0+31, decided once for the warp where it
// can be: every row of the warp keeps them (amax <= C0 and bmin >= C0 + 31), or
// every row drops them (bmax < C0 or amin > C0 + 31); otherwise each row tests its
// columns.  The bounds are the warp's extremes of a and b (warp-uniform branches).
template <int C0>
__device__ __forceinline__ void range_chunk(float (&x)[64], int a, int b, int amin, int amax,
                                            int bmin, int bmax) {
  if (!(amax <= C0 && bmin >= C0 + 31)) RangeCols<C0, C0 + 32>::apply(x, a, b);
}

// Tabulated rule: the row's four mask words of a PARTIAL block, keys kv0 .. kv0+127
// (bit i of w[c]: key kv0 + 32c + i), loaded before the block's S is waited for,
// so that the load's latency overlaps that wait (kv0 is a multiple of 128; the
// words are read in 8-byte pairs, the alignment the bitmap is checked for).
template <int MK>
__device__ __forceinline__ void mask_fetch(const uint32_t* brow, int kv0, uint32_t (&w)[4]) {
  if constexpr (MK == kMaskBitmap) {
    const int2 w01 = ldg_nc_v2(reinterpret_cast<const int32_t*>(brow + (kv0 >> 5)));
    const int2 w23 = ldg_nc_v2(reinterpret_cast<const int32_t*>(brow + (kv0 >> 5) + 2));
    w[0] = static_cast<uint32_t>(w01.x);
    w[1] = static_cast<uint32_t>(w01.y);
    w[2] = static_cast<uint32_t>(w23.x);
    w[3] = static_cast<uint32_t>(w23.y);
  } else {
#pragma unroll
    for (int c = 0; c < 4; ++c) w[c] = 0u;
  }
}

// Mask rule on 64 columns of a PARTIAL block: column i (key kv0 + i) is live iff
// a <= i <= b (causal / window interval, clipped to the keys that exist) and, for
// documents, doc_id[kv0 + i] == dq; for a tabulated mask, iff its bit in the words
// w0 (columns 0-31) and w1 (32-63) from mask_fetch is set.  Dead entries become
// -inf.  `ext` = (min a, max a, min b, max b) over the warp's 32 rows (interval
// rule).
template <int MK>
__device__ __forceinline__ void apply_mask(const Params& p, float (&x)[64], int a, int b, int4 ext,
                                           int kv0, int dq, const int32_t* docs, uint32_t w0,
                                           uint32_t w1) {
  if constexpr (MK == kMaskBitmap) {
    MaskCols<0>::doc(x, a, b, w0);
    MaskCols<32>::doc(x, a, b, w1);
  } else if constexpr (MK == kMaskDoc) {
    // bit i of `same[c]`: the document of key kv0 + c*32 + i equals the row's; keys
    // past S read the last id (in bounds) and are excluded by the range anyway.  Lane
    // i fetches the ids of keys i and 32 + i; then one pass per distinct document
    // among the warp's rows (one pass unless a document starts inside the warp's 32
    // rows): the ballot of "key's id == that document" gives its rows their bits.
    // The loop condition is warp-uniform, so every ballot is taken by all lanes.
    const int lane = threadIdx.x & 31;
    const int kid0 = ldg_nc(docs + min(kv0 + lane, p.S - 1));
    const int kid1 = ldg_nc(docs + min(kv0 + 32 + lane, p.S - 1));
    uint32_t same[2] = {0u, 0u};
    uint32_t todo = 0xffffffffu;  // lanes whose document has no pass yet
    while (todo != 0u) {
      const int v = __shfl_sync(0xffffffffu, dq, __ffs(todo) - 1);
      const uint32_t b0 = __ballot_sync(0xffffffffu, kid0 == v);
      const uint32_t b1 = __ballot_sync(0xffffffffu, kid1 == v);
      const bool mine = dq == v;
      if (mine) {
        same[0] = b0;
        same[1] = b1;
      }
      todo &= ~__ballot_sync(0xffffffffu, mine);
    }
    MaskCols<0>::doc(x, a, b, same[0]);
    MaskCols<32>::doc(x, a, b, same[1]);
  } else {
    range_chunk<0>(x, a, b, ext.x, ext.y, ext.z, ext.w);
    range_chunk<32>(x, a, b, ext.x, ext.y, ext.z, ext.w);
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

// x = log2(e) * c * tanh(s * scale / c), the softcap in log2 units.
__device__ __forceinline__ void softcap64(const Params& p, float (&x)[64]) {
#pragma unroll
  for (int i = 0; i < 64; i += 2) {
    const float2 e = make_float2(ex2_approx(x[i] * p.cap_k), ex2_approx(x[i + 1] * p.cap_k));
    const float2 r = make_float2(rcp_approx(e.x + 1.f), rcp_approx(e.y + 1.f));
    const float2 v = fma2(r, make_float2(-2.f * p.cap_a, -2.f * p.cap_a), make_float2(p.cap_a, p.cap_a));
    x[i] = v.x;
    x[i + 1] = v.y;
  }
}

// O *= alpha on this thread's row (all D columns), in TMEM.
template <int D>
__device__ __forceinline__ void rescale_o_rows(uint32_t t_o, float alpha) {
#pragma unroll 1
  for (int c = 0; c < D / 32; ++c) {
    uint32_t r[32];
    tmem_ld32(t_o + c * 32, r);
    tmem_wait_ld();
    reg_fence32(r);
#pragma unroll
    for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * alpha);
    tmem_st32(t_o + c * 32, r);
  }
}

// p = exp2(x * xs - m) for 64 keys, rounded to 16-bit pairs into ph[32]; returns the
// sum of the fp32 p.
__device__ __forceinline__ float exp_pack64(const float (&x)[64], float xs, float neg_mu, bool bf16,
                                            uint32_t (&ph)[32]) {
  float2 sums[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) sums[i] = make_float2(0.f, 0.f);
  const float2 xs2 = make_float2(xs, xs), nm2 = make_float2(neg_mu, neg_mu);
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const float2 a2 = fma2(make_float2(x[2 * i], x[2 * i + 1]), xs2, nm2);
    const float2 pp = make_float2(ex2_approx(a2.x), ex2_approx(a2.y));
    sums[i & 3] = add2(sums[i & 3], pp);
    ph[i] = pack2(pp.x, pp.y, bf16);
  }
  sums[0] = add2(add2(sums[0], sums[1]), add2(sums[2], sums[3]));
  return sums[0].x + sums[0].y;
}

// Softmax warpgroup of one slot: thread t owns row t of the slot's 128-row tile
// (TMEM lane t), so row max and row sum need no shuffles.
template <int D, int MK, bool BHM, bool SC>
__device__ void softmax_role(Smem<D>& sm, const Params& p, uint32_t tmem, int slot,
                             const CUtensorMap* tmap_o) {
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
  const float xs = SC ? 1.f : p.scale_log2;
  const bool split = p.split_p != 0 && !C::kSepP;
  UnitIter<BHM> it;
  it.init(p, slot);
  int blk = 0, units = 0;
  Unit un;

  while (it.pop(p, un)) {
    const int row = un.qblk * kBlockN + t;
    const bool valid = row < p.L;
    if (un.n == 0) {
      const size_t orow = static_cast<size_t>(un.bh) * p.L + row;
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + orow * D);
      if (valid) {
#pragma unroll
        for (int i = 0; i < D / 8; ++i) dst[i] = make_uint4(0, 0, 0, 0);
        if (p.lse) p.lse[orow] = -INFINITY;
      }
      continue;
    }
    // this unit's mask instance: its document ids / bitmap rows (pointers formed
    // where they are used, like the key range below)
    auto docs_of = [&]() {
      return MK == kMaskDoc ? p.doc_id + static_cast<size_t>(un.inst) * p.doc_len : nullptr;
    };
    const int dq_own = (MK == kMaskDoc && valid) ? __ldg(docs_of() + row) : 0;
    // rows past L (only ever above the valid ones, so lane 0 is valid if any lane is)
    // take lane 0's document: they add no document to the warp's passes in apply_mask.
    // The shuffle is taken by every lane, outside any short-circuited expression.
    const int dq0 = __shfl_sync(0xffffffffu, dq_own, 0);
    const int dq = valid ? dq_own : dq0;
    // tabulated mask: this row's words (rows past L read the last row, unused)
    auto brow_of = [&]() {
      return MK == kMaskBitmap ? p.bitmap + (static_cast<size_t>(un.inst) * p.L +
                                             min(un.qblk * kBlockN + t, p.L - 1)) *
                                                p.bitmap_words
                               : nullptr;
    };
    // live keys of this row: kv in [lo, hi] (and, for documents, doc_id[kv] == dq;
    // for a tabulated mask, its bit); only the causal rules bound hi by the row.
    // Formed where a PARTIAL block needs them, so that no register holds them
    // through the block loop.
    // Both bounds are non-decreasing in the row, so over the warp's 32 rows their
    // extremes are those of its first and last row: `mask_span` forms a block's
    // bounds for this row (a, b) and the warp's extremes without a warp reduction.
    auto key_range = [&](int r, int& lo, int& hi) {
      hi = MK == kMaskBitmap ? p.S - 1 : min(r, p.S - 1);
      lo = p.mask_kind == FA_MASK_SLIDING_WINDOW_CAUSAL ? max(r - p.window + 1, 0) : 0;
    };
    auto mask_span = [&](int kv0, int& a, int& b, int4& ext) {
      const int r = un.qblk * kBlockN + t;
      int lo, hi;
      key_range(r, lo, hi);
      a = lo - kv0;
      b = hi - kv0;
      ext = make_int4(0, 0, 0, 0);
      if constexpr (MK == kMaskRange) {
        const int rw = r - (t & 31);
        int lo0, hi0, lo1, hi1;
        key_range(rw, lo0, hi0);
        key_range(rw + 31, lo1, hi1);
        ext = make_int4(lo0 - kv0, lo1 - kv0, hi0 - kv0, hi1 - kv0);
      }
    };
    float m = -INFINITY, l = 0.f;  // running max (log2 units) and running sum
    int kvb = block_index(p, un, 0);

    for (int j = 0; j < un.n; ++j) {
      const bool full = j >= un.np;
      const int kvb_next = j + 1 < un.n ? block_index(p, un, j + 1) : 0;
      // a PARTIAL block's tabulated-mask words, loaded before S is waited for
      uint32_t mw[4] = {0u, 0u, 0u, 0u};
      if (!full) mask_fetch<MK>(brow_of(), kvb * kBlockN, mw);
      if (!wait_warp(sm, &sm.s_full[slot], blk & 1, p)) return;
      tc_fence_after();
      if constexpr (C::kStageO) {
        // The previous unit's TMA store has had a block's wait to read its staging
        // tile (that unit's Q buffer): once it has, the tile goes back to the
        // producer.
        if (j == 0 && units > 0 && (t & 31) == 0) {
          bulk_wait_read_all();
          mbar_arrive(&sm.q_empty[slot][(units - 1) % C::kQBuf]);
        }
      }
      if constexpr (C::kSepP) {
        // Separate-P layout: the whole row of S (128 columns) comes into registers at
        // once, S is released to the MMA warp right away, and P is written per half.
        float x[128];
        load_s_half(t_s, *reinterpret_cast<float(*)[64]>(x));
        load_s_half(t_s + 64, *reinterpret_cast<float(*)[64]>(x + 64));
        tc_fence_before();
        __syncwarp();
        if ((t & 31) == 0) mbar_arrive(&sm.s_empty[slot]);
        if constexpr (SC) softcap64(p, *reinterpret_cast<float(*)[64]>(x)), softcap64(p, *reinterpret_cast<float(*)[64]>(x + 64));
        if (!full) {
          int a, b;
          int4 e;
          mask_span(kvb * kBlockN, a, b, e);
          apply_mask<MK>(p, *reinterpret_cast<float(*)[64]>(x), a, b, e, kvb * kBlockN, dq, docs_of(),
                         mw[0], mw[1]);
          apply_mask<MK>(p, *reinterpret_cast<float(*)[64]>(x + 64), a - 64, b - 64,
                         make_int4(e.x - 64, e.y - 64, e.z - 64, e.w - 64), kvb * kBlockN + 64, dq,
                         docs_of(), mw[2], mw[3]);
        }
        const float mb = fmaxf(row_max64(*reinterpret_cast<float(*)[64]>(x)),
                               row_max64(*reinterpret_cast<float(*)[64]>(x + 64))) * xs;
        const float m_new = fmaxf(m, mb);
        float alpha = 1.f;
        bool rescale_o = false;
        if (m_new > m + p.rescale_thr) {
          if (m != -INFINITY) {
            alpha = ex2_approx(m - m_new);
            l *= alpha;
            rescale_o = true;
          }
          m = m_new;
        }
        const float neg_mu = (m == -INFINITY) ? 0.f : -m;
        uint32_t ph[32];
        l += exp_pack64(*reinterpret_cast<float(*)[64]>(x), xs, neg_mu, bf16, ph);
        // The previous PV of this slot must be done before P is overwritten or O
        // rescaled; waiting here, after the first half's exponentials, hides it.
        if (blk > 0 && !wait_warp(sm, &sm.pv_done[slot], (blk - 1) & 1, p)) return;
        tc_fence_after();
        if (__any_sync(0xffffffffu, rescale_o)) rescale_o_rows<D>(t_o, alpha);
        tmem_st32(t_p, ph);
        l += exp_pack64(*reinterpret_cast<float(*)[64]>(x + 64), xs, neg_mu, bf16, ph);
        tmem_st32(t_p + 32, ph);
      } else {
      // Pass 1: the block's row max from the raw scores (a PARTIAL block's masked
        // entries excluded).  The softcap is monotone, so the max of the capped scores
        // is the cap of the raw max.  Pass 2 then turns each half of 64 keys into P with
        // that one max: P_hi of half h goes to P columns [32h, 32h + 32); with the
        // split, P_lo goes to columns 64 + [32h, 32h + 32), held in registers until
        // half 1 has been read (in the aliased layout those columns are still S).
        int a, b;  // live columns of the block: a <= i <= b
        int4 e;
        mask_span(kvb * kBlockN, a, b, e);
        float rmax = -INFINITY;
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          float x[64];
          load_s_half(t_s + h * 64, x);
          if (!full)
            apply_mask<MK>(p, x, a - h * 64, b - h * 64,
                           make_int4(e.x - h * 64, e.y - h * 64, e.z - h * 64, e.w - h * 64),
                           kvb * kBlockN + h * 64, dq, docs_of(), h ? mw[2] : mw[0],
                           h ? mw[3] : mw[1]);
          rmax = fmaxf(rmax, row_max64(x));
        }
        float mb = rmax;
        if (rmax != -INFINITY) {
          if constexpr (SC) {
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
        if (m_new > m + p.rescale_thr) {
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
            reg_fence32(r);
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
          if constexpr (SC) {  // x = log2(e) * c * tanh(s * scale / c)
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
          if (!full)
            apply_mask<MK>(p, x, a - h * 64, b - h * 64,
                           make_int4(e.x - h * 64, e.y - h * 64, e.z - h * 64, e.w - h * 64),
                           kvb * kBlockN + h * 64, dq, docs_of(), h ? mw[2] : mw[0],
                           h ? mw[3] : mw[1]);
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
      }
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if ((t & 31) == 0) mbar_arrive(&sm.p_full[slot]);
      ++blk;
      kvb = kvb_next;
    }

    // epilogue: O / l -> out, LSE (the output row is formed here, not kept in
    // registers through the block loop)
    if (!wait_warp(sm, &sm.o_full[slot], units & 1, p)) return;
    tc_fence_after();
    const size_t orow = static_cast<size_t>(un.bh) * p.L + un.qblk * kBlockN + t;
    const float inv = l > 0.f ? 1.f / l : 0.f;
    if (C::kStageO && un.n <= stage_max_blocks<MK>()) {
      // O comes into registers and is released to the next unit's PV at once; the
      // warp writes its 32 rows into the staging tile (128-byte rows, 16-byte chunk
      // c of row r at chunk c ^ (r % 8): the layout of the map's 128-byte swizzle,
      // and conflict-free for one row per thread) and lane 0 stores them with TMA.
      // Rows past L are clipped by the map's extent.
      uint32_t pk[32];  // the row as 16-bit pairs
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t r[32];
        tmem_ld32(t_o + c * 32, r);
        tmem_wait_ld();
        reg_fence32(r);
#pragma unroll
        for (int i = 0; i < 16; ++i)
          pk[16 * c + i] = pack2(__uint_as_float(r[2 * i]) * inv, __uint_as_float(r[2 * i + 1]) * inv, bf16);
      }
      tc_fence_before();
      __syncwarp();
      // The lane index is read here (a volatile read), so that the staging
      // addresses below are formed here and not kept in registers across the
      // block loop, where every register is taken.
      const int lane = lane_id_volatile();
      if (lane == 0) mbar_arrive(&sm.o_empty[slot]);
      // the unit's Q tile: its MMAs are done (o_full), and the producer refills it
      // only after this warp releases it, in the next unit's first block
      const int qb = units % C::kQBuf;
      uint8_t* rowp = sm.q[slot][qb] + (wq * 32 + lane) * 128;
      uint8_t* tile = rowp - lane * 128;
#pragma unroll
      for (int c = 0; c < 8; ++c)
        *reinterpret_cast<uint4*>(rowp + ((c ^ (lane & 7)) << 4)) =
            make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
      fence_proxy_async_shared();
      __syncwarp();
      const int row0 = un.qblk * kBlockN + wq * 32;
      if (lane == 0 && row0 < p.L) {
        tma_store_3d(tmap_o, tile, 0, row0, un.bh);
        bulk_commit_group();
      }
    } else {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + orow * D);
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(t_o + c * 32, r);
        tmem_wait_ld();
        reg_fence32(r);
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
    }
    if (valid && p.lse) p.lse[orow] = l > 0.f ? (m + log2f(l)) * kLn2 : -INFINITY;
    ++units;
  }
}

template <int D, int MK, bool BHM, bool SC>
__global__ void __launch_bounds__(kThreads, 1)
fwd_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
           const __grid_constant__ CUtensorMap tmap_v, const __grid_constant__ CUtensorMap tmap_o,
           const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  Smem<D>& sm = *reinterpret_cast<Smem<D>*>(smem_raw + ((1024u - (base & 1023u)) & 1023u));
  const int warp = threadIdx.x >> 5;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kNumSlots; ++s) {
      for (int b = 0; b < Cfg<D>::kQBuf; ++b) {
        mbar_init(&sm.q_full[s][b], 1);
        // the MMA warp's commit, and with O staged in it, one arrival per softmax warp
        mbar_init(&sm.q_empty[s][b], Cfg<D>::kStageO ? 1 + 4 : 1);
      }
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.s_empty[s], 4);
      mbar_init(&sm.pv_done[s], 1);
      mbar_init(&sm.p_full[s], 4);   // one arrival per softmax warp
      mbar_init(&sm.o_full[s], 1);
      mbar_init(&sm.o_empty[s], 4);
      for (int i = 0; i < Cfg<D>::kKRing; ++i) {
        mbar_init(&sm.k_full[s][i], 1);
        mbar_init(&sm.k_empty[s][i], 1);
      }
      for (int i = 0; i < Cfg<D>::kVRing; ++i) {
        mbar_init(&sm.v_full[s][i], 1);
        mbar_init(&sm.v_empty[s][i], 1);
      }
    }
    mbar_init(&sm.drain, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kProducerWarp && (threadIdx.x & 31) == 0) {
    prefetch_tensormap(&tmap_q);  // the other producer warp shares the cached maps
    prefetch_tensormap(&tmap_k);
    prefetch_tensormap(&tmap_v);
    if (Cfg<D>::kStageO) prefetch_tensormap(&tmap_o);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&sm.tmem_base, Cfg<D>::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  // Launched as a programmatic dependent: everything above overlaps the end of the
  // previous kernel on the stream (typically the block-mask build); nothing in
  // global memory is read before this wait.
  grid_dep_wait();

  // Role dispatch; the final rendezvous is a named barrier over all threads.
  if (warp < kSoftmaxWarps) {
    softmax_role<D, MK, BHM, SC>(sm, p, tmem, warp / 4, &tmap_o);
    // the warp's TMA stores of O (issued by lane 0) complete before the CTA exits
    if (Cfg<D>::kStageO && (threadIdx.x & 31) == 0) bulk_wait_all();
    tc_fence_before();
    named_barrier_sync(1, kThreads);
    return;
  }
  if (warp == kProducerWarp || warp == kProducerWarp + 1) {
    // one copy of the producer code for both slots (the slot is a runtime value)
    producer_role<D, BHM>(warp - kProducerWarp, sm, p, &tmap_q, &tmap_k, &tmap_v);
  } else if (warp == kMmaWarp) {
    mma_role<D, BHM>(sm, p, tmem);
  }
  tc_fence_before();
  named_barrier_sync(1, kThreads);
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, Cfg<D>::kTmemCols);
  }
}

// ---------------------------------------------------------------- host side
// The forward's Q, K, V (and out) maps: 128-row boxes, one per 64 columns.
bool make_map(CUtensorMap* map, const void* ptr, bool bf16, int D, int rows, int bh) {
  return make_tile_map(map, ptr, bf16, D, rows, bh, kBlockN);
}

template <int D, int MK, bool BHM, bool SC>
fa_status launch(const void* q, const void* k, const void* v, bool bf16, int BH, int L, int S,
                 const Params& prm, cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  if (!make_map(&tq, q, bf16, D, L, BH)) return FA_ERR_CUDA;
  // With S == 0 no K/V tile is ever loaded; the maps only need to be well formed.
  const int BHkv = BH / prm.kv_group;
  if (!make_map(&tk, S > 0 ? k : q, bf16, D, S > 0 ? S : L, S > 0 ? BHkv : BH)) return FA_ERR_CUDA;
  if (!make_map(&tv, S > 0 ? v : q, bf16, D, S > 0 ? S : L, S > 0 ? BHkv : BH)) return FA_ERR_CUDA;
  // out, stored by the softmax warps 32 rows at a time (D = 64)
  CUtensorMap to;
  if (!make_tile_map(&to, prm.out, bf16, D, L, BH, 32)) return FA_ERR_CUDA;
  const size_t smem = sizeof(Smem<D>) + 1024;
  int dev = 0;
  FA_CUDA_CHECK(cudaGetDevice(&dev));
  {
    static std::mutex mu;
    static bool done[kMaxDevices] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
    if (!done[dev]) {
      FA_CUDA_CHECK(cudaFuncSetAttribute(fwd_kernel<D, MK, BHM, SC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem)));
      done[dev] = true;
    }
  }
  const int sms = num_sms_current_device();
  if (sms <= 0) return FA_ERR_CUDA;
  const int want = (prm.num_units + kNumSlots - 1) / kNumSlots;
  const int grid = want < sms ? want : sms;
  FA_CUDA_CHECK(launch_pdl(fwd_kernel<D, MK, BHM, SC>, dim3(grid), dim3(kThreads), smem, stream, tq, tk,
                           tv, to, prm));
  return FA_OK;
}

}  // namespace
}  // namespace fa

extern "C" size_t fa_fwd_workspace_bytes(void) { return 256; }

namespace fa {
namespace {

// The instantiation for a head dim, mask family, (broadcast or per-instance) mask and
// score_mod: each kernel holds only the code it runs, which keeps it small enough
// for the instruction caches.
template <bool BHM, bool SC>
fa_status launch_family(int kind, int D, const void* q, const void* k, const void* v, bool b16,
                        int L, int S, const Params& prm, cudaStream_t s) {
  switch (mask_family(kind) * 2 + (D == 64 ? 0 : 1)) {
    case kMaskRange * 2: return launch<64, kMaskRange, BHM, SC>(q, k, v, b16, prm.BH, L, S, prm, s);
    case kMaskRange * 2 + 1: return launch<128, kMaskRange, BHM, SC>(q, k, v, b16, prm.BH, L, S, prm, s);
    case kMaskDoc * 2: return launch<64, kMaskDoc, BHM, SC>(q, k, v, b16, prm.BH, L, S, prm, s);
    case kMaskDoc * 2 + 1: return launch<128, kMaskDoc, BHM, SC>(q, k, v, b16, prm.BH, L, S, prm, s);
    case kMaskBitmap * 2: return launch<64, kMaskBitmap, BHM, SC>(q, k, v, b16, prm.BH, L, S, prm, s);
    default: return launch<128, kMaskBitmap, BHM, SC>(q, k, v, b16, prm.BH, L, S, prm, s);
  }
}

fa_status fwd_impl(const void* q, const void* k, const void* v, int32_t dtype, int32_t B, int32_t H,
                   int32_t Hkv, int32_t L, int32_t S, int32_t D, const fa_block_mask* bm,
                   int32_t score_kind, float softcap, float scale, void* out, float* lse,
                   void* workspace, void* stream) {
  if (bm == nullptr || workspace == nullptr) return FA_ERR_INVALID_ARG;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_INVALID_ARG;
  if (B < 0 || H < 0 || L < 0 || S < 0) return FA_ERR_INVALID_ARG;
  if (Hkv < 1 || (H > 0 && H % Hkv != 0) || (H == 0 && Hkv != 1)) return FA_ERR_INVALID_ARG;
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
  // Alignment of everything the kernel reads or writes, checked here so that a
  // misaligned pointer is an argument error and never a device fault: Q, K, V, out
  // (TMA tiles, 16-byte stores) 16 bytes; the schedule table (8-byte loads) and a
  // tabulated mask (8-byte loads of word pairs) 8 bytes; block lists, document ids,
  // LSE and the error word 4 bytes.
  auto misaligned = [](const void* ptr, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) != 0;
  };
  if (misaligned(q, 16) || misaligned(out, 16) || (S > 0 && (misaligned(k, 16) || misaligned(v, 16))))
    return FA_ERR_INVALID_ARG;
  if (misaligned(lse, 4) || misaligned(workspace, 4)) return FA_ERR_INVALID_ARG;
  if (bm->kv_num_blocks == nullptr || bm->full_kv_num_blocks == nullptr || bm->q_order == nullptr ||
      (bm->n_kv_blocks > 0 && (bm->kv_indices == nullptr || bm->full_kv_indices == nullptr)))
    return FA_ERR_INVALID_ARG;
  if (misaligned(bm->q_order, 8) || misaligned(bm->kv_indices, 4) ||
      misaligned(bm->full_kv_indices, 4))
    return FA_ERR_INVALID_ARG;
  if (bm->kind == FA_MASK_DOCUMENT_CAUSAL && (bm->doc_id == nullptr || misaligned(bm->doc_id, 4)))
    return FA_ERR_INVALID_ARG;
  if (bm->kind == FA_MASK_BITMAP && S > 0 && (bm->bitmap == nullptr || misaligned(bm->bitmap, 8)))
    return FA_ERR_INVALID_ARG;
  // per-(batch, head) masks: one instance per batch element and / or head (0 reads as 1)
  const int mb = bm->mask_batch > 1 ? bm->mask_batch : 1;
  const int mh = bm->mask_heads > 1 ? bm->mask_heads : 1;
  if ((mb != 1 && mb != B) || (mh != 1 && mh != H)) return FA_ERR_INVALID_ARG;

  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(D));
  Params prm{};
  prm.kv_idx = bm->kv_indices;
  prm.full_idx = bm->full_kv_indices;
  prm.sched = bm->q_order;
  prm.doc_id = bm->doc_id;
  prm.bitmap = bm->bitmap;
  prm.bitmap_words = 4 * bm->n_kv_blocks;
  prm.n_q = bm->n_q_blocks;
  prm.mask_b = mb > 1 ? 1 : 0;
  prm.mask_h = mh > 1 ? 1 : 0;
  prm.mask_heads = mh;
  prm.doc_len = L > S ? L : S;
  prm.out = out;
  prm.lse = lse;
  prm.err = static_cast<int32_t*>(workspace);
  prm.BH = static_cast<int>(BH64);
  prm.H = H;
  prm.Hkv = Hkv;
  prm.kv_group = H > 0 ? H / Hkv : 1;
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
  // bf16 P carries 8 significant bits; in a peaked row the largest weights set the
  // error.  D = 64: P always uses the exact running max (threshold 0), so each
  // row's largest weight is exactly 1.  D = 128 (P overwrites S, O rescales are
  // kept rare): P is fed as hi + lo, ~16 bits.  fp16 P (11 significant bits) is fed
  // as one term, with the deferred rescale.
  prm.split_p = (dtype == FA_BF16 && D == 128) ? 1 : 0;
  prm.rescale_thr = (dtype == FA_BF16 && D == 64) ? 0.f : 8.f;
  prm.timeout_ns = 2000000000ull;
  if (debug_stall(&prm.timeout_ns)) prm.stall_mma = 1;
  const cudaStream_t s = as_stream(stream);
  const bool b16 = dtype == FA_BF16;
  const bool bhm = (prm.mask_b | prm.mask_h) != 0;
  if (prm.softcap_on) {
    return bhm ? launch_family<true, true>(bm->kind, D, q, k, v, b16, L, S, prm, s)
               : launch_family<false, true>(bm->kind, D, q, k, v, b16, L, S, prm, s);
  }
  return bhm ? launch_family<true, false>(bm->kind, D, q, k, v, b16, L, S, prm, s)
             : launch_family<false, false>(bm->kind, D, q, k, v, b16, L, S, prm, s);
}

}  // namespace
}  // namespace fa

extern "C" fa_status fa_flex_attention_fwd(const void* q, const void* k, const void* v,
                                           int32_t dtype, int32_t B, int32_t H, int32_t L,
                                           int32_t S, int32_t D, const fa_block_mask* bm,
                                           int32_t score_kind, float softcap, float scale,
                                           void* out, float* lse, void* workspace,
                                           void* stream) {
  return fa::fwd_impl(q, k, v, dtype, B, H, H > 0 ? H : 1, L, S, D, bm, score_kind, softcap, scale,
                      out, lse, workspace, stream);
}

extern "C" fa_status fa_flex_attention_fwd_gqa(const void* q, const void* k, const void* v,
                                               int32_t dtype, int32_t B, int32_t H, int32_t H_kv,
                                               int32_t L, int32_t S, int32_t D,
                                               const fa_block_mask* bm, int32_t score_kind,
                                               float softcap, float scale, void* out, float* lse,
                                               void* workspace, void* stream) {
  return fa::fwd_impl(q, k, v, dtype, B, H, H_kv, L, S, D, bm, score_kind, softcap, scale, out,
                      lse, workspace, stream);
}
