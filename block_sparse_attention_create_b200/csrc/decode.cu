// Decode against a KV cache (SDPA tutorial, section 4, pitfall 3): L new queries
// after S - L cached keys, the causal mask aligned to the lower right (query i sits
// at key position S - L + i), optionally within a window of W keys, or no mask.
// L is small (a token or a short chunk), S long, so the work is reading K and V
// once: the path is bound by HBM.
//
// Split-KV: CTA (split, b * Hkv + kvh) takes every query row that reads K/V head
// kvh -- the H / Hkv query heads of the group times the L queries, R <= 32 rows --
// against one contiguous chunk of keys, streamed through shared memory in 64-key
// tiles by TMA (128-byte swizzle, a ring of stages, bounded mbarrier waits).  It
// leaves the chunk's running max, sum and unnormalised output per row in the
// workspace; a second kernel merges the chunks of each row (rescaling each by
// 2^(m_chunk - m)) into out and LSE.  Chunks no row can see (sliding window) load
// nothing.  Two kernels do the chunk: for R <= 8 rows (grouped-query decode of one
// or a few tokens) `decode_mma_kernel`, whose warps keep private softmax states and
// run both products on warp-level tensor-core tiles, so the instruction stream stays
// well below the HBM time; for more rows `decode_split_kernel` on the CUDA cores.
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

constexpr int kTile = 64;            // keys per K/V tile
constexpr int kMaxRows = FA_DECODE_MAX_ROWS;
// CTAs per SM of the chunk kernel for R rows: the tensor-core kernel runs three
// (two at D = 128 for R > 8, twice the accumulators); the CUDA-core kernel
// (R <= 32) runs 8 warps, two CTAs per SM, at D = 128 and 4 warps, three per SM, at
// D = 64.  The grid is sized for that many CTAs.
__host__ __device__ constexpr int split_ctas_per_sm(int D) { return D == 128 ? 2 : 3; }
__host__ __device__ constexpr int dec_ctas_per_sm(int D, int rows) {
  return rows <= 8 ? 3 : (rows <= 16 ? (D == 128 ? 2 : 3) : split_ctas_per_sm(D));
}
template <int D>
struct DecCfg {
  static constexpr int kThreads = D == 128 ? 256 : 128;
};
constexpr int kBoxBytes = kTile * 128;  // one TMA box: 64 keys x 64 elements
// K/V tiles in flight per CTA: a ring of stages(D, RM) tiles, plus L2 prefetches
// of the tiles kPrefetch further on, so that enough bytes are on their way to cover
// the DRAM latency (one 32 KB tile per CTA was not).  Three stages, except at D =
// 128 with 32 rows, where two keep two CTAs per SM in shared memory.
__host__ __device__ constexpr int dec_stages(int D, int RM) { return D == 128 && RM == 32 ? 2 : 3; }
constexpr int kPrefetch = 4;
constexpr int kDecWorkspaceHeader = 256;  // word 0: device error flags
constexpr float kDecLog2e = 1.4426950408889634f;
constexpr float kDecLn2 = 0.6931471805599453f;

struct DecParams {
  const uint16_t* q;  // (B, H, L, D)
  void* out;          // (B, H, L, D)
  float* lse;         // (B, H, L) or null
  float* part;        // per (b, h, i, split): m, l, O[D]
  int32_t* err;
  int H, Hkv, G, L, S, nsplit, chunk, mask, window, softcap_on, is_bf16;
  float q_scale;  // folded into Q: scale * log2(e), or scale alone under the softcap
  float cap_c;    // softcap c
  float cap_a;    // c * log2(e)
  unsigned long long timeout_ns;
  int stall_loads;  // testing hook: no K/V tile is loaded (see fa_debug_set_mma_stall)
};

template <int D, int RM>
struct __align__(1024) DecSmem {
  static constexpr int kStages = dec_stages(D, RM);
  uint8_t k[kStages][D / 64][kBoxBytes];
  uint8_t v[kStages][D / 64][kBoxBytes];
  float qs[RM][D];
  float sc[RM][kTile];
  float m[RM], l[RM], alpha[RM];
  uint64_t full[dec_stages(D, RM)];
  volatile int abort_flag;
};

__device__ __forceinline__ float load16(const uint16_t* ptr, bool bf16) {
  const uint16_t u = __ldg(ptr);
  return bf16 ? __uint_as_float(static_cast<uint32_t>(u) << 16)
              : __half2float(__ushort_as_half(u));
}

// 8 consecutive 16-bit values -> fp32.
__device__ __forceinline__ void unpack8(const uint4 raw, bool bf16, float (&f)[8]) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    if (bf16) {
      f[2 * i] = __uint_as_float(w[i] << 16);
      f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    } else {
      const float2 h = __half22float2(*reinterpret_cast<const __half2*>(&w[i]));
      f[2 * i] = h.x;
      f[2 * i + 1] = h.y;
    }
  }
}

// 16-byte chunk c (elements 8c .. 8c+7) of key row j of a tile: box c / 8, swizzled
// position (c % 8) ^ (j % 8) inside the row's 128 bytes.
template <int NB>
__device__ __forceinline__ uint4 tile_chunk(const uint8_t (&tile)[NB][kBoxBytes], int j, int c) {
  return *reinterpret_cast<const uint4*>(&tile[c >> 3][j * 128 + (((c & 7) ^ (j & 7)) << 4)]);
}

template <class Sm>
__device__ __forceinline__ bool dec_wait(Sm& sm, uint64_t* bar, uint32_t parity,
                                         const DecParams& p) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
#pragma unroll 1  // inlined at every wait site: keep the code small
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

// RM: bound on the rows R (the path launches it with RM = 32 for R > 8; at most 8
// rows take decode_mma_kernel).  With RM <= 8 every PV thread keeps all rows
// for one 16-byte column chunk over a subset of the tile's keys (key group), and
// the key groups are summed once per CTA at the end; with RM = 32 a thread keeps
// a few rows over all keys.
template <int D, int RM>
__global__ void __launch_bounds__(DecCfg<D>::kThreads, split_ctas_per_sm(D))
decode_split_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                    const __grid_constant__ DecParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  using Sm = DecSmem<D, RM>;
  constexpr int kStages = Sm::kStages;
  Sm& sm = *reinterpret_cast<Sm*>(smem_raw + ((1024u - (base & 1023u)) & 1023u));
  constexpr int kThr = DecCfg<D>::kThreads;
  constexpr int kWarps = kThr / 32;
  constexpr int kRowGroups = kThr / kTile;        // score threads per key
  constexpr int kChunks = D / 8;                  // 16-byte chunks of a row
  constexpr int kGroups = kThr / kChunks;         // PV thread groups (rows or keys)
  constexpr bool kKeyGroups = RM <= 8;
  constexpr int kRowsPer = kKeyGroups ? RM : RM / kGroups;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, bkv = blockIdx.y;
  const int b = bkv / p.Hkv, kvh = bkv - b * p.Hkv;
  const int R = p.G * p.L;
  const bool bf16 = p.is_bf16 != 0;

  // keys of this chunk that some row can see: the window's lower edge for row 0
  int k_start = split * p.chunk;
  const int c1 = min(p.S, k_start + p.chunk);
  if (p.mask == FA_DECODE_SLIDING_WINDOW) k_start = max(k_start, p.S - p.L - p.window + 1);
  const int ntiles = k_start < c1 ? (c1 - k_start + kTile - 1) / kTile : 0;

  if (tid == 0) {
    for (int b = 0; b < kStages; ++b) mbar_init(&sm.full[b], 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  // query rows r = g * L + i (query head kvh * G + g, query i), scaled
  for (int e = tid; e < R * D; e += kThr) {
    const int r = e / D, d = e - (e / D) * D;
    const int g = r / p.L, i = r - g * p.L;
    const size_t qi = (static_cast<size_t>(b * p.H + kvh * p.G + g) * p.L + i) * D + d;
    sm.qs[r][d] = load16(p.q + qi, bf16) * p.q_scale;
  }
  for (int r = tid; r < R; r += kThr) {
    sm.m[r] = -INFINITY;
    sm.l[r] = 0.f;
  }
  __syncthreads();

  const uint64_t pol = policy_evict_first();
  auto issue = [&](int t) {
    const int buf = t % kStages;
    const int k0 = k_start + t * kTile;
    fence_proxy_async_shared();
    mbar_arrive_expect_tx(&sm.full[buf], 2 * (D / 64) * kBoxBytes);
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_load_3d(sm.k[buf][c], &tk, &sm.full[buf], c * 64, k0, bkv, pol);
      tma_load_3d(sm.v[buf][c], &tv, &sm.full[buf], c * 64, k0, bkv, pol);
    }
  };
  auto prefetch = [&](int t) {  // tile t into L2
    const int k0 = k_start + t * kTile;
#pragma unroll
    for (int c = 0; c < D / 64; ++c) {
      tma_prefetch_3d(&tk, c * 64, k0, bkv);
      tma_prefetch_3d(&tv, c * 64, k0, bkv);
    }
  };
  if (tid == 0 && !p.stall_loads) {
    for (int u = 0; u < kStages - 1 && u < ntiles; ++u) issue(u);
    for (int u = kStages - 1; u < kStages - 1 + kPrefetch && u < ntiles; ++u) prefetch(u);
  }

  const int oc = tid % kChunks, og = tid / kChunks;  // PV: 16-byte chunk, row group
  float o[kRowsPer][8];
#pragma unroll
  for (int k = 0; k < kRowsPer; ++k)
#pragma unroll
    for (int e = 0; e < 8; ++e) o[k][e] = 0.f;

  int t = 0;
  for (; t < ntiles; ++t) {
    const int buf = t % kStages;
    const int k0 = k_start + t * kTile;
    // tile t + kStages - 1 goes to the buffer released after tile t - 1
    if (tid == 0 && !p.stall_loads) {
      if (t + kStages - 1 < ntiles) issue(t + kStages - 1);
      if (t + kStages - 1 + kPrefetch < ntiles) prefetch(t + kStages - 1 + kPrefetch);
    }
    const bool ok = dec_wait(sm, &sm.full[buf], (t / kStages) & 1, p);
    if (!__syncthreads_and(ok)) break;

    {
      // scores: thread = (key j, row group rg); rows r = rg, rg + kRowGroups, ...
      constexpr int kRowsS = RM / kRowGroups > 0 ? RM / kRowGroups : 1;
      const int j = tid & (kTile - 1), rg = tid / kTile;
      // two independent packed partial sums per row keep the FMA chains short
      float2 acc[kRowsS][2];
#pragma unroll
      for (int k = 0; k < kRowsS; ++k) acc[k][0] = acc[k][1] = make_float2(0.f, 0.f);
#pragma unroll
      for (int c = 0; c < kChunks; ++c) {
        float kf[8];
        unpack8(tile_chunk(sm.k[buf], j, c), bf16, kf);
#pragma unroll
        for (int k = 0; k < kRowsS; ++k) {
          const int r = rg + kRowGroups * k;
          if (r < R) {
            const float4 qa = *reinterpret_cast<const float4*>(&sm.qs[r][c * 8]);
            const float4 qb = *reinterpret_cast<const float4*>(&sm.qs[r][c * 8 + 4]);
            acc[k][0] = fma2(make_float2(qa.x, qa.y), make_float2(kf[0], kf[1]), acc[k][0]);
            acc[k][1] = fma2(make_float2(qa.z, qa.w), make_float2(kf[2], kf[3]), acc[k][1]);
            acc[k][0] = fma2(make_float2(qb.x, qb.y), make_float2(kf[4], kf[5]), acc[k][0]);
            acc[k][1] = fma2(make_float2(qb.z, qb.w), make_float2(kf[6], kf[7]), acc[k][1]);
          }
        }
      }
      const int kv = k0 + j;
#pragma unroll
      for (int k = 0; k < kRowsS; ++k) {
        const int r = rg + kRowGroups * k;
        if (r < R) {
          const int pos = p.S - p.L + (r % p.L);  // the query's key position
          bool keep = kv < c1;
          if (p.mask != FA_DECODE_FULL) keep = keep && kv <= pos;
          if (p.mask == FA_DECODE_SLIDING_WINDOW) keep = keep && pos - kv < p.window;
          float s = (acc[k][0].x + acc[k][0].y) + (acc[k][1].x + acc[k][1].y);
          if (p.softcap_on) s = p.cap_a * tanhf(s / p.cap_c);
          sm.sc[r][j] = keep ? s : -INFINITY;
        }
      }
    }
    __syncthreads();

    // online softmax: warp w takes rows w, w + 4, ...; lane holds keys lane, lane + 32
    for (int r = warp; r < R; r += kWarps) {
      const float s0 = sm.sc[r][lane], s1 = sm.sc[r][lane + 32];
      float mx = fmaxf(s0, s1);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      const float m_old = sm.m[r];
      const float m_new = fmaxf(m_old, mx);
      const float mu = m_new == -INFINITY ? 0.f : m_new;  // a row with no key yet: p = 0
      const float p0 = ex2_approx(s0 - mu), p1 = ex2_approx(s1 - mu);
      float sum = p0 + p1;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      sm.sc[r][lane] = p0;
      sm.sc[r][lane + 32] = p1;
      __syncwarp();
      if (lane == 0) {
        const float a = ex2_approx(m_old - mu);  // 0 while the row had no key
        sm.alpha[r] = a;
        sm.l[r] = sm.l[r] * a + sum;
        sm.m[r] = m_new;
      }
    }
    __syncthreads();

    // O += P V: thread = (16-byte chunk oc of a V row, group og: rows or keys)
    if constexpr (kKeyGroups) {
      // rescale only when some row's max moved (alpha is exactly 1 otherwise: ex2(0));
      // the test reads the same shared values in every thread, so it is CTA-uniform
      bool moved = false;
#pragma unroll
      for (int r = 0; r < RM; ++r) moved |= r < R && sm.alpha[r] != 1.f;
      if (moved) {
#pragma unroll
        for (int r = 0; r < RM; ++r) {
          const float a = r < R ? sm.alpha[r] : 0.f;
#pragma unroll
          for (int e = 0; e < 8; ++e) o[r][e] *= a;
        }
      }
      const int nk = min(kTile, c1 - k0);
      for (int j = og; j < nk; j += kGroups) {
        float vf[8];
        unpack8(tile_chunk(sm.v[buf], j, oc), bf16, vf);
#pragma unroll
        for (int r = 0; r < RM; ++r) {
          const float pj = r < R ? sm.sc[r][j] : 0.f;
          const float2 p2 = make_float2(pj, pj);
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const float2 acc2 = fma2(p2, make_float2(vf[e], vf[e + 1]), make_float2(o[r][e], o[r][e + 1]));
            o[r][e] = acc2.x;
            o[r][e + 1] = acc2.y;
          }
        }
      }
    } else {
      float al[kRowsPer];
#pragma unroll
      for (int k = 0; k < kRowsPer; ++k) {
        const int r = og + kGroups * k;
        al[k] = r < R ? sm.alpha[r] : 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) o[k][e] *= al[k];
      }
      const int nk = min(kTile, c1 - k0);
      for (int j = 0; j < nk; ++j) {
        float vf[8];
        unpack8(tile_chunk(sm.v[buf], j, oc), bf16, vf);
#pragma unroll
        for (int k = 0; k < kRowsPer; ++k) {
          const int r = og + kGroups * k;
          if (r < R) {
            const float pj = sm.sc[r][j];
#pragma unroll
            for (int e = 0; e < 8; ++e) o[k][e] = fmaf(pj, vf[e], o[k][e]);
          }
        }
      }
    }
    __syncthreads();  // tile buffer and scores free
  }

  if (t < ntiles) {
    // aborted: let the copies still in flight (tiles t .. t + kStages - 1) land,
    // bounded, before the CTA exits
    if (tid == 0 && !p.stall_loads) {
      const uint64_t t0 = globaltimer_ns();
      for (int u = t; u < min(ntiles, t + kStages); ++u)
        while (!mbar_try_wait(&sm.full[u % kStages], (u / kStages) & 1) &&
               globaltimer_ns() - t0 < p.timeout_ns) {
        }
    }
    return;
  }

  // this chunk's partial result per row
  if constexpr (kKeyGroups) {
    // sum the key groups through shared memory: the K and V tile buffers (adjacent,
    // free now) hold [kGroups][RM][D] floats
    float* red = reinterpret_cast<float*>(&sm.k[0][0][0]);
    static_assert(sizeof(Sm::k) + sizeof(Sm::v) >= sizeof(float) * kGroups * RM * D,
                  "reduction space");
#pragma unroll
    for (int r = 0; r < RM; ++r)
#pragma unroll
      for (int e = 0; e < 8; ++e) red[(og * RM + r) * D + oc * 8 + e] = o[r][e];
    __syncthreads();
    for (int x = tid; x < R * D; x += kThr) {
      const int r = x / D, d = x - (x / D) * D;
      float sum = 0.f;
#pragma unroll
      for (int gk = 0; gk < kGroups; ++gk) sum += red[(gk * RM + r) * D + d];
      const int g = r / p.L, i = r - g * p.L;
      const size_t row = static_cast<size_t>(b * p.H + kvh * p.G + g) * p.L + i;
      float* rec = p.part + (row * p.nsplit + split) * (D + 2);
      if (d == 0) {
        rec[0] = sm.m[r];
        rec[1] = sm.l[r];
      }
      rec[2 + d] = sum;
    }
  } else {
#pragma unroll
    for (int k = 0; k < kRowsPer; ++k) {
      const int r = og + kGroups * k;
      if (r < R) {
        const int g = r / p.L, i = r - g * p.L;
        const size_t row = static_cast<size_t>(b * p.H + kvh * p.G + g) * p.L + i;
        float* rec = p.part + (row * p.nsplit + split) * (D + 2);
        if (oc == 0) {
          rec[0] = sm.m[r];
          rec[1] = sm.l[r];
        }
#pragma unroll
        for (int e = 0; e < 8; ++e) rec[2 + oc * 8 + e] = o[k][e];
      }
    }
  }
}

// ---------------------------------------------------------------- at most 16 rows
// The common grouped-query decode (R = (H / H_kv) * L <= 16 rows per K/V head) on
// warp-level tensor-core tiles (16 x 8 x 16), with each warp keeping its own online
// softmax state over its keys, so that a tile needs no barrier across the CTA.
// Warp w of the 4 compute warps takes keys 16w .. 16w + 15 of every 64-key tile;
// the rows come in NT = ceil(R / 8) column tiles of 8 (the MMA's N), each sharing
// the A fragments loaded for the others:
//   S^T (16 keys x 8 rows) = K_w Q^T      (A = K rows by ldmatrix from the swizzled
//                                          TMA tile, B = Q^T held in registers for
//                                          the whole chunk; rows past R are zero)
//   O^T (D x 8 rows)      += V_w^T P      (A = V^T by transposing ldmatrix, B = P:
//                                          the S^T fragment rounded to 16 bits and
//                                          transposed in registers by movmatrix)
// Lane l holds rows 8t + 2(l % 4) and 8t + 2(l % 4) + 1 of tile t of both
// fragments, so its online softmax state and its share of O belong to the same
// rows.  A fifth warp keeps the ring of tiles full; the 4 warps' states are merged
// at the end.  The score is the fp32 accumulation of 16-bit products, scaled in
// fp32.
constexpr int kMdWarps = 4;                      // compute warps
constexpr int kMdThreads = (kMdWarps + 1) * 32;  // + the producer warp
constexpr int kMdRows = 16;                      // rows this kernel takes (NT <= 2)

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]) : "r"(addr));
}
__device__ __forceinline__ uint32_t movm_trans(uint32_t a) {
  uint32_t d;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(d) : "r"(a));
  return d;
}
// d += a b: m16n8k16, 16-bit A and B of one type, fp32 accumulators
template <bool BF16>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  if constexpr (BF16) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}
// Shared-memory address of 16-byte chunk c (elements 8c .. 8c + 7) of key row j of a
// swizzled tile: box c / 8, position (c % 8) ^ (j % 8) inside the row's 128 bytes.
template <int NB>
__device__ __forceinline__ uint32_t chunk_addr(const uint8_t (&tile)[NB][kBoxBytes], int j, int c) {
  return smem_u32(&tile[c >> 3][j * 128 + (((c & 7) ^ (j & 7)) << 4)]);
}
__device__ __forceinline__ uint32_t pack_16(float lo, float hi, bool bf16) {
  if (bf16) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

template <int D, int NT>
struct __align__(1024) MdSmem {
  static constexpr int kStages = D == 128 ? 2 : 3;
  uint8_t k[kStages][D / 64][kBoxBytes];
  uint8_t v[kStages][D / 64][kBoxBytes];
  float wm[kMdWarps][8 * NT], wl[kMdWarps][8 * NT];
  uint64_t full[kStages], empty[kStages];
  volatile int abort_flag;
};

template <int D, bool BF16, int NT>
__global__ void __launch_bounds__(kMdThreads, dec_ctas_per_sm(D, 8 * NT))
decode_mma_kernel(const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                  const __grid_constant__ DecParams p) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t base = smem_u32(smem_raw);
  using Sm = MdSmem<D, NT>;
  constexpr int kRows = 8 * NT;
  constexpr int kStages = Sm::kStages;
  constexpr int kKs = D / 16;  // k-steps of S = 16-dim slices; m-tiles of O^T
  Sm& sm = *reinterpret_cast<Sm*>(smem_raw + ((1024u - (base & 1023u)) & 1023u));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, bkv = blockIdx.y;
  const int b = bkv / p.Hkv, kvh = bkv - b * p.Hkv;
  const int R = p.G * p.L;

  int k_start = split * p.chunk;
  const int c1 = min(p.S, k_start + p.chunk);
  if (p.mask == FA_DECODE_SLIDING_WINDOW) k_start = max(k_start, p.S - p.L - p.window + 1);
  const int ntiles = k_start < c1 ? (c1 - k_start + kTile - 1) / kTile : 0;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kMdWarps);
    }
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();

  // this lane's rows in both fragments (8t + 2q, 8t + 2q + 1 of tile t) and its key /
  // dim row (l / 4)
  const int q4 = lane & 3, g8 = lane >> 2;
  const int n0 = 2 * q4, n1 = 2 * q4 + 1;  // rows within a tile
  float m[NT][2], l[NT][2];
  float o[NT][kKs][4];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
    m[nt][0] = m[nt][1] = -INFINITY;
    l[nt][0] = l[nt][1] = 0.f;
#pragma unroll
    for (int t = 0; t < kKs; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) o[nt][t][e] = 0.f;
  }

  if (warp == kMdWarps) {
    // producer: tile t into stage t % kStages once the warps have released the tile
    // that used it.  No L2 prefetch here: with the tiles consumed at this rate the
    // prefetched tiles of the CTAs in flight outgrew L2 and were read twice (16% over
    // K + V with four tiles ahead, 4% with none).
    if (lane == 0 && !p.stall_loads) {
      const uint64_t pol = policy_evict_first();
      int t = 0;
      for (; t < ntiles; ++t) {
        const int buf = t % kStages;
        if (t >= kStages && !dec_wait(sm, &sm.empty[buf], ((t / kStages) - 1) & 1, p)) break;
        const int k0 = k_start + t * kTile;
        fence_proxy_async_shared();
        mbar_arrive_expect_tx(&sm.full[buf], 2 * (D / 64) * kBoxBytes);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(sm.k[buf][c], &tk, &sm.full[buf], c * 64, k0, bkv, pol);
          tma_load_3d(sm.v[buf][c], &tv, &sm.full[buf], c * 64, k0, bkv, pol);
        }
      }
      // the last kStages tiles issued may still be in flight if the compute warps
      // stopped early: let them land (bounded) before the CTA exits
      const uint64_t t0 = globaltimer_ns();
      for (int u = max(0, t - kStages); u < t; ++u)
        while (!mbar_try_wait(&sm.full[u % kStages], (u / kStages) & 1) &&
               globaltimer_ns() - t0 < p.timeout_ns) {
        }
    }
  } else {
    // Q^T as the B fragments of S^T: tile nt, slice ks, lane holds Q[row 8 nt + g8]
    // [16 ks + 2 q4 + {0, 1}] and the same 8 dims further on; rows past R are zero
    uint32_t qb[NT][kKs][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int r = 8 * nt + g8;
      const bool live = r < R;
      const int g = live ? r / p.L : 0, i = live ? r - g * p.L : 0;
      const uint16_t* qrow = p.q + (static_cast<size_t>(b * p.H + kvh * p.G + g) * p.L + i) * D;
#pragma unroll
      for (int ks = 0; ks < kKs; ++ks) {
        qb[nt][ks][0] = live ? __ldg(reinterpret_cast<const unsigned int*>(qrow + 16 * ks + 2 * q4)) : 0u;
        qb[nt][ks][1] = live ? __ldg(reinterpret_cast<const unsigned int*>(qrow + 16 * ks + 8 + 2 * q4)) : 0u;
      }
    }
    // ldmatrix row of this lane: matrix lane / 8, row lane % 8
    const int mi = lane >> 3, mr = lane & 7;
    for (int t = 0; t < ntiles; ++t) {
      const int buf = t % kStages;
      if (!__all_sync(0xffffffffu, dec_wait(sm, &sm.full[buf], (t / kStages) & 1, p))) break;
      const int k0 = k_start + t * kTile;
      // S^T = K_w Q^T: A = keys 16 warp + (0..15) x dims 16 ks + (0..15); the four 8x8
      // matrices are (keys 0-7, dims 0-7), (keys 8-15, dims 0-7), (keys 0-7, dims
      // 8-15), (keys 8-15, dims 8-15); one A fragment serves every row tile
      float s[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
      {
        const int key = 16 * warp + mr + 8 * (mi & 1);
#pragma unroll
        for (int ks = 0; ks < kKs; ++ks) {
          uint32_t a[4];
          ldsm_x4(chunk_addr(sm.k[buf], key, 2 * ks + (mi >> 1)), a);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma16816<BF16>(s[nt], a, qb[nt][ks][0], qb[nt][ks][1]);
        }
      }
      // s[nt][0], s[nt][1]: key 16 warp + g8, rows 8 nt + n0, n1; s[nt][2], s[nt][3]: key + 8
      const int kva = k0 + 16 * warp + g8, kvb = kva + 8;
      uint32_t pb[NT][2];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        const int r0 = 8 * nt + n0, r1 = 8 * nt + n1;
        const int pos0 = p.S - p.L + (r0 < R ? r0 % p.L : 0);
        const int pos1 = p.S - p.L + (r1 < R ? r1 % p.L : 0);
        float x[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int kv = e < 2 ? kva : kvb;
          const int n = (e & 1) ? r1 : r0;
          const int pos = (e & 1) ? pos1 : pos0;
          float v = s[nt][e] * p.q_scale;
          if (p.softcap_on) v = p.cap_a * tanhf(v / p.cap_c);
          bool keep = n < R && kv < c1;
          if (p.mask != FA_DECODE_FULL) keep = keep && kv <= pos;
          if (p.mask == FA_DECODE_SLIDING_WINDOW) keep = keep && pos - kv < p.window;
          x[e] = keep ? v : -INFINITY;
        }
        // online softmax per row over the warp's 16 keys (lanes with the same l % 4)
        float mx0 = fmaxf(x[0], x[2]), mx1 = fmaxf(x[1], x[3]);
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, off));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, off));
        }
        const float mn0 = fmaxf(m[nt][0], mx0), mn1 = fmaxf(m[nt][1], mx1);
        const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
        const float p0 = ex2_approx(x[0] - mu0), p1 = ex2_approx(x[1] - mu1);
        const float p2 = ex2_approx(x[2] - mu0), p3 = ex2_approx(x[3] - mu1);
        float sm0 = p0 + p2, sm1 = p1 + p3;
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          sm0 += __shfl_xor_sync(0xffffffffu, sm0, off);
          sm1 += __shfl_xor_sync(0xffffffffu, sm1, off);
        }
        const float al0 = ex2_approx(m[nt][0] - mu0), al1 = ex2_approx(m[nt][1] - mu1);
        l[nt][0] = l[nt][0] * al0 + sm0;
        l[nt][1] = l[nt][1] * al1 + sm1;
        m[nt][0] = mn0;
        m[nt][1] = mn1;
        if (al0 != 1.f || al1 != 1.f) {
#pragma unroll
          for (int mt = 0; mt < kKs; ++mt) {
            o[nt][mt][0] *= al0;
            o[nt][mt][1] *= al1;
            o[nt][mt][2] *= al0;
            o[nt][mt][3] *= al1;
          }
        }
        // P as the B fragment of O^T += V^T P: transpose the two 8x8 halves
        pb[nt][0] = movm_trans(pack_16(p0, p1, BF16));
        pb[nt][1] = movm_trans(pack_16(p2, p3, BF16));
      }
      // A = V^T: dims 16 mt + (0..15) x keys 16 warp + (0..15); matrices (dims 0-7,
      // keys 0-7), (dims 8-15, keys 0-7), (dims 0-7, keys 8-15), (dims 8-15, keys
      // 8-15), each the transpose of 8 key rows x 8 dims of the tile
      {
        const int key = 16 * warp + mr + 8 * (mi >> 1);
#pragma unroll
        for (int mt = 0; mt < kKs; ++mt) {
          uint32_t a[4];
          ldsm_x4_trans(chunk_addr(sm.v[buf], key, 2 * mt + (mi & 1)), a);
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) mma16816<BF16>(o[nt][mt], a, pb[nt][0], pb[nt][1]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[buf]);
    }
  }
  __syncthreads();
  if (sm.abort_flag) return;

  // merge the 4 warps' states per row.  The tile buffers are free now and hold the
  // warps' O^T: red[warp][row][D]
  float* red = reinterpret_cast<float*>(&sm.k[0][0][0]);
  static_assert(sizeof(Sm::k) + sizeof(Sm::v) >= sizeof(float) * kMdWarps * kRows * D,
                "reduction space");
  if (warp < kMdWarps) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int r0 = 8 * nt + n0, r1 = 8 * nt + n1;
#pragma unroll
      for (int mt = 0; mt < kKs; ++mt) {
        const int d = 16 * mt + g8;
        red[(warp * kRows + r0) * D + d] = o[nt][mt][0];
        red[(warp * kRows + r1) * D + d] = o[nt][mt][1];
        red[(warp * kRows + r0) * D + d + 8] = o[nt][mt][2];
        red[(warp * kRows + r1) * D + d + 8] = o[nt][mt][3];
      }
      if (g8 == 0) {
        sm.wm[warp][r0] = m[nt][0];
        sm.wm[warp][r1] = m[nt][1];
        sm.wl[warp][r0] = l[nt][0];
        sm.wl[warp][r1] = l[nt][1];
      }
    }
  }
  __syncthreads();
  for (int xi = tid; xi < R * D; xi += kMdThreads) {
    const int rr = xi / D, d = xi - (xi / D) * D;
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < kMdWarps; ++w) mx = fmaxf(mx, sm.wm[w][rr]);
    float lsum = 0.f, acc = 0.f;
    if (mx != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kMdWarps; ++w) {
        const float a = ex2_approx(sm.wm[w][rr] - mx);  // 0 for a warp that saw no key
        lsum = fmaf(a, sm.wl[w][rr], lsum);
        acc = fmaf(a, red[(w * kRows + rr) * D + d], acc);
      }
    }
    const int g = rr / p.L, i = rr - g * p.L;
    const size_t row = static_cast<size_t>(b * p.H + kvh * p.G + g) * p.L + i;
    float* rec = p.part + (row * p.nsplit + split) * (D + 2);
    if (d == 0) {
      rec[0] = mx;
      rec[1] = lsum;
    }
    rec[2 + d] = acc;
  }
}

// One CTA per query row, one thread per output column: merge the chunks.
template <int D>
__global__ void __launch_bounds__(D) decode_combine_kernel(const __grid_constant__ DecParams p) {
  const size_t row = blockIdx.x;
  const int d = threadIdx.x;
  const float* rec0 = p.part + row * p.nsplit * (D + 2);
  float mx = -INFINITY;
  for (int s = 0; s < p.nsplit; ++s) mx = fmaxf(mx, rec0[static_cast<size_t>(s) * (D + 2)]);
  float l = 0.f, acc = 0.f;
  if (mx != -INFINITY) {
    for (int s = 0; s < p.nsplit; ++s) {
      const float* rec = rec0 + static_cast<size_t>(s) * (D + 2);
      const float w = ex2_approx(rec[0] - mx);  // 0 for a chunk that saw no key
      l = fmaf(w, rec[1], l);
      acc = fmaf(w, rec[2 + d], acc);
    }
  }
  const float o = l > 0.f ? acc / l : 0.f;
  uint16_t* dst = static_cast<uint16_t*>(p.out) + row * D + d;
  if (p.is_bf16) {
    *reinterpret_cast<__nv_bfloat16*>(dst) = __float2bfloat16_rn(o);
  } else {
    *reinterpret_cast<__half*>(dst) = __float2half_rn(o);
  }
  if (d == 0 && p.lse) p.lse[row] = l > 0.f ? (mx + log2f(l)) * kDecLn2 : -INFINITY;
}

// ---------------------------------------------------------------- host side
// Chunking of the keys over the (B * Hkv) groups, whole tiles.  The CTAs run in
// waves of (SMs x CTAs per SM); the time is about (waves) x (tiles per chunk
// + a fixed cost per CTA), so the split count is chosen to minimise that product --
// a grid just past a whole number of waves leaves most SMs idle in its last wave.
// The plan is a function of the shape alone (B200: 148 SMs), so the workspace size
// that depends on it needs no device.
void decode_plan(int B, int Hkv, int S, int D, int rows, int* nsplit, int* chunk) {
  constexpr int kSms = 148;
  constexpr int kCtaCost = 2;  // prologue and merge record, in tile units
  const int64_t groups = static_cast<int64_t>(B) * Hkv > 0 ? static_cast<int64_t>(B) * Hkv : 1;
  const int tiles = S > 0 ? (S + kTile - 1) / kTile : 1;
  const int64_t slots = static_cast<int64_t>(kSms) * dec_ctas_per_sm(D, rows);
  int best_tiles = tiles;
  int64_t best_cost = INT64_MAX;
  for (int n = 1; n <= tiles && n <= 256; ++n) {
    const int per = (tiles + n - 1) / n;      // tiles per chunk
    const int used = (tiles + per - 1) / per; // splits actually used
    if (used != n) continue;
    const int64_t waves = (groups * used + slots - 1) / slots;
    const int64_t cost = waves * (per + kCtaCost);
    if (cost < best_cost) {
      best_cost = cost;
      best_tiles = per;
    }
  }
  *chunk = best_tiles * kTile;
  *nsplit = S > 0 ? (S + *chunk - 1) / *chunk : 1;
}

template <int D, bool BF16, int NT>
fa_status decode_mma_launch(const void* k, const void* v, int B, int S, const DecParams& prm,
                            cudaStream_t stream) {
  CUtensorMap tk, tv;
  // With S == 0 no tile is loaded; the maps only need to be well formed.
  const void* kp = S > 0 ? k : prm.q;
  const void* vp = S > 0 ? v : prm.q;
  const int rows = S > 0 ? S : 1, bh = S > 0 ? B * prm.Hkv : 1;
  if (!make_tile_map(&tk, kp, BF16, D, rows, bh, kTile)) return FA_ERR_CUDA;
  if (!make_tile_map(&tv, vp, BF16, D, rows, bh, kTile)) return FA_ERR_CUDA;
  const size_t smem = sizeof(MdSmem<D, NT>) + 1024;
  int dev = 0;
  FA_CUDA_CHECK(cudaGetDevice(&dev));
  {
    static std::mutex mu;
    static bool done[kMaxDevices] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
    if (!done[dev]) {
      FA_CUDA_CHECK(cudaFuncSetAttribute(decode_mma_kernel<D, BF16, NT>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem)));
      done[dev] = true;
    }
  }
  const dim3 grid(prm.nsplit, B * prm.Hkv);
  decode_mma_kernel<D, BF16, NT><<<grid, kMdThreads, smem, stream>>>(tk, tv, prm);
  FA_CUDA_CHECK(cudaGetLastError());
  decode_combine_kernel<D><<<B * prm.H * prm.L, D, 0, stream>>>(prm);
  FA_CUDA_CHECK(cudaGetLastError());
  return FA_OK;
}

template <int D, int RM>
fa_status decode_launch(const void* k, const void* v, bool bf16, int B, int S, const DecParams& prm,
                        cudaStream_t stream) {
  CUtensorMap tk, tv;
  // With S == 0 no tile is loaded; the maps only need to be well formed.
  const void* kp = S > 0 ? k : prm.q;
  const void* vp = S > 0 ? v : prm.q;
  const int rows = S > 0 ? S : 1, bh = S > 0 ? B * prm.Hkv : 1;
  if (!make_tile_map(&tk, kp, bf16, D, rows, bh, kTile)) return FA_ERR_CUDA;
  if (!make_tile_map(&tv, vp, bf16, D, rows, bh, kTile)) return FA_ERR_CUDA;
  const size_t smem = sizeof(DecSmem<D, RM>) + 1024;
  int dev = 0;
  FA_CUDA_CHECK(cudaGetDevice(&dev));
  {
    static std::mutex mu;
    static bool done[kMaxDevices] = {};
    std::lock_guard<std::mutex> lock(mu);
    if (dev < 0 || dev >= kMaxDevices) return FA_ERR_UNSUPPORTED;
    if (!done[dev]) {
      FA_CUDA_CHECK(cudaFuncSetAttribute(decode_split_kernel<D, RM>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         static_cast<int>(smem)));
      done[dev] = true;
    }
  }
  const dim3 grid(prm.nsplit, B * prm.Hkv);
  decode_split_kernel<D, RM><<<grid, DecCfg<D>::kThreads, smem, stream>>>(tk, tv, prm);
  FA_CUDA_CHECK(cudaGetLastError());
  decode_combine_kernel<D><<<B * prm.H * prm.L, D, 0, stream>>>(prm);
  FA_CUDA_CHECK(cudaGetLastError());
  return FA_OK;
}

}  // namespace
}  // namespace fa

extern "C" size_t fa_decode_workspace_bytes(int32_t B, int32_t H, int32_t H_kv, int32_t L,
                                            int32_t S, int32_t D) {
  if (B < 0 || H < 0 || H_kv < 1 || L < 0 || S < 0 || D < 0) return 0;
  int nsplit = 0, chunk = 0;
  fa::decode_plan(B, H_kv, S, D, H_kv > 0 && H > 0 ? (H / H_kv) * L : L, &nsplit, &chunk);
  return fa::kDecWorkspaceHeader + static_cast<size_t>(B) * H * L * nsplit * (D + 2) * sizeof(float);
}

extern "C" fa_status fa_flex_attention_decode(const void* q, const void* k, const void* v,
                                              int32_t dtype, int32_t B, int32_t H, int32_t H_kv,
                                              int32_t L, int32_t S, int32_t D, int32_t mask,
                                              int32_t window, int32_t score_kind, float softcap,
                                              float scale, void* out, float* lse, void* workspace,
                                              size_t workspace_bytes, void* stream) {
  using namespace fa;
  if (dtype != FA_BF16 && dtype != FA_FP16) return FA_ERR_INVALID_ARG;
  if (B < 0 || H < 0 || L < 0 || S < 0 || H_kv < 1 || (H > 0 && H % H_kv != 0))
    return FA_ERR_INVALID_ARG;
  if (S > FA_MAX_LEN) return FA_ERR_INVALID_ARG;
  if (mask < FA_DECODE_FULL || mask > FA_DECODE_SLIDING_WINDOW) return FA_ERR_INVALID_ARG;
  if (mask == FA_DECODE_SLIDING_WINDOW && window < 1) return FA_ERR_INVALID_ARG;
  if (score_kind != FA_SCORE_NONE && score_kind != FA_SCORE_TANH_SOFTCAP) return FA_ERR_INVALID_ARG;
  if (score_kind == FA_SCORE_TANH_SOFTCAP && !(softcap > 0.f && std::isfinite(softcap)))
    return FA_ERR_INVALID_ARG;
  if (!std::isfinite(scale)) return FA_ERR_INVALID_ARG;
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  const int G = H > 0 ? H / H_kv : 1;
  if (static_cast<int64_t>(G) * L > kMaxRows) return FA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H * L == 0) return FA_OK;
  if (static_cast<int64_t>(B) * H * L > INT32_MAX || static_cast<int64_t>(B) * H_kv > 65535)
    return FA_ERR_UNSUPPORTED;
  if (workspace == nullptr || workspace_bytes < fa_decode_workspace_bytes(B, H, H_kv, L, S, D))
    return FA_ERR_INVALID_ARG;
  if (q == nullptr || out == nullptr || (S > 0 && (k == nullptr || v == nullptr)))
    return FA_ERR_INVALID_ARG;
  // Q, K, V (TMA tiles and 16-byte loads), out and the workspace: 16 bytes; LSE
  // (4-byte stores): 4 bytes.  Checked here so that a misaligned pointer is an
  // argument error, never a device fault.
  auto misaligned = [](const void* ptr, uintptr_t a) {
    return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) != 0;
  };
  if (misaligned(q, 16) || misaligned(out, 16) || misaligned(workspace, 16) ||
      (S > 0 && (misaligned(k, 16) || misaligned(v, 16))) || misaligned(lse, 4))
    return FA_ERR_INVALID_ARG;

  DecParams prm{};
  prm.q = static_cast<const uint16_t*>(q);
  prm.out = out;
  prm.lse = lse;
  prm.err = static_cast<int32_t*>(workspace);
  prm.part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + kDecWorkspaceHeader);
  prm.H = H;
  prm.Hkv = H_kv;
  prm.G = G;
  prm.L = L;
  prm.S = S;
  decode_plan(B, H_kv, S, D, G * L, &prm.nsplit, &prm.chunk);
  prm.mask = mask;
  prm.window = mask == FA_DECODE_SLIDING_WINDOW ? window : 0;
  prm.softcap_on = score_kind == FA_SCORE_TANH_SOFTCAP ? 1 : 0;
  prm.is_bf16 = dtype == FA_BF16 ? 1 : 0;
  const float sc = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(D));
  prm.q_scale = prm.softcap_on ? sc : sc * kDecLog2e;
  prm.cap_c = prm.softcap_on ? softcap : 1.f;
  prm.cap_a = prm.softcap_on ? softcap * kDecLog2e : 0.f;
  prm.timeout_ns = 2000000000ull;
  if (debug_stall(&prm.timeout_ns)) prm.stall_loads = 1;
  const cudaStream_t s = as_stream(stream);
  const bool b16 = dtype == FA_BF16;
  const int rows = G * L;
  // up to 16 rows (one or two of the MMA's 8-row N tiles): the tensor-core chunk
  // kernel; more: the CUDA-core one
  if (D == 64) {
    if (rows <= 8)
      return b16 ? decode_mma_launch<64, true, 1>(k, v, B, S, prm, s)
                 : decode_mma_launch<64, false, 1>(k, v, B, S, prm, s);
    if (rows <= kMdRows)
      return b16 ? decode_mma_launch<64, true, 2>(k, v, B, S, prm, s)
                 : decode_mma_launch<64, false, 2>(k, v, B, S, prm, s);
    return decode_launch<64, 32>(k, v, b16, B, S, prm, s);
  }
  if (rows <= 8)
    return b16 ? decode_mma_launch<128, true, 1>(k, v, B, S, prm, s)
               : decode_mma_launch<128, false, 1>(k, v, B, S, prm, s);
  if (rows <= kMdRows)
    return b16 ? decode_mma_launch<128, true, 2>(k, v, B, S, prm, s)
               : decode_mma_launch<128, false, 2>(k, v, B, S, prm, s);
  return decode_launch<128, 32>(k, v, b16, B, S, prm, s);
}
