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
// nothing.  The chunk kernel, `decode_mma_kernel`, gives its warps private softmax
// states and runs both products on warp-level tensor-core tiles, so the instruction
// stream stays well below the HBM time; up to 16 rows one CTA takes them all, beyond
// that one CTA per 16 rows, neighbours in launch order, so K and V still come from
// DRAM about once.
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
// CTAs per SM of the chunk kernel for R rows: three (two at D = 128 for R > 8, with
// twice the accumulators).  The grid is sized for that many CTAs.
__host__ __device__ constexpr int dec_ctas_per_sm(int D, int rows) {
  return rows <= 8 ? 3 : (D == 128 ? 2 : 3);
}
// Tensor-core kernel: CTAs per (chunk, K/V head), each taking 16 of the R rows (one
// for R <= 16).
__host__ __device__ constexpr int dec_row_tiles(int rows) { return rows <= 16 ? 1 : (rows + 15) / 16; }
constexpr int kBoxBytes = kTile * 128;  // one TMA box: 64 keys x 64 elements
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
  int row_tiles;  // tensor-core kernel: CTAs per (chunk, K/V head), each taking 16 rows
  float q_scale;  // folded into Q: scale * log2(e), or scale alone under the softcap
  float cap_c;    // softcap c
  float cap_a;    // c * log2(e)
  unsigned long long timeout_ns;
  int stall_loads;  // testing hook: no K/V tile is loaded (see fa_debug_set_mma_stall)
};

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

// ---------------------------------------------------------------- chunk kernel
// Grouped-query decode (R = (H / H_kv) * L <= 32 rows per K/V head, 16 per CTA) on
// warp-level tensor-core tiles (16 x 8 x 16), with each warp keeping its own online
// softmax state over its keys, so that a tile needs no barrier across the CTA.
// Warp w of the 4 compute warps takes keys 16w .. 16w + 15 of every 64-key tile;
// the CTA's rows come in NT = 1 or 2 column tiles of 8 (the MMA's N), each sharing
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
  // blockIdx.x = chunk * row_tiles + row tile: the CTAs of one chunk's row tiles are
  // neighbours in launch order, so they read the same K / V tiles at about the same
  // time and all but the first find them in L2
  const int split = blockIdx.x / p.row_tiles, bkv = blockIdx.y;
  const int rbase = (blockIdx.x - split * p.row_tiles) * kRows;  // first row of this CTA
  const int b = bkv / p.Hkv, kvh = bkv - b * p.Hkv;
  const int R = min(p.G * p.L - rbase, kRows);  // rows of this CTA: rbase .. rbase + R - 1

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
  // Launched as a programmatic dependent: nothing in global memory is read before
  // the previous kernel on the stream has finished.  The merge kernel may launch
  // as soon as every CTA is running (it waits for this grid before reading).
  grid_dep_wait();
  grid_dep_launch_dependents();

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
      const int g = live ? (rbase + r) / p.L : 0, i = live ? rbase + r - g * p.L : 0;
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
        const int pos0 = p.S - p.L + (r0 < R ? (rbase + r0) % p.L : 0);
        const int pos1 = p.S - p.L + (r1 < R ? (rbase + r1) % p.L : 0);
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
    const int g = (rbase + rr) / p.L, i = rbase + rr - g * p.L;
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
  grid_dep_wait();  // the chunk kernel's records are complete
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
  const int64_t groups = (static_cast<int64_t>(B) * Hkv > 0 ? static_cast<int64_t>(B) * Hkv : 1) *
                        dec_row_tiles(rows);
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
  const dim3 grid(prm.nsplit * prm.row_tiles, B * prm.Hkv);
  FA_CUDA_CHECK(launch_pdl(decode_mma_kernel<D, BF16, NT>, grid, dim3(kMdThreads), smem, stream,
                           tk, tv, prm));
  FA_CUDA_CHECK(launch_pdl(decode_combine_kernel<D>, dim3(B * prm.H * prm.L), dim3(D), 0, stream,
                           prm));
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
  prm.row_tiles = dec_row_tiles(G * L);
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
  // the tensor-core chunk kernel: one 8-row column tile up to 8 rows, else two,
  // with a CTA per 16 rows beyond 16
  if (D == 64) {
    if (rows <= 8)
      return b16 ? decode_mma_launch<64, true, 1>(k, v, B, S, prm, s)
                 : decode_mma_launch<64, false, 1>(k, v, B, S, prm, s);
    return b16 ? decode_mma_launch<64, true, 2>(k, v, B, S, prm, s)
               : decode_mma_launch<64, false, 2>(k, v, B, S, prm, s);
  }
  if (rows <= 8)
    return b16 ? decode_mma_launch<128, true, 1>(k, v, B, S, prm, s)
               : decode_mma_launch<128, false, 1>(k, v, B, S, prm, s);
  return b16 ? decode_mma_launch<128, true, 2>(k, v, B, S, prm, s)
             : decode_mma_launch<128, false, 2>(k, v, B, S, prm, s);
}
