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
// Three kernels: delta (a warp per row); dQ, one CTA per 128-query tile in the
// forward's schedule order; dK and dV, one CTA per 128-key tile over its column
// lists and the query heads that share its K/V head.  Every output tile is owned by
// one CTA (no atomics; dQ recomputes S and dP instead of accumulating into global
// memory).  The products run on the tensor cores as warp-level mma.sync
// m16n8k16 tiles (16-bit operands, fp32 accumulation) fed from shared memory by
// cp.async double buffering; P and dS enter the second products rounded to the
// input dtype, as in FlashAttention-2.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "fa_internal.h"

namespace fa {
namespace {

constexpr int kBwdWarps = 8;
constexpr float kBwdLog2e = 1.4426950408889634f;

struct BwdParams {
  const uint16_t *q, *k, *v, *out, *dout;
  const float* lse;
  float* delta;
  uint16_t *dq, *dk, *dv;
  const int32_t *kv_num, *kv_idx, *full_num, *full_idx;      // row lists
  const int32_t *q_num, *q_idx, *full_q_num, *full_q_idx;   // column lists
  const int32_t* sched;                                      // forward's q-block order
  const int32_t* doc_id;
  const uint32_t* bitmap;
  int B, H, Hkv, G, L, S, n_q, n_kv, kind, window, softcap_on, is_bf16;
  float scale, cap_c;
};

__device__ __forceinline__ float2 load_pair(const uint16_t* ptr, bool bf16) {
  const uint32_t u = __ldg(reinterpret_cast<const unsigned int*>(ptr));
  if (bf16) return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
  return __half22float2(*reinterpret_cast<const __half2*>(&u));
}

__device__ __forceinline__ void store_pair(uint16_t* ptr, float2 x, bool bf16) {
  if (bf16) {
    *reinterpret_cast<__nv_bfloat162*>(ptr) = __floats2bfloat162_rn(x.x, x.y);
  } else {
    *reinterpret_cast<__half2*>(ptr) = __floats2half2_rn(x.x, x.y);
  }
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// The mask rule for (query i, key j) inside a PARTIAL block (FULL blocks skip it).
__device__ __forceinline__ bool pair_live(const BwdParams& p, int i, int j) {
  switch (p.kind) {
    case FA_MASK_CAUSAL: return j <= i;
    case FA_MASK_SLIDING_WINDOW_CAUSAL: return j <= i && i - j < p.window;
    case FA_MASK_DOCUMENT_CAUSAL: return j <= i && __ldg(p.doc_id + i) == __ldg(p.doc_id + j);
    default: {
      const uint32_t w = __ldg(p.bitmap + static_cast<size_t>(i) * 4 * p.n_kv + (j >> 5));
      return ((w >> (j & 31)) & 1u) != 0u;
    }
  }
}

// P and dS of one pair from the two dot products (natural-log LSE of the row).
__device__ __forceinline__ void pair_grads(const BwdParams& p, float qk, float dov, float lse2,
                                           float delta, float& pij, float& dsij) {
  const float t = qk * p.scale;
  float s = t, dcap = 1.f;
  if (p.softcap_on) {
    const float th = tanhf(t / p.cap_c);
    s = p.cap_c * th;
    dcap = 1.f - th * th;
  }
  pij = exp2f(s * kBwdLog2e - lse2);
  dsij = pij * (dov - delta) * dcap;
}

// delta_i = rowsum(dO_i * O_i): one warp per row of (B * H * L).
template <int D>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_delta_kernel(const BwdParams p) {
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kBwdWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<int64_t>(p.B) * p.H * p.L) return;
  const bool bf16 = p.is_bf16 != 0;
  float acc = 0.f;
#pragma unroll
  for (int e = 0; e < D / 64; ++e) {
    const int64_t off = row * D + 2 * lane + 64 * e;
    const float2 o = load_pair(p.out + off, bf16), g = load_pair(p.dout + off, bf16);
    acc = fmaf(o.x, g.x, fmaf(o.y, g.y, acc));
  }
  acc = warp_sum(acc);
  if (lane == 0) p.delta[row] = acc;
}

// ---- tensor-core tiles (mma.sync m16n8k16, fp32 accumulate) ---------------------
//
// Fragment layouts (PTX ISA, "Matrix fragments for mma.m16n8k16"): lane = 4 g + t.
// A 16x16 (row): {(g, 2t..2t+1), (g+8, 2t..), (g, 2t+8..), (g+8, 2t+8..)}.
// B 16x8 (col):  {(k = 2t..2t+1, n = g), (k = 2t+8.., n = g)}.
// C 16x8 fp32:   {(g, 2t), (g, 2t+1), (g+8, 2t), (g+8, 2t+1)}.
// Two adjacent C tiles of a 16-row product, rounded to 16 bits, are the A operand
// of a 16-deep k step: how P and dS feed the second product without shared memory.
// Shared-memory tiles are row-major with rows padded to D + 8 elements, so the
// eight 16-byte rows of one ldmatrix land in eight different bank groups.

__device__ __forceinline__ uint32_t smem_addr(const void* ptr) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(ptr));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

template <bool BF>
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  if constexpr (BF) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  } else {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, "
        "{%4, %5, %6, %7}, {%8, %9}, {%0, %1, %2, %3};\n"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  }
}

// Two floats as one 16-bit pair, the first in the low half.
template <bool BF>
__device__ __forceinline__ uint32_t pack16(float lo, float hi) {
  if constexpr (BF) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
  } else {
    const __half2 h = __floats2half2_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
  }
}

// 16-byte global -> shared copy; with valid == false the 16 bytes are zero-filled
// and nothing is read.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, bool valid) {
  const int n = valid ? 16 : 0;
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src), "r"(n));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N));
}

// Rows [r0, r0 + R) of a (rows x D) 16-bit tensor into a padded shared tile; rows at
// or past n_rows are zero.  All threads of the CTA take part.
template <int D, int R>
__device__ __forceinline__ void load_tile(uint16_t* tile, const uint16_t* src, int64_t r0,
                                          int64_t n_rows) {
  constexpr int kChunks = D / 8, LD = D + 8;
  for (int c = threadIdx.x; c < R * kChunks; c += kBwdWarps * 32) {
    const int r = c / kChunks, col = (c - r * kChunks) * 8;
    const bool ok = r0 + r < n_rows;
    const uint16_t* g = src + (ok ? (r0 + r) * D + col : 0);
    cp_async16(smem_addr(tile + r * LD + col), g, ok);
  }
}

// Per row of a query tile: lse * log2(e), or +inf for rows past L and rows with no
// live key (P = exp2(s - inf) = 0 there), and delta.
__device__ __forceinline__ void row_stats(const BwdParams& p, int64_t bh, int64_t i, float& l2,
                                          float& dl) {
  l2 = INFINITY;
  dl = 0.f;
  if (i < p.L) {
    const float l = p.lse[bh * p.L + i];
    if (l != -INFINITY) {
      l2 = l * kBwdLog2e;
      dl = p.delta[bh * p.L + i];
    }
  }
}

// Entry t of a block list: the t-th PARTIAL block, then the FULL ones after np.
__device__ __forceinline__ int list_entry(const int32_t* idx, const int32_t* fidx, int np,
                                          int64_t base, int t, bool& full) {
  full = t >= np;
  return full ? __ldg(fidx + base + (t - np)) : __ldg(idx + base + t);
}

// dK, dV of one 128-key tile (b, kv head, kv block), over the query heads of its
// group and the q blocks of its column lists, BR query rows at a time.  Warp w owns
// keys 16 w .. 16 w + 15 and computes the transposed products:
//   S^T = K Q^T,  dP^T = V dO^T  (16 x BR),  then  dV += P^T dO,  dK += dS^T Q.
template <int D>
struct DkdvTile {
  static constexpr int BR = D == 64 ? 64 : 32;
  static constexpr int LD = D + 8;
  static constexpr size_t kSmem =
      (2 * 128 + 4 * BR) * LD * sizeof(uint16_t) + 4 * BR * sizeof(float);
};

template <int D, bool BF>
__global__ void __launch_bounds__(kBwdWarps * 32, 1) bwd_dkdv_mma_kernel(const BwdParams p) {
  using T = DkdvTile<D>;
  constexpr int BR = T::BR, LD = T::LD, KT = D / 16, NQ = BR / 8, ND = D / 8, SUBS = 128 / BR;
  extern __shared__ __align__(16) uint16_t smem[];
  uint16_t* Ks = smem;                  // [128][LD]
  uint16_t* Vs = Ks + 128 * LD;         // [128][LD]
  uint16_t* Qs = Vs + 128 * LD;         // [2][BR][LD]
  uint16_t* Gs = Qs + 2 * BR * LD;      // [2][BR][LD]  dO
  float* Ls = reinterpret_cast<float*>(Gs + 2 * BR * LD);  // [2][BR]
  float* Dl = Ls + 2 * BR;                                 // [2][BR]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const int64_t n_kvbh = static_cast<int64_t>(p.B) * p.Hkv;
  const int jb = static_cast<int>(blockIdx.x / n_kvbh);   // column-major: longest columns first
  const int64_t kvbh = blockIdx.x - static_cast<int64_t>(jb) * n_kvbh;
  const int64_t b = kvbh / p.Hkv, kvh = kvbh - b * p.Hkv;
  const int j0 = jb * 128;

  load_tile<D, 128>(Ks, p.k, kvbh * p.S + j0, kvbh * p.S + p.S);
  load_tile<D, 128>(Vs, p.v, kvbh * p.S + j0, kvbh * p.S + p.S);
  cp_async_commit();

  const int np = p.n_q > 0 ? __ldg(p.q_num + jb) : 0;
  const int nf = p.n_q > 0 ? __ldg(p.full_q_num + jb) : 0;
  const int nblk = np + nf;
  const int n_it = p.G * nblk * SUBS;
  const int64_t list_base = static_cast<int64_t>(jb) * p.n_q;

  // iteration it -> (query head in the group, list entry, BR-row slice)
  auto decode = [&](int it, int64_t& bh, int& i0, bool& full) {
    const int sub = it % SUBS, rest = it / SUBS;
    const int t = rest % nblk, gg = rest / nblk;
    const int ib = list_entry(p.q_idx, p.full_q_idx, np, list_base, t, full);
    i0 = ib * 128 + sub * BR;
    bh = b * p.H + kvh * p.G + gg;
  };
  auto prefetch = [&](int it, int st) {
    int64_t bh;
    int i0;
    bool full;
    decode(it, bh, i0, full);
    load_tile<D, BR>(Qs + st * BR * LD, p.q, bh * p.L + i0, bh * p.L + p.L);
    load_tile<D, BR>(Gs + st * BR * LD, p.dout, bh * p.L + i0, bh * p.L + p.L);
    for (int r = threadIdx.x; r < BR; r += kBwdWarps * 32)
      row_stats(p, bh, static_cast<int64_t>(i0) + r, Ls[st * BR + r], Dl[st * BR + r]);
  };

  if (n_it > 0) prefetch(0, 0);
  cp_async_commit();
  cp_async_wait<1>();  // the K / V tile
  __syncthreads();

  // K and V rows of this warp as A operands: held in registers for the whole
  // column at D = 64, re-read from shared memory per use at D = 128 (registers)
  constexpr bool kHold = D == 64;
  constexpr int KH = kHold ? KT : 1;
  const int a_row = 16 * warp + (lane & 7) + 8 * ((lane >> 3) & 1);
  const int a_col = 8 * (lane >> 4);
  uint32_t kf[KH][4], vf[KH][4];
  if constexpr (kHold) {
#pragma unroll
    for (int kk = 0; kk < KT; ++kk) {
      ldsm_x4(kf[kk], smem_addr(Ks + a_row * LD + kk * 16 + a_col));
      ldsm_x4(vf[kk], smem_addr(Vs + a_row * LD + kk * 16 + a_col));
    }
  }
  const int kr0 = j0 + 16 * warp + g;  // key of C rows g; kr0 + 8 for rows g + 8

  float dk[ND][4], dv[ND][4];
#pragma unroll
  for (int n = 0; n < ND; ++n)
#pragma unroll
    for (int c = 0; c < 4; ++c) dk[n][c] = dv[n][c] = 0.f;

  for (int it = 0; it < n_it; ++it) {
    const int st = it & 1;
    if (it + 1 < n_it) prefetch(it + 1, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    int64_t bh;
    int i0;
    bool full;
    decode(it, bh, i0, full);
    const uint16_t* Qt = Qs + st * BR * LD;
    const uint16_t* Gt = Gs + st * BR * LD;
    const float* Lt = Ls + st * BR;
    const float* Dt = Dl + st * BR;

    float s[NQ][4], dp[NQ][4];
#pragma unroll
    for (int n = 0; n < NQ; ++n)
#pragma unroll
      for (int c = 0; c < 4; ++c) s[n][c] = dp[n][c] = 0.f;
    {
      // B operands: Q / dO rows (n = query, k = d), two 8-query tiles per ldmatrix
      const int row = (lane & 7) + 8 * (lane >> 4);
      const int col = 8 * ((lane >> 3) & 1);
#pragma unroll
      for (int kk = 0; kk < KT; ++kk) {
        uint32_t ka[4], va[4];
        if constexpr (kHold) {
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            ka[r] = kf[kk][r];
            va[r] = vf[kk][r];
          }
        } else {
          ldsm_x4(ka, smem_addr(Ks + a_row * LD + kk * 16 + a_col));
          ldsm_x4(va, smem_addr(Vs + a_row * LD + kk * 16 + a_col));
        }
#pragma unroll
        for (int n2 = 0; n2 < NQ / 2; ++n2) {
          uint32_t bq[4], bg[4];
          ldsm_x4(bq, smem_addr(Qt + (n2 * 16 + row) * LD + kk * 16 + col));
          ldsm_x4(bg, smem_addr(Gt + (n2 * 16 + row) * LD + kk * 16 + col));
          mma16816<BF>(s[2 * n2], ka, bq[0], bq[1]);
          mma16816<BF>(s[2 * n2 + 1], ka, bq[2], bq[3]);
          mma16816<BF>(dp[2 * n2], va, bg[0], bg[1]);
          mma16816<BF>(dp[2 * n2 + 1], va, bg[2], bg[3]);
        }
      }
    }
    // P^T and dS^T in place of S^T and dP^T
#pragma unroll
    for (int n = 0; n < NQ; ++n) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int qc = n * 8 + 2 * tq + (c & 1);
        const int j = kr0 + 8 * (c >> 1), i = i0 + qc;
        float pij, dsij;
        pair_grads(p, s[n][c], dp[n][c], Lt[qc], Dt[qc], pij, dsij);
        bool keep = j < p.S;
        if (!full) keep = keep && i < p.L && pair_live(p, i, j);
        s[n][c] = keep ? pij : 0.f;
        dp[n][c] = keep ? dsij : 0.f;
      }
    }
    // dV += P^T dO, dK += dS^T Q: B operands dO / Q (k = query, n = d) by transposed loads
    {
      const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
      const int col = 8 * (lane >> 4);
#pragma unroll
      for (int kq = 0; kq < BR / 16; ++kq) {
        const uint32_t ap[4] = {pack16<BF>(s[2 * kq][0], s[2 * kq][1]),
                                pack16<BF>(s[2 * kq][2], s[2 * kq][3]),
                                pack16<BF>(s[2 * kq + 1][0], s[2 * kq + 1][1]),
                                pack16<BF>(s[2 * kq + 1][2], s[2 * kq + 1][3])};
        const uint32_t ad[4] = {pack16<BF>(dp[2 * kq][0], dp[2 * kq][1]),
                                pack16<BF>(dp[2 * kq][2], dp[2 * kq][3]),
                                pack16<BF>(dp[2 * kq + 1][0], dp[2 * kq + 1][1]),
                                pack16<BF>(dp[2 * kq + 1][2], dp[2 * kq + 1][3])};
#pragma unroll
        for (int n2 = 0; n2 < ND / 2; ++n2) {
          uint32_t bg[4], bq[4];
          ldsm_x4_trans(bg, smem_addr(Gt + (kq * 16 + row) * LD + n2 * 16 + col));
          ldsm_x4_trans(bq, smem_addr(Qt + (kq * 16 + row) * LD + n2 * 16 + col));
          mma16816<BF>(dv[2 * n2], ap, bg[0], bg[1]);
          mma16816<BF>(dv[2 * n2 + 1], ap, bg[2], bg[3]);
          mma16816<BF>(dk[2 * n2], ad, bq[0], bq[1]);
          mma16816<BF>(dk[2 * n2 + 1], ad, bq[2], bq[3]);
        }
      }
    }
    __syncthreads();  // this stage is refilled by the next iteration's prefetch
  }
  cp_async_wait<0>();

  const bool bf16 = BF;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int j = kr0 + 8 * h;
    if (j >= p.S) continue;
    const int64_t off = (kvbh * p.S + j) * D + 2 * tq;
#pragma unroll
    for (int n = 0; n < ND; ++n) {
      store_pair(p.dk + off + n * 8,
                 make_float2(dk[n][2 * h] * p.scale, dk[n][2 * h + 1] * p.scale), bf16);
      store_pair(p.dv + off + n * 8, make_float2(dv[n][2 * h], dv[n][2 * h + 1]), bf16);
    }
  }
}

// dQ of one 128-query tile (b, h, q block), over the kv blocks of its row lists, BC
// keys at a time.  Warp w owns queries 16 w .. 16 w + 15:
//   S = Q K^T,  dP = dO V^T  (16 x BC),  then  dQ += dS K.
// Tiles run in the forward's schedule order (longest rows first).
template <int D>
struct DqTile {
  static constexpr int BC = D == 64 ? 64 : 32;
  static constexpr int LD = D + 8;
  static constexpr size_t kSmem = (2 * 128 + 4 * BC) * LD * sizeof(uint16_t);
};

template <int D, bool BF>
__global__ void __launch_bounds__(kBwdWarps * 32, 1) bwd_dq_mma_kernel(const BwdParams p) {
  using T = DqTile<D>;
  constexpr int BC = T::BC, LD = T::LD, KT = D / 16, NK = BC / 8, ND = D / 8, SUBS = 128 / BC;
  extern __shared__ __align__(16) uint16_t smem[];
  uint16_t* Qs = smem;                 // [128][LD]
  uint16_t* Gs = Qs + 128 * LD;        // [128][LD]  dO
  uint16_t* Ks = Gs + 128 * LD;        // [2][BC][LD]
  uint16_t* Vs = Ks + 2 * BC * LD;     // [2][BC][LD]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, tq = lane & 3;
  const int64_t n_bh = static_cast<int64_t>(p.B) * p.H;
  const int rank = static_cast<int>(blockIdx.x / n_bh);
  const int64_t bh = blockIdx.x - static_cast<int64_t>(rank) * n_bh;
  const int qb = p.sched != nullptr ? __ldg(p.sched + 2 * rank) : rank;
  const int64_t kvbh = (bh / p.H) * p.Hkv + (bh % p.H) / p.G;
  const int i0 = qb * 128;

  load_tile<D, 128>(Qs, p.q, bh * p.L + i0, bh * p.L + p.L);
  load_tile<D, 128>(Gs, p.dout, bh * p.L + i0, bh * p.L + p.L);
  cp_async_commit();

  const int np = __ldg(p.kv_num + qb), nf = __ldg(p.full_num + qb);
  const int n_it = (np + nf) * SUBS;
  const int64_t list_base = static_cast<int64_t>(qb) * p.n_kv;
  auto decode = [&](int it, int& j0, bool& full) {
    const int jb = list_entry(p.kv_idx, p.full_idx, np, list_base, it / SUBS, full);
    j0 = jb * 128 + (it % SUBS) * BC;
  };
  auto prefetch = [&](int it, int st) {
    int j0;
    bool full;
    decode(it, j0, full);
    load_tile<D, BC>(Ks + st * BC * LD, p.k, kvbh * p.S + j0, kvbh * p.S + p.S);
    load_tile<D, BC>(Vs + st * BC * LD, p.v, kvbh * p.S + j0, kvbh * p.S + p.S);
  };

  if (n_it > 0) prefetch(0, 0);
  cp_async_commit();
  cp_async_wait<1>();  // the Q / dO tile
  __syncthreads();

  uint32_t qf[KT][4], gf[KT][4];
  {
    const int row = 16 * warp + (lane & 7) + 8 * ((lane >> 3) & 1);
    const int col = 8 * (lane >> 4);
#pragma unroll
    for (int kk = 0; kk < KT; ++kk) {
      ldsm_x4(qf[kk], smem_addr(Qs + row * LD + kk * 16 + col));
      ldsm_x4(gf[kk], smem_addr(Gs + row * LD + kk * 16 + col));
    }
  }
  const int qr0 = i0 + 16 * warp + g;  // query of C rows g; qr0 + 8 for rows g + 8
  float l2[2], dl[2];
  row_stats(p, bh, qr0, l2[0], dl[0]);
  row_stats(p, bh, qr0 + 8, l2[1], dl[1]);

  float dq[ND][4];
#pragma unroll
  for (int n = 0; n < ND; ++n)
#pragma unroll
    for (int c = 0; c < 4; ++c) dq[n][c] = 0.f;

  for (int it = 0; it < n_it; ++it) {
    const int st = it & 1;
    if (it + 1 < n_it) prefetch(it + 1, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    int j0;
    bool full;
    decode(it, j0, full);
    const uint16_t* Kt = Ks + st * BC * LD;
    const uint16_t* Vt = Vs + st * BC * LD;

    float s[NK][4], dp[NK][4];
#pragma unroll
    for (int n = 0; n < NK; ++n)
#pragma unroll
      for (int c = 0; c < 4; ++c) s[n][c] = dp[n][c] = 0.f;
    {
      // B operands: K / V rows (n = key, k = d)
      const int row = (lane & 7) + 8 * (lane >> 4);
      const int col = 8 * ((lane >> 3) & 1);
#pragma unroll
      for (int kk = 0; kk < KT; ++kk) {
#pragma unroll
        for (int n2 = 0; n2 < NK / 2; ++n2) {
          uint32_t bk[4], bv[4];
          ldsm_x4(bk, smem_addr(Kt + (n2 * 16 + row) * LD + kk * 16 + col));
          ldsm_x4(bv, smem_addr(Vt + (n2 * 16 + row) * LD + kk * 16 + col));
          mma16816<BF>(s[2 * n2], qf[kk], bk[0], bk[1]);
          mma16816<BF>(s[2 * n2 + 1], qf[kk], bk[2], bk[3]);
          mma16816<BF>(dp[2 * n2], gf[kk], bv[0], bv[1]);
          mma16816<BF>(dp[2 * n2 + 1], gf[kk], bv[2], bv[3]);
        }
      }
    }
#pragma unroll
    for (int n = 0; n < NK; ++n) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int h = c >> 1;
        const int i = qr0 + 8 * h, j = j0 + n * 8 + 2 * tq + (c & 1);
        float pij, dsij;
        pair_grads(p, s[n][c], dp[n][c], l2[h], dl[h], pij, dsij);
        bool keep = j < p.S;
        if (!full) keep = keep && i < p.L && pair_live(p, i, j);
        dp[n][c] = keep ? dsij : 0.f;
      }
    }
    // dQ += dS K: B operand K (k = key, n = d) by transposed loads
    {
      const int row = (lane & 7) + 8 * ((lane >> 3) & 1);
      const int col = 8 * (lane >> 4);
#pragma unroll
      for (int kq = 0; kq < BC / 16; ++kq) {
        const uint32_t ad[4] = {pack16<BF>(dp[2 * kq][0], dp[2 * kq][1]),
                                pack16<BF>(dp[2 * kq][2], dp[2 * kq][3]),
                                pack16<BF>(dp[2 * kq + 1][0], dp[2 * kq + 1][1]),
                                pack16<BF>(dp[2 * kq + 1][2], dp[2 * kq + 1][3])};
#pragma unroll
        for (int n2 = 0; n2 < ND / 2; ++n2) {
          uint32_t bk[4];
          ldsm_x4_trans(bk, smem_addr(Kt + (kq * 16 + row) * LD + n2 * 16 + col));
          mma16816<BF>(dq[2 * n2], ad, bk[0], bk[1]);
          mma16816<BF>(dq[2 * n2 + 1], ad, bk[2], bk[3]);
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();

  const bool bf16 = BF;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int i = qr0 + 8 * h;
    if (i >= p.L) continue;
    const int64_t off = (bh * p.L + i) * D + 2 * tq;
#pragma unroll
    for (int n = 0; n < ND; ++n)
      store_pair(p.dq + off + n * 8,
                 make_float2(dq[n][2 * h] * p.scale, dq[n][2 * h + 1] * p.scale), bf16);
  }
}

template <int D, bool BF>
fa_status bwd_launch(const BwdParams& prm, cudaStream_t s) {
  const int64_t rows = static_cast<int64_t>(prm.B) * prm.H * prm.L;
  const int64_t krows = static_cast<int64_t>(prm.B) * prm.Hkv * prm.S;
  const unsigned threads = kBwdWarps * 32;
  if (rows > 0) {
    const unsigned qgrid = static_cast<unsigned>((rows + kBwdWarps - 1) / kBwdWarps);
    bwd_delta_kernel<D><<<qgrid, threads, 0, s>>>(prm);
    FA_CUDA_CHECK(cudaGetLastError());
    FA_CUDA_CHECK(cudaFuncSetAttribute(bwd_dq_mma_kernel<D, BF>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(DqTile<D>::kSmem)));
    const unsigned grid = static_cast<unsigned>(static_cast<int64_t>(prm.n_q) * prm.B * prm.H);
    bwd_dq_mma_kernel<D, BF><<<grid, threads, DqTile<D>::kSmem, s>>>(prm);
    FA_CUDA_CHECK(cudaGetLastError());
  }
  if (krows > 0) {
    FA_CUDA_CHECK(cudaFuncSetAttribute(bwd_dkdv_mma_kernel<D, BF>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(DkdvTile<D>::kSmem)));
    const unsigned grid = static_cast<unsigned>(static_cast<int64_t>(prm.n_kv) * prm.B * prm.Hkv);
    bwd_dkdv_mma_kernel<D, BF><<<grid, threads, DkdvTile<D>::kSmem, s>>>(prm);
    FA_CUDA_CHECK(cudaGetLastError());
  }
  return FA_OK;
}

}  // namespace
}  // namespace fa

extern "C" size_t fa_bwd_workspace_bytes(int32_t B, int32_t H, int32_t L) {
  if (B < 0 || H < 0 || L < 0) return 0;
  return static_cast<size_t>(B) * H * L * sizeof(float) + 256;
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
  if (bm->mask_batch > 1 || bm->mask_heads > 1) return FA_ERR_UNSUPPORTED;  // broadcast masks only
  if (D != 64 && D != 128) return FA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(B) * H * L == 0 && static_cast<int64_t>(B) * H_kv * S == 0) return FA_OK;
  if (static_cast<int64_t>(B) * H * L > (int64_t{1} << 33) ||
      static_cast<int64_t>(B) * H_kv * S > (int64_t{1} << 33))
    return FA_ERR_UNSUPPORTED;
  if (workspace == nullptr || workspace_bytes < fa_bwd_workspace_bytes(B, H, L))
    return FA_ERR_INVALID_ARG;
  const bool any_q = static_cast<int64_t>(B) * H * L > 0, any_k = static_cast<int64_t>(B) * H_kv * S > 0;
  if (any_q && (q == nullptr || out == nullptr || dout == nullptr || lse == nullptr || dq == nullptr))
    return FA_ERR_INVALID_ARG;
  if (any_k && (k == nullptr || v == nullptr || dk == nullptr || dv == nullptr))
    return FA_ERR_INVALID_ARG;
  if (bm->n_q_blocks > 0 && (bm->kv_num_blocks == nullptr || bm->full_kv_num_blocks == nullptr))
    return FA_ERR_INVALID_ARG;
  if (bm->n_q_blocks > 0 && bm->n_kv_blocks > 0 &&
      (bm->kv_indices == nullptr || bm->full_kv_indices == nullptr || q_num_blocks == nullptr ||
       q_indices == nullptr || full_q_num_blocks == nullptr || full_q_indices == nullptr))
    return FA_ERR_INVALID_ARG;
  if (bm->kind == FA_MASK_DOCUMENT_CAUSAL && bm->doc_id == nullptr) return FA_ERR_INVALID_ARG;
  if (bm->kind == FA_MASK_BITMAP && S > 0 && bm->bitmap == nullptr) return FA_ERR_INVALID_ARG;
  // q, k, v, dout are staged by 16-byte cp.async copies; the rest is accessed in
  // 4-byte pairs / floats
  auto off16 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) != 0; };
  auto off4 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 3u) != 0; };
  if (off16(q) || off16(k) || off16(v) || off16(dout) || off4(out) || off4(dq) || off4(dk) ||
      off4(dv) || off4(workspace) || off4(lse))
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
  prm.delta = static_cast<float*>(workspace);
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
  prm.softcap_on = score_kind == FA_SCORE_TANH_SOFTCAP ? 1 : 0;
  prm.is_bf16 = dtype == FA_BF16 ? 1 : 0;
  prm.scale = scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(D));
  prm.cap_c = prm.softcap_on ? softcap : 1.f;
  const cudaStream_t s = as_stream(stream);
  if (D == 64) return prm.is_bf16 ? bwd_launch<64, true>(prm, s) : bwd_launch<64, false>(prm, s);
  return prm.is_bf16 ? bwd_launch<128, true>(prm, s) : bwd_launch<128, false>(prm, s);
}
