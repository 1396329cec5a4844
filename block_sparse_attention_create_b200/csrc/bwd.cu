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
// One warp per query row for dQ and one warp per key row for dK / dV, so every
// output row is owned by one warp (no atomics); a lane holds pairs of columns
// 2 * lane + 64 e.  A first, CUDA-core implementation: correct for every mask
// family and grouped-query heads, not tuned.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "fa_internal.h"

namespace fa {
namespace {

constexpr int kBwdWarps = 8;
constexpr int kBwdBlock = FA_BLOCK;
constexpr float kBwdLog2e = 1.4426950408889634f;

struct BwdParams {
  const uint16_t *q, *k, *v, *out, *dout;
  const float* lse;
  float* delta;
  uint16_t *dq, *dk, *dv;
  const int32_t *kv_num, *kv_idx, *full_num, *full_idx;      // row lists
  const int32_t *q_num, *q_idx, *full_q_num, *full_q_idx;   // column lists
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

// dQ: warp per query row (b, h, i), over the kv blocks of its q-block row.
template <int D>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_dq_kernel(const BwdParams p) {
  constexpr int E = D / 64;  // column pairs per lane
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kBwdWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= static_cast<int64_t>(p.B) * p.H * p.L) return;
  const bool bf16 = p.is_bf16 != 0;
  const int64_t bh = row / p.L;
  const int i = static_cast<int>(row - bh * p.L);
  const int64_t kvbh = (bh / p.H) * p.Hkv + (bh % p.H) / p.G;
  float2 q[E], g[E], dq[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int64_t off = row * D + 2 * lane + 64 * e;
    q[e] = load_pair(p.q + off, bf16);
    g[e] = load_pair(p.dout + off, bf16);
    dq[e] = make_float2(0.f, 0.f);
  }
  const float lse = p.lse[row];
  if (lse != -INFINITY) {  // a row with no live key has no gradient
    const float lse2 = lse * kBwdLog2e, delta = p.delta[row];
    const int qb = i / kBwdBlock;
    const int np = __ldg(p.kv_num + qb), nf = __ldg(p.full_num + qb);
    for (int t = 0; t < np + nf; ++t) {
      const bool full = t >= np;
      const int jb = full ? __ldg(p.full_idx + static_cast<size_t>(qb) * p.n_kv + (t - np))
                          : __ldg(p.kv_idx + static_cast<size_t>(qb) * p.n_kv + t);
      const int j1 = min(p.S, (jb + 1) * kBwdBlock);
      for (int j = jb * kBwdBlock; j < j1; ++j) {
        if (!full && !pair_live(p, i, j)) continue;  // uniform across the warp
        const int64_t koff = (kvbh * p.S + j) * D + 2 * lane;
        float2 kk[E];
        float qk = 0.f, dov = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          kk[e] = load_pair(p.k + koff + 64 * e, bf16);
          const float2 vv = load_pair(p.v + koff + 64 * e, bf16);
          qk = fmaf(q[e].x, kk[e].x, fmaf(q[e].y, kk[e].y, qk));
          dov = fmaf(g[e].x, vv.x, fmaf(g[e].y, vv.y, dov));
        }
        qk = warp_sum(qk);
        dov = warp_sum(dov);
        float pij, dsij;
        pair_grads(p, qk, dov, lse2, delta, pij, dsij);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          dq[e].x = fmaf(dsij, kk[e].x, dq[e].x);
          dq[e].y = fmaf(dsij, kk[e].y, dq[e].y);
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e)
    store_pair(p.dq + row * D + 2 * lane + 64 * e,
               make_float2(dq[e].x * p.scale, dq[e].y * p.scale), bf16);
}

// dK, dV: warp per key row (b, kv head, j), over the query heads that share the
// K/V head and the q blocks of its kv-block column.
template <int D>
__global__ void __launch_bounds__(kBwdWarps * 32) bwd_dkdv_kernel(const BwdParams p) {
  constexpr int E = D / 64;
  const int64_t krow = static_cast<int64_t>(blockIdx.x) * kBwdWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (krow >= static_cast<int64_t>(p.B) * p.Hkv * p.S) return;
  const bool bf16 = p.is_bf16 != 0;
  const int64_t kvbh = krow / p.S;
  const int j = static_cast<int>(krow - kvbh * p.S);
  const int64_t b = kvbh / p.Hkv, kvh = kvbh - b * p.Hkv;
  float2 kk[E], vv[E], dk[E], dv[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int64_t off = krow * D + 2 * lane + 64 * e;
    kk[e] = load_pair(p.k + off, bf16);
    vv[e] = load_pair(p.v + off, bf16);
    dk[e] = dv[e] = make_float2(0.f, 0.f);
  }
  const int jb = j / kBwdBlock;
  // no query rows (L == 0): no column lists were built, and no gradient flows
  const int np = p.n_q > 0 ? __ldg(p.q_num + jb) : 0;
  const int nf = p.n_q > 0 ? __ldg(p.full_q_num + jb) : 0;
  for (int g = 0; g < p.G; ++g) {
    const int64_t bh = b * p.H + kvh * p.G + g;
    for (int t = 0; t < np + nf; ++t) {
      const bool full = t >= np;
      const int ib = full ? __ldg(p.full_q_idx + static_cast<size_t>(jb) * p.n_q + (t - np))
                          : __ldg(p.q_idx + static_cast<size_t>(jb) * p.n_q + t);
      const int i1 = min(p.L, (ib + 1) * kBwdBlock);
      for (int i = ib * kBwdBlock; i < i1; ++i) {
        if (!full && !pair_live(p, i, j)) continue;
        const int64_t row = bh * p.L + i;
        const float lse = p.lse[row];
        if (lse == -INFINITY) continue;
        const int64_t qoff = row * D + 2 * lane;
        float2 q[E], go[E];
        float qk = 0.f, dov = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          q[e] = load_pair(p.q + qoff + 64 * e, bf16);
          go[e] = load_pair(p.dout + qoff + 64 * e, bf16);
          qk = fmaf(q[e].x, kk[e].x, fmaf(q[e].y, kk[e].y, qk));
          dov = fmaf(go[e].x, vv[e].x, fmaf(go[e].y, vv[e].y, dov));
        }
        qk = warp_sum(qk);
        dov = warp_sum(dov);
        float pij, dsij;
        pair_grads(p, qk, dov, lse * kBwdLog2e, p.delta[row], pij, dsij);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          dv[e].x = fmaf(pij, go[e].x, dv[e].x);
          dv[e].y = fmaf(pij, go[e].y, dv[e].y);
          dk[e].x = fmaf(dsij, q[e].x, dk[e].x);
          dk[e].y = fmaf(dsij, q[e].y, dk[e].y);
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int64_t off = krow * D + 2 * lane + 64 * e;
    store_pair(p.dk + off, make_float2(dk[e].x * p.scale, dk[e].y * p.scale), bf16);
    store_pair(p.dv + off, dv[e], bf16);
  }
}

template <int D>
fa_status bwd_launch(const BwdParams& prm, cudaStream_t s) {
  const int64_t rows = static_cast<int64_t>(prm.B) * prm.H * prm.L;
  const int64_t krows = static_cast<int64_t>(prm.B) * prm.Hkv * prm.S;
  const unsigned threads = kBwdWarps * 32;
  if (rows > 0) {
    const unsigned qgrid = static_cast<unsigned>((rows + kBwdWarps - 1) / kBwdWarps);
    bwd_delta_kernel<D><<<qgrid, threads, 0, s>>>(prm);
    FA_CUDA_CHECK(cudaGetLastError());
    bwd_dq_kernel<D><<<qgrid, threads, 0, s>>>(prm);
    FA_CUDA_CHECK(cudaGetLastError());
  }
  if (krows > 0) {
    const unsigned kgrid = static_cast<unsigned>((krows + kBwdWarps - 1) / kBwdWarps);
    bwd_dkdv_kernel<D><<<kgrid, threads, 0, s>>>(prm);
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
  auto misaligned = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 3u) != 0; };
  if (misaligned(q) || misaligned(k) || misaligned(v) || misaligned(out) || misaligned(dout) ||
      misaligned(dq) || misaligned(dk) || misaligned(dv) || misaligned(workspace))
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
  if (D == 64) return bwd_launch<64>(prm, s);
  return bwd_launch<128>(prm, s);
}
