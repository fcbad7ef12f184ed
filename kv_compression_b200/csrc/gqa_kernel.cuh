// gqa_kernel.cuh -- LCA decode for grouped-query attention (GQA) on CUDA cores,
// fp32 accumulation.
//
// "Latent-Condensed Transformer for Efficient Long Context Modeling",
// section 2, "Condensacao Dual-Path" (the semantic component is pooled with
// the query-aware group softmax, the positional component is taken from the
// top-scoring token), extended to GQA as section 3, item 3 allows.  In a GQA
// cache the key carries the position (RoPE) and the value the content, so for
// each query head and each group G_j of the section-2 segmentation:
//   s_t = q . k_t,  w_t = softmax_{t in G_j}(s_t),  a_j = lowest-index argmax,
//   condensed entry: key k_{a_j} (logit s_{a_j} = max_{G_j} s), value sum_t w_t v_t;
// window tokens stand for themselves, and attention runs over
// [condensed || window].  As an online softmax over tokens: a grouped token
// weighs e^{S_j - M} w_t = e^{s_t - M} / den_j (S_j = m_j), a window token
// e^{s_t - M}; O = sum_t P_t v_t.
//
// One CTA per (context split, KV head, sequence) serves the r = H / H_kv query
// heads that share the KV head, so each K and V row is read from HBM once per
// step.  With r <= 16 heads the score block is r x tile, too thin a contraction
// for the tensor cores; several CTAs per SM hide the load latency.  Per tile:
//   load      the tile's K and V rows of this KV head into shared memory,
//             16-byte vector loads (the cache is [B][L][H_kv][d], rows strided)
//   scores    one warp per token, lanes over dims, r warp sums
//   condense  one thread per (head, group): max, anchor, den, in-group weights
//   max       one warp per head: the tile's largest entry, the rescale factor
//   weights   one thread per (head, token); Z by one warp per head
//   O         one thread per (head, value dim): O = O alpha + sum_t P_t v_t
// The split partial (M, Z, O) of each head is merged by the combine kernel.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "checks.cuh"

namespace lca {

constexpr int kGqaThreads = 256;
constexpr int kGqaWarps = kGqaThreads / 32;
constexpr int kGqaMaxR = 16;        // query heads per KV head
constexpr int kGqaMaxD = 256;       // d_k and d_v
constexpr int kGqaMaxOut = kGqaMaxR * kGqaMaxD / kGqaThreads;   // O values per thread

struct GqaParams {
  const void* q;     // [B][H][d_k]
  const void* k;     // [B][L][H_kv][d_k]
  const void* v;     // [B][L][H_kv][d_v]
  int B, H, H_kv, r, d_k, d_v;
  int64_t L;
  int g;             // group size (1 when nG == 0)
  int64_t nG;
  int64_t win0;      // first window token: n_G g
  int64_t split_len; // tokens per split (a multiple of g)
  int tile;          // tokens per tile (a multiple of g)
  int n_split;
  int32_t* anchor;   // [B][H][nG] or null when nG == 0
  float* part_o;     // [B * n_split][H][d_v]
  float* part_mz;    // [B * n_split][H][2]
  int64_t ws_slots;
  int* err;
};

template <typename T>
__device__ __forceinline__ float gqa_elem(const T* p);
template <>
__device__ __forceinline__ float gqa_elem<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float gqa_elem<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

// Shared memory of one CTA (floats unless noted): q [r][d_k] | s [r][tile] |
// pw [r][tile] | glog [r][tile] | M, Z, alpha [r] each | K tile [tile][d_k] T |
// V tile [tile][d_v] T.
__host__ __device__ inline size_t gqa_smem_bytes(int r, int d_k, int d_v, int tile, int elem) {
  const size_t f = (size_t)r * d_k + 3 * (size_t)r * tile + 3 * (size_t)r;
  const size_t fb = (f * 4 + 15) / 16 * 16;
  return fb + (size_t)tile * (d_k + d_v) * elem;
}

__device__ __forceinline__ float gqa_warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float gqa_warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

template <typename T>
__global__ void __launch_bounds__(kGqaThreads) lca_gqa_kernel(const GqaParams p) {
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = p.r, d_k = p.d_k, d_v = p.d_v, tile = p.tile;
  extern __shared__ __align__(16) uint8_t gsm[];
  float* qs = reinterpret_cast<float*>(gsm);          // [r][d_k]
  float* s = qs + r * d_k;                            // [r][tile]
  float* pw = s + r * tile;                           // [r][tile]
  float* glog = pw + r * tile;                        // [r][tile]
  float* Ms = glog + r * tile;                        // [r]
  float* Zs = Ms + r;                                 // [r]
  float* As = Zs + r;                                 // [r]
  const size_t fbytes = (((size_t)r * d_k + 3 * (size_t)r * tile + 3 * (size_t)r) * 4 + 15) / 16 * 16;
  T* ks = reinterpret_cast<T*>(gsm + fbytes);         // [tile][d_k]
  T* vs = ks + (size_t)tile * d_k;                    // [tile][d_v]

  const int h0 = kvh * r;
  const T* qg = static_cast<const T*>(p.q) + ((int64_t)b * p.H + h0) * d_k;
  for (int i = tid; i < r * d_k; i += kGqaThreads) qs[i] = gqa_elem(qg + i);
  if (tid < r) { Ms[tid] = -INFINITY; Zs[tid] = 0.f; }

  const int64_t s0 = (int64_t)split * p.split_len;
  const int64_t s1 = (p.L < s0 + p.split_len) ? p.L : s0 + p.split_len;
  const int64_t row_stride = (int64_t)p.H_kv;          // rows of one KV head are H_kv rows apart
  const T* kg = static_cast<const T*>(p.k) + ((int64_t)b * p.L * row_stride + kvh) * d_k;
  const T* vg = static_cast<const T*>(p.v) + ((int64_t)b * p.L * row_stride + kvh) * d_v;
  constexpr int kVec = 16 / sizeof(T);                // elements per 16-byte load

  float o[kGqaMaxOut];
#pragma unroll
  for (int k = 0; k < kGqaMaxOut; ++k) o[k] = 0.f;
  __syncthreads();

  for (int64_t t0 = s0; t0 < s1; t0 += tile) {
    const int n = (int)((int64_t)tile < s1 - t0 ? (int64_t)tile : s1 - t0);
    // ---- load the tile's K and V rows of this KV head
    {
      const int kc = d_k / kVec, vc = d_v / kVec;
      for (int i = tid; i < n * kc; i += kGqaThreads) {
        const int tt = i / kc, c = i - tt * kc;
        *reinterpret_cast<uint4*>(ks + (size_t)tt * d_k + c * kVec) =
            __ldg(reinterpret_cast<const uint4*>(kg + (t0 + tt) * row_stride * d_k) + c);
      }
      for (int i = tid; i < n * vc; i += kGqaThreads) {
        const int tt = i / vc, c = i - tt * vc;
        *reinterpret_cast<uint4*>(vs + (size_t)tt * d_v + c * kVec) =
            __ldg(reinterpret_cast<const uint4*>(vg + (t0 + tt) * row_stride * d_v) + c);
      }
    }
    __syncthreads();
    // ---- scores: one warp per token, lanes over dims, every head of the KV head
    for (int tt = warp; tt < n; tt += kGqaWarps) {
      float acc[kGqaMaxR];
#pragma unroll
      for (int h = 0; h < kGqaMaxR; ++h) acc[h] = 0.f;
      const T* krow = ks + (size_t)tt * d_k;
      for (int d = lane; d < d_k; d += 32) {
        const float kv = gqa_elem(krow + d);
#pragma unroll
        for (int h = 0; h < kGqaMaxR; ++h)
          if (h < r) acc[h] = fmaf(qs[h * d_k + d], kv, acc[h]);
      }
#pragma unroll
      for (int h = 0; h < kGqaMaxR; ++h) {
        if (h < r) {
          const float v = gqa_warp_sum(acc[h]);
          if (lane == 0) s[h * tile + tt] = v;
        }
      }
    }
    __syncthreads();
    // ---- condense: one thread per (head, group start); the group's logit is its max
    for (int i = tid; i < r * n; i += kGqaThreads) {
      const int h = i / n, tt = i - h * n;
      const int64_t t = t0 + tt;
      if (t < p.win0 && (t % p.g) == 0 && LCA_CHECK(p.err, tt + p.g <= tile, 0xC21)) {
        const float* sh = s + h * tile;
        float m = sh[tt];
        int amax = tt;
        for (int u = tt + 1; u < tt + p.g; ++u)
          if (sh[u] > m) { m = sh[u]; amax = u; }   // strict: the lowest index keeps a tie
        float den = 0.f;
        for (int u = tt; u < tt + p.g; ++u) den += expf(sh[u] - m);
        const float inv = 1.f / den;
        for (int u = tt; u < tt + p.g; ++u) pw[h * tile + u] = expf(sh[u] - m) * inv;   // w_t
        glog[h * tile + tt] = m;
        if (LCA_CHECK(p.err, t / p.g < p.nG, 0xC22))
          p.anchor[((int64_t)b * p.H + h0 + h) * p.nG + t / p.g] = (int32_t)(t0 + amax);
      }
    }
    __syncthreads();
    // ---- the tile's largest entry per head (one warp per head) and the rescale factor
    for (int h = warp; h < r; h += kGqaWarps) {
      float mx = -INFINITY;
      for (int tt = lane; tt < n; tt += 32) {
        const int64_t t = t0 + tt;
        if (t < p.win0) {
          if ((t % p.g) == 0) mx = fmaxf(mx, glog[h * tile + tt]);
        } else {
          mx = fmaxf(mx, s[h * tile + tt]);
        }
      }
      mx = gqa_warp_max(mx);
      if (lane == 0) {
        const float Mn = fmaxf(Ms[h], mx);
        As[h] = expf(Ms[h] - Mn);    // 0 on the first tile (M = -inf)
        Ms[h] = Mn;
      }
    }
    __syncthreads();
    // ---- per-token weights
    for (int i = tid; i < r * n; i += kGqaThreads) {
      const int h = i / n, tt = i - h * n;
      const int64_t t = t0 + tt;
      float wgt;
      if (t < p.win0) {
        const int gs = tt - (int)(t % p.g);           // the group's start within the tile
        wgt = expf(glog[h * tile + gs] - Ms[h]) * pw[h * tile + tt];
      } else {
        wgt = expf(s[h * tile + tt] - Ms[h]);
      }
      pw[h * tile + tt] = wgt;
    }
    __syncthreads();
    // ---- Z: one warp per head
    for (int h = warp; h < r; h += kGqaWarps) {
      float z = 0.f;
      for (int tt = lane; tt < n; tt += 32) z += pw[h * tile + tt];
      z = gqa_warp_sum(z);
      if (lane == 0) Zs[h] = Zs[h] * As[h] + z;
    }
    // ---- O = O alpha + sum_t P_t v_t, one thread per (head, value dim)
#pragma unroll
    for (int k = 0; k < kGqaMaxOut; ++k) {
      const int idx = tid + k * kGqaThreads;
      if (idx < r * d_v) {
        const int h = idx / d_v, d = idx - h * d_v;
        float acc = o[k] * As[h];
        const float* ph = pw + h * tile;
        for (int tt = 0; tt < n; ++tt) acc = fmaf(ph[tt], gqa_elem(vs + (size_t)tt * d_v + d), acc);
        o[k] = acc;
      }
    }
    __syncthreads();
  }

  const int64_t slot = (int64_t)b * p.n_split + split;
  if (!LCA_CHECK(p.err, slot < p.ws_slots, 0xC23)) return;
#pragma unroll
  for (int k = 0; k < kGqaMaxOut; ++k) {
    const int idx = tid + k * kGqaThreads;
    if (idx < r * d_v) {
      const int h = idx / d_v, d = idx - h * d_v;
      p.part_o[(slot * p.H + h0 + h) * (int64_t)d_v + d] = o[k];
    }
  }
  if (tid < r) {
    p.part_mz[(slot * p.H + h0 + tid) * 2 + 0] = Ms[tid];
    p.part_mz[(slot * p.H + h0 + tid) * 2 + 1] = Zs[tid];
  }
}

}  // namespace lca
