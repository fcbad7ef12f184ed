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
//   condensed entry: key k_{a_j} (logit s_{a_j} = m_j = max_{G_j} s), value sum_t w_t v_t;
// window tokens stand for themselves, and attention runs over
// [condensed || window].  As an online softmax over tokens: a grouped token
// weighs e^{m_j - M} w_t = e^{s_t - M} / den_j (den_j = sum_{G_j} e^{s_t - m_j}),
// a window token e^{s_t - M}; the group adds e^{m_j - M} to Z; O = sum_t P_t v_t.
//
// One CTA per (context split, KV head, sequence) serves the r = H / H_kv query
// heads that share the KV head, so each K and V row is read from HBM once per
// step.  With r <= 16 heads the score block is r x 64, too thin a contraction
// for the tensor cores.  Per 64-token tile:
//   load      the next tile's K and V rows of this KV head stream into the other
//             shared-memory buffer (cp.async, 16 bytes a copy) while this one is
//             used; K rows are padded by 16 bytes so the score reads are
//             conflict-free
//   scores    one lane per token (warps 2 i and 2 i + 1 take the tile's two halves
//             for heads i, i + 4, i + 8, i + 12): 16-byte row loads, the heads'
//             q read as broadcast float4, no reduction
//   condense  one thread per (head, token), the heads' 64 tokens in two
//             consecutive warps, so a group of g <= 32 tokens is g neighbouring
//             lanes: butterfly max and sum, ballot for the lowest-index argmax
//             (a 64-token group joins its two warps through shared memory)
//   max, Z    warp reductions per (head, half tile), combined by one thread per head
//   O         one thread per (slice of the tile's tokens, pair of value dims), for all
//             r heads: each V element is read from shared memory once and used r
//             times; the slices' partial sums are added once, at the end
// The number of heads a lane or thread serves, SLOTS = ceil(r / 4), is a template
// parameter, so no work is issued for head slots beyond r; the dot products and O
// run on packed fp32 pairs (two multiply-adds per instruction).
// The split partial (M, Z, O) of each head is merged by the combine kernel.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "checks.cuh"
#include "ptx.cuh"

namespace lca {

constexpr int kGqaThreads = 256;
constexpr int kGqaWarps = kGqaThreads / 32;
constexpr int kGqaTile = 64;                                        // tokens per tile
constexpr int kGqaMaxR = 16;                                        // query heads per KV head
constexpr int kGqaMaxD = 256;                                       // d_k and d_v

struct GqaParams {
  const void* q;     // [B][H][d_k]
  const void* k;     // [B][L][H_kv][d_k]
  const void* v;     // [B][L][H_kv][d_v]
  int B, H, H_kv, r, d_k, d_v;
  int64_t L;
  int g;             // group size, a power of two <= 64 (1 when nG == 0)
  int64_t nG;
  int64_t win0;      // first window token: n_G g
  int64_t split_len; // tokens per split (a multiple of 64)
  int n_split;
  int32_t* anchor;   // [B][H][nG] or null when nG == 0
  float* part_o;     // [B * n_split][H][d_v]
  float* part_mz;    // [B * n_split][H][2]
  int64_t ws_slots;
  int* err;
};

// Elements of one 16-byte copy, and a K row's stride in shared memory (16 bytes of padding).
template <typename T>
__host__ __device__ constexpr int gqa_vec() { return 16 / (int)sizeof(T); }
template <typename T>
__host__ __device__ inline int gqa_kstride(int d_k) { return d_k + gqa_vec<T>(); }

// Shared memory (floats first): q [r][d_k] | s [r][64] | pw [r][64] | wpart, zpart
// [r][2] | gstat [r][2][4] | M, Z, alpha [r] | then two buffers of K [64][kstride]
// and V [64][d_v] elements.
__host__ __device__ inline size_t gqa_float_bytes(int r, int d_k) {
  const size_t f = (size_t)r * d_k + 2 * (size_t)r * kGqaTile + 4 * (size_t)r + 8 * (size_t)r + 3 * (size_t)r;
  return (f * 4 + 15) / 16 * 16;
}
template <typename T>
__host__ __device__ inline size_t gqa_smem_bytes(int r, int d_k, int d_v) {
  // the tile buffers, which at the end also hold the token slices' partial O
  // (512 r floats: (256 / (d_v / 2)) slices x r heads x d_v)
  const size_t tiles = 2 * (size_t)kGqaTile * (gqa_kstride<T>(d_k) + d_v) * sizeof(T);
  const size_t red = 512 * (size_t)r * sizeof(float);
  return gqa_float_bytes(r, d_k) + (tiles > red ? tiles : red);
}

__device__ __forceinline__ void gqa_cp_async16(void* smem_dst, const void* gmem_src) {
  const uint32_t d = static_cast<uint32_t>(__cvta_generic_to_shared(smem_dst));
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gmem_src) : "memory");
}
__device__ __forceinline__ void gqa_cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void gqa_cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

template <typename T>
__device__ __forceinline__ void gqa_unpack(const uint4& raw, float* f);
template <>
__device__ __forceinline__ void gqa_unpack<float>(const uint4& raw, float* f) {
  f[0] = __uint_as_float(raw.x); f[1] = __uint_as_float(raw.y);
  f[2] = __uint_as_float(raw.z); f[3] = __uint_as_float(raw.w);
}
template <>
__device__ __forceinline__ void gqa_unpack<__nv_bfloat16>(const uint4& raw, float* f) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}
// two consecutive elements (an even index: 4- or 8-byte aligned) as floats
template <typename T>
__device__ __forceinline__ void gqa_pair(const T* p, float& a, float& b);
template <>
__device__ __forceinline__ void gqa_pair<float>(const float* p, float& a, float& b) {
  const float2 v = *reinterpret_cast<const float2*>(p);
  a = v.x;
  b = v.y;
}
template <>
__device__ __forceinline__ void gqa_pair<__nv_bfloat16>(const __nv_bfloat16* p, float& a, float& b) {
  const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
  a = __uint_as_float(u << 16);
  b = __uint_as_float(u & 0xffff0000u);
}
template <typename T>
__device__ __forceinline__ float gqa_elem(const T* p);
template <>
__device__ __forceinline__ float gqa_elem<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float gqa_elem<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

template <typename T, int SLOTS>
__global__ void __launch_bounds__(kGqaThreads, 3) lca_gqa_kernel(const GqaParams p) {
  static_assert(SLOTS >= 1 && 4 * SLOTS <= kGqaMaxR, "head slots");
  constexpr int kVec = gqa_vec<T>();
  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int r = p.r, d_k = p.d_k, d_v = p.d_v, g = p.g;
  const int kstride = gqa_kstride<T>(d_k);
  extern __shared__ __align__(16) uint8_t gsm[];
  float* qs = reinterpret_cast<float*>(gsm);          // [r][d_k]
  float* s = qs + r * d_k;                            // [r][64] scores
  float* pw = s + r * kGqaTile;                       // [r][64] token weights
  float* wpart = pw + r * kGqaTile;                   // [r][2] half-tile maxima
  float* zpart = wpart + 2 * r;                       // [r][2] half-tile weight sums
  float* gstat = zpart + 2 * r;                       // [r][2][4] half-group m, den, anchor (64-token groups)
  float* Ms = gstat + 8 * r;
  float* Zs = Ms + r;
  float* As = Zs + r;
  T* kbuf = reinterpret_cast<T*>(gsm + gqa_float_bytes(r, d_k));   // [2][64][kstride]
  T* vbuf = kbuf + 2 * kGqaTile * kstride;                          // [2][64][d_v]

  const int h0 = kvh * r;
  const T* qg = static_cast<const T*>(p.q) + ((int64_t)b * p.H + h0) * d_k;
  for (int i = tid; i < r * d_k; i += kGqaThreads) qs[i] = gqa_elem(qg + i);
  if (tid < r) { Ms[tid] = -INFINITY; Zs[tid] = 0.f; }

  const int64_t s0 = (int64_t)split * p.split_len;
  const int64_t s1 = (p.L < s0 + p.split_len) ? p.L : s0 + p.split_len;
  const int64_t rs = p.H_kv;                           // a KV head's rows are H_kv rows apart
  const T* kg = static_cast<const T*>(p.k) + ((int64_t)b * p.L * rs + kvh) * d_k;
  const T* vg = static_cast<const T*>(p.v) + ((int64_t)b * p.L * rs + kvh) * d_v;

  // this thread's first (row, chunk) of the K and V copies; later ones step by
  // 256 chunks (the divisions are done once)
  const int kc = d_k / kVec, vc = d_v / kVec;
  const int k_row0 = tid / kc, k_c0 = tid - k_row0 * kc;
  const int v_row0 = tid / vc, v_c0 = tid - v_row0 * vc;
  const int k_rstep = kGqaThreads / kc, k_cstep = kGqaThreads - k_rstep * kc;
  const int v_rstep = kGqaThreads / vc, v_cstep = kGqaThreads - v_rstep * vc;
  auto issue = [&](int64_t t0, int bf) {
    const int n = (int)(s1 - t0 < kGqaTile ? s1 - t0 : kGqaTile);
    T* kd = kbuf + bf * kGqaTile * kstride;
    T* vd = vbuf + bf * kGqaTile * d_v;
    const T* ks = kg + t0 * rs * d_k;
    const T* vs = vg + t0 * rs * d_v;
    for (int tt = k_row0, c = k_c0; tt < n;) {
      gqa_cp_async16(kd + tt * kstride + c * kVec, ks + (int64_t)tt * rs * d_k + c * kVec);
      tt += k_rstep;
      c += k_cstep;
      if (c >= kc) { c -= kc; ++tt; }
    }
    for (int tt = v_row0, c = v_c0; tt < n;) {
      gqa_cp_async16(vd + tt * d_v + c * kVec, vs + (int64_t)tt * rs * d_v + c * kVec);
      tt += v_rstep;
      c += v_cstep;
      if (c >= vc) { c -= vc; ++tt; }
    }
    gqa_cp_commit();
  };

  // O: thread = (token slice tg, value-dim pair dp), all r heads; d_v / 2 is a power
  // of two in [16, 128], so there are 256 / (d_v / 2) slices of d_v / 8 tokens
  const int npairs = d_v / 2;
  const int lg_np = __ffs(npairs) - 1;
  const int dp = tid & (npairs - 1), tg = tid >> lg_np;
  const int tpg = npairs >> 2;                        // tokens per slice, a multiple of 4
  float o0[4 * SLOTS], o1[4 * SLOTS];
#pragma unroll
  for (int h = 0; h < 4 * SLOTS; ++h) { o0[h] = 0.f; o1[h] = 0.f; }
  if (s0 < s1) issue(s0, 0);
  __syncthreads();

  int bf = 0;
  for (int64_t t0 = s0; t0 < s1; t0 += kGqaTile, bf ^= 1) {
    const int n = (int)(s1 - t0 < kGqaTile ? s1 - t0 : kGqaTile);
    if (t0 + kGqaTile < s1) {
      issue(t0 + kGqaTile, bf ^ 1);
      gqa_cp_wait<1>();
    } else {
      gqa_cp_wait<0>();
    }
    __syncthreads();
    const T* kb = kbuf + bf * kGqaTile * kstride;
    const T* vb = vbuf + bf * kGqaTile * d_v;

    // ---- scores: lane = token of the warp's half tile, heads hg, hg + 4, ...
    {
      const int hg = warp >> 1;
      const int tt = (warp & 1) * 32 + lane;
      uint64_t acc[SLOTS];   // packed (even dims, odd dims) partial sums
#pragma unroll
      for (int i = 0; i < SLOTS; ++i) acc[i] = ptx::f32x2(0.f, 0.f);
      if (tt < n) {
        const T* krow = kb + tt * kstride;
        for (int c = 0; c < d_k; c += kVec) {
          float kf[kVec];
          gqa_unpack<T>(*reinterpret_cast<const uint4*>(krow + c), kf);
          uint64_t k2[kVec / 2];
#pragma unroll
          for (int e = 0; e < kVec / 2; ++e) k2[e] = ptx::f32x2(kf[2 * e], kf[2 * e + 1]);
#pragma unroll
          for (int i = 0; i < SLOTS; ++i) {
            const int h = hg + 4 * i;
            if (h < r) {
              const float4* qv = reinterpret_cast<const float4*>(qs + h * d_k + c);
#pragma unroll
              for (int e = 0; e < kVec / 4; ++e) {
                const float4 q4 = qv[e];
                acc[i] = ptx::fma_f32x2(ptx::f32x2(q4.x, q4.y), k2[2 * e], acc[i]);
                acc[i] = ptx::fma_f32x2(ptx::f32x2(q4.z, q4.w), k2[2 * e + 1], acc[i]);
              }
            }
          }
        }
#pragma unroll
        for (int i = 0; i < SLOTS; ++i) {
          if (hg + 4 * i < r) {
            float a0, a1;
            ptx::f32x2_split(acc[i], a0, a1);
            s[(hg + 4 * i) * kGqaTile + tt] = a0 + a1;
          }
        }
      }
    }
    __syncthreads();

    // ---- condense and the tile's entries: thread per (head, token)
    const bool tile_groups = t0 < p.win0;               // tile-uniform (g = 1 included)
    float sv[SLOTS], dn[SLOTS];
    bool gr[SLOTS];
#pragma unroll
    for (int k = 0; k < SLOTS; ++k) {
      const int idx = tid + k * kGqaThreads;
      const bool active = idx < r * kGqaTile;           // warp-uniform (r * 64 is a multiple of 32)
      const int h = idx >> 6, tt = idx & (kGqaTile - 1);
      const int64_t t = t0 + tt;
      const bool valid = active && tt < n;
      sv[k] = valid ? s[h * kGqaTile + tt] : -INFINITY;
      gr[k] = valid && t < p.win0;
      dn[k] = 1.f;
      float ent = gr[k] ? -INFINITY : sv[k];             // a window token is its own entry
      if (tile_groups) {
        // groups are aligned to g and the window starts on a group boundary, so a
        // group's lanes agree on gr; an invalid lane is never in a valid group
        const int W = g < 32 ? g : 32;
        float m = sv[k];
        for (int off = 1; off < W; off <<= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        const int base = lane & ~(W - 1);
        const uint32_t gmask = W == 32 ? 0xffffffffu : (((1u << W) - 1u) << base);
        const uint32_t ties = __ballot_sync(0xffffffffu, sv[k] == m) & gmask;
        int a = __ffs(ties) - 1 - base;                  // lowest index among the maxima
        float den = gr[k] ? expf(sv[k] - m) : 0.f;
        for (int off = 1; off < W; off <<= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
        if (g > 32) {
          // a 64-token group: the head's two warps meet in shared memory (warp half 0 first,
          // so both form the same bits and a tie keeps half 0's anchor)
          const int half = tt >> 5;
          if (active && lane == 0) {
            float* gs = gstat + (h * 2 + half) * 4;
            gs[0] = m; gs[1] = den; gs[2] = __int_as_float(a + 32 * half);
          }
          __syncthreads();
          if (active) {
            const float* g0 = gstat + h * 8;
            const float m0 = g0[0], m1 = g0[4];
            const float mm = fmaxf(m0, m1);
            const float f0 = m0 == -INFINITY ? 0.f : expf(m0 - mm), f1 = m1 == -INFINITY ? 0.f : expf(m1 - mm);
            const float den2 = g0[1] * f0 + g0[5] * f1;
            a = m1 > m0 ? __float_as_int(g0[6]) : __float_as_int(g0[2]);
            den = den2;
            m = mm;
          }
          __syncthreads();
        }
        dn[k] = den;
        if (gr[k]) {
          const bool leader = (tt & (g - 1)) == 0;
          if (leader) {
            ent = m;                                     // the condensed logit s_{a_j} = m_j
            if (LCA_CHECK(p.err, t / g < p.nG && a >= 0 && a < g, 0xC21))
              p.anchor[((int64_t)b * p.H + h0 + h) * p.nG + t / g] = (int32_t)(t + a);
          }
        }
      }
      // the tile's largest entry per (head, half tile)
      float mx = ent;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      if (active && lane == 0) wpart[h * 2 + (tt >> 5)] = mx;
    }
    __syncthreads();
    if (tid < r) {
      const float Mn = fmaxf(Ms[tid], fmaxf(wpart[2 * tid], wpart[2 * tid + 1]));
      As[tid] = expf(Ms[tid] - Mn);                      // 0 on the first tile (M = -inf)
      Ms[tid] = Mn;
    }
    __syncthreads();
    // ---- per-token weights and Z
#pragma unroll
    for (int k = 0; k < SLOTS; ++k) {
      const int idx = tid + k * kGqaThreads;
      const bool active = idx < r * kGqaTile;
      const int h = idx >> 6, tt = idx & (kGqaTile - 1);
      float wgt = 0.f;
      if (active && sv[k] != -INFINITY) {
        wgt = expf(sv[k] - Ms[h]);
        if (gr[k]) wgt /= dn[k];
      }
      if (active) pw[h * kGqaTile + tt] = wgt;
      float z = wgt;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
      if (active && lane == 0) zpart[h * 2 + (tt >> 5)] = z;
    }
    __syncthreads();
    if (tid < r) Zs[tid] = Zs[tid] * As[tid] + (zpart[2 * tid] + zpart[2 * tid + 1]);
    // ---- O = O alpha + sum_t P_t v_t over this thread's token slice, every head
    {
#pragma unroll
      for (int h = 0; h < 4 * SLOTS; ++h)
        if (h < r) { o0[h] *= As[h]; o1[h] *= As[h]; }
      const int ta = tg * tpg;
      const int tb = ta + tpg < n ? ta + tpg : n;     // rows past n are never read
      int tt = ta;
      for (; tt + 4 <= tb; tt += 4) {
        float v0[4], v1[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) gqa_pair<T>(vb + (tt + e) * d_v + 2 * dp, v0[e], v1[e]);
#pragma unroll
        for (int h = 0; h < 4 * SLOTS; ++h) {
          if (h < r) {
            const float4 w4 = *reinterpret_cast<const float4*>(pw + h * kGqaTile + tt);
            const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              o0[h] = fmaf(wv[e], v0[e], o0[h]);
              o1[h] = fmaf(wv[e], v1[e], o1[h]);
            }
          }
        }
      }
      for (; tt < tb; ++tt) {
        float v0, v1;
        gqa_pair<T>(vb + tt * d_v + 2 * dp, v0, v1);
#pragma unroll
        for (int h = 0; h < 4 * SLOTS; ++h) {
          if (h < r) {
            const float wt = pw[h * kGqaTile + tt];
            o0[h] = fmaf(wt, v0, o0[h]);
            o1[h] = fmaf(wt, v1, o1[h]);
          }
        }
      }
    }
    __syncthreads();
  }

  const int64_t slot = (int64_t)b * p.n_split + split;
  if (!LCA_CHECK(p.err, slot < p.ws_slots, 0xC23)) return;
  // the token slices' partial sums meet in shared memory (the tile buffers are
  // free now) and are added in slice order
  {
    float* red = reinterpret_cast<float*>(kbuf);      // [slice][r][d_v]
#pragma unroll
    for (int h = 0; h < 4 * SLOTS; ++h) {
      if (h < r) {
        red[(tg * r + h) * d_v + 2 * dp] = o0[h];
        red[(tg * r + h) * d_v + 2 * dp + 1] = o1[h];
      }
    }
    __syncthreads();
    const int n_slices = kGqaThreads >> lg_np;
    for (int i = tid; i < r * npairs; i += kGqaThreads) {
      const int h = i >> lg_np, d = 2 * (i & (npairs - 1));
      float a0 = 0.f, a1 = 0.f;
      for (int sl = 0; sl < n_slices; ++sl) {
        a0 += red[(sl * r + h) * d_v + d];
        a1 += red[(sl * r + h) * d_v + d + 1];
      }
      *reinterpret_cast<float2*>(p.part_o + (slot * p.H + h0 + h) * (int64_t)d_v + d) = make_float2(a0, a1);
    }
  }
  if (tid < r) {
    p.part_mz[(slot * p.H + h0 + tid) * 2 + 0] = Ms[tid];
    p.part_mz[(slot * p.H + h0 + tid) * 2 + 1] = Zs[tid];
  }
}

}  // namespace lca
