// condense_kernel.cuh -- build a stored, head-shared condensed cache.
//
// "Latent-Condensed Transformer for Efficient Long Context Modeling": the
// cache and decode gains of section 4 ("Eficiencia") come from keeping each
// condensed group instead of its tokens.  A stored entry is condensed once,
// with the query of the step that condenses it, and one entry serves every
// head: the pooling weights and the anchor come from the head-mean score
//   s_bar_t = (1/H) sum_h (q_c^h . c_t + q_r^h . k_t) = q_bar_c . c_t + q_bar_r . k_t
// (the mean of the heads' scores is the score of the mean query), then, as in
// section 2 step 2, w_t = softmax over the group of s_bar_t, a_j = the lowest
// index with the largest s_bar_t, and the entry is (c_bar_j = sum w_t c_t,
// k_{a_j}).
//
// lca_condense_kernel: grid (blocks per sequence, B), 256 threads; each block
// first forms the mean query of its sequence in shared memory (fp32), then
// each warp condenses one group at a time: per token the warp's lanes split
// the dims of the score (a warp-wide sum), and the pooled latent is kept as an
// online softmax-weighted sum (running max, rescale on a rise), so every
// cache row is read once.  The entry is stored in the cache's element type.
// lca_copy_rows_kernel: copies the window rows after the condensed entries.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "simt_kernel.cuh"

namespace lca {

constexpr int kCondThreads = 256;
constexpr int kCondWarps = kCondThreads / 32;
constexpr int kCondMaxPerLane = kSimtMaxDc / 32;   // latent dims a lane holds

struct CondenseParams {
  const void* q_c;    // [B][H][d_c]
  const void* q_r;    // [B][H][d_r]
  const void* c_kv;   // [B][L][d_c]
  const void* k_r;    // [B][L][d_r]
  int B, H, d_c, d_r;
  int64_t L;
  int g;
  int64_t j0, n;      // groups j0 .. j0 + n - 1 (tokens below L)
  void* c_dst;        // entry jj of sequence b -> row b * dst_rows + dst_row0 + jj
  void* k_dst;
  int64_t dst_rows, dst_row0;
  int32_t* anchor;    // [B][n] absolute positions
  int* err;           // device error word (range checks)
};

template <typename T>
__device__ __forceinline__ void store_elem(T* p, float v);
template <>
__device__ __forceinline__ void store_elem<float>(float* p, float v) { *p = v; }
template <>
__device__ __forceinline__ void store_elem<__nv_bfloat16>(__nv_bfloat16* p, float v) {
  *p = __float2bfloat16_rn(v);
}

template <typename T>
__global__ void __launch_bounds__(kCondThreads) lca_condense_kernel(const CondenseParams p) {
  extern __shared__ float cq[];              // the mean query: [d_c + d_r] floats
  const int b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int dq = p.d_c + p.d_r;
  const T* qc_b = static_cast<const T*>(p.q_c) + (int64_t)b * p.H * p.d_c;
  const T* qr_b = static_cast<const T*>(p.q_r) + (int64_t)b * p.H * p.d_r;
  const float inv_h = 1.f / (float)p.H;
  for (int d = tid; d < dq; d += kCondThreads) {
    float acc = 0.f;
    if (d < p.d_c) {
      for (int h = 0; h < p.H; ++h) acc += load_elem(qc_b + (int64_t)h * p.d_c + d);
    } else {
      for (int h = 0; h < p.H; ++h) acc += load_elem(qr_b + (int64_t)h * p.d_r + (d - p.d_c));
    }
    cq[d] = acc * inv_h;
  }
  __syncthreads();

  const T* c_b = static_cast<const T*>(p.c_kv) + (int64_t)b * p.L * p.d_c;
  const T* k_b = static_cast<const T*>(p.k_r) + (int64_t)b * p.L * p.d_r;
  T* cd = static_cast<T*>(p.c_dst);
  T* kd = static_cast<T*>(p.k_dst);
  for (int64_t jj = (int64_t)blockIdx.x * kCondWarps + warp; jj < p.n;
       jj += (int64_t)gridDim.x * kCondWarps) {
    const int64_t t0 = (p.j0 + jj) * p.g;
    if (!LCA_CHECK(p.err, t0 + p.g <= p.L && p.dst_row0 + jj < p.dst_rows, 0xC21)) continue;
    float acc[kCondMaxPerLane];
#pragma unroll
    for (int k = 0; k < kCondMaxPerLane; ++k) acc[k] = 0.f;
    float m = -INFINITY, den = 0.f;
    int a = 0;
    for (int u = 0; u < p.g; ++u) {
      const T* crow = c_b + (t0 + u) * p.d_c;
      const T* krow = k_b + (t0 + u) * p.d_r;
      float cv[kCondMaxPerLane];
      float part = 0.f;
#pragma unroll
      for (int k = 0; k < kCondMaxPerLane; ++k) {
        const int d = lane + 32 * k;
        cv[k] = d < p.d_c ? load_elem(crow + d) : 0.f;
        part = fmaf(d < p.d_c ? cq[d] : 0.f, cv[k], part);
      }
      for (int d = lane; d < p.d_r; d += 32) part = fmaf(cq[p.d_c + d], load_elem(krow + d), part);
      const float s = warp_sum(part);          // the same bits in every lane
      if (s > m) {                             // strict: the lowest index keeps a tie
        const float alpha = __expf(m - s);     // 0 on the first token
        den *= alpha;
#pragma unroll
        for (int k = 0; k < kCondMaxPerLane; ++k) acc[k] *= alpha;
        m = s;
        a = u;
      }
      const float e = __expf(s - m);
      den += e;
#pragma unroll
      for (int k = 0; k < kCondMaxPerLane; ++k) acc[k] = fmaf(e, cv[k], acc[k]);
    }
    const float inv = 1.f / den;
    const int64_t row = (int64_t)b * p.dst_rows + p.dst_row0 + jj;
#pragma unroll
    for (int k = 0; k < kCondMaxPerLane; ++k) {
      const int d = lane + 32 * k;
      if (d < p.d_c) store_elem(cd + row * p.d_c + d, acc[k] * inv);
    }
    const T* ka = k_b + (t0 + a) * p.d_r;      // the anchor's RoPE key, copied as stored
    for (int d = lane; d < p.d_r; d += 32) kd[row * p.d_r + d] = ka[d];
    if (lane == 0) p.anchor[(int64_t)b * p.n + jj] = (int32_t)(t0 + a);
  }
}

// The same for bf16 latents with d_c = 512 and d_r = 64 (every benchmark
// shape): lane l owns latent dims [16 l, 16 l + 16) -- two 16-byte loads a
// row -- and RoPE dims [2 l, 2 l + 2); four tokens' rows are loaded before
// their scores are reduced, so a warp keeps several rows in flight.
constexpr int kCondFastDc = 512, kCondFastDr = 64, kCondBatch = 4;

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float* f) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__global__ void __launch_bounds__(kCondThreads) lca_condense_fast_kernel(const CondenseParams p) {
  __shared__ float cq[kCondFastDc + kCondFastDr];   // the mean query
  const int b = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const __nv_bfloat16* qc_b = static_cast<const __nv_bfloat16*>(p.q_c) + (int64_t)b * p.H * kCondFastDc;
  const __nv_bfloat16* qr_b = static_cast<const __nv_bfloat16*>(p.q_r) + (int64_t)b * p.H * kCondFastDr;
  const float inv_h = 1.f / (float)p.H;
  for (int d = tid; d < kCondFastDc + kCondFastDr; d += kCondThreads) {
    float acc = 0.f;
    if (d < kCondFastDc) {
      for (int h = 0; h < p.H; ++h) acc += load_elem(qc_b + (int64_t)h * kCondFastDc + d);
    } else {
      for (int h = 0; h < p.H; ++h) acc += load_elem(qr_b + (int64_t)h * kCondFastDr + (d - kCondFastDc));
    }
    cq[d] = acc * inv_h;
  }
  __syncthreads();
  float qc[16], qr[2];
#pragma unroll
  for (int i = 0; i < 16; ++i) qc[i] = cq[16 * lane + i];
  qr[0] = cq[kCondFastDc + 2 * lane];
  qr[1] = cq[kCondFastDc + 2 * lane + 1];

  const uint8_t* c_b = static_cast<const uint8_t*>(p.c_kv) + (int64_t)b * p.L * kCondFastDc * 2;
  const uint8_t* k_b = static_cast<const uint8_t*>(p.k_r) + (int64_t)b * p.L * kCondFastDr * 2;
  uint8_t* cd = static_cast<uint8_t*>(p.c_dst);
  uint8_t* kd = static_cast<uint8_t*>(p.k_dst);
  for (int64_t jj = (int64_t)blockIdx.x * kCondWarps + warp; jj < p.n;
       jj += (int64_t)gridDim.x * kCondWarps) {
    const int64_t t0 = (p.j0 + jj) * p.g;
    if (!LCA_CHECK(p.err, t0 + p.g <= p.L && p.dst_row0 + jj < p.dst_rows, 0xC22)) continue;
    float acc[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) acc[i] = 0.f;
    float m = -INFINITY, den = 0.f;
    int a = 0;
    for (int u0 = 0; u0 < p.g; u0 += kCondBatch) {
      uint4 cv[kCondBatch][2];
      uint32_t kv[kCondBatch];
#pragma unroll
      for (int e = 0; e < kCondBatch; ++e) {
        const int u = u0 + e < p.g ? u0 + e : p.g - 1;     // a short group repeats its last row
        const uint4* crow = reinterpret_cast<const uint4*>(c_b + (t0 + u) * (kCondFastDc * 2)) + 2 * lane;
        cv[e][0] = __ldg(crow);
        cv[e][1] = __ldg(crow + 1);
        kv[e] = __ldg(reinterpret_cast<const uint32_t*>(k_b + (t0 + u) * (kCondFastDr * 2)) + lane);
      }
      float part[kCondBatch];
#pragma unroll
      for (int e = 0; e < kCondBatch; ++e) {
        float f[16];
        bf16x8_to_f32(cv[e][0], f);
        bf16x8_to_f32(cv[e][1], f + 8);
        float s = 0.f;
#pragma unroll
        for (int i = 0; i < 16; ++i) s = fmaf(qc[i], f[i], s);
        s = fmaf(qr[0], __uint_as_float(kv[e] << 16), s);
        s = fmaf(qr[1], __uint_as_float(kv[e] & 0xFFFF0000u), s);
        part[e] = s;
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
#pragma unroll
        for (int e = 0; e < kCondBatch; ++e) part[e] += __shfl_xor_sync(0xffffffffu, part[e], o);
#pragma unroll
      for (int e = 0; e < kCondBatch; ++e) {
        if (u0 + e >= p.g) break;                          // warp-uniform
        const float s = part[e];                           // the same bits in every lane
        float f[16];
        bf16x8_to_f32(cv[e][0], f);
        bf16x8_to_f32(cv[e][1], f + 8);
        if (s > m) {                                       // strict: the lowest index keeps a tie
          const float alpha = __expf(m - s);               // 0 on the first token
          den *= alpha;
#pragma unroll
          for (int i = 0; i < 16; ++i) acc[i] *= alpha;
          m = s;
          a = u0 + e;
        }
        const float w = __expf(s - m);
        den += w;
#pragma unroll
        for (int i = 0; i < 16; ++i) acc[i] = fmaf(w, f[i], acc[i]);
      }
    }
    const float inv = 1.f / den;
    const int64_t row = (int64_t)b * p.dst_rows + p.dst_row0 + jj;
    uint32_t packed[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const __nv_bfloat162 v = __floats2bfloat162_rn(acc[2 * i] * inv, acc[2 * i + 1] * inv);
      packed[i] = *reinterpret_cast<const uint32_t*>(&v);
    }
    uint4* cdst = reinterpret_cast<uint4*>(cd + row * (kCondFastDc * 2)) + 2 * lane;
    cdst[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    cdst[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    // the anchor's RoPE key, copied as stored
    reinterpret_cast<uint32_t*>(kd + row * (kCondFastDr * 2))[lane] =
        __ldg(reinterpret_cast<const uint32_t*>(k_b + (t0 + a) * (kCondFastDr * 2)) + lane);
    if (lane == 0) p.anchor[(int64_t)b * p.n + jj] = (int32_t)(t0 + a);
  }
}

// Copy rows [src_row0, src_row0 + n) of every sequence (src_rows rows each) to
// rows [dst_row0, dst_row0 + n) (dst_rows rows each), `row_bytes` bytes a row
// (a multiple of 16), 16 bytes per thread.
struct CopyRowsParams {
  const uint8_t* src;
  uint8_t* dst;
  int64_t src_rows, src_row0, dst_rows, dst_row0, n, row_bytes;
  int B;
};

__global__ void lca_copy_rows_kernel(const CopyRowsParams p) {
  const int64_t per_seq = p.n * (p.row_bytes / 16);
  const int64_t total = per_seq * p.B;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int64_t b = i / per_seq;
    const int64_t r = i - b * per_seq;
    const int64_t row = r / (p.row_bytes / 16);
    const int64_t col = r - row * (p.row_bytes / 16);
    const uint4* s = reinterpret_cast<const uint4*>(p.src + ((b * p.src_rows + p.src_row0 + row) * p.row_bytes)) + col;
    uint4* d = reinterpret_cast<uint4*>(p.dst + ((b * p.dst_rows + p.dst_row0 + row) * p.row_bytes)) + col;
    *d = *s;
  }
}

}  // namespace lca
