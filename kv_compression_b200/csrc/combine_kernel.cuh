// combine_kernel.cuh -- merge the per-split partials (M, Z, O) of one
// (sequence, head) into out = sum_i e^{M_i - M} O_i / sum_i e^{M_i - M} Z_i,
// M = max_i M_i: the online-softmax merge (Milakov & Gimelshein 2018), here
// applied to the ranges a long context is split into on one GPU.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace lca {

constexpr int kCombineThreads = 128;
constexpr int kCombineMaxParts = 1024;   // per (sequence, head); the plan keeps far fewer

struct CombineParams {
  const float* part_o;   // [slots][H][d_c]
  const float* part_mz;  // [slots][H][2]
  float* out;            // [B][H][d_c]
  int B, H, d_c;
  // Slots of sequence b.
  //   mode 0: slots b*n_split .. b*n_split + n_split - 1
  //   mode 1: the units (b, tile) are cut into G contiguous ranges, range c =
  //           [c*U/G, (c+1)*U/G) with U = B * tiles_per_seq; range c writes the
  //           partial of sequence b into slot b + c.
  int mode;
  int n_split;
  int64_t tiles_per_seq;
  int64_t G;
  int wait_prior;        // 1: launched as a programmatic dependent of the producer grid
};

__device__ __forceinline__ int64_t range_owner(int64_t u, int64_t U, int64_t G) {
  return ((u + 1) * G - 1) / U;  // largest c with floor(c*U/G) <= u
}

// Grid: (H, B, d_c / kCombineThreads); one thread per latent dimension.
__global__ void __launch_bounds__(kCombineThreads) lca_combine_kernel(const CombineParams p) {
  __shared__ float scale[kCombineMaxParts];
  __shared__ float red[kCombineThreads / 32];
  if (p.wait_prior) ptx::griddep_wait();
  const int h = blockIdx.x, b = blockIdx.y, tid = threadIdx.x;
  int64_t first, count;
  if (p.mode == 0) {
    first = (int64_t)b * p.n_split;
    count = p.n_split;
  } else {
    const int64_t U = (int64_t)p.B * p.tiles_per_seq;
    const int64_t c0 = range_owner((int64_t)b * p.tiles_per_seq, U, p.G);
    const int64_t c1 = range_owner((int64_t)(b + 1) * p.tiles_per_seq - 1, U, p.G);
    first = b + c0;
    count = c1 - c0 + 1;
  }
  if (count > kCombineMaxParts) count = kCombineMaxParts;  // the host never plans more
  // M = max_i M_i (partials read in parallel)
  float m = -INFINITY;
  for (int64_t i = tid; i < count; i += kCombineThreads)
    m = fmaxf(m, p.part_mz[((first + i) * p.H + h) * 2]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((tid & 31) == 0) red[tid >> 5] = m;
  __syncthreads();
  float M = red[0];
#pragma unroll
  for (int w = 1; w < kCombineThreads / 32; ++w) M = fmaxf(M, red[w]);
  __syncthreads();
  // factors e^{M_i - M} and Z = sum_i e^{M_i - M} Z_i
  float z = 0.f;
  for (int64_t i = tid; i < count; i += kCombineThreads) {
    const float* mz = p.part_mz + ((first + i) * p.H + h) * 2;
    const float f = expf(mz[0] - M);
    scale[i] = f;
    z = fmaf(f, mz[1], z);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xffffffffu, z, o);
  if ((tid & 31) == 0) red[tid >> 5] = z;
  __syncthreads();
  float Z = 0.f;
#pragma unroll
  for (int w = 0; w < kCombineThreads / 32; ++w) Z += red[w];
  const float invZ = 1.f / Z;
  // out[d] = sum_i f_i O_i[d] / Z with eight loads in flight
  const int d = blockIdx.z * kCombineThreads + tid;
  if (d >= p.d_c) return;
  const int64_t stride = (int64_t)p.H * p.d_c;
  const float* po = p.part_o + (first * p.H + h) * (int64_t)p.d_c + d;
  float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int64_t i = 0;
  for (; i + 8 <= count; i += 8) {
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = po[(i + k) * stride];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = fmaf(scale[i + k], v[k], acc[k]);
  }
  for (; i < count; ++i) acc[0] = fmaf(scale[i], po[i * stride], acc[0]);
  const float sum = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
  p.out[((int64_t)b * p.H + h) * p.d_c + d] = sum * invZ;
}

}  // namespace lca
