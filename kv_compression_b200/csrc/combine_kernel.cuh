// combine_kernel.cuh -- merge the per-split partials (M, Z, O) of one
// (sequence, head) into out = sum_i e^{M_i - M} O_i / sum_i e^{M_i - M} Z_i,
// M = max_i M_i: the online-softmax merge (Milakov & Gimelshein 2018), here
// applied to the ranges a long context is split into on one GPU.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace lca {

constexpr int kCombineThreads = 128;

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

__global__ void __launch_bounds__(kCombineThreads) lca_combine_kernel(const CombineParams p) {
  if (p.wait_prior) ptx::griddep_wait();
  const int h = blockIdx.x, b = blockIdx.y;
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
  float M = -INFINITY;
  for (int64_t i = 0; i < count; ++i) M = fmaxf(M, p.part_mz[((first + i) * p.H + h) * 2]);
  float Z = 0.f;
  for (int64_t i = 0; i < count; ++i) {
    const float* mz = p.part_mz + ((first + i) * p.H + h) * 2;
    Z += expf(mz[0] - M) * mz[1];
  }
  const float invZ = 1.f / Z;
  for (int d = threadIdx.x; d < p.d_c; d += kCombineThreads) {
    float acc = 0.f;
    for (int64_t i = 0; i < count; ++i) {
      const float sc = expf(p.part_mz[((first + i) * p.H + h) * 2] - M);
      acc = fmaf(sc, p.part_o[((first + i) * p.H + h) * p.d_c + d], acc);
    }
    p.out[((int64_t)b * p.H + h) * p.d_c + d] = acc * invZ;
  }
}

}  // namespace lca
