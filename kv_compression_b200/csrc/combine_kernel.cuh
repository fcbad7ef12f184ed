// combine_kernel.cuh -- merge the per-split partials (M, Z, O) of one
// (sequence, head) into out = sum_i e^{M_i - M} O_i / sum_i e^{M_i - M} Z_i,
// M = max_i M_i: the online-softmax merge (Milakov & Gimelshein 2018), here
// applied to the ranges a long context is split into on one GPU.
#pragma once
#include <cstdint>

#include "checks.cuh"
#include "paged_kernel.cuh"
#include "ptx.cuh"

namespace lca {

constexpr int kCombineThreads = 128;
constexpr int kCombineVec = 4;    // latent dims per thread

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
  //   mode 2: slots b, B + b, 2B + b, ... (n_split of them): partials stacked
  //           by part, merged across parts (lca_merge_partials)
  //   mode 3: as mode 1 over sequences of their own lengths: U, G and the
  //           first tile and tile count of each sequence from the paged
  //           metadata (a sequence without tiles has no partial: NaN out)
  int mode;
  int n_split;
  int64_t tiles_per_seq;
  int64_t G;
  int wait_prior;        // 1: launched as a programmatic dependent of the producer grid
  const int* meta;       // mode 3: the paged metadata
  float* out_mz;         // non-null: write the merged (M, Z) to out_mz [B][H][2] and the
                         // unnormalised sum O to out (a partial for a later merge)
  int64_t n_slots;       // slots readable in part_o / part_mz (range checks)
  int* err;              // device error word (range checks; null: none)
  int vec;               // 1: d_c % 4 == 0 and part_o, out 16-byte aligned (vector loads and stores)
};

__device__ __forceinline__ int64_t range_owner(int64_t u, int64_t U, int64_t G) {
  return ((u + 1) * G - 1) / U;  // largest c with floor(c*U/G) <= u
}

// Grid: (H, B, d_c / (kCombineThreads * kCombineVec)); each thread takes
// kCombineVec consecutive latent dimensions (one 16-byte load per partial when
// the rows allow it).  The slots of the block's (sequence, head) are found once
// per block.  One pass over the partials, kChunk at a time: every (M_i, Z_i)
// and O_i[d] of a chunk is loaded at once, then merged online -- the running
// max rises to the chunk's and the sums are rescaled -- so the kernel waits for
// memory about once per chunk.  Each thread forms Z itself (a few
// exponentials) instead of sharing it through a block reduction.
__global__ void __launch_bounds__(kCombineThreads, 4) lca_combine_kernel(const CombineParams p) {
  constexpr int kChunk = 8;
  if (p.wait_prior) ptx::griddep_wait();
  // The next step's main kernel may start its prologue now; it waits for this
  // grid to complete before touching global memory.
  ptx::griddep_launch_dependents();
  const int h = blockIdx.x, b = blockIdx.y;
  __shared__ int64_t s_first, s_count;
  if (threadIdx.x == 0) {
    int64_t first, count;
    if (p.mode == 0) {
      first = (int64_t)b * p.n_split;
      count = p.n_split;
    } else if (p.mode == 2) {
      first = b;
      count = p.n_split;
    } else if (p.mode == 3) {
      const int64_t U = p.meta[0], G = p.meta[1];
      const int4 rec = meta_seq(p.meta)[b];
      first = b;
      count = 0;
      if (rec.w > 0 && G > 0) {
        const int64_t c0 = range_owner(rec.y, U, G);
        const int64_t c1 = range_owner((int64_t)rec.y + rec.w - 1, U, G);
        first = b + c0;
        count = c1 - c0 + 1;
      }
    } else {
      const int64_t U = (int64_t)p.B * p.tiles_per_seq;
      const int64_t c0 = range_owner((int64_t)b * p.tiles_per_seq, U, p.G);
      const int64_t c1 = range_owner((int64_t)(b + 1) * p.tiles_per_seq - 1, U, p.G);
      first = b + c0;
      count = c1 - c0 + 1;
    }
    const int64_t step = p.mode == 2 ? p.B : 1;
    if (count > 0 && p.err && !LCA_CHECK(p.err, first + (count - 1) * step < p.n_slots, 0xC11))
      count = 0;
    s_first = first;
    s_count = count;
  }
  __syncthreads();
  const int64_t first = s_first, count = s_count;
  const int64_t slot_step = p.mode == 2 ? p.B : 1;
  const int d = (blockIdx.z * kCombineThreads + threadIdx.x) * kCombineVec;
  if (d >= p.d_c) return;
  const int nd = p.d_c - d < kCombineVec ? p.d_c - d : kCombineVec;
  const bool vec = p.vec && nd == kCombineVec;
  const int64_t stride = (int64_t)p.H * p.d_c * slot_step;
  const float* po = p.part_o + (first * p.H + h) * (int64_t)p.d_c + d;
  const float2* pmz = reinterpret_cast<const float2*>(p.part_mz) + first * p.H + h;
  float M = -INFINITY, Z = 0.f;
  float acc[kCombineVec] = {0.f, 0.f, 0.f, 0.f};
  for (int64_t i0 = 0; i0 < count; i0 += kChunk) {
    const int n = (int)(count - i0 < kChunk ? count - i0 : kChunk);
    float2 mz[kChunk];
    float4 o[kChunk];
#pragma unroll
    for (int k = 0; k < kChunk; ++k) {
      mz[k] = make_float2(-INFINITY, 0.f);
      o[k] = make_float4(0.f, 0.f, 0.f, 0.f);
      if (k < n) {
        mz[k] = pmz[(i0 + k) * slot_step * p.H];
        const float* src = po + (i0 + k) * stride;
        if (vec) {
          o[k] = *reinterpret_cast<const float4*>(src);
        } else {
          o[k].x = src[0];
          if (nd > 1) o[k].y = src[1];
          if (nd > 2) o[k].z = src[2];
          if (nd > 3) o[k].w = src[3];
        }
      }
    }
    float mc = M;
#pragma unroll
    for (int k = 0; k < kChunk; ++k) mc = fmaxf(mc, mz[k].x);
    if (mc == -INFINITY) continue;            // only empty partials so far
    const float f = expf(M - mc);             // 0 while M is still -inf
    Z *= f;
#pragma unroll
    for (int j = 0; j < kCombineVec; ++j) acc[j] *= f;
#pragma unroll
    for (int k = 0; k < kChunk; ++k) {
      if (k < n) {
        const float w = expf(mz[k].x - mc);    // 0 for an empty partial (M_i = -inf)
        Z = fmaf(w, mz[k].y, Z);
        acc[0] = fmaf(w, o[k].x, acc[0]);
        acc[1] = fmaf(w, o[k].y, acc[1]);
        acc[2] = fmaf(w, o[k].z, acc[2]);
        acc[3] = fmaf(w, o[k].w, acc[3]);
      }
    }
    M = mc;
  }
  float* dst = p.out + ((int64_t)b * p.H + h) * p.d_c + d;
  float r[kCombineVec];
#pragma unroll
  for (int j = 0; j < kCombineVec; ++j) r[j] = p.out_mz ? acc[j] : acc[j] / Z;
  if (vec) {
    *reinterpret_cast<float4*>(dst) = make_float4(r[0], r[1], r[2], r[3]);
  } else {
    for (int j = 0; j < nd; ++j) dst[j] = r[j];
  }
  if (p.out_mz && d == 0) {
    p.out_mz[((int64_t)b * p.H + h) * 2 + 0] = M;
    p.out_mz[((int64_t)b * p.H + h) * 2 + 1] = Z;
  }
}

}  // namespace lca
