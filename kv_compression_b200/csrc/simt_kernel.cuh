// simt_kernel.cuh -- LCA / dense-MLA decode on CUDA cores, fp32 accumulation.
//
// Used for fp32 latents (where tensor-core TF32 would not hold a 1e-5
// tolerance) and for shapes the tcgen05 kernel does not take.  One CTA per
// (split of the context, head, sequence).  Within a split, tiles of whole
// groups are processed as:
//   scores      s_t = q_c.c_t + q_r.k_t, one warp per token (lanes over dims);
//   condense    per group (one thread each): max, lowest-index argmax (anchor),
//               group-local softmax weights, condensed logit
//               S_j = sum_t w_t sc_t + sr_{a_j}  (q_c.c_bar_j without forming c_bar_j);
//   attend      online softmax over [condensed || window] entries: per-token
//               weight P_t = exp(S_j - M) w_t in a group, exp(s_t - M) in the window;
//               O = O * alpha + sum_t P_t c_t.
// "Latent-Condensed Transformer for Efficient Long Context Modeling",
// section 2, "O Algoritmo LCA", steps 1-3.  The split partial (M, Z, O) is
// merged by the combine kernel (online-softmax merge).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "checks.cuh"
#include "paged_kernel.cuh"

namespace lca {

constexpr int kSimtThreads = 256;
constexpr int kSimtWarps = kSimtThreads / 32;

template <typename T>
__device__ __forceinline__ float load_elem(const T* p);
template <>
__device__ __forceinline__ float load_elem<float>(const float* p) {
  return __ldg(p);
}
template <>
__device__ __forceinline__ float load_elem<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(__ldg(p));
}

struct SimtParams {
  const void* q_c;
  const void* q_r;
  const void* c_kv;
  const void* k_r;
  int B, H, d_c, d_r;
  int64_t L;
  int g;             // group size (1 when nG == 0)
  int64_t nG;        // number of condensed groups
  int64_t split_len; // tokens per split (a multiple of g)
  int tile;          // tokens per tile (a multiple of g, <= kSimtTileMax)
  int n_split;
  int32_t* anchor;   // [B][H][nG] or null when nG == 0
  float* part_o;     // [B * n_split][H][d_c]
  float* part_mz;    // [B * n_split][H][2]
  int64_t bias_rows; // rows [0, bias_rows) get `bias` added to their score (stored-cache
  float bias;        // decode: the condensed entries; 0 rows otherwise)
  int64_t win0;      // first window token, in this cache's rows (n_G g for a whole context)
  int64_t pos0;      // position of row 0 in the context: anchors are written as pos0 + row
  int64_t ws_slots;  // slots of part_o / part_mz (range checks)
  int* err;          // device error word (range checks)
  int64_t anchor_stride;     // anchors of (b, h) start at (b H + h) anchor_stride
  // paged, variable-length decode (meta != null): c_kv / k_r are the pools,
  // sequence b has meta_seq(meta)[b].x tokens, token t in row
  // block_table[b table_stride + t / page_size] page_size + t % page_size
  const int* meta;
  const int32_t* block_table;
  int64_t table_stride;   // block-table entries from one sequence's row to the next (0: one shared row)
  int page_size;
  int64_t num_pages;
};

constexpr int kSimtTileMax = 1024;
constexpr int kSimtMaxDc = 1024;

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// Block-wide reduction (sum or max) through `red` (kSimtWarps floats).
template <bool kMax>
__device__ __forceinline__ float block_reduce(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  v = kMax ? warp_max(v) : warp_sum(v);
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
  for (int i = 1; i < kSimtWarps; ++i) r = kMax ? fmaxf(r, red[i]) : r + red[i];
  return r;
}

template <typename T>
__global__ void __launch_bounds__(kSimtThreads)
lca_simt_kernel(const SimtParams p) {
  const int split = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  extern __shared__ float smem[];
  float* qc = smem;                    // [d_c]
  float* qr = qc + p.d_c;              // [d_r]
  float* sc = qr + p.d_r;              // [tile] semantic score
  float* sr = sc + kSimtTileMax;       // [tile] positional score
  float* pw = sr + kSimtTileMax;       // [tile] per-token attention weight
  float* glog = pw + kSimtTileMax;     // [tile] condensed logit of the group starting here
  float* red = glog + kSimtTileMax;    // [kSimtWarps]
  int64_t* rowix = reinterpret_cast<int64_t*>(red + kSimtWarps);   // [tile] pool row (paged)

  const T* qc_g = static_cast<const T*>(p.q_c) + ((int64_t)b * p.H + h) * p.d_c;
  const T* qr_g = static_cast<const T*>(p.q_r) + ((int64_t)b * p.H + h) * p.d_r;
  const bool paged = p.meta != nullptr;
  const T* c_g = static_cast<const T*>(p.c_kv) + (paged ? 0 : (int64_t)b * p.L * p.d_c);
  const T* k_g = static_cast<const T*>(p.k_r) + (paged ? 0 : (int64_t)b * p.L * p.d_r);
  for (int i = tid; i < p.d_c; i += kSimtThreads) qc[i] = load_elem(qc_g + i);
  for (int i = tid; i < p.d_r; i += kSimtThreads) qr[i] = load_elem(qr_g + i);

  // this sequence's length, groups and split (paged: its own, from the metadata)
  int64_t L = p.L, nG = p.nG, win0 = p.win0, split_len = p.split_len;
  if (paged) {
    const int4 rec = meta_seq(p.meta)[b];
    L = rec.x;
    nG = rec.z;
    win0 = nG * p.g;
    split_len = (L + p.n_split - 1) / p.n_split;
    split_len = (split_len + p.g - 1) / p.g * p.g;
  }
  const int64_t s0 = (int64_t)split * split_len;
  const int64_t s1 = (L < s0 + split_len) ? L : s0 + split_len;

  constexpr int kDPerThread = kSimtMaxDc / kSimtThreads;
  float o[kDPerThread];
#pragma unroll
  for (int k = 0; k < kDPerThread; ++k) o[k] = 0.f;
  float M = -INFINITY, Z = 0.f;
  __syncthreads();

  for (int64_t t0 = s0; t0 < s1; t0 += p.tile) {
    const int n = (int)((int64_t)p.tile < s1 - t0 ? (int64_t)p.tile : s1 - t0);
    // ---- the rows of this tile's tokens
    for (int tt = tid; tt < n; tt += kSimtThreads)
      if (LCA_CHECK(p.err, tt < kSimtTileMax, 0xC05))
        rowix[tt] = paged ? paged_row(p.block_table, p.table_stride, p.page_size, p.num_pages, b, t0 + tt,
                                      p.err, 0xA02)
                          : t0 + tt;
    __syncthreads();
    // ---- scores, one warp per token
    for (int tt = warp; tt < n; tt += kSimtWarps) {
      const T* crow = c_g + rowix[tt] * p.d_c;
      const T* krow = k_g + rowix[tt] * p.d_r;
      float a = 0.f, r = 0.f;
      for (int d = lane; d < p.d_c; d += 32) a = fmaf(qc[d], load_elem(crow + d), a);
      for (int d = lane; d < p.d_r; d += 32) r = fmaf(qr[d], load_elem(krow + d), r);
      a = warp_sum(a);
      r = warp_sum(r);
      if (t0 + tt < p.bias_rows) r += p.bias;
      if (lane == 0 && LCA_CHECK(p.err, tt < kSimtTileMax, 0xC01)) { sc[tt] = a; sr[tt] = r; }
    }
    __syncthreads();
    // ---- condense: one thread per group, starting token of the group
    for (int tt = tid; tt < n; tt += kSimtThreads) {
      const int64_t t = t0 + tt;
      if (t < win0 && (t % p.g) == 0 && LCA_CHECK(p.err, tt + p.g <= kSimtTileMax, 0xC02)) {
        float m = sc[tt] + sr[tt];
        int amax = tt;
        for (int u = tt + 1; u < tt + p.g; ++u) {
          const float s = sc[u] + sr[u];
          if (s > m) { m = s; amax = u; }   // strict: the lowest index keeps a tie
        }
        float den = 0.f, num = 0.f;
        for (int u = tt; u < tt + p.g; ++u) {
          const float e = expf(sc[u] + sr[u] - m);
          den += e;
          num = fmaf(e, sc[u], num);
        }
        glog[tt] = num / den + sr[amax];
        const float inv = 1.f / den;
        for (int u = tt; u < tt + p.g; ++u) pw[u] = expf(sc[u] + sr[u] - m) * inv;  // w_t
        if (LCA_CHECK(p.err, t / p.g < nG, 0xC03))
          p.anchor[((int64_t)b * p.H + h) * p.anchor_stride + t / p.g] = (int32_t)(p.pos0 + t0 + amax);
      }
    }
    __syncthreads();
    // ---- tile maximum over entries (condensed logits and window scores)
    float lmax = -INFINITY;
    for (int tt = tid; tt < n; tt += kSimtThreads) {
      const int64_t t = t0 + tt;
      if (t < win0) {
        if ((t % p.g) == 0) lmax = fmaxf(lmax, glog[tt]);
      } else {
        lmax = fmaxf(lmax, sc[tt] + sr[tt]);
      }
    }
    const float tmax = block_reduce<true>(lmax, red);
    const float Mn = fmaxf(M, tmax);
    const float alpha = expf(M - Mn);  // 0 on the first tile (M = -inf)
    // ---- per-token weights
    float lz = 0.f;
    for (int tt = tid; tt < n; tt += kSimtThreads) {
      const int64_t t = t0 + tt;
      float w;
      if (t < win0) {
        const int64_t gs = tt - (t % p.g);            // group start within the tile
        w = expf(glog[gs] - Mn) * pw[tt];           // group weight x in-group weight
      } else {
        w = expf(sc[tt] + sr[tt] - Mn);
      }
      pw[tt] = w;
      lz += w;
    }
    const float tz = block_reduce<false>(lz, red);  // contains __syncthreads: pw is complete
    Z = Z * alpha + tz;
    M = Mn;
    // ---- O = O * alpha + sum_t P_t c_t, threads over latent dims
#pragma unroll
    for (int k = 0; k < kDPerThread; ++k) o[k] *= alpha;
    for (int tt = 0; tt < n; ++tt) {
      const float w = pw[tt];
      const T* crow = c_g + rowix[tt] * p.d_c;
#pragma unroll
      for (int k = 0; k < kDPerThread; ++k) {
        const int d = tid + k * kSimtThreads;
        if (d < p.d_c) o[k] = fmaf(w, load_elem(crow + d), o[k]);
      }
    }
    __syncthreads();
  }

  const int64_t slot = (int64_t)b * p.n_split + split;
  if (!LCA_CHECK(p.err, slot < p.ws_slots, 0xC04)) return;
  float* po = p.part_o + (slot * p.H + h) * p.d_c;
#pragma unroll
  for (int k = 0; k < kDPerThread; ++k) {
    const int d = tid + k * kSimtThreads;
    if (d < p.d_c) po[d] = o[k];
  }
  if (tid == 0) {
    p.part_mz[(slot * p.H + h) * 2 + 0] = M;
    p.part_mz[(slot * p.H + h) * 2 + 1] = Z;
  }
}

}  // namespace lca
