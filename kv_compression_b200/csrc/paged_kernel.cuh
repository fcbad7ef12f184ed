// paged_kernel.cuh -- per-call metadata of the paged, variable-length decode.
//
// A paged batch keeps each sequence's latent rows in pages of page_size rows
// (a multiple of 64) of one pool, listed per sequence in a block table, and
// gives every sequence its own length L_b (device array).  Each sequence is
// decoded exactly as a contiguous cache of L_b rows: its own n_G(b) groups and
// window ("Latent-Condensed Transformer for Efficient Long Context Modeling",
// section 2, "O Algoritmo LCA", step 1).  The lengths stay on the device, so
// one call needs no host round trip and can be captured in a CUDA graph.
//
// A prefill chunk is the same batch for n queries of one sequence: query b
// sits at position pos0 + b and condenses its own causal prefix, so its length
// is pos0 + b + 1 and every query reads the one block-table row (row stride 0).
//
// lca_paged_meta_kernel (one CTA) reads the lengths (or forms them from pos0)
// and writes, for the decode kernels and the combine:
//
//   meta[0] U        tiles of all sequences (tile = kT tokens of the chosen kernel)
//   meta[1] G_eff    tile ranges used: min(G, U); range c = [c U / G_eff, (c+1) U / G_eff)
//   meta[2] bad      1 if some length was out of range
//   seq[b]  int4     {L_b, first tile of b in the concatenation, n_G(b), tiles of b}, b <= B
//                    (a length outside [1, cap] or with n_G(b) > anchor_stride is set
//                    to 0 -- no tiles, no output -- and raises the device input bit)
//   range[c] int2    {sequence, tile within it} of range c's first tile
#pragma once
#include <cstdint>

namespace lca {

constexpr int kErrInput = 4;          // device error word bit: a length or page entry out of range
constexpr int kMetaThreads = 1024;
constexpr int kMetaHeader = 4;        // ints before the per-sequence records

__host__ __device__ inline int64_t meta_ints(int B, int64_t ranges) {
  return kMetaHeader + 4LL * (B + 1) + 2 * ranges;
}
__host__ __device__ inline int4* meta_seq(int* meta) { return reinterpret_cast<int4*>(meta + kMetaHeader); }
__host__ __device__ inline const int4* meta_seq(const int* meta) {
  return reinterpret_cast<const int4*>(meta + kMetaHeader);
}
__host__ __device__ inline int2* meta_range(int* meta, int B) {
  return reinterpret_cast<int2*>(meta + kMetaHeader + 4 * (B + 1));
}
__host__ __device__ inline const int2* meta_range(const int* meta, int B) {
  return reinterpret_cast<const int2*>(meta + kMetaHeader + 4 * (B + 1));
}

__device__ __forceinline__ void input_error(int* err, int where) {
  if (atomicOr(err, kErrInput) == 0) atomicExch(err + 1, where);
}

// The pool row of token `tok` of sequence b: its page from the block table,
// checked against the pool (an entry outside [0, num_pages) raises the device
// input bit, and page 0 is read instead, so no access leaves the pool).
__device__ __forceinline__ int64_t paged_row(const int32_t* table, int64_t row_stride, int page_size,
                                             int64_t num_pages, int64_t b, int64_t tok, int* err,
                                             int where) {
  const uint32_t ps = (uint32_t)page_size;
  const uint32_t t = (uint32_t)tok;
  const uint32_t j = t / ps;
  int64_t page = table[b * row_stride + j];
  if (page < 0 || page >= num_pages) {
    input_error(err, where);
    page = 0;
  }
  return page * page_size + (t - j * ps);
}

struct MetaParams {
  const int32_t* seq_lens;   // [B] device; null: a prefill chunk, length pos0 + b + 1
  int64_t pos0;
  int B;
  int64_t cap;               // the longest valid length: min(max_L, max_pages * page_size)
  int g, w;
  int64_t anchor_stride;     // anchors per (b, h); n_G(b) must not exceed it
  int kT;                    // tokens per tile of the decode kernel (0: no ranges)
  int64_t G;                 // tile ranges asked for
  int* meta;
  int* err;
};

__global__ void __launch_bounds__(kMetaThreads) lca_paged_meta_kernel(const MetaParams p) {
  __shared__ int64_t warp_sum[kMetaThreads / 32];
  __shared__ int bad_s;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  if (tid == 0) bad_s = 0;
  __syncthreads();
  // each thread takes `per` consecutive sequences
  const int per = (p.B + kMetaThreads - 1) / kMetaThreads;
  const int b0 = tid * per;
  const int b1 = min(p.B, b0 + per);
  int64_t local = 0;
  bool bad = false;
  for (int b = b0; b < b1; ++b) {
    const int64_t L = p.seq_lens ? (int64_t)p.seq_lens[b] : p.pos0 + b + 1;
    const int64_t nG = L > p.w ? (L - p.w) / p.g : 0;
    const bool ok = L >= 1 && L <= p.cap && nG <= p.anchor_stride;
    bad = bad || !ok;
    if (ok && p.kT > 0) local += (L + p.kT - 1) / p.kT;
  }
  // exclusive scan of the tile counts over threads
  int64_t incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int64_t v = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += v;
  }
  if (lane == 31) warp_sum[warp] = incl;
  if (bad) bad_s = 1;
  __syncthreads();
  int64_t before = 0;
  for (int k = 0; k < warp; ++k) before += warp_sum[k];
  int64_t start = before + incl - local;
  int4* seq = meta_seq(p.meta);
  for (int b = b0; b < b1; ++b) {
    int64_t L = p.seq_lens ? (int64_t)p.seq_lens[b] : p.pos0 + b + 1;
    int64_t nG = L > p.w ? (L - p.w) / p.g : 0;
    if (!(L >= 1 && L <= p.cap && nG <= p.anchor_stride)) L = 0, nG = 0;
    const int64_t tiles = p.kT > 0 ? (L + p.kT - 1) / p.kT : 0;
    seq[b] = make_int4((int)L, (int)start, (int)nG, (int)tiles);
    start += tiles;
  }
  int64_t U = 0;
  for (int k = 0; k < kMetaThreads / 32; ++k) U += warp_sum[k];
  const int64_t Ge = p.kT > 0 ? (U < p.G ? U : p.G) : 0;
  if (tid == 0) {
    seq[p.B] = make_int4(0, (int)U, 0, 0);
    p.meta[0] = (int)U;
    p.meta[1] = (int)Ge;
    p.meta[2] = bad_s;
    p.meta[3] = 0;
    if (bad_s) input_error(p.err, 0xA01);
  }
  __syncthreads();   // the records above are visible to the whole block
  // first (sequence, tile) of each range: the last sequence whose first tile
  // is at or before the range's first unit (it holds that unit: a sequence
  // without tiles starts where the next one does)
  int2* rng = meta_range(p.meta, p.B);
  for (int64_t c = tid; c < Ge; c += kMetaThreads) {
    const int64_t u0 = c * U / Ge;
    int lo = 0, hi = p.B - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (seq[mid].y <= u0) lo = mid; else hi = mid - 1;
    }
    rng[c] = make_int2(lo, (int)(u0 - seq[lo].y));
  }
}

}  // namespace lca
