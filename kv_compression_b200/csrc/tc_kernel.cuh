// tc_kernel.cuh -- LCA / dense-MLA decode with tcgen05 tensor cores, TMEM
// accumulators and TMA tile loads (sm_100a), bf16 latents, fp32 accumulation.
//
// What one CTA computes ("Latent-Condensed Transformer for Efficient Long
// Context Modeling", section 2, "O Algoritmo LCA", steps 1-3) for 16 heads of
// one sequence over a contiguous range of 128-token tiles:
//   scores     S^T[128 tokens x 16 heads] = [C_KV | K_R]_tile . [q_c | q_r]^T,
//              two TMEM accumulators, sc (K = 512) and sr (K = 64), because the
//              condensed logit needs the semantic part on its own;
//   condense   (step 2) per group and head: max and lowest-index argmax (the
//              anchor a_j), den_j = sum e^{s_t - m_j}, num_j = sum e^{s_t - m_j} sc_t
//              and the condensed logit S_j = num_j / den_j + sr_{a_j}
//              (= q_c.c_bar_j + q_r.k_{a_j}; c_bar_j is never formed).  A thread
//              holds one token row; a group of g <= 32 tokens is g neighbouring
//              lanes of a warp and reduces by butterfly shuffles, a group of 64
//              or 128 tokens merges the partial statistics of its warps;
//   attend     (step 3) softmax over [condensed || window] against a reference
//              max M per head.  A grouped token weighs
//              p_j w_t = e^{S_j - M} e^{s_t - m_j} / den_j, written e^{s_t + k_j - M}
//              with k_j = S_j - m_j - ln den_j; a window token weighs e^{s_t - M}:
//              one exponential per (token, head).  The bf16 weights go to shared
//              memory and O^T[512 x 16] += C_KV_tile^T . P^T accumulates in TMEM.
//              M only rises when an entry exceeds it by more than 2^8; then Z and
//              O^T (in TMEM) are rescaled.
// The range's partial (M, Z, O) goes to the workspace; the combine kernel
// merges the ranges of a sequence.
//
// Each C_KV byte is read from HBM once.  Of a tile's four 128-dim column
// pairs, pair 3 stays in shared memory from its load until O^T += C^T P^T has
// used it; pairs 0-2 are loaded for the scores and loaded again, from L2, for
// O.  So the scores of tile i+1 complete while the softmax of tile i runs.
// Two threads issue MMAs: the scores of a tile as its pairs land, O of a tile
// once its P is written.
//
// Roles (352 threads): warp 0 lane 0 issues TMA loads; warp 1 allocates TMEM
// and its lane 0 issues the score MMAs; warps 2-9 (256 threads) do the
// softmax, two warps per TMEM lane quarter, each owning 8 of the 16 heads;
// warp 10 lane 0 issues the O MMAs.
// Shared memory: five column-pair slots ([128 tokens][2 x 64 dims] each,
// 128-byte swizzle), two K_R slots, the query block (9 x [16 heads][64 dims])
// and two P buffers.
// Every mbarrier wait is bounded; when a bound runs out the CTA records the
// error, stops issuing work, waits for its own copies and MMAs in flight,
// frees TMEM and exits.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "checks.cuh"
#include "paged_kernel.cuh"
#include "ptx.cuh"

namespace lca {
namespace tc {

constexpr int kHC = 16;                    // heads per CTA (MMA N)
constexpr int kHH = 8;                     // heads per softmax thread
constexpr int kT = 128;                    // tokens per tile (MMA M of the score MMA)
constexpr int kDC = 512;                   // latent width
constexpr int kDR = 64;                    // RoPE key width
constexpr int kChunk = kT * 128;           // [128 rows][64 bf16] = 16 KB
constexpr int kPairBytes = 2 * kChunk;     // two 64-dim chunks = 128 latent dims
constexpr int kPairsPerTile = kDC / 128;
constexpr int kNPair = 5;                  // C_KV pair slots: ring A then ring B
constexpr int kNA = 3;                     // ring A: column pairs 0-2 (one slot each), streamed
constexpr int kHeld = kPairsPerTile - kNA; // pairs per tile held in ring B until O
constexpr int kNB = kNPair - kNA;          // ring B slots: the held pairs of two tiles
static_assert(kNB == 2 * kHeld, "ring B holds the held pairs of two tiles");
constexpr int kNKr = 2;                    // K_R slots
constexpr int kQChunk = kHC * 128;         // [16 heads][64 bf16] = 2 KB
constexpr int kQBytes = 9 * kQChunk;       // 8 chunks of q_c, 1 of q_r
constexpr int kPBytes = kT * kHC * 2;      // P^T tile, bf16
constexpr int kSoftmaxWarps = 8;
constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
constexpr int kOWarp = 2 + kSoftmaxWarps;   // issues O^T += C^T P^T
constexpr int kThreads = 32 * (kOWarp + 1);
constexpr int kTmemCols = 128;
constexpr int kSoftmaxBar = 1;             // named barrier of the softmax warps
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleLog2 = 8.f;        // M rises once an entry exceeds it by 2^8

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int kOffPair = 0;
constexpr int kOffKr = kOffPair + kNPair * kPairBytes;
constexpr int kOffQ = kOffKr + kNKr * kChunk;
constexpr int kOffP = kOffQ + kQBytes;
constexpr int kOffGpart = kOffP + 2 * kPBytes;          // float4 [4 quarters][16]: m, den, num, sr_a
constexpr int kOffGanc = kOffGpart + 4 * kHC * 16;      // int [4][16]: row of the partial argmax
constexpr int kOffWmax = kOffGanc + 4 * kHC * 4;        // float [4][16]: max entry per quarter
constexpr int kOffZred = kOffWmax + 4 * kHC * 4;        // float [4][16]
constexpr int kOffBar = kOffZred + 4 * kHC * 4;
constexpr int kNumBars = 2 * kNPair + 2 * kNA + 2 * kNKr + 2 + 4 * 2 + 2;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 16;
constexpr int kSmemAlloc = kSmemBytes + 1024;          // alignment slack
static_assert(kSmemAlloc <= 232448, "shared memory budget of one sm_100 CTA");

// TMEM columns: S buffer b: sc at 32b, sr at 32b + 16;  O^T block m: 64 + 16m
constexpr uint32_t kColS = 0;
constexpr uint32_t kColO = 64;

// error word bits (device error word [0]); [1] holds where the first one happened
constexpr int kErrTimeout = 1;

struct TcParams {
  CUtensorMap tm_c;    // c_kv  as [B*L rows][512], box [128 rows][64], 128B swizzle
  CUtensorMap tm_k;    // k_r   as [B*L rows][64],  box [128 rows][64], 128B swizzle
  CUtensorMap tm_qc;   // q_c   as [B*H rows][512], box [16 rows][64],  128B swizzle
  CUtensorMap tm_qr;   // q_r   as [B*H rows][64],  box [16 rows][64],  128B swizzle
  int B, H;
  int64_t L;
  int64_t nG;          // condensed groups (0: dense attention)
  int64_t tiles_per_seq;
  int64_t U;           // B * tiles_per_seq
  int64_t G;           // number of tile ranges (CTA groups); G <= U
  int n_hb;            // head blocks: H / 16
  int32_t* anchor;     // [B][H][nG]
  float* part_o;       // [slots][H][512]
  float* part_mz;      // [slots][H][2]
  int* err;            // device error word [2]
  uint64_t timeout_ns;
  int debug_skip_load;
  int64_t bias_rows;   // rows [0, bias_rows) get `bias` added to their score (stored-cache
  float bias;          // decode with n_G = 0: the condensed entries; 0 rows otherwise)
  int64_t win0;        // first window token, in this cache's rows (n_G g for a whole context)
  int64_t pos0;        // position of row 0 in the context (a slice's offset): anchors are
                       // written as pos0 + row, and groups start at rows that are multiples of g
  int64_t ws_slots;    // slots of part_o / part_mz (range checks)
  int64_t anchor_stride;   // anchors of (b, h) start at (b H + h) anchor_stride
  // Paged, variable-length decode (meta != null): tm_c / tm_k cover the pools
  // with a 64-row box, and a tile's two 64-token halves are loaded from their
  // own pages; sequence b's token t is row
  // block_table[b table_stride + t / page_size] page_size + t % page_size, and its
  // length, groups, tiles and the ranges come from the metadata (L, nG, U, G,
  // tiles_per_seq, win0 above are then unused; page_size is a multiple of 64).
  const int* meta;
  const int32_t* block_table;
  int64_t table_stride;   // block-table entries from one sequence's row to the next (0: one shared row)
  int page_size;
  int64_t num_pages;
};

struct Bars {
  // Ring A slot s holds column pair s, loaded alternately for the scores and
  // (again) for O; each use has its own full/empty pair, so that every barrier
  // is waited on by one thread, phase after phase.
  uint64_t* full_as;  // [kNA]  scores load landed
  uint64_t* full_ar;  // [kNA]  reload for O landed
  uint64_t* empty_as; // [kNA]  released after the score MMAs
  uint64_t* empty_ar; // [kNA]  released after O += C^T P^T
  uint64_t* full_b;   // [kNB]  ring B
  uint64_t* empty_b;  // [kNB]  released after O += C^T P^T of the slot's tile
  uint64_t* full_k;   // [kNKr]
  uint64_t* empty_k;  // [kNKr]
  uint64_t* q_full;
  uint64_t* q_empty;
  uint64_t* s_full;   // [2]  scores of a tile are in TMEM
  uint64_t* s_empty;  // [2]  the softmax has read the S buffer
  uint64_t* p_full;   // [2]  P is in shared memory and O^T is consistent
  uint64_t* o_full;   // [2]  O^T += C^T P^T of the tile using P buffer b is done
  uint64_t* drain;    // [2]  every MMA of the score / O issuer is done
};

// Records a timeout: raises the CTA's abort flag and the device error word.
__device__ __forceinline__ void record_timeout(volatile int* abort, const TcParams& p, int where) {
  *abort = 1;
  if (atomicOr(p.err, kErrTimeout) == 0) atomicExch(p.err + 1, where);
}

// Bounded wait, the loop after a first probe that found the phase incomplete.
// Returns false when the CTA's abort flag is set (if honoured) or when the
// bound runs out (then the flag and the error word are set).  The thread
// sleeps in hardware between probes (up to 100 ns each, woken when the phase
// completes), so waiting threads take few issue slots from the softmax warps
// on their sub-partition; a longer hint (1 us) measured 1% slower.
__device__ __noinline__ bool bounded_wait_slow(uint64_t* bar, uint32_t parity, volatile int* abort,
                                               const TcParams& p, int where, bool honour_abort) {
  constexpr uint32_t kSleepNs = 100;
  if (ptx::mbar_try_wait_sleep(bar, parity, kSleepNs)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (ptx::mbar_try_wait_sleep(bar, parity, kSleepNs)) return true;
    if (honour_abort && *abort) return false;
    if ((spin & 7u) == 0 && ptx::globaltimer_ns() - t0 > p.timeout_ns) {
      record_timeout(abort, p, where);
      return false;
    }
  }
}

// Bounded wait: the first probe plain and inline, because most waits find the
// phase complete and a first probe with a suspend-time hint (or a call) cost
// the hand-off time.
__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                             const TcParams& p, int where, bool honour_abort) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  return bounded_wait_slow(bar, parity, abort, p, where, honour_abort);
}

// A wait of a whole warp: every lane probes the same phase once inline (one
// shared-memory request for the warp, no divergent branch); a lane that finds
// it incomplete takes the sleeping bounded loop.  The warp reconverges here
// even when the caller ignores the verdict, so no lane waits at the next
// aligned tcgen05 instruction instead.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          const TcParams& p, int where) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const bool ok = bounded_wait_slow(bar, parity, abort, p, where, true);
  __syncwarp();
  return ok;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Statistics of one group for each of a thread's kHH heads, over W aligned
// neighbouring lanes (one token each): the max m, the lane a of its first
// occurrence (the anchor), den = sum e^{s - m}, num = sum e^{s - m} sc and the
// anchor's sr.  Butterfly rounds run over all heads at once.  Every lane of a
// group ends with the same bits: each step combines the same two values, in
// either order, and max and + are commutative.
template <int W>
__device__ __forceinline__ void group_stats(const float (&s)[kHH], const float (&sc)[kHH],
                                            const float (&sr)[kHH], int lane, float (&m)[kHH],
                                            int (&a)[kHH], float (&den)[kHH], float (&num)[kHH],
                                            float (&sra)[kHH]) {
#pragma unroll
  for (int h = 0; h < kHH; ++h) m[h] = s[h];
#pragma unroll
  for (int off = 1; off < W; off <<= 1)
#pragma unroll
    for (int h = 0; h < kHH; ++h) m[h] = fmaxf(m[h], __shfl_xor_sync(0xffffffffu, m[h], off));
  const int base = lane & ~(W - 1);
#pragma unroll
  for (int h = 0; h < kHH; ++h) {
    const uint32_t ties = __ballot_sync(0xffffffffu, s[h] == m[h]);
    const uint32_t mine = W == 32 ? ties : (ties >> base) & ((1u << (W & 31)) - 1u);
    a[h] = base + __ffs(mine) - 1;         // lowest index among the maxima
    const float e = ex2(fmaf(s[h], kLog2e, -m[h] * kLog2e));
    den[h] = e;
    num[h] = e * sc[h];
  }
#pragma unroll
  for (int off = 1; off < W; off <<= 1)
#pragma unroll
    for (int h = 0; h < kHH; ++h) {
      den[h] += __shfl_xor_sync(0xffffffffu, den[h], off);
      num[h] += __shfl_xor_sync(0xffffffffu, num[h], off);
    }
#pragma unroll
  for (int h = 0; h < kHH; ++h) sra[h] = __shfl_sync(0xffffffffu, sr[h], a[h]);
}

template <int LOG2G, bool kPaged>
__global__ void __launch_bounds__(kThreads, 1) lca_tc_kernel(const __grid_constant__ TcParams p) {
  constexpr int g = 1 << LOG2G;
  static_assert(g <= kT, "a group must fit in one tile");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  Bars bb;
  bb.full_as = bars;
  bb.full_ar = bb.full_as + kNA;
  bb.empty_as = bb.full_ar + kNA;
  bb.empty_ar = bb.empty_as + kNA;
  bb.full_b = bb.empty_ar + kNA;
  bb.empty_b = bb.full_b + kNB;
  bb.full_k = bb.empty_b + kNB;
  bb.empty_k = bb.full_k + kNKr;
  bb.q_full = bb.empty_k + kNKr;
  bb.q_empty = bb.q_full + 1;
  bb.s_full = bb.q_empty + 1;
  bb.s_empty = bb.s_full + 2;
  bb.p_full = bb.s_empty + 2;
  bb.o_full = bb.p_full + 2;
  bb.drain = bb.o_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int hb = blockIdx.x % p.n_hb;
  const int64_t c = blockIdx.x / p.n_hb;
  const int h0 = hb * kHC;
  constexpr bool paged = kPaged;   // a separate instantiation: the contiguous loops stay as they were
  // The CTA's range of tiles, for sequences of tiles_per_seq tiles each; a
  // paged batch takes its range from the metadata once the previous kernel in
  // the stream is done (below).
  int64_t u0 = c * p.U / p.G;
  int64_t n_tiles = (c + 1) * p.U / p.G - u0;
  // (sequence, tile within it) of the range's first tile; each role then steps
  // its own copy once per tile rather than dividing
  int64_t seq0 = u0 / p.tiles_per_seq;
  int64_t tile0 = u0 - seq0 * p.tiles_per_seq;
  auto seq_tiles = [&](int64_t b) -> int64_t {
    if constexpr (kPaged) return (int64_t)meta_seq(p.meta)[b].w;
    else return p.tiles_per_seq;
  };
  // the next (sequence, tile); a paged batch's sequences without tiles are
  // passed over (tps: tiles of the current sequence)
  auto step = [&](int64_t& seq, int64_t& tile, int64_t& tps) {
    if constexpr (kPaged) {
      if (++tile == tps) {
        tile = 0;
        do {
          ++seq;
          tps = seq < p.B ? seq_tiles(seq) : 1;
        } while (tps == 0);
      }
    } else {
      if (++tile == p.tiles_per_seq) { tile = 0; ++seq; }
    }
  };
  // first rows of a tile's two 64-token halves in the C_KV / K_R tensor maps
  // (contiguous: one 128-row box from the first).  A paged half that starts at
  // or past the sequence's end reads the first half's rows again: they are
  // cleared before use, and no table entry past the sequence's end is read.
  auto tile_rows = [&](int64_t b, int64_t tile, int32_t& ra, int32_t& rb) {
    if constexpr (!kPaged) {
      ra = (int32_t)(b * p.L + tile * kT);
      rb = ra + kT / 2;
      return;
    }
    const int64_t Lb = meta_seq(p.meta)[b].x;
    const int64_t tok = tile * kT;
    ra = (int32_t)paged_row(p.block_table, p.table_stride, p.page_size, p.num_pages, b, tok, p.err, 0xA04);
    rb = tok + kT / 2 < Lb ? (int32_t)paged_row(p.block_table, p.table_stride, p.page_size, p.num_pages, b,
                                                 tok + kT / 2, p.err, 0xA04)
                           : ra;
  };

  if (tid == 0) {
    for (int i = 0; i < kNA; ++i) {
      ptx::mbar_init(&bb.full_as[i], 1); ptx::mbar_init(&bb.full_ar[i], 1);
      ptx::mbar_init(&bb.empty_as[i], 1); ptx::mbar_init(&bb.empty_ar[i], 1);
    }
    for (int i = 0; i < kNB; ++i) { ptx::mbar_init(&bb.full_b[i], 1); ptx::mbar_init(&bb.empty_b[i], 1); }
    for (int i = 0; i < kNKr; ++i) { ptx::mbar_init(&bb.full_k[i], 1); ptx::mbar_init(&bb.empty_k[i], 1); }
    ptx::mbar_init(bb.q_full, 1);
    ptx::mbar_init(bb.q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bb.s_full[i], 1);
      ptx::mbar_init(&bb.s_empty[i], kSoftmaxWarps);
      ptx::mbar_init(&bb.p_full[i], kSoftmaxWarps);
      ptx::mbar_init(&bb.o_full[i], 1);
    }
    ptx::mbar_init(&bb.drain[0], 1);
    ptx::mbar_init(&bb.drain[1], 1);
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Launched as a programmatic dependent: the prologue above may overlap the end
  // of the previous kernel in the stream, and nothing below reads or writes
  // global memory before that kernel has completed and its writes are visible.
  // The combine that follows may be scheduled from here on; it waits the same way.
  // Start the range's first tile and query block on their way into L2 while the
  // previous kernel may still run: an L2 prefetch returns no data to this CTA,
  // and L2 holds every later write to those lines, so nothing read after the
  // wait below can be stale.  (One tile: prefetching two measured no better.)
  if (tid == 0 && !paged) {
    const int32_t frow = (int32_t)(seq0 * p.L + tile0 * kT);
    for (int cc = 0; cc < 8; ++cc) ptx::tma_prefetch_l2_2d(&p.tm_c, 64 * cc, frow);
    ptx::tma_prefetch_l2_2d(&p.tm_k, 0, frow);
    const int32_t qrow = (int32_t)(seq0 * p.H + h0);
    for (int k = 0; k < 8; ++k) ptx::tma_prefetch_l2_2d(&p.tm_qc, 64 * k, qrow);
    ptx::tma_prefetch_l2_2d(&p.tm_qr, 0, qrow);
  }
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();
  if constexpr (kPaged) {
    const int64_t U = p.meta[0], Ge = p.meta[1];
    u0 = 0;
    n_tiles = 0;
    seq0 = 0;
    tile0 = 0;
    if (c < Ge) {
      u0 = c * U / Ge;
      n_tiles = (c + 1) * U / Ge - u0;
      const int2 rg = meta_range(p.meta, p.B)[c];
      seq0 = rg.x;
      tile0 = rg.y;
    }
  }
  const int64_t tps0 = n_tiles > 0 ? seq_tiles(seq0) : 1;

  if (warp == 0 && lane == 0) {
    // ===================================================== TMA producer
    // Two rings of 32 KB column-pair slots.  Ring B (two slots) holds pair 3 of
    // a tile from its load until O += C^T P^T of that tile, for two tiles at a
    // time.  Ring A (one slot per pair 0-2) streams each of those pairs twice:
    // once for the scores (kept in L2 with an evict-last hint) and once more,
    // read back from L2, for O.  So the scores of tile i+1 complete while the
    // softmax of tile i runs, and the softmaxes follow each other directly.
    // Per tile the load order is
    //   K_R(i), A: i.p0, i.p1, i.p2,  B: i.p3,  A: (i-1).p0', p1', p2'
    // and the last tile's reloads come after the loop; each load waits only on
    // MMAs that need no later load of this order.
    ptx::prefetch_tmap(&p.tm_c);
    ptx::prefetch_tmap(&p.tm_k);
    ptx::prefetch_tmap(&p.tm_qc);
    ptx::prefetch_tmap(&p.tm_qr);
    const uint64_t keep = ptx::l2_policy_evict_last();    // pairs 0-2: read again from L2
    const uint64_t once = ptx::l2_policy_evict_first();   // read once
    // last phase issued on each full barrier (-1: none), so that every copy can
    // be waited for before the CTA exits
    int issued_as[kNA], issued_ar[kNA], issued_b[kNB], issued_k[kNKr];
#pragma unroll
    for (int i = 0; i < kNA; ++i) { issued_as[i] = -1; issued_ar[i] = -1; }
#pragma unroll
    for (int i = 0; i < kNB; ++i) issued_b[i] = -1;
#pragma unroll
    for (int i = 0; i < kNKr; ++i) issued_k[i] = -1;
    int issued_q = -1;
    int64_t nb = 0, nk = 0;
    int seg = -1;
    int64_t cur_b = -1;
    bool ok = true;
    const int64_t T = n_tiles;
    auto issue = [&](uint64_t* full, int slot, int32_t row, int32_t row_b, int pr, uint64_t policy) {
      if (!LCA_CHECK(p.err, slot >= 0 && slot < kNPair && pr >= 0 && pr < kPairsPerTile, 0xD01)) return;
      ptx::mbar_arrive_expect_tx(full, kPairBytes);
      uint8_t* dst = smem + kOffPair + slot * kPairBytes;
      if constexpr (!kPaged) {
        ptx::tma_load_2d_hint(dst, &p.tm_c, 128 * pr, row, full, policy);
        ptx::tma_load_2d_hint(dst + kChunk, &p.tm_c, 128 * pr + 64, row, full, policy);
      } else {   // 64-row boxes: the second half lands 8 KB (eight swizzle atoms) further on
        for (int ch = 0; ch < 2; ++ch) {
          ptx::tma_load_2d_hint(dst + ch * kChunk, &p.tm_c, 128 * pr + 64 * ch, row, full, policy);
          ptx::tma_load_2d_hint(dst + ch * kChunk + kChunk / 2, &p.tm_c, 128 * pr + 64 * ch, row_b, full,
                                policy);
        }
      }
    };
    // ring A, pair pr (slot pr) of tile i for its scores.  The slot's previous content:
    // nothing (i = 0), the scores load of tile 0 (i = 1), else the reload of i-2.
    auto load_scores_a = [&](int64_t i, int32_t row, int32_t row_b, int pr) -> bool {
      if (i == 1 && !bounded_wait(&bb.empty_as[pr], 0, abort_flag, p, 0x102, true)) return false;
      if (i >= 2 && !bounded_wait(&bb.empty_ar[pr], (uint32_t)(i - 2) & 1, abort_flag, p, 0x102, true))
        return false;
      issue(&bb.full_as[pr], pr, row, row_b, pr, keep);
#pragma unroll
      for (int q = 0; q < kNA; ++q) if (q == pr) issued_as[q] = (int)i;
      return true;
    };
    // ring A, pair pr of tile j again for O.  The slot's previous content: the
    // scores load of tile j+1, or for the last tile the reload of j-1 (the
    // scores load of tile 0 when it is the only tile).
    auto load_reload_a = [&](int64_t j, int32_t row, int32_t row_b, int pr) -> bool {
      bool w;
      if (j + 1 < T) w = bounded_wait(&bb.empty_as[pr], (uint32_t)(j + 1) & 1, abort_flag, p, 0x103, true);
      else if (j >= 1) w = bounded_wait(&bb.empty_ar[pr], (uint32_t)(j - 1) & 1, abort_flag, p, 0x103, true);
      else w = bounded_wait(&bb.empty_as[pr], 0, abort_flag, p, 0x103, true);
      if (!w) return false;
      issue(&bb.full_ar[pr], pr, row, row_b, pr, once);
#pragma unroll
      for (int q = 0; q < kNA; ++q) if (q == pr) issued_ar[q] = (int)j;
      return true;
    };
    // ring B: the next slot, after O of the tile two back that held it
    auto load_b = [&](int32_t row, int32_t row_b, int pr) -> bool {
      const int cs = (int)(nb % kNB);
      const int ck = (int)(nb / kNB);
      if (ck >= 1 && !bounded_wait(&bb.empty_b[cs], (ck - 1) & 1, abort_flag, p, 0x104, true)) return false;
      issue(&bb.full_b[cs], kNA + cs, row, row_b, pr, once);
#pragma unroll
      for (int q = 0; q < kNB; ++q) if (q == cs) issued_b[q] = ck;
      ++nb;
      return true;
    };
    int64_t pseq = seq0, ptile = tile0;
    int64_t ptps = tps0;
    int32_t prev_row = 0, prev_row_b = 0;   // first rows of the previous tile's halves
    // each tile's rows are looked up a tile ahead (a paged batch reads its
    // block table), so that the lookup's latency passes during the waits
    int32_t next_row = 0, next_row_b = 0;
    if (kPaged && n_tiles > 0) tile_rows(pseq, ptile, next_row, next_row_b);
    for (int64_t i = 0; i < n_tiles && ok; ++i) {
      const int64_t b = pseq;
      if (b != cur_b) {
        cur_b = b;
        ++seg;
        if (seg >= 1) ok = bounded_wait(bb.q_empty, (seg - 1) & 1, abort_flag, p, 0x100, true);
        if (!ok) break;
        ptx::mbar_arrive_expect_tx(bb.q_full, kQBytes);
        const int32_t qrow = (int32_t)(b * p.H + h0);
        for (int k = 0; k < 8; ++k)
          ptx::tma_load_2d(smem + kOffQ + k * kQChunk, &p.tm_qc, 64 * k, qrow, bb.q_full);
        ptx::tma_load_2d(smem + kOffQ + 8 * kQChunk, &p.tm_qr, 0, qrow, bb.q_full);
        issued_q = seg;
      }
      int32_t row = next_row, row_b = next_row_b;
      if constexpr (!kPaged) tile_rows(b, ptile, row, row_b);
      {
        const int ks = (int)(nk % kNKr);
        const int kk = (int)(nk / kNKr);
        if (kk >= 1) ok = bounded_wait(&bb.empty_k[ks], (kk - 1) & 1, abort_flag, p, 0x101, true);
        if (!ok) break;
        if (!(p.debug_skip_load && nk == 0)) {
          ptx::mbar_arrive_expect_tx(&bb.full_k[ks], kChunk);
          ptx::tma_load_2d_hint(smem + kOffKr + ks * kChunk, &p.tm_k, 0, row, &bb.full_k[ks], once);
          if constexpr (kPaged)
            ptx::tma_load_2d_hint(smem + kOffKr + ks * kChunk + kChunk / 2, &p.tm_k, 0, row_b, &bb.full_k[ks],
                                  once);
#pragma unroll
          for (int q = 0; q < kNKr; ++q) if (q == ks) issued_k[q] = kk;
        }
        ++nk;
      }
      for (int pr = 0; pr < kNA && ok; ++pr) ok = load_scores_a(i, row, row_b, pr);
      for (int pr = kNA; pr < kPairsPerTile && ok; ++pr) ok = load_b(row, row_b, pr);
      for (int pr = 0; pr < kNA && ok && i >= 1; ++pr) ok = load_reload_a(i - 1, prev_row, prev_row_b, pr);
      prev_row = row;
      prev_row_b = row_b;
      step(pseq, ptile, ptps);
      if (kPaged && i + 1 < n_tiles) tile_rows(pseq, ptile, next_row, next_row_b);
    }
    for (int pr = 0; pr < kNA && ok && T > 0; ++pr)
      ok = load_reload_a(T - 1, prev_row, prev_row_b, pr);   // the last tile
    // Let every copy this thread started land before the CTA can exit.
#pragma unroll
    for (int i = 0; i < kNA; ++i) {
      if (issued_as[i] >= 0) bounded_wait(&bb.full_as[i], issued_as[i] & 1, abort_flag, p, 0x1F0, false);
      if (issued_ar[i] >= 0) bounded_wait(&bb.full_ar[i], issued_ar[i] & 1, abort_flag, p, 0x1F0, false);
    }
#pragma unroll
    for (int i = 0; i < kNB; ++i)
      if (issued_b[i] >= 0) bounded_wait(&bb.full_b[i], issued_b[i] & 1, abort_flag, p, 0x1F0, false);
#pragma unroll
    for (int i = 0; i < kNKr; ++i)
      if (issued_k[i] >= 0) bounded_wait(&bb.full_k[i], issued_k[i] & 1, abort_flag, p, 0x1F1, false);
    if (issued_q >= 0) bounded_wait(bb.q_full, issued_q & 1, abort_flag, p, 0x1F2, false);
  } else if (warp == 1 && lane == 0) {
    // ===================================================== score MMA issuer
    // Tile t: K_R (sr first), then column pairs 0-2 from ring A (each slot
    // released after its MMAs) and pair 3 from ring B (held for O), each once
    // it has landed; also waits for the S buffer to be released and, for a new
    // sequence part, for the query block.
    constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(kT, kHC, 0, 0);   // K-major A and B
    // Descriptor templates; a K step adds (bytes >> 4) to the start-address field.
    const uint64_t d_pair = ptx::smem_desc(ptx::smem_u32(smem + kOffPair), 16, 1024, ptx::kSwizzle128B);
    const uint64_t d_kr = ptx::smem_desc(ptx::smem_u32(smem + kOffKr), 16, 1024, ptx::kSwizzle128B);
    const uint64_t d_q = ptx::smem_desc(ptx::smem_u32(smem + kOffQ), 16, 1024, ptx::kSwizzle128B);
    int seg = -1;
    int64_t cur_b = -1;
    bool ok = true;
    int64_t sseq = seq0, stile = tile0, stps = tps0;
    for (int64_t t = 0; t < n_tiles && ok; ++t, step(sseq, stile, stps)) {
      const int64_t b = sseq;
      const bool last_in_seg = t + 1 == n_tiles || stile + 1 == (kPaged ? stps : p.tiles_per_seq);
      const int buf = (int)(t & 1);
      if (b != cur_b) {
        cur_b = b;
        ++seg;
        ok = bounded_wait(bb.q_full, seg & 1, abort_flag, p, 0x200, true);
        if (!ok) break;
      }
      if (t >= 2)
        ok = bounded_wait(&bb.s_empty[buf], (uint32_t)((t >> 1) - 1) & 1, abort_flag, p, 0x201, true);
      if (ok) ok = bounded_wait(&bb.full_k[t % kNKr], (uint32_t)(t / kNKr) & 1, abort_flag, p, 0x202, true);
      if (!ok) break;
      ptx::tc_fence_after();
      {  // sr = K_R . q_r^T
        const uint32_t d_sr = tmem + kColS + 32 * buf + 16;
        const uint64_t a0 = d_kr + (uint64_t)(((t % kNKr) * kChunk) >> 4);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          ptx::mma_bf16_ss(d_sr, a0 + (uint64_t)((32 * k) >> 4),
                           d_q + (uint64_t)((8 * kQChunk + 32 * k) >> 4), kIdescS, k > 0);
        ptx::mma_commit(&bb.empty_k[t % kNKr]);
      }
      for (int pr = 0; pr < kPairsPerTile; ++pr) {   // sc += C_KV[:, pair] . q_c[pair]^T
        const int64_t n = kHeld * t + (pr - kNA);     // ring B index of a held pair
        const int cs = pr < kNA ? pr : kNA + (int)(n % kNB);   // shared-memory slot
        if (!LCA_CHECK(p.err, cs >= 0 && cs < kNPair && buf < 2, 0xD02)) { ok = false; break; }
        ok = pr < kNA ? bounded_wait(&bb.full_as[pr], (uint32_t)t & 1, abort_flag, p, 0x203, true)
                      : bounded_wait(&bb.full_b[cs - kNA], (uint32_t)(n / kNB) & 1, abort_flag, p, 0x203, true);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t d_sc = tmem + kColS + 32 * buf;
        const uint64_t a0 = d_pair + (uint64_t)((cs * kPairBytes) >> 4);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
#pragma unroll
          for (int k = 0; k < 4; ++k)
            ptx::mma_bf16_ss(d_sc, a0 + (uint64_t)((ch * kChunk + 32 * k) >> 4),
                             d_q + (uint64_t)(((2 * pr + ch) * kQChunk + 32 * k) >> 4), kIdescS,
                             (pr | ch | k) != 0);
        }
        if (pr < kNA) ptx::mma_commit(&bb.empty_as[pr]);   // ring A: read again later from L2
      }
      if (!ok) break;
      ptx::mma_commit(&bb.s_full[buf]);
      if (last_in_seg) ptx::mma_commit(bb.q_empty);
    }
    // Every MMA issued here must finish before TMEM is freed.
    ptx::mma_commit(&bb.drain[0]);
    bounded_wait(&bb.drain[0], 0, abort_flag, p, 0x2F0, false);
  } else if (warp == kOWarp && lane == 0) {
    // ===================================================== O MMA issuer
    // Tile j once its P is written: O^T += C^T P^T over pair 3 (held in ring B)
    // and pairs 0-2 (loaded again into ring A), releasing each slot after; a
    // sequence part starts the accumulator afresh.
    constexpr uint32_t kIdescP = ptx::idesc_bf16_f32(128, kHC, 1, 1);  // MN-major A and B
    // A = C^T, M = 128 latent dims (two 64-dim atoms 16 KB apart), K = 16 tokens
    const uint64_t d_ct = ptx::smem_desc(ptx::smem_u32(smem + kOffPair), kChunk, 1024, ptx::kSwizzle128B);
    // B = P^T, N = 16 heads (8-head core blocks 2 KB apart), K = 16 tokens
    const uint64_t d_pt = ptx::smem_desc(ptx::smem_u32(smem + kOffP), 128, 2048, ptx::kSwizzleNone);
    int64_t oseq = seq0, otile = tile0, otps = tps0;
    for (int64_t j = 0; j < n_tiles; ++j, step(oseq, otile, otps)) {
      const int buf = (int)(j & 1);
      if (!bounded_wait(&bb.p_full[buf], (uint32_t)(j >> 1) & 1, abort_flag, p, 0x204, true)) break;
      ptx::tc_fence_after();
      const uint32_t acc0 = (j > 0 && otile > 0) ? 1u : 0u;   // a sequence part starts afresh
      const uint64_t bpt = d_pt + (uint64_t)((buf * kPBytes) >> 4);
#pragma unroll 1
      for (int mm = 0; mm < kPairsPerTile; ++mm) {
        const int m = (mm + kNA) % kPairsPerTile;   // held pairs (ring B) first, then the reloads
        const int64_t n = kHeld * j + (m - kNA);      // ring B index of a held pair
        const int cs = m >= kNA ? kNA + (int)(n % kNB) : m;  // shared-memory slot
        if (!LCA_CHECK(p.err, cs >= 0 && cs < kNPair && m < kPairsPerTile, 0xD03)) break;
        const bool okw = m >= kNA ? bounded_wait(&bb.full_b[cs - kNA], (uint32_t)(n / kNB) & 1, abort_flag, p, 0x206, true)
                                  : bounded_wait(&bb.full_ar[m], (uint32_t)j & 1, abort_flag, p, 0x206, true);
        if (!okw) break;
        ptx::tc_fence_after();
        const uint32_t d_o = tmem + kColO + 16 * m;
        const uint64_t act = d_ct + (uint64_t)((cs * kPairBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::mma_bf16_ss(d_o, act + (uint64_t)(kk * (2048 >> 4)),
                           bpt + (uint64_t)(kk * (256 >> 4)), kIdescP, kk > 0 ? 1u : acc0);
        ptx::mma_commit(m >= kNA ? &bb.empty_b[cs - kNA] : &bb.empty_ar[m]);
      }
      ptx::mma_commit(&bb.o_full[buf]);
    }
    ptx::mma_commit(&bb.drain[1]);
    bounded_wait(&bb.drain[1], 0, abort_flag, p, 0x2F1, false);
  } else if (warp >= 2 && warp < kOWarp) {
    // ===================================================== softmax warps
    // A failed wait only raises the abort flag; the softmax warps leave the
    // tile loop together, at the one checkpoint barrier of each tile, so no
    // warp is ever left waiting at a named barrier.
    const int q4 = warp & 3;             // TMEM lane quarter this warp may access
    const int hh = (warp - 2) >> 2;      // which 8 of the 16 heads
    const int row = q4 * 32 + lane;      // token row of the tile owned by this thread
    const uint32_t t_cols = tmem + ((uint32_t)(q4 * 32) << 16) + kHH * hh;   // lane, first head column
    float4* gpart = reinterpret_cast<float4*>(smem + kOffGpart);   // [4][16]
    int* ganc = reinterpret_cast<int*>(smem + kOffGanc);           // [4][16]
    float* wmax_s = reinterpret_cast<float*>(smem + kOffWmax);     // [4][16]
    float* zred = reinterpret_cast<float*>(smem + kOffZred);       // [4][16]
    uint8_t* pbase = smem + kOffP;

    float Zt[kHH], Mh[kHH];    // this thread's rows' share of Z; the reference max
#pragma unroll
    for (int h = 0; h < kHH; ++h) { Zt[h] = 0.f; Mh[h] = -INFINITY; }

    int64_t cseq = seq0, ctile = tile0, ctps = tps0;
    // the current sequence's length, groups and first window token
    int64_t sL = 0, snG = 0, swin0 = 0, s_of = -1;
    for (int64_t i = 0; i < n_tiles; ++i, step(cseq, ctile, ctps)) {
      const int64_t b = cseq, tile = ctile;
      const bool last_in_seg = i + 1 == n_tiles || tile + 1 == (kPaged ? ctps : p.tiles_per_seq);
      if constexpr (kPaged) {
        if (b != s_of) {
          s_of = b;
          const int4 rec = meta_seq(p.meta)[b];
          sL = rec.x;
          snG = rec.z;
          swin0 = snG * g;
        }
      } else {
        sL = p.L;
        snG = p.nG;
        swin0 = p.win0;
      }
      const int buf = (int)(i & 1);
      const int kb = (int)(i >> 1);
      warp_wait(&bb.s_full[buf], kb & 1, abort_flag, p, 0x300);
      ptx::tc_fence_after();
      float sc[kHH], sr[kHH], s[kHH];
      ptx::tmem_ld8(t_cols + kColS + 32 * buf, sc);
      ptx::tmem_ld8(t_cols + kColS + 32 * buf + 16, sr);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bb.s_empty[buf]);
#pragma unroll
      for (int h = 0; h < kHH; ++h) s[h] = sc[h] + sr[h];

      const int64_t tok0 = tile * kT;
      const int64_t t = tok0 + row;
      const bool valid = t < sL;
      const bool grouped = t < swin0;
      if (t < p.bias_rows) {
#pragma unroll
        for (int h = 0; h < kHH; ++h) s[h] += p.bias;
      }
      const bool tile_groups = (g > 1) && (tok0 < swin0);   // tile-uniform
      int32_t* anc = p.anchor + ((int64_t)b * p.H + h0 + kHH * hh) * p.anchor_stride;

      // ---- step 2: condense; ent = the softmax entry this token stands for
      float kj[kHH], ent[kHH];
#pragma unroll
      for (int h = 0; h < kHH; ++h) { kj[h] = 0.f; ent[h] = valid ? s[h] : -INFINITY; }
      if (g == 1 && grouped) {
#pragma unroll
        for (int h = 0; h < kHH; ++h)
          if (LCA_CHECK(p.err, t < snG && h0 + kHH * hh + h < p.H, 0xD04))
            anc[(int64_t)h * p.anchor_stride + t] = (int32_t)(p.pos0 + t);
      }
      if (tile_groups) {
        const int64_t jg = t / g;                 // this token's group (if grouped)
        constexpr int W = g < 32 ? g : 32;
        float m[kHH], den[kHH], num[kHH], sra[kHH];
        int a[kHH];
        group_stats<W>(s, sc, sr, lane, m, a, den, num, sra);
        if (g > 32) {
          // 64 or 128 tokens: merge the per-warp statistics of the group's warps
#pragma unroll
          for (int h = 0; h < kHH; ++h)
            if (lane == 0) {
              gpart[q4 * kHC + kHH * hh + h] = make_float4(m[h], den[h], num[h], sra[h]);
              ganc[q4 * kHC + kHH * hh + h] = q4 * 32 + a[h];
            }
          ptx::named_bar_sync(kSoftmaxBar, kSoftmaxThreads);
          constexpr int NQ = g / 32 > 0 ? g / 32 : 1;   // lane quarters per group
          const int qb = q4 & ~(NQ - 1);
#pragma unroll
          for (int h = 0; h < kHH; ++h) {
            float4 r = gpart[qb * kHC + kHH * hh + h];
            int ar = ganc[qb * kHC + kHH * hh + h];
#pragma unroll
            for (int k = 1; k < NQ; ++k) {
              const float4 o = gpart[(qb + k) * kHC + kHH * hh + h];
              const float mm = fmaxf(r.x, o.x);
              const float f1 = ex2((r.x - mm) * kLog2e), f2 = ex2((o.x - mm) * kLog2e);
              r.y = r.y * f1 + o.y * f2;
              r.z = r.z * f1 + o.z * f2;
              if (o.x > r.x) { ar = ganc[(qb + k) * kHC + kHH * hh + h]; r.w = o.w; }   // a tie keeps the lower row
              r.x = mm;
            }
            m[h] = r.x; den[h] = r.y; num[h] = r.z; sra[h] = r.w; a[h] = ar;
          }
        } else {
#pragma unroll
          for (int h = 0; h < kHH; ++h) a[h] += q4 * 32;   // lane -> tile row
        }
        if (grouped) {
#pragma unroll
          for (int h = 0; h < kHH; ++h) {
            const float S = __fdividef(num[h], den[h]) + sra[h];
            kj[h] = S - m[h] - lg2(den[h]) * kLn2;
            ent[h] = S;
          }
          const bool writer = g > 32 ? (lane == 0 && (q4 & (g / 32 - 1)) == 0) : (lane & (W - 1)) == 0;
          if (writer) {
#pragma unroll
            for (int h = 0; h < kHH; ++h)
              if (LCA_CHECK(p.err, jg < snG && a[h] >= 0 && a[h] < kT, 0xD05))
                anc[(int64_t)h * p.anchor_stride + jg] = (int32_t)(p.pos0 + tok0 + a[h]);
          }
        }
      }

      // ---- step 3: reference max.  The first tile of a sequence part sets it
      // to the tile's largest entry; later it rises only when an entry exceeds
      // it by more than 2^8, and then Z and O^T are rescaled.  The checkpoint
      // barrier ORs "abort, or take this slow path" over the softmax threads.
      const bool first = i == 0 || tile == 0;
      bool need = first;
#pragma unroll
      for (int h = 0; h < kHH; ++h) need = need || (ent[h] - Mh[h]) * kLog2e > kRescaleLog2;
      if (ptx::named_bar_or(kSoftmaxBar, kSoftmaxThreads, need || *abort_flag != 0)) {
        if (ptx::named_bar_or(kSoftmaxBar, kSoftmaxThreads, *abort_flag != 0)) break;
#pragma unroll
        for (int h = 0; h < kHH; ++h) {
          float v = ent[h];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
          if (lane == 0) wmax_s[q4 * kHC + kHH * hh + h] = v;
        }
        ptx::named_bar_sync(kSoftmaxBar, kSoftmaxThreads);
        float alpha[kHH];
        bool rescale = false;
#pragma unroll
        for (int h = 0; h < kHH; ++h) {
          const int hc = kHH * hh + h;
          const float mt = fmaxf(fmaxf(wmax_s[hc], wmax_s[kHC + hc]),
                                 fmaxf(wmax_s[2 * kHC + hc], wmax_s[3 * kHC + hc]));
          alpha[h] = 1.f;
          if (first) {
            Mh[h] = mt;
          } else if ((mt - Mh[h]) * kLog2e > kRescaleLog2) {
            alpha[h] = ex2((Mh[h] - mt) * kLog2e);
            Mh[h] = mt;
            rescale = true;
          }
        }
        if (rescale) {   // the same decision in every lane of a warp (same heads)
#pragma unroll
          for (int h = 0; h < kHH; ++h) Zt[h] *= alpha[h];
          // O^T of the previous tile must be complete before it is scaled
          warp_wait(&bb.o_full[(i - 1) & 1], (uint32_t)((i - 1) >> 1) & 1, abort_flag, p, 0x303);
          ptx::tc_fence_after();
#pragma unroll
          for (int m = 0; m < kPairsPerTile; ++m) {
            float o[kHH];
            ptx::tmem_ld8(t_cols + kColO + 16 * m, o);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int h = 0; h < kHH; ++h) o[h] *= alpha[h];
            ptx::tmem_st8(t_cols + kColO + 16 * m, o);
          }
          ptx::tmem_wait_st();
        }
      }

      // ---- per-token weights into the P^T tile
      uint32_t pk[kHH / 2];
#pragma unroll
      for (int h2 = 0; h2 < kHH / 2; ++h2) {
        float pv[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int h = 2 * h2 + e;
          pv[e] = valid ? ex2(fmaf(s[h] + kj[h], kLog2e, -Mh[h] * kLog2e)) : 0.f;
        }
        pk[h2] = pack_bf16x2(pv[0], pv[1]);
        const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&pk[h2]);
        Zt[2 * h2] += __low2float(v);          // Z from the rounded P
        Zt[2 * h2 + 1] += __high2float(v);
      }
      // A paged sequence's last tile: the rows past its last token, in the four
      // pair slots O reads (pair 3 held in ring B, pairs 0-2 reloaded into ring
      // A), hold whatever the pool has there.  Their weights are 0, but 0 x NaN
      // is not, so the softmax warps clear them before P is released.  The
      // reload cannot be overtaken: the slot's next load waits for O of this
      // tile, which waits for P.
      if (kPaged && (tile + 1) * kT > sL) {
        const int n_valid = (int)(sL - tile * kT);
        for (int pr = 0; pr < kNA; ++pr) warp_wait(&bb.full_ar[pr], (uint32_t)i & 1, abort_flag, p, 0x306);
        const int held = kNA + (int)((kHeld * i) % kNB);
        for (int idx = (warp - 2) * 32 + lane; idx < 4 * 2 * kT * 8; idx += kSoftmaxThreads) {
          const int row = (idx >> 3) & (kT - 1);    // 8 chunks of 16 bytes a row
          const int sl = idx >> 11;                 // slot 0-2 (ring A) or 3 (ring B)
          const int slot = sl < kNA ? sl : held;
          if (row >= n_valid)
            *reinterpret_cast<uint4*>(smem + kOffPair + slot * kPairBytes + ((idx >> 10) & 1) * kChunk +
                                      row * 128 + (idx & 7) * 16) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      // the P buffer is free once O of the tile two back is done
      if (i >= 2) warp_wait(&bb.o_full[buf], (uint32_t)((i - 2) >> 1) & 1, abort_flag, p, 0x305);
      // MN-major core matrices: token row -> K, head -> N (8-head blocks 2 KB apart)
      uint8_t* prow = pbase + buf * kPBytes + hh * 2048 + (row >> 3) * 128 + (row & 7) * 16;
      if (LCA_CHECK(p.err, prow + 16 <= pbase + 2 * kPBytes, 0xD06))
        *reinterpret_cast<uint4*>(prow) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      ptx::fence_proxy_async_smem();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bb.p_full[buf]);

      if (last_in_seg) {
        // the partial of the range's part of sequence b
        const int64_t slot = b + c;
        const bool slot_ok = LCA_CHECK(p.err, slot < p.ws_slots, 0xD07);
        warp_wait(&bb.o_full[buf], (uint32_t)kb & 1, abort_flag, p, 0x304);
        ptx::tc_fence_after();
#pragma unroll 1
        for (int m = 0; m < kPairsPerTile; ++m) {
          float o[kHH];
          ptx::tmem_ld8(t_cols + kColO + 16 * m, o);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < kHH; ++h)
            if (slot_ok) p.part_o[(slot * p.H + h0 + kHH * hh + h) * kDC + 128 * m + row] = o[h];
        }
        ptx::tc_fence_before();
#pragma unroll
        for (int h = 0; h < kHH; ++h) {
          float z = Zt[h];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
          if (lane == 0) zred[q4 * kHC + kHH * hh + h] = z;
        }
        ptx::named_bar_sync(kSoftmaxBar, kSoftmaxThreads);
        if (q4 == 2 && lane < kHH && slot_ok) {   // warps 2 and 6: heads 0-7 and 8-15
          float Mv = 0.f;
#pragma unroll
          for (int h = 0; h < kHH; ++h) if (h == lane) Mv = Mh[h];
          const int hc = kHH * hh + lane;
          const float z = (zred[hc] + zred[kHC + hc]) + (zred[2 * kHC + hc] + zred[3 * kHC + hc]);
          p.part_mz[(slot * p.H + h0 + hc) * 2 + 0] = Mv;
          p.part_mz[(slot * p.H + h0 + hc) * 2 + 1] = z;
        }
        ptx::named_bar_sync(kSoftmaxBar, kSoftmaxThreads);
#pragma unroll
        for (int h = 0; h < kHH; ++h) { Zt[h] = 0.f; Mh[h] = -INFINITY; }
      }
    }
  }

  // ===================================================== teardown
  // Lanes that skipped a one-lane role wait for their lane 0 first.
  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace tc
}  // namespace lca
