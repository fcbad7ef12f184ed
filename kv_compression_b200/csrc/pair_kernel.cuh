// pair_kernel.cuh -- LCA / dense-MLA decode for 128 heads sharing one latent,
// on a cluster of two CTAs that split the latent width: tcgen05 tensor cores,
// TMEM accumulators and operands, TMA tile loads, distributed shared memory
// (sm_100a), bf16 latents, fp32 accumulation.
//
// What one cluster computes ("Latent-Condensed Transformer for Efficient Long
// Context Modeling", section 2, "O Algoritmo LCA", steps 1-3) for 128 heads of
// one sequence over a contiguous range of 64-token tiles.  CTA r of the pair
// holds latent dims [256 r, 256 r + 256) of every tile.  Heads sit in TMEM
// lanes (head m = lane m); CTA r owns the 16-head blocks m with
// (m / 16) % 2 == r, so every lane quarter -- every SM sub-partition -- holds
// 16 own heads and 16 of the other CTA's ("peer") heads.
//   scores     S_r[128 heads x 64 tokens] = Q_c[:, dims_r] . C_KV[tile, dims_r]^T
//              (partial over its own dims) and sr = q_r . K_R^T, in TMEM (q_r
//              itself sits in TMEM as the A operand).  Each CTA sends the
//              partial scores of its peer heads to the other CTA (st.async into
//              its shared memory, per lane quarter), so each head's full score
//              sc_t = S_0 + S_1 is formed by the CTA that owns the head;
//   condense   (step 2) two threads hold one head, 32 consecutive tokens each,
//              so a group of g <= 32 tokens is reduced inside a thread: max,
//              lowest-index argmax (the anchor a_j), e_t = e^{s_t - m_j},
//              den_j = sum e_t, num_j = sum e_t sc_t and the condensed logit
//              S_j = num_j / den_j + sr_{a_j}; a 64-token group merges its two
//              threads with a shuffle;
//   attend     (step 3) softmax over [condensed || window] against a reference
//              max M per head: a grouped token weighs e_t e^{S_j - M} / den_j,
//              a window token e^{s_t - M}.  The bf16 weights P[128 heads x 64
//              tokens] are the A operand of O[128 heads x 256 dims_r] +=
//              P . C_KV[tile, dims_r], read from shared memory: the owner
//              writes its heads' rows into its own P buffer and copies them
//              (bulk shared-to-distributed-shared copies) into the peer's, so
//              O of a tile starts as soon as both halves have landed.  M rises
//              only when an entry exceeds it by more than 2^8; the owner
//              rescales its O rows, and the factors (with one flag per lane
//              quarter) travel with P so that the O MMA issuer of the other
//              CTA has its shipper warps rescale that CTA's copy of the rows
//              first (rare).
// Each CTA writes its dims of every head's partial O, the owner CTA the
// head's (M, Z); the combine kernel merges the ranges of a sequence.
//
// Every C_KV byte is read from HBM once and into shared memory once (each CTA
// loads only its half); K_R is loaded by both CTAs.
//
// TMEM (512 columns): O at 0 (256), partial sc in two buffers at 256 and 320,
// sr at 384 (one buffer: it is read at the start of a tile), q_r of a sequence
// in two buffers at 448 and 480 (bf16 pairs).
//
// Roles (352 threads): warp 0 lane 0 issues TMA loads; warp 1 allocates TMEM
// and its lane 0 issues the score MMAs; warp 2 lane 0 issues the O MMAs and
// decides, from the peer's per-quarter flags, whether a tile needs the peer
// rows rescaled; warps 3-6 run the softmax of the own heads of lane quarter
// (warp % 4) and load each sequence's q_r into TMEM; warps 7-10 tell the peer
// when their quarter's softmax has read the received partials (the
// cluster-scope release, kept off the softmax warps), ship the partial scores
// of the peer heads of their quarter a tile ahead and, one tile behind,
// rescale (on request) and write out those heads' O rows.
// Completion of O is only ever waited on barriers whose every phase the
// waiter observes in order (a parity wait on a barrier two phases ahead would
// pass early).  Waits suspend in hardware (mbarrier.try_wait) and are bounded;
// when a bound runs out the CTA records the error, stops issuing work, waits
// for its own copies and MMAs in flight, frees TMEM and exits after its peer.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>

#include "checks.cuh"
#include "paged_kernel.cuh"
#include "ptx.cuh"

namespace lca {
namespace pair {

constexpr int kHeads = 128;                 // heads per cluster: M of every MMA
constexpr int kOwn = 64;                    // heads whose softmax a CTA runs
constexpr int kT = 64;                      // tokens per tile: N of the score MMAs
constexpr int kHalfT = 32;                  // tokens per softmax thread
constexpr int kDC = 512;                    // latent width
constexpr int kDR = 64;                     // RoPE key width
constexpr int kDim = kDC / 2;               // latent dims per CTA
constexpr int kAtoms = kDim / 64;           // [rows][64 dims] 128B-swizzled atoms per tile half
constexpr int kNS = 3;                      // C_KV stages
constexpr int kNKr = 2;                     // K_R slots
constexpr int kQcAtom = kHeads * 128;       // [128 heads][64 bf16] = 16 KB
constexpr int kCAtom = kT * 128;            // [64 tokens][64 bf16] = 8 KB
constexpr int kStage = kAtoms * kCAtom;     // 32 KB
constexpr int kKrBytes = kT * 128;          // 8 KB
constexpr int kPBytes = kHeads * kT * 2;    // P[128 heads][64 tokens] bf16, K-major, 16 KB
constexpr int kRecvBytes = kOwn * kT * 4;   // partial scores from the peer, 16 KB
// Messages travel per lane quarter: the 16 heads of quarter q come from the
// peer's warp of the same quarter and complete their own barrier, so a
// quarter waits only for its rows and each barrier takes a quarter of the
// transaction updates.
constexpr int kRecvQBytes = kRecvBytes / 4;               // 16 heads x 64 tokens x 4 B
constexpr int kFacChunk = 20;                             // 16 factors, a flag word, 3 words of padding
constexpr int kPQBytes = 16 * kT * 2 + kFacChunk * 4;     // 16 rows of P + their factors and flag
constexpr int kThreads = 32 * 11;
constexpr int kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.f;

// shared memory map (offsets from a 1024-byte aligned base; equal in both CTAs)
constexpr int kOffQc = 0;
constexpr int kOffC = kOffQc + kAtoms * kQcAtom;
constexpr int kOffKr = kOffC + kNS * kStage;
constexpr int kOffP = kOffKr + kNKr * kKrBytes;            // [2] P tiles
constexpr int kOffRecv = kOffP + 2 * kPBytes;
// [2 buffers][4 quarters][2 CTAs] chunks of kFacChunk floats: the rescale
// factors of a quarter's 16 rows of one CTA, then a flag word (1 when one of
// them is not 1), copied to the peer with the rows of P
constexpr int kOffAlpha = kOffRecv + kRecvBytes;
constexpr int kOffFlag = kOffAlpha + 2 * 4 * 2 * kFacChunk * 4;   // int [4]: peer rows need a rescale
constexpr int kOffBar = kOffFlag + 16;
constexpr int kNumBars = 53;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 16;
constexpr int kSmemAlloc = kSmemBytes + 1024;
static_assert(kSmemAlloc <= 232448, "shared memory budget of one sm_100 CTA");
static_assert(kOffC % 1024 == 0 && kOffKr % 1024 == 0 && kOffP % 1024 == 0, "swizzle atoms");
static_assert(kOffRecv % 16 == 0 && kOffAlpha % 16 == 0 && kOffBar % 8 == 0, "st.async targets and barriers");

// TMEM columns
constexpr uint32_t kColO = 0;       // O [128 heads x 256 dims] fp32
constexpr uint32_t kColSc = 256;    // partial sc, buffer b at 256 + 64 b
constexpr uint32_t kColSr = 384;    // sr
constexpr uint32_t kColQr = 448;    // q_r, buffer b at 448 + 32 b (64 bf16 = 32 columns a row)

constexpr int kErrTimeout = 1;

struct PairParams {
  CUtensorMap tm_c;    // c_kv as [B*L rows][512], box [64 rows][64], 128B swizzle
  CUtensorMap tm_k;    // k_r  as [B*L rows][64],  box [64 rows][64], 128B swizzle
  CUtensorMap tm_qc;   // q_c  as [B*H rows][512], box [128 rows][64], 128B swizzle
  const __nv_bfloat16* q_r;   // [B][H][64]
  int B, H;
  int64_t L;
  int64_t nG;          // condensed groups in these rows (0: dense attention)
  int64_t tiles_per_seq;
  int64_t U;           // B * tiles_per_seq
  int64_t G;           // tile ranges; cluster (c, hb) takes range c, heads 128 hb ..
  int n_hb;            // H / 128
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
  // Paged, variable-length decode (meta != null): tm_c / tm_k cover the pools,
  // [num_pages * page_size rows]; sequence b's token t is row
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
  uint64_t* c_full;      // [kNS] a tile's C_KV half landed
  uint64_t* c_empty;     // [kNS] released after O of that tile
  uint64_t* kr_full;     // [kNKr]
  uint64_t* kr_empty;    // [kNKr] released after the sr MMAs
  uint64_t* q_full;      // Q_c of a sequence landed
  uint64_t* q_empty;     // the last score MMA of a sequence is done
  uint64_t* qr_full;     // [2] q_r of sequence segment s is in TMEM buffer s & 1
  uint64_t* qr_empty;    // [2] the last sr MMA that read buffer s & 1 is done
  uint64_t* s_full;      // [2] the scores (partial sc in buffer b, then sr) of a tile are in TMEM
  uint64_t* sc_full;     // [2] the partial sc of a tile is in buffer b
  uint64_t* sc_empty;    // [2] softmax and shipper warps have read partial sc buffer b
  uint64_t* sr_empty;    // the softmax warps have read sr
  uint64_t* recv_full;   // [4] quarter q of the peer's partial scores landed (transaction bytes)
  uint64_t* recv_free;   // [4] the peer's quarter q has read the partial scores sent to it
  uint64_t* recv_used;   // [4] this CTA's softmax warp of quarter q has read the received partials
  uint64_t* p_local;     // [2] the own rows of P buffer b are written (one barrier per buffer: a
                         // single one could run two phases ahead of the O issuer's wait)
  uint64_t* p_remote;    // [2] the peer's rows of P buffer b landed, all four quarters (transaction bytes)
  uint64_t* p_free;      // [2 x 2] index 2 c + b: O of CTA c done with P buffer b (and every O before)
  uint64_t* part_written; // the shippers wrote out their rows of a sequence part (one phase per part)
  uint64_t* dec;         // [4] the O issuer's decision for a tile (flag: rescale the peer rows)
  uint64_t* resc_go;     // every O issued before a rescale request is done
  uint64_t* resc_done;   // the shippers rescaled the peer rows as asked
  uint64_t* part_done;   // the last O of a sequence part is done (one phase per part)
  uint64_t* drain;       // [2]
};

__device__ __forceinline__ void record_timeout(volatile int* abort, const PairParams& p, int where) {
  *abort = 1;
  if (atomicOr(p.err, kErrTimeout) == 0) atomicExch(p.err + 1, where);
}

// Bounded wait.  Each probe is an mbarrier.try_wait at CTA scope, which
// suspends the thread in hardware until the phase completes or a short
// system-defined limit passes.  The first probe is inline (most waits find
// the phase complete); the loop with its time bound is out of line.  CTA scope
// suffices for every barrier here, including those the peer completes: data
// from the peer lands in this CTA's shared memory before its transaction bytes
// complete the phase (st.async, bulk copies), and the peer's remote arrivals
// and multicast MMA commits only report that it has finished reading or
// writing its own copies.  A cluster-scope acquire on each probe measured
// about 0.3 us per wait.
__device__ __noinline__ bool bounded_wait_slow(uint64_t* bar, uint32_t parity, volatile int* abort,
                                               const PairParams& p, int where, bool honour_abort) {
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (honour_abort && *abort) return false;
    if ((spin & 7u) == 0 && ptx::globaltimer_ns() - t0 > p.timeout_ns) {
      record_timeout(abort, p, where);
      return false;
    }
  }
}

__device__ __forceinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                             const PairParams& p, int where, bool honour_abort) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  return bounded_wait_slow(bar, parity, abort, p, where, honour_abort);
}

// A wait of a whole warp: every lane probes the same phase (one shared-memory
// request for the warp, no divergent branch and no broadcast of a verdict),
// and each lane acquires the phase itself.  A lane that finds the phase
// incomplete takes the bounded loop; the warp reconverges at its next
// warp-wide instruction.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          const PairParams& p, int where) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  return bounded_wait_slow(bar, parity, abort, p, where, true);
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Maximum of s[0..N), the lowest index attaining it and sr at that index, as
// a pairwise tree: depth log2 N instead of a chain of N dependent selects.  A
// node keeps its left (lower-index) half unless the right half's maximum is
// strictly greater, so each subtree returns its lowest-index maximum.
template <int N>
__device__ __forceinline__ void tree_argmax(const float* s, const float* sr, int base, float& m, int& a,
                                            float& sra) {
  if constexpr (N == 1) {
    m = s[0];
    a = base;
    sra = sr[0];
  } else {
    float m0, m1, r0, r1;
    int a0, a1;
    tree_argmax<N / 2>(s, sr, base, m0, a0, r0);
    tree_argmax<N / 2>(s + N / 2, sr + N / 2, base + N / 2, m1, a1, r1);
    const bool right = m1 > m0;
    m = right ? m1 : m0;
    a = right ? a1 : a0;
    sra = right ? r1 : r0;
  }
}

// Statistics of one group held by one thread: x[0..N) the semantic scores,
// sr[0..N) the positional ones; on return e[] holds e_t = e^{s_t - m}.
// m = max s_t, a = the lowest index attaining it, sra = sr_a, den = sum e_t,
// num = sum e_t sc_t.
// The elementwise work runs on packed fp32 pairs (two tokens per instruction).
template <int N>
__device__ __forceinline__ void group_stats(const float* x, const float* sr, float* e, float& m, int& a,
                                            float& sra, float& den, float& num) {
  if constexpr (N == 1) {
    m = x[0] + sr[0];
    a = 0;
    sra = sr[0];
    e[0] = 1.f;
    den = 1.f;
    num = x[0];
  } else {
    float s[N];
#pragma unroll
    for (int t = 0; t < N; t += 2)
      ptx::f32x2_split(ptx::add_f32x2(ptx::f32x2(x[t], x[t + 1]), ptx::f32x2(sr[t], sr[t + 1])), s[t], s[t + 1]);
    tree_argmax<N>(s, sr, 0, m, a, sra);
    const float mb = -m * kLog2e;
    const uint64_t l2e = ptx::f32x2(kLog2e, kLog2e), mb2 = ptx::f32x2(mb, mb);
    uint64_t nacc = ptx::f32x2(0.f, 0.f), dacc = ptx::f32x2(0.f, 0.f);
#pragma unroll
    for (int t = 0; t < N; t += 2) {
      float u0, u1;
      ptx::f32x2_split(ptx::fma_f32x2(ptx::f32x2(s[t], s[t + 1]), l2e, mb2), u0, u1);
      e[t] = ex2(u0);
      e[t + 1] = ex2(u1);
      const uint64_t ee = ptx::f32x2(e[t], e[t + 1]);
      nacc = ptx::fma_f32x2(ee, ptx::f32x2(x[t], x[t + 1]), nacc);
      dacc = ptx::add_f32x2(dacc, ee);
    }
    float n0, n1, d0, d1;
    ptx::f32x2_split(nacc, n0, n1);
    ptx::f32x2_split(dacc, d0, d1);
    num = n0 + n1;
    den = d0 + d1;
  }
}

template <int LOG2G, bool kPaged>
__global__ void __launch_bounds__(kThreads, 1) lca_pair_kernel(const __grid_constant__ PairParams p) {
  constexpr int g = 1 << LOG2G;
  static_assert(g <= kT, "a group must fit in one tile");
  constexpr int GW = g < kHalfT ? g : kHalfT;   // tokens of one group held by one thread
  constexpr int NGT = kHalfT / GW;              // groups (or group halves) per thread
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int r = (int)ptx::cluster_ctarank();     // 0 or 1
  const int peer = r ^ 1;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  Bars bb;
  bb.c_full = bars;
  bb.c_empty = bb.c_full + kNS;
  bb.kr_full = bb.c_empty + kNS;
  bb.kr_empty = bb.kr_full + kNKr;
  bb.q_full = bb.kr_empty + kNKr;
  bb.q_empty = bb.q_full + 1;
  bb.qr_full = bb.q_empty + 1;
  bb.qr_empty = bb.qr_full + 2;
  bb.s_full = bb.qr_empty + 2;
  bb.sc_full = bb.s_full + 2;
  bb.sc_empty = bb.sc_full + 2;
  bb.sr_empty = bb.sc_empty + 2;
  bb.recv_full = bb.sr_empty + 1;
  bb.recv_free = bb.recv_full + 4;
  bb.p_local = bb.recv_free + 4;
  bb.p_remote = bb.p_local + 2;
  bb.p_free = bb.p_remote + 2;
  bb.part_written = bb.p_free + 4;
  bb.dec = bb.part_written + 1;
  bb.resc_go = bb.dec + 4;
  bb.resc_done = bb.resc_go + 1;
  bb.part_done = bb.resc_done + 1;
  bb.drain = bb.part_done + 1;
  bb.recv_used = bb.drain + 2;
  static_assert(2 * kNS + 2 * kNKr + 2 + 2 + 2 + 2 + 2 + 2 + 1 + 4 + 4 + 2 + 2 + 4 + 1 + 2 + 1 + 1 + 1 + 2 + 4 + 2 ==
                    kNumBars,
                "barrier count");
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);
  volatile int* dec_flag = reinterpret_cast<volatile int*>(smem + kOffFlag);
  float* recv = reinterpret_cast<float*>(smem + kOffRecv);
  float* alpha_s = reinterpret_cast<float*>(smem + kOffAlpha);
  // the chunk of (P buffer, lane quarter, CTA)
  auto fac_chunk = [&](int buf, int q, int rank) -> int { return ((buf * 4 + q) * 2 + rank) * kFacChunk; };

  const int64_t cl = blockIdx.x >> 1;
  const int hb = (int)(cl % p.n_hb);
  const int64_t c = cl / p.n_hb;
  const int h0 = hb * kHeads;
  constexpr bool paged = kPaged;   // a separate instantiation: the contiguous loops stay as they were
  // The cluster's range of tiles, for sequences of tiles_per_seq tiles each; a
  // paged batch takes its range from the metadata once the previous kernel in
  // the stream is done (below).
  int64_t u0 = c * p.U / p.G;
  int64_t n_tiles = (c + 1) * p.U / p.G - u0;
  int64_t seq0 = u0 / p.tiles_per_seq;
  int64_t tile0 = u0 - seq0 * p.tiles_per_seq;
  auto seq_tiles = [&](int64_t b) -> int64_t {
    if constexpr (kPaged) return (int64_t)meta_seq(p.meta)[b].w;
    else return p.tiles_per_seq;
  };
  // the next (sequence, tile) of the range; a paged batch's sequences without
  // tiles are passed over (tps: tiles of the current sequence)
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
  auto last_of_part = [&](int64_t i, int64_t tile, int64_t tps) {
    if constexpr (kPaged) return i + 1 == n_tiles || tile + 1 == tps;
    else return i + 1 == n_tiles || tile + 1 == p.tiles_per_seq;
  };
  // first row of a tile's 64 tokens in the C_KV / K_R tensor maps
  auto tile_row = [&](int64_t b, int64_t tile) -> int32_t {
    if constexpr (!kPaged) return (int32_t)(b * p.L + tile * kT);
    else return (int32_t)paged_row(p.block_table, p.table_stride, p.page_size, p.num_pages, b, tile * kT, p.err,
                                   0xA03);
  };

  if (tid == 0) {
    for (int i = 0; i < kNS; ++i) { ptx::mbar_init(&bb.c_full[i], 1); ptx::mbar_init(&bb.c_empty[i], 1); }
    for (int i = 0; i < kNKr; ++i) { ptx::mbar_init(&bb.kr_full[i], 1); ptx::mbar_init(&bb.kr_empty[i], 1); }
    ptx::mbar_init(bb.q_full, 1);
    ptx::mbar_init(bb.q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bb.qr_full[i], 4);          // the 4 softmax warps
      ptx::mbar_init(&bb.qr_empty[i], 1);
      ptx::mbar_init(&bb.s_full[i], 1);
      ptx::mbar_init(&bb.sc_full[i], 1);
      ptx::mbar_init(&bb.sc_empty[i], 8);         // 4 softmax + 4 shipper warps
      ptx::mbar_init(&bb.dec[i], 1);
      ptx::mbar_init(&bb.dec[2 + i], 1);
      ptx::mbar_init(&bb.drain[i], 1);
    }
    for (int i = 0; i < 4; ++i) ptx::mbar_init(&bb.p_free[i], 1);   // one O commit (multicast)
    ptx::mbar_init(bb.sr_empty, 4);               // the 4 softmax warps
    for (int q = 0; q < 4; ++q) {
      ptx::mbar_init(&bb.recv_full[q], 1);        // armed with its transaction bytes
      ptx::mbar_init(&bb.recv_free[q], 1);        // the peer's shipper warp of quarter q
      ptx::mbar_init(&bb.recv_used[q], 1);        // this CTA's softmax warp of quarter q
    }
    ptx::mbar_init(&bb.p_remote[0], 1);           // armed with the four quarters' transaction bytes
    ptx::mbar_init(&bb.p_remote[1], 1);
    ptx::mbar_init(&bb.p_local[0], 4);            // the 4 softmax warps
    ptx::mbar_init(&bb.p_local[1], 4);
    ptx::mbar_init(bb.part_written, 4);           // the 4 shipper warps
    ptx::mbar_init(bb.resc_go, 1);
    ptx::mbar_init(bb.resc_done, 4);
    ptx::mbar_init(bb.part_done, 1);
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
    // the first phases of the barriers the peer completes with transaction bytes
    ptx::mbar_arrive_expect_tx(&bb.p_remote[0], 4 * kPQBytes);
    ptx::mbar_arrive_expect_tx(&bb.p_remote[1], 4 * kPQBytes);
    for (int q = 0; q < 4; ++q) {
      ptx::mbar_arrive_expect_tx(&bb.recv_full[q], kRecvQBytes);
    }
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  // Both CTAs' barriers are initialised before either CTA touches the other's.
  ptx::cluster_sync();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // Programmatic dependent launch: nothing below touches global memory before
  // the previous kernel in the stream has completed; its first tile and query
  // block are only prefetched into L2 (no data reaches this CTA).
  if (tid == 0 && !paged) {
    const int32_t frow = (int32_t)(seq0 * p.L + tile0 * kT);
    for (int a = 0; a < kAtoms; ++a) ptx::tma_prefetch_l2_2d(&p.tm_c, kDim * r + 64 * a, frow);
    ptx::tma_prefetch_l2_2d(&p.tm_k, 0, frow);
    const int32_t qrow = (int32_t)(seq0 * p.H + h0);
    for (int a = 0; a < kAtoms; ++a) ptx::tma_prefetch_l2_2d(&p.tm_qc, kDim * r + 64 * a, qrow);
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
    // Per tile: K_R into its slot (after the sr MMAs of the tile two back), then
    // this CTA's half of C_KV into its stage (after O of the tile kNS back).
    ptx::prefetch_tmap(&p.tm_c);
    ptx::prefetch_tmap(&p.tm_k);
    ptx::prefetch_tmap(&p.tm_qc);
    const uint64_t once = ptx::l2_policy_evict_first();
    int issued_c[kNS], issued_k[kNKr];
#pragma unroll
    for (int i = 0; i < kNS; ++i) issued_c[i] = -1;
#pragma unroll
    for (int i = 0; i < kNKr; ++i) issued_k[i] = -1;
    int issued_q = -1, seg = -1;
    int64_t cur_b = -1;
    bool ok = true;
    int64_t pseq = seq0, ptile = tile0, ptps = tps0;
    // each tile's row is looked up a tile ahead (a paged batch reads its block
    // table), so that the lookup's latency passes during the waits
    int32_t row_next = (kPaged && n_tiles > 0) ? tile_row(pseq, ptile) : 0;
    for (int64_t i = 0; i < n_tiles && ok; ++i) {
      const int64_t b = pseq;
      if (b != cur_b) {
        cur_b = b;
        ++seg;
        if (seg >= 1) ok = bounded_wait(bb.q_empty, (seg - 1) & 1, abort_flag, p, 0x500, true);
        if (!ok) break;
        ptx::mbar_arrive_expect_tx(bb.q_full, kAtoms * kQcAtom);
        const int32_t qrow = (int32_t)(b * p.H + h0);
        for (int a = 0; a < kAtoms; ++a)
          ptx::tma_load_2d(smem + kOffQc + a * kQcAtom, &p.tm_qc, kDim * r + 64 * a, qrow, bb.q_full);
        issued_q = seg;
      }
      const int32_t row = kPaged ? row_next : tile_row(b, ptile);
      {
        const int ks = (int)(i % kNKr);
        const int kk = (int)(i / kNKr);
        if (kk >= 1) ok = bounded_wait(&bb.kr_empty[ks], (kk - 1) & 1, abort_flag, p, 0x501, true);
        if (!ok) break;
        if (!(p.debug_skip_load && i == 0)) {
          ptx::mbar_arrive_expect_tx(&bb.kr_full[ks], kKrBytes);
          ptx::tma_load_2d_hint(smem + kOffKr + ks * kKrBytes, &p.tm_k, 0, row, &bb.kr_full[ks], once);
#pragma unroll
          for (int q = 0; q < kNKr; ++q) if (q == ks) issued_k[q] = kk;
        }
      }
      {
        const int cs = (int)(i % kNS);
        const int ck = (int)(i / kNS);
        if (ck >= 1) ok = bounded_wait(&bb.c_empty[cs], (ck - 1) & 1, abort_flag, p, 0x502, true);
        if (!ok) break;
        if (!LCA_CHECK(p.err, cs < kNS && (int64_t)row < (paged ? p.num_pages * p.page_size : (int64_t)p.B * p.L),
                       0xE01)) { ok = false; break; }
        ptx::mbar_arrive_expect_tx(&bb.c_full[cs], kStage);
        uint8_t* dst = smem + kOffC + cs * kStage;
        for (int a = 0; a < kAtoms; ++a)
          ptx::tma_load_2d_hint(dst + a * kCAtom, &p.tm_c, kDim * r + 64 * a, row, &bb.c_full[cs], once);
#pragma unroll
        for (int q = 0; q < kNS; ++q) if (q == cs) issued_c[q] = ck;
      }
      step(pseq, ptile, ptps);
      if (kPaged && i + 1 < n_tiles) row_next = tile_row(pseq, ptile);
    }
    // Let every copy this thread started land before the CTA can exit.
#pragma unroll
    for (int i = 0; i < kNS; ++i)
      if (issued_c[i] >= 0) bounded_wait(&bb.c_full[i], issued_c[i] & 1, abort_flag, p, 0x5F0, false);
#pragma unroll
    for (int i = 0; i < kNKr; ++i)
      if (issued_k[i] >= 0) bounded_wait(&bb.kr_full[i], issued_k[i] & 1, abort_flag, p, 0x5F1, false);
    if (issued_q >= 0) bounded_wait(bb.q_full, issued_q & 1, abort_flag, p, 0x5F2, false);
  } else if (warp == 1 && lane == 0) {
    // ===================================================== score MMA issuer
    // Tile t: the partial sc[128 x 64] = Q_c[:, dims_r] . C_KV[tile, dims_r]^T
    // into buffer t & 1 (signalled on its own, for the shippers), then
    // sr[128 x 64] = q_r . K_R^T (A from TMEM) into the one sr buffer once the
    // softmax has read the previous tile's.
    constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(kHeads, kT, 0, 0);   // K-major A and B
    const uint64_t d_qc = ptx::smem_desc(ptx::smem_u32(smem + kOffQc), 16, 1024, ptx::kSwizzle128B);
    const uint64_t d_c = ptx::smem_desc(ptx::smem_u32(smem + kOffC), 16, 1024, ptx::kSwizzle128B);
    const uint64_t d_kr = ptx::smem_desc(ptx::smem_u32(smem + kOffKr), 16, 1024, ptx::kSwizzle128B);
    int seg = -1;
    int64_t cur_b = -1;
    bool ok = true;
    int64_t sseq = seq0, stile = tile0, stps = tps0;
    for (int64_t t = 0; t < n_tiles && ok; ++t, step(sseq, stile, stps)) {
      const int64_t b = sseq;
      const bool last_in_seg = last_of_part(t, stile, stps);
      const int buf = (int)(t & 1);
      bool new_seg = false;
      if (b != cur_b) {
        cur_b = b;
        ++seg;
        new_seg = true;
        ok = bounded_wait(bb.q_full, seg & 1, abort_flag, p, 0x600, true);
        if (!ok) break;
      }
      if (t >= 2) ok = bounded_wait(&bb.sc_empty[buf], (uint32_t)((t >> 1) - 1) & 1, abort_flag, p, 0x601, true);
      if (ok) ok = bounded_wait(&bb.kr_full[t % kNKr], (uint32_t)(t / kNKr) & 1, abort_flag, p, 0x602, true);
      if (ok) ok = bounded_wait(&bb.c_full[t % kNS], (uint32_t)(t / kNS) & 1, abort_flag, p, 0x603, true);
      if (!ok) break;
      ptx::tc_fence_after();
      {
        const uint32_t d_s = tmem + kColSc + 64u * buf;
        const uint64_t b0 = d_c + (uint64_t)(((t % kNS) * kStage) >> 4);
#pragma unroll
        for (int a = 0; a < kAtoms; ++a)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            ptx::mma_bf16_ss(d_s, d_qc + (uint64_t)((a * kQcAtom + 32 * k) >> 4),
                             b0 + (uint64_t)((a * kCAtom + 32 * k) >> 4), kIdescS, (a | k) != 0);
      }
      ptx::mma_commit(&bb.sc_full[buf]);
      if (t >= 1) ok = bounded_wait(bb.sr_empty, (uint32_t)(t - 1) & 1, abort_flag, p, 0x604, true);
      if (ok && new_seg) ok = bounded_wait(&bb.qr_full[seg & 1], (uint32_t)(seg >> 1) & 1, abort_flag, p, 0x605, true);
      if (!ok) break;
      ptx::tc_fence_after();
      {
        const uint32_t a_qr = tmem + kColQr + 32u * (uint32_t)(seg & 1);
        const uint64_t b0 = d_kr + (uint64_t)(((t % kNKr) * kKrBytes) >> 4);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          ptx::mma_bf16_ts(tmem + kColSr, a_qr + 8u * k, b0 + (uint64_t)((32 * k) >> 4), kIdescS, k > 0);
        ptx::mma_commit(&bb.kr_empty[t % kNKr]);
      }
      ptx::mma_commit(&bb.s_full[buf]);
      if (last_in_seg) {
        ptx::mma_commit(bb.q_empty);
        ptx::mma_commit(&bb.qr_empty[seg & 1]);
      }
    }
    ptx::mma_commit(&bb.drain[0]);
    bounded_wait(&bb.drain[0], 0, abort_flag, p, 0x6F0, false);
  } else if (warp == 2 && lane == 0) {
    // ===================================================== O MMA issuer
    // Tile j once P buffer j & 1 is complete (own rows, the peer's rows and
    // factors), and, when a sequence part ended with the tile before, once the
    // shippers have written out their rows of it.  The decision for tile j
    // goes to the shippers on one of four barriers (they run at most three
    // tiles behind: O of tile j needs the peer's partials of tile j, which
    // the peer sends once this CTA's shippers have finished tile j - 3): if a
    // peer factor is not 1, the shippers rescale those heads' O rows first
    // (rare).  Then O[128 x 256] += P[128 x 64] . C_KV[tile, dims_r] (A
    // K-major from the P buffer, B MN-major from the tile's stage), four K
    // steps of 16 tokens; a sequence part starts afresh.  The release of the
    // P buffer is signalled in both CTAs (each writes into the other's).
    constexpr uint32_t kIdescO = ptx::idesc_bf16_f32(kHeads, kDim, 0, 1);   // A K-major, B MN-major
    const uint64_t d_p = ptx::smem_desc(ptx::smem_u32(smem + kOffP), 16, 1024, ptx::kSwizzle128B);
    const uint64_t d_cb = ptx::smem_desc(ptx::smem_u32(smem + kOffC), kCAtom, 1024, ptx::kSwizzle128B);
    int n_resc = 0, n_pw = 0;
    int64_t oseq = seq0, otile = tile0, otps = tps0;
    for (int64_t j = 0; j < n_tiles; ++j, step(oseq, otile, otps)) {
      const int buf = (int)(j & 1);
      if (!bounded_wait(&bb.p_local[buf], (uint32_t)(j >> 1) & 1, abort_flag, p, 0x700, true)) break;
      if (!bounded_wait(&bb.p_remote[buf], (uint32_t)(j >> 1) & 1, abort_flag, p, 0x701, true)) break;
      // this buffer takes the peer's rows of tile j + 2 next; the peer writes
      // them only after this CTA's O of tile j is done
      if (j + 2 < n_tiles)
        ptx::mbar_arrive_expect_tx(&bb.p_remote[buf], 4 * kPQBytes);
      // a part ended with the tile before: the shippers have written out their
      // rows of it before this tile's O starts the next part over them
      if (j > 0 && otile == 0) {
        if (!bounded_wait(bb.part_written, (uint32_t)n_pw & 1, abort_flag, p, 0x702, true)) break;
        ++n_pw;
      }
      bool resc = false;
      if (j > 0 && otile > 0) {   // a factor of the peer's rows is not 1: one flag per quarter
        const volatile float* al = alpha_s;
        resc = (__float_as_int(al[fac_chunk(buf, 0, peer) + 16]) | __float_as_int(al[fac_chunk(buf, 1, peer) + 16]) |
                __float_as_int(al[fac_chunk(buf, 2, peer) + 16]) | __float_as_int(al[fac_chunk(buf, 3, peer) + 16])) != 0;
      }
      if (resc) ptx::mma_commit(bb.resc_go);       // lands once every O issued so far is done
      dec_flag[j & 3] = resc ? 1 : 0;
      ptx::mbar_arrive(&bb.dec[j & 3]);
      if (resc) {
        if (!bounded_wait(bb.resc_done, (uint32_t)n_resc & 1, abort_flag, p, 0x703, true)) break;
        ++n_resc;
      }
      ptx::tc_fence_after();
      const uint32_t acc0 = (j > 0 && otile > 0) ? 1u : 0u;
      const int cs = (int)(j % kNS);
      const uint64_t a0 = d_p + (uint64_t)((buf * kPBytes) >> 4);
      const uint64_t b0 = d_cb + (uint64_t)((cs * kStage) >> 4);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        ptx::mma_bf16_ss(tmem + kColO, a0 + (uint64_t)((32 * k) >> 4), b0 + (uint64_t)((2048 * k) >> 4), kIdescO,
                         k > 0 ? 1u : acc0);
      ptx::mma_commit(&bb.c_empty[cs]);
      ptx::mma_commit_multicast(&bb.p_free[2 * r + buf], (uint16_t)0x3);
      if (last_of_part(j, otile, otps)) ptx::mma_commit(bb.part_done);
    }
    ptx::mma_commit(&bb.drain[1]);
    bounded_wait(&bb.drain[1], 0, abort_flag, p, 0x7F0, false);
  } else if (warp >= 3 && warp <= 6) {
    // ===================================================== softmax (own heads of quarter q)
    // Thread (hi, k): head m = 32 q + 16 r + hi, tokens 32 k .. 32 k + 31 of a tile.
    const int q = warp & 3;
    const int hi = lane & 15, k = lane >> 4;
    const int m = 32 * q + 16 * r + hi;          // TMEM lane, P row, factor index
    const int mp = 32 * q + 16 * peer + hi;      // the peer head of the same lane slot
    const int ol = 16 * q + hi;                  // row in the receive buffer
    const int h = h0 + m;
    const uint32_t lanes = (uint32_t)(32 * q + 16 * r) << 16;
    const uint32_t lanes_peer = (uint32_t)(32 * q + 16 * peer) << 16;
    const uint32_t peer_p_remote0 = ptx::mapa(ptx::smem_u32(&bb.p_remote[0]), peer);
    const uint32_t peer_p_remote1 = ptx::mapa(ptx::smem_u32(&bb.p_remote[1]), peer);
    const int row0 = 32 * q + 16 * r;            // this warp's 16 P rows (2 KB) and factors
    bool copy_pending = false;
    // q_r of sequence `seq` (segment s) into TMEM buffer s & 1, both lane
    // halves of this quarter: this thread's 32 dims of its own and its peer head
    auto load_qr = [&](int64_t seq, int s) -> bool {
      if (s >= 2 && !warp_wait(&bb.qr_empty[s & 1], (uint32_t)((s >> 1) - 1) & 1, abort_flag, p, 0x807))
        return false;
      uint32_t own[16], oth[16];
      const uint4* src_own = reinterpret_cast<const uint4*>(p.q_r + ((int64_t)seq * p.H + h0 + m) * kDR + 32 * k);
      const uint4* src_oth = reinterpret_cast<const uint4*>(p.q_r + ((int64_t)seq * p.H + h0 + mp) * kDR + 32 * k);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const uint4 a = __ldg(src_own + v), b2 = __ldg(src_oth + v);
        own[4 * v] = a.x; own[4 * v + 1] = a.y; own[4 * v + 2] = a.z; own[4 * v + 3] = a.w;
        oth[4 * v] = b2.x; oth[4 * v + 1] = b2.y; oth[4 * v + 2] = b2.z; oth[4 * v + 3] = b2.w;
      }
      ptx::tc_fence_after();
      ptx::tmem_st16x2_16(tmem + lanes + kColQr + 32u * (uint32_t)(s & 1), own);
      ptx::tmem_st16x2_16(tmem + lanes_peer + kColQr + 32u * (uint32_t)(s & 1), oth);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bb.qr_full[s & 1]);
      return true;
    };
    float M = -INFINITY, Z = 0.f;
    // A sequence part's partial (this head's O row over this CTA's dims, and
    // (M, Z)) is written out one tile later, just before that tile's P: the
    // next tile then starts without waiting for the part's last O, which may
    // wait for a rescale by the shippers, who reach it only once this warp
    // has started the next tile.  O of the next tile, which starts the next
    // part over these rows, needs that tile's P, so it comes after.
    bool pend = false;
    int pend_buf = 0;
    uint32_t pend_par = 0;
    int64_t pend_slot = 0;
    float pend_M = 0.f, pend_Z = 0.f;
    auto write_part = [&]() -> bool {
      const bool slot_ok = LCA_CHECK(p.err, pend_slot < p.ws_slots, 0xE06);
      // the part's last O is done once its P buffer is released
      if (!warp_wait(&bb.p_free[2 * r + pend_buf], pend_par, abort_flag, p, 0x806)) return false;
      ptx::tc_fence_after();
      float* dst = p.part_o + (pend_slot * p.H + h) * (int64_t)kDC + kDim * r + 32 * k;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        float o[32];
        ptx::tmem_ld16x2_32(tmem + lanes + kColO + 64u * cc, o);
        ptx::tmem_wait_ld();
#pragma unroll
        for (int t = 0; t < 32; t += 4)
          if (slot_ok)
            *reinterpret_cast<float4*>(dst + 64 * cc + t) = make_float4(o[t], o[t + 1], o[t + 2], o[t + 3]);
      }
      ptx::tc_fence_before();
      if (k == 0 && slot_ok) {
        p.part_mz[(pend_slot * p.H + h) * 2 + 0] = pend_M;
        p.part_mz[(pend_slot * p.H + h) * 2 + 1] = pend_Z;
      }
      pend = false;
      return true;
    };
    int64_t cseq = seq0, ctile = tile0, ctps = tps0;
    // the current sequence's length, groups and first window token
    // (32-bit: token positions fit, anchors are int32 and B L rows are bounded by
    // the TMA coordinates; the registers are short here)
    int32_t sL = 0, snG = 0, swin0 = 0;
    int64_t s_of = -1;
    int seg = 0;
    int64_t i = 0;
    bool ok = n_tiles > 0 ? load_qr(seq0, 0) : true;
    for (; i < n_tiles && ok; ++i, step(cseq, ctile, ctps)) {
      const int64_t b = cseq, tile = ctile;
      if constexpr (kPaged) {
        if (b != s_of) {
          s_of = b;
          const int4 rec = meta_seq(p.meta)[b];
          sL = rec.x;
          snG = rec.z;
          swin0 = snG * g;
        }
      } else {
        sL = (int32_t)p.L;
        snG = (int32_t)p.nG;
        swin0 = (int32_t)p.win0;
      }
      const int buf = (int)(i & 1);
      if (!warp_wait(&bb.s_full[buf], (uint32_t)(i >> 1) & 1, abort_flag, p, 0x800)) break;
      if (!warp_wait(&bb.recv_full[q], (uint32_t)i & 1, abort_flag, p, 0x801)) break;
      ptx::tc_fence_after();
      float x[kHalfT], sr[kHalfT];
      ptx::tmem_ld16x2_32(tmem + lanes + kColSc + 64u * buf, x);
      ptx::tmem_ld16x2_32(tmem + lanes + kColSr, sr);
      ptx::tmem_wait_ld();
      {  // the peer's partial scores over its dims (16-byte chunks swizzled by head)
        const float* rrow = recv + ol * kT;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const int phys = (8 * k + j) ^ (ol & 15);
          const float4 v = *reinterpret_cast<const float4*>(rrow + 4 * phys);
          ptx::f32x2_split(ptx::add_f32x2(ptx::f32x2(x[4 * j], x[4 * j + 1]), ptx::f32x2(v.x, v.y)), x[4 * j],
                           x[4 * j + 1]);
          ptx::f32x2_split(ptx::add_f32x2(ptx::f32x2(x[4 * j + 2], x[4 * j + 3]), ptx::f32x2(v.z, v.w)),
                           x[4 * j + 2], x[4 * j + 3]);
        }
      }
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(&bb.sc_empty[buf]);
        ptx::mbar_arrive(bb.sr_empty);
        // this quarter's buffer takes the next tile's partials: armed before the
        // peer may send them
        if (i + 1 < n_tiles) ptx::mbar_arrive_expect_tx(&bb.recv_full[q], kRecvQBytes);
        // the received partials are read: the quarter's shipper tells the peer
        ptx::mbar_arrive(&bb.recv_used[q]);
      }
      // the next sequence's q_r, for the sr MMA of the tile after this one
      if (last_of_part(i, tile, ctps) && i + 1 < n_tiles) {
        ++seg;
        int64_t nb = b + 1;
        if constexpr (kPaged)
          while (nb + 1 < p.B && seq_tiles(nb) == 0) ++nb;
        if (!load_qr(nb, seg)) break;
      }

      const int32_t tile0 = (int32_t)tile * kT;         // first token of the tile
      const int32_t tok0 = tile0 + kHalfT * k;
      int32_t* anc = p.anchor + ((int64_t)b * p.H + h) * p.anchor_stride;
      const bool first = i == 0 || tile == 0;
      float alpha = 1.f;
      uint32_t pk[kHalfT / 2];

      // Steps 2 and 3 for this thread's 32 tokens.  kFast: the whole tile is
      // condensed (g > 1, tile before the window), so no per-token choice.
      auto tile_math = [&](auto fast_tag) {
        constexpr bool kFast = decltype(fast_tag)::value;
        float s[kHalfT];
        // this thread's tokens before the sequence end, with the bias, and grouped,
        // as counts (32-bit compares against each token's constant offset; unused,
        // so not formed, when the whole tile is condensed)
        const int n_in = (int)(sL - tok0 < 0 ? 0 : (sL - tok0 > kHalfT ? kHalfT : sL - tok0));
        const int n_bias = (int)(p.bias_rows - tok0 < 0 ? 0 : (p.bias_rows - tok0 > kHalfT ? kHalfT : p.bias_rows - tok0));
        const int n_grp = (int)(swin0 - tok0 < 0 ? 0 : (swin0 - tok0 > kHalfT ? kHalfT : swin0 - tok0));
        // Some of this thread's groups are condensed: the window starts at a
        // multiple of g, which may fall inside the thread's 32 tokens, so the
        // choice is made per group (grp[]).  For g = 64 a group is the whole
        // tile, and the choice is the same for both threads of a head.
        const bool half_groups = kFast || ((g > 1) && (tok0 < swin0));
        bool grp[NGT];
#pragma unroll
        for (int gi = 0; gi < NGT; ++gi) grp[gi] = kFast || (half_groups && gi * GW < n_grp);

        float f[NGT], Sg[NGT], deng[NGT], own_den[NGT], ent = -INFINITY;
        if constexpr (!kFast && g == 1) {
#pragma unroll
          for (int t = 0; t < kHalfT; ++t)
            if (t < n_grp && LCA_CHECK(p.err, tok0 + t < snG, 0xE05))
              anc[tok0 + t] = (int32_t)(p.pos0 + tok0 + t);
        }
        if (half_groups) {
          int ag[NGT];
          float srag[NGT], numg[NGT], mg[NGT];
#pragma unroll
          for (int gi = 0; gi < NGT; ++gi) {
            group_stats<GW>(x + gi * GW, sr + gi * GW, s + gi * GW, mg[gi], ag[gi], srag[gi], deng[gi],
                            numg[gi]);
            ag[gi] += gi * GW + kHalfT * k;          // tile-relative
            own_den[gi] = deng[gi];
            f[gi] = 1.f;
          }
          if constexpr (g > kHalfT) {
            // a 64-token group: merge the head's two threads (half 0 first, so
            // both form the same bits; a tie keeps half 0's anchor)
            const float om = __shfl_xor_sync(0xffffffffu, mg[0], 16);
            const float od = __shfl_xor_sync(0xffffffffu, deng[0], 16);
            const float on = __shfl_xor_sync(0xffffffffu, numg[0], 16);
            const float os = __shfl_xor_sync(0xffffffffu, srag[0], 16);
            const int oa = __shfl_xor_sync(0xffffffffu, ag[0], 16);
            const float m0 = k == 0 ? mg[0] : om, m1 = k == 0 ? om : mg[0];
            const float d0 = k == 0 ? deng[0] : od, d1 = k == 0 ? od : deng[0];
            const float n0 = k == 0 ? numg[0] : on, n1 = k == 0 ? on : numg[0];
            const float s0 = k == 0 ? srag[0] : os, s1 = k == 0 ? os : srag[0];
            const int a0 = k == 0 ? ag[0] : oa, a1 = k == 0 ? oa : ag[0];
            const float mm = fmaxf(m0, m1);
            const float f0 = ex2((m0 - mm) * kLog2e), f1 = ex2((m1 - mm) * kLog2e);
            deng[0] = d0 * f0 + d1 * f1;
            numg[0] = n0 * f0 + n1 * f1;
            const bool take1 = m1 > m0;
            srag[0] = take1 ? s1 : s0;
            ag[0] = take1 ? a1 : a0;
            f[0] = k == 0 ? f0 : f1;                 // this thread's e_t are relative to its own max
          }
#pragma unroll
          for (int gi = 0; gi < NGT; ++gi) {
            Sg[gi] = __fdividef(numg[gi], deng[gi]) + srag[gi];
            if (grp[gi]) ent = fmaxf(ent, Sg[gi]);
          }
          if (g <= kHalfT || k == 0) {
#pragma unroll
            for (int gi = 0; gi < NGT; ++gi) {
              const int32_t jg = (tile0 + (g <= kHalfT ? kHalfT * k + gi * GW : 0)) / g;
              if (grp[gi] && LCA_CHECK(p.err, jg >= 0 && jg < snG && ag[gi] >= 0 && ag[gi] < kT, 0xE04))
                anc[jg] = (int32_t)p.pos0 + tile0 + ag[gi];
            }
          }
          if constexpr (!kFast) {
#pragma unroll
            for (int gi = 0; gi < NGT; ++gi) {
              if (!grp[gi]) {   // a window group inside this half: its tokens stand for themselves
#pragma unroll
                for (int t = 0; t < GW; ++t) {
                  s[gi * GW + t] = x[gi * GW + t] + sr[gi * GW + t];
                  if (gi * GW + t < n_in) ent = fmaxf(ent, s[gi * GW + t]);
                }
              }
            }
          }
        } else {   // window tokens (and g = 1): the entry is the token itself
#pragma unroll
          for (int t = 0; t < kHalfT; ++t) {
            s[t] = x[t] + sr[t] + (t < n_bias ? p.bias : 0.f);
            if (t < n_in) ent = fmaxf(ent, s[t]);
          }
        }

        // ---- step 3: the head's reference max (both threads of the head agree)
        const float tmax = fmaxf(ent, __shfl_xor_sync(0xffffffffu, ent, 16));
        if (first) {
          M = tmax;
        } else if ((tmax - M) * kLog2e > kRescaleLog2) {
          alpha = ex2((M - tmax) * kLog2e);
          M = tmax;
        }
        Z *= alpha;

        // ---- per-token weights (this thread's 32 bf16 of its head's P row); Z
        // gains e^{S_j - M} per whole condensed group in this thread (the
        // tokens' weights sum to it), its share for a split 64-token group,
        // and each window token's weight
        if (half_groups) {
#pragma unroll
          for (int gi = 0; gi < NGT; ++gi) {
            if (grp[gi]) {
              const float eS = ex2((Sg[gi] - M) * kLog2e);
              if constexpr (g > kHalfT) {
                f[gi] *= __fdividef(eS, deng[gi]);
                Z += own_den[gi] * f[gi];
              } else {
                f[gi] = __fdividef(eS, deng[gi]);
                Z += eS;
              }
            }
          }
        }
        const float mb = -M * kLog2e;
        if constexpr (kFast) {   // every token is grouped: one packed multiply per pair
#pragma unroll
          for (int t2 = 0; t2 < kHalfT / 2; ++t2) {
            const float ff = f[(2 * t2) / GW];
            float a0, a1;
            ptx::f32x2_split(ptx::mul_f32x2(ptx::f32x2(s[2 * t2], s[2 * t2 + 1]), ptx::f32x2(ff, ff)), a0, a1);
            pk[t2] = pack_bf16x2(a0, a1);
          }
        } else {
#pragma unroll
          for (int t2 = 0; t2 < kHalfT / 2; ++t2) {
            float pv[2];
#pragma unroll
            for (int e2 = 0; e2 < 2; ++e2) {
              const int t = 2 * t2 + e2;
              float v;
              if (grp[t / GW]) {
                v = s[t] * f[t / GW];
              } else {
                v = t < n_in ? ex2(fmaf(s[t], kLog2e, mb)) : 0.f;
                Z += v;
              }
              pv[e2] = v;
            }
            pk[t2] = pack_bf16x2(pv[0], pv[1]);
          }
        }
      };
      const bool fast = g > 1 && tile0 + kT <= swin0;   // warp-uniform
      if (fast) tile_math(std::true_type{});
      else tile_math(std::false_type{});
      if (*abort_flag) break;

      const bool any_resc = __any_sync(0xffffffffu, alpha != 1.f);
      if (any_resc) {
        // this head's O row must be complete (O of tile i - 1) before it is
        // scaled here; this warp saw buffer (i - 1) & 1's earlier release when
        // it wrote P of tile i - 1
        const int pb = (int)((i - 1) & 1);
        if (!warp_wait(&bb.p_free[2 * r + pb], (uint32_t)((i - 1) >> 1) & 1, abort_flag, p, 0x803)) break;
        ptx::tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          float o[32];
          const uint32_t ta = tmem + lanes + kColO + 64u * cc;
          ptx::tmem_ld16x2_32(ta, o);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) o[t] *= alpha;
          ptx::tmem_st16x2_32(ta, o);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
      }
      if (pend && !write_part()) break;
      // A paged sequence's last tile: its stage rows past the last token hold
      // whatever the pool has there.  Their weights are 0, but 0 x NaN is not,
      // so the four softmax warps clear those rows before O reads the stage
      // (the score MMAs are done with it; the fence below orders the stores).
      if (kPaged && (tile + 1) * kT > sL) {
        const int n_valid = (int)(sL - tile * kT);
        uint8_t* st = smem + kOffC + (int)(i % kNS) * kStage;
        for (int idx = (warp - 3) * 32 + lane; idx < kAtoms * kT * 8; idx += 128) {
          const int row = (idx >> 3) & (kT - 1);   // 8 chunks of 16 bytes a row, in every atom
          if (row >= n_valid)
            *reinterpret_cast<uint4*>(st + (idx >> 9) * kCAtom + row * 128 + (idx & 7) * 16) =
                make_uint4(0u, 0u, 0u, 0u);
        }
      }
      // ---- this head's P row and factor into this CTA's P buffer (free once
      // its O of tile i - 2 is done; the previous copy out of it has read it)
      if (i >= 2 && !warp_wait(&bb.p_free[2 * r + buf], (uint32_t)((i >> 1) - 1) & 1, abort_flag, p, 0x804))
        break;
      if (lane == 0 && copy_pending) {
        ptx::bulk_wait_group_read0();
        copy_pending = false;
      }
      __syncwarp();
      {
        uint8_t* row = smem + kOffP + buf * kPBytes + m * 128;
#pragma unroll
        for (int j = 0; j < 4; ++j)
          *reinterpret_cast<uint4*>(row + 16 * ((4 * k + j) ^ (m & 7))) =
              make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
        if (k == 0) alpha_s[fac_chunk(buf, q, r) + hi] = alpha;
        if (lane == 0) alpha_s[fac_chunk(buf, q, r) + 16] = __int_as_float(any_resc ? 1 : 0);
      }
      ptx::fence_proxy_async_smem();                 // visible to the MMA's and the copy's reads
      __syncwarp();
      // ---- the same 16 rows and factors into the peer's P buffer (free once
      // the peer's O of tile i - 2 is done): two bulk copies, same offsets
      if (i >= 2 && !warp_wait(&bb.p_free[2 * peer + buf], (uint32_t)((i >> 1) - 1) & 1, abort_flag, p, 0x805))
        break;
      if (lane == 0) {
        const uint32_t bar = buf ? peer_p_remote1 : peer_p_remote0;
        const uint8_t* rows = smem + kOffP + buf * kPBytes + row0 * 128;
        const float* fac = alpha_s + fac_chunk(buf, q, r);
        ptx::bulk_copy_to_peer(ptx::mapa(ptx::smem_u32(rows), peer), rows, 16 * 128, bar);
        ptx::bulk_copy_to_peer(ptx::mapa(ptx::smem_u32(fac), peer), fac, kFacChunk * 4, bar);
        ptx::bulk_commit_group();
        copy_pending = true;
        ptx::mbar_arrive(&bb.p_local[buf]);
      }

      if (last_of_part(i, tile, ctps)) {   // written out before the next tile's P
        pend = true;
        pend_buf = buf;
        pend_par = (uint32_t)(i >> 1) & 1;
        pend_slot = b + c;
        pend_M = M;
        pend_Z = Z + __shfl_xor_sync(0xffffffffu, Z, 16);
        M = -INFINITY;
        Z = 0.f;
      }
    }
    if (pend && i == n_tiles) write_part();
    if (lane == 0 && copy_pending) ptx::bulk_wait_group_read0();
    // The peer O issuer's releases of the last two P buffers (multicast into
    // this CTA's shared memory) have landed before this CTA exits.
    if (lane == 0 && q == 0 && i == n_tiles) {
      for (int64_t t = n_tiles - 2; t < n_tiles; ++t)
        if (t >= 0 && !bounded_wait(&bb.p_free[2 * peer + (t & 1)], (uint32_t)(t >> 1) & 1, abort_flag, p, 0x8F0, true))
          break;
    }
  } else if (warp >= 7) {
    // ===================================================== shipper (peer heads of quarter q)
    // Thread (hi, k): peer head m = 32 q + 16 peer + hi, tokens 32 k .. of a tile.
    // Iteration i: tell the peer that this CTA's softmax has read the partials
    // of tile i, and send it those of tile i + 1; then, one tile behind, do what
    // O of tile i - 1 asked of these heads' O rows: the rescale (rare), and at
    // the end of a sequence part the write-out.
    const int q = warp & 3;
    const int hi = lane & 15, k = lane >> 4;
    const int m = 32 * q + 16 * peer + hi;
    const int olp = 16 * q + hi;                 // the head's row in the peer's receive buffer
    const uint32_t lanes = (uint32_t)(32 * q + 16 * peer) << 16;
    const uint32_t peer_row = ptx::mapa(ptx::smem_u32(recv + olp * kT), peer);
    const uint32_t peer_recv_full = ptx::mapa(ptx::smem_u32(&bb.recv_full[q]), peer);
    const uint32_t peer_recv_free = ptx::mapa(ptx::smem_u32(&bb.recv_free[q]), peer);
    int n_resc = 0, n_part = 0;
    // This CTA's softmax warp of quarter q has read the partials of tile t: the
    // peer may overwrite them.  The release at cluster scope is taken here, off
    // the softmax warp's path; it covers the softmax's reads, which its
    // CTA-scope release on recv_used ordered before this warp's acquire.
    auto forward = [&](int64_t t) -> bool {
      if (!warp_wait(&bb.recv_used[q], (uint32_t)t & 1, abort_flag, p, 0x905)) return false;
      if (lane == 0) ptx::mbar_arrive_remote(peer_recv_free);
      return true;
    };
    auto ship = [&](int64_t t) -> bool {
      const int buf = (int)(t & 1);
      if (t >= 1 && !forward(t - 1)) return false;
      if (!warp_wait(&bb.sc_full[buf], (uint32_t)(t >> 1) & 1, abort_flag, p, 0x900)) return false;
      ptx::tc_fence_after();
      float v[32];
      ptx::tmem_ld16x2_32(tmem + lanes + kColSc + 64u * buf, v);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bb.sc_empty[buf]);
      if (t >= 1 && !warp_wait(&bb.recv_free[q], (uint32_t)(t - 1) & 1, abort_flag, p, 0x901)) return false;
#pragma unroll
      for (int j = 0; j < 8; ++j)
        ptx::st_async_v4(peer_row + 16u * (uint32_t)((8 * k + j) ^ (olp & 15)), __float_as_uint(v[4 * j]),
                         __float_as_uint(v[4 * j + 1]), __float_as_uint(v[4 * j + 2]),
                         __float_as_uint(v[4 * j + 3]), peer_recv_full);
      return true;
    };
    // what O of tile j needed of these heads' rows, done after O of tile j
    auto behind = [&](int64_t j, int64_t b, int64_t tile, int64_t tps) -> bool {
      if (!warp_wait(&bb.dec[j & 3], (uint32_t)(j >> 2) & 1, abort_flag, p, 0x902)) return false;
      if (dec_flag[j & 3]) {
        // every O before tile j is done (one phase per request, seen in order)
        const float a = alpha_s[fac_chunk((int)(j & 1), q, peer) + hi];
        if (!warp_wait(bb.resc_go, (uint32_t)n_resc & 1, abort_flag, p, 0x903)) return false;
        ++n_resc;
        ptx::tc_fence_after();
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          float o[32];
          const uint32_t ta = tmem + lanes + kColO + 64u * cc;
          ptx::tmem_ld16x2_32(ta, o);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; ++t) o[t] *= a;
          ptx::tmem_st16x2_32(ta, o);
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bb.resc_done);
      }
      if (last_of_part(j, tile, tps)) {
        const int64_t slot = b + c;
        if (!LCA_CHECK(p.err, slot < p.ws_slots, 0xE08)) return false;
        // the last O of the part is done (one phase per part, seen in order)
        if (!warp_wait(bb.part_done, (uint32_t)n_part & 1, abort_flag, p, 0x904)) return false;
        ++n_part;
        ptx::tc_fence_after();
        float* dst = p.part_o + (slot * p.H + h0 + m) * (int64_t)kDC + kDim * r + 32 * k;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          float o[32];
          ptx::tmem_ld16x2_32(tmem + lanes + kColO + 64u * cc, o);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int t = 0; t < 32; t += 4)
            *reinterpret_cast<float4*>(dst + 64 * cc + t) = make_float4(o[t], o[t + 1], o[t + 2], o[t + 3]);
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bb.part_written);
      }
      return true;
    };
    bool ok = n_tiles > 0 ? ship(0) : true;
    int64_t bseq = seq0, btile = tile0, btps = tps0;   // (sequence, tile) of tile i - 1
    int64_t i = 0;
    for (; i < n_tiles && ok; ++i) {
      if (i + 1 < n_tiles && !(ok = ship(i + 1))) break;
      if (i >= 1) {
        if (!(ok = behind(i - 1, bseq, btile, btps))) break;
        step(bseq, btile, btps);
      }
    }
    if (ok && i == n_tiles && n_tiles > 0) {
      behind(n_tiles - 1, bseq, btile, btps);
      // the peer's release of the last partial scores has landed here before this CTA exits
      if (forward(n_tiles - 1) && lane == 0)
        bounded_wait(&bb.recv_free[q], (uint32_t)(n_tiles - 1) & 1, abort_flag, p, 0x9F0, true);
    }
  }

  // ===================================================== teardown
  __syncwarp();
  ptx::tc_fence_before();
  __syncthreads();
  // Neither CTA leaves while the other may still write its shared memory.
  ptx::cluster_sync();
  ptx::tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace pair
}  // namespace lca
