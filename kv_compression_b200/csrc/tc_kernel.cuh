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
//              anchor a_j), the group-local softmax sums den_j = sum e^{s_t - m_j}
//              and num_j = sum e^{s_t - m_j} sc_t, and the condensed logit
//              S_j = num_j / den_j + sr_{a_j}  (= q_c.c_bar_j + q_r.k_{a_j}; c_bar_j
//              is never formed).  Each thread scans an 8-token segment of one
//              head; a group of g > 8 tokens merges its segments by shuffles;
//   attend     (step 3) online softmax over [condensed || window].  A grouped
//              token's weight p_j w_t = e^{S_j - M} e^{s_t - m_j} / den_j is
//              written e^{s_t + k_j - M} with k_j = S_j - m_j - ln den_j, a window
//              token's e^{s_t - M}: one exponential per (token, head).  The
//              weights go to shared memory as bf16 and O^T[512 x 16] +=
//              C_KV_tile^T . P^T is one more MMA chain per tile.
// The range's partial (M, Z, O) goes to the workspace; the combine kernel
// merges the ranges of a sequence.
//
// Roles (320 threads): warp 0 lane 0 issues TMA loads and L2 prefetches two
// tiles ahead; warp 1 allocates TMEM and its lane 0 issues MMAs; warps 2-9
// (256 threads) do the softmax work, two warps per TMEM lane quarter, each
// owning 8 of the 16 heads.  C_KV is read twice per tile: once for the scores
// (kept in L2 with an evict-last hint) and once more, from L2, for O = C^T P^T
// after the softmax.  MMA order: scores(i), then O(i-1); each column pair
// leaves shared memory as soon as its MMAs are done, so the softmax of tile i
// overlaps the tensor work of tiles i-1 and i+1 and the loads keep streaming.
// Shared memory: a ring of five 32 KB slots for C_KV column pairs ([128
// tokens][2 x 64 dims], 128-byte swizzle), two 16 KB K_R slots (each reused to
// stage its tile's scores once the score MMA is done), the query block
// (9 x [16 heads][64 dims]) and two P buffers.
// Every mbarrier wait is bounded; when a bound runs out the CTA records the
// error, stops issuing work, waits for its own copies and MMAs in flight,
// frees TMEM and exits.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace lca {
namespace tc {

constexpr int kHC = 16;                    // heads per CTA (MMA N)
constexpr int kT = 128;                    // tokens per tile (MMA M of the score MMA)
constexpr int kDC = 512;                   // latent width
constexpr int kDR = 64;                    // RoPE key width
constexpr int kChunk = kT * 128;           // [128 rows][64 bf16] = 16 KB
constexpr int kPairBytes = 2 * kChunk;     // two 64-dim chunks = 128 latent dims
constexpr int kNPair = 5;                  // C_KV pair slots
constexpr int kNKr = 2;                    // K_R slots
constexpr int kQChunk = kHC * 128;         // [16 heads][64 bf16] = 2 KB
constexpr int kQBytes = 9 * kQChunk;       // 8 chunks of q_c, 1 of q_r
constexpr int kPBytes = kT * kHC * 2;      // P^T tile, bf16
constexpr int kSoftmaxWarps = 8;
constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
constexpr int kThreads = 64 + kSoftmaxThreads;
constexpr int kHH = kHC / 2;               // heads per softmax thread
constexpr int kTmemCols = 256;
constexpr int kSoftmaxBar = 1;             // named barrier of the softmax warps
constexpr int kMaxGroupsPerTile = 64;      // g >= 2 (g = 1 takes the per-token path)
constexpr int kPrefetchAhead = 2;          // tiles brought into L2 ahead of their loads
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

// shared memory map (offsets from a 1024-byte aligned base)
constexpr int kOffPair = 0;
constexpr int kOffKr = kOffPair + kNPair * kPairBytes;
constexpr int kOffQ = kOffKr + kNKr * kChunk;
constexpr int kOffP = kOffQ + kQBytes;
constexpr int kOffK = kOffP + 2 * kPBytes;                  // float [64 groups][16 heads]: k_j
constexpr int kOffGmax = kOffK + kMaxGroupsPerTile * kHC * 4;  // float [16]: max_j S_j of the tile
constexpr int kOffWmax = kOffGmax + kHC * 4;                // float [4][16]: max window score
constexpr int kOffZred = kOffWmax + 4 * kHC * 4;            // float [4][16]
constexpr int kOffBar = kOffZred + 4 * kHC * 4;
constexpr int kNumBars = 2 * kNPair + 2 * kNKr + 2 + 5 * 2 + 1;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 16;
constexpr int kSmemAlloc = kSmemBytes + 1024;          // alignment slack
static_assert(kSmemAlloc <= 232448, "shared memory budget of one sm_100 CTA");

// TMEM columns: S buffer b: sc at 32b, sr at 32b + 16;  O tile b: 64 + 64b + 16m
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
};

struct Bars {
  uint64_t* full_c;   // [kNPair]
  uint64_t* empty_c;  // [kNPair]
  uint64_t* full_k;   // [kNKr]
  uint64_t* empty_k;  // [kNKr]  released by the softmax warps (they stage scores there)
  uint64_t* q_full;
  uint64_t* q_empty;
  uint64_t* s_full;   // [2]
  uint64_t* s_empty;  // [2]
  uint64_t* p_full;   // [2]
  uint64_t* o_full;   // [2]
  uint64_t* o_empty;  // [2]
  uint64_t* drain;
};

// Bounded wait.  Returns false when the CTA's abort flag is set (if honoured)
// or when the bound runs out (then the flag and the error word are set).
__device__ __noinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          const TcParams& p, int where, bool honour_abort) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (ptx::mbar_try_wait(bar, parity)) return true;
    if (honour_abort && *abort) return false;
    if ((spin & 63u) == 0 && ptx::globaltimer_ns() - t0 > p.timeout_ns) {
      *abort = 1;
      if (atomicOr(p.err, kErrTimeout) == 0) atomicExch(p.err + 1, where);
      return false;
    }
  }
}

// Warp-uniform bounded wait: lane 0 polls, the verdict is broadcast.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          const TcParams& p, int where) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = bounded_wait(bar, parity, abort, p, where, true);
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
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

// Score staging in a K_R slot: [128 rows][32 floats] (sc of 16 heads, then sr),
// float4 columns XOR-swizzled by row so that threads reading the same step of
// different segments hit different banks.
__device__ __forceinline__ int stage_idx(int row, int col) {
  const int sw = ((row ^ (row >> 3)) & 7) << 2;
  return row * 32 + (col ^ sw);
}

// Fold the O^T tile in TMEM buffer `ob` (its use `okb`) into the register
// accumulator: O = O * al + O_tile, for this thread's latent rows and 8 heads.
__device__ __forceinline__ void fold_o(float (&O)[4][kHH], const float (&al)[kHH], int ob, int okb,
                                       uint32_t t_cols, const Bars& bb, volatile int* abort_flag,
                                       const TcParams& p) {
  warp_wait(&bb.o_full[ob], okb & 1, abort_flag, p, 0x303);
  ptx::tc_fence_after();
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    float ot[kHH];
    ptx::tmem_ld8(t_cols + kColO + 64 * ob + 16 * m, ot);
    ptx::tmem_wait_ld();
#pragma unroll
    for (int h = 0; h < kHH; ++h) O[m][h] = fmaf(O[m][h], al[h], ot[h]);
  }
  ptx::tc_fence_before();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(&bb.o_empty[ob]);
}

// Group statistics over v in [v0, v0 + n) of a thread's 8-token segment.
struct GroupStat {
  float m;    // max score
  int a;      // tile row of the first maximum
  float den;  // sum e^{s - m}
  float num;  // sum e^{s - m} sc
};

template <int N>
__device__ __forceinline__ GroupStat scan_group(const float (&x)[8], const float (&c)[8], int v0,
                                                int row0) {
  GroupStat r;
  r.m = x[v0];
  r.a = row0 + v0;
#pragma unroll
  for (int v = 1; v < N; ++v)
    if (x[v0 + v] > r.m) { r.m = x[v0 + v]; r.a = row0 + v0 + v; }   // strict: lowest index keeps a tie
  const float mb = r.m * kLog2e;
  r.den = 0.f;
  r.num = 0.f;
#pragma unroll
  for (int v = 0; v < N; ++v) {
    const float e = ex2(fmaf(x[v0 + v], kLog2e, -mb));
    r.den += e;
    r.num = fmaf(e, c[v0 + v], r.num);
  }
  return r;
}

template <int LOG2G>
__global__ void __launch_bounds__(kThreads, 1) lca_tc_kernel(const __grid_constant__ TcParams p) {
  constexpr int g = 1 << LOG2G;
  static_assert(g <= kT, "a group must fit in one tile");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBar);
  Bars bb;
  bb.full_c = bars;
  bb.empty_c = bb.full_c + kNPair;
  bb.full_k = bb.empty_c + kNPair;
  bb.empty_k = bb.full_k + kNKr;
  bb.q_full = bb.empty_k + kNKr;
  bb.q_empty = bb.q_full + 1;
  bb.s_full = bb.q_empty + 1;
  bb.s_empty = bb.s_full + 2;
  bb.p_full = bb.s_empty + 2;
  bb.o_full = bb.p_full + 2;
  bb.o_empty = bb.o_full + 2;
  bb.drain = bb.o_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int hb = blockIdx.x % p.n_hb;
  const int64_t c = blockIdx.x / p.n_hb;
  const int h0 = hb * kHC;
  const int64_t u0 = c * p.U / p.G;
  const int64_t u1 = (c + 1) * p.U / p.G;
  const int64_t win0 = p.nG * g;

  if (tid == 0) {
    for (int i = 0; i < kNPair; ++i) { ptx::mbar_init(&bb.full_c[i], 1); ptx::mbar_init(&bb.empty_c[i], 1); }
    for (int i = 0; i < kNKr; ++i) {
      ptx::mbar_init(&bb.full_k[i], 1);
      ptx::mbar_init(&bb.empty_k[i], kSoftmaxWarps);
    }
    ptx::mbar_init(bb.q_full, 1);
    ptx::mbar_init(bb.q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bb.s_full[i], 1);
      ptx::mbar_init(&bb.s_empty[i], kSoftmaxWarps);
      ptx::mbar_init(&bb.p_full[i], kSoftmaxWarps);
      ptx::mbar_init(&bb.o_full[i], 1);
      ptx::mbar_init(&bb.o_empty[i], kSoftmaxWarps);
    }
    ptx::mbar_init(bb.drain, 1);
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

  if (warp == 0 && lane == 0) {
    // ===================================================== TMA producer
    // Load order = MMA consumption order: for tile i, K_R(i) and the four
    // column pairs of C_KV(i) for the scores, then the four pairs of tile i-1
    // again for O(i-1) (read back from L2), and after the last tile the pairs
    // of that tile.  Each pair slot is freed as soon as its MMAs are done, so
    // shared memory never has to hold a whole tile across the softmax.
    ptx::prefetch_tmap(&p.tm_c);
    ptx::prefetch_tmap(&p.tm_k);
    ptx::prefetch_tmap(&p.tm_qc);
    ptx::prefetch_tmap(&p.tm_qr);
    const uint64_t keep = ptx::l2_policy_evict_last();    // first read: keep for the second
    const uint64_t drop = ptx::l2_policy_evict_first();   // second read: last use
    auto tile_row = [&](int64_t u) -> int32_t {
      return (int32_t)((u / p.tiles_per_seq) * p.L + (u % p.tiles_per_seq) * kT);
    };
    auto prefetch_tile = [&](int64_t u) {
      const int32_t row = tile_row(u);
      ptx::tma_prefetch_l2_2d(&p.tm_k, 0, row);
      for (int ch = 0; ch < 8; ++ch) ptx::tma_prefetch_l2_2d(&p.tm_c, 64 * ch, row);
    };
    for (int64_t u = u0 + 1; u < u0 + kPrefetchAhead && u < u1; ++u) prefetch_tile(u);
    int issued_c[kNPair], issued_k[kNKr];
#pragma unroll
    for (int i = 0; i < kNPair; ++i) issued_c[i] = -1;
#pragma unroll
    for (int i = 0; i < kNKr; ++i) issued_k[i] = -1;
    int issued_q = -1;
    int64_t nc = 0, nk = 0;
    int seg = -1;
    int64_t cur_b = -1;
    bool ok = true;
    // the four pairs of the tile at `row` into the next ring slots
    auto load_pairs = [&](int32_t row, uint64_t policy) -> bool {
      for (int pr = 0; pr < 4; ++pr) {
        const int cs = (int)(nc % kNPair);
        const int ck = (int)(nc / kNPair);
        if (ck >= 1 && !bounded_wait(&bb.empty_c[cs], (ck - 1) & 1, abort_flag, p, 0x102, true))
          return false;
        ptx::mbar_arrive_expect_tx(&bb.full_c[cs], kPairBytes);
        uint8_t* dst = smem + kOffPair + cs * kPairBytes;
        ptx::tma_load_2d_hint(dst, &p.tm_c, 128 * pr, row, &bb.full_c[cs], policy);
        ptx::tma_load_2d_hint(dst + kChunk, &p.tm_c, 128 * pr + 64, row, &bb.full_c[cs], policy);
#pragma unroll
        for (int q = 0; q < kNPair; ++q) if (q == cs) issued_c[q] = ck;
        ++nc;
      }
      return true;
    };
    for (int64_t u = u0; u < u1 && ok; ++u) {
      const int64_t b = u / p.tiles_per_seq;
      if (u + kPrefetchAhead < u1) prefetch_tile(u + kPrefetchAhead);
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
      const int32_t row = tile_row(u);
      {
        const int ks = (int)(nk % kNKr);
        const int kk = (int)(nk / kNKr);
        if (kk >= 1) ok = bounded_wait(&bb.empty_k[ks], (kk - 1) & 1, abort_flag, p, 0x101, true);
        if (!ok) break;
        if (!(p.debug_skip_load && nk == 0)) {
          ptx::mbar_arrive_expect_tx(&bb.full_k[ks], kChunk);
          ptx::tma_load_2d(smem + kOffKr + ks * kChunk, &p.tm_k, 0, row, &bb.full_k[ks]);
#pragma unroll
          for (int q = 0; q < kNKr; ++q) if (q == ks) issued_k[q] = kk;
        }
        ++nk;
      }
      ok = load_pairs(row, keep);                       // scores(u)
      if (ok && u > u0) ok = load_pairs(tile_row(u - 1), drop);   // O(u-1)
    }
    if (ok && u1 > u0) load_pairs(tile_row(u1 - 1), drop);        // O(last)
    // Let every copy this thread started land before the CTA can exit.
#pragma unroll
    for (int i = 0; i < kNPair; ++i)
      if (issued_c[i] >= 0) bounded_wait(&bb.full_c[i], issued_c[i] & 1, abort_flag, p, 0x1F0, false);
#pragma unroll
    for (int i = 0; i < kNKr; ++i)
      if (issued_k[i] >= 0) bounded_wait(&bb.full_k[i], issued_k[i] & 1, abort_flag, p, 0x1F1, false);
    if (issued_q >= 0) bounded_wait(bb.q_full, issued_q & 1, abort_flag, p, 0x1F2, false);
  } else if (warp == 1 && lane == 0) {
    // ===================================================== MMA issuer
    constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(kT, kHC, 0, 0);   // K-major A and B
    constexpr uint32_t kIdescP = ptx::idesc_bf16_f32(128, kHC, 1, 1);  // MN-major A and B
    // Descriptor templates; a K step adds (bytes >> 4) to the start-address field.
    const uint64_t d_pair = ptx::smem_desc(ptx::smem_u32(smem + kOffPair), 16, 1024, ptx::kSwizzle128B);
    const uint64_t d_kr = ptx::smem_desc(ptx::smem_u32(smem + kOffKr), 16, 1024, ptx::kSwizzle128B);
    const uint64_t d_q = ptx::smem_desc(ptx::smem_u32(smem + kOffQ), 16, 1024, ptx::kSwizzle128B);
    // A = C^T, M = 128 latent dims (two 64-dim atoms 16 KB apart), K = 16 tokens
    const uint64_t d_ct = ptx::smem_desc(ptx::smem_u32(smem + kOffPair), kChunk, 1024, ptx::kSwizzle128B);
    // B = P^T, N = 16 heads (8-head core blocks 2 KB apart), K = 16 tokens
    const uint64_t d_pt = ptx::smem_desc(ptx::smem_u32(smem + kOffP), 128, 2048, ptx::kSwizzleNone);
    int64_t nc = 0, nk = 0, i = 0;
    int seg = -1;
    int64_t cur_b = -1;
    bool ok = true;

    // O^T(j) = C_KV(j)^T . P^T(j): the next four ring entries hold tile j's pairs again
    auto issue_pc = [&](int64_t j) -> bool {
      const int buf = (int)(j & 1), kb = (int)(j >> 1);
      if (!bounded_wait(&bb.p_full[buf], kb & 1, abort_flag, p, 0x204, true)) return false;
      if (kb >= 1 && !bounded_wait(&bb.o_empty[buf], (kb - 1) & 1, abort_flag, p, 0x205, true))
        return false;
      const uint64_t bpt = d_pt + (uint64_t)((buf * kPBytes) >> 4);
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        const int cs = (int)(nc % kNPair);
        if (!bounded_wait(&bb.full_c[cs], (int)(nc / kNPair) & 1, abort_flag, p, 0x206, true))
          return false;
        ptx::tc_fence_after();
        const uint32_t d_o = tmem + kColO + 64 * buf + 16 * m;
        const uint64_t act = d_ct + (uint64_t)((cs * kPairBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ptx::mma_bf16_ss(d_o, act + (uint64_t)(kk * (2048 >> 4)), bpt + (uint64_t)(kk * (256 >> 4)),
                           kIdescP, kk > 0);
        ptx::mma_commit(&bb.empty_c[cs]);
        ++nc;
      }
      ptx::mma_commit(&bb.o_full[buf]);
      return true;
    };
    // scores(i) for column pair `pr` into sc of S buffer `buf`; frees the slot
    auto issue_sc_pair = [&](int buf, int pr) -> bool {
      const int cs = (int)(nc % kNPair);
      if (!bounded_wait(&bb.full_c[cs], (int)(nc / kNPair) & 1, abort_flag, p, 0x203, true))
        return false;
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
      ptx::mma_commit(&bb.empty_c[cs]);
      ++nc;
      return true;
    };

    for (int64_t u = u0; u < u1 && ok; ++u, ++i) {
      const int64_t b = u / p.tiles_per_seq;
      const bool last_in_seg = (u + 1 == u1) || ((u + 1) / p.tiles_per_seq != b);
      if (b != cur_b) {
        cur_b = b;
        ++seg;
        ok = bounded_wait(bb.q_full, seg & 1, abort_flag, p, 0x200, true);
        if (!ok) break;
      }
      const int buf = (int)(i & 1);
      const int kb = (int)(i >> 1);
      if (kb >= 1) ok = bounded_wait(&bb.s_empty[buf], (kb - 1) & 1, abort_flag, p, 0x201, true);
      if (!ok) break;
      // ---- scores(i): sr = K_R . q_r^T, sc = C_KV . q_c^T
      {
        const int ks = (int)(nk % kNKr);
        ok = bounded_wait(&bb.full_k[ks], (int)(nk / kNKr) & 1, abort_flag, p, 0x202, true);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t d_sr = tmem + kColS + 32 * buf + 16;
        const uint64_t a0 = d_kr + (uint64_t)((ks * kChunk) >> 4);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          ptx::mma_bf16_ss(d_sr, a0 + (uint64_t)((32 * k) >> 4),
                           d_q + (uint64_t)((8 * kQChunk + 32 * k) >> 4), kIdescS, k > 0);
        ++nk;
      }
      ok = issue_sc_pair(buf, 0) && issue_sc_pair(buf, 1) && issue_sc_pair(buf, 2) &&
           issue_sc_pair(buf, 3);
      if (!ok) break;
      ptx::mma_commit(&bb.s_full[buf]);   // also tells the softmax warps the K_R slot is read
      if (last_in_seg) ptx::mma_commit(bb.q_empty);
      // ---- O(i-1), its softmax done while scores(i) ran
      if (i > 0) ok = issue_pc(i - 1);
    }
    if (ok && i > 0) issue_pc(i - 1);
    // Every MMA issued here must finish before TMEM is freed.
    ptx::mma_commit(bb.drain);
    bounded_wait(bb.drain, 0, abort_flag, p, 0x2F0, false);
  } else if (warp >= 2) {
    // ===================================================== softmax warps
    // A failed wait only raises the abort flag; the softmax warps leave the
    // tile loop together, at the one checkpoint barrier of each tile, so no
    // warp is ever left waiting at a named barrier.
    const int q4 = warp & 3;             // TMEM lane quarter this warp may access
    const int hh = (warp - 2) >> 2;      // which 8 of the 16 heads
    const int row = q4 * 32 + lane;      // token row of the tile owned by this thread
    const int st = tid - 64;             // 0..255 among the softmax threads
    const uint32_t t_lane = tmem + ((uint32_t)(q4 * 32) << 16);
    const uint32_t t_cols = t_lane + kHH * hh;   // this thread's 8 head columns
    float* ks_tab = reinterpret_cast<float*>(smem + kOffK);      // [64][16] k_j
    float* gmax_s = reinterpret_cast<float*>(smem + kOffGmax);   // [16]
    float* wmax_s = reinterpret_cast<float*>(smem + kOffWmax);   // [4][16]
    float* zred = reinterpret_cast<float*>(smem + kOffZred);     // [4][16]
    uint8_t* pbase = smem + kOffP;
    // group phase: thread st scans tokens [8 sg, 8 sg + 8) of head gh
    const int gh = st >> 4;
    const int sg = st & 15;

    float O[4][kHH];
    float Zt[kHH], Mh[kHH], apend[kHH];
#pragma unroll
    for (int h = 0; h < kHH; ++h) {
      Zt[h] = 0.f; Mh[h] = -INFINITY; apend[h] = 0.f;
#pragma unroll
      for (int m = 0; m < 4; ++m) O[m][h] = 0.f;
    }
    bool pending = false;
    int pbuf = 0, pkb = 0;
    int64_t i = 0;

    for (int64_t u = u0; u < u1; ++u, ++i) {
      const int64_t b = u / p.tiles_per_seq, tile = u % p.tiles_per_seq;
      const bool last_in_seg = (u + 1 == u1) || ((u + 1) / p.tiles_per_seq != b);
      const int buf = (int)(i & 1);
      const int kb = (int)(i >> 1);
      const int ks = (int)(i % kNKr);
      float* stage = reinterpret_cast<float*>(smem + kOffKr + ks * kChunk);
      warp_wait(&bb.s_full[buf], kb & 1, abort_flag, p, 0x300);
      ptx::tc_fence_after();
      float sc[kHH], sr[kHH];
      ptx::tmem_ld8(t_cols + kColS + 32 * buf, sc);
      ptx::tmem_ld8(t_cols + kColS + 32 * buf + 16, sr);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bb.s_empty[buf]);

      const int64_t tok0 = tile * kT;
      const int64_t t = tok0 + row;
      const bool valid = t < p.L;
      const bool grouped = t < win0;
      // tile-uniform flags
      const bool tile_groups = (g > 1) && (tok0 < win0);
      const bool tile_tokens = (g == 1) || (tok0 + kT > win0);   // per-token entries present
      float s[kHH];
#pragma unroll
      for (int h = 0; h < kHH; ++h) s[h] = sc[h] + sr[h];

      if (tile_groups) {
        *reinterpret_cast<float4*>(stage + stage_idx(row, kHH * hh)) =
            make_float4(sc[0], sc[1], sc[2], sc[3]);
        *reinterpret_cast<float4*>(stage + stage_idx(row, kHH * hh + 4)) =
            make_float4(sc[4], sc[5], sc[6], sc[7]);
        *reinterpret_cast<float4*>(stage + stage_idx(row, 16 + kHH * hh)) =
            make_float4(sr[0], sr[1], sr[2], sr[3]);
        *reinterpret_cast<float4*>(stage + stage_idx(row, 16 + kHH * hh + 4)) =
            make_float4(sr[4], sr[5], sr[6], sr[7]);
      }
      ptx::named_bar_sync(kSoftmaxBar, kSoftmaxThreads);          // B1: staged scores visible

      if (tile_groups) {
        // ---- step 2: this thread's 8-token segment of head gh
        const int row0 = 8 * sg;
        float x[8], cv[8];
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          cv[v] = stage[stage_idx(row0 + v, gh)];
          x[v] = cv[v] + stage[stage_idx(row0 + v, 16 + gh)];   // the same fp32 sum as s above
        }
        float gm = -INFINITY;
        if (g >= 8) {
          GroupStat r = scan_group<8>(x, cv, 0, row0);
          // merge the g/8 segments of a group (consecutive lanes)
#pragma unroll
          for (int off = 1; off < (g >= 8 ? g / 8 : 1); off <<= 1) {
            const float om = __shfl_xor_sync(0xffffffffu, r.m, off);
            const int oa = __shfl_xor_sync(0xffffffffu, r.a, off);
            const float od = __shfl_xor_sync(0xffffffffu, r.den, off);
            const float on = __shfl_xor_sync(0xffffffffu, r.num, off);
            const float mm = fmaxf(r.m, om);
            const float f1 = ex2((r.m - mm) * kLog2e), f2 = ex2((om - mm) * kLog2e);
            r.den = r.den * f1 + od * f2;
            r.num = r.num * f1 + on * f2;
            if (om > r.m || (om == r.m && oa < r.a)) r.a = oa;
            r.m = mm;
          }
          const int j = row0 / g;                    // group within the tile
          const int64_t jg = tok0 / g + j;            // group within the sequence
          if (jg < p.nG) {
            const float S = __fdividef(r.num, r.den) + stage[stage_idx(r.a, 16 + gh)];
            gm = S;
            if ((sg & (g / 8 - 1)) == 0) {
              ks_tab[j * kHC + gh] = S - r.m - lg2(r.den) * kLn2;
              p.anchor[((int64_t)b * p.H + h0 + gh) * p.nG + jg] = (int32_t)(tok0 + r.a);
            }
          }
        } else {
#pragma unroll
          for (int q = 0; q < 8 / g; ++q) {
            const GroupStat r = scan_group<(g < 8 ? g : 1)>(x, cv, q * g, row0);
            const int j = row0 / g + q;
            const int64_t jg = tok0 / g + j;
            if (jg < p.nG) {
              const float S = __fdividef(r.num, r.den) + stage[stage_idx(r.a, 16 + gh)];
              gm = fmaxf(gm, S);
              ks_tab[j * kHC + gh] = S - r.m - lg2(r.den) * kLn2;
              p.anchor[((int64_t)b * p.H + h0 + gh) * p.nG + jg] = (int32_t)(tok0 + r.a);
            }
          }
        }
        // max over the head's 16 segments (lanes 16*(gh&1) .. +15)
#pragma unroll
        for (int off = 1; off < 16; off <<= 1) gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, off));
        if (sg == 0) gmax_s[gh] = gm;
      }
      if (tile_tokens) {
        // window tokens (and g = 1, where every grouped token is its own entry)
        const bool own = valid && (!grouped || g == 1);
        if (g == 1 && grouped) {
#pragma unroll
          for (int h = 0; h < kHH; ++h)
            p.anchor[((int64_t)b * p.H + h0 + kHH * hh + h) * p.nG + t] = (int32_t)t;
        }
#pragma unroll
        for (int h = 0; h < kHH; ++h) {
          float v = own ? s[h] : -INFINITY;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
          if (lane == 0) wmax_s[q4 * kHC + kHH * hh + h] = v;
        }
      }
      // B2, checkpoint: the only place the softmax warps leave the loop early
      const bool stop = ptx::named_bar_or(kSoftmaxBar, kSoftmaxThreads, *abort_flag != 0);
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bb.empty_k[ks]);   // staging in the K_R slot is done
      if (stop) break;

      // ---- step 3: tile maximum over entries, per-token weights
      float alpha[kHH], mb[kHH], kt[kHH];
#pragma unroll
      for (int h = 0; h < kHH; ++h) {
        const int hg = kHH * hh + h;
        float mt = tile_groups ? gmax_s[hg] : -INFINITY;
        if (tile_tokens)
          mt = fmaxf(mt, fmaxf(fmaxf(wmax_s[hg], wmax_s[kHC + hg]),
                               fmaxf(wmax_s[2 * kHC + hg], wmax_s[3 * kHC + hg])));
        const float mn = fmaxf(Mh[h], mt);
        alpha[h] = ex2((Mh[h] - mn) * kLog2e);   // 0 on the first tile of a range
        Mh[h] = mn;
        mb[h] = mn * kLog2e;
        kt[h] = 0.f;
      }
      if (grouped && g > 1) {
        const float* kr = ks_tab + (row / g) * kHC + kHH * hh;
        const float4 k0 = *reinterpret_cast<const float4*>(kr);
        const float4 k1 = *reinterpret_cast<const float4*>(kr + 4);
        kt[0] = k0.x; kt[1] = k0.y; kt[2] = k0.z; kt[3] = k0.w;
        kt[4] = k1.x; kt[5] = k1.y; kt[6] = k1.z; kt[7] = k1.w;
      }
      float pv[kHH];
#pragma unroll
      for (int h = 0; h < kHH; ++h) pv[h] = valid ? ex2(fmaf(s[h] + kt[h], kLog2e, -mb[h])) : 0.f;
      // ---- P^T tile, bf16, MN-major core matrices: token row -> K, head -> N
      uint32_t pk[4];
#pragma unroll
      for (int h2 = 0; h2 < 4; ++h2) {
        pk[h2] = pack_bf16x2(pv[2 * h2], pv[2 * h2 + 1]);
        const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&pk[h2]);
        Zt[2 * h2] = fmaf(Zt[2 * h2], alpha[2 * h2], __low2float(v));   // Z from the rounded P
        Zt[2 * h2 + 1] = fmaf(Zt[2 * h2 + 1], alpha[2 * h2 + 1], __high2float(v));
      }
      uint8_t* prow = pbase + buf * kPBytes + (row >> 3) * 128 + (row & 7) * 16 + hh * 2048;
      *reinterpret_cast<uint4*>(prow) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bb.p_full[buf]);

      // ---- fold the previous tile's O^T; at a range end also this tile's, then write
      if (pending) fold_o(O, apend, pbuf, pkb, t_cols, bb, abort_flag, p);
#pragma unroll
      for (int h = 0; h < kHH; ++h) apend[h] = alpha[h];
      pending = true;
      pbuf = buf;
      pkb = kb;
      if (last_in_seg) {
        fold_o(O, alpha, buf, kb, t_cols, bb, abort_flag, p);
        pending = false;
        const int64_t slot = b + c;
#pragma unroll
        for (int h = 0; h < kHH; ++h) {
          float* po = p.part_o + (slot * p.H + h0 + kHH * hh + h) * kDC;
#pragma unroll
          for (int m = 0; m < 4; ++m) po[128 * m + row] = O[m][h];
          float z = Zt[h];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
          if (lane == 0) zred[q4 * kHC + kHH * hh + h] = z;
        }
        ptx::named_bar_sync(kSoftmaxBar, kSoftmaxThreads);
        if (q4 == 0 && lane < kHH) {
          float Mv = 0.f;
#pragma unroll
          for (int h = 0; h < kHH; ++h) if (h == lane) Mv = Mh[h];
          const int hg = kHH * hh + lane;
          const float z = zred[hg] + zred[kHC + hg] + zred[2 * kHC + hg] + zred[3 * kHC + hg];
          p.part_mz[(slot * p.H + h0 + hg) * 2 + 0] = Mv;
          p.part_mz[(slot * p.H + h0 + hg) * 2 + 1] = z;
        }
        ptx::named_bar_sync(kSoftmaxBar, kSoftmaxThreads);
#pragma unroll
        for (int h = 0; h < kHH; ++h) {
          Zt[h] = 0.f; Mh[h] = -INFINITY;
#pragma unroll
          for (int m = 0; m < 4; ++m) O[m][h] = 0.f;
        }
      }
    }
  }

  // ===================================================== teardown
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
