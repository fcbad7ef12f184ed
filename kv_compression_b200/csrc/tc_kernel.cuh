// tc_kernel.cuh -- LCA / dense-MLA decode with tcgen05 tensor cores, TMEM
// accumulators and TMA tile loads (sm_100a), bf16 latents, fp32 accumulation.
//
// What one CTA computes ("Latent-Condensed Transformer for Efficient Long
// Context Modeling", section 2, "O Algoritmo LCA", steps 1-3) for 16 heads of
// one sequence over a contiguous range of 128-token tiles:
//   scores     S^T[128 tokens x 16 heads] = [C_KV | K_R]_tile . [q_c | q_r]^T,
//              two TMEM accumulators, sc (K = 512) and sr (K = 64), because the
//              condensed logit needs the semantic part on its own;
//   condense   (step 2) one thread per (group, head) runs over the g tokens of
//              its group: max and lowest-index argmax (the anchor a_j), the
//              group-local softmax sums den_j = sum e^{s_t - m_j} and
//              num_j = sum e^{s_t - m_j} sc_t, and the condensed logit
//              S_j = num_j / den_j + sr_{a_j}  (= q_c.c_bar_j + q_r.k_{a_j};
//              c_bar_j is never formed);
//   attend     (step 3) online softmax over [condensed || window].  A grouped
//              token's weight p_j w_t = e^{S_j - M} e^{s_t - m_j} / den_j is
//              written e^{s_t + k_j - M} with k_j = S_j - m_j - ln den_j, a window
//              token's e^{s_t - M}: one exponential per (token, head).  The
//              weights go to shared memory as bf16 and O^T[512 x 16] +=
//              C_KV_tile^T . P^T is one more MMA per tile.
// The range's partial (M, Z, O) goes to the workspace; the combine kernel
// merges the ranges of a sequence.
//
// Roles (192 threads): warp 0 lane 0 issues TMA loads; warp 1 allocates TMEM
// and its lane 0 issues MMAs; warps 2-5 (128 threads, one per TMEM lane) do
// the softmax work.  Shared memory: a ring of five 32 KB slots for C_KV
// column pairs ([128 tokens][2 x 64 dims], 128-byte swizzle), two 16 KB K_R
// slots (each reused to stage its tile's scores once the score MMA is done),
// the query block (9 x [16 heads][64 dims]) and two P buffers.
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
constexpr int kThreads = 192;
constexpr int kTmemCols = 256;
constexpr int kSoftmaxBar = 1;             // named barrier of the 4 softmax warps
constexpr int kMaxGroupsPerTile = 64;      // g >= 2 (g = 1 takes the per-token path)
constexpr float kLog2e = 1.4426950408889634f;

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

// Score staging in a K_R slot: [128 rows][32 floats] (sc of 16 heads, then sr),
// float4 columns XOR-swizzled by (row ^ group-of-row) so that the group phase
// (threads on different groups, same step) reads distinct banks.
template <int LOG2G>
__device__ __forceinline__ int stage_idx(int row, int col) {
  const int sw = ((row ^ (row >> LOG2G)) & 7) << 2;
  return row * 32 + (col ^ sw);
}

// Fold the O^T tile in TMEM buffer `ob` (its use `okb`) into the register
// accumulator: O = O * al + O_tile.  Thread = latent row of each 128-row block.
__device__ __forceinline__ void fold_o(float (&O)[4][kHC], const float (&al)[kHC], int ob, int okb,
                                       uint32_t t_lane, const Bars& bb, volatile int* abort_flag,
                                       const TcParams& p) {
  warp_wait(&bb.o_full[ob], okb & 1, abort_flag, p, 0x303);
  ptx::tc_fence_after();
#pragma unroll
  for (int m = 0; m < 4; ++m) {
    float ot[kHC];
    ptx::tmem_ld16(t_lane + kColO + 64 * ob + 16 * m, ot);
    ptx::tmem_wait_ld();
#pragma unroll
    for (int h = 0; h < kHC; ++h) O[m][h] = fmaf(O[m][h], al[h], ot[h]);
  }
  ptx::tc_fence_before();
  __syncwarp();
  if ((threadIdx.x & 31) == 0) ptx::mbar_arrive(&bb.o_empty[ob]);
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
    for (int i = 0; i < kNKr; ++i) { ptx::mbar_init(&bb.full_k[i], 1); ptx::mbar_init(&bb.empty_k[i], 4); }
    ptx::mbar_init(bb.q_full, 1);
    ptx::mbar_init(bb.q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bb.s_full[i], 1);
      ptx::mbar_init(&bb.s_empty[i], 4);
      ptx::mbar_init(&bb.p_full[i], 4);
      ptx::mbar_init(&bb.o_full[i], 1);
      ptx::mbar_init(&bb.o_empty[i], 4);
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
    ptx::prefetch_tmap(&p.tm_c);
    ptx::prefetch_tmap(&p.tm_k);
    ptx::prefetch_tmap(&p.tm_qc);
    ptx::prefetch_tmap(&p.tm_qr);
    int issued_c[kNPair], issued_k[kNKr];
    for (int i = 0; i < kNPair; ++i) issued_c[i] = -1;
    for (int i = 0; i < kNKr; ++i) issued_k[i] = -1;
    int issued_q = -1;
    int64_t nc = 0, nk = 0;
    int seg = -1;
    int64_t cur_b = -1;
    bool ok = true;
    for (int64_t u = u0; u < u1 && ok; ++u) {
      const int64_t b = u / p.tiles_per_seq, tile = u % p.tiles_per_seq;
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
      const int32_t row = (int32_t)(b * p.L + tile * kT);
      {
        const int ks = (int)(nk % kNKr);
        const int kk = (int)(nk / kNKr);
        if (kk >= 1) ok = bounded_wait(&bb.empty_k[ks], (kk - 1) & 1, abort_flag, p, 0x101, true);
        if (!ok) break;
        if (!(p.debug_skip_load && nk == 0)) {
          ptx::mbar_arrive_expect_tx(&bb.full_k[ks], kChunk);
          ptx::tma_load_2d(smem + kOffKr + ks * kChunk, &p.tm_k, 0, row, &bb.full_k[ks]);
          issued_k[ks] = kk;
        }
        ++nk;
      }
      for (int pr = 0; pr < 4 && ok; ++pr) {
        const int cs = (int)(nc % kNPair);
        const int ck = (int)(nc / kNPair);
        if (ck >= 1) ok = bounded_wait(&bb.empty_c[cs], (ck - 1) & 1, abort_flag, p, 0x102, true);
        if (!ok) break;
        ptx::mbar_arrive_expect_tx(&bb.full_c[cs], kPairBytes);
        uint8_t* dst = smem + kOffPair + cs * kPairBytes;
        ptx::tma_load_2d(dst, &p.tm_c, 128 * pr, row, &bb.full_c[cs]);
        ptx::tma_load_2d(dst + kChunk, &p.tm_c, 128 * pr + 64, row, &bb.full_c[cs]);
        issued_c[cs] = ck;
        ++nc;
      }
    }
    // Let every copy this thread started land before the CTA can exit.
    for (int i = 0; i < kNPair; ++i)
      if (issued_c[i] >= 0) bounded_wait(&bb.full_c[i], issued_c[i] & 1, abort_flag, p, 0x1F0, false);
    for (int i = 0; i < kNKr; ++i)
      if (issued_k[i] >= 0) bounded_wait(&bb.full_k[i], issued_k[i] & 1, abort_flag, p, 0x1F1, false);
    if (issued_q >= 0) bounded_wait(bb.q_full, issued_q & 1, abort_flag, p, 0x1F2, false);
  } else if (warp == 1 && lane == 0) {
    // ===================================================== MMA issuer
    constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(kT, kHC, 0, 0);   // K-major A and B
    constexpr uint32_t kIdescP = ptx::idesc_bf16_f32(128, kHC, 1, 1);  // MN-major A and B
    const uint32_t s_pair = ptx::smem_u32(smem + kOffPair);
    const uint32_t s_kr = ptx::smem_u32(smem + kOffKr);
    const uint32_t s_q = ptx::smem_u32(smem + kOffQ);
    const uint32_t s_p = ptx::smem_u32(smem + kOffP);
    int64_t nc = 0, nk = 0, i = 0;
    int seg = -1;
    int64_t cur_b = -1;
    bool ok = true;
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
      const uint32_t d_sc = tmem + kColS + 32 * buf;
      const uint32_t d_sr = d_sc + 16;
      // ---- sr = K_R tile . q_r^T
      {
        const int ks = (int)(nk % kNKr);
        ok = bounded_wait(&bb.full_k[ks], (int)(nk / kNKr) & 1, abort_flag, p, 0x202, true);
        if (!ok) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint64_t a = ptx::smem_desc(s_kr + ks * kChunk + 32 * k, 16, 1024, ptx::kSwizzle128B);
          const uint64_t bq = ptx::smem_desc(s_q + 8 * kQChunk + 32 * k, 16, 1024, ptx::kSwizzle128B);
          ptx::mma_bf16_ss(d_sr, a, bq, kIdescS, k > 0);
        }
        ++nk;
      }
      // ---- sc = C_KV tile . q_c^T, one column pair (128 dims) per ring slot
      int slotp[4];
      for (int pr = 0; pr < 4; ++pr) {
        const int cs = (int)(nc % kNPair);
        ok = bounded_wait(&bb.full_c[cs], (int)(nc / kNPair) & 1, abort_flag, p, 0x203, true);
        if (!ok) break;
        ptx::tc_fence_after();
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const uint64_t a = ptx::smem_desc(s_pair + cs * kPairBytes + ch * kChunk + 32 * k, 16,
                                              1024, ptx::kSwizzle128B);
            const uint64_t bq = ptx::smem_desc(s_q + (2 * pr + ch) * kQChunk + 32 * k, 16, 1024,
                                               ptx::kSwizzle128B);
            ptx::mma_bf16_ss(d_sc, a, bq, kIdescS, (pr | ch | k) != 0);
          }
        }
        slotp[pr] = cs;
        ++nc;
      }
      if (!ok) break;
      ptx::mma_commit(&bb.s_full[buf]);   // also tells the softmax warps the K_R slot is read
      if (last_in_seg) ptx::mma_commit(bb.q_empty);
      // ---- O^T tile = C_KV tile^T . P^T, four 128-dim blocks
      ok = bounded_wait(&bb.p_full[buf], kb & 1, abort_flag, p, 0x204, true);
      if (ok && kb >= 1) ok = bounded_wait(&bb.o_empty[buf], (kb - 1) & 1, abort_flag, p, 0x205, true);
      if (!ok) break;
      ptx::tc_fence_after();
      for (int m = 0; m < 4; ++m) {
        const uint32_t d_o = tmem + kColO + 64 * buf + 16 * m;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // A = C^T: M = 128 latent dims (two 64-dim atoms 16 KB apart), K = 16 tokens
          const uint64_t a = ptx::smem_desc(s_pair + slotp[m] * kPairBytes + kk * 2048, kChunk,
                                            1024, ptx::kSwizzle128B);
          // B = P^T: N = 16 heads (8-head core blocks 2 KB apart), K = 16 tokens
          const uint64_t bp = ptx::smem_desc(s_p + buf * kPBytes + kk * 256, 128, 2048,
                                             ptx::kSwizzleNone);
          ptx::mma_bf16_ss(d_o, a, bp, kIdescP, kk > 0);
        }
        ptx::mma_commit(&bb.empty_c[slotp[m]]);
      }
      ptx::mma_commit(&bb.o_full[buf]);
    }
    // Every MMA issued here must finish before TMEM is freed.
    ptx::mma_commit(bb.drain);
    bounded_wait(bb.drain, 0, abort_flag, p, 0x2F0, false);
  } else if (warp >= 2) {
    // ===================================================== softmax warps
    // A failed wait only raises the abort flag; the four warps leave the tile
    // loop together, at the one checkpoint barrier of each tile, so no warp
    // is ever left waiting at a named barrier.
    const int q4 = warp & 3;             // TMEM lane quarter this warp may access
    const int row = q4 * 32 + lane;      // token row of the tile owned by this thread
    const int st = tid - 64;             // 0..127 among the softmax threads
    const uint32_t t_lane = tmem + ((uint32_t)(q4 * 32) << 16);
    float* ks_tab = reinterpret_cast<float*>(smem + kOffK);      // [64][16] k_j
    float* gmax_s = reinterpret_cast<float*>(smem + kOffGmax);   // [16]
    float* wmax_s = reinterpret_cast<float*>(smem + kOffWmax);   // [4][16]
    float* zred = reinterpret_cast<float*>(smem + kOffZred);     // [4][16]
    uint8_t* pbase = smem + kOffP;
    // group phase: threads per head (consecutive), groups per thread
    constexpr int kGt = kT / g;                          // groups per tile
    constexpr int kTpH = kGt < 8 ? kGt : 8;
    constexpr int kGpt = kGt / kTpH;
    constexpr int kActive = kHC * kTpH;
    constexpr int kUnroll = g < 16 ? g : 16;             // full unroll would spill for g >= 64

    float O[4][kHC];
    float Zt[kHC], Mh[kHC], apend[kHC];
#pragma unroll
    for (int h = 0; h < kHC; ++h) {
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
      float sc[kHC], sr[kHC];
      ptx::tmem_ld16(t_lane + kColS + 32 * buf, sc);
      ptx::tmem_ld16(t_lane + kColS + 32 * buf + 16, sr);
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
      float s[kHC];
#pragma unroll
      for (int h = 0; h < kHC; ++h) s[h] = sc[h] + sr[h];

      if (tile_groups) {
#pragma unroll
        for (int c4 = 0; c4 < 8; ++c4) {
          const float4 v = c4 < 4 ? make_float4(sc[4 * c4], sc[4 * c4 + 1], sc[4 * c4 + 2], sc[4 * c4 + 3])
                                  : make_float4(sr[4 * c4 - 16], sr[4 * c4 - 15], sr[4 * c4 - 14],
                                                sr[4 * c4 - 13]);
          *reinterpret_cast<float4*>(stage + stage_idx<LOG2G>(row, 4 * c4)) = v;
        }
      }
      ptx::named_bar_sync(kSoftmaxBar, 128);                     // B1: staged scores visible

      if (tile_groups && st < kActive) {
        // ---- step 2, one thread per (group, head)
        const int h = st / kTpH;
        const int j0 = st % kTpH;
        float gm = -INFINITY;
#pragma unroll
        for (int r = 0; r < kGpt; ++r) {
          const int j = j0 + kTpH * r;                 // group within the tile
          const int64_t jg = tok0 / g + j;             // group within the sequence
          if (jg < p.nG) {
            const int r0 = j * g;
            float m = -INFINITY;
            int a = 0;
#pragma unroll kUnroll
            for (int v = 0; v < g; ++v) {
              const float x = stage[stage_idx<LOG2G>(r0 + v, h)] + stage[stage_idx<LOG2G>(r0 + v, 16 + h)];
              if (x > m) { m = x; a = v; }             // strict: the lowest index keeps a tie
            }
            float den = 0.f, num = 0.f;
            const float mb = m * kLog2e;
#pragma unroll kUnroll
            for (int v = 0; v < g; ++v) {
              const float scv = stage[stage_idx<LOG2G>(r0 + v, h)];
              const float x = scv + stage[stage_idx<LOG2G>(r0 + v, 16 + h)];
              const float e = ex2(fmaf(x, kLog2e, -mb));
              den += e;
              num = fmaf(e, scv, num);
            }
            const float sra = stage[stage_idx<LOG2G>(r0 + a, 16 + h)];   // K_R score of the anchor
            const float S = __fdividef(num, den) + sra;                 // condensed logit
            ks_tab[j * kHC + h] = S - m - __logf(den);                  // k_j
            gm = fmaxf(gm, S);
            p.anchor[((int64_t)b * p.H + h0 + h) * p.nG + jg] = (int32_t)(tok0 + r0 + a);
          }
        }
#pragma unroll
        for (int off = 1; off < kTpH; off <<= 1)
          gm = fmaxf(gm, __shfl_xor_sync(0xffffffffu, gm, off));
        if (j0 == 0) gmax_s[h] = gm;
      }
      if (tile_tokens) {
        // window tokens (and g = 1, where every grouped token is its own entry)
        const bool own = valid && (!grouped || g == 1);
        if (g == 1 && grouped) {
#pragma unroll
          for (int h = 0; h < kHC; ++h)
            p.anchor[((int64_t)b * p.H + h0 + h) * p.nG + t] = (int32_t)t;
        }
#pragma unroll
        for (int h = 0; h < kHC; ++h) {
          float v = own ? s[h] : -INFINITY;
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
          if (lane == 0) wmax_s[q4 * kHC + h] = v;
        }
      }
      // B2, checkpoint: the only place the softmax warps leave the loop early
      const bool stop = ptx::named_bar_or(kSoftmaxBar, 128, *abort_flag != 0);
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bb.empty_k[ks]);   // staging in the K_R slot is done
      if (stop) break;

      // ---- step 3: tile maximum over entries, per-token weights
      float alpha[kHC], mb[kHC];
#pragma unroll
      for (int h = 0; h < kHC; ++h) {
        float mt = tile_groups ? gmax_s[h] : -INFINITY;
        if (tile_tokens)
          mt = fmaxf(mt, fmaxf(fmaxf(wmax_s[h], wmax_s[kHC + h]),
                               fmaxf(wmax_s[2 * kHC + h], wmax_s[3 * kHC + h])));
        const float mn = fmaxf(Mh[h], mt);
        alpha[h] = ex2((Mh[h] - mn) * kLog2e);   // 0 on the first tile of a range
        Mh[h] = mn;
        mb[h] = mn * kLog2e;
      }
      float pv[kHC];
      if (grouped && g > 1) {
        const float* kr = ks_tab + (row / g) * kHC;
#pragma unroll
        for (int h4 = 0; h4 < 4; ++h4) {
          const float4 k4 = *reinterpret_cast<const float4*>(kr + 4 * h4);
          pv[4 * h4 + 0] = ex2(fmaf(s[4 * h4 + 0] + k4.x, kLog2e, -mb[4 * h4 + 0]));
          pv[4 * h4 + 1] = ex2(fmaf(s[4 * h4 + 1] + k4.y, kLog2e, -mb[4 * h4 + 1]));
          pv[4 * h4 + 2] = ex2(fmaf(s[4 * h4 + 2] + k4.z, kLog2e, -mb[4 * h4 + 2]));
          pv[4 * h4 + 3] = ex2(fmaf(s[4 * h4 + 3] + k4.w, kLog2e, -mb[4 * h4 + 3]));
        }
      } else {
#pragma unroll
        for (int h = 0; h < kHC; ++h) pv[h] = valid ? ex2(fmaf(s[h], kLog2e, -mb[h])) : 0.f;
      }
      // ---- P^T tile, bf16, MN-major core matrices: token row -> K, head -> N
      uint32_t pk[8];
#pragma unroll
      for (int h2 = 0; h2 < 8; ++h2) {
        pk[h2] = pack_bf16x2(pv[2 * h2], pv[2 * h2 + 1]);
        const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&pk[h2]);
        Zt[2 * h2] = fmaf(Zt[2 * h2], alpha[2 * h2], __low2float(v));   // Z from the rounded P
        Zt[2 * h2 + 1] = fmaf(Zt[2 * h2 + 1], alpha[2 * h2 + 1], __high2float(v));
      }
      uint8_t* prow = pbase + buf * kPBytes + (row >> 3) * 128 + (row & 7) * 16;
      *reinterpret_cast<uint4*>(prow) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      *reinterpret_cast<uint4*>(prow + 2048) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bb.p_full[buf]);

      // ---- fold the previous tile's O^T; at a range end also this tile's, then write
      if (pending) fold_o(O, apend, pbuf, pkb, t_lane, bb, abort_flag, p);
#pragma unroll
      for (int h = 0; h < kHC; ++h) apend[h] = alpha[h];
      pending = true;
      pbuf = buf;
      pkb = kb;
      if (last_in_seg) {
        fold_o(O, alpha, buf, kb, t_lane, bb, abort_flag, p);
        pending = false;
        const int64_t slot = b + c;
#pragma unroll
        for (int h = 0; h < kHC; ++h) {
          float* po = p.part_o + (slot * p.H + h0 + h) * kDC;
#pragma unroll
          for (int m = 0; m < 4; ++m) po[128 * m + row] = O[m][h];
          float z = Zt[h];
#pragma unroll
          for (int off = 16; off > 0; off >>= 1) z += __shfl_xor_sync(0xffffffffu, z, off);
          if (lane == 0) zred[q4 * kHC + h] = z;
        }
        ptx::named_bar_sync(kSoftmaxBar, 128);
        if (warp == 2 && lane < kHC) {
          float Mv = 0.f;
#pragma unroll
          for (int h = 0; h < kHC; ++h) if (h == lane) Mv = Mh[h];
          const float z = zred[lane] + zred[kHC + lane] + zred[2 * kHC + lane] + zred[3 * kHC + lane];
          p.part_mz[(slot * p.H + h0 + lane) * 2 + 0] = Mv;
          p.part_mz[(slot * p.H + h0 + lane) * 2 + 1] = z;
        }
        ptx::named_bar_sync(kSoftmaxBar, 128);
#pragma unroll
        for (int h = 0; h < kHC; ++h) {
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
