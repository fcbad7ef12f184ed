// pair_kernel.cuh -- LCA / dense-MLA decode for 128 heads sharing one latent,
// on a cluster of two CTAs that split the latent width: tcgen05 tensor cores,
// TMEM accumulators, TMA tile loads, distributed shared memory (sm_100a),
// bf16 latents, fp32 accumulation.
//
// What one cluster computes ("Latent-Condensed Transformer for Efficient Long
// Context Modeling", section 2, "O Algoritmo LCA", steps 1-3) for 128 heads of
// one sequence over a contiguous range of 64-token tiles.  CTA r of the pair
// holds latent dims [256 r, 256 r + 256) of every tile, and runs the softmax
// of heads [64 r, 64 r + 64):
//   scores     S_r[128 heads x 64 tokens] = Q_c[:, dims_r] . C_KV[tile, dims_r]^T
//              (partial over its own dims, every head) and sr = q_r . K_R^T
//              (its own heads), both in TMEM with heads in lanes.  Each CTA
//              sends the partial scores of the other CTA's heads to it
//              (st.async into its shared memory), so that each head's full
//              score sc_t = S_0 + S_1 is formed by the CTA that owns the head;
//   condense   (step 2) one thread holds one head and 32 consecutive tokens, so
//              a group of g <= 32 tokens is reduced inside the thread: max,
//              lowest-index argmax (the anchor a_j), e_t = e^{s_t - m_j},
//              den_j = sum e_t, num_j = sum e_t sc_t and the condensed logit
//              S_j = num_j / den_j + sr_{a_j}.  A 64-token group merges the
//              statistics of the head's two threads through shared memory;
//   attend     (step 3) softmax over [condensed || window] against a reference
//              max M per head: a grouped token weighs e_t e^{S_j - M} / den_j,
//              a window token e^{s_t - M}.  The bf16 weights P[128 heads x 64
//              tokens] (own rows written here, the other rows copied in by the
//              peer) feed O[128 heads x 256 dims_r] += P . C_KV[tile, dims_r],
//              accumulated in TMEM.  M rises only when an entry exceeds it by
//              more than 2^8; then the head's O rows are rescaled in both CTAs
//              (the factor travels with P).
// Each CTA writes its dims of every head's partial O, the owner CTA the
// head's (M, Z); the combine kernel merges the ranges of a sequence.
//
// Every C_KV byte is read from HBM once and into shared memory once (each CTA
// loads only its half); K_R is loaded by both CTAs.
//
// Roles (352 threads): warp 0 lane 0 issues TMA loads; warp 1 allocates TMEM
// and its lane 0 issues the score MMAs; warp 2 lane 0 issues the O MMAs;
// warps 3-10 are "quarter warps": warp w may access TMEM lanes 32 (w % 4) ..
// +31.  In the two quarters that hold the CTA's own heads, two warps each run
// the softmax (token halves 0 and 1 of a tile).  In the other two quarters
// one warp ships the partial scores to the peer and one applies the peer's
// rescale factors to those heads' O rows.
// Every mbarrier wait is bounded; when a bound runs out the CTA records the
// error, stops issuing work, waits for its own copies and MMAs in flight,
// frees TMEM and exits after its peer.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

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
constexpr int kQrBytes = kOwn * 128;        // the own heads' q_r, 8 KB
constexpr int kPBytes = kHeads * kT * 2;    // P[128 heads][64 tokens] bf16, 16 KB
constexpr int kPOwnBytes = kOwn * kT * 2;   // the rows a CTA writes, 8 KB
constexpr int kRecvBytes = kOwn * kT * 4;   // partial scores from the peer, 16 KB
constexpr int kAlphaOwnBytes = kOwn * 4;
constexpr int kSoftmaxThreads = 128;        // four softmax warps
constexpr int kThreads = 32 * 11;
constexpr int kTmemCols = 512;
constexpr int kSoftmaxBar = 1;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kRescaleLog2 = 8.f;

// shared memory map (offsets from a 1024-byte aligned base; equal in both CTAs)
constexpr int kOffQc = 0;
constexpr int kOffQr = kOffQc + kAtoms * kQcAtom;
constexpr int kOffC = kOffQr + kQrBytes;
constexpr int kOffKr = kOffC + kNS * kStage;
constexpr int kOffP = kOffKr + kNKr * kKrBytes;
constexpr int kOffRecv = kOffP + kPBytes;
constexpr int kOffAlpha = kOffRecv + kRecvBytes;           // float [128]: rescale factor per head
constexpr int kOffGst = kOffAlpha + kHeads * 4;            // float4 [2][64]: 64-token group halves
constexpr int kOffGan = kOffGst + 2 * kOwn * 16;           // int [2][64]
constexpr int kOffMt = kOffGan + 2 * kOwn * 4;             // float [2][64]: tile maxima
constexpr int kOffZt = kOffMt + 2 * kOwn * 4;              // float [2][64]: Z halves
constexpr int kOffBar = kOffZt + 2 * kOwn * 4;
constexpr int kNumBars = 2 * kNS + 2 * kNKr + 2 + 2 + 2 + 2 + 2 + 1 + 2 + 2;
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 16;
constexpr int kSmemAlloc = kSmemBytes + 1024;
static_assert(kSmemAlloc <= 232448, "shared memory budget of one sm_100 CTA");
static_assert(kOffQr >= 8192, "the peer-row offset of the q_r descriptor stays inside the CTA");
static_assert(kOffC % 1024 == 0 && kOffKr % 1024 == 0 && kOffP % 1024 == 0, "swizzle atoms");

// TMEM columns: S buffer b: partial sc at 128 b, sr at 128 b + 64;  O at 256.
constexpr uint32_t kColO = 256;

constexpr int kErrTimeout = 1;

struct PairParams {
  CUtensorMap tm_c;    // c_kv as [B*L rows][512], box [64 rows][64], 128B swizzle
  CUtensorMap tm_k;    // k_r  as [B*L rows][64],  box [64 rows][64], 128B swizzle
  CUtensorMap tm_qc;   // q_c  as [B*H rows][512], box [128 rows][64], 128B swizzle
  CUtensorMap tm_qr;   // q_r  as [B*H rows][64],  box [64 rows][64], 128B swizzle
  int B, H;
  int64_t L;
  int64_t nG;          // condensed groups (0: dense attention)
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
};

struct Bars {
  uint64_t* c_full;      // [kNS] a tile's C_KV half landed
  uint64_t* c_empty;     // [kNS] released after O of that tile
  uint64_t* kr_full;     // [kNKr]
  uint64_t* kr_empty;    // [kNKr] released after the sr MMAs
  uint64_t* q_full;
  uint64_t* q_empty;
  uint64_t* s_full;      // [2] the scores of a tile are in TMEM
  uint64_t* s_empty;     // [2] the softmax and shipper warps have read them
  uint64_t* recv_full;   // the peer's partial scores of a tile landed (transaction bytes)
  uint64_t* recv_free;   // the peer has read the partial scores this CTA sent it
  uint64_t* p_local;     // the own rows of P are written
  uint64_t* p_remote;    // the peer's rows of P and its rescale factors landed
  uint64_t* lanes_ready; // the peer heads' O rows are rescaled (if asked)
  uint64_t* o_done;      // [2] O of a tile is done in CTA 0 / CTA 1 (both CTAs arrive)
  uint64_t* drain;       // [2]
};

__device__ __forceinline__ void record_timeout(volatile int* abort, const PairParams& p, int where) {
  *abort = 1;
  if (atomicOr(p.err, kErrTimeout) == 0) atomicExch(p.err + 1, where);
}

// Bounded wait.  `cluster`: acquire at cluster scope (barriers that the peer
// CTA arrives on or completes transactions on).
__device__ __noinline__ bool bounded_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          const PairParams& p, int where, bool honour_abort,
                                          bool cluster) {
  auto probe = [&]() {
    return cluster ? ptx::mbar_try_wait_cluster(bar, parity) : ptx::mbar_try_wait(bar, parity);
  };
  if (probe()) return true;
  const uint64_t t0 = ptx::globaltimer_ns();
  for (uint32_t spin = 1;; ++spin) {
    if (probe()) return true;
    if (honour_abort && *abort) return false;
    if ((spin & 63u) == 0 && ptx::globaltimer_ns() - t0 > p.timeout_ns) {
      record_timeout(abort, p, where);
      return false;
    }
  }
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort,
                                          const PairParams& p, int where, bool cluster) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = bounded_wait(bar, parity, abort, p, where, true, cluster);
  __syncwarp();
  return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
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

template <int LOG2G>
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
  bb.s_full = bb.q_empty + 1;
  bb.s_empty = bb.s_full + 2;
  bb.recv_full = bb.s_empty + 2;
  bb.recv_free = bb.recv_full + 1;
  bb.p_local = bb.recv_free + 1;
  bb.p_remote = bb.p_local + 1;
  bb.lanes_ready = bb.p_remote + 1;
  bb.o_done = bb.lanes_ready + 1;
  bb.drain = bb.o_done + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + kOffMisc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffMisc + 4);

  const int64_t cl = blockIdx.x >> 1;
  const int hb = (int)(cl % p.n_hb);
  const int64_t c = cl / p.n_hb;
  const int h0 = hb * kHeads;
  const int64_t u0 = c * p.U / p.G;
  const int64_t u1 = (c + 1) * p.U / p.G;
  const int64_t n_tiles = u1 - u0;
  const int64_t win0 = p.win0;
  const int64_t seq0 = u0 / p.tiles_per_seq;
  const int64_t tile0 = u0 - seq0 * p.tiles_per_seq;
  auto step = [&](int64_t& seq, int64_t& tile) {
    if (++tile == p.tiles_per_seq) { tile = 0; ++seq; }
  };

  if (tid == 0) {
    for (int i = 0; i < kNS; ++i) { ptx::mbar_init(&bb.c_full[i], 1); ptx::mbar_init(&bb.c_empty[i], 1); }
    for (int i = 0; i < kNKr; ++i) { ptx::mbar_init(&bb.kr_full[i], 1); ptx::mbar_init(&bb.kr_empty[i], 1); }
    ptx::mbar_init(bb.q_full, 1);
    ptx::mbar_init(bb.q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(&bb.s_full[i], 1);
      ptx::mbar_init(&bb.s_empty[i], 6);          // 4 softmax + 2 shipper warps
      ptx::mbar_init(&bb.o_done[i], 1);
      ptx::mbar_init(&bb.drain[i], 1);
    }
    ptx::mbar_init(bb.recv_full, 1);              // armed with its transaction bytes
    ptx::mbar_init(bb.recv_free, 4);              // the peer's 4 softmax warps
    ptx::mbar_init(bb.p_local, 4);                // this CTA's 4 softmax warps
    ptx::mbar_init(bb.p_remote, 1);               // armed with its transaction bytes
    ptx::mbar_init(bb.lanes_ready, 2);            // the 2 rescale (checker) warps
    *abort_flag = 0;
    ptx::fence_mbarrier_init();
    // phase 0 of the two barriers the peer completes with transaction bytes
    ptx::mbar_arrive_expect_tx(bb.recv_full, kRecvBytes);
    ptx::mbar_arrive_expect_tx(bb.p_remote, kPOwnBytes + kAlphaOwnBytes);
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
  if (tid == 0) {
    const int32_t frow = (int32_t)(seq0 * p.L + tile0 * kT);
    for (int a = 0; a < kAtoms; ++a) ptx::tma_prefetch_l2_2d(&p.tm_c, kDim * r + 64 * a, frow);
    ptx::tma_prefetch_l2_2d(&p.tm_k, 0, frow);
    const int32_t qrow = (int32_t)(seq0 * p.H + h0);
    for (int a = 0; a < kAtoms; ++a) ptx::tma_prefetch_l2_2d(&p.tm_qc, kDim * r + 64 * a, qrow);
  }
  ptx::griddep_wait();
  ptx::griddep_launch_dependents();

  if (warp == 0 && lane == 0) {
    // ===================================================== TMA producer
    // Per tile: K_R into its slot (after the sr MMAs of the tile two back), then
    // this CTA's half of C_KV into its stage (after O of the tile kNS back).
    ptx::prefetch_tmap(&p.tm_c);
    ptx::prefetch_tmap(&p.tm_k);
    ptx::prefetch_tmap(&p.tm_qc);
    ptx::prefetch_tmap(&p.tm_qr);
    const uint64_t once = ptx::l2_policy_evict_first();
    int issued_c[kNS], issued_k[kNKr];
#pragma unroll
    for (int i = 0; i < kNS; ++i) issued_c[i] = -1;
#pragma unroll
    for (int i = 0; i < kNKr; ++i) issued_k[i] = -1;
    int issued_q = -1, seg = -1;
    int64_t cur_b = -1;
    bool ok = true;
    int64_t pseq = seq0, ptile = tile0;
    for (int64_t i = 0; i < n_tiles && ok; ++i, step(pseq, ptile)) {
      const int64_t b = pseq;
      if (b != cur_b) {
        cur_b = b;
        ++seg;
        if (seg >= 1) ok = bounded_wait(bb.q_empty, (seg - 1) & 1, abort_flag, p, 0x500, true, false);
        if (!ok) break;
        ptx::mbar_arrive_expect_tx(bb.q_full, kAtoms * kQcAtom + kQrBytes);
        const int32_t qrow = (int32_t)(b * p.H + h0);
        for (int a = 0; a < kAtoms; ++a)
          ptx::tma_load_2d(smem + kOffQc + a * kQcAtom, &p.tm_qc, kDim * r + 64 * a, qrow, bb.q_full);
        ptx::tma_load_2d(smem + kOffQr, &p.tm_qr, 0, qrow + kOwn * r, bb.q_full);
        issued_q = seg;
      }
      const int32_t row = (int32_t)(b * p.L + ptile * kT);
      {
        const int ks = (int)(i % kNKr);
        const int kk = (int)(i / kNKr);
        if (kk >= 1) ok = bounded_wait(&bb.kr_empty[ks], (kk - 1) & 1, abort_flag, p, 0x501, true, false);
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
        if (ck >= 1) ok = bounded_wait(&bb.c_empty[cs], (ck - 1) & 1, abort_flag, p, 0x502, true, false);
        if (!ok) break;
        ptx::mbar_arrive_expect_tx(&bb.c_full[cs], kStage);
        uint8_t* dst = smem + kOffC + cs * kStage;
        for (int a = 0; a < kAtoms; ++a)
          ptx::tma_load_2d_hint(dst + a * kCAtom, &p.tm_c, kDim * r + 64 * a, row, &bb.c_full[cs], once);
#pragma unroll
        for (int q = 0; q < kNS; ++q) if (q == cs) issued_c[q] = ck;
      }
    }
    // Let every copy this thread started land before the CTA can exit.
#pragma unroll
    for (int i = 0; i < kNS; ++i)
      if (issued_c[i] >= 0) bounded_wait(&bb.c_full[i], issued_c[i] & 1, abort_flag, p, 0x5F0, false, false);
#pragma unroll
    for (int i = 0; i < kNKr; ++i)
      if (issued_k[i] >= 0) bounded_wait(&bb.kr_full[i], issued_k[i] & 1, abort_flag, p, 0x5F1, false, false);
    if (issued_q >= 0) bounded_wait(bb.q_full, issued_q & 1, abort_flag, p, 0x5F2, false, false);
  } else if (warp == 1 && lane == 0) {
    // ===================================================== score MMA issuer
    // Tile t into S buffer t & 1:  sr[128 x 64] = q_r . K_R^T (the own heads'
    // rows are real; the rest of A is whatever precedes or follows the own q_r
    // block and lands in TMEM lanes nobody reads), then the partial
    // sc[128 x 64] = Q_c[:, dims_r] . C_KV[tile, dims_r]^T.
    constexpr uint32_t kIdescS = ptx::idesc_bf16_f32(kHeads, kT, 0, 0);   // K-major A and B
    const uint64_t d_qc = ptx::smem_desc(ptx::smem_u32(smem + kOffQc), 16, 1024, ptx::kSwizzle128B);
    const uint64_t d_qr = ptx::smem_desc(ptx::smem_u32(smem + kOffQr) - (uint32_t)(r * kQrBytes), 16, 1024,
                                         ptx::kSwizzle128B);
    const uint64_t d_c = ptx::smem_desc(ptx::smem_u32(smem + kOffC), 16, 1024, ptx::kSwizzle128B);
    const uint64_t d_kr = ptx::smem_desc(ptx::smem_u32(smem + kOffKr), 16, 1024, ptx::kSwizzle128B);
    int seg = -1;
    int64_t cur_b = -1;
    bool ok = true;
    int64_t sseq = seq0, stile = tile0;
    for (int64_t t = 0; t < n_tiles && ok; ++t, step(sseq, stile)) {
      const int64_t b = sseq;
      const bool last_in_seg = t + 1 == n_tiles || stile + 1 == p.tiles_per_seq;
      const int buf = (int)(t & 1);
      if (b != cur_b) {
        cur_b = b;
        ++seg;
        ok = bounded_wait(bb.q_full, seg & 1, abort_flag, p, 0x600, true, false);
        if (!ok) break;
      }
      if (t >= 2) ok = bounded_wait(&bb.s_empty[buf], (uint32_t)((t >> 1) - 1) & 1, abort_flag, p, 0x601, true, false);
      if (ok) ok = bounded_wait(&bb.kr_full[t % kNKr], (uint32_t)(t / kNKr) & 1, abort_flag, p, 0x602, true, false);
      if (ok) ok = bounded_wait(&bb.c_full[t % kNS], (uint32_t)(t / kNS) & 1, abort_flag, p, 0x603, true, false);
      if (!ok) break;
      ptx::tc_fence_after();
      const uint32_t d_s = tmem + 128u * buf;
      {
        const uint64_t b0 = d_kr + (uint64_t)(((t % kNKr) * kKrBytes) >> 4);
#pragma unroll
        for (int k = 0; k < 4; ++k)
          ptx::mma_bf16_ss(d_s + 64, d_qr + (uint64_t)((32 * k) >> 4), b0 + (uint64_t)((32 * k) >> 4), kIdescS,
                           k > 0);
        ptx::mma_commit(&bb.kr_empty[t % kNKr]);
      }
      {
        const uint64_t b0 = d_c + (uint64_t)(((t % kNS) * kStage) >> 4);
#pragma unroll
        for (int a = 0; a < kAtoms; ++a)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            ptx::mma_bf16_ss(d_s, d_qc + (uint64_t)((a * kQcAtom + 32 * k) >> 4),
                             b0 + (uint64_t)((a * kCAtom + 32 * k) >> 4), kIdescS, (a | k) != 0);
      }
      ptx::mma_commit(&bb.s_full[buf]);
      if (last_in_seg) ptx::mma_commit(bb.q_empty);
    }
    ptx::mma_commit(&bb.drain[0]);
    bounded_wait(&bb.drain[0], 0, abort_flag, p, 0x6F0, false, false);
  } else if (warp == 2 && lane == 0) {
    // ===================================================== O MMA issuer
    // Tile j once P is complete (own rows, the peer's rows) and the peer heads'
    // O rows are rescaled where asked:  O[128 x 256] += P[128 x 64] . C_KV[tile, dims_r]
    // (B read MN-major from the tile's stage), four K steps of 16 tokens.  A
    // sequence part starts the accumulator afresh.  Completion is signalled in
    // both CTAs (the peer copies its next P rows only after this O is done).
    constexpr uint32_t kIdescO = ptx::idesc_bf16_f32(kHeads, kDim, 0, 1);   // A K-major, B MN-major
    const uint64_t d_p = ptx::smem_desc(ptx::smem_u32(smem + kOffP), 16, 1024, ptx::kSwizzle128B);
    const uint64_t d_cb = ptx::smem_desc(ptx::smem_u32(smem + kOffC), kCAtom, 1024, ptx::kSwizzle128B);
    int64_t oseq = seq0, otile = tile0;
    for (int64_t j = 0; j < n_tiles; ++j, step(oseq, otile)) {
      if (!bounded_wait(bb.p_local, (uint32_t)j & 1, abort_flag, p, 0x700, true, false)) break;
      if (!bounded_wait(bb.p_remote, (uint32_t)j & 1, abort_flag, p, 0x701, true, true)) break;
      if (j + 1 < n_tiles) ptx::mbar_arrive_expect_tx(bb.p_remote, kPOwnBytes + kAlphaOwnBytes);
      if (!bounded_wait(bb.lanes_ready, (uint32_t)j & 1, abort_flag, p, 0x702, true, false)) break;
      ptx::tc_fence_after();
      const uint32_t acc0 = (j > 0 && otile > 0) ? 1u : 0u;
      const int cs = (int)(j % kNS);
      const uint64_t b0 = d_cb + (uint64_t)((cs * kStage) >> 4);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        ptx::mma_bf16_ss(tmem + kColO, d_p + (uint64_t)((32 * k) >> 4), b0 + (uint64_t)((2048 * k) >> 4), kIdescO,
                         k > 0 ? 1u : acc0);
      ptx::mma_commit(&bb.c_empty[cs]);
      ptx::mma_commit_multicast(&bb.o_done[r], (uint16_t)0x3);
    }
    ptx::mma_commit(&bb.drain[1]);
    bounded_wait(&bb.drain[1], 0, abort_flag, p, 0x7F0, false, false);
  } else if (warp >= 3) {
    // ===================================================== quarter warps
    const int q = warp & 3;                   // TMEM lane quarter this warp may access
    const int k = (warp - 3) >> 2;            // 0 or 1
    const int hl = 32 * q + lane;             // head within the cluster's 128 (TMEM lane)
    const uint32_t lanes = (uint32_t)(32 * q) << 16;
    const bool own = (q >> 1) == r;
    float* recv = reinterpret_cast<float*>(smem + kOffRecv);
    float* alpha_s = reinterpret_cast<float*>(smem + kOffAlpha);
    if (own) {
      // ------------------------------------------------- softmax (head hl, tokens 32 k .. 32 k + 31)
      const int ol = hl - kOwn * r;
      const int h = h0 + hl;
      float4* gst = reinterpret_cast<float4*>(smem + kOffGst);   // [2][64]
      int* gan = reinterpret_cast<int*>(smem + kOffGan);         // [2][64]
      float* mt_s = reinterpret_cast<float*>(smem + kOffMt);     // [2][64]
      float* zt_s = reinterpret_cast<float*>(smem + kOffZt);     // [2][64]
      uint8_t* pbuf = smem + kOffP;
      const bool armer = q == 2 * r && k == 0;                     // arms recv_full
      const bool copier = armer && lane == 0;                      // copies the own P rows to the peer
      const uint32_t peer_recv_free = ptx::mapa(ptx::smem_u32(bb.recv_free), peer);
      const uint32_t peer_p_remote = ptx::mapa(ptx::smem_u32(bb.p_remote), peer);
      const uint32_t peer_prow = ptx::mapa(ptx::smem_u32(pbuf + r * kPOwnBytes), peer);
      const uint32_t peer_alpha = ptx::mapa(ptx::smem_u32(alpha_s + kOwn * r), peer);
      bool copy_pending = false;
      float M = -INFINITY, Z = 0.f;
      int64_t cseq = seq0, ctile = tile0;
      for (int64_t i = 0; i < n_tiles; ++i, step(cseq, ctile)) {
        const int64_t b = cseq, tile = ctile;
        const bool last_in_seg = i + 1 == n_tiles || tile + 1 == p.tiles_per_seq;
        const int buf = (int)(i & 1);
        warp_wait(&bb.s_full[buf], (uint32_t)(i >> 1) & 1, abort_flag, p, 0x800, false);
        warp_wait(bb.recv_full, (uint32_t)i & 1, abort_flag, p, 0x801, true);
        ptx::tc_fence_after();
        // x: the partial sc, then sc, then (grouped) e_t or (window) s_t
        float x[kHalfT], sr[kHalfT];
        ptx::tmem_ld32(tmem + lanes + 128u * buf + 32u * k, x);
        ptx::tmem_ld32(tmem + lanes + 128u * buf + 64u + 32u * k, sr);
        ptx::tmem_wait_ld();
        {  // the peer's partial scores over its dims (16-byte chunks swizzled by head)
          const float* rrow = recv + ol * kT;
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int phys = (8 * k + j) ^ (ol & 15);
            const float4 v = *reinterpret_cast<const float4*>(rrow + 4 * phys);
            x[4 * j] += v.x; x[4 * j + 1] += v.y; x[4 * j + 2] += v.z; x[4 * j + 3] += v.w;
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          ptx::mbar_arrive(&bb.s_empty[buf]);
          if (armer && i + 1 < n_tiles) ptx::mbar_arrive_expect_tx(bb.recv_full, kRecvBytes);
          ptx::mbar_arrive_remote(peer_recv_free);   // the peer may send the next tile's partials
        }

        const int64_t tok0 = tile * kT + kHalfT * k;
        // Some of this thread's groups are condensed: the window starts at a
        // multiple of g, which may fall inside the thread's 32 tokens, so the
        // choice is made per group (grp[]).  For g = 64 a group is the whole
        // tile, and the choice is the same in all four warps.
        const bool half_groups = (g > 1) && (tok0 < win0);
        bool grp[NGT];
#pragma unroll
        for (int gi = 0; gi < NGT; ++gi) grp[gi] = half_groups && (tok0 + gi * GW < win0);
        int32_t* anc = p.anchor + ((int64_t)b * p.H + h) * p.nG;

        // ---- step 2: condense; a grouped token's weight is e_t * f[group]
        float f[NGT], Sg[NGT], deng[NGT], ent = -INFINITY;
        if constexpr (g == 1) {
#pragma unroll
          for (int t = 0; t < kHalfT; ++t)
            if (tok0 + t < win0) anc[tok0 + t] = (int32_t)(p.pos0 + tok0 + t);
        }
        if (half_groups) {
          float mg[NGT], numg[NGT], srag[NGT];
          int ag[NGT];
#pragma unroll
          for (int gi = 0; gi < NGT; ++gi) {
            if (!grp[gi]) {   // a window group inside this half: its tokens stand for themselves
#pragma unroll
              for (int t = 0; t < GW; ++t) {
                x[gi * GW + t] += sr[gi * GW + t];
                if (tok0 + gi * GW + t < p.L) ent = fmaxf(ent, x[gi * GW + t]);
              }
              mg[gi] = 0.f; ag[gi] = 0; deng[gi] = 1.f; numg[gi] = 0.f; srag[gi] = 0.f; f[gi] = 1.f;
              continue;
            }
            float m = x[gi * GW] + sr[gi * GW], sra = sr[gi * GW];
            int a = 0;
#pragma unroll
            for (int t = 1; t < GW; ++t) {
              const float st = x[gi * GW + t] + sr[gi * GW + t];
              if (st > m) { m = st; a = t; sra = sr[gi * GW + t]; }   // strict: lowest index wins ties
            }
            float den = 0.f, num = 0.f;
#pragma unroll
            for (int t = 0; t < GW; ++t) {
              const float sc = x[gi * GW + t];
              const float et = ex2((sc + sr[gi * GW + t] - m) * kLog2e);
              den += et;
              num = fmaf(et, sc, num);
              x[gi * GW + t] = et;
            }
            mg[gi] = m; ag[gi] = gi * GW + a; deng[gi] = den; numg[gi] = num; srag[gi] = sra;
            f[gi] = 1.f;
          }
          if constexpr (g > kHalfT) {
            // a 64-token group: merge the two halves (half 0 first, so both
            // threads form the same bits; a tie keeps half 0's anchor)
            gst[k * kOwn + ol] = make_float4(mg[0], deng[0], numg[0], srag[0]);
            gan[k * kOwn + ol] = kHalfT * k + ag[0];
            ptx::named_bar_sync(kSoftmaxBar, kSoftmaxThreads);
            const float4 v0 = gst[ol], v1 = gst[kOwn + ol];
            const int a0 = gan[ol], a1 = gan[kOwn + ol];
            const float mm = fmaxf(v0.x, v1.x);
            const float f0 = ex2((v0.x - mm) * kLog2e), f1 = ex2((v1.x - mm) * kLog2e);
            deng[0] = v0.y * f0 + v1.y * f1;
            numg[0] = v0.z * f0 + v1.z * f1;
            const bool take1 = v1.x > v0.x;
            srag[0] = take1 ? v1.w : v0.w;
            ag[0] = take1 ? a1 : a0;                   // tile-relative
            f[0] = k == 0 ? f0 : f1;                   // this half's e_t are relative to its own max
          } else {
#pragma unroll
            for (int gi = 0; gi < NGT; ++gi) ag[gi] += kHalfT * k;   // tile-relative
          }
#pragma unroll
          for (int gi = 0; gi < NGT; ++gi) {
            Sg[gi] = __fdividef(numg[gi], deng[gi]) + srag[gi];
            if (grp[gi]) ent = fmaxf(ent, Sg[gi]);
          }
          if (g <= kHalfT || k == 0) {
#pragma unroll
            for (int gi = 0; gi < NGT; ++gi) {
              const int64_t jg = (tile * kT + (g <= kHalfT ? kHalfT * k + gi * GW : 0)) / g;
              if (grp[gi]) anc[jg] = (int32_t)(p.pos0 + tile * kT + ag[gi]);
            }
          }
        } else {   // window tokens (and g = 1): the entry is the token itself
#pragma unroll
          for (int t = 0; t < kHalfT; ++t) {
            x[t] += sr[t] + (tok0 + t < p.bias_rows ? p.bias : 0.f);
            if (tok0 + t < p.L) ent = fmaxf(ent, x[t]);
          }
        }

        // ---- step 3: reference max (see the file comment); the checkpoint
        // barrier ORs "abort, or take this slow path" over the softmax threads.
        const bool first = i == 0 || tile == 0;
        if (copier && copy_pending) {   // the P rows of the previous tile were read by the copy
          ptx::bulk_wait_group_read0();
          copy_pending = false;
        }
        float alpha = 1.f;
        const bool need = first || (ent - M) * kLog2e > kRescaleLog2;
        if (ptx::named_bar_or(kSoftmaxBar, kSoftmaxThreads, need || *abort_flag != 0)) {
          if (ptx::named_bar_or(kSoftmaxBar, kSoftmaxThreads, *abort_flag != 0)) break;
          mt_s[k * kOwn + ol] = ent;
          ptx::named_bar_sync(kSoftmaxBar, kSoftmaxThreads);
          const float mt = fmaxf(mt_s[ol], mt_s[kOwn + ol]);
          if (first) {
            M = mt;
          } else if ((mt - M) * kLog2e > kRescaleLog2) {
            alpha = ex2((M - mt) * kLog2e);
            M = mt;
          }
          if (__any_sync(0xffffffffu, alpha != 1.f)) {
            Z *= alpha;
            // this head's O row (this half of the dims) must be complete before scaling
            warp_wait(&bb.o_done[r], (uint32_t)(i - 1) & 1, abort_flag, p, 0x803, false);
            ptx::tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < 4; ++cc) {
              float o[32];
              const uint32_t ta = tmem + lanes + kColO + 128u * k + 32u * cc;
              ptx::tmem_ld32(ta, o);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int t = 0; t < 32; ++t) o[t] *= alpha;
              ptx::tmem_st32(ta, o);
            }
            ptx::tmem_wait_st();
          }
          ptx::named_bar_sync(kSoftmaxBar, kSoftmaxThreads);   // mt_s may be rewritten next tile
        }
        if (k == 0) alpha_s[hl] = alpha;     // travels to the peer with P

        // ---- per-token weights, this thread's 64 bytes of its head's P row
        uint32_t pk[kHalfT / 2];
        if (half_groups) {
#pragma unroll
          for (int gi = 0; gi < NGT; ++gi)
            if (grp[gi]) f[gi] *= __fdividef(ex2((Sg[gi] - M) * kLog2e), deng[gi]);
        }
#pragma unroll
        for (int t2 = 0; t2 < kHalfT / 2; ++t2) {
          float pv[2];
#pragma unroll
          for (int e2 = 0; e2 < 2; ++e2) {
            const int t = 2 * t2 + e2;
            const bool valid = tok0 + t < p.L;
            float v;
            if (grp[t / GW]) v = x[t] * f[t / GW];
            else v = valid ? ex2(fmaf(x[t], kLog2e, -M * kLog2e)) : 0.f;
            pv[e2] = v;
          }
          pk[t2] = pack_bf16x2(pv[0], pv[1]);
          const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(&pk[t2]);
          Z += __low2float(v) + __high2float(v);   // Z from the rounded P
        }
        // the own P rows are free once O of the previous tile is done here
        if (i >= 1) warp_wait(&bb.o_done[r], (uint32_t)(i - 1) & 1, abort_flag, p, 0x804, false);
        {
          uint8_t* prow = pbuf + hl * 128;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int phys = (4 * k + j) ^ (hl & 7);
            *reinterpret_cast<uint4*>(prow + 16 * phys) =
                make_uint4(pk[4 * j], pk[4 * j + 1], pk[4 * j + 2], pk[4 * j + 3]);
          }
        }
        ptx::fence_proxy_async_smem();
        ptx::named_bar_sync(kSoftmaxBar, kSoftmaxThreads);   // every own row and factor written
        if (copier) {
          // the peer's P rows are free once O of the previous tile is done there
          bool okp = true;
          if (i >= 1) okp = bounded_wait(&bb.o_done[peer], (uint32_t)(i - 1) & 1, abort_flag, p, 0x805, true, true);
          if (okp) {
            ptx::bulk_copy_to_peer(peer_prow, pbuf + r * kPOwnBytes, kPOwnBytes, peer_p_remote);
            ptx::bulk_copy_to_peer(peer_alpha, alpha_s + kOwn * r, kAlphaOwnBytes, peer_p_remote);
            ptx::bulk_commit_group();
            copy_pending = true;
          }
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bb.p_local);

        if (last_in_seg) {
          // the partial of the range's part of sequence b: this head's O row over
          // this CTA's dims (half k of them), and (owner) its (M, Z)
          const int64_t slot = b + c;
          warp_wait(&bb.o_done[r], (uint32_t)i & 1, abort_flag, p, 0x806, false);
          ptx::tc_fence_after();
          float* dst = p.part_o + (slot * p.H + h) * (int64_t)kDC + kDim * r + 128 * k;
#pragma unroll 1
          for (int cc = 0; cc < 4; ++cc) {
            float o[32];
            ptx::tmem_ld32(tmem + lanes + kColO + 128u * k + 32u * cc, o);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int t = 0; t < 32; t += 4)
              *reinterpret_cast<float4*>(dst + 32 * cc + t) = make_float4(o[t], o[t + 1], o[t + 2], o[t + 3]);
          }
          ptx::tc_fence_before();
          zt_s[k * kOwn + ol] = Z;
          ptx::named_bar_sync(kSoftmaxBar, kSoftmaxThreads);
          if (k == 0) {
            p.part_mz[(slot * p.H + h) * 2 + 0] = M;
            p.part_mz[(slot * p.H + h) * 2 + 1] = zt_s[ol] + zt_s[kOwn + ol];
          }
          ptx::named_bar_sync(kSoftmaxBar, kSoftmaxThreads);
          M = -INFINITY;
          Z = 0.f;
        }
      }
      if (copier) {
        if (copy_pending) ptx::bulk_wait_group_read0();
        // the peer's last O-completion signal has landed here before this CTA exits
        if (n_tiles > 0) bounded_wait(&bb.o_done[peer], (uint32_t)(n_tiles - 1) & 1, abort_flag, p, 0x8F0, true, true);
      }
    } else if (k == 0) {
      // ------------------------------------------------- shipper: the peer heads' partial scores
      const int olp = hl - kOwn * peer;           // the head's row in the peer's receive buffer
      const uint32_t peer_row = ptx::mapa(ptx::smem_u32(recv + olp * kT), peer);
      const uint32_t peer_recv_full = ptx::mapa(ptx::smem_u32(bb.recv_full), peer);
      int64_t i = 0;
      for (; i < n_tiles; ++i) {
        const int buf = (int)(i & 1);
        if (!warp_wait(&bb.s_full[buf], (uint32_t)(i >> 1) & 1, abort_flag, p, 0x900, false)) break;
        ptx::tc_fence_after();
        float v0[32], v1[32];
        ptx::tmem_ld32(tmem + lanes + 128u * buf, v0);
        ptx::tmem_ld32(tmem + lanes + 128u * buf + 32u, v1);
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bb.s_empty[buf]);
        if (i >= 1 && !warp_wait(bb.recv_free, (uint32_t)(i - 1) & 1, abort_flag, p, 0x901, true)) break;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          ptx::st_async_v4(peer_row + 16u * (uint32_t)(j ^ (olp & 15)), __float_as_uint(v0[4 * j]),
                           __float_as_uint(v0[4 * j + 1]), __float_as_uint(v0[4 * j + 2]),
                           __float_as_uint(v0[4 * j + 3]), peer_recv_full);
#pragma unroll
        for (int j = 0; j < 8; ++j)
          ptx::st_async_v4(peer_row + 16u * (uint32_t)((8 + j) ^ (olp & 15)), __float_as_uint(v1[4 * j]),
                           __float_as_uint(v1[4 * j + 1]), __float_as_uint(v1[4 * j + 2]),
                           __float_as_uint(v1[4 * j + 3]), peer_recv_full);
      }
      // the peer's release of the last tile has landed here before this CTA exits
      if (i == n_tiles && n_tiles > 0 && lane == 0)
        bounded_wait(bb.recv_free, (uint32_t)(n_tiles - 1) & 1, abort_flag, p, 0x9F0, true, true);
    } else {
      // ------------------------------------------------- checker: the peer heads' rescale factors
      int64_t cseq = seq0, ctile = tile0;
      for (int64_t i = 0; i < n_tiles; ++i, step(cseq, ctile)) {
        const int64_t b = cseq, tile = ctile;
        const bool last_in_seg = i + 1 == n_tiles || tile + 1 == p.tiles_per_seq;
        if (!warp_wait(bb.p_remote, (uint32_t)i & 1, abort_flag, p, 0xA00, true)) break;
        const float a = alpha_s[hl];
        if (__any_sync(0xffffffffu, a != 1.f) && i >= 1) {
          if (!warp_wait(&bb.o_done[r], (uint32_t)(i - 1) & 1, abort_flag, p, 0xA01, false)) break;
          ptx::tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < 8; ++cc) {
            float o[32];
            const uint32_t ta = tmem + lanes + kColO + 32u * cc;
            ptx::tmem_ld32(ta, o);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int t = 0; t < 32; ++t) o[t] *= a;
            ptx::tmem_st32(ta, o);
          }
          ptx::tmem_wait_st();
        }
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(bb.lanes_ready);
        if (last_in_seg) {
          const int64_t slot = b + c;
          if (!warp_wait(&bb.o_done[r], (uint32_t)i & 1, abort_flag, p, 0xA02, false)) break;
          ptx::tc_fence_after();
          float* dst = p.part_o + (slot * p.H + h0 + hl) * (int64_t)kDC + kDim * r;
#pragma unroll 1
          for (int cc = 0; cc < 8; ++cc) {
            float o[32];
            ptx::tmem_ld32(tmem + lanes + kColO + 32u * cc, o);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int t = 0; t < 32; t += 4)
              *reinterpret_cast<float4*>(dst + 32 * cc + t) = make_float4(o[t], o[t + 1], o[t + 2], o[t + 3]);
          }
          ptx::tc_fence_before();
        }
      }
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
