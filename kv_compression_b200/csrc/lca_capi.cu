// lca_capi.cu -- the C ABI declared in include/lca.h: plans, argument checks,
// kernel choice, TMA descriptor encoding and launches.  No exception crosses
// the ABI and nothing here aborts; every CUDA error becomes a status code.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>

#include "lca.h"
#include "checks.cuh"
#include "combine_kernel.cuh"
#include "condense_kernel.cuh"
#include "gqa_kernel.cuh"
#include "paged_kernel.cuh"
#include "pair_kernel.cuh"
#include "simt_kernel.cuh"
#include "tc_kernel.cuh"

struct lca_plan {
  int B, H, d_c, d_r;
  lca_dtype dt;
  int64_t max_L;
  int device;
  int num_sms;
  bool tc_shape;           // the tcgen05 kernel can take this shape
  bool pair_shape;         // the two-CTA tcgen05 kernel can take this shape (H % 128 == 0)
  int pair_clusters;       // two-CTA clusters resident at once on this device
  int64_t ws_slots;
  float* part_o;           // [ws_slots][H][d_c]
  float* part_mz;          // [ws_slots][H][2]
  int* meta;               // paged-decode metadata, lca::meta_ints(B, ws_slots) ints
  int* err;                // [2]: flags, where
  int last_site;           // where of the last error lca_get_device_error reported
  // options
  bool force_simt;
  int kernel_pref;         // 0: automatic, else the lca_plan_kernel code to use
  int num_ctas;
  uint64_t timeout_ns;
  int debug_skip_load;
  cudaEvent_t timing_event;  // recorded between the main and the combine kernel when set
  int64_t bias_rows;         // set only for the duration of an lca_decode_stored call
  float bias;
  // lca_decode_host staging (allocated on first use)
  void* st_qc;
  void* st_qr;
  void* st_c;
  void* st_k;
  float* st_out;
  int32_t* st_anc;
};

// Fixed device scratch of lca_decode_noalloc (zero at module load): split
// partials [slots][H][d_c] and [slots][H][2] floats, then the device error
// word (2 ints).  Only lca_decode_noalloc uses it, through the address that
// cudaGetSymbolAddress gives for the current device.  A call may use at most
// min(kNoAllocOFloats / (H d_c), kNoAllocMzFloats / (2 H)) slots, so that both
// regions hold every slot it writes.
constexpr size_t kNoAllocOFloats = (size_t)4 << 20;              // 16 MiB of partial outputs
constexpr size_t kNoAllocMzFloats = kNoAllocOFloats / 256;       // 64 KiB of (M, Z) pairs
constexpr size_t kNoAllocErrOffset = kNoAllocOFloats + kNoAllocMzFloats;
static __device__ __align__(256) float lca_noalloc_scratch[kNoAllocErrOffset + 64];

namespace {

constexpr int64_t kDefaultTimeoutNs = 2000000000LL;  // 2 s bound on any in-kernel wait

size_t elem_size(lca_dtype dt) { return dt == LCA_F32 ? 4 : 2; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool is_pow2(int x) { return x > 0 && (x & (x - 1)) == 0; }

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Splits of the CUDA-core kernel: about two CTAs per SM overall.
int simt_target_splits(const lca_plan* p) {
  const int64_t bh = (int64_t)p->B * p->H;
  return (int)std::max<int64_t>(1, ceil_div(2LL * p->num_sms, bh));
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// bf16 matrix [rows][inner], box [box_rows][64], 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t gdim[2] = {inner, rows};
  const cuuint64_t gstride[1] = {inner * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim, gstride, box,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

enum Kernel { kNone = 0, kSimt = 1, kTc = 2, kPair = 3 };

// Where the rows of one call sit in the context: a whole context (win0 = n_G g,
// pos0 = 0) or one slice of a context-sharded decode; and whether the combine
// writes the normalised output or a partial (M, Z, unnormalised O).
struct Slice {
  int64_t win0;
  int64_t pos0;
  float* out_mz;
};

// A paged, variable-length batch (lca_decode_paged): the pools' pages, the
// block table and the device lengths; cap bounds every length.
struct Paged {
  const int32_t* block_table;
  int64_t max_pages;        // pages a sequence may have (bounds every length)
  int64_t table_stride;     // entries from one sequence's table row to the next (0: one shared row)
  int page_size;
  int64_t num_pages;
  const int32_t* seq_lens;  // null: a prefill chunk, query b's length pos0 + b + 1
  int64_t pos0;
  int64_t cap;
  int64_t anchor_stride;
  int g, w;     // the segmentation every sequence's n_G(b) follows
};

// The metadata of a paged call (lengths checked, tiles of kT tokens, G ranges)
// into the plan's metadata buffer; stream-ordered before the decode kernel.
lca_status launch_meta(const lca_plan* p, const Paged& pg, int kT, int64_t G, cudaStream_t stream) {
  lca::MetaParams mp = {};
  mp.seq_lens = pg.seq_lens;
  mp.pos0 = pg.pos0;
  mp.B = p->B;
  mp.cap = pg.cap;
  mp.g = pg.g;
  mp.w = pg.w;
  mp.anchor_stride = pg.anchor_stride;
  mp.kT = kT;
  mp.G = G;
  mp.meta = p->meta;
  mp.err = p->err;
  lca::lca_paged_meta_kernel<<<1, lca::kMetaThreads, 0, stream>>>(mp);
  return cudaGetLastError() == cudaSuccess ? LCA_OK : LCA_ERR_CUDA;
}

bool tc_group_ok(int64_t nG, int g, int gmax) { return nG == 0 || (is_pow2(g) && g <= gmax); }

// The kernel for (n_G, g): the two-CTA tcgen05 kernel where H is a multiple of
// 128 and g <= 64, else the 16-head tcgen05 kernel (H a multiple of 16,
// g <= 128), else the CUDA-core kernel.  LCA_OPT_FORCE_SIMT / LCA_OPT_KERNEL
// narrow the choice; a forced kernel that cannot take the shape gives kNone.
Kernel choose(const lca_plan* p, int64_t nG, int g) {
  const bool pair_ok = p->pair_shape && tc_group_ok(nG, g, lca::pair::kT);
  const bool tc_ok = p->tc_shape && tc_group_ok(nG, g, lca::tc::kT);
  const bool simt_ok = nG == 0 || g <= lca::kSimtTileMax;
  int pref = p->force_simt ? kSimt : p->kernel_pref;
  if (pref == kPair) return pair_ok ? kPair : kNone;
  if (pref == kTc) return tc_ok ? kTc : kNone;
  if (pref == kSimt) return simt_ok ? kSimt : kNone;
  if (pair_ok) return kPair;
  if (tc_ok) return kTc;
  if (simt_ok) return kSimt;
  return kNone;
}

lca_status launch_combine(const lca_plan* p, const lca::CombineParams& cp_in, cudaStream_t stream,
                          bool pdl) {
  lca::CombineParams cp = cp_in;
  if (cp.mode != 2) {          // the plan's workspace; a merge reads the caller's n_split parts
    cp.n_slots = p->ws_slots;
    cp.err = p->err;
  } else {
    cp.n_slots = (int64_t)cp.n_split * p->B;
    cp.err = p->err;
  }
  cp.vec = (p->d_c % lca::kCombineVec == 0) && (reinterpret_cast<uintptr_t>(cp.part_o) % 16 == 0) &&
           (reinterpret_cast<uintptr_t>(cp.out) % 16 == 0) ? 1 : 0;
  constexpr int kDimsPerBlock = lca::kCombineThreads * lca::kCombineVec;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p->H, (unsigned)p->B, (unsigned)((p->d_c + kDimsPerBlock - 1) / kDimsPerBlock));
  cfg.blockDim = dim3(lca::kCombineThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (cudaLaunchKernelEx(&cfg, lca::lca_combine_kernel, cp) != cudaSuccess) return LCA_ERR_CUDA;
  return LCA_OK;
}

lca_status run_simt(lca_plan* p, const void* q_c, const void* q_r, const void* c_kv,
                    const void* k_r, int64_t L, int g, int64_t nG, float* out, int32_t* anchor,
                    cudaStream_t stream, const Slice& sl, const Paged* pg = nullptr) {
  const int ge = nG > 0 ? g : 1;
  const int tile = ge * std::max(1, 256 / ge);
  // a paged batch: every sequence is cut into the same number of splits of
  // its own length (in the kernel); lengths are known only on the device
  int64_t split_len = ceil_div(L, simt_target_splits(p));
  split_len = ceil_div(split_len, ge) * ge;
  const int64_t n_split = pg ? simt_target_splits(p) : ceil_div(L, split_len);
  if ((int64_t)p->B * n_split > p->ws_slots) return LCA_ERR_UNSUPPORTED;
  if (pg) {
    const lca_status st = launch_meta(p, *pg, 0, 0, stream);
    if (st != LCA_OK) return st;
  }
  lca::SimtParams sp = {};
  sp.q_c = q_c; sp.q_r = q_r; sp.c_kv = c_kv; sp.k_r = k_r;
  sp.B = p->B; sp.H = p->H; sp.d_c = p->d_c; sp.d_r = p->d_r;
  sp.L = L; sp.g = ge; sp.nG = nG; sp.split_len = split_len; sp.tile = tile;
  sp.n_split = (int)n_split; sp.anchor = anchor; sp.part_o = p->part_o; sp.part_mz = p->part_mz;
  sp.bias_rows = p->bias_rows; sp.bias = p->bias; sp.win0 = sl.win0; sp.pos0 = sl.pos0;
  sp.ws_slots = p->ws_slots; sp.err = p->err;
  sp.anchor_stride = pg ? pg->anchor_stride : nG;
  if (pg) {
    sp.meta = p->meta; sp.block_table = pg->block_table; sp.table_stride = pg->table_stride;
    sp.page_size = pg->page_size; sp.num_pages = pg->num_pages;
  }
  const size_t smem = (size_t)(p->d_c + p->d_r + 4 * lca::kSimtTileMax + lca::kSimtWarps) * 4 +
                      (size_t)lca::kSimtTileMax * sizeof(int64_t);
  dim3 grid((unsigned)n_split, (unsigned)p->H, (unsigned)p->B);
  if (p->dt == LCA_F32)
    lca::lca_simt_kernel<float><<<grid, lca::kSimtThreads, smem, stream>>>(sp);
  else
    lca::lca_simt_kernel<__nv_bfloat16><<<grid, lca::kSimtThreads, smem, stream>>>(sp);
  if (cudaGetLastError() != cudaSuccess) return LCA_ERR_CUDA;
  if (p->timing_event && cudaEventRecord(p->timing_event, stream) != cudaSuccess) return LCA_ERR_CUDA;
  lca::CombineParams cp = {};
  cp.part_o = p->part_o; cp.part_mz = p->part_mz; cp.out = out;
  cp.B = p->B; cp.H = p->H; cp.d_c = p->d_c; cp.mode = 0; cp.n_split = (int)n_split;
  cp.wait_prior = 0; cp.out_mz = sl.out_mz;
  return launch_combine(p, cp, stream, false);
}

constexpr int kMaxDevices = 64;

// One bit per device: the kernel's shared-memory limit is set there.  Setting
// it twice is harmless, so two threads racing on a first call only repeat it.
bool device_flag_set(std::atomic<uint64_t>& flags, int device) {
  return device >= 0 && device < kMaxDevices && ((flags.load(std::memory_order_acquire) >> device) & 1u);
}
void device_flag_mark(std::atomic<uint64_t>& flags, int device) {
  if (device >= 0 && device < kMaxDevices)
    flags.fetch_or(uint64_t(1) << device, std::memory_order_acq_rel);
}

template <int LOG2G, bool kPaged>
cudaError_t launch_tc(const lca::tc::TcParams& tp, unsigned grid, cudaStream_t stream, int device) {
  static std::atomic<uint64_t> configured{0};
  if (!device_flag_set(configured, device)) {
    cudaError_t e = cudaFuncSetAttribute(lca::tc::lca_tc_kernel<LOG2G, kPaged>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         lca::tc::kSmemAlloc);
    if (e != cudaSuccess) return e;
    device_flag_mark(configured, device);
  }
  // Programmatic stream serialization: the kernel's prologue (barrier init,
  // TMEM allocation) may overlap the previous kernel's tail; the kernel waits on
  // griddepcontrol before its first global access.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid, 1, 1);
  cfg.blockDim = dim3(lca::tc::kThreads, 1, 1);
  cfg.dynamicSmemBytes = lca::tc::kSmemAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, lca::tc::lca_tc_kernel<LOG2G, kPaged>, tp);
}

template <bool kPaged>
cudaError_t launch_tc_gp(int g, const lca::tc::TcParams& tp, unsigned grid, cudaStream_t stream,
                         int device) {
  switch (g) {
    case 1: return launch_tc<0, kPaged>(tp, grid, stream, device);
    case 2: return launch_tc<1, kPaged>(tp, grid, stream, device);
    case 4: return launch_tc<2, kPaged>(tp, grid, stream, device);
    case 8: return launch_tc<3, kPaged>(tp, grid, stream, device);
    case 16: return launch_tc<4, kPaged>(tp, grid, stream, device);
    case 32: return launch_tc<5, kPaged>(tp, grid, stream, device);
    case 64: return launch_tc<6, kPaged>(tp, grid, stream, device);
    case 128: return launch_tc<7, kPaged>(tp, grid, stream, device);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_tc_g(int g, const lca::tc::TcParams& tp, unsigned grid, cudaStream_t stream,
                        int device) {
  return tp.meta ? launch_tc_gp<true>(g, tp, grid, stream, device) : launch_tc_gp<false>(g, tp, grid, stream, device);
}

lca_status run_tc(lca_plan* p, const void* q_c, const void* q_r, const void* c_kv,
                  const void* k_r, int64_t L, int g, int64_t nG, float* out, int32_t* anchor,
                  cudaStream_t stream, const Slice& sl, const Paged* pg = nullptr) {
  lca::tc::TcParams tp;
  std::memset(&tp, 0, sizeof(tp));
  const uint64_t rows = pg ? (uint64_t)pg->num_pages * (uint64_t)pg->page_size : (uint64_t)p->B * (uint64_t)L;
  if (rows > (uint64_t)INT32_MAX) return LCA_ERR_UNSUPPORTED;   // TMA row coordinates are int32
  const uint64_t qrows = (uint64_t)p->B * (uint64_t)p->H;
  // a paged tile's two 64-token halves may sit in two pages: 64-row boxes
  const uint32_t box = pg ? lca::tc::kT / 2 : lca::tc::kT;
  if (!make_map(&tp.tm_c, c_kv, 512, rows, box) || !make_map(&tp.tm_k, k_r, 64, rows, box) ||
      !make_map(&tp.tm_qc, q_c, 512, qrows, 16) || !make_map(&tp.tm_qr, q_r, 64, qrows, 16))
    return LCA_ERR_CUDA;
  const int n_hb = p->H / lca::tc::kHC;
  const int64_t tps = pg ? 0 : ceil_div(L, lca::tc::kT);
  const int64_t U = (int64_t)p->B * tps;
  const int ctas = p->num_ctas > 0 ? p->num_ctas : p->num_sms;
  // a paged batch's tile count is known on the device only: it uses
  // min(G, U) of these ranges (the metadata)
  int64_t G = std::max<int64_t>(1, pg ? ctas / n_hb : std::min<int64_t>(ctas / n_hb, U));
  G = std::min<int64_t>(G, p->ws_slots - p->B + 1);    // range c writes slot b + c
  if (G < 1) return LCA_ERR_UNSUPPORTED;
  if (pg) {
    const lca_status st = launch_meta(p, *pg, lca::tc::kT, G, stream);
    if (st != LCA_OK) return st;
  }
  tp.B = p->B; tp.H = p->H; tp.L = L; tp.nG = nG;
  tp.tiles_per_seq = pg ? 1 : tps; tp.U = U; tp.G = G; tp.n_hb = n_hb;
  tp.anchor = anchor; tp.part_o = p->part_o; tp.part_mz = p->part_mz; tp.err = p->err;
  tp.timeout_ns = p->timeout_ns; tp.debug_skip_load = p->debug_skip_load;
  tp.bias_rows = p->bias_rows; tp.bias = p->bias; tp.win0 = sl.win0; tp.pos0 = sl.pos0;
  tp.ws_slots = p->ws_slots;
  tp.anchor_stride = pg ? pg->anchor_stride : nG;
  if (pg) {
    tp.meta = p->meta; tp.block_table = pg->block_table; tp.table_stride = pg->table_stride;
    tp.page_size = pg->page_size; tp.num_pages = pg->num_pages;
  }
  const unsigned grid = (unsigned)(G * n_hb);
  if (launch_tc_g(nG > 0 ? g : 1, tp, grid, stream, p->device) != cudaSuccess) return LCA_ERR_CUDA;
  if (p->timing_event && cudaEventRecord(p->timing_event, stream) != cudaSuccess) return LCA_ERR_CUDA;
  lca::CombineParams cp = {};
  cp.part_o = p->part_o; cp.part_mz = p->part_mz; cp.out = out;
  cp.B = p->B; cp.H = p->H; cp.d_c = p->d_c; cp.mode = pg ? 3 : 1; cp.tiles_per_seq = tps; cp.G = G;
  cp.wait_prior = 1; cp.out_mz = sl.out_mz; cp.meta = p->meta;
  return launch_combine(p, cp, stream, true);
}

template <int LOG2G, bool kPaged>
cudaError_t launch_pair(const lca::pair::PairParams& pp, unsigned clusters, cudaStream_t stream, int device) {
  static std::atomic<uint64_t> configured{0};
  if (!device_flag_set(configured, device)) {
    cudaError_t e = cudaFuncSetAttribute(lca::pair::lca_pair_kernel<LOG2G, kPaged>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         lca::pair::kSmemAlloc);
    if (e != cudaSuccess) return e;
    device_flag_mark(configured, device);
  }
  // Clusters of two CTAs (one per SM), launched as a programmatic dependent
  // like the 16-head kernel.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters, 1, 1);
  cfg.blockDim = dim3(lca::pair::kThreads, 1, 1);
  cfg.dynamicSmemBytes = lca::pair::kSmemAlloc;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, lca::pair::lca_pair_kernel<LOG2G, kPaged>, pp);
}

template <bool kPaged>
cudaError_t launch_pair_gp(int g, const lca::pair::PairParams& pp, unsigned clusters, cudaStream_t stream,
                           int device) {
  switch (g) {
    case 1: return launch_pair<0, kPaged>(pp, clusters, stream, device);
    case 2: return launch_pair<1, kPaged>(pp, clusters, stream, device);
    case 4: return launch_pair<2, kPaged>(pp, clusters, stream, device);
    case 8: return launch_pair<3, kPaged>(pp, clusters, stream, device);
    case 16: return launch_pair<4, kPaged>(pp, clusters, stream, device);
    case 32: return launch_pair<5, kPaged>(pp, clusters, stream, device);
    case 64: return launch_pair<6, kPaged>(pp, clusters, stream, device);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_pair_g(int g, const lca::pair::PairParams& pp, unsigned clusters, cudaStream_t stream,
                          int device) {
  return pp.meta ? launch_pair_gp<true>(g, pp, clusters, stream, device)
                 : launch_pair_gp<false>(g, pp, clusters, stream, device);
}

// Two-CTA clusters of the pair kernel that fit on the device at once (one
// wave); 0 when the query fails.
int pair_cluster_capacity(int num_sms) {
  cudaError_t e = cudaFuncSetAttribute(lca::pair::lca_pair_kernel<4, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       lca::pair::kSmemAlloc);
  if (e != cudaSuccess) { cudaGetLastError(); return num_sms / 2; }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(num_sms & ~1), 1, 1);
  cfg.blockDim = dim3(lca::pair::kThreads, 1, 1);
  cfg.dynamicSmemBytes = lca::pair::kSmemAlloc;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, lca::pair::lca_pair_kernel<4, false>, &cfg) != cudaSuccess || n < 1) {
    cudaGetLastError();
    return num_sms / 2;
  }
  return n;
}

lca_status run_pair(lca_plan* p, const void* q_c, const void* q_r, const void* c_kv,
                    const void* k_r, int64_t L, int g, int64_t nG, float* out, int32_t* anchor,
                    cudaStream_t stream, const Slice& sl, const Paged* pg = nullptr) {
  lca::pair::PairParams pp;
  std::memset(&pp, 0, sizeof(pp));
  const uint64_t rows = pg ? (uint64_t)pg->num_pages * (uint64_t)pg->page_size : (uint64_t)p->B * (uint64_t)L;
  if (rows > (uint64_t)INT32_MAX) return LCA_ERR_UNSUPPORTED;   // TMA row coordinates are int32
  const uint64_t qrows = (uint64_t)p->B * (uint64_t)p->H;
  if (!make_map(&pp.tm_c, c_kv, 512, rows, lca::pair::kT) ||
      !make_map(&pp.tm_k, k_r, 64, rows, lca::pair::kT) ||
      !make_map(&pp.tm_qc, q_c, 512, qrows, lca::pair::kHeads))
    return LCA_ERR_CUDA;
  pp.q_r = static_cast<const __nv_bfloat16*>(q_r);
  const int n_hb = p->H / lca::pair::kHeads;
  const int64_t tps = pg ? 0 : ceil_div(L, lca::pair::kT);
  const int64_t U = (int64_t)p->B * tps;
  const int64_t clusters = p->num_ctas > 0 ? std::max(1, p->num_ctas / 2) : p->pair_clusters;
  // a paged batch's tile count is known on the device only: it uses
  // min(G, U) of these ranges (the metadata)
  int64_t G = std::max<int64_t>(1, pg ? clusters / n_hb : std::min<int64_t>(clusters / n_hb, U));
  G = std::min<int64_t>(G, p->ws_slots - p->B + 1);    // range c writes slot b + c
  if (G < 1) return LCA_ERR_UNSUPPORTED;
  if (pg) {
    const lca_status st = launch_meta(p, *pg, lca::pair::kT, G, stream);
    if (st != LCA_OK) return st;
  }
  pp.B = p->B; pp.H = p->H; pp.L = L; pp.nG = nG;
  pp.tiles_per_seq = pg ? 1 : tps; pp.U = U; pp.G = G; pp.n_hb = n_hb;
  pp.anchor = anchor; pp.part_o = p->part_o; pp.part_mz = p->part_mz; pp.err = p->err;
  pp.timeout_ns = p->timeout_ns; pp.debug_skip_load = p->debug_skip_load;
  pp.bias_rows = p->bias_rows; pp.bias = p->bias; pp.win0 = sl.win0; pp.pos0 = sl.pos0;
  pp.ws_slots = p->ws_slots;
  pp.anchor_stride = pg ? pg->anchor_stride : nG;
  if (pg) {
    pp.meta = p->meta; pp.block_table = pg->block_table; pp.table_stride = pg->table_stride;
    pp.page_size = pg->page_size; pp.num_pages = pg->num_pages;
  }
  if (launch_pair_g(nG > 0 ? g : 1, pp, (unsigned)(G * n_hb), stream, p->device) != cudaSuccess)
    return LCA_ERR_CUDA;
  if (p->timing_event && cudaEventRecord(p->timing_event, stream) != cudaSuccess) return LCA_ERR_CUDA;
  lca::CombineParams cp = {};
  cp.part_o = p->part_o; cp.part_mz = p->part_mz; cp.out = out;
  cp.B = p->B; cp.H = p->H; cp.d_c = p->d_c; cp.mode = pg ? 3 : 1; cp.tiles_per_seq = tps; cp.G = G;
  cp.wait_prior = 1; cp.out_mz = sl.out_mz; cp.meta = p->meta;
  return launch_combine(p, cp, stream, true);
}

lca_status check_common(const lca_plan* p, const void* q_c, const void* q_r, const void* c_kv,
                        const void* k_r, int64_t L, const float* out) {
  if (!p || !q_c || !q_r || !c_kv || !k_r || !out) return LCA_ERR_INVALID_ARG;
  if (L < 1 || L > p->max_L) return LCA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return LCA_ERR_CUDA;
  if (dev != p->device) return LCA_ERR_PLAN_MISMATCH;
  return LCA_OK;
}

}  // namespace
extern "C" int64_t lca_num_groups(int64_t L, int g, int w);
namespace {

// One decode over `L` cache rows of a context: n_G groups in those rows (the
// anchor stride), window from row sl.win0, anchors offset by sl.pos0.
lca_status decode_rows(lca_plan* p, const void* q_c, const void* q_r, const void* c_kv,
                       const void* k_r, int64_t L, int g, int64_t nG, float* out, int32_t* anchor,
                       void* stream, const Slice& sl) {
  lca_status st = check_common(p, q_c, q_r, c_kv, k_r, L, out);
  if (st != LCA_OK) return st;
  if (nG > 0 && !anchor) return LCA_ERR_INVALID_ARG;
  const Kernel k = choose(p, nG, g);
  if (k == kNone) return LCA_ERR_UNSUPPORTED;
  if (!aligned16(q_c) || !aligned16(q_r) || !aligned16(c_kv) || !aligned16(k_r) ||
      !aligned16(out) || (nG > 0 && !aligned16(anchor)) || (sl.out_mz && !aligned16(sl.out_mz)))
    return LCA_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (k == kPair) return run_pair(p, q_c, q_r, c_kv, k_r, L, g, nG, out, anchor, s, sl);
  if (k == kTc) return run_tc(p, q_c, q_r, c_kv, k_r, L, g, nG, out, anchor, s, sl);
  return run_simt(p, q_c, q_r, c_kv, k_r, L, g, nG, out, anchor, s, sl);
}

lca_status decode_impl(lca_plan* p, const void* q_c, const void* q_r, const void* c_kv,
                       const void* k_r, int64_t L, int g, int w, float* out, int32_t* anchor,
                       void* stream, bool dense) {
  int64_t nG = 0;
  if (!dense) {
    if (g < 1 || w < 0) return LCA_ERR_INVALID_ARG;
    nG = lca_num_groups(L, g, w);
  }
  const Slice whole = {nG * (dense ? 1 : g), 0, nullptr};
  return decode_rows(p, q_c, q_r, c_kv, k_r, L, dense ? 1 : g, nG, out, anchor, stream, whole);
}

lca_status launch_condense(const lca_plan* p, const lca::CondenseParams& cp, cudaStream_t stream) {
  if (cp.n <= 0) return LCA_OK;
  const int64_t per_seq = std::max<int64_t>(1, std::min<int64_t>(ceil_div(cp.n, lca::kCondWarps),
                                                                 ceil_div(4LL * p->num_sms, p->B)));
  dim3 grid((unsigned)per_seq, (unsigned)p->B, 1);
  const size_t smem = (size_t)(p->d_c + p->d_r) * sizeof(float);
  const bool fast = p->dt == LCA_BF16 && p->d_c == lca::kCondFastDc && p->d_r == lca::kCondFastDr &&
                    aligned16(cp.c_kv) && aligned16(cp.c_dst) && aligned16(cp.k_r) && aligned16(cp.k_dst);
  if (fast)
    lca::lca_condense_fast_kernel<<<grid, lca::kCondThreads, 0, stream>>>(cp);
  else if (p->dt == LCA_F32)
    lca::lca_condense_kernel<float><<<grid, lca::kCondThreads, smem, stream>>>(cp);
  else
    lca::lca_condense_kernel<__nv_bfloat16><<<grid, lca::kCondThreads, smem, stream>>>(cp);
  return cudaGetLastError() == cudaSuccess ? LCA_OK : LCA_ERR_CUDA;
}

lca_status launch_copy_rows(const lca::CopyRowsParams& rp, cudaStream_t stream) {
  if (rp.n <= 0) return LCA_OK;
  const int64_t total = rp.B * rp.n * (rp.row_bytes / 16);
  const unsigned blocks = (unsigned)std::max<int64_t>(1, std::min<int64_t>(ceil_div(total, 256), 4096));
  lca::lca_copy_rows_kernel<<<blocks, 256, 0, stream>>>(rp);
  return cudaGetLastError() == cudaSuccess ? LCA_OK : LCA_ERR_CUDA;
}

void free_staging(lca_plan* p) {
  cudaFree(p->st_qc); cudaFree(p->st_qr); cudaFree(p->st_c); cudaFree(p->st_k);
  cudaFree(p->st_out); cudaFree(p->st_anc);
  p->st_qc = p->st_qr = p->st_c = p->st_k = nullptr;
  p->st_out = nullptr;
  p->st_anc = nullptr;
}


// lca_decode_paged and lca_prefill_paged: argument checks, kernel choice, and
// the three launches (metadata, decode, combine).
lca_status paged_impl(lca_plan* p, const void* q_c, const void* q_r, const void* c_pool, const void* k_pool,
                      int64_t num_pages, int page_size, const int32_t* block_table, int64_t max_pages,
                      int64_t table_stride, const int32_t* seq_lens, int64_t pos0, int g, int w, float* out,
                      int32_t* anchor, int64_t anchor_stride, void* stream) {
  if (!p || !q_c || !q_r || !c_pool || !k_pool || !block_table || !out) return LCA_ERR_INVALID_ARG;
  if (num_pages < 1 || page_size < 64 || (page_size % 64) != 0 || max_pages < 1 || g < 1 || w < 0 ||
      anchor_stride < 0)
    return LCA_ERR_INVALID_ARG;
  if ((uint64_t)num_pages * (uint64_t)page_size > (uint64_t)INT32_MAX) return LCA_ERR_UNSUPPORTED;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return LCA_ERR_CUDA;
  if (dev != p->device) return LCA_ERR_PLAN_MISMATCH;
  Paged pg;
  pg.block_table = block_table; pg.max_pages = max_pages; pg.table_stride = table_stride;
  pg.page_size = page_size; pg.num_pages = num_pages; pg.seq_lens = seq_lens; pg.pos0 = pos0;
  pg.g = g; pg.w = w;
  pg.cap = std::min<int64_t>(p->max_L, max_pages * (int64_t)page_size);
  const int64_t nG_cap = lca_num_groups(pg.cap, g, w);
  if (nG_cap > 0 && !anchor) return LCA_ERR_INVALID_ARG;
  pg.anchor_stride = anchor ? anchor_stride : INT64_MAX;
  const Kernel k = choose(p, nG_cap, g);
  if (k == kNone) return LCA_ERR_UNSUPPORTED;
  if (!aligned16(q_c) || !aligned16(q_r) || !aligned16(c_pool) || !aligned16(k_pool) || !aligned16(out) ||
      (anchor && !aligned16(anchor)) || (reinterpret_cast<uintptr_t>(block_table) & 3u) != 0 ||
      (reinterpret_cast<uintptr_t>(seq_lens) & 3u) != 0)
    return LCA_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const Slice whole = {0, 0, nullptr};
  const int ge = nG_cap > 0 ? g : 1;
  if (k == kPair) return run_pair(p, q_c, q_r, c_pool, k_pool, 0, ge, nG_cap, out, anchor, s, whole, &pg);
  if (k == kTc) return run_tc(p, q_c, q_r, c_pool, k_pool, 0, ge, nG_cap, out, anchor, s, whole, &pg);
  return run_simt(p, q_c, q_r, c_pool, k_pool, 0, ge, nG_cap, out, anchor, s, whole, &pg);
}

// GQA LCA decode on the CUDA-core kernel: one CTA per (split, KV head,
// sequence) over the r = H / H_kv query heads of the KV head.
template <typename T, int SLOTS>
cudaError_t gqa_setup(int device, size_t smem, int* per_sm) {
  static std::atomic<uint64_t> configured{0};
  constexpr size_t kMaxSmem = 227 * 1024;
  if (!device_flag_set(configured, device)) {
    const cudaError_t e = cudaFuncSetAttribute(lca::lca_gqa_kernel<T, SLOTS>,
                                               cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kMaxSmem);
    if (e != cudaSuccess) return e;
    device_flag_mark(configured, device);
  }
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(per_sm, lca::lca_gqa_kernel<T, SLOTS>, lca::kGqaThreads,
                                                    smem) != cudaSuccess || *per_sm < 1) {
    cudaGetLastError();
    *per_sm = 1;
  }
  return cudaSuccess;
}

template <typename T, int SLOTS>
void gqa_launch(const lca::GqaParams& gp, dim3 grid, size_t smem, cudaStream_t stream) {
  lca::lca_gqa_kernel<T, SLOTS><<<grid, lca::kGqaThreads, smem, stream>>>(gp);
}

// GQA LCA decode on the CUDA-core kernel: one CTA per (split, KV head,
// sequence) over the r = H / H_kv query heads of the KV head; the kernel is
// instantiated for ceil(r / 4) head slots.
lca_status run_gqa(lca_plan* p, const void* q, const void* k, const void* v, int64_t L, int H_kv, int g,
                   int64_t nG, float* out, int32_t* anchor, cudaStream_t stream) {
  const int r = p->H / H_kv;
  const int slots = (r + 3) / 4;
  const int ge = nG > 0 ? g : 1;
  const bool f32 = p->dt == LCA_F32;
  const size_t smem = f32 ? lca::gqa_smem_bytes<float>(r, p->d_r, p->d_c)
                          : lca::gqa_smem_bytes<__nv_bfloat16>(r, p->d_r, p->d_c);
  if (smem > 227 * 1024) return LCA_ERR_UNSUPPORTED;
  // Splits: as many CTAs as are resident at once (one wave, so no tail wave
  // runs half empty), at least one per (sequence, KV head).
  int per_sm = 1;
  cudaError_t e = cudaErrorInvalidValue;
  switch (slots * 2 + (f32 ? 0 : 1)) {
    case 2: e = gqa_setup<float, 1>(p->device, smem, &per_sm); break;
    case 3: e = gqa_setup<__nv_bfloat16, 1>(p->device, smem, &per_sm); break;
    case 4: e = gqa_setup<float, 2>(p->device, smem, &per_sm); break;
    case 5: e = gqa_setup<__nv_bfloat16, 2>(p->device, smem, &per_sm); break;
    case 6: e = gqa_setup<float, 3>(p->device, smem, &per_sm); break;
    case 7: e = gqa_setup<__nv_bfloat16, 3>(p->device, smem, &per_sm); break;
    case 8: e = gqa_setup<float, 4>(p->device, smem, &per_sm); break;
    case 9: e = gqa_setup<__nv_bfloat16, 4>(p->device, smem, &per_sm); break;
  }
  if (e != cudaSuccess) return LCA_ERR_CUDA;
  const int64_t units = (int64_t)p->B * H_kv;
  int64_t n_split = std::max<int64_t>(1, ((int64_t)per_sm * p->num_sms) / units);
  n_split = std::min<int64_t>(n_split, p->ws_slots / p->B);
  n_split = std::min<int64_t>(n_split, ceil_div(L, lca::kGqaTile));
  if (n_split < 1) return LCA_ERR_UNSUPPORTED;
  const int64_t split_len = ceil_div(ceil_div(L, n_split), lca::kGqaTile) * lca::kGqaTile;
  n_split = ceil_div(L, split_len);
  lca::GqaParams gp = {};
  gp.q = q; gp.k = k; gp.v = v;
  gp.B = p->B; gp.H = p->H; gp.H_kv = H_kv; gp.r = r; gp.d_k = p->d_r; gp.d_v = p->d_c;
  gp.L = L; gp.g = ge; gp.nG = nG; gp.win0 = nG * ge; gp.split_len = split_len;
  gp.n_split = (int)n_split; gp.anchor = anchor; gp.part_o = p->part_o; gp.part_mz = p->part_mz;
  gp.ws_slots = p->ws_slots; gp.err = p->err;
  dim3 grid((unsigned)n_split, (unsigned)H_kv, (unsigned)p->B);
  switch (slots * 2 + (f32 ? 0 : 1)) {
    case 2: gqa_launch<float, 1>(gp, grid, smem, stream); break;
    case 3: gqa_launch<__nv_bfloat16, 1>(gp, grid, smem, stream); break;
    case 4: gqa_launch<float, 2>(gp, grid, smem, stream); break;
    case 5: gqa_launch<__nv_bfloat16, 2>(gp, grid, smem, stream); break;
    case 6: gqa_launch<float, 3>(gp, grid, smem, stream); break;
    case 7: gqa_launch<__nv_bfloat16, 3>(gp, grid, smem, stream); break;
    case 8: gqa_launch<float, 4>(gp, grid, smem, stream); break;
    case 9: gqa_launch<__nv_bfloat16, 4>(gp, grid, smem, stream); break;
  }
  if (cudaGetLastError() != cudaSuccess) return LCA_ERR_CUDA;
  if (p->timing_event && cudaEventRecord(p->timing_event, stream) != cudaSuccess) return LCA_ERR_CUDA;
  lca::CombineParams cp = {};
  cp.part_o = p->part_o; cp.part_mz = p->part_mz; cp.out = out;
  cp.B = p->B; cp.H = p->H; cp.d_c = p->d_c; cp.mode = 0; cp.n_split = (int)n_split;
  return launch_combine(p, cp, stream, false);
}
}  // namespace

extern "C" {

int64_t lca_num_groups(int64_t L, int g, int w) {
  if (g < 1 || w < 0 || L < 1) return -1;
  return L > (int64_t)w ? (L - (int64_t)w) / g : 0;
}

const char* lca_status_string(lca_status s) {
  switch (s) {
    case LCA_OK: return "ok";
    case LCA_ERR_INVALID_ARG: return "invalid argument";
    case LCA_ERR_UNSUPPORTED: return "unsupported shape, dtype or group size";
    case LCA_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
    case LCA_ERR_CUDA: return "CUDA error";
    case LCA_ERR_DEVICE_TIMEOUT: return "a bounded in-kernel wait ran out";
    case LCA_ERR_PLAN_MISMATCH: return "plan made for another shape or device";
    case LCA_ERR_NO_MEMORY: return "out of memory";
    case LCA_ERR_DEVICE_CHECK: return "a kernel index failed its range check (debug build)";
    case LCA_ERR_DEVICE_INPUT: return "a sequence length or block-table entry on the device was out of range";
  }
  return "unknown status";
}

lca_status lca_plan_create(int B, int H, int d_c, int d_r, lca_dtype dt, int64_t max_L,
                           lca_plan** out_plan) {
  if (!out_plan || B < 1 || H < 1 || d_c < 1 || d_r < 1 || max_L < 1) return LCA_ERR_INVALID_ARG;
  if (dt != LCA_F32 && dt != LCA_BF16) return LCA_ERR_INVALID_ARG;
  if (d_c > lca::kSimtMaxDc || d_r > 256 || H > 4096 || (d_c % 8) != 0 || (d_r % 8) != 0)
    return LCA_ERR_UNSUPPORTED;
  lca_plan* p = new (std::nothrow) lca_plan;
  if (!p) return LCA_ERR_NO_MEMORY;
  std::memset(p, 0, sizeof(*p));
  p->B = B; p->H = H; p->d_c = d_c; p->d_r = d_r; p->dt = dt; p->max_L = max_L;
  p->timeout_ns = kDefaultTimeoutNs;
  if (cudaGetDevice(&p->device) != cudaSuccess ||
      cudaDeviceGetAttribute(&p->num_sms, cudaDevAttrMultiProcessorCount, p->device) !=
          cudaSuccess) {
    delete p;
    return LCA_ERR_CUDA;
  }
  p->tc_shape = dt == LCA_BF16 && d_c == lca::tc::kDC && d_r == lca::tc::kDR &&
                (H % lca::tc::kHC) == 0;
  p->pair_shape = p->tc_shape && (H % lca::pair::kHeads) == 0;
  p->pair_clusters = p->pair_shape ? pair_cluster_capacity(p->num_sms) : 0;
  const int64_t simt_slots = (int64_t)B * simt_target_splits(p);
  const int64_t tc_slots = p->tc_shape ? (int64_t)B + p->num_sms : 0;
  p->ws_slots = std::max(simt_slots, tc_slots);
  // the GQA kernel's splits (about four CTAs per SM over B x H_kv), where the
  // partials of that many slots take at most 64 MiB
  const int64_t gqa_slots = (int64_t)B * ceil_div(4LL * p->num_sms, B);
  if ((size_t)gqa_slots * H * d_c * sizeof(float) <= ((size_t)64 << 20))
    p->ws_slots = std::max(p->ws_slots, gqa_slots);
  const size_t o_bytes = (size_t)p->ws_slots * H * d_c * sizeof(float);
  const size_t mz_bytes = (size_t)p->ws_slots * H * 2 * sizeof(float);
  const size_t meta_bytes = (size_t)lca::meta_ints(B, p->ws_slots) * sizeof(int);
  if (cudaMalloc(&p->part_o, o_bytes) != cudaSuccess ||
      cudaMalloc(&p->part_mz, mz_bytes) != cudaSuccess ||
      cudaMalloc(&p->meta, meta_bytes) != cudaSuccess ||
      cudaMalloc(&p->err, 2 * sizeof(int)) != cudaSuccess ||
      cudaMemset(p->err, 0, 2 * sizeof(int)) != cudaSuccess) {
    cudaFree(p->part_o); cudaFree(p->part_mz); cudaFree(p->meta); cudaFree(p->err);
    cudaGetLastError();
    delete p;
    return LCA_ERR_NO_MEMORY;
  }
  *out_plan = p;
  return LCA_OK;
}

lca_status lca_plan_destroy(lca_plan* p) {
  if (!p) return LCA_OK;
  cudaFree(p->part_o); cudaFree(p->part_mz); cudaFree(p->meta); cudaFree(p->err);
  free_staging(p);
  delete p;
  return LCA_OK;
}

lca_status lca_plan_set(lca_plan* p, lca_option opt, int64_t v) {
  if (!p) return LCA_ERR_INVALID_ARG;
  switch (opt) {
    case LCA_OPT_FORCE_SIMT: p->force_simt = v != 0; return LCA_OK;
    case LCA_OPT_NUM_CTAS:
      if (v < 0 || v > p->num_sms) return LCA_ERR_INVALID_ARG;  // one resident wave only
      p->num_ctas = (int)v;
      return LCA_OK;
    case LCA_OPT_WAIT_TIMEOUT_NS:
      if (v < 1000 || v > 60LL * 1000000000LL) return LCA_ERR_INVALID_ARG;
      p->timeout_ns = (uint64_t)v;
      return LCA_OK;
    case LCA_OPT_DEBUG_SKIP_LOAD: p->debug_skip_load = v != 0; return LCA_OK;
    case LCA_OPT_KERNEL:
      if (v < 0 || v > kPair) return LCA_ERR_INVALID_ARG;
      p->kernel_pref = (int)v;
      return LCA_OK;
  }
  return LCA_ERR_INVALID_ARG;
}

lca_status lca_plan_set_timing_event(lca_plan* p, void* event) {
  if (!p) return LCA_ERR_INVALID_ARG;
  p->timing_event = static_cast<cudaEvent_t>(event);
  return LCA_OK;
}

int lca_plan_kernel(lca_plan* p, int64_t L, int g, int w) {
  if (!p || L < 1 || g < 1 || w < 0) return 0;
  return (int)choose(p, lca_num_groups(L, g, w), g);
}

lca_status lca_decode(lca_plan* p, const void* q_c, const void* q_r, const void* c_kv,
                      const void* k_r, int64_t L, int g, int w, float* out, int32_t* anchor,
                      void* stream) {
  return decode_impl(p, q_c, q_r, c_kv, k_r, L, g, w, out, anchor, stream, false);
}

lca_status mla_decode(lca_plan* p, const void* q_c, const void* q_r, const void* c_kv,
                      const void* k_r, int64_t L, float* out, void* stream) {
  return decode_impl(p, q_c, q_r, c_kv, k_r, L, 1, 0, out, nullptr, stream, true);
}

lca_status lca_decode_host(lca_plan* p, const void* h_q_c, const void* h_q_r, const void* h_c_kv,
                           const void* h_k_r, int64_t L, int g, int w, float* h_out,
                           int32_t* h_anchor, void* stream) {
  if (!p || !h_q_c || !h_q_r || !h_c_kv || !h_k_r || !h_out) return LCA_ERR_INVALID_ARG;
  if (L < 1 || L > p->max_L || g < 1 || w < 0) return LCA_ERR_INVALID_ARG;
  const int64_t nG = lca_num_groups(L, g, w);
  if (nG > 0 && !h_anchor) return LCA_ERR_INVALID_ARG;
  const size_t es = elem_size(p->dt);
  const size_t qc_b = (size_t)p->B * p->H * p->d_c * es, qr_b = (size_t)p->B * p->H * p->d_r * es;
  const size_t c_b = (size_t)p->B * L * p->d_c * es, k_b = (size_t)p->B * L * p->d_r * es;
  const size_t o_b = (size_t)p->B * p->H * p->d_c * sizeof(float);
  const size_t a_b = (size_t)p->B * p->H * (size_t)std::max<int64_t>(nG, 0) * sizeof(int32_t);
  if (!p->st_qc) {
    const size_t cmax = (size_t)p->B * p->max_L * p->d_c * es;
    const size_t kmax = (size_t)p->B * p->max_L * p->d_r * es;
    const size_t amax = (size_t)p->B * p->H * (size_t)p->max_L * sizeof(int32_t);
    if (cudaMalloc(&p->st_qc, qc_b) != cudaSuccess || cudaMalloc(&p->st_qr, qr_b) != cudaSuccess ||
        cudaMalloc(&p->st_c, cmax) != cudaSuccess || cudaMalloc(&p->st_k, kmax) != cudaSuccess ||
        cudaMalloc(&p->st_out, o_b) != cudaSuccess || cudaMalloc(&p->st_anc, amax) != cudaSuccess) {
      free_staging(p);
      cudaGetLastError();
      return LCA_ERR_NO_MEMORY;
    }
  }
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(p->st_qc, h_q_c, qc_b, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(p->st_qr, h_q_r, qr_b, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(p->st_c, h_c_kv, c_b, cudaMemcpyHostToDevice, s) != cudaSuccess ||
      cudaMemcpyAsync(p->st_k, h_k_r, k_b, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return LCA_ERR_CUDA;
  lca_status st = lca_decode(p, p->st_qc, p->st_qr, p->st_c, p->st_k, L, g, w, p->st_out,
                             nG > 0 ? p->st_anc : nullptr, stream);
  if (st != LCA_OK) return st;
  if (cudaMemcpyAsync(h_out, p->st_out, o_b, cudaMemcpyDeviceToHost, s) != cudaSuccess) return LCA_ERR_CUDA;
  if (nG > 0 && cudaMemcpyAsync(h_anchor, p->st_anc, a_b, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return LCA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return LCA_ERR_CUDA;
  return LCA_OK;
}

int64_t lca_stored_rows(int64_t L, int g, int w) {
  const int64_t nG = lca_num_groups(L, g, w);
  if (nG < 0) return -1;
  return nG + (L - nG * g);
}

lca_status lca_condense(lca_plan* p, const void* q_c, const void* q_r, const void* c_kv,
                        const void* k_r, int64_t L, int g, int64_t j0, int64_t n, void* c_dst,
                        void* k_dst, int64_t dst_rows, int64_t dst_row0, int32_t* anchor,
                        void* stream) {
  if (!p || !q_c || !q_r || !c_kv || !k_r || !c_dst || !k_dst || (n > 0 && !anchor))
    return LCA_ERR_INVALID_ARG;
  if (L < 1 || L > p->max_L || g < 1 || j0 < 0 || n < 0 || (j0 + n) * (int64_t)g > L)
    return LCA_ERR_INVALID_ARG;
  if (dst_row0 < 0 || dst_rows < dst_row0 + n) return LCA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return LCA_ERR_CUDA;
  if (dev != p->device) return LCA_ERR_PLAN_MISMATCH;
  lca::CondenseParams cp = {};
  cp.q_c = q_c; cp.q_r = q_r; cp.c_kv = c_kv; cp.k_r = k_r;
  cp.B = p->B; cp.H = p->H; cp.d_c = p->d_c; cp.d_r = p->d_r; cp.L = L; cp.g = g;
  cp.j0 = j0; cp.n = n; cp.c_dst = c_dst; cp.k_dst = k_dst; cp.dst_rows = dst_rows;
  cp.dst_row0 = dst_row0; cp.anchor = anchor; cp.err = p->err;
  return launch_condense(p, cp, static_cast<cudaStream_t>(stream));
}

lca_status lca_build_stored(lca_plan* p, const void* q_c, const void* q_r, const void* c_kv,
                            const void* k_r, int64_t L, int g, int w, void* c_store, void* k_store,
                            int32_t* anchor, void* stream) {
  if (!p || !q_c || !q_r || !c_kv || !k_r || !c_store || !k_store) return LCA_ERR_INVALID_ARG;
  if (L < 1 || L > p->max_L || g < 1 || w < 0) return LCA_ERR_INVALID_ARG;
  const int64_t nG = lca_num_groups(L, g, w);
  if (nG > 0 && !anchor) return LCA_ERR_INVALID_ARG;
  const int64_t rows = lca_stored_rows(L, g, w);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (!aligned16(c_kv) || !aligned16(k_r) || !aligned16(c_store) || !aligned16(k_store))
    return LCA_ERR_ALIGNMENT;
  lca_status st = lca_condense(p, q_c, q_r, c_kv, k_r, L, g, 0, nG, c_store, k_store, rows, 0,
                               anchor, stream);
  if (st != LCA_OK) return st;
  const size_t es = elem_size(p->dt);
  lca::CopyRowsParams rc = {};
  rc.src = static_cast<const uint8_t*>(c_kv); rc.dst = static_cast<uint8_t*>(c_store);
  rc.src_rows = L; rc.src_row0 = nG * g; rc.dst_rows = rows; rc.dst_row0 = nG; rc.n = L - nG * g;
  rc.row_bytes = (int64_t)p->d_c * (int64_t)es; rc.B = p->B;
  if ((st = launch_copy_rows(rc, s)) != LCA_OK) return st;
  lca::CopyRowsParams rk = rc;
  rk.src = static_cast<const uint8_t*>(k_r); rk.dst = static_cast<uint8_t*>(k_store);
  rk.row_bytes = (int64_t)p->d_r * (int64_t)es;
  return launch_copy_rows(rk, s);
}

lca_status lca_decode_stored(lca_plan* p, const void* q_c, const void* q_r, const void* c_store,
                             const void* k_store, int64_t n_rows, int64_t n_cond, float bias,
                             float* out, void* stream) {
  if (!p || n_cond < 0 || n_cond > n_rows) return LCA_ERR_INVALID_ARG;
  p->bias_rows = n_cond;
  p->bias = bias;
  const lca_status st =
      decode_impl(p, q_c, q_r, c_store, k_store, n_rows, 1, 0, out, nullptr, stream, true);
  p->bias_rows = 0;
  p->bias = 0.f;
  return st;
}

int64_t lca_slice_groups(int64_t L, int g, int w, int64_t pos0, int64_t n_tok) {
  const int64_t nG = lca_num_groups(L, g, w);
  if (nG < 0 || pos0 < 0 || n_tok < 0 || pos0 + n_tok > L) return -1;
  const int64_t win0 = nG * g, end = pos0 + n_tok;
  if ((pos0 < win0 && pos0 % g != 0) || (end < win0 && end % g != 0)) return -1;   // a cut group
  const int64_t lo = pos0 < win0 ? pos0 / g : nG;
  const int64_t hi = end < win0 ? end / g : nG;
  return hi > lo ? hi - lo : 0;
}

lca_status lca_decode_partial(lca_plan* p, const void* q_c, const void* q_r, const void* c_slice,
                              const void* k_slice, int64_t n_tok, int64_t pos0, int64_t L, int g,
                              int w, float* part_mz, float* part_o, int32_t* anchor, void* stream) {
  if (!p || !part_mz || !part_o || g < 1 || w < 0 || L < 1) return LCA_ERR_INVALID_ARG;
  const int64_t ng = lca_slice_groups(L, g, w, pos0, n_tok);
  if (ng < 0) return LCA_ERR_INVALID_ARG;
  const int64_t win0 = lca_num_groups(L, g, w) * g;
  // The slice's own rows hold its groups: rows past n_tok (a partial last tile
  // reads the next sequence's rows) must never count as grouped.
  const Slice sl = {std::min<int64_t>(n_tok, std::max<int64_t>(0, win0 - pos0)), pos0, part_mz};
  if (n_tok == 0) {   // an empty slice: M = -inf, Z = 0, O = 0 (the combine over no parts)
    if (!aligned16(part_mz) || !aligned16(part_o)) return LCA_ERR_ALIGNMENT;
    lca::CombineParams cp = {};
    cp.part_o = p->part_o; cp.part_mz = p->part_mz; cp.out = part_o; cp.out_mz = part_mz;
    cp.B = p->B; cp.H = p->H; cp.d_c = p->d_c; cp.mode = 0; cp.n_split = 0;
    return launch_combine(p, cp, static_cast<cudaStream_t>(stream), false);
  }
  // a slice that starts inside the window holds no group: any g will do
  const int gg = ng > 0 ? g : 1;
  return decode_rows(p, q_c, q_r, c_slice, k_slice, n_tok, gg, ng, part_o, ng > 0 ? anchor : nullptr,
                     stream, sl);
}

lca_status lca_merge_partials(lca_plan* p, int n_parts, const float* part_mz, const float* part_o,
                              float* out, void* stream) {
  if (!p || n_parts < 1 || !part_mz || !part_o || !out) return LCA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return LCA_ERR_CUDA;
  if (dev != p->device) return LCA_ERR_PLAN_MISMATCH;
  lca::CombineParams cp = {};
  cp.part_o = part_o; cp.part_mz = part_mz; cp.out = out;
  cp.B = p->B; cp.H = p->H; cp.d_c = p->d_c; cp.mode = 2; cp.n_split = n_parts;
  return launch_combine(p, cp, static_cast<cudaStream_t>(stream), false);
}

lca_status lca_get_device_error(lca_plan* p, void* stream) {
  if (!p) return LCA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int host[2] = {0, 0};
  if (cudaStreamSynchronize(s) != cudaSuccess) return LCA_ERR_CUDA;
  if (cudaMemcpy(host, p->err, sizeof(host), cudaMemcpyDeviceToHost) != cudaSuccess)
    return LCA_ERR_CUDA;
  if (host[0] != 0 && cudaMemset(p->err, 0, sizeof(host)) != cudaSuccess) return LCA_ERR_CUDA;
  if (host[0] != 0) p->last_site = host[1];
  if (host[0] & lca::kErrCheck) return LCA_ERR_DEVICE_CHECK;
  if (host[0] & lca::kErrInput) return LCA_ERR_DEVICE_INPUT;
  return host[0] != 0 ? LCA_ERR_DEVICE_TIMEOUT : LCA_OK;
}

int lca_get_device_error_site(const lca_plan* p) { return p ? p->last_site : 0; }

lca_status lca_decode_gqa(lca_plan* p, const void* q, const void* k_cache, const void* v_cache, int64_t L,
                          int n_kv_heads, int g, int w, float* out, int32_t* anchor, void* stream) {
  if (!p || !q || !k_cache || !v_cache || !out) return LCA_ERR_INVALID_ARG;
  if (L < 1 || L > p->max_L || g < 1 || w < 0 || n_kv_heads < 1 || p->H % n_kv_heads != 0)
    return LCA_ERR_INVALID_ARG;
  if (p->H / n_kv_heads > lca::kGqaMaxR || p->d_c > lca::kGqaMaxD || p->d_r > lca::kGqaMaxD ||
      !is_pow2(p->d_c) || p->d_c < 32)
    return LCA_ERR_UNSUPPORTED;
  const int64_t nG = lca_num_groups(L, g, w);
  if (nG > 0 && !(is_pow2(g) && g <= lca::kGqaTile)) return LCA_ERR_UNSUPPORTED;
  if (nG > 0 && !anchor) return LCA_ERR_INVALID_ARG;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return LCA_ERR_CUDA;
  if (dev != p->device) return LCA_ERR_PLAN_MISMATCH;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
      (nG > 0 && !aligned16(anchor)))
    return LCA_ERR_ALIGNMENT;
  if ((uint64_t)p->B * (uint64_t)L * (uint64_t)n_kv_heads > (uint64_t)INT64_MAX / 1024) return LCA_ERR_UNSUPPORTED;
  return run_gqa(p, q, k_cache, v_cache, L, n_kv_heads, g, nG, out, nG > 0 ? anchor : nullptr,
                 static_cast<cudaStream_t>(stream));
}

lca_status lca_decode_paged(lca_plan* p, const void* q_c, const void* q_r, const void* c_pool,
                            const void* k_pool, int64_t num_pages, int page_size,
                            const int32_t* block_table, int64_t max_pages, const int32_t* seq_lens,
                            int g, int w, float* out, int32_t* anchor, int64_t anchor_stride,
                            void* stream) {
  if (!seq_lens) return LCA_ERR_INVALID_ARG;
  return paged_impl(p, q_c, q_r, c_pool, k_pool, num_pages, page_size, block_table, max_pages, max_pages,
                    seq_lens, 0, g, w, out, anchor, anchor_stride, stream);
}

lca_status lca_prefill_paged(lca_plan* p, const void* q_c, const void* q_r, const void* c_pool,
                             const void* k_pool, int64_t num_pages, int page_size,
                             const int32_t* block_table_row, int64_t max_pages, int64_t pos0, int g, int w,
                             float* out, int32_t* anchor, int64_t anchor_stride, void* stream) {
  if (!p || pos0 < 0 || pos0 + p->B > std::min<int64_t>(p->max_L, max_pages * (int64_t)page_size))
    return LCA_ERR_INVALID_ARG;
  return paged_impl(p, q_c, q_r, c_pool, k_pool, num_pages, page_size, block_table_row, max_pages, 0,
                    nullptr, pos0, g, w, out, anchor, anchor_stride, stream);
}

// For callers that may not allocate device memory when they decode -- a
// server whose memory is all reserved up front by its own pool (a cudaMalloc
// here would fail or fragment it) and that cannot keep a plan per shape --
// this entry point runs the same kernels as lca_decode with the fixed
// file-scope scratch above in place of a plan's workspace, and allocates
// nothing.  The first call on a device looks up the scratch's address there
// (cudaGetSymbolAddress), its SM count and how many two-CTA clusters fit
// (cudaOccupancyMaxActiveClusters), under a mutex, so concurrent first
// calls from several host threads are safe; later calls read the cached
// values without locking.
lca_status lca_decode_noalloc(int B, int H, int d_c, int d_r, lca_dtype dt, const void* q_c,
                              const void* q_r, const void* c_kv, const void* k_r, int64_t L, int g,
                              int w, float* out, int32_t* anchor, void* stream) {
  static std::atomic<float*> scratch[kMaxDevices];   // the scratch's address, per device
  static std::atomic<int> sms[kMaxDevices];
  static std::atomic<int> pair_clusters[kMaxDevices];
  static std::mutex first_call;
  if (B < 1 || H < 1 || d_c < 1 || d_r < 1 || L < 1 || g < 1 || w < 0) return LCA_ERR_INVALID_ARG;
  if (!q_c || !q_r || !c_kv || !k_r || !out) return LCA_ERR_INVALID_ARG;
  if (dt != LCA_F32 && dt != LCA_BF16) return LCA_ERR_INVALID_ARG;
  if (d_c > lca::kSimtMaxDc || d_r > 256 || H > 4096 || (d_c % 8) != 0 || (d_r % 8) != 0)
    return LCA_ERR_UNSUPPORTED;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return LCA_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return LCA_ERR_UNSUPPORTED;
  if (!scratch[dev].load(std::memory_order_acquire)) {
    std::lock_guard<std::mutex> lock(first_call);
    if (!scratch[dev].load(std::memory_order_acquire)) {
      void* ptr = nullptr;
      int n_sm = 0;
      if (cudaGetSymbolAddress(&ptr, lca_noalloc_scratch) != cudaSuccess) return LCA_ERR_CUDA;
      if (cudaDeviceGetAttribute(&n_sm, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return LCA_ERR_CUDA;
      sms[dev].store(n_sm, std::memory_order_relaxed);
      pair_clusters[dev].store(pair_cluster_capacity(n_sm), std::memory_order_relaxed);
      scratch[dev].store(static_cast<float*>(ptr), std::memory_order_release);
    }
  }
  float* base = scratch[dev].load(std::memory_order_acquire);
  // Split slots that fit BOTH regions of the scratch: partial outputs (H d_c
  // floats a slot) and (M, Z) pairs (2 H floats a slot).  Fewer than B slots
  // is a shape beyond the scratch's limit.
  const int64_t cap_o = (int64_t)(kNoAllocOFloats / ((size_t)H * (size_t)d_c));
  const int64_t cap_mz = (int64_t)(kNoAllocMzFloats / ((size_t)2 * (size_t)H));
  const int64_t cap = std::min(cap_o, cap_mz);
  if (cap < B) return LCA_ERR_UNSUPPORTED;
  lca_plan plan;
  std::memset(&plan, 0, sizeof(plan));
  plan.B = B; plan.H = H; plan.d_c = d_c; plan.d_r = d_r; plan.dt = dt; plan.max_L = L;
  plan.device = dev;
  plan.num_sms = sms[dev].load(std::memory_order_relaxed);
  plan.tc_shape = dt == LCA_BF16 && d_c == lca::tc::kDC && d_r == lca::tc::kDR &&
                  (H % lca::tc::kHC) == 0;
  plan.pair_shape = plan.tc_shape && (H % lca::pair::kHeads) == 0;
  plan.pair_clusters = pair_clusters[dev].load(std::memory_order_relaxed);
  // run_simt refuses a launch that needs more slots; the tensor-core paths cut
  // the context into at most cap - B + 1 tile ranges
  plan.ws_slots = cap;
  plan.part_o = base;
  plan.part_mz = base + kNoAllocOFloats;
  plan.err = reinterpret_cast<int*>(base + kNoAllocErrOffset);
  plan.timeout_ns = kDefaultTimeoutNs;
  // The kernels only OR into the error word, so it must start each call at zero.
  if (cudaMemsetAsync(plan.err, 0, 2 * sizeof(int), static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return LCA_ERR_CUDA;
  return decode_impl(&plan, q_c, q_r, c_kv, k_r, L, g, w, out, anchor, stream, false);
}

}  // extern "C"
