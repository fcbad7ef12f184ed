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
#include "combine_kernel.cuh"
#include "simt_kernel.cuh"
#include "tc_kernel.cuh"

struct lca_plan {
  int B, H, d_c, d_r;
  lca_dtype dt;
  int64_t max_L;
  int device;
  int num_sms;
  bool tc_shape;           // the tcgen05 kernel can take this shape
  int64_t ws_slots;
  float* part_o;           // [ws_slots][H][d_c]
  float* part_mz;          // [ws_slots][H][2]
  int* err;                // [2]: flags, where
  // options
  bool force_simt;
  int num_ctas;
  uint64_t timeout_ns;
  int debug_skip_load;
  cudaEvent_t timing_event;  // recorded between the main and the combine kernel when set
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

enum Kernel { kNone = 0, kSimt = 1, kTc = 2 };

Kernel choose(const lca_plan* p, int64_t nG, int g) {
  if (p->tc_shape && !p->force_simt && (nG == 0 || (is_pow2(g) && g <= 128))) return kTc;
  if (nG == 0 || g <= lca::kSimtTileMax) return kSimt;
  return kNone;
}

lca_status launch_combine(const lca_plan* p, const lca::CombineParams& cp, cudaStream_t stream,
                          bool pdl) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)p->H, (unsigned)p->B,
                     (unsigned)((p->d_c + lca::kCombineThreads - 1) / lca::kCombineThreads));
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
                    cudaStream_t stream) {
  const int ge = nG > 0 ? g : 1;
  const int tile = ge * std::max(1, 256 / ge);
  int64_t split_len = ceil_div(L, simt_target_splits(p));
  split_len = ceil_div(split_len, ge) * ge;
  const int64_t n_split = ceil_div(L, split_len);
  if ((int64_t)p->B * n_split > p->ws_slots) return LCA_ERR_UNSUPPORTED;
  lca::SimtParams sp;
  sp.q_c = q_c; sp.q_r = q_r; sp.c_kv = c_kv; sp.k_r = k_r;
  sp.B = p->B; sp.H = p->H; sp.d_c = p->d_c; sp.d_r = p->d_r;
  sp.L = L; sp.g = ge; sp.nG = nG; sp.split_len = split_len; sp.tile = tile;
  sp.n_split = (int)n_split; sp.anchor = anchor; sp.part_o = p->part_o; sp.part_mz = p->part_mz;
  const size_t smem = (size_t)(p->d_c + p->d_r + 4 * lca::kSimtTileMax + lca::kSimtWarps) * 4;
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
  cp.wait_prior = 0;
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

template <int LOG2G>
cudaError_t launch_tc(const lca::tc::TcParams& tp, unsigned grid, cudaStream_t stream, int device) {
  static std::atomic<uint64_t> configured{0};
  if (!device_flag_set(configured, device)) {
    cudaError_t e = cudaFuncSetAttribute(lca::tc::lca_tc_kernel<LOG2G>,
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
  return cudaLaunchKernelEx(&cfg, lca::tc::lca_tc_kernel<LOG2G>, tp);
}

cudaError_t launch_tc_g(int g, const lca::tc::TcParams& tp, unsigned grid, cudaStream_t stream,
                        int device) {
  switch (g) {
    case 1: return launch_tc<0>(tp, grid, stream, device);
    case 2: return launch_tc<1>(tp, grid, stream, device);
    case 4: return launch_tc<2>(tp, grid, stream, device);
    case 8: return launch_tc<3>(tp, grid, stream, device);
    case 16: return launch_tc<4>(tp, grid, stream, device);
    case 32: return launch_tc<5>(tp, grid, stream, device);
    case 64: return launch_tc<6>(tp, grid, stream, device);
    case 128: return launch_tc<7>(tp, grid, stream, device);
  }
  return cudaErrorInvalidValue;
}

lca_status run_tc(lca_plan* p, const void* q_c, const void* q_r, const void* c_kv,
                  const void* k_r, int64_t L, int g, int64_t nG, float* out, int32_t* anchor,
                  cudaStream_t stream) {
  lca::tc::TcParams tp;
  std::memset(&tp, 0, sizeof(tp));
  const uint64_t rows = (uint64_t)p->B * (uint64_t)L;
  if (rows > (uint64_t)INT32_MAX) return LCA_ERR_UNSUPPORTED;   // TMA row coordinates are int32
  const uint64_t qrows = (uint64_t)p->B * (uint64_t)p->H;
  if (!make_map(&tp.tm_c, c_kv, 512, rows, 128) || !make_map(&tp.tm_k, k_r, 64, rows, 128) ||
      !make_map(&tp.tm_qc, q_c, 512, qrows, 16) || !make_map(&tp.tm_qr, q_r, 64, qrows, 16))
    return LCA_ERR_CUDA;
  const int n_hb = p->H / lca::tc::kHC;
  const int64_t tps = ceil_div(L, lca::tc::kT);
  const int64_t U = (int64_t)p->B * tps;
  const int ctas = p->num_ctas > 0 ? p->num_ctas : p->num_sms;
  const int64_t G = std::max<int64_t>(1, std::min<int64_t>(ctas / n_hb, U));
  if ((int64_t)p->B + G - 1 > p->ws_slots) return LCA_ERR_UNSUPPORTED;
  tp.B = p->B; tp.H = p->H; tp.L = L; tp.nG = nG;
  tp.tiles_per_seq = tps; tp.U = U; tp.G = G; tp.n_hb = n_hb;
  tp.anchor = anchor; tp.part_o = p->part_o; tp.part_mz = p->part_mz; tp.err = p->err;
  tp.timeout_ns = p->timeout_ns; tp.debug_skip_load = p->debug_skip_load;
  const unsigned grid = (unsigned)(G * n_hb);
  if (launch_tc_g(nG > 0 ? g : 1, tp, grid, stream, p->device) != cudaSuccess) return LCA_ERR_CUDA;
  if (p->timing_event && cudaEventRecord(p->timing_event, stream) != cudaSuccess) return LCA_ERR_CUDA;
  lca::CombineParams cp = {};
  cp.part_o = p->part_o; cp.part_mz = p->part_mz; cp.out = out;
  cp.B = p->B; cp.H = p->H; cp.d_c = p->d_c; cp.mode = 1; cp.tiles_per_seq = tps; cp.G = G;
  cp.wait_prior = 1;
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

lca_status decode_impl(lca_plan* p, const void* q_c, const void* q_r, const void* c_kv,
                       const void* k_r, int64_t L, int g, int w, float* out, int32_t* anchor,
                       void* stream, bool dense) {
  lca_status st = check_common(p, q_c, q_r, c_kv, k_r, L, out);
  if (st != LCA_OK) return st;
  int64_t nG = 0;
  if (!dense) {
    if (g < 1 || w < 0) return LCA_ERR_INVALID_ARG;
    nG = lca_num_groups(L, g, w);
    if (nG > 0 && !anchor) return LCA_ERR_INVALID_ARG;
  }
  const Kernel k = choose(p, nG, g);
  if (k == kNone) return LCA_ERR_UNSUPPORTED;
  if (!aligned16(q_c) || !aligned16(q_r) || !aligned16(c_kv) || !aligned16(k_r) ||
      !aligned16(out) || (nG > 0 && !aligned16(anchor)))
    return LCA_ERR_ALIGNMENT;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (k == kTc) return run_tc(p, q_c, q_r, c_kv, k_r, L, g, nG, out, anchor, s);
  return run_simt(p, q_c, q_r, c_kv, k_r, L, g, nG, out, anchor, s);
}

void free_staging(lca_plan* p) {
  cudaFree(p->st_qc); cudaFree(p->st_qr); cudaFree(p->st_c); cudaFree(p->st_k);
  cudaFree(p->st_out); cudaFree(p->st_anc);
  p->st_qc = p->st_qr = p->st_c = p->st_k = nullptr;
  p->st_out = nullptr;
  p->st_anc = nullptr;
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
  const int64_t simt_slots = (int64_t)B * simt_target_splits(p);
  const int64_t tc_slots = p->tc_shape ? (int64_t)B + p->num_sms : 0;
  p->ws_slots = std::max(simt_slots, tc_slots);
  const size_t o_bytes = (size_t)p->ws_slots * H * d_c * sizeof(float);
  const size_t mz_bytes = (size_t)p->ws_slots * H * 2 * sizeof(float);
  if (cudaMalloc(&p->part_o, o_bytes) != cudaSuccess ||
      cudaMalloc(&p->part_mz, mz_bytes) != cudaSuccess ||
      cudaMalloc(&p->err, 2 * sizeof(int)) != cudaSuccess ||
      cudaMemset(p->err, 0, 2 * sizeof(int)) != cudaSuccess) {
    cudaFree(p->part_o); cudaFree(p->part_mz); cudaFree(p->err);
    cudaGetLastError();
    delete p;
    return LCA_ERR_NO_MEMORY;
  }
  *out_plan = p;
  return LCA_OK;
}

lca_status lca_plan_destroy(lca_plan* p) {
  if (!p) return LCA_OK;
  cudaFree(p->part_o); cudaFree(p->part_mz); cudaFree(p->err);
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

lca_status lca_get_device_error(lca_plan* p, void* stream) {
  if (!p) return LCA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int host[2] = {0, 0};
  if (cudaStreamSynchronize(s) != cudaSuccess) return LCA_ERR_CUDA;
  if (cudaMemcpy(host, p->err, sizeof(host), cudaMemcpyDeviceToHost) != cudaSuccess)
    return LCA_ERR_CUDA;
  if (host[0] != 0 && cudaMemset(p->err, 0, sizeof(host)) != cudaSuccess) return LCA_ERR_CUDA;
  return host[0] != 0 ? LCA_ERR_DEVICE_TIMEOUT : LCA_OK;
}

// For callers that may not allocate device memory when they decode -- a
// server whose memory is all reserved up front by its own pool (a cudaMalloc
// here would fail or fragment it) and that cannot keep a plan per shape --
// this entry point runs the same kernels as lca_decode with the fixed
// file-scope scratch above in place of a plan's workspace, and allocates
// nothing.  The first call on a device looks up the scratch's address there
// (cudaGetSymbolAddress) and its SM count, under a mutex, so concurrent first
// calls from several host threads are safe; later calls read the cached
// values without locking.
lca_status lca_decode_noalloc(int B, int H, int d_c, int d_r, lca_dtype dt, const void* q_c,
                              const void* q_r, const void* c_kv, const void* k_r, int64_t L, int g,
                              int w, float* out, int32_t* anchor, void* stream) {
  static std::atomic<float*> scratch[kMaxDevices];   // the scratch's address, per device
  static std::atomic<int> sms[kMaxDevices];
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
  plan.ws_slots = cap;   // run_simt and run_tc refuse a launch that needs more slots
  plan.part_o = base;
  plan.part_mz = base + kNoAllocOFloats;
  plan.err = reinterpret_cast<int*>(base + kNoAllocErrOffset);
  plan.timeout_ns = kDefaultTimeoutNs;
  if (plan.tc_shape) {   // as many tile ranges as the scratch holds partials for
    const int64_t n_hb = H / lca::tc::kHC;
    plan.num_ctas = (int)std::min<int64_t>(plan.num_sms, n_hb * (cap - B + 1));
    if (plan.num_ctas < n_hb) plan.num_ctas = (int)n_hb;
  }
  // The kernels only OR into the error word, so it must start each call at zero.
  if (cudaMemsetAsync(plan.err, 0, 2 * sizeof(int), static_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return LCA_ERR_CUDA;
  return decode_impl(&plan, q_c, q_r, c_kv, k_r, L, g, w, out, anchor, stream, false);
}

}  // extern "C"
