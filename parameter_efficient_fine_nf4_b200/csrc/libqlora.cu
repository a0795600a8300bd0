// libqlora: C ABI of the QLoRA linear layer on sm_100a.
//
// One translation unit: the kernels (nf4_kernels.cuh, gemm_tc.cuh) and the
// host entry points declared in include/qlora.h.  The host code validates
// arguments, carves the caller's workspace, builds TMA tensor maps and
// launches kernels on the caller's stream.  It never allocates device memory.
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

#include <cuda.h>
#include <cuda_runtime.h>
#include <dlfcn.h>
#include <nccl.h>

#include "../../include/qlora.h"
#include "adam_kernels.cuh"
#include "deploy_kernels.cuh"
#include "gemm_tc.cuh"
#include "nf4_gemm.cuh"
#include "nf4_kernels.cuh"
#include "ptx.cuh"

namespace qlora {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kSMs = 148;

std::atomic<int64_t> g_launches{0};

// --------------------------------------------------------------- NF4 table
// [P1] 4-bit NormalFloat paragraph: levels at N(0,1) quantiles, 2^(k-1)
// negative and 2^(k-1)+1 positive points with one shared zero dropped, and
// an exact zero; normalised so the ends are -1 and +1.  The outermost
// probability is not printed on the pages; this library uses
// p_max = 1 - (1/2)(1/32 + 1/30) and spaces each side's probabilities evenly
// from p_max down to 1/2.  Quantiles by Newton's method on the normal CDF in
// long double (monotone convergence from 0 because the CDF is concave on
// the positive half-line).
long double normal_cdf(long double x) { return 0.5L * erfcl(-x / sqrtl(2.0L)); }

long double normal_quantile(long double p) {
  if (p == 0.5L) return 0.0L;
  const long double inv_sqrt_2pi = 0.398942280401432677939946059934381868L;
  long double x = 0.0L;
  for (int it = 0; it < 200; ++it) {
    const long double f = normal_cdf(x) - p;
    const long double dfdx = inv_sqrt_2pi * expl(-0.5L * x * x);
    const long double dx = f / dfdx;
    x -= dx;
    if (fabsl(dx) <= 1e-19L * (1.0L + fabsl(x))) break;
  }
  return x;
}

struct HostTables {
  float levels[16];
  float thresholds[15];
  EncTable enc;
  bool enc_ok;
};

HostTables build_tables() {
  HostTables t;
  const long double pmax = 1.0L - 0.5L * (1.0L / 32.0L + 1.0L / 30.0L);
  long double v[16];
  int n = 0;
  for (int i = 0; i < 7; ++i) v[n++] = -normal_quantile(pmax - i * (pmax - 0.5L) / 7.0L);
  v[n++] = 0.0L;
  for (int i = 7; i >= 0; --i) v[n++] = normal_quantile(pmax - i * (pmax - 0.5L) / 8.0L);
  const long double top = normal_quantile(pmax);
  for (int i = 0; i < 16; ++i) t.levels[i] = (float)(v[i] / top);
  t.levels[0] = -1.0f;
  t.levels[15] = 1.0f;
  for (int i = 0; i < 15; ++i) {
    const double mid = 0.5 * ((double)t.levels[i] + (double)t.levels[i + 1]);  // exact
    float f = (float)mid;
    if ((double)f <= mid) f = nextafterf(f, 2.0f);
    t.thresholds[i] = f;
  }
  t.enc_ok = true;
  memset(&t.enc, 0, sizeof(t.enc));
  for (int i = 0; i < 15; ++i) t.enc.thr[i] = t.thresholds[i];
  t.enc.thr[15] = INFINITY;
  for (int j = 0; j < kEncBins; ++j) {
    const double lo = ((double)j - 64.5) / 64.0;
    const double hi = ((double)j - 63.5) / 64.0;
    int base = 0, inside = 0;
    for (int i = 0; i < 15; ++i) {
      const double th = (double)t.thresholds[i];
      if (th <= lo) ++base;
      else if (th <= hi) ++inside;
    }
    if (inside > 1) t.enc_ok = false;      // the table form needs at most one per bin
    t.enc.base[j] = (uint8_t)base;
  }
  // the fast encoder's coarser bins, rint(16 x) = j - 16, same construction
  for (int j = 0; j < kFastBins; ++j) {
    const double lo = ((double)j - 16.5) / 16.0;
    const double hi = ((double)j - 15.5) / 16.0;
    int base = 0, inside = 0;
    for (int i = 0; i < 15; ++i) {
      const double th = (double)t.thresholds[i];
      if (th <= lo) ++base;
      else if (th <= hi) ++inside;
    }
    if (inside > 1) t.enc_ok = false;
    t.enc.fbase[j] = (uint32_t)base;
    t.enc.fthr[j] = t.enc.thr[base];
  }
  return t;
}

const HostTables& tables() {
  static const HostTables t = build_tables();
  return t;
}

// --------------------------------------------------------------- device setup
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (EncodeTiledFn) nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

std::mutex g_init_mu;
bool g_dev_ready[kMaxDevices] = {false};
unsigned long long g_dev_ctx[kMaxDevices] = {0};
int g_dev_sms[kMaxDevices] = {0};
int g_dev_pair_clusters[kMaxDevices] = {0};
// per device, for few-token clusters of 9..16 CTAs: how many the device
// holds at once (0 where not known)
int g_dev_cluster_fit[kMaxDevices][kSmMaxSplits + 1] = {};
// Which build of the NF4 base GEMM runs for more than 64 tokens: 0 = chosen by
// shape, 1 = one CTA per tile, 2 = CTA pairs (both give the same bits).
std::atomic<int> g_nf4_gemm_mode{0};

// Unique id of the calling thread's current CUDA context, 0 if there is none
// yet.  Ids are never reused within a process, so a device reset (which
// destroys the context; the next runtime call creates a new one) changes it.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);
unsigned long long current_ctx_id() {
  static const CtxGetCurrentFn get_cur = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (CtxGetCurrentFn) nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  static const CtxGetIdFn get_id = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (CtxGetIdFn) nullptr;
    return reinterpret_cast<CtxGetIdFn>(p);
  }();
  if (get_cur == nullptr || get_id == nullptr) return 0;
  CUcontext c = nullptr;
  if (get_cur(&c) != CUDA_SUCCESS || c == nullptr) return 0;
  unsigned long long id = 0;
  if (get_id(c, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// SM count of the current device (persistent grids are sized to it).
int current_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices || g_dev_sms[dev] <= 0)
    return kSMs;
  return g_dev_sms[dev];
}

template <int BN, int KSUB = 1>
cudaError_t set_gemm_attrs() {
  return cudaFuncSetAttribute(gemm_tc_kernel<BN, KSUB>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              GemmCfg<BN, KSUB>::kSmemBytes);
}

template <bool kDx, bool kPair>
cudaError_t set_nf4_gemm_attrs() {
  using Cfg = Nf4Cfg<kPair>;
  const cudaError_t e = cudaFuncSetAttribute(gemm_nf4_kernel<kDx, kPair>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes);
  if (e != cudaSuccess) return e;
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, gemm_nf4_kernel<kDx, kPair>) != cudaSuccess) return cudaErrorInvalidValue;
  return fa.maxThreadsPerBlock >= Cfg::kThreads ? cudaSuccess : cudaErrorLaunchOutOfResources;
}

// Clusters of two CTAs of the paired NF4 GEMM that fit on the device at once.
int pair_clusters_on_device() {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3(2 * kSMs);
  cfg.blockDim = dim3(Nf4Cfg<true>::kThreads);
  cfg.dynamicSmemBytes = Nf4Cfg<true>::kSmemBytes;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, gemm_nf4_kernel<false, true>, &cfg) != cudaSuccess) return 0;
  return n;
}

// How many clusters of s few-token CTAs (s = 9..16, the largest configuration,
// two CTAs per SM) the device holds at once; 0 where the query fails.
void small_cluster_fit(int (&fit)[kSmMaxSplits + 1]) {
  for (int sz = 0; sz <= kSmMaxSplits; ++sz) fit[sz] = 0;
  for (int sz = 9; sz <= kSmMaxSplits; ++sz) {
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)sz);
    cfg.blockDim = dim3(kSmThreads);
    cfg.dynamicSmemBytes = SmallCfg<64>::kSmem;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)sz;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, gemm_nf4_small_kernel<SRC_TMA_K, OUT_U, 64>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    fit[sz] = n;
  }
}

template <int kSrc, int kOut, int TN>
cudaError_t set_small_attrs_one() {
  const cudaError_t e = cudaFuncSetAttribute(gemm_nf4_small_kernel<kSrc, kOut, TN>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, SmallCfg<TN>::kSmem);
  if (e != cudaSuccess) return e;
  // clusters of up to 16 depth splits (beyond the portable 8) where the
  // device schedules them (small_max_splits checks)
  if (cudaFuncSetAttribute(gemm_nf4_small_kernel<kSrc, kOut, TN>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) !=
      cudaSuccess)
    cudaGetLastError();
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, gemm_nf4_small_kernel<kSrc, kOut, TN>) != cudaSuccess)
    return cudaErrorInvalidValue;
  return fa.maxThreadsPerBlock >= kSmThreads ? cudaSuccess : cudaErrorLaunchOutOfResources;
}
template <int kSrc, int kOut>
cudaError_t set_small_attrs_tn() {
  cudaError_t e = set_small_attrs_one<kSrc, kOut, 16>();
  if (e == cudaSuccess) e = set_small_attrs_one<kSrc, kOut, 32>();
  if (e == cudaSuccess) e = set_small_attrs_one<kSrc, kOut, 64>();
  return e;
}
cudaError_t set_small_attrs() {
  cudaError_t e = set_small_attrs_tn<SRC_NF4_ROWS, OUT_BF16>();
  if (e == cudaSuccess) e = set_small_attrs_tn<SRC_NF4_COLS, OUT_BF16>();
  if (e == cudaSuccess) e = set_small_attrs_tn<SRC_TMA_K, OUT_U>();
  if (e == cudaSuccess) e = set_small_attrs_tn<SRC_TMA_MN, OUT_HILO>();
  if (e == cudaSuccess) e = set_small_attrs_tn<SRC_TMA_MN, OUT_U>();
  return e;
}

template <bool kMerge, int KS>
cudaError_t set_deploy_attrs() {
  const cudaError_t e = cudaFuncSetAttribute(lora_deploy_kernel<kMerge, KS>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             DeployCfg<kMerge, KS>::kSmemBytes);
  if (e != cudaSuccess) return e;
  // the kernel's register cap must leave room for its whole block
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, lora_deploy_kernel<kMerge, KS>) != cudaSuccess) return cudaErrorInvalidValue;
  return fa.maxThreadsPerBlock >= kDeployThreads ? cudaSuccess : cudaErrorLaunchOutOfResources;
}

int ensure_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return QLORA_ERR_NO_DEVICE;
  if (dev < 0 || dev >= kMaxDevices) return QLORA_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lk(g_init_mu);
  // the kernel attributes below belong to the context: set them again when
  // the context has changed (after a device reset)
  const unsigned long long ctx = current_ctx_id();
  if (g_dev_ready[dev] && ctx != 0 && ctx == g_dev_ctx[dev]) return QLORA_OK;
  g_dev_ready[dev] = false;
  int major = 0, minor = 0;
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  if (major != 10 || minor != 0) return QLORA_ERR_NO_DEVICE;
  cudaDeviceGetAttribute(&g_dev_sms[dev], cudaDevAttrMultiProcessorCount, dev);
  if (encode_fn() == nullptr) return QLORA_ERR_CUDA;
  if (!tables().enc_ok) return QLORA_ERR_CUDA;
  if (set_gemm_attrs<64>() != cudaSuccess || set_gemm_attrs<128>() != cudaSuccess ||
      set_gemm_attrs<64, 2>() != cudaSuccess || set_gemm_attrs<64, 4>() != cudaSuccess ||
      set_gemm_attrs<128, 2>() != cudaSuccess ||
      set_gemm_attrs<256>() != cudaSuccess || set_deploy_attrs<true, 1>() != cudaSuccess ||
      set_deploy_attrs<true, 2>() != cudaSuccess || set_deploy_attrs<false, 1>() != cudaSuccess ||
      set_deploy_attrs<false, 2>() != cudaSuccess || set_nf4_gemm_attrs<false, false>() != cudaSuccess ||
      set_nf4_gemm_attrs<true, false>() != cudaSuccess || set_nf4_gemm_attrs<false, true>() != cudaSuccess ||
      set_nf4_gemm_attrs<true, true>() != cudaSuccess || set_small_attrs() != cudaSuccess)
    return QLORA_ERR_CUDA;
  g_dev_pair_clusters[dev] = pair_clusters_on_device();
  small_cluster_fit(g_dev_cluster_fit[dev]);
  g_dev_ctx[dev] = current_ctx_id();
  g_dev_ready[dev] = true;
  return QLORA_OK;
}

// --------------------------------------------------------------- profiling
struct ProfRec {
  std::string name;
  double flops, bytes;
  cudaEvent_t start, stop;
};
std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<ProfRec> g_prof;
std::vector<cudaEvent_t> g_event_pool;

cudaEvent_t take_event() {
  if (!g_event_pool.empty()) {
    cudaEvent_t e = g_event_pool.back();
    g_event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

// Launch wrapper: counts the launch, checks the launch error and, when
// profiling, brackets it with events on the launch stream.
template <typename F>
int launch(const char* name, double flops, double bytes, cudaStream_t stream, F&& fn) {
  cudaEvent_t a = nullptr, b = nullptr;
  bool prof = false;
  {
    std::lock_guard<std::mutex> lk(g_prof_mu);
    prof = g_prof_on;
    if (prof) {
      a = take_event();
      b = take_event();
    }
  }
  if (prof) cudaEventRecord(a, stream);
  fn();
  cudaError_t err = cudaGetLastError();
  g_launches.fetch_add(1);
  if (prof) {
    cudaEventRecord(b, stream);
    std::lock_guard<std::mutex> lk(g_prof_mu);
    g_prof.push_back(ProfRec{name, flops, bytes, a, b});
  }
  return err == cudaSuccess ? QLORA_OK : QLORA_ERR_CUDA;
}

// --------------------------------------------------------------- helpers
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }
// fp32 product rounded once (the double product of two floats is exact)
inline float mul_rn_f32(float a, float b) { return (float)((double)a * (double)b); }
inline int64_t nf4_storage_bytes(int64_t d, int64_t k) {
  const int64_t n_b = d * k / 64;
  return d * k / 2 + n_b + 4 * ((n_b + 255) / 256) + 4;
}
inline int grid_for(int64_t n, int threads) {
  int64_t g = cdiv(n, threads);
  const int64_t cap = (int64_t)kSMs * 16;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return (int)g;
}

// bf16 2-D tensor map: `inner` contiguous elements per row, `outer` rows,
// `ld` elements between rows; box = 64 (inner, 128 bytes) x box_outer.
bool make_map(CUtensorMap* map, const void* base, int64_t inner, int64_t outer, int64_t ld,
              int box_outer) {
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 2)};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_outer};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = encode_fn()(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims,
                           strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                           CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// uint8 2-D tensor map (for the NF4 codes): `inner` bytes per row, `outer`
// rows, `ld` bytes between rows; 128-byte swizzle unless given.
bool make_map_u8(CUtensorMap* map, const void* base, int64_t inner, int64_t outer, int64_t ld,
                 int box_inner, int box_outer, CUtensorMapSwizzle sw = CU_TENSOR_MAP_SWIZZLE_128B) {
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)ld};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = encode_fn()(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides,
                           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// fp32 2-D tensor map without swizzle: `inner` contiguous elements per row,
// `outer` rows, `ld` elements between rows (a multiple of 4), box
// box_inner x box_outer (box_inner * 4 a multiple of 16 bytes).
bool make_map_f32(CUtensorMap* map, const void* base, int64_t inner, int64_t outer, int64_t ld, int box_inner,
                  int box_outer) {
  cuuint64_t dims[2] = {(cuuint64_t)inner, (cuuint64_t)outer};
  cuuint64_t strides[1] = {(cuuint64_t)(ld * 4)};
  cuuint32_t box[2] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer};
  cuuint32_t estr[2] = {1u, 1u};
  CUresult r = encode_fn()(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
                           estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Layouts of the per-call block scales (nf4_block_scales): the forward reads
// them transposed (block column s: rows n contiguous, row stride round4(d)),
// dX row-major (row n: block columns contiguous, row stride round4(k / 64)).
inline int64_t scales_ld_fwd(int64_t d) { return (d + 3) / 4 * 4; }
inline int64_t scales_ld_dx(int64_t k) { return (k / 64 + 3) / 4 * 4; }

// Merge / unmerge through the bulk-copy deploy kernel (r <= 128).
template <bool kMerge, int KS>
int launch_deploy_t(const qlora_nf4_t* q, const uint16_t* W, const uint16_t* A, const uint16_t* Bp,
                    int r, int r8, int64_t d, int64_t k, float s, uint16_t* out, cudaStream_t st) {
  CUtensorMap mA, mB, mIo, mOut;
  if (!make_map(&mA, Bp, r8, d, r8, 128)) return QLORA_ERR_CUDA;     // B rows, K-major
  if (!make_map(&mB, A, k, r, k, 64)) return QLORA_ERR_CUDA;         // A columns, MN-major
  if (!make_map(&mOut, out, k, d, k, 32)) return QLORA_ERR_CUDA;      // per-warp 32 x 64 stores
  if (kMerge) {
    if (!make_map_u8(&mIo, q->codes, k / 2, d, k / 2, 128, 128)) return QLORA_ERR_CUDA;
  } else {
    if (!make_map(&mIo, W, k, d, k, 128)) return QLORA_ERR_CUDA;
  }
  DeployArgs a;
  memset(&a, 0, sizeof(a));
  a.d = (int)d; a.k = (int)k; a.r = r;
  a.tiles_m = (int)cdiv(d, 128);
  a.tiles_n = (int)cdiv(k, 256);
  a.alpha = kMerge ? s : -s;
  if (kMerge) { a.absmax_q = q->absmax_q; a.scale2 = q->scale2; a.mean = q->mean; }
  memcpy(a.levels, tables().levels, sizeof(a.levels));
  const int64_t units = (int64_t)a.tiles_m * a.tiles_n;
  const dim3 grid((unsigned)std::min<int64_t>(units, current_sms()));
  const double bytes = (double)d * k * (kMerge ? 2.5 : 4.0);
  return launch(kMerge ? "lora_merge" : "lora_unmerge", 2.0 * d * (double)k * r, bytes, st, [&] {
    lora_deploy_kernel<kMerge, KS><<<grid, kDeployThreads, DeployCfg<kMerge, KS>::kSmemBytes, st>>>(mA, mB, mIo, mOut, a);
  });
}

int launch_deploy(bool merge, const qlora_nf4_t* q, const uint16_t* W, const uint16_t* A,
                  const uint16_t* Bp, int r, int r8, int64_t d, int64_t k, float s, uint16_t* out,
                  cudaStream_t st) {
  if (merge) return r <= 64 ? launch_deploy_t<true, 1>(q, W, A, Bp, r, r8, d, k, s, out, st)
                            : launch_deploy_t<true, 2>(q, W, A, Bp, r, r8, d, k, s, out, st);
  return r <= 64 ? launch_deploy_t<false, 1>(q, W, A, Bp, r, r8, d, k, s, out, st)
                 : launch_deploy_t<false, 2>(q, W, A, Bp, r, r8, d, k, s, out, st);
}

// One GEMM operand as stored in global memory.
struct Operand {
  const void* ptr = nullptr;
  int64_t inner = 0, outer = 0, ld = 0;   // bf16 elements
  int mn_major = 0;                       // 1: the M (or N) index is the contiguous one
};

inline Operand kmajor(const void* p, int64_t K, int64_t rows, int64_t ld) {
  Operand o; o.ptr = p; o.inner = K; o.outer = rows; o.ld = ld; o.mn_major = 0; return o;
}
inline Operand mnmajor(const void* p, int64_t MN, int64_t K, int64_t ld) {
  Operand o; o.ptr = p; o.inner = MN; o.outer = K; o.ld = ld; o.mn_major = 1; return o;
}

struct GemmPlan {
  int M, N, K0, K1 = 0;
  Operand a0, b0, a1, b1;
  int splits = 1;
  int bn = 256;
  int ksub = 1;      // 64-wide K sub-blocks per pipeline stage
};

template <int BN, int KSUB = 1>
int launch_gemm_bn(const char* name, const GemmPlan& g, GemmArgs args, cudaStream_t st) {
  CUtensorMap m[4];
  memset(m, 0, sizeof(m));
  const Operand* ops[4] = {&g.a0, &g.b0, &g.a1, &g.b1};
  const int nops = g.K1 > 0 ? 4 : 2;
  for (int i = 0; i < nops; ++i) {
    const Operand& o = *ops[i];
    const bool is_a = (i % 2) == 0;
    const int box_outer = o.mn_major ? 64 : (is_a ? kBM : BN);
    if (!make_map(&m[i], o.ptr, o.inner, o.outer, o.ld, box_outer)) return QLORA_ERR_CUDA;
  }
  if (nops == 2) { m[2] = m[0]; m[3] = m[1]; }
  args.M = g.M; args.N = g.N; args.K0 = g.K0; args.K1 = g.K1;
  args.a0_mn = g.a0.mn_major; args.b0_mn = g.b0.mn_major;
  args.a1_mn = g.K1 > 0 ? g.a1.mn_major : 0; args.b1_mn = g.K1 > 0 ? g.b1.mn_major : 0;
  args.tiles_m = (int)cdiv(g.M, kBM);
  args.tiles_n = (int)cdiv(g.N, BN);
  args.group_m = 16;
  args.k_per_split = (int)round_up(cdiv(g.K0, g.splits), kBK);
  const int splits = (int)cdiv(g.K0, args.k_per_split);
  const auto& T = tables();
  memcpy(args.levels, T.levels, sizeof(args.levels));
  // bf16 outputs of the 256-wide kernel leave through shared staging and TMA
  // stores when the rows are 16-byte aligned
  CUtensorMap mo = m[0];
  args.tma_store = 0;
  if (BN == 256 && args.epi == EPI_BF16 && aligned16(args.out) && (args.ldo % 8) == 0 &&
      args.n_store == g.N) {
    if (!make_map(&mo, args.out, g.N, g.M, args.ldo, 32)) return QLORA_ERR_CUDA;
    args.tma_store = 1;
  }
  // persistent: one CTA per SM (or per unit when there are fewer units)
  const int64_t units = (int64_t)args.tiles_m * args.tiles_n * splits;
  dim3 grid((unsigned)std::min<int64_t>(units, current_sms()), 1, 1);
  const double flops = 2.0 * g.M * (double)g.N * (g.K0 + g.K1);
  return launch(name, flops, 0.0, st, [&] {
    gemm_tc_kernel<BN, KSUB><<<grid, kGemmThreads, GemmCfg<BN, KSUB>::kSmemBytes, st>>>(m[0], m[1], m[2], m[3], mo,
                                                                                        args);
  });
}

int launch_gemm(const char* name, const GemmPlan& g, const GemmArgs& args, cudaStream_t st) {
  for (const Operand* o : {&g.a0, &g.b0}) {
    if (!aligned16(o->ptr) || (o->ld * 2) % 16 != 0) return QLORA_ERR_MISALIGNED;
  }
  if (g.K1 > 0) {
    for (const Operand* o : {&g.a1, &g.b1})
      if (!aligned16(o->ptr) || (o->ld * 2) % 16 != 0) return QLORA_ERR_MISALIGNED;
  }
  switch (g.bn) {
    case 64:
      if (g.ksub >= 4) return launch_gemm_bn<64, 4>(name, g, args, st);
      if (g.ksub == 2) return launch_gemm_bn<64, 2>(name, g, args, st);
      return launch_gemm_bn<64>(name, g, args, st);
    case 128:
      if (g.ksub >= 2) return launch_gemm_bn<128, 2>(name, g, args, st);
      return launch_gemm_bn<128>(name, g, args, st);
    default: return launch_gemm_bn<256>(name, g, args, st);
  }
}

inline int bn_for_rank(int r) { return r <= 64 ? 64 : (r <= 128 ? 128 : 256); }

// 64-wide K sub-blocks per pipeline stage of the adapter GEMMs.  These stream
// a T x k (or T x d) activation against a rank-r operand and are bound by
// HBM; wider stages fetch 256 (U, G) or 128 (dA, dB) contiguous columns of
// every activation row at once: 13-15 % faster than one sub-block per stage
// at the 8192 -> 22016 projection pair, 16384 tokens.
constexpr int kAdapterKSub = 4;    // U = X A^T and G = dY B: K-major rows of X / dY
constexpr int kGradKSub = 2;       // dA, dB: T-reductions over MN-major X / dY

GemmArgs blank_args() {
  GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.alpha = 1.0f;
  a.alpha2 = 1.0f;
  return a;
}

// Workspace carving (256-byte aligned pieces).
struct Carver {
  uint8_t* base;
  size_t off = 0;
  void* take(size_t bytes) {
    void* p = base ? base + off : nullptr;
    off += (size_t)round_up((int64_t)bytes, 256);
    return p;
  }
};

int check_nf4(const qlora_nf4_t* q) {
  if (!q || !q->codes || !q->absmax_q || !q->scale2 || !q->mean) return QLORA_ERR_INVALID_ARG;
  if (q->block != kBlock || q->block2 != kBlock2) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (q->d < 1 || q->k < 64 || q->k % 64 != 0) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (q->d > (int64_t)1 << 31 || q->k > (int64_t)1 << 31 || q->d * q->k >= ((int64_t)1 << 34))
    return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(q->codes)) return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

int check_rank(int r, float alpha) {
  if (r < 1 || r > 256) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!(alpha > 0.0f) || !std::isfinite(alpha)) return QLORA_ERR_INVALID_ARG;
  return QLORA_OK;
}

#define QLORA_TRY(x)            \
  do {                          \
    int _s = (x);               \
    if (_s != QLORA_OK) return _s; \
  } while (0)

int dequantize_into(const qlora_nf4_t* q, uint16_t* W, cudaStream_t st) {
  const int64_t n_units = q->d * q->k / 8;
  const auto& T = tables();
  NF4Levels lv;
  memcpy(lv.q, T.levels, sizeof(lv.q));
  const int grid = std::max(1, std::min<int>((int)cdiv(n_units, 256 * 4), current_sms() * 8));
  const double bytes = (double)q->d * q->k * 2.5;
  return launch("nf4_dequantize", 0.0, bytes, st, [&] {
    nf4_dequantize_kernel<<<grid, 256, 0, st>>>(reinterpret_cast<const uint32_t*>(q->codes), q->absmax_q,
                                                q->scale2, q->mean, n_units,
                                                reinterpret_cast<uint4*>(W), lv);
  });
}

// B (d x r) with rows padded to r8 columns, when r is not a multiple of 8.
const uint16_t* padded_B(const uint16_t* B, int64_t d, int r, int r8, uint16_t* ws, cudaStream_t st,
                         int* status) {
  if (r == r8) return B;
  *status = launch("pad_cols_bf16", 0.0, 0.0, st, [&] {
    pad_cols_bf16<<<grid_for(d * r8, 256), 256, 0, st>>>(B, d, r, ws, r8);
  });
  return ws;
}

// Few-token plan of gemm_nf4_small_kernel: tokens padded to TN, 128-row
// tiles of the Mw output features, the main depth split so that about three
// CTAs per SM are busy, while every split keeps at least eight K-steps and a
// row tile has at most kSmMaxSplits splits (the last CTA's reduction keeps
// all of them in flight).
constexpr int64_t kSmallT = 64;
struct SmallPlan {
  int tn = 16, tiles_m = 1, splits = 1;
};
SmallPlan small_plan(int64_t Mw, int64_t K0, int64_t T) {
  SmallPlan sp;
  sp.tn = T <= 16 ? 16 : (T <= 32 ? 32 : 64);
  sp.tiles_m = (int)cdiv(Mw, 128);
  const int steps0 = (int)cdiv(K0, 64);
  // two CTAs of the few-token kernel fit on an SM; one wave of them
  const int want = std::max(1, (int)(2 * kSMs / sp.tiles_m));
  // at least 4 K-steps per split; more than the portable 8 splits only where
  // the device holds every cluster of that size at once (checked per size)
  int splits = std::max(1, std::min(std::min(want, steps0 / 4), kSmMaxSplits));
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) dev = -1;
  while (splits > 8 && (dev < 0 || g_dev_cluster_fit[dev][splits] < sp.tiles_m)) --splits;
  sp.splits = splits;
  return sp;
}

// Forward workspace: bf16 s*U (the rank-r operand of the extension), B
// padded to r8 columns and the block scales of the dequantising GEMM (the
// few-token kernels keep their split partials in shared memory).  No copy of
// the weight: the QLoRA path dequantises inside the GEMM and plain LoRA reads
// the caller's W.
struct FwdWs {
  uint16_t* sU; uint16_t* Bp;
  uint16_t* Xm;            // LoRA dropout: the masked adapter input
  uint16_t* Bcat; float* Uall;   // several adapters: B_0..B_{n-1} side by side, U of every adapter
  float* scales;           // fp32 block scales of the NF4 weight (forward layout)
  size_t bytes;
};
// `r` is the rank seen by the GEMMs (n r for a stack of n adapters of rank r).
FwdWs carve_fwd(void* ws, int64_t d, int64_t k, int r, int64_t T, bool dropout = false, bool multi = false) {
  Carver c{reinterpret_cast<uint8_t*>(ws)};
  const int64_t r8 = round_up(r, 8);
  FwdWs w;
  w.sU = (uint16_t*)c.take((size_t)(std::max<int64_t>(T, 1) * r8 * 2));
  w.Bp = (uint16_t*)c.take((size_t)(d * r8 * 2));
  w.Xm = dropout ? (uint16_t*)c.take((size_t)(std::max<int64_t>(T, 1) * k * 2)) : nullptr;
  w.Bcat = multi ? (uint16_t*)c.take((size_t)(d * r * 2)) : nullptr;
  w.Uall = multi ? (float*)c.take((size_t)(std::max<int64_t>(T, 1) * r * 4)) : nullptr;
  w.scales = (float*)c.take((size_t)(k / 64 * scales_ld_fwd(d) * 4));
  w.bytes = c.off;
  return w;
}

int splits_for(int64_t tiles, int64_t K) {
  int s = 1;
  while (tiles * s < 2 * kSMs && (K / (s * 2)) >= 1024 && s < 32) s *= 2;
  return s;
}

// Effective split count of a K range cut into 64-aligned pieces (the kernel
// derives the same value from k_per_split).
int eff_splits(int64_t K, int splits) {
  const int64_t per = round_up(cdiv(K, splits), kBK);
  return (int)cdiv(K, per);
}

struct BwdWs {
  uint16_t* Us2; uint16_t* Gs2; uint16_t* Bp; float* partA; float* partB;
  uint16_t* Xm;            // LoRA dropout: the masked adapter input
  uint16_t* Bcat; float* Gall; float* dBcat;   // several adapters
  float* scales;           // fp32 block scales of the NF4 weight (dX layout)
  float* sGf;              // T <= 64: s G in fp32 (T x r), operand of the CUDA-core dA
  float* sUf;              // T <= 64, several adapters: s U scattered into the token's block (T x r)
  int rp, halves, splitsA, splitsB; size_t bytes;
};
// Backward workspace.  U and G enter the T-reductions (dB, dA) as two bf16
// terms, hi = bf16(v) and lo = bf16(v - hi), stored side by side in rows of
// 2*rp columns (rp = r rounded up to 32); with rp <= 128 one GEMM with N = 2*rp
// multiplies both and the epilogue adds the paired columns, otherwise the two
// halves run as two GEMMs whose partial outputs are summed.
BwdWs carve_bwd(void* ws, int64_t d, int64_t k, int r, int64_t T, bool dropout = false, bool multi = false) {
  Carver c{reinterpret_cast<uint8_t*>(ws)};
  const int64_t r8 = round_up(r, 8);
  const int64_t Tm = std::max<int64_t>(T, 1);
  BwdWs w;
  w.rp = (int)round_up(r, 32);
  w.halves = w.rp > 128 ? 2 : 1;
  w.Us2 = (uint16_t*)c.take((size_t)(Tm * 2 * w.rp * 2));
  w.Gs2 = (uint16_t*)c.take((size_t)(Tm * 2 * w.rp * 2));
  w.Bp = (uint16_t*)c.take((size_t)(d * r8 * 2));
  w.splitsA = eff_splits(Tm, splits_for(cdiv(k, kBM), Tm));
  w.splitsB = eff_splits(Tm, splits_for(cdiv(d, kBM), Tm));
  const int64_t pa = (int64_t)w.splitsA * w.halves, pb = (int64_t)w.splitsB * w.halves;
  w.partA = (float*)c.take((size_t)(pa > 1 ? pa * r * k * 4 : 0));
  w.partB = (float*)c.take((size_t)(pb > 1 ? pb * d * r * 4 : 0));
  w.sGf = (T >= 1 && T <= kSmallT) ? (float*)c.take((size_t)(T * r * 4)) : nullptr;
  w.sUf = (T >= 1 && T <= kSmallT && multi) ? (float*)c.take((size_t)(T * r * 4)) : nullptr;
  w.Xm = dropout ? (uint16_t*)c.take((size_t)(Tm * k * 2)) : nullptr;
  w.Bcat = multi ? (uint16_t*)c.take((size_t)(d * r * 2)) : nullptr;
  w.Gall = multi ? (float*)c.take((size_t)(Tm * r * 4)) : nullptr;
  w.dBcat = multi ? (float*)c.take((size_t)(d * r * 4)) : nullptr;
  w.scales = (float*)c.take((size_t)(d * scales_ld_dx(k) * 4));
  w.bytes = c.off;
  return w;
}

// One T-reduction GEMM of the adapter gradients: out (M x r, or r x M when
// transposed) = big^T hilo, big an MN-major T x M bf16 matrix, hilo the
// T x 2rp hi/lo operand.  Deterministic: partials are reduced in fixed order.
int adapter_grad_gemm(const char* name, const uint16_t* big, int64_t M, int64_t T, const uint16_t* hilo,
                      int r, int rp, int halves, int splits, bool transposed, float* out,
                      float* part, cudaStream_t st, float alpha = 1.0f) {
  const int nparts = splits * halves;
  const int64_t plane = M * r;
  for (int h = 0; h < halves; ++h) {
    GemmPlan g;
    g.M = (int)M; g.K0 = (int)T; g.splits = splits; g.ksub = kGradKSub;
    g.a0 = mnmajor(big, M, T, M);
    GemmArgs a = blank_args();
    a.epi = transposed ? EPI_F32_T : EPI_F32;
    a.alpha = alpha;
    a.n_store = r;
    a.ldo = transposed ? M : r;
    if (halves == 1) {
      g.N = 2 * rp; g.bn = 2 * rp;
      g.b0 = mnmajor(hilo, 2 * rp, T, 2 * rp);
      a.pair_offset = rp;
    } else {
      g.N = r; g.bn = 256;
      g.b0 = mnmajor(hilo + (size_t)h * rp, r, T, 2 * rp);
    }
    if (nparts > 1) {
      a.out = part + (size_t)h * splits * plane;
      a.split_stride = plane;
    } else {
      a.out = out;
    }
    QLORA_TRY(launch_gemm(name, g, a, st));
  }
  if (nparts > 1) {
    QLORA_TRY(launch("splitk_reduce_f32", 0.0, (double)plane * 4 * (nparts + 1), st, [&] {
      splitk_reduce_f32<<<grid_for(plane, 256), 256, 0, st>>>(part, nparts, plane, out);
    }));
  }
  return QLORA_OK;
}

int pair_clusters() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 0;
  return g_dev_pair_clusters[dev];
}

// CTA pairs halve each SM's share of the decode at the same MMA work per SM;
// measured faster than one CTA per tile at every shape from 65 to 16384
// tokens, so they are the default wherever clusters of two fit.
bool nf4_use_pair() {
  const int mode = g_nf4_gemm_mode.load();
  return mode != 1 && pair_clusters() > 0;
}

// Base GEMM on the NF4 weight with the rank-r extension (gemm_nf4_kernel):
//   forward (dx = false): out = Y (T x d)  = [X | sU][W' | B]^T,  a1 = sU (T x r8, ld r8), b1 = B (d x r8)
//   dX      (dx = true):  out = dX (T x k) = [dY | sG][W' ; A],    a1 = sG (T x r, ld a1_ld), b1 = A (r x k)
int launch_nf4_gemm(bool dx, const qlora_nf4_t* q, const float* scales, const uint16_t* act, int64_t T,
                    const uint16_t* a1, int64_t a1_inner, int64_t a1_ld, const uint16_t* b1, int r, int r8,
                    uint16_t* out, cudaStream_t st) {
  const int64_t d = q->d, k = q->k;
  Nf4GemmArgs a;
  memset(&a, 0, sizeof(a));
  a.M = (int)T;
  a.N = (int)(dx ? k : d);
  a.K0 = (int)(dx ? d : k);
  a.K1 = r;
  const bool pair = nf4_use_pair();
  a.tiles_m = (int)cdiv(T, pair ? 512 : 256);
  a.tiles_n = (int)cdiv(a.N, 256);
  a.group_m = pair ? 4 : 8;
  memcpy(a.levels, tables().levels, sizeof(a.levels));
  CUtensorMap mA0, mC, mS, mA1, mB1, mO;
  // codes and scales: a pair's CTA loads the half of the weight tile it decodes
  if (dx) {
    if (!make_map_f32(&mS, scales, k / 64, d, scales_ld_dx(k), 4, 64)) return QLORA_ERR_CUDA;
  } else {
    if (!make_map_f32(&mS, scales, d, k / 64, scales_ld_fwd(d), pair ? 128 : 256, 1)) return QLORA_ERR_CUDA;
  }
  if (!make_map(&mA0, act, a.K0, T, a.K0, 128)) return QLORA_ERR_CUDA;
  if (dx) {
    if (pair) {
      if (!make_map_u8(&mC, q->codes, k / 2, d, k / 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_64B)) return QLORA_ERR_CUDA;
    } else {
      if (!make_map_u8(&mC, q->codes, k / 2, d, k / 2, 128, 64, CU_TENSOR_MAP_SWIZZLE_128B)) return QLORA_ERR_CUDA;
    }
  } else {
    if (!make_map_u8(&mC, q->codes, k / 2, d, k / 2, 32, pair ? 128 : 256, CU_TENSOR_MAP_SWIZZLE_32B))
      return QLORA_ERR_CUDA;
  }
  if (r == 0) {
    mA1 = mA0;
    mB1 = mA0;
  } else {
    if (!make_map(&mA1, a1, a1_inner, T, a1_ld, 128)) return QLORA_ERR_CUDA;
    if (dx) {
      if (!make_map(&mB1, b1, k, r, k, 64)) return QLORA_ERR_CUDA;        // A columns, MN-major
    } else {
      // B rows, K-major (a pair's CTA loads its 128 of the tile's 256 rows)
      if (!make_map(&mB1, b1, r8, d, r8, pair ? 128 : 256)) return QLORA_ERR_CUDA;
    }
  }
  mO = mA0;
  a.out = out;
  a.ldo = a.N;
  a.tma_store = 0;
  if (aligned16(out) && (a.N % 8) == 0) {
    if (!make_map(&mO, out, a.N, T, a.N, 32)) return QLORA_ERR_CUDA;
    a.tma_store = 1;
  }
  const double flops = 2.0 * (double)T * a.N * ((double)a.K0 + r);
  const char* name = dx ? "gemm_nf4_dx" : "gemm_nf4_fwd";
  const int64_t units = (int64_t)a.tiles_m * a.tiles_n;
  if (!pair) {
    const dim3 grid((unsigned)std::min<int64_t>(units, current_sms()));
    return launch(name, flops, 0.0, st, [&] {
      if (dx)
        gemm_nf4_kernel<true, false>
            <<<grid, Nf4Cfg<false>::kThreads, Nf4Cfg<false>::kSmemBytes, st>>>(mA0, mC, mS, mA1, mB1, mO, a);
      else
        gemm_nf4_kernel<false, false>
            <<<grid, Nf4Cfg<false>::kThreads, Nf4Cfg<false>::kSmemBytes, st>>>(mA0, mC, mS, mA1, mB1, mO, a);
    });
  }
  // CTA pairs: units of 512 rows, one cluster of two per unit, as many
  // clusters as fit at once
  const int64_t clusters = std::min<int64_t>(units, std::max(1, pair_clusters()));
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = dim3((unsigned)(2 * clusters));
  cfg.blockDim = dim3(Nf4Cfg<true>::kThreads);
  cfg.dynamicSmemBytes = Nf4Cfg<true>::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return launch(name, flops, 0.0, st, [&] {
    if (dx)
      cudaLaunchKernelEx(&cfg, gemm_nf4_kernel<true, true>, mA0, mC, mS, mA1, mB1, mO, a);
    else
      cudaLaunchKernelEx(&cfg, gemm_nf4_kernel<false, true>, mA0, mC, mS, mA1, mB1, mO, a);
  });
}

// One few-token GEMM (gemm_nf4_small_kernel): out^T (Mw x T) = Wside * act^T
// over K0 (+ the rank-r extension for the NF4 products), depth split over
// CTAs, partials summed in split order by the last CTA of each row tile.
struct SmallJob {
  int src = SRC_NF4_ROWS, out = OUT_BF16;
  const char* name = "";
  const qlora_nf4_t* q = nullptr;                         // NF4 sources
  const void* w = nullptr;                                // bf16 sources: the tensor tiles are cut from
  int64_t w_inner = 0, w_outer = 0, w_ld = 0;
  const uint16_t* act = nullptr;                          // T x K0 activations (row stride K0)
  int64_t K0 = 0, Mw = 0;
  int r = 0, r8 = 0;                                      // extension (NF4 sources)
  const uint16_t* a1 = nullptr;
  int64_t a1_inner = 0, a1_ld = 0;
  const uint16_t* w1 = nullptr;
  float* f32_out = nullptr;
  int ldf = 0, nf = 0;
  uint16_t* b16_out = nullptr;
  int ldb = 0, nb = 0, lo_off = 0;
  float scale = 1.0f, f32_scale = 1.0f;
};

// One launch of the few-token kernel; the depth splits of a row tile form a
// cluster (consecutive blocks) when there are several.
template <int kSrc, int kOut, int TN>
cudaError_t small_launch_tn(dim3 grid, int splits, cudaStream_t st, const CUtensorMap& a, const CUtensorMap& w,
                            const CUtensorMap& w1, const CUtensorMap& a1, const Nf4SmallArgs& p) {
  cudaLaunchConfig_t cfg;
  memset(&cfg, 0, sizeof(cfg));
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kSmThreads);
  cfg.dynamicSmemBytes = SmallCfg<TN>::kSmem;
  cfg.stream = st;
  // programmatic dependent launch: the kernel's prologue may overlap the
  // previous kernel of the stream (the kernel waits for it before touching
  // global memory)
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  at[1].id = cudaLaunchAttributeClusterDimension;
  at[1].val.clusterDim.x = (unsigned)splits;
  at[1].val.clusterDim.y = 1;
  at[1].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = splits > 1 ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, gemm_nf4_small_kernel<kSrc, kOut, TN>, a, w, w1, a1, p);
}
template <int kSrc, int kOut>
void small_dispatch(int tn, dim3 grid, int splits, cudaStream_t st, const CUtensorMap& a, const CUtensorMap& w,
                    const CUtensorMap& w1, const CUtensorMap& a1, const Nf4SmallArgs& p) {
  switch (tn) {
    case 16: small_launch_tn<kSrc, kOut, 16>(grid, splits, st, a, w, w1, a1, p); break;
    case 32: small_launch_tn<kSrc, kOut, 32>(grid, splits, st, a, w, w1, a1, p); break;
    default: small_launch_tn<kSrc, kOut, 64>(grid, splits, st, a, w, w1, a1, p); break;
  }
}

int launch_small(const SmallJob& j, int64_t T, cudaStream_t st) {
  const SmallPlan sp = small_plan(j.Mw, j.K0, T);
  Nf4SmallArgs a;
  memset(&a, 0, sizeof(a));
  a.T = (int)T;
  a.Mw = (int)j.Mw;
  a.K0 = (int)j.K0;
  a.K1 = j.r;
  a.tiles_m = sp.tiles_m;
  a.splits = sp.splits;
  a.f32_out = j.f32_out;
  a.ldf = j.ldf;
  a.nf = j.nf;
  a.b16_out = j.b16_out;
  a.ldb = j.ldb;
  a.nb = j.nb;
  a.lo_off = j.lo_off;
  a.scale = j.scale;
  a.f32_scale = j.f32_scale;
  memcpy(a.levels, tables().levels, sizeof(a.levels));
  CUtensorMap mAct, mW, mW1, mAct1;
  if (!make_map(&mAct, j.act, j.K0, T, j.K0, sp.tn)) return QLORA_ERR_CUDA;
  double bytes = 0.0;
  if (j.src == SRC_NF4_ROWS || j.src == SRC_NF4_COLS) {
    const int64_t d = j.q->d, k = j.q->k;
    bytes = (double)nf4_storage_bytes(d, k);
    a.absmax_q = j.q->absmax_q;
    a.scale2 = j.q->scale2;
    a.mean = j.q->mean;
    a.kb = (int)(k / 64);
    if (j.src == SRC_NF4_COLS) {
      if (!make_map_u8(&mW, j.q->codes, k / 2, d, k / 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_64B)) return QLORA_ERR_CUDA;
    } else {
      if (!make_map_u8(&mW, j.q->codes, k / 2, d, k / 2, 32, 128, CU_TENSOR_MAP_SWIZZLE_32B)) return QLORA_ERR_CUDA;
    }
    if (j.r == 0) {
      mW1 = mW;
      mAct1 = mAct;
    } else {
      if (j.src == SRC_NF4_COLS) {
        if (!make_map(&mW1, j.w1, k, j.r, k, 64)) return QLORA_ERR_CUDA;          // A columns, MN-major
      } else {
        if (!make_map(&mW1, j.w1, j.r8, d, j.r8, 128)) return QLORA_ERR_CUDA;     // B rows, K-major
      }
      if (!make_map(&mAct1, j.a1, j.a1_inner, T, j.a1_ld, sp.tn)) return QLORA_ERR_CUDA;
    }
  } else {
    const int box_outer = j.src == SRC_TMA_MN ? 64 : 128;
    if (!make_map(&mW, j.w, j.w_inner, j.w_outer, j.w_ld, box_outer)) return QLORA_ERR_CUDA;
    mW1 = mW;
    mAct1 = mAct;
  }
  const dim3 grid((unsigned)(sp.tiles_m * sp.splits));
  const double flops = 2.0 * (double)T * j.Mw * ((double)j.K0 + j.r);
  return launch(j.name, flops, bytes, st, [&] {
    switch (j.src) {
      case SRC_NF4_ROWS: small_dispatch<SRC_NF4_ROWS, OUT_BF16>(sp.tn, grid, sp.splits, st, mAct, mW, mW1, mAct1, a); break;
      case SRC_NF4_COLS: small_dispatch<SRC_NF4_COLS, OUT_BF16>(sp.tn, grid, sp.splits, st, mAct, mW, mW1, mAct1, a); break;
      case SRC_TMA_K: small_dispatch<SRC_TMA_K, OUT_U>(sp.tn, grid, sp.splits, st, mAct, mW, mW1, mAct1, a); break;
      default:
        if (j.out == OUT_U)
          small_dispatch<SRC_TMA_MN, OUT_U>(sp.tn, grid, sp.splits, st, mAct, mW, mW1, mAct1, a);
        else
          small_dispatch<SRC_TMA_MN, OUT_HILO>(sp.tn, grid, sp.splits, st, mAct, mW, mW1, mAct1, a);
        break;
    }
  });
}

// a' of every block of q into `out`, transposed (forward) or row-major (dX).
int block_scales(const qlora_nf4_t* q, bool transposed, float* out, cudaStream_t st) {
  const int64_t d = q->d, kb = q->k / 64;
  const int64_t ld = transposed ? scales_ld_fwd(d) : scales_ld_dx(q->k);
  const dim3 grid((unsigned)cdiv(kb, 32), (unsigned)cdiv(d, 32));
  return launch("nf4_block_scales", 0.0, (double)d * kb * 5, st, [&] {
    nf4_block_scales<<<grid, 256, 0, st>>>(q->absmax_q, q->scale2, q->mean, d, kb, transposed ? 1 : 0, ld, out);
  });
}

// A second stream of the calling thread on the current device, with two
// events, for work that may run beside the main stream's (fork / join by
// events, so that stream capture into a CUDA graph turns it into parallel
// branches).  Per thread, so that concurrent callers never share it.
struct SideStream {
  cudaStream_t st = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
  unsigned long long ctx = 0;
};
SideStream* side_stream() {
  thread_local SideStream side[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  SideStream& s = side[dev];
  const unsigned long long ctx = current_ctx_id();
  if (s.st == nullptr || s.ctx != ctx) {
    // a new context (first use, or after a device reset): the old handles
    // belonged to the old one
    s.st = nullptr;
    s.fork = s.join = nullptr;
    if (cudaStreamCreateWithFlags(&s.st, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&s.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&s.join, cudaEventDisableTiming) != cudaSuccess) {
      s.st = nullptr;
      return nullptr;
    }
    s.ctx = ctx;
  }
  return &s;
}

// dA (r x k) and dB (d x r) of a few tokens on CUDA cores (adapter_grads_small).
int grads_small(const uint16_t* X, const uint16_t* dY, const float* U, const float* sG, float s, int64_t T,
                int64_t d, int64_t k, int r, float* dA, float* dB, cudaStream_t st) {
  // four columns of dA / four rows of dB per thread (k % 64 == 0, d % 8 == 0)
  const int kblk = (int)cdiv(k / 4, kGradThreads);
  const int nb_a = r * kblk;
  const int nb_b = (int)cdiv(d / 4, kGradThreads / r);
  const double n = (double)r * k + (double)d * r;
  return launch("adapter_grads_small", 2.0 * (double)T * n, n * 4, st, [&] {
    cudaLaunchConfig_t cfg;
    memset(&cfg, 0, sizeof(cfg));
    cfg.gridDim = dim3((unsigned)(nb_a + nb_b));
    cfg.blockDim = dim3(kGradThreads);
    cfg.stream = st;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    at[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    cudaLaunchKernelEx(&cfg, adapter_grads_small, X, dY, U, sG, s, (int)T, (int)d, (int)k, r, kblk, nb_a, dA, dB);
  });
}

// Forward on a bf16 d x k weight W (plain LoRA: the caller's W) or, when `q`
// is given, on the NF4 weight dequantised inside the GEMM (W unused).
// A stack of n unmerged adapters of rank ra chosen per token (idx[t]); the
// GEMMs then see rank n ra with A = [A_0; ...; A_{n-1}] and B = [B_0 | ... ],
// and every rank-r operand is scattered into the token's block.
struct MultiAdapter {
  int n, ra;
  const int32_t* idx;
  AdapterScales sc;
};

// With LoRA dropout (`keep` given, rate p): the adapter path reads the masked
// input X * keep (in the workspace) and U is scaled by c = 1 / (1 - p), so
// U = D(X) A^T with D(X) = X * keep / (1 - p); the frozen path reads X.
int fwd_core(const qlora_nf4_t* q, const uint16_t* W, int64_t d, int64_t k, const uint16_t* A, const uint16_t* B, int r,
             float alpha, const uint16_t* X, int64_t T, uint16_t* Y, float* U_save, const FwdWs& w,
             cudaStream_t st, const uint8_t* keep = nullptr, float c = 1.0f,
             const MultiAdapter* ma = nullptr) {
  const float s = alpha / (float)r;
  const uint16_t* Xa = X;
  if (keep) {
    QLORA_TRY(launch("apply_keep_bf16", 0.0, (double)T * k * 4.125, st, [&] {
      apply_keep_bf16<<<grid_for(T * k / 8, 256), 256, 0, st>>>(reinterpret_cast<const uint4*>(X), keep, T * k / 8,
                                                                reinterpret_cast<uint4*>(w.Xm));
    }));
    Xa = w.Xm;
  }
  const float su = keep ? mul_rn_f32(s, c) : s;
  const int r8 = (int)round_up(r, 8);
  int pst = QLORA_OK;
  const uint16_t* Bp = padded_B(B, d, r, r8, w.Bp, st, &pst);
  QLORA_TRY(pst);

  if (T > kSmallT && q) {
    // block scales for the dequantising GEMM (the few-token kernels form
    // them from the stored constants themselves)
    QLORA_TRY(block_scales(q, true, w.scales, st));
  }
  // U = X A^T (fp32 to U_save), sU = bf16(s U) (operand of the extension)
  if (T <= kSmallT) {
    SmallJob j;
    j.src = SRC_TMA_K; j.out = OUT_U; j.name = "gemm_lora_down_small";
    j.w = A; j.w_inner = k; j.w_outer = r; j.w_ld = k;
    j.act = Xa; j.K0 = k; j.Mw = r8;
    j.f32_out = ma ? w.Uall : U_save; j.ldf = r; j.nf = r; j.f32_scale = c;
    j.b16_out = w.sU; j.ldb = r8; j.nb = ma ? 0 : r8; j.scale = su;
    QLORA_TRY(launch_small(j, T, st));
  } else {
    GemmPlan g;
    g.M = (int)T; g.N = r; g.K0 = (int)k; g.bn = bn_for_rank(r); g.ksub = kAdapterKSub;
    g.a0 = kmajor(Xa, k, T, k);
    g.b0 = kmajor(A, k, r, k);
    GemmArgs a = blank_args();
    a.epi = EPI_F32; a.out = ma ? w.Uall : U_save; a.ldo = r; a.alpha = c; a.n_store = r;
    if (!ma) { a.out2 = w.sU; a.ldo2 = r8; a.alpha2 = su; a.n_store2 = r8; }
    QLORA_TRY(launch_gemm("gemm_lora_down", g, a, st));
  }
  if (ma) {
    // each token's own U and its scaled block of sU
    QLORA_TRY(launch("scatter_adapter_u", 0.0, 0.0, st, [&] {
      scatter_adapter_u<<<grid_for(T * r8, 256), 256, 0, st>>>(w.Uall, ma->idx, T, ma->ra, ma->n, r8, ma->sc,
                                                               U_save, w.sU);
    }));
  }
  // Y = [X | sU] [W | B]^T
  if (q && T <= kSmallT) {
    SmallJob j;
    j.src = SRC_NF4_ROWS; j.out = OUT_BF16; j.name = "gemm_nf4_small_fwd";
    j.q = q; j.act = X; j.K0 = k; j.Mw = d;
    j.r = r; j.r8 = r8; j.a1 = w.sU; j.a1_inner = r8; j.a1_ld = r8; j.w1 = Bp;
    j.b16_out = Y; j.ldb = (int)d; j.nb = (int)d;
    return launch_small(j, T, st);
  }
  if (q) return launch_nf4_gemm(false, q, w.scales, X, T, w.sU, r8, r8, Bp, r, r8, Y, st);
  {
    GemmPlan g;
    g.M = (int)T; g.N = (int)d; g.K0 = (int)k; g.K1 = r; g.bn = 256;
    g.a0 = kmajor(X, k, T, k);
    g.b0 = kmajor(W, k, d, k);
    g.a1 = kmajor(w.sU, r8, T, r8);
    g.b1 = kmajor(Bp, r8, d, r8);
    GemmArgs a = blank_args();
    a.epi = EPI_BF16; a.out = Y; a.ldo = d; a.n_store = (int)d;
    QLORA_TRY(launch_gemm("gemm_fwd_main", g, a, st));
  }
  return QLORA_OK;
}

// Backward on a bf16 d x k weight W (plain LoRA) or, when `q` is given, on
// the NF4 weight dequantised inside the dX GEMM (W unused).
int bwd_dx_base(const qlora_nf4_t* q, const uint16_t* W, int64_t d, int64_t k, const uint16_t* A, int r, int r8,
                int rp, const uint16_t* dY, int64_t T, uint16_t* dX, const BwdWs& w, cudaStream_t st,
                bool with_rank);

// With LoRA dropout (`keep` given, c = 1 / (1 - p)), the gradients of the
// forward above: dA = c s G^T (X * keep), dB as without dropout (U_saved is
// the dropped-out U), and the adapter term of dX passes back through the same
// mask, dX = dY W' + keep * (c s G A), added onto the base product by a
// second rank-r GEMM because the mask is elementwise.
int bwd_core(const qlora_nf4_t* q, const uint16_t* W, int64_t d, int64_t k, const uint16_t* A, const uint16_t* B, int r,
             float alpha, const uint16_t* X, const float* U_saved, const uint16_t* dY, int64_t T,
             uint16_t* dX, float* dA, float* dB, const BwdWs& w, cudaStream_t st,
             const uint8_t* keep = nullptr, float c = 1.0f, const MultiAdapter* ma = nullptr) {
  const float s = alpha / (float)r;
  const uint16_t* Xa = X;
  if (keep) {
    QLORA_TRY(launch("apply_keep_bf16", 0.0, (double)T * k * 4.125, st, [&] {
      apply_keep_bf16<<<grid_for(T * k / 8, 256), 256, 0, st>>>(reinterpret_cast<const uint4*>(X), keep, T * k / 8,
                                                                reinterpret_cast<uint4*>(w.Xm));
    }));
    Xa = w.Xm;
  }
  const int r8 = (int)round_up(r, 8);
  const int bnr = bn_for_rank(r);

  int pst = QLORA_OK;
  const uint16_t* Bp = padded_B(B, d, r, r8, w.Bp, st, &pst);
  QLORA_TRY(pst);
  const int rp = w.rp;
  if (T > kSmallT && q) QLORA_TRY(block_scales(q, false, w.scales, st));
  // Few tokens, several adapters, no dropout: G of every adapter in fp32, the
  // token's s_i U and s_i G scattered into its block, then dA (the stack) and
  // dB (side by side) in one CUDA-core kernel; the bf16 s G of the dX
  // extension as before.  With one adapter this is the arithmetic of the
  // single-adapter path below, so both give the same bits.
  if (T <= kSmallT && ma && !keep) {
    SmallJob j;
    j.src = SRC_TMA_MN; j.out = OUT_U; j.name = "gemm_lora_g_small";
    j.w = Bp; j.w_inner = r8; j.w_outer = d; j.w_ld = r8;
    j.act = dY; j.K0 = d; j.Mw = rp;
    j.f32_out = w.Gall; j.ldf = r; j.nf = r; j.nb = 0;
    QLORA_TRY(launch_small(j, T, st));
    QLORA_TRY(launch("scatter_adapter_hilo", 0.0, 0.0, st, [&] {
      scatter_adapter_hilo<<<grid_for(T * rp, 256), 256, 0, st>>>(w.Gall, 0, ma->idx, T, ma->ra, ma->n, rp,
                                                                  ma->sc, w.Gs2);
    }));
    QLORA_TRY(launch("scatter_adapter_f32", 0.0, 0.0, st, [&] {
      scatter_adapter_f32<<<grid_for(T * r, 256), 256, 0, st>>>(U_saved, 1, ma->idx, T, ma->ra, ma->n, ma->sc,
                                                               w.sUf);
    }));
    QLORA_TRY(launch("scatter_adapter_f32", 0.0, 0.0, st, [&] {
      scatter_adapter_f32<<<grid_for(T * r, 256), 256, 0, st>>>(w.Gall, 0, ma->idx, T, ma->ra, ma->n, ma->sc,
                                                               w.sGf);
    }));
    QLORA_TRY(grads_small(X, dY, w.sUf, w.sGf, 1.0f, T, d, k, r, dA, w.dBcat, st));
    QLORA_TRY(launch("uncat_adapters_db", 0.0, 0.0, st, [&] {
      uncat_adapters_db<<<grid_for(d * r, 256), 256, 0, st>>>(w.dBcat, d, ma->ra, ma->n, dB);
    }));
    return bwd_dx_base(q, W, d, k, A, r, r8, rp, dY, T, dX, w, st, true);
  }
  // Few tokens, one adapter, no dropout: G gives s G in fp32 (and the bf16
  // operand of the dX extension), then dA and dB in one CUDA-core kernel.
  if (T <= kSmallT && !ma && !keep) {
    SmallJob j;
    j.src = SRC_TMA_MN; j.out = OUT_U; j.name = "gemm_lora_g_small";
    j.w = Bp; j.w_inner = r8; j.w_outer = d; j.w_ld = r8;
    j.act = dY; j.K0 = d; j.Mw = rp;
    j.f32_out = w.sGf; j.ldf = r; j.nf = r; j.f32_scale = s;
    j.b16_out = w.Gs2; j.ldb = 2 * rp; j.nb = rp; j.scale = s;
    QLORA_TRY(launch_small(j, T, st));
    // dA and dB (which need only G) on a side stream, beside dX
    SideStream* side = side_stream();
    if (side == nullptr) return QLORA_ERR_CUDA;
    if (cudaEventRecord(side->fork, st) != cudaSuccess || cudaStreamWaitEvent(side->st, side->fork, 0) != cudaSuccess)
      return QLORA_ERR_CUDA;
    const int gst = grads_small(X, dY, U_saved, w.sGf, s, T, d, k, r, dA, dB, side->st);
    const int xst = bwd_dx_base(q, W, d, k, A, r, r8, rp, dY, T, dX, w, st, true);
    // join (always, so that a capture in progress stays well formed)
    if (cudaEventRecord(side->join, side->st) != cudaSuccess || cudaStreamWaitEvent(st, side->join, 0) != cudaSuccess)
      return QLORA_ERR_CUDA;
    return gst != QLORA_OK ? gst : xst;
  }
  // Us2 = hi/lo of bf16(s U)
  if (ma) {
    QLORA_TRY(launch("scatter_adapter_hilo", 0.0, 0.0, st, [&] {
      scatter_adapter_hilo<<<grid_for(T * rp, 256), 256, 0, st>>>(U_saved, 1, ma->idx, T, ma->ra, ma->n, rp,
                                                                  ma->sc, w.Us2);
    }));
  } else {
    QLORA_TRY(launch("scale_f32_to_bf16_hilo", 0.0, (double)T * r * 8, st, [&] {
      scale_f32_to_bf16_hilo<<<grid_for(T * rp, 256), 256, 0, st>>>(U_saved, T, r, s, w.Us2, rp);
    }));
  }
  // G = dY B  ->  Gs2 = hi/lo of bf16(s G)
  if (T <= kSmallT) {
    SmallJob j;
    j.src = SRC_TMA_MN; j.out = OUT_HILO; j.name = "gemm_lora_g_small";
    j.w = Bp; j.w_inner = r8; j.w_outer = d; j.w_ld = r8;
    j.act = dY; j.K0 = d; j.Mw = rp;
    j.b16_out = w.Gs2; j.ldb = 2 * rp; j.nb = rp; j.lo_off = rp; j.scale = s;
    if (ma) {
      // every adapter's G in fp32, scattered below
      j.out = OUT_U; j.name = "gemm_lora_g_small";
      j.f32_out = w.Gall; j.ldf = r; j.nf = r; j.nb = 0; j.lo_off = 0;
    }
    QLORA_TRY(launch_small(j, T, st));
  } else {
    GemmPlan g;
    g.M = (int)T; g.N = r; g.K0 = (int)d; g.bn = bnr; g.ksub = kAdapterKSub;
    g.a0 = kmajor(dY, d, T, d);
    g.b0 = mnmajor(Bp, r8, d, r8);
    GemmArgs a = blank_args();
    if (ma) {
      a.epi = EPI_F32; a.out = w.Gall; a.ldo = r; a.n_store = r; a.alpha = 1.0f;
    } else {
      a.epi = EPI_F32; a.out = nullptr; a.n_store = 0;
      a.out2 = w.Gs2; a.ldo2 = 2 * rp; a.alpha2 = s; a.n_store2 = rp; a.lo_offset = rp;
    }
    QLORA_TRY(launch_gemm("gemm_lora_g", g, a, st));
  }
  if (ma) {
    QLORA_TRY(launch("scatter_adapter_hilo", 0.0, 0.0, st, [&] {
      scatter_adapter_hilo<<<grid_for(T * rp, 256), 256, 0, st>>>(w.Gall, 0, ma->idx, T, ma->ra, ma->n, rp,
                                                                  ma->sc, w.Gs2);
    }));
  }
  // dB = dY^T (s U)   (M = d, N = r, K = T); several adapters: every
  // adapter's dB side by side, then split into the stack
  QLORA_TRY(adapter_grad_gemm("gemm_lora_dB", dY, d, T, w.Us2, r, rp, w.halves, w.splitsB,
                              false, ma ? w.dBcat : dB, w.partB, st));
  if (ma) {
    QLORA_TRY(launch("uncat_adapters_db", 0.0, 0.0, st, [&] {
      uncat_adapters_db<<<grid_for(d * r, 256), 256, 0, st>>>(w.dBcat, d, ma->ra, ma->n, dB);
    }));
  }
  // dA^T = X^T (s G)  (M = k, N = r, K = T), stored transposed into dA (r x k)
  QLORA_TRY(adapter_grad_gemm("gemm_lora_dA", Xa, k, T, w.Gs2, r, rp, w.halves, w.splitsA,
                              true, dA, w.partA, st, c));
  if (keep) {
    // dX = dY W' first (no rank-r extension), then += keep * c (s G) A
    QLORA_TRY(bwd_dx_base(q, W, d, k, A, r, r8, rp, dY, T, dX, w, st, false));
    GemmPlan g;
    g.M = (int)T; g.N = (int)k; g.K0 = r; g.bn = 256;
    g.a0 = kmajor(w.Gs2, r, T, 2 * rp);          // hi part of s G
    g.b0 = mnmajor(A, k, r, k);
    GemmArgs a = blank_args();
    a.epi = EPI_DROPOUT; a.out = dX; a.ldo = k; a.n_store = (int)k; a.alpha = c;
    a.keep = keep; a.ldk = k;
    return launch_gemm("gemm_dropout_dx", g, a, st);
  }
  return bwd_dx_base(q, W, d, k, A, r, r8, rp, dY, T, dX, w, st, true);
}

// dX = dY W' (+ (s G) A when `with_rank` is set): the base GEMM of the
// backward, on the NF4 weight or on a bf16 W.
int bwd_dx_base(const qlora_nf4_t* q, const uint16_t* W, int64_t d, int64_t k, const uint16_t* A, int r, int r8,
                int rp, const uint16_t* dY, int64_t T, uint16_t* dX, const BwdWs& w, cudaStream_t st,
                bool with_rank) {
  const int re = with_rank ? r : 0;
  // dX = [dY | sG] [W ; A]   (M = T, N = k, K = d + r)
  if (q && T <= kSmallT) {
    SmallJob j;
    j.src = SRC_NF4_COLS; j.out = OUT_BF16; j.name = "gemm_nf4_small_dx";
    j.q = q; j.act = dY; j.K0 = d; j.Mw = k;
    j.r = re; j.r8 = r8; j.a1 = w.Gs2; j.a1_inner = r; j.a1_ld = 2 * rp; j.w1 = A;
    j.b16_out = dX; j.ldb = (int)k; j.nb = (int)k;
    return launch_small(j, T, st);
  }
  if (q) return launch_nf4_gemm(true, q, w.scales, dY, T, w.Gs2, r, 2 * rp, A, re, r8, dX, st);
  {
    GemmPlan g;
    g.M = (int)T; g.N = (int)k; g.K0 = (int)d; g.K1 = re; g.bn = 256;
    g.a0 = kmajor(dY, d, T, d);
    g.b0 = mnmajor(W, k, d, k);
    g.a1 = kmajor(w.Gs2, r, T, 2 * rp);          // hi part of s G
    g.b1 = mnmajor(A, k, r, k);
    GemmArgs a = blank_args();
    a.epi = EPI_BF16; a.out = dX; a.ldo = k; a.n_store = (int)k;
    QLORA_TRY(launch_gemm("gemm_bwd_dx", g, a, st));
  }
  return QLORA_OK;
}

// Shared argument checks of the two backward entry points (T > 0).
int check_bwd_args(const uint16_t* A, const uint16_t* X, const float* U_saved, const uint16_t* dY,
                   uint16_t* dX, float* dA, float* dB, void* ws, int64_t d, int64_t T) {
  if (!X || !U_saved || !dY || !dX || !ws) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(X) || !aligned16(dY) || !aligned16(dX) || !aligned16(dA) ||
      !aligned16(dB) || !aligned16(U_saved) || !aligned16(ws))
    return QLORA_ERR_MISALIGNED;
  if (T > ((int64_t)1 << 31)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (d % 8 != 0) return QLORA_ERR_UNSUPPORTED_SHAPE;   // dY rows must be 16-byte aligned for TMA
  return QLORA_OK;
}

int zero_adapter_grads(float* dA, float* dB, int64_t d, int64_t k, int r, cudaStream_t st) {
  QLORA_TRY(ensure_device());
  if (cudaMemsetAsync(dA, 0, (size_t)r * k * 4, st) != cudaSuccess) return QLORA_ERR_CUDA;
  if (cudaMemsetAsync(dB, 0, (size_t)d * r * 4, st) != cudaSuccess) return QLORA_ERR_CUDA;
  return QLORA_OK;
}
}  // namespace
}  // namespace qlora

using namespace qlora;

// Scratch of qlora_nf4_quantize_noalloc: room for the fp32 block constants and
// fp64 group sums of QLORA_NOALLOC_MAX_WEIGHTS weights.  In host code this
// name is only a stand-in for the device array; its device address comes from
// cudaGetSymbolAddress, once per device.
static constexpr size_t kNoallocScratchBytes =
    (size_t)(QLORA_NOALLOC_MAX_WEIGHTS / 16) + (size_t)(QLORA_NOALLOC_MAX_WEIGHTS / 2048) + 256;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

namespace {
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[64] = {nullptr};
unsigned long long g_noalloc_ctx[64] = {0};

// Device address of g_noalloc_scratch on the current device: looked up on the
// first call per device (with that device current) and cached together with
// the id of the context it belongs to; a call in another context (after a
// device reset) looks it up again instead of using a stale address.
int noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return QLORA_ERR_NO_DEVICE;
  const unsigned long long ctx = current_ctx_id();
  if (ctx == 0) return QLORA_ERR_NO_DEVICE;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (g_noalloc_ptr[dev] == nullptr || g_noalloc_ctx[dev] != ctx) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return QLORA_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = ctx;
  }
  *out = g_noalloc_ptr[dev];
  return QLORA_OK;
}
}  // namespace

// =====================================================================
// C ABI
// =====================================================================
namespace {
// NCCL entry points, resolved from libnccl.so.2 at the first use (a process
// that already loaded NCCL, such as one running torch.distributed, gets that
// copy).
struct NcclApi {
  bool ok = false;
  decltype(&ncclGetUniqueId) get_unique_id = nullptr;
  decltype(&ncclCommInitRank) comm_init_rank = nullptr;
  decltype(&ncclCommDestroy) comm_destroy = nullptr;
  decltype(&ncclAllReduce) all_reduce = nullptr;
  decltype(&ncclGroupStart) group_start = nullptr;
  decltype(&ncclGroupEnd) group_end = nullptr;
};
NcclApi load_nccl() {
  NcclApi a;
  void* h = dlopen("libnccl.so.2", RTLD_NOW | RTLD_GLOBAL);
  if (h == nullptr) return a;
  a.get_unique_id = reinterpret_cast<decltype(a.get_unique_id)>(dlsym(h, "ncclGetUniqueId"));
  a.comm_init_rank = reinterpret_cast<decltype(a.comm_init_rank)>(dlsym(h, "ncclCommInitRank"));
  a.comm_destroy = reinterpret_cast<decltype(a.comm_destroy)>(dlsym(h, "ncclCommDestroy"));
  a.all_reduce = reinterpret_cast<decltype(a.all_reduce)>(dlsym(h, "ncclAllReduce"));
  a.group_start = reinterpret_cast<decltype(a.group_start)>(dlsym(h, "ncclGroupStart"));
  a.group_end = reinterpret_cast<decltype(a.group_end)>(dlsym(h, "ncclGroupEnd"));
  a.ok = a.get_unique_id && a.comm_init_rank && a.comm_destroy && a.all_reduce && a.group_start && a.group_end;
  return a;
}
const NcclApi& nccl_api() {
  static const NcclApi api = load_nccl();
  return api;
}
}  // namespace

extern "C" {

const char* qlora_strerror(int s) {
  switch (s) {
    case QLORA_OK: return "ok";
    case QLORA_ERR_INVALID_ARG: return "invalid argument";
    case QLORA_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
    case QLORA_ERR_MISALIGNED: return "pointer or leading dimension not 16-byte aligned";
    case QLORA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case QLORA_ERR_CUDA: return "CUDA error";
    case QLORA_ERR_TIMEOUT: return "device wait timed out";
    case QLORA_ERR_NO_DEVICE: return "no sm_100 device is current";
    case QLORA_ERR_EXCEEDS_STATIC_SCRATCH:
      return "d*k exceeds the static scratch of qlora_nf4_quantize_noalloc (2^28 weights)";
    case QLORA_ERR_NCCL: return "NCCL unavailable or an NCCL call failed";
    default: return "unknown status";
  }
}

int qlora_version(void) { return 100; }

// ------------------------------------------------------------ data parallel

int qlora_comm_unique_id(uint8_t* id) {
  if (id == nullptr) return QLORA_ERR_INVALID_ARG;
  const NcclApi& n = nccl_api();
  if (!n.ok) return QLORA_ERR_NCCL;
  ncclUniqueId u;
  if (n.get_unique_id(&u) != ncclSuccess) return QLORA_ERR_NCCL;
  static_assert(sizeof(u.internal) == QLORA_NCCL_ID_BYTES, "NCCL unique id size");
  memcpy(id, u.internal, QLORA_NCCL_ID_BYTES);
  return QLORA_OK;
}

int qlora_comm_init(const uint8_t* id, int nranks, int rank, void** comm) {
  if (id == nullptr || comm == nullptr || nranks < 1 || rank < 0 || rank >= nranks) return QLORA_ERR_INVALID_ARG;
  *comm = nullptr;
  const NcclApi& n = nccl_api();
  if (!n.ok) return QLORA_ERR_NCCL;
  ncclUniqueId u;
  memcpy(u.internal, id, QLORA_NCCL_ID_BYTES);
  ncclComm_t c = nullptr;
  if (n.comm_init_rank(&c, nranks, u, rank) != ncclSuccess) return QLORA_ERR_NCCL;
  *comm = c;
  return QLORA_OK;
}

int qlora_comm_destroy(void* comm) {
  if (comm == nullptr) return QLORA_ERR_INVALID_ARG;
  const NcclApi& n = nccl_api();
  if (!n.ok) return QLORA_ERR_NCCL;
  return n.comm_destroy(static_cast<ncclComm_t>(comm)) == ncclSuccess ? QLORA_OK : QLORA_ERR_NCCL;
}

int qlora_grad_allreduce(void* comm, float* dA, int64_t nA, float* dB, int64_t nB, qlora_stream_t stream) {
  if (comm == nullptr || nA < 0 || nB < 0 || (nA > 0 && dA == nullptr) || (nB > 0 && dB == nullptr))
    return QLORA_ERR_INVALID_ARG;
  const NcclApi& n = nccl_api();
  if (!n.ok) return QLORA_ERR_NCCL;
  const ncclComm_t c = static_cast<ncclComm_t>(comm);
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (n.group_start() != ncclSuccess) return QLORA_ERR_NCCL;
  ncclResult_t r = ncclSuccess;
  if (nA > 0) r = n.all_reduce(dA, dA, (size_t)nA, ncclFloat32, ncclSum, c, st);
  if (r == ncclSuccess && nB > 0) r = n.all_reduce(dB, dB, (size_t)nB, ncclFloat32, ncclSum, c, st);
  const ncclResult_t e = n.group_end();
  return (r == ncclSuccess && e == ncclSuccess) ? QLORA_OK : QLORA_ERR_NCCL;
}

int qlora_nf4_levels(float* levels16, float* thresholds15) {
  const auto& T = tables();
  if (levels16) memcpy(levels16, T.levels, sizeof(T.levels));
  if (thresholds15) memcpy(thresholds15, T.thresholds, sizeof(T.thresholds));
  return QLORA_OK;
}

int64_t qlora_launch_count(void) { return g_launches.load(); }

int qlora_set_nf4_gemm_mode(int mode) {
  if (mode < 0 || mode > 2) return QLORA_ERR_INVALID_ARG;
  g_nf4_gemm_mode.store(mode);
  return QLORA_OK;
}

size_t qlora_quantize_workspace_bytes(int64_t d, int64_t k) {
  if (d < 1 || k < 1) return 0;
  const int64_t n_b = d * k / kBlock;
  const int64_t n_g = cdiv(n_b, kBlock2);
  return (size_t)(round_up(n_b * 4, 256) + round_up(n_g * 8, 256) + 256);
}

int qlora_nf4_quantize(const float* W0, int64_t d, int64_t k, int block, qlora_nf4_t* out,
                       void* ws, size_t ws_bytes, qlora_stream_t stream) {
  if (!W0 || !out || !out->codes || !out->absmax_q || !out->scale2 || !out->mean)
    return QLORA_ERR_INVALID_ARG;
  if (block != kBlock) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (d < 1 || k < 64 || k % 64 != 0 || d * k >= ((int64_t)1 << 34)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(W0) || !aligned16(out->codes)) return QLORA_ERR_MISALIGNED;
  if (!ws || ws_bytes < qlora_quantize_workspace_bytes(d, k)) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  QLORA_TRY(ensure_device());
  out->d = d; out->k = k; out->block = kBlock; out->block2 = kBlock2;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int64_t n_b = d * k / kBlock;
  const int64_t n_g = cdiv(n_b, kBlock2);
  Carver c{reinterpret_cast<uint8_t*>(ws)};
  float* absmax = (float*)c.take((size_t)(n_b * 4));
  double* gsum = (double*)c.take((size_t)(n_g * 8));
  unsigned int* ticket = (unsigned int*)c.take(4);
  const auto& T = tables();
  const double bytes1 = (double)d * k * 4.5 + (double)n_b * 4;
  if (cudaMemsetAsync(ticket, 0, sizeof(unsigned int), st) != cudaSuccess) return QLORA_ERR_CUDA;
  QLORA_TRY(launch("nf4_quantize_phase1", 0.0, bytes1, st, [&] {
    nf4_quantize_phase1<<<(unsigned)std::min<int64_t>(n_g, 4 * (int64_t)current_sms()), 256, 0, st>>>(
        W0, n_b, n_g, reinterpret_cast<uint32_t*>(out->codes), absmax, gsum, ticket, out->mean, T.enc);
  }));
  QLORA_TRY(launch("nf4_quantize_dq", 0.0, (double)n_b * 5 + n_g * 4, st, [&] {
    nf4_quantize_dq<<<(unsigned)cdiv(n_g, kDqGroups), 256, 0, st>>>(absmax, n_g, n_b, out->mean,
                                                                   out->absmax_q, out->scale2);
  }));
  return QLORA_OK;
}

int qlora_nf4_quantize_noalloc(const float* W0, int64_t d, int64_t k, int block, qlora_nf4_t* out,
                               qlora_stream_t stream) {
  if (d >= 1 && k >= 1 && d * k > QLORA_NOALLOC_MAX_WEIGHTS) return QLORA_ERR_EXCEEDS_STATIC_SCRATCH;
  QLORA_TRY(ensure_device());
  void* scratch = nullptr;
  QLORA_TRY(noalloc_scratch(&scratch));
  return qlora_nf4_quantize(W0, d, k, block, out, scratch, kNoallocScratchBytes, stream);
}

int qlora_nf4_dequantize(const qlora_nf4_t* q, uint16_t* W_out, qlora_stream_t stream) {
  QLORA_TRY(check_nf4(q));
  if (!W_out) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(W_out)) return QLORA_ERR_MISALIGNED;
  QLORA_TRY(ensure_device());
  return dequantize_into(q, W_out, reinterpret_cast<cudaStream_t>(stream));
}

size_t qlora_fwd_workspace_bytes(int64_t d, int64_t k, int r, int64_t T) {
  if (d < 1 || k < 1 || r < 1 || T < 0) return 0;
  return carve_fwd(nullptr, d, k, r, T).bytes;
}


int qlora_fwd(const qlora_nf4_t* q, const uint16_t* A, const uint16_t* B, int r, float alpha,
              const uint16_t* X, int64_t T, uint16_t* Y, float* U_save, void* ws, size_t ws_bytes,
              qlora_stream_t stream) {
  QLORA_TRY(check_nf4(q));
  QLORA_TRY(check_rank(r, alpha));
  if (T < 0) return QLORA_ERR_INVALID_ARG;
  if (T == 0) return QLORA_OK;
  if (!A || !B || !X || !Y || !U_save || !ws) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(X) || !aligned16(Y) || !aligned16(U_save) || !aligned16(ws))
    return QLORA_ERR_MISALIGNED;
  const int64_t d = q->d, k = q->k;
  if (T > ((int64_t)1 << 31)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  FwdWs w = carve_fwd(ws, d, k, r, T);
  if (ws_bytes < w.bytes) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  QLORA_TRY(ensure_device());
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return fwd_core(q, nullptr, d, k, A, B, r, alpha, X, T, Y, U_save, w, st);
}

size_t lora_fwd_workspace_bytes(int64_t d, int64_t k, int r, int64_t T) {
  if (d < 1 || k < 1 || r < 1 || T < 0) return 0;
  return carve_fwd(nullptr, d, k, r, T).bytes;
}

int lora_fwd(const uint16_t* W, int64_t d, int64_t k, const uint16_t* A, const uint16_t* B, int r,
             float alpha, const uint16_t* X, int64_t T, uint16_t* Y, float* U_save, void* ws,
             size_t ws_bytes, qlora_stream_t stream) {
  QLORA_TRY(check_rank(r, alpha));
  if (d < 1 || k < 1 || T < 0) return QLORA_ERR_INVALID_ARG;
  if (T == 0) return QLORA_OK;
  if (!W || !A || !B || !X || !Y || !U_save || !ws) return QLORA_ERR_INVALID_ARG;
  if (k % 8 != 0 || d > ((int64_t)1 << 31) || k > ((int64_t)1 << 31) || T > ((int64_t)1 << 31))
    return QLORA_ERR_UNSUPPORTED_SHAPE;
  if (!aligned16(W) || !aligned16(A) || !aligned16(X) || !aligned16(Y) || !aligned16(U_save) ||
      !aligned16(ws))
    return QLORA_ERR_MISALIGNED;
  FwdWs w = carve_fwd(ws, d, k, r, T);
  if (ws_bytes < w.bytes) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  QLORA_TRY(ensure_device());
  return fwd_core(nullptr, W, d, k, A, B, r, alpha, X, T, Y, U_save, w, reinterpret_cast<cudaStream_t>(stream));
}

size_t qlora_bwd_workspace_bytes(int64_t d, int64_t k, int r, int64_t T) {
  if (d < 1 || k < 1 || r < 1 || T < 0) return 0;
  return carve_bwd(nullptr, d, k, r, T).bytes;
}


int qlora_bwd(const qlora_nf4_t* q, const uint16_t* A, const uint16_t* B, int r, float alpha,
              const uint16_t* X, const float* U_saved, const uint16_t* dY, int64_t T, uint16_t* dX,
              float* dA, float* dB, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  QLORA_TRY(check_nf4(q));
  QLORA_TRY(check_rank(r, alpha));
  if (T < 0) return QLORA_ERR_INVALID_ARG;
  if (!A || !B || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  const int64_t d = q->d, k = q->k;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) return zero_adapter_grads(dA, dB, d, k, r, st);
  QLORA_TRY(check_bwd_args(A, X, U_saved, dY, dX, dA, dB, ws, d, T));
  BwdWs w = carve_bwd(ws, d, k, r, T);
  if (ws_bytes < w.bytes) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  QLORA_TRY(ensure_device());
  return bwd_core(q, nullptr, d, k, A, B, r, alpha, X, U_saved, dY, T, dX, dA, dB, w, st);
}

// Several adapters: host-side checks and the stack descriptor.
static int make_multi(int n, int r, const float* alphas, const int32_t* idx, MultiAdapter* ma) {
  if (n < 1 || n > kMaxAdapters || !alphas || !idx) return QLORA_ERR_INVALID_ARG;
  if (r < 1 || (int64_t)n * r > 256) return QLORA_ERR_UNSUPPORTED_SHAPE;
  ma->n = n;
  ma->ra = r;
  ma->idx = idx;
  memset(&ma->sc, 0, sizeof(ma->sc));
  for (int i = 0; i < n; ++i) {
    if (!(alphas[i] > 0.0f) || !std::isfinite(alphas[i])) return QLORA_ERR_INVALID_ARG;
    ma->sc.s[i] = alphas[i] / (float)r;
  }
  return QLORA_OK;
}

size_t qlora_fwd_multi_workspace_bytes(int64_t d, int64_t k, int n, int r, int64_t T) {
  if (d < 1 || k < 1 || n < 1 || r < 1 || T < 0) return 0;
  return carve_fwd(nullptr, d, k, n * r, T, false, true).bytes;
}

int qlora_fwd_multi(const qlora_nf4_t* q, int n, const uint16_t* As, const uint16_t* Bs, int r,
                    const float* alphas, const int32_t* idx, const uint16_t* X, int64_t T, uint16_t* Y,
                    float* U_save, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  QLORA_TRY(check_nf4(q));
  MultiAdapter ma;
  QLORA_TRY(make_multi(n, r, alphas, idx, &ma));
  if (T < 0) return QLORA_ERR_INVALID_ARG;
  if (T == 0) return QLORA_OK;
  if (!As || !Bs || !X || !Y || !U_save || !ws) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(As) || !aligned16(X) || !aligned16(Y) || !aligned16(U_save) || !aligned16(ws) ||
      (reinterpret_cast<uintptr_t>(idx) & 3u) != 0)
    return QLORA_ERR_MISALIGNED;
  const int64_t d = q->d, k = q->k;
  if (T > ((int64_t)1 << 31)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  const int R = n * r;
  FwdWs w = carve_fwd(ws, d, k, R, T, false, true);
  if (ws_bytes < w.bytes) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  QLORA_TRY(ensure_device());
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  QLORA_TRY(launch("cat_adapters_b", 0.0, 0.0, st, [&] {
    cat_adapters_b<<<grid_for(d * R, 256), 256, 0, st>>>(Bs, d, r, n, w.Bcat);
  }));
  // alpha only sets s = alpha / R, which the stack path does not use
  return fwd_core(q, nullptr, d, k, As, w.Bcat, R, (float)R, X, T, Y, U_save, w, st, nullptr, 1.0f, &ma);
}

size_t qlora_bwd_multi_workspace_bytes(int64_t d, int64_t k, int n, int r, int64_t T) {
  if (d < 1 || k < 1 || n < 1 || r < 1 || T < 0) return 0;
  return carve_bwd(nullptr, d, k, n * r, T, false, true).bytes;
}

int qlora_bwd_multi(const qlora_nf4_t* q, int n, const uint16_t* As, const uint16_t* Bs, int r,
                    const float* alphas, const int32_t* idx, const uint16_t* X, const float* U_saved,
                    const uint16_t* dY, int64_t T, uint16_t* dX, float* dAs, float* dBs, void* ws,
                    size_t ws_bytes, qlora_stream_t stream) {
  QLORA_TRY(check_nf4(q));
  MultiAdapter ma;
  QLORA_TRY(make_multi(n, r, alphas, idx, &ma));
  if (T < 0) return QLORA_ERR_INVALID_ARG;
  if (!As || !Bs || !dAs || !dBs) return QLORA_ERR_INVALID_ARG;
  const int64_t d = q->d, k = q->k;
  const int R = n * r;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) return zero_adapter_grads(dAs, dBs, d, k, R, st);
  QLORA_TRY(check_bwd_args(As, X, U_saved, dY, dX, dAs, dBs, ws, d, T));
  if ((reinterpret_cast<uintptr_t>(idx) & 3u) != 0) return QLORA_ERR_MISALIGNED;
  BwdWs w = carve_bwd(ws, d, k, R, T, false, true);
  if (ws_bytes < w.bytes) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  QLORA_TRY(ensure_device());
  QLORA_TRY(launch("cat_adapters_b", 0.0, 0.0, st, [&] {
    cat_adapters_b<<<grid_for(d * R, 256), 256, 0, st>>>(Bs, d, r, n, w.Bcat);
  }));
  return bwd_core(q, nullptr, d, k, As, w.Bcat, R, (float)R, X, U_saved, dY, T, dX, dAs, dBs, w, st, nullptr,
                  1.0f, &ma);
}

static int check_dropout(const uint8_t* keep, float p) {
  if (!(p >= 0.0f && p < 1.0f)) return QLORA_ERR_INVALID_ARG;
  if (p > 0.0f && !keep) return QLORA_ERR_INVALID_ARG;
  if (p > 0.0f && !aligned16(keep)) return QLORA_ERR_MISALIGNED;
  return QLORA_OK;
}

// c = fp32(1 / (1 - p)), the inverted-dropout scale of the kept elements
static float dropout_scale(float p) { return (float)(1.0 / (1.0 - (double)p)); }

size_t qlora_fwd_dropout_workspace_bytes(int64_t d, int64_t k, int r, int64_t T) {
  if (d < 1 || k < 1 || r < 1 || T < 0) return 0;
  return carve_fwd(nullptr, d, k, r, T, true).bytes;
}

int qlora_fwd_dropout(const qlora_nf4_t* q, const uint16_t* A, const uint16_t* B, int r, float alpha,
                      const uint16_t* X, const uint8_t* keep, float p, int64_t T, uint16_t* Y, float* U_save,
                      void* ws, size_t ws_bytes, qlora_stream_t stream) {
  QLORA_TRY(check_dropout(keep, p));
  if (p == 0.0f) return qlora_fwd(q, A, B, r, alpha, X, T, Y, U_save, ws, ws_bytes, stream);
  QLORA_TRY(check_nf4(q));
  QLORA_TRY(check_rank(r, alpha));
  if (T < 0) return QLORA_ERR_INVALID_ARG;
  if (T == 0) return QLORA_OK;
  if (!A || !B || !X || !Y || !U_save || !ws) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(X) || !aligned16(Y) || !aligned16(U_save) || !aligned16(ws))
    return QLORA_ERR_MISALIGNED;
  const int64_t d = q->d, k = q->k;
  if (T > ((int64_t)1 << 31)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  FwdWs w = carve_fwd(ws, d, k, r, T, true);
  if (ws_bytes < w.bytes) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  QLORA_TRY(ensure_device());
  return fwd_core(q, nullptr, d, k, A, B, r, alpha, X, T, Y, U_save, w, reinterpret_cast<cudaStream_t>(stream),
                  keep, dropout_scale(p));
}

size_t qlora_bwd_dropout_workspace_bytes(int64_t d, int64_t k, int r, int64_t T) {
  if (d < 1 || k < 1 || r < 1 || T < 0) return 0;
  return carve_bwd(nullptr, d, k, r, T, true).bytes;
}

int qlora_bwd_dropout(const qlora_nf4_t* q, const uint16_t* A, const uint16_t* B, int r, float alpha,
                      const uint16_t* X, const uint8_t* keep, float p, const float* U_saved, const uint16_t* dY,
                      int64_t T, uint16_t* dX, float* dA, float* dB, void* ws, size_t ws_bytes,
                      qlora_stream_t stream) {
  QLORA_TRY(check_dropout(keep, p));
  if (p == 0.0f) return qlora_bwd(q, A, B, r, alpha, X, U_saved, dY, T, dX, dA, dB, ws, ws_bytes, stream);
  QLORA_TRY(check_nf4(q));
  QLORA_TRY(check_rank(r, alpha));
  if (T < 0) return QLORA_ERR_INVALID_ARG;
  if (!A || !B || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  const int64_t d = q->d, k = q->k;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) return zero_adapter_grads(dA, dB, d, k, r, st);
  QLORA_TRY(check_bwd_args(A, X, U_saved, dY, dX, dA, dB, ws, d, T));
  BwdWs w = carve_bwd(ws, d, k, r, T, true);
  if (ws_bytes < w.bytes) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  QLORA_TRY(ensure_device());
  return bwd_core(q, nullptr, d, k, A, B, r, alpha, X, U_saved, dY, T, dX, dA, dB, w, st, keep, dropout_scale(p));
}

size_t lora_bwd_workspace_bytes(int64_t d, int64_t k, int r, int64_t T) {
  if (d < 1 || k < 1 || r < 1 || T < 0) return 0;
  return carve_bwd(nullptr, d, k, r, T).bytes;
}

int lora_bwd(const uint16_t* W, int64_t d, int64_t k, const uint16_t* A, const uint16_t* B, int r,
             float alpha, const uint16_t* X, const float* U_saved, const uint16_t* dY, int64_t T,
             uint16_t* dX, float* dA, float* dB, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  QLORA_TRY(check_rank(r, alpha));
  if (d < 1 || k < 1 || T < 0) return QLORA_ERR_INVALID_ARG;
  if (!W || !A || !B || !dA || !dB) return QLORA_ERR_INVALID_ARG;
  if (k % 8 != 0 || d > ((int64_t)1 << 31) || k > ((int64_t)1 << 31)) return QLORA_ERR_UNSUPPORTED_SHAPE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (T == 0) return zero_adapter_grads(dA, dB, d, k, r, st);
  if (!aligned16(W)) return QLORA_ERR_MISALIGNED;
  QLORA_TRY(check_bwd_args(A, X, U_saved, dY, dX, dA, dB, ws, d, T));
  BwdWs w = carve_bwd(ws, d, k, r, T);
  if (ws_bytes < w.bytes) return QLORA_ERR_WORKSPACE_TOO_SMALL;
  QLORA_TRY(ensure_device());
  return bwd_core(nullptr, W, d, k, A, B, r, alpha, X, U_saved, dY, T, dX, dA, dB, w, st);
}

size_t lora_merge_workspace_bytes(int64_t d, int64_t k, int r) {
  if (d < 1 || k < 1 || r < 1) return 0;
  return (size_t)round_up(d * round_up(r, 8) * 2, 256);
}

static int merge_common(const qlora_nf4_t* q, const uint16_t* W, const uint16_t* A, const uint16_t* B,
                        int r, float alpha, int64_t d, int64_t k, uint16_t* out, void* ws,
                        size_t ws_bytes, cudaStream_t st, bool merge) {
  if (!A || !B || !out) return QLORA_ERR_INVALID_ARG;
  if (!aligned16(A) || !aligned16(out) || (W && !aligned16(W))) return QLORA_ERR_MISALIGNED;
  const int r8 = (int)round_up(r, 8);
  if (r8 != r && (!ws || ws_bytes < lora_merge_workspace_bytes(d, k, r)))
    return QLORA_ERR_WORKSPACE_TOO_SMALL;
  if (r8 != r && !aligned16(ws)) return QLORA_ERR_MISALIGNED;
  QLORA_TRY(ensure_device());
  const float s = alpha / (float)r;
  int pst = QLORA_OK;
  const uint16_t* Bp = padded_B(B, d, r, r8, reinterpret_cast<uint16_t*>(ws), st, &pst);
  QLORA_TRY(pst);
  if (r <= 128) return launch_deploy(merge, q, W, A, Bp, r, r8, d, k, s, out, st);
  GemmPlan g;
  g.M = (int)d; g.N = (int)k; g.K0 = r; g.bn = 256;
  g.a0 = kmajor(Bp, r8, d, r8);
  g.b0 = mnmajor(A, k, r, k);
  GemmArgs a = blank_args();
  a.out = out; a.ldo = k; a.n_store = (int)k;
  if (merge) {
    a.epi = EPI_MERGE; a.alpha = s;
    a.codes = q->codes; a.absmax_q = q->absmax_q; a.scale2 = q->scale2; a.mean = q->mean;
  } else {
    a.epi = EPI_UNMERGE; a.alpha = -s; a.w_in = W; a.ldw = k;
  }
  return launch_gemm(merge ? "lora_merge" : "lora_unmerge", g, a, st);
}

int lora_merge(const qlora_nf4_t* q, const uint16_t* A, const uint16_t* B, int r, float alpha,
               uint16_t* W_out, void* ws, size_t ws_bytes, qlora_stream_t stream) {
  QLORA_TRY(check_nf4(q));
  QLORA_TRY(check_rank(r, alpha));
  return merge_common(q, nullptr, A, B, r, alpha, q->d, q->k, W_out, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream), true);
}

int lora_adam_step(float* master, uint16_t* weight_bf16, float* m, float* v, const float* grad, int64_t n,
                   int64_t step, float lr, float beta1, float beta2, float eps, float weight_decay,
                   qlora_stream_t stream) {
  if (!master || !weight_bf16 || !m || !v || !grad || n < 0 || step < 1) return QLORA_ERR_INVALID_ARG;
  if (!(lr >= 0.f) || !(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f) || !(eps >= 0.f) ||
      !(weight_decay >= 0.f))
    return QLORA_ERR_INVALID_ARG;
  if (!aligned16(master) || !aligned16(weight_bf16) || !aligned16(m) || !aligned16(v) || !aligned16(grad))
    return QLORA_ERR_MISALIGNED;
  if (n == 0) return QLORA_OK;
  QLORA_TRY(ensure_device());
  AdamArgs a;
  a.lr = lr; a.beta1 = beta1; a.beta2 = beta2;
  a.omb1 = (float)(1.0 - (double)beta1);
  a.omb2 = (float)(1.0 - (double)beta2);
  a.c1 = (float)(1.0 / (1.0 - std::pow((double)beta1, (double)step)));
  a.c2 = (float)(1.0 / (1.0 - std::pow((double)beta2, (double)step)));
  a.eps = eps; a.wd = weight_decay;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return launch("lora_adam_step", 0.0, 30.0 * (double)n, st, [&] {
    adam_step_kernel<<<grid_for(cdiv(n, 4), 256), 256, 0, st>>>(master, weight_bf16, m, v, grad, n, a);
  });
}

int lora_unmerge(const uint16_t* W, const uint16_t* A, const uint16_t* B, int r, float alpha,
                 int64_t d, int64_t k, uint16_t* W0_out, void* ws, size_t ws_bytes,
                 qlora_stream_t stream) {
  QLORA_TRY(check_rank(r, alpha));
  if (!W) return QLORA_ERR_INVALID_ARG;
  if (d < 1 || k < 64 || k % 64 != 0 || d > ((int64_t)1 << 31) || k > ((int64_t)1 << 31))
    return QLORA_ERR_UNSUPPORTED_SHAPE;
  return merge_common(nullptr, W, A, B, r, alpha, d, k, W0_out, ws, ws_bytes,
                      reinterpret_cast<cudaStream_t>(stream), false);
}

int qlora_get_device_status(qlora_stream_t stream, int* status) {
  if (!status) return QLORA_ERR_INVALID_ARG;
  QLORA_TRY(ensure_device());
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return QLORA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_status, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_status, &zero, sizeof(int)) != cudaSuccess) return QLORA_ERR_CUDA;
  *status = v;
  return QLORA_OK;
}

int qlora_selftest_wait_timeout(int limit_us, qlora_stream_t stream) {
  if (limit_us < 1 || limit_us > 2000000) return QLORA_ERR_INVALID_ARG;
  QLORA_TRY(ensure_device());
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  return launch("selftest_wait", 0.0, 0.0, st, [&] {
    selftest_wait_kernel<<<1, 32, 0, st>>>((unsigned long long)limit_us * 1000ull);
  });
}

int qlora_profile_begin(void) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  for (auto& r : g_prof) {
    g_event_pool.push_back(r.start);
    g_event_pool.push_back(r.stop);
  }
  g_prof.clear();
  g_prof_on = true;
  return QLORA_OK;
}

int qlora_profile_end(qlora_kernel_stat_t* out, int capacity, int* n_out) {
  std::lock_guard<std::mutex> lk(g_prof_mu);
  g_prof_on = false;
  std::vector<qlora_kernel_stat_t> agg;
  int status = QLORA_OK;
  for (auto& r : g_prof) {
    if (cudaEventSynchronize(r.stop) != cudaSuccess) { status = QLORA_ERR_CUDA; continue; }
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.start, r.stop) != cudaSuccess) { status = QLORA_ERR_CUDA; continue; }
    qlora_kernel_stat_t* slot = nullptr;
    for (auto& a : agg)
      if (strncmp(a.name, r.name.c_str(), sizeof(a.name)) == 0) slot = &a;
    if (!slot) {
      qlora_kernel_stat_t z;
      memset(&z, 0, sizeof(z));
      strncpy(z.name, r.name.c_str(), sizeof(z.name) - 1);
      agg.push_back(z);
      slot = &agg.back();
    }
    slot->launches += 1;
    slot->total_ms += ms;
    slot->flops += r.flops;
    slot->bytes += r.bytes;
  }
  for (auto& r : g_prof) {
    g_event_pool.push_back(r.start);
    g_event_pool.push_back(r.stop);
  }
  g_prof.clear();
  const int n = (int)agg.size();
  if (n_out) *n_out = n;
  if (out)
    for (int i = 0; i < n && i < capacity; ++i) out[i] = agg[i];
  return status;
}

}  // extern "C"
