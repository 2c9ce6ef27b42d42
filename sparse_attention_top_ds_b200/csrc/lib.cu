// lib.cu -- the C ABI of libdstopk.so (declared in include/ds_topk.h):
// argument checks, launch-shape choice and kernel launches.  One translation
// unit holds every kernel, so device symbols (the status word) resolve here.
#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "../../include/ds_topk.h"
#include "ptx.cuh"
#include "topk_kernel.cuh"
#include "topk_stash_kernel.cuh"
#include "indexer_kernel.cuh"
#include "attention_kernel.cuh"
#include "qproj_kernel.cuh"
#include "compress_kernel.cuh"

namespace dstopk {

// Per-device status word: kernels record the first device-side error here.
static __device__ int g_status;

constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  bool supported = false;
  int num_sms = 0;
  int* status = nullptr;     // device address of g_status on this device
  void* scratch = nullptr;   // grow-only scratch: [B, S] score rows of the indexer paths
  size_t scratch_bytes = 0;
  void* sel_state = nullptr;  // indexer + top-k: key histograms of the rows (zero between calls)
  size_t sel_state_bytes = 0;
  void* attn_scratch = nullptr;  // sparse attention: per-chunk partial results, grow-only
  size_t attn_scratch_bytes = 0;
};

static std::mutex g_mu;
static DeviceState g_dev[kMaxDevices];

// Limit of the kernels' bounded waits, in ns (0: kWaitLimitNs), read at each
// launch; and the number of scorer launches still to carry the planted fault
// that makes one of their waits run out (testing the failure detection).
static std::atomic<long long> g_wait_ns{0};
static std::atomic<int> g_planted{0};

static uint64_t wait_limit() { return (uint64_t)g_wait_ns.load(std::memory_order_relaxed); }

static int take_planted_fault() {
  int n = g_planted.load(std::memory_order_relaxed);
  while (n > 0 && !g_planted.compare_exchange_weak(n, n - 1, std::memory_order_relaxed)) {
  }
  return n > 0 ? 1 : 0;
}

static cudaError_t indexer_setup();
template <int NT>
static cudaError_t set_stash_smem(int bytes) {
  cudaError_t e = cudaFuncSetAttribute(topk_stash_kernel<F32Keys, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(topk_stash_kernel<BF16Keys, NT>, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  return e;
}
static bool topk_cluster16_ok();
static int g_max_cluster = 8;  // largest cluster the top-k launch may use

// Launch attribute: the kernel may start while the previous kernel on the
// stream finishes (every kernel launched with it waits, with griddepcontrol,
// before it touches global memory).  DS_NO_PDL=1 turns it off (comparisons).
static bool pdl_on() {
  static const bool on = getenv("DS_NO_PDL") == nullptr;
  return on;
}
static void set_pdl(cudaLaunchAttribute& a) {
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
}

// Set-up once per device, with that device current: capability check, the
// status word's address, and the kernels' shared-memory limits.
static int device_state(DeviceState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  DeviceState& s = g_dev[dev];
  if (!s.ready) {
    int major = 0, sms = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return DS_ERR_CUDA;
    if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return DS_ERR_CUDA;
    s.supported = (major == 10);
    s.num_sms = sms;
    if (s.supported) {
      if (cudaGetSymbolAddress(reinterpret_cast<void**>(&s.status), g_status) != cudaSuccess) return DS_ERR_CUDA;
      const int smem_max = 227 * 1024;
      cudaError_t e = cudaSuccess;
      e = cudaFuncSetAttribute(topk_cluster_kernel<F32Keys, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(topk_cluster_kernel<F32Keys, 512>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(topk_cluster_kernel<BF16Keys, 256>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max);
      if (e == cudaSuccess)
        e = cudaFuncSetAttribute(topk_cluster_kernel<BF16Keys, 512>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem_max);
      if (e == cudaSuccess) e = set_stash_smem<kTsThreads>(smem_max);
      if (e == cudaSuccess) e = indexer_setup();
      if (e != cudaSuccess) return DS_ERR_CUDA;
      g_max_cluster = topk_cluster16_ok() ? 16 : 8;
    }
    s.ready = true;
  }
  if (!s.supported) return DS_ERR_UNSUPPORTED;
  *out = &s;
  return DS_OK;
}

// ------------------------------------------------------------------ top-k

struct TopkShape {
  int cluster;   // CTAs per row
  int slice;     // elements per CTA
  int threads;   // threads per CTA
};

// Launch shape: a cluster of C CTAs per row (C <= 8, or 16 where the device
// allows non-portable clusters), enough CTAs to fill every SM several times
// over, but no slice below 1024 scores.  Shared memory does not hold the
// scores, so the slice size is free.
constexpr int kMaxRowElems = 1 << 24;

static bool choose_topk_shape(int batch, int n, int num_sms, TopkShape* out) {
  if (n > kMaxRowElems) return false;
  int C = 1;
  const long target = 4L * num_sms;
  const char* force = getenv("DS_TOPK_CLUSTER");  // tuning sweeps only
  if (force) {
    C = atoi(force);
    if (C != 1 && C != 2 && C != 4 && C != 8 && C != 16) C = 8;
    if (C > g_max_cluster) C = g_max_cluster;
  } else {
    const int cmax = batch >= 8 ? min(8, g_max_cluster) : g_max_cluster;
    while (C < cmax && (long)batch * C < target && (n + 2 * C - 1) / (2 * C) >= 1024) C *= 2;
  }
  int slice = (n + C - 1) / C;
  slice = (slice + 7) / 8 * 8;
  out->cluster = C;
  out->slice = slice;
  // 512 threads measured faster for up to 16 rows, 256 for more
  out->threads = batch <= 16 ? 512 : 256;
  const char* nt = getenv("DS_TOPK_THREADS");      // tuning sweeps only
  if (nt && (atoi(nt) == 256 || atoi(nt) == 512)) out->threads = atoi(nt);
  return true;
}

// Clusters of 16 CTAs are non-portable: allow them only where the device
// can run at least one.
static bool topk_cluster16_ok() {
  auto kern = topk_cluster_kernel<F32Keys, 256>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  cudaFuncSetAttribute(topk_cluster_kernel<F32Keys, 512>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  cudaFuncSetAttribute(topk_cluster_kernel<BF16Keys, 256>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  cudaFuncSetAttribute(topk_cluster_kernel<BF16Keys, 512>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  cudaFuncSetAttribute(topk_hist_select_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(16, 1, 1);
  cfg.blockDim = dim3(256, 1, 1);
  cfg.dynamicSmemBytes = (size_t)kTopkSmemBytes;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 16;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return n >= 1;
}

template <class K, int NT>
static cudaError_t launch_topk(const TopkParams& p, int C, cudaStream_t st) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(p.batch * C), 1, 1);
  cfg.blockDim = dim3(NT, 1, 1);
  cfg.dynamicSmemBytes = (size_t)kTopkSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  set_pdl(attr[1]);
  cfg.attrs = attr;
  cfg.numAttrs = pdl_on() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, topk_cluster_kernel<K, NT>, p);
}

// One-pass stash kernel.  Launch shape: one CTA per row, or C = 2 or 4 CTAs
// per row (a cluster) while the rows would leave more than half of the SMs
// idle and every slice keeps at least 32768 scores.
static int topk_stash_enqueue(const void* scores, int batch, int n, int k, int dtype, const int32_t* valid_len,
                              int32_t* out_idx, void* out_val, int return_value, int sorted_index,
                              cudaStream_t st, DeviceState* s, uint32_t* ghist = nullptr) {
  if (n > kMaxRowElems) return DS_ERR_ARG;
  int C = 1;
  const char* force = getenv("DS_TOPK_CLUSTER");  // tuning sweeps only
  if (force) {
    C = atoi(force);
    if (C != 1 && C != 2 && C != 4) C = 1;
  } else {
    while (C < kTsMaxCluster && (long)batch * 2 * C <= s->num_sms && n / (2 * C) >= 32768) C *= 2;
  }
  int slice = (n + C - 1) / C;
  slice = (slice + 7) / 8 * 8;
  TsParams p;
  memset(&p, 0, sizeof(p));
  p.scores = scores;
  p.ghist = dtype == DS_F32 ? ghist : nullptr;
  p.valid_len = valid_len;
  p.out_idx = out_idx;
  p.out_val = out_val;
  p.batch = batch;
  p.n = n;
  p.k = k;
  p.slice = slice;
  p.return_value = return_value ? 1 : 0;
  p.sorted = sorted_index ? 1 : 0;
  p.status = s->status;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(batch * C), 1, 1);
  cfg.blockDim = dim3(kTsThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)ts_smem_bytes(C);
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  set_pdl(attr[1]);
  cfg.attrs = attr;
  cfg.numAttrs = pdl_on() ? 2 : 1;
  const cudaError_t e = dtype == DS_F32 ? cudaLaunchKernelEx(&cfg, topk_stash_kernel<F32Keys, kTsThreads>, p)
                                        : cudaLaunchKernelEx(&cfg, topk_stash_kernel<BF16Keys, kTsThreads>, p);
  return e == cudaSuccess ? DS_OK : DS_ERR_CUDA;
}

// Two kernels: with many rows (>= 64) the one-pass stash kernel, whose rows
// fill the SMs with one or two CTAs each; with fewer rows the cluster kernel
// (topk_kernel.cuh), which spreads a row over up to 16 CTAs and has the
// shorter fixed chain of steps (both measured on each side of the boundary).
// DS_TOPK_KERNEL=stash / cluster picks one regardless (tests and comparisons).
static int topk_enqueue(const void* scores, int batch, int n, int k, int dtype, const int32_t* valid_len,
                        int32_t* out_idx, void* out_val, int return_value, int sorted_index, cudaStream_t st,
                        DeviceState* s) {
  bool stash = batch >= 64;
  const char* pick = getenv("DS_TOPK_KERNEL");
  if (pick && strcmp(pick, "stash") == 0) stash = true;
  if (pick && strcmp(pick, "cluster") == 0) stash = false;
  if (stash)
    return topk_stash_enqueue(scores, batch, n, k, dtype, valid_len, out_idx, out_val, return_value, sorted_index,
                              st, s);
  TopkShape sh;
  if (!choose_topk_shape(batch, n, s->num_sms, &sh)) return DS_ERR_ARG;
  TopkParams p;
  p.scores = scores;
  p.valid_len = valid_len;
  p.out_idx = out_idx;
  p.out_val = out_val;
  p.status = s->status;
  p.batch = batch;
  p.n = n;
  p.k = k;
  p.slice = sh.slice;
  p.return_value = return_value ? 1 : 0;
  p.sorted = sorted_index ? 1 : 0;
  cudaError_t e;
  if (dtype == DS_F32)
    e = sh.threads == 512 ? launch_topk<F32Keys, 512>(p, sh.cluster, st) : launch_topk<F32Keys, 256>(p, sh.cluster, st);
  else
    e = sh.threads == 512 ? launch_topk<BF16Keys, 512>(p, sh.cluster, st)
                          : launch_topk<BF16Keys, 256>(p, sh.cluster, st);
  return e == cudaSuccess ? DS_OK : DS_ERR_CUDA;
}


// ------------------------------------------------------------------ indexer

static PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

// Ring shapes of the weighted-sum kernel (K chunks per stage, S stages), in
// order of preference: the first whose shared memory fits the row's chunk count
// is launched.  Deeper rings of smaller stages (2 x 3, 1 x 4 .. 1 x 7) were no
// faster on the decode workload: the stream is bound by each SM's copy rate.
struct PvCfg {
  int K, S;
  void (*fn)(AttnParams);
  int (*bytes)(int);
};
template <int K, int S>
static int pv_bytes(int NS) {
  return PvSmem<K, S>::bytes(NS);
}
#define DS_PV_CFG(k, s) {k, s, sparse_attn_pv_kernel<k, s>, pv_bytes<k, s>}
static const PvCfg kPvCfg[] = {DS_PV_CFG(4, 2), DS_PV_CFG(3, 2), DS_PV_CFG(2, 2), DS_PV_CFG(1, 2)};
#undef DS_PV_CFG
static constexpr int kPvCfgs = (int)(sizeof(kPvCfg) / sizeof(kPvCfg[0]));

static const PvCfg* pv_pick(int NS) {
  const int lim = 227 * 1024;
  for (int i = 0; i < kPvCfgs; ++i)
    if (kPvCfg[i].bytes(NS) <= lim) return &kPvCfg[i];
  return nullptr;
}

template <int NT, int HP, int ST, bool SEL = false>
static cudaError_t set_score_smem() {
  return cudaFuncSetAttribute(indexer_score_kernel<NT, HP, ST, SEL>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              ScoreCfg<NT, HP, ST, SEL>::kSmemBytes);
}

// Called once per device from device_state (under its lock).
static cudaError_t indexer_setup() {
  if (!g_encode) {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
    if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn) return cudaErrorNotSupported;
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }
  cudaError_t e = set_score_smem<1, 64, 4>();
  if (e == cudaSuccess) e = set_score_smem<2, 64, 4>();
  if (e == cudaSuccess) e = set_score_smem<4, 64, 4>();
  if (e == cudaSuccess) e = set_score_smem<8, 32, 4>();
  if (e == cudaSuccess) e = set_score_smem<8, 16, 4>();
  if (e == cudaSuccess) e = set_score_smem<1, 32, 4>();
  if (e == cudaSuccess) e = set_score_smem<1, 16, 4>();
  if (e == cudaSuccess) e = set_score_smem<1, 64, 4, true>();
  if (e == cudaSuccess) e = set_score_smem<2, 64, 4, true>();
  if (e == cudaSuccess) e = set_score_smem<4, 64, 4, true>();
  if (e == cudaSuccess) e = set_score_smem<1, 32, 4, true>();
  if (e == cudaSuccess) e = set_score_smem<1, 16, 4, true>();
  if (e == cudaSuccess) e = set_score_smem<4, 32, 4, true>();
  if (e == cudaSuccess) e = set_score_smem<4, 16, 4, true>();
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(topk_hist_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, HsSmem::kBytes);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(sparse_attn_score_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             AttnSmem::bytes(kAttnMaxD));
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(indexer_qproj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kQpTok * kQpMaxIn * 2 + 8 * 32 * 33 * 4);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(indexer_qproj_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, QtSmem::kBytes);
  for (int i = 0; e == cudaSuccess && i < kPvCfgs; ++i)
    e = cudaFuncSetAttribute(kPvCfg[i].fn, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
  return e;
}

// bf16 tensor maps with 128-byte swizzle: queries [B][H][128] in boxes of
// (64 channels, HP heads, NT rows); keys [S][128] in boxes of (64, 128).
static bool encode_maps(const void* q, const void* kc, int B, int H, int S, int HP, int NT, CUtensorMap* tq,
                        CUtensorMap* tk) {
  cuuint64_t qdims[3] = {128, (cuuint64_t)H, (cuuint64_t)B};
  cuuint64_t qstr[2] = {256, (cuuint64_t)H * 256};
  cuuint32_t qbox[3] = {64, (cuuint32_t)HP, (cuuint32_t)NT};
  cuuint32_t one3[3] = {1, 1, 1};
  CUresult r = g_encode(tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), qdims, qstr, qbox, one3,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return false;
  cuuint64_t kdims[2] = {128, (cuuint64_t)S};
  cuuint64_t kstr[1] = {256};
  cuuint32_t kbox[2] = {64, 128};
  cuuint32_t one2[2] = {1, 1};
  r = g_encode(tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(kc), kdims, kstr, kbox, one2,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Keys viewed as (64 channels, S positions, 2 channel halves, nk caches),
// caches kstride rows apart, in boxes of (64, 128, 2, 1): one copy is a whole
// 128-position tile, its two 64-channel halves one after the other.
static bool encode_kmap(const void* kc, int S, int nk, long long kstride, CUtensorMap* tk) {
  cuuint64_t dims[4] = {64, (cuuint64_t)S, 2, (cuuint64_t)nk};
  cuuint64_t str[3] = {256, 128, (cuuint64_t)(kstride > 0 ? kstride : S) * 256};
  cuuint32_t box[4] = {64, 128, 2, 1};
  cuuint32_t one[4] = {1, 1, 1, 1};
  return g_encode(tk, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(kc), dims, str, box, one,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int NT, int HP, int ST>
static int launch_score(const void* q, const void* kc, const float* w, int B, int H, int S, const int32_t* vl,
                        float* out, long long kstride, cudaStream_t st, DeviceState* s) {
  using Cfg = ScoreCfg<NT, HP, ST>;
  CUtensorMap tq, tk;
  if (!encode_maps(q, kc, B, H, S, HP, NT, &tq, &tk)) return DS_ERR_ARG;
  const bool per_row = kstride > 0;
  if (per_row && NT != 1) return DS_ERR_ARG;
  if (!encode_kmap(kc, S, per_row ? B : 1, kstride, &tk)) return DS_ERR_ARG;
  const int ntiles = (S + 127) / 128;
  const int groups = (B + NT - 1) / NT;
  // spread one group's tiles over several CTAs only while there are fewer
  // groups than SMs
  long tpc = ((long)groups * ntiles + s->num_sms - 1) / s->num_sms;
  if (tpc < 1) tpc = 1;
  if (tpc > ntiles) tpc = ntiles;
  const int cpg = (int)((ntiles + tpc - 1) / tpc);
  ScoreParams p;
  memset(&p, 0, sizeof(p));
  p.w = w;
  p.valid_len = vl;
  p.out = out;
  p.status = s->status;
  p.B = B;
  p.H = H;
  p.S = S;
  p.tiles_per_cta = (int)tpc;
  p.ctas_per_group = cpg;
  p.key_per_row = per_row ? 1 : 0;
  p.wait_ns = wait_limit();
  p.fault = take_planted_fault();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(groups * cpg), 1, 1);
  cfg.blockDim = dim3(Cfg::kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)Cfg::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  set_pdl(attr[0]);
  cfg.attrs = attr;
  cfg.numAttrs = pdl_on() ? 1 : 0;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, indexer_score_kernel<NT, HP, ST>, tq, tk, p);
  return e == cudaSuccess ? DS_OK : DS_ERR_CUDA;
}

// kstride: rows from one row's key cache to the next (0: one cache for every row).
static int score_enqueue(const void* q, const void* kc, const float* w, int B, int H, int S, const int32_t* vl,
                         float* out, cudaStream_t st, DeviceState* s, long long kstride = 0) {
  if (kstride > 0) {  // a cache per row: one row per CTA group
    if (H > 32) return launch_score<1, 64, 4>(q, kc, w, B, H, S, vl, out, kstride, st, s);
    if (H > 16) return launch_score<1, 32, 4>(q, kc, w, B, H, S, vl, out, kstride, st, s);
    return launch_score<1, 16, 4>(q, kc, w, B, H, S, vl, out, kstride, st, s);
  }
  if (H > 32) {
    const char* force = getenv("DS_SCORE_ROWS");  // tuning sweeps only: rows per CTA group
    if (force && B > 2) {
      const int nt = atoi(force);
      if (nt == 1) return launch_score<1, 64, 4>(q, kc, w, B, H, S, vl, out, 0, st, s);
      if (nt == 2) return launch_score<2, 64, 4>(q, kc, w, B, H, S, vl, out, 0, st, s);
      if (nt == 4) return launch_score<4, 64, 4>(q, kc, w, B, H, S, vl, out, 0, st, s);
    }
    if (B == 1) return launch_score<1, 64, 4>(q, kc, w, B, H, S, vl, out, 0, st, s);
    if (B == 2) return launch_score<2, 64, 4>(q, kc, w, B, H, S, vl, out, 0, st, s);
    // 5..8 rows: two rows per CTA (measured faster than eight per CTA, whose
    // 128 KiB query tile every CTA must load)
    if (B <= 4 || B > 8) return launch_score<4, 64, 4>(q, kc, w, B, H, S, vl, out, 0, st, s);
    return launch_score<2, 64, 4>(q, kc, w, B, H, S, vl, out, 0, st, s);
  }
  if (H > 16) return launch_score<8, 32, 4>(q, kc, w, B, H, S, vl, out, 0, st, s);
  return launch_score<8, 16, 4>(q, kc, w, B, H, S, vl, out, 0, st, s);
}

static int indexer_check(const void* q, const void* kc, const float* w, int B, int H, int d, int S) {
  if (!q || !kc || !w || B <= 0 || H <= 0 || H > DS_INDEXER_MAX_HEADS || d != DS_INDEXER_DIM || S <= 0)
    return DS_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(q) & 15u) || (reinterpret_cast<uintptr_t>(kc) & 15u) ||
      (reinterpret_cast<uintptr_t>(w) & 3u))
    return DS_ERR_ARG;
  return DS_OK;
}

// Grow-only per-device scratch; the caller holds no lock.
static void* get_scratch(DeviceState* s, size_t bytes) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (s->scratch_bytes >= bytes) return s->scratch;
  if (s->scratch) cudaFree(s->scratch);
  s->scratch = nullptr;
  s->scratch_bytes = 0;
  void* p = nullptr;
  if (cudaMalloc(&p, bytes) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  s->scratch = p;
  s->scratch_bytes = bytes;
  return p;
}

// ---- indexer + top-k (the path of ds_indexer_topk and ds_indexer_topk_ex)
//
// The scorer also counts every valid score in an exact histogram of its key's
// top 12 bits (per row, added into global memory), and the selection starts
// from the threshold bin those counts give, with no sampling.  Rows split over
// several scorer CTAs (few rows, as in decode): topk_hist_select_kernel, a
// cluster per row.  Whole rows per scorer CTA (many rows, as in prefill): the
// one-pass stash kernel streams each row once and stashes what is at or above
// the bin.  Selecting inside the scorer's CTAs (whose selection tail leaves the
// tensor pipe idle) or beside them measured slower on this GPU.

// Grow-only buffer that is all zero whenever no call is in flight: zeroed when
// (re)allocated, and every launch that uses it leaves it zero again.
static void* get_zeroed_state(DeviceState* s, size_t bytes) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (s->sel_state_bytes >= bytes) return s->sel_state;
  if (s->sel_state) cudaFree(s->sel_state);
  s->sel_state = nullptr;
  s->sel_state_bytes = 0;
  void* p = nullptr;
  if (cudaMalloc(&p, bytes) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  if (cudaMemset(p, 0, bytes) != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) {
    cudaFree(p);
    return nullptr;
  }
  s->sel_state = p;
  s->sel_state_bytes = bytes;
  return p;
}

// Scorer CTAs per group of NT rows for the scores-with-histograms launch (the
// same spread as score_enqueue's, capped by the 16-bit counters).
template <int NT, int HP, int ST>
static int hist_groups_split(int B, int S, const DeviceState* s, int* tpc_out) {
  using Cfg = ScoreCfg<NT, HP, ST, true>;
  const int ntiles = (S + 127) / 128;
  const int groups = (B + NT - 1) / NT;
  long tpc = ((long)groups * ntiles + s->num_sms - 1) / s->num_sms;
  tpc = std::max(1L, std::min(tpc, (long)std::min(ntiles, Cfg::kMaxTilesPerCta)));
  *tpc_out = (int)tpc;
  return (int)((ntiles + tpc - 1) / tpc);
}

// One scorer launch: scores of the valid positions to out [B, S], key counts
// added into ghist [B, 4096].
template <int NT, int HP, int ST>
static int launch_score_hist(const void* q, const void* kc, const float* w, int B, int H, int S, const int32_t* vl,
                             long long kstride, float* out, uint32_t* ghist, cudaStream_t st, DeviceState* s) {
  using Cfg = ScoreCfg<NT, HP, ST, true>;
  CUtensorMap tq, tk;
  if (!encode_maps(q, kc, B, H, S, HP, NT, &tq, &tk)) return DS_ERR_ARG;
  const bool per_row = kstride > 0;
  if (per_row && NT != 1) return DS_ERR_ARG;
  if (!encode_kmap(kc, S, per_row ? B : 1, kstride, &tk)) return DS_ERR_ARG;
  int tpc = 0;
  const int cpg = hist_groups_split<NT, HP, ST>(B, S, s, &tpc);
  ScoreParams p;
  memset(&p, 0, sizeof(p));
  p.w = w;
  p.valid_len = vl;
  p.out = out;
  p.status = s->status;
  p.B = B;
  p.H = H;
  p.S = S;
  p.tiles_per_cta = tpc;
  p.ctas_per_group = cpg;
  p.key_per_row = per_row ? 1 : 0;
  p.ghist = ghist;
  p.wait_ns = wait_limit();
  p.fault = take_planted_fault();
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(((B + NT - 1) / NT) * cpg), 1, 1);
  cfg.blockDim = dim3(Cfg::kThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)Cfg::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  set_pdl(attr[0]);
  cfg.attrs = attr;
  cfg.numAttrs = pdl_on() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, indexer_score_kernel<NT, HP, ST, true>, tq, tk, p) == cudaSuccess ? DS_OK
                                                                                                    : DS_ERR_CUDA;
}

// One selection launch over B rows: a cluster of C CTAs per row, as many as
// keep every slice at 1024 scores or more and the rows' CTAs within the SM count.
static int launch_hist_select(const float* scores, uint32_t* ghist, const int32_t* vl, int32_t* out_idx,
                              float* out_score, int B, int S, int k, int sorted, cudaStream_t st, DeviceState* s) {
  int C = 1;
  int cmax = g_max_cluster;
  if (const char* f = getenv("DS_HS_CLUSTER")) {  // tuning sweeps only: the largest cluster allowed
    const int v = atoi(f);
    if (v == 1 || v == 2 || v == 4 || v == 8 || v == 16) cmax = std::min(cmax, v);
  }
  while (2 * C <= cmax && (long)B * 2 * C <= s->num_sms && S / (2 * C) >= 1024) C *= 2;
  HsParams h;
  memset(&h, 0, sizeof(h));
  h.scores = scores;
  h.ghist = ghist;
  h.valid_len = vl;
  h.out_idx = out_idx;
  h.out_score = out_score;
  h.B = B;
  h.S = S;
  h.k = k;
  h.slice = ((S + C - 1) / C + 3) / 4 * 4;
  h.sorted = sorted;
  h.status = s->status;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(B * C), 1, 1);
  cfg.blockDim = dim3(kHsThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)HsSmem::kBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)C;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  set_pdl(attr[1]);
  cfg.attrs = attr;
  cfg.numAttrs = pdl_on() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, topk_hist_select_kernel, h) == cudaSuccess ? DS_OK : DS_ERR_CUDA;
}

template <int NT, int HP, int ST>
static int indexer_topk_rows(const void* q, const void* kc, const float* w, int B, int H, int S, const int32_t* vl,
                             int k, int sorted, int32_t* out_idx, float* out_score, long long kstride,
                             cudaStream_t st, DeviceState* s) {
  float* sc = static_cast<float*>(get_scratch(s, (size_t)B * (size_t)S * sizeof(float)));
  if (!sc) return DS_ERR_NOMEM;
  int tpc = 0;
  if (hist_groups_split<NT, HP, ST>(B, S, s, &tpc) > 1) {
    uint32_t* gh = static_cast<uint32_t*>(get_zeroed_state(s, (size_t)B * kSelBins * sizeof(uint32_t)));
    if (!gh) return DS_ERR_NOMEM;
    const int rc = launch_score_hist<NT, HP, ST>(q, kc, w, B, H, S, vl, kstride, sc, gh, st, s);
    if (rc != DS_OK) return rc;
    return launch_hist_select(sc, gh, vl, out_idx, out_score, B, S, k, sorted, st, s);
  }
  // whole rows: the scorer's counts give the stash kernel its threshold
  uint32_t* gh = static_cast<uint32_t*>(get_zeroed_state(s, (size_t)B * kSelBins * sizeof(uint32_t)));
  if (!gh) return DS_ERR_NOMEM;
  const int rc = launch_score_hist<NT, HP, ST>(q, kc, w, B, H, S, vl, kstride, sc, gh, st, s);
  if (rc != DS_OK) return rc;
  return topk_stash_enqueue(sc, B, S, k, DS_F32, vl, out_idx, out_score, out_score != nullptr, sorted, st, s, gh);
}

// Rows per CTA group: as for the scores alone (two rows for 2 and 5..8 rows,
// one for one row, four otherwise); one row with a key cache per row; four
// rows with 32 or fewer heads (N = 128 or 64).
static int fused_enqueue(const void* q, const void* kc, const float* w, int B, int H, int S, const int32_t* vl,
                         int k, int sorted, int32_t* out_idx, float* out_score, long long kstride, cudaStream_t st,
                         DeviceState* s) {
  if (kstride > 0) {
    if (H > 32) return indexer_topk_rows<1, 64, 4>(q, kc, w, B, H, S, vl, k, sorted, out_idx, out_score, kstride, st, s);
    if (H > 16) return indexer_topk_rows<1, 32, 4>(q, kc, w, B, H, S, vl, k, sorted, out_idx, out_score, kstride, st, s);
    return indexer_topk_rows<1, 16, 4>(q, kc, w, B, H, S, vl, k, sorted, out_idx, out_score, kstride, st, s);
  }
  if (H > 32) {
    if (B == 1) return indexer_topk_rows<1, 64, 4>(q, kc, w, B, H, S, vl, k, sorted, out_idx, out_score, 0, st, s);
    if (B == 2 || (B >= 5 && B <= 8))
      return indexer_topk_rows<2, 64, 4>(q, kc, w, B, H, S, vl, k, sorted, out_idx, out_score, 0, st, s);
    return indexer_topk_rows<4, 64, 4>(q, kc, w, B, H, S, vl, k, sorted, out_idx, out_score, 0, st, s);
  }
  if (H > 16) return indexer_topk_rows<4, 32, 4>(q, kc, w, B, H, S, vl, k, sorted, out_idx, out_score, 0, st, s);
  return indexer_topk_rows<4, 16, 4>(q, kc, w, B, H, S, vl, k, sorted, out_idx, out_score, 0, st, s);
}

// ---- sparse attention over the selected rows

// Queries [rows][D] bf16 viewed as (64 channels, rows, D/64 blocks): one box
// of (64, 128, D/64) is a head tile's queries, block by block, 128-byte swizzle.
static bool encode_attn_q(const void* q, long long rows, int D, CUtensorMap* tq) {
  cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)(D / 64)};
  cuuint64_t str[2] = {(cuuint64_t)D * 2, 128};
  cuuint32_t box[3] = {64, (cuuint32_t)kAttnHeads, (cuuint32_t)(D / 64)};
  cuuint32_t one[3] = {1, 1, 1};
  const CUresult r = g_encode(tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, str, box, one,
                              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Partial results of one call stay below this; larger batches run in pieces.
constexpr size_t kAttnScratchCap = size_t(512) << 20;

static void* get_attn_scratch(DeviceState* s, size_t bytes) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (s->attn_scratch_bytes >= bytes) return s->attn_scratch;
  if (s->attn_scratch) cudaFree(s->attn_scratch);
  s->attn_scratch = nullptr;
  s->attn_scratch_bytes = 0;
  void* p = nullptr;
  if (cudaMalloc(&p, bytes) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  s->attn_scratch = p;
  s->attn_scratch_bytes = bytes;
  return p;
}

static int attention_enqueue(const uint16_t* q, const uint16_t* kv, long long kv_bstride_rows, int T,
                             const int32_t* idx, int k, const uint16_t* win, int W, const int32_t* win_len,
                             const float* sink, int B, int H, int D, float scale, uint16_t* out, float* lse,
                             cudaStream_t st, DeviceState* s) {
  const int HT = (H + kAttnHeads - 1) / kAttnHeads;
  const int NS = (k + W + kAttnRows - 1) / kAttnRows;
  // per batch row and chunk: a bf16 weight tile and (max, sum) per head of
  // every head tile, and the chunk's rows as D/64 row tiles
  const size_t tile_row = (size_t)HT * NS * kAttnTile;
  const size_t vt_row = (size_t)(D / 64) * NS * kRowTile;
  const size_t ml_row = (size_t)HT * NS * kAttnHeads * sizeof(float2);
  const size_t per_row = tile_row + vt_row + ml_row;
  int per = B;
  if (NS > 0 && per_row * (size_t)B > kAttnScratchCap) per = (int)std::max<size_t>(1, kAttnScratchCap / per_row);
  uint8_t* ptile = nullptr;
  uint8_t* vtile = nullptr;
  float2* ml = nullptr;
  if (NS > 0) {
    uint8_t* base = static_cast<uint8_t*>(get_attn_scratch(s, per_row * (size_t)per));
    if (!base) return DS_ERR_NOMEM;
    ptile = base;
    vtile = base + tile_row * (size_t)per;
    ml = reinterpret_cast<float2*>(vtile + vt_row * (size_t)per);
  }
  const float kLog2e = 1.4426950408889634f;
  for (int b0 = 0; b0 < B; b0 += per) {
    const int nb = std::min(per, B - b0);
    AttnParams p;
    memset(&p, 0, sizeof(p));
    p.wait_ns = wait_limit();
    p.kv = kv + (size_t)b0 * (size_t)kv_bstride_rows * D;
    p.kv_bstride = kv_bstride_rows * (long long)D;
    p.win = win ? win + (size_t)b0 * W * D : nullptr;
    p.idx = idx ? idx + (size_t)b0 * k : nullptr;
    p.win_len = win_len ? win_len + b0 : nullptr;
    p.sink = sink;
    p.ptile = ptile;
    p.vtile = vtile;
    p.ml = ml;
    p.out = out + (size_t)b0 * H * D;
    p.lse = lse ? lse + (size_t)b0 * H : nullptr;
    p.status = s->status;
    p.T = T;
    p.k = k;
    p.W = W;
    p.B = nb;
    p.H = H;
    p.D = D;
    p.HT = HT;
    p.NS = NS;
    p.scale_log2 = scale * kLog2e;
    cudaLaunchAttribute attr[1];
    set_pdl(attr[0]);
    if (NS > 0) {
      CUtensorMap tq;
      if (!encode_attn_q(q + (size_t)b0 * H * D, (long long)nb * H, D, &tq)) return DS_ERR_ARG;
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)NS, (unsigned)HT, (unsigned)nb);
      cfg.blockDim = dim3(kAttnThreads, 1, 1);
      cfg.dynamicSmemBytes = (size_t)AttnSmem::bytes(D);
      cfg.stream = st;
      cfg.attrs = attr;
      cfg.numAttrs = pdl_on() ? 1 : 0;
      if (cudaLaunchKernelEx(&cfg, sparse_attn_score_kernel, tq, p) != cudaSuccess) return DS_ERR_CUDA;
    }
    // chunks of a row split over a cluster pair while one CTA per column slice
    // would leave more than half of the SMs idle
    const int G = (NS > 1 && 2L * (D / kPvSlice) * HT * nb <= s->num_sms) ? 2 : 1;
    const PvCfg* pc = pv_pick(NS);
    if (!pc) return DS_ERR_ARG;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(D / kPvSlice), (unsigned)G, (unsigned)(HT * nb));
    cfg.blockDim = dim3(kPvWarps * 32, 1, 1);
    cfg.dynamicSmemBytes = (size_t)pc->bytes(NS);
    cfg.stream = st;
    cudaLaunchAttribute pattr[2];
    int na = 0;
    if (pdl_on()) set_pdl(pattr[na++]);
    if (G == 2) {
      pattr[na].id = cudaLaunchAttributeClusterDimension;
      pattr[na].val.clusterDim.x = 1;
      pattr[na].val.clusterDim.y = 2;
      pattr[na].val.clusterDim.z = 1;
      ++na;
    }
    cfg.attrs = pattr;
    cfg.numAttrs = na;
    if (cudaLaunchKernelEx(&cfg, pc->fn, p) != cudaSuccess) return DS_ERR_CUDA;
  }
  return DS_OK;
}

// ---- indexer query projection on the tensor cores (input width a multiple of 64)

// A [rows][d_in] bf16 matrix viewed as (64 channels, rows, d_in/64 blocks), in
// boxes of (64, box_rows, bpb): rows block by block, 128-byte swizzle.
static bool encode_rowblocks(const void* base, long long rows, int d_in, int box_rows, int bpb, CUtensorMap* m) {
  cuuint64_t dims[3] = {64, (cuuint64_t)rows, (cuuint64_t)(d_in / 64)};
  cuuint64_t str[2] = {(cuuint64_t)d_in * 2, 128};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, (cuuint32_t)bpb};
  cuuint32_t one[3] = {1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, str, box, one,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

static int qproj_tc_enqueue(const void* x, const void* wq, const void* ww, int T, int d_in, int heads, int d,
                            void* q_out, float* w_out, cudaStream_t st, DeviceState* s) {
  const int nq = heads * d;
  const int nqb = nq / 128;
  const int nrb = nqb + (ww ? 1 : 0);
  const int nblk = d_in / 64;
  const int ntg = (T + kQtTok - 1) / kQtTok;
  // split the input width over a cluster pair while one CTA per row block
  // would leave more than half of the SMs idle
  const int G = (nblk % 2 == 0 && 2 * nrb * ntg <= s->num_sms) ? 2 : 1;
  const int per = nblk / G;
  const int bpb = per % 4 == 0 ? 4 : 1;
  CUtensorMap twq, tww, tx;
  if (!encode_rowblocks(wq, nq, d_in, 128, bpb, &twq)) return DS_ERR_ARG;
  if (!encode_rowblocks(ww ? ww : wq, ww ? heads : nq, d_in, 128, bpb, &tww)) return DS_ERR_ARG;
  if (!encode_rowblocks(x, T, d_in, kQtTok, bpb, &tx)) return DS_ERR_ARG;
  QtParams p;
  memset(&p, 0, sizeof(p));
  p.wait_ns = wait_limit();
  p.q = static_cast<uint16_t*>(q_out);
  p.w = w_out;
  p.status = s->status;
  p.T = T;
  p.nq = nq;
  p.heads = heads;
  p.nblk = nblk;
  p.bpb = bpb;
  p.nqb = nqb;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)nrb, (unsigned)G, (unsigned)ntg);
  cfg.blockDim = dim3(128, 1, 1);
  cfg.dynamicSmemBytes = (size_t)QtSmem::kBytes;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  int na = 0;
  if (pdl_on()) set_pdl(attr[na++]);
  if (G == 2) {
    attr[na].id = cudaLaunchAttributeClusterDimension;
    attr[na].val.clusterDim.x = 1;
    attr[na].val.clusterDim.y = 2;
    attr[na].val.clusterDim.z = 1;
    ++na;
  }
  cfg.attrs = attr;
  cfg.numAttrs = na;
  return cudaLaunchKernelEx(&cfg, indexer_qproj_tc_kernel, twq, tww, tx, p) == cudaSuccess ? DS_OK : DS_ERR_CUDA;
}

}  // namespace dstopk

using namespace dstopk;

extern "C" int ds_topk(const void* scores, int batch, int n, int k, int dtype, const int32_t* valid_len,
                       int32_t* out_idx, void* out_val, int return_value, int sorted_index, void* stream) {
  if (!scores || !out_idx || batch <= 0 || n <= 0 || k <= 0 || k > DS_MAX_K) return DS_ERR_ARG;
  if (dtype != DS_F32 && dtype != DS_BF16) return DS_ERR_ARG;
  if (return_value && !out_val) return DS_ERR_ARG;
  if (n > kMaxRowElems) return DS_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(scores) & (dtype == DS_F32 ? 3u : 1u)) != 0) return DS_ERR_ARG;
  DeviceState* s = nullptr;
  const int rc = device_state(&s);
  if (rc != DS_OK) return rc;
  return topk_enqueue(scores, batch, n, k, dtype, valid_len, out_idx, out_val, return_value, sorted_index,
                      static_cast<cudaStream_t>(stream), s);
}

extern "C" int ds_get_device_status(void* stream) {
  DeviceState* s = nullptr;
  const int rc = device_state(&s);
  if (rc != DS_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int host = 0;
  if (cudaMemcpyAsync(&host, s->status, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess) return DS_ERR_CUDA;
  if (cudaMemsetAsync(s->status, 0, sizeof(int), st) != cudaSuccess) return DS_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return DS_ERR_CUDA;
  return host;
}

extern "C" int ds_set_wait_limit(int64_t ns) {
  if (ns < 0 || ns > kMaxWaitLimitNs) return DS_ERR_ARG;
  g_wait_ns.store((long long)ns, std::memory_order_relaxed);
  return DS_OK;
}

extern "C" int ds_plant_wait_fault(int launches) {
  if (launches < 0) return DS_ERR_ARG;
  g_planted.store(launches, std::memory_order_relaxed);
  return DS_OK;
}

extern "C" int ds_debug_build(void) { return kDebugChecks ? 1 : 0; }

namespace dstopk {
// A read-only pass over a buffer (16-byte loads, 8 in flight per thread, the
// buffer split evenly over the CTAs): what a one-pass kernel over the same
// bytes cannot beat.
static __device__ uint32_t g_floor_sink;
__global__ void __launch_bounds__(1024) read_floor_kernel(const uint4* p, long long words) {
  const long long per = (words + gridDim.x - 1) / gridDim.x;
  const long long w0 = (long long)blockIdx.x * per;
  const long long w1 = w0 + per < words ? w0 + per : words;
  uint32_t acc = 0u;
  for (long long base = w0; base < w1; base += 8 * 1024) {
    uint4 v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const long long w = base + u * 1024 + threadIdx.x;
      v[u] = w < w1 ? __ldcs(p + w) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) acc ^= v[u].x ^ v[u].y ^ v[u].z ^ v[u].w;
  }
  if (acc == 0x9E3779B9u) g_floor_sink = acc;  // keeps the loads
}
}  // namespace dstopk

extern "C" int ds_read_floor(const void* p, int64_t bytes, int ctas, void* stream) {
  if (!p || (reinterpret_cast<uintptr_t>(p) & 15u) || bytes <= 0 || (bytes & 15) || ctas < 1 || ctas > 65535)
    return DS_ERR_ARG;
  DeviceState* s = nullptr;
  const int rc = device_state(&s);
  if (rc != DS_OK) return rc;
  read_floor_kernel<<<ctas, 1024, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<const uint4*>(p), bytes / 16);
  return cudaGetLastError() == cudaSuccess ? DS_OK : DS_ERR_CUDA;
}

extern "C" int ds_debug_stash_stamps(uint64_t* host_dst, int ctas) {
#ifdef DS_DEBUG
  if (!host_dst || ctas < 1 || ctas > kTsStampCtas) return DS_ERR_ARG;
  DeviceState* s = nullptr;
  const int rc = device_state(&s);
  if (rc != DS_OK) return rc;
  const size_t n = (size_t)ctas * kTsStampSlots * sizeof(unsigned long long);
  if (cudaMemcpyFromSymbol(host_dst, ts_stamps, n) != cudaSuccess) return DS_ERR_CUDA;
  void* d = nullptr;
  if (cudaGetSymbolAddress(&d, ts_stamps) != cudaSuccess) return DS_ERR_CUDA;
  return cudaMemset(d, 0, sizeof(ts_stamps)) == cudaSuccess && cudaDeviceSynchronize() == cudaSuccess ? DS_OK
                                                                                                   : DS_ERR_CUDA;
#else
  (void)host_dst;
  (void)ctas;
  return DS_ERR_UNSUPPORTED;
#endif
}

extern "C" const char* ds_strerror(int code) {
  switch (code) {
    case DS_OK: return "DS_OK";
    case DS_ERR_ARG: return "DS_ERR_ARG: invalid argument";
    case DS_ERR_CUDA: return "DS_ERR_CUDA: CUDA runtime error";
    case DS_ERR_TIMEOUT: return "DS_ERR_TIMEOUT: a bounded device wait ran out";
    case DS_ERR_UNSUPPORTED: return "DS_ERR_UNSUPPORTED: device is not sm_100";
    case DS_ERR_NOMEM: return "DS_ERR_NOMEM: scratch allocation failed";
    case DS_ERR_RANGE: return "DS_ERR_RANGE: an input read on the device was out of range (DS_DEBUG build)";
    default: return "unknown status";
  }
}

extern "C" void ds_release(void) {
  std::lock_guard<std::mutex> lock(g_mu);
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) cur = -1;
  for (int d = 0; d < kMaxDevices; ++d) {
    DeviceState& st = g_dev[d];
    if (st.scratch || st.sel_state || st.attn_scratch) {
      if (cudaSetDevice(d) == cudaSuccess) {
        if (st.scratch) cudaFree(st.scratch);
        if (st.sel_state) cudaFree(st.sel_state);
        if (st.attn_scratch) cudaFree(st.attn_scratch);
      }
      st.attn_scratch = nullptr;
      st.attn_scratch_bytes = 0;
      st.scratch = nullptr;
      st.scratch_bytes = 0;
      st.sel_state = nullptr;
      st.sel_state_bytes = 0;
    }
  }
  if (cur >= 0) cudaSetDevice(cur);
}

extern "C" int ds_indexer_score(const void* q, const void* kcache, const float* w, int batch, int heads, int d,
                                int S, const int32_t* valid_len, float* out_score, void* stream) {
  int rc = indexer_check(q, kcache, w, batch, heads, d, S);
  if (rc != DS_OK) return rc;
  if (!out_score) return DS_ERR_ARG;
  DeviceState* s = nullptr;
  rc = device_state(&s);
  if (rc != DS_OK) return rc;
  return score_enqueue(q, kcache, w, batch, heads, S, valid_len, out_score, static_cast<cudaStream_t>(stream), s);
}

extern "C" int ds_indexer_topk(const void* q, const void* kcache, const float* w, int batch, int heads, int d, int S,
                               const int32_t* valid_len, int k, int32_t* out_idx, float* out_score, void* stream) {
  int rc = indexer_check(q, kcache, w, batch, heads, d, S);
  if (rc != DS_OK) return rc;
  if (!out_idx || k <= 0 || k > DS_MAX_K) return DS_ERR_ARG;
  if (S > kMaxRowElems) return DS_ERR_ARG;
  DeviceState* s = nullptr;
  rc = device_state(&s);
  if (rc != DS_OK) return rc;
  return fused_enqueue(q, kcache, w, batch, heads, S, valid_len, k, 0, out_idx, out_score, 0,
                       static_cast<cudaStream_t>(stream), s);
}

// ------------------------------------------------------------------ allocation-free indexer + top-k
//
// Some callers cannot call cudaMalloc at all: a serving engine that reserves
// all device memory for its own pool up front, code that runs while another
// framework is capturing a CUDA graph in a mode that forbids allocation, or a
// latency-critical path that cannot afford the device-wide synchronisation a
// first cudaMalloc may cause.  ds_indexer_topk_noalloc serves them: its score
// rows go to a fixed array in the library's own device memory instead of the
// grow-only scratch buffer.  Every GPU that loads the library holds this array
// (1 MiB) until the process exits.

constexpr int kNoAllocScores = 262144;  // floats: batch * S may not exceed this (1 MiB)

// The array itself.  In host code this name is only a host-side stand-in, not
// a device address; the device address comes from cudaGetSymbolAddress below.
static __device__ __align__(256) float g_noalloc_scores[kNoAllocScores];

static float* g_noalloc_ptr[kMaxDevices];  // device address of g_noalloc_scores, per device

// Once per device, with that device current (the first call on the device).
static int noalloc_scores_ptr(float** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DS_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scores) != cudaSuccess || !p) return DS_ERR_CUDA;
    g_noalloc_ptr[dev] = static_cast<float*>(p);
  }
  *out = g_noalloc_ptr[dev];
  return DS_OK;
}

extern "C" int ds_indexer_topk_noalloc(const void* q, const void* kcache, const float* w, int batch, int heads,
                                       int d, int S, const int32_t* valid_len, int k, int32_t* out_idx,
                                       float* out_score, void* stream) {
  int rc = indexer_check(q, kcache, w, batch, heads, d, S);
  if (rc != DS_OK) return rc;
  if (!out_idx || k <= 0 || k > DS_MAX_K) return DS_ERR_ARG;
  if ((long)batch * (long)S > (long)kNoAllocScores) return DS_ERR_ARG;  // beyond the fixed array
  DeviceState* s = nullptr;
  rc = device_state(&s);
  if (rc != DS_OK) return rc;
  float* scores = nullptr;
  rc = noalloc_scores_ptr(&scores);
  if (rc != DS_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The scorer writes every position of every row (-inf at and past
  // valid_len, and -inf at the positions left when one of its waits runs
  // out) before the selection reads it, so nothing left over from an earlier
  // call is ever read and the array needs no clearing.
  rc = score_enqueue(q, kcache, w, batch, heads, S, valid_len, scores, st, s);
  if (rc != DS_OK) return rc;
  return topk_enqueue(scores, batch, S, k, DS_F32, valid_len, out_idx, out_score, out_score != nullptr, 0, st, s);
}

extern "C" int ds_sparse_attention(const void* q, const void* kv, int64_t kv_batch_stride, int T, const int32_t* idx,
                                   int k, const void* win, int W, const int32_t* win_len, const float* sink,
                                   int batch, int heads, int d, float scale, void* out, float* lse, void* stream) {
  auto misaligned = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0; };
  if (!q || !kv || !out || batch <= 0 || batch > 65535 || heads <= 0 || heads > DS_ATTN_MAX_HEADS) return DS_ERR_ARG;
  if ((long)batch * ((heads + 127) / 128) > 65535) return DS_ERR_ARG;  // grid z of the weighted-sum kernel
  if (d < 64 || d > DS_ATTN_MAX_DIM || d % 64 != 0 || T <= 0 || kv_batch_stride < 0) return DS_ERR_ARG;
  if (k < 0 || k > DS_MAX_K || (k > 0 && !idx) || W < 0 || W > DS_ATTN_MAX_WINDOW || (W > 0 && !win))
    return DS_ERR_ARG;
  if (!(scale == scale) || scale > 3.0e38f || scale < -3.0e38f) return DS_ERR_ARG;
  if (misaligned(q, 16) || misaligned(kv, 16) || misaligned(out, 16) || (win && misaligned(win, 16)) ||
      (idx && misaligned(idx, 4)) || (win_len && misaligned(win_len, 4)) || (sink && misaligned(sink, 4)) ||
      (lse && misaligned(lse, 4)))
    return DS_ERR_ARG;
  DeviceState* s = nullptr;
  const int rc = device_state(&s);
  if (rc != DS_OK) return rc;
  return attention_enqueue(static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(kv), (long long)kv_batch_stride,
                           T, idx, k, static_cast<const uint16_t*>(win), W, win_len, sink, batch, heads, d, scale,
                           static_cast<uint16_t*>(out), lse, static_cast<cudaStream_t>(stream), s);
}

extern "C" int ds_indexer_qproj(const void* x, const void* wq, const void* ww, int T, int d_in, int heads, int d,
                                void* q_out, float* w_out, void* stream) {
  auto misaligned = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0; };
  if (!x || !wq || !q_out || (ww == nullptr) != (w_out == nullptr)) return DS_ERR_ARG;
  if (T <= 0 || T > 65535 * kQpTok || heads <= 0 || heads > DS_INDEXER_MAX_HEADS || d != DS_INDEXER_DIM) return DS_ERR_ARG;
  if (d_in < 8 || d_in > kQpMaxIn || d_in % 8 != 0) return DS_ERR_ARG;
  if (misaligned(x, 16) || misaligned(wq, 16) || (ww && misaligned(ww, 16)) || misaligned(q_out, 2) ||
      (w_out && misaligned(w_out, 4)))
    return DS_ERR_ARG;
  DeviceState* s = nullptr;
  const int rc = device_state(&s);
  if (rc != DS_OK) return rc;
  if (d_in % 64 == 0) return qproj_tc_enqueue(x, wq, ww, T, d_in, heads, d, q_out, w_out, static_cast<cudaStream_t>(stream), s);
  QpParams p;
  p.x = static_cast<const uint16_t*>(x);
  p.wq = static_cast<const uint16_t*>(wq);
  p.ww = static_cast<const uint16_t*>(ww);
  p.q = static_cast<uint16_t*>(q_out);
  p.w = w_out;
  p.T = T;
  p.d_in = d_in;
  p.heads = heads;
  p.nq = heads * d;
  p.nrows = p.nq + (ww ? heads : 0);
  const int ntasks = (p.nrows + kQpRows - 1) / kQpRows;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)std::min((ntasks + 7) / 8, s->num_sms), (unsigned)((T + kQpTok - 1) / kQpTok), 1);
  cfg.blockDim = dim3(kQpThreads, 1, 1);
  cfg.dynamicSmemBytes = (size_t)kQpTok * d_in * 2 + 8 * 32 * 33 * 4;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  set_pdl(attr[0]);
  cfg.attrs = attr;
  cfg.numAttrs = pdl_on() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, indexer_qproj_kernel, p) == cudaSuccess ? DS_OK : DS_ERR_CUDA;
}

extern "C" int ds_indexer_topk_ex(const void* q, const void* kcache, int64_t kcache_batch_stride, const float* w,
                                  int batch, int heads, int d, int S, const int32_t* valid_len, int k,
                                  int sorted_index, int32_t* out_idx, float* out_score, void* stream) {
  int rc = indexer_check(q, kcache, w, batch, heads, d, S);
  if (rc != DS_OK) return rc;
  if (!out_idx || k <= 0 || k > DS_MAX_K || S > kMaxRowElems) return DS_ERR_ARG;
  if (kcache_batch_stride < 0 || (kcache_batch_stride > 0 && kcache_batch_stride < S)) return DS_ERR_ARG;
  if (sorted_index != 0 && sorted_index != 1) return DS_ERR_ARG;
  DeviceState* s = nullptr;
  rc = device_state(&s);
  if (rc != DS_OK) return rc;
  return fused_enqueue(q, kcache, w, batch, heads, S, valid_len, k, sorted_index, out_idx, out_score,
                       (long long)kcache_batch_stride, static_cast<cudaStream_t>(stream), s);
}

extern "C" int ds_compress_fold(const void* rows, int batch, int D, int64_t rows_batch_stride, const void* gate,
                                void* out, int64_t out_batch_stride, void* stream) {
  auto misaligned = [](const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) != 0; };
  if (!rows || !gate || !out || batch <= 0 || batch > (1 << 24)) return DS_ERR_ARG;
  if (D < 8 || D > kCfMaxD || D % 8 != 0) return DS_ERR_ARG;
  if (rows_batch_stride < 4LL * D || rows_batch_stride % 8 != 0) return DS_ERR_ARG;
  if (out_batch_stride < (int64_t)D || out_batch_stride % 8 != 0) return DS_ERR_ARG;
  if (misaligned(rows, 16) || misaligned(gate, 16) || misaligned(out, 16)) return DS_ERR_ARG;
  DeviceState* s = nullptr;
  const int rc = device_state(&s);
  if (rc != DS_OK) return rc;
  CfParams p;
  p.rows = static_cast<const uint16_t*>(rows);
  p.gate = static_cast<const uint16_t*>(gate);
  p.out = static_cast<uint16_t*>(out);
  p.rows_bstride = (long long)rows_batch_stride;
  p.out_bstride = (long long)out_batch_stride;
  p.B = batch;
  p.D = D;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)((batch + kCfWarps - 1) / kCfWarps), 1, 1);
  cfg.blockDim = dim3(kCfWarps * 32, 1, 1);
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[1];
  set_pdl(attr[0]);
  cfg.attrs = attr;
  cfg.numAttrs = pdl_on() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, compress_fold_kernel, p) == cudaSuccess ? DS_OK : DS_ERR_CUDA;
}
