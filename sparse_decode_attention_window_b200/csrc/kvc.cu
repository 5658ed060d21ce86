// libkvc: host side of the C ABI declared in include/kvc.h. Every entry point
// validates its arguments on the host, picks a kernel and launches it on the
// caller's stream; nothing here allocates device memory. All kernels live in
// the headers included below (one translation unit, one device error word).
#include <cstdio>
#include <cstdarg>
#include <cstdlib>
#include <cstring>
#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <string>
#include <tuple>

#include "common.cuh"
#include "score_simt.cuh"
#include "cache.cuh"
#include "score_sm100.cuh"
#include "score_cl.cuh"
#include "select.cuh"
#include "decode.cuh"
#include "decode_mma.cuh"
#include "decode_tc.cuh"
#include "profile.cuh"

namespace {

thread_local std::string g_last_error;
std::atomic<unsigned long long> g_launches{0};

void count_launches(unsigned n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

kvc_status fail(kvc_status st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return st;
}

kvc_status check_launch(const char* what) {
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(KVC_ERR_CUDA, "%s: launch failed: %s", what, cudaGetErrorString(e));
  g_last_error.clear();
  return KVC_OK;
}

struct DevInfo {
  int sms = 0;
  int cc_major = 0, cc_minor = 0;
  int smem_optin = 0;
};

constexpr int kMaxDevices = 64;
DevInfo g_dev[kMaxDevices];
std::once_flag g_dev_once[kMaxDevices];

kvc_status dev_info(DevInfo** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(KVC_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(KVC_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::call_once(g_dev_once[dev], [dev] {
    cudaDeviceGetAttribute(&g_dev[dev].sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&g_dev[dev].cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&g_dev[dev].cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
    cudaDeviceGetAttribute(&g_dev[dev].smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  });
  *out = &g_dev[dev];
  return KVC_OK;
}

// Opt a kernel in to `bytes` of dynamic shared memory. The attribute is set once per
// (kernel, device) and raised only when a larger size is asked for, so repeated calls
// (and calls made while a stream is being captured into a graph) do no driver work.
std::mutex g_smem_mu;
std::map<std::pair<const void*, int>, size_t> g_smem_set;

template <typename K>
kvc_status set_smem(K kernel, size_t bytes, const char* what) {
  if (bytes <= 48 * 1024) return KVC_OK;
  int dev = 0;
  cudaGetDevice(&dev);
  const auto key = std::make_pair(reinterpret_cast<const void*>(kernel), dev);
  std::lock_guard<std::mutex> lk(g_smem_mu);
  auto it = g_smem_set.find(key);
  if (it != g_smem_set.end() && it->second >= bytes) return KVC_OK;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return fail(KVC_ERR_CUDA, "%s: shared memory %zu B: %s", what, bytes, cudaGetErrorString(e));
  g_smem_set[key] = bytes;
  return KVC_OK;
}

size_t esize(int dtype) { return dtype == KVC_FP32 ? 4 : 2; }

kvc_status check_shape(const kvc_shape* sh, bool need_window) {
  if (!sh) return fail(KVC_ERR_INVALID_ARG, "shape is NULL");
  if (sh->n_slots <= 0 || sh->G <= 0 || sh->d <= 0 || sh->L <= 0)
    return fail(KVC_ERR_SHAPE, "n_slots, G, d, L must be positive (got %d, %d, %d, %d)", sh->n_slots, sh->G,
                sh->d, sh->L);
  if (sh->dtype != KVC_BF16 && sh->dtype != KVC_FP32) return fail(KVC_ERR_INVALID_ARG, "bad dtype %d", sh->dtype);
  if (sh->d != 64 && sh->d != 128) return fail(KVC_ERR_UNSUPPORTED, "head dim %d (supported: 64, 128)", sh->d);
  if (need_window && (sh->w <= 0 || sh->w > sh->L))
    return fail(KVC_ERR_SHAPE, "window w = %d must be in [1, L = %d]", sh->w, sh->L);
  if (sh->n_kv_heads <= 0 || sh->batch <= 0) return fail(KVC_ERR_SHAPE, "n_kv_heads and batch must be positive");
  return KVC_OK;
}

// Kernel-path overrides for cross-checks, set only through kvc_diag_set_path (process-wide;
// all zero = the automatic choice every production call makes). Nothing else changes them.
std::atomic<int> g_diag[KVC_DIAG_KNOBS];

int diag(int knob) { return g_diag[knob].load(std::memory_order_relaxed); }

// bf16 scoring on the CUDA-core kernels
bool force_simt() { return diag(KVC_DIAG_SCORE) == KVC_DIAG_SCORE_SIMT; }
// tensor-core scoring in its two-launch form (pass 1, merge, pass 2)
bool force_two_pass_score() { return diag(KVC_DIAG_SCORE) == KVC_DIAG_SCORE_TWO_PASS; }
// tensor-core scoring in its earlier slot-cluster form with 128-key tiles (both passes in one
// launch, few slots), else two-launch
bool force_cluster_score() { return diag(KVC_DIAG_SCORE) == KVC_DIAG_SCORE_CLUSTER; }
// CTAs per slot of the slot-cluster scoring (0: chosen from the shape)
int diag_cluster_k() { return diag(KVC_DIAG_SCORE_K); }
// selection at one CTA per slot where slot clusters would run
bool force_cta_select() { return diag(KVC_DIAG_SELECT) == KVC_DIAG_SELECT_CTA; }
// the grid-stride compaction kernel instead of the one-wave kernel
bool force_old_compact() { return diag(KVC_DIAG_COMPACT) == KVC_DIAG_COMPACT_GRID; }
// bf16 decode on the CUDA-core kernel
bool force_simt_decode() { return diag(KVC_DIAG_DECODE) == KVC_DIAG_DECODE_SIMT; }
// bf16, d = 128 decode on the tcgen05 kernel (decode_tc.cuh: slower than the mma.sync
// kernel on B200, kept as a cross-check and measurement path)
bool force_tc_decode() { return diag(KVC_DIAG_DECODE) == KVC_DIAG_DECODE_TC; }
// the token-range decode split even for few slots
bool force_token_split() { return diag(KVC_DIAG_DECODE_SPLIT) == KVC_DIAG_SPLIT_TOKENS; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---- workspace layouts
struct ScoreWs {
  size_t part_off, part_bytes;   // float2 partial row statistics
  size_t lse_off, lse_bytes;     // float per window row
  size_t keys_off, keys_bytes;   // gathered chunk keys (tensor-core path)
  size_t total;
};

ScoreWs score_ws_layout(const kvc_shape* sh, int C, int sms) {
  const int R = sh->G * sh->w;
  const long long N = C > 0 ? C : sh->L;
  const long long nblk_simt = (N + kvc::SIMT_TB - 1) / kvc::SIMT_TB;
  const long long nsplit_tc = kvc::tc_num_splits(sh->n_slots, N, sms);
  const long long nparts = nblk_simt > nsplit_tc ? nblk_simt : nsplit_tc;
  ScoreWs w{};
  w.part_off = 0;
  w.part_bytes = align_up((size_t)sh->n_slots * nparts * R * sizeof(float2), 256);
  w.lse_off = w.part_off + w.part_bytes;
  w.lse_bytes = align_up((size_t)sh->n_slots * R * sizeof(float), 256);
  w.keys_off = w.lse_off + w.lse_bytes;
  w.keys_bytes = C > 0 ? align_up((size_t)sh->n_slots * C * sh->d * esize(sh->dtype), 256) : 0;
  w.total = w.keys_off + w.keys_bytes;
  return w;
}

struct DecodeWs {
  size_t part_off, part_bytes, cnt_off, cnt_bytes, total;
};

DecodeWs decode_ws_layout(const kvc_shape* sh, int sms) {
  DecodeWs w{};
  w.cnt_off = 0;
  w.cnt_bytes = align_up((size_t)(sh->n_slots + 1) * sizeof(int), 256);
  w.part_off = w.cnt_bytes;
  w.part_bytes = align_up((size_t)(sms + sh->n_slots) * kvc::partial_stride(sh->G, sh->d) * sizeof(float), 256);
  w.total = w.part_off + w.part_bytes;
  return w;
}

// ---- decode dispatch
template <typename T, int D, int G>
kvc_status launch_decode(const kvc::DecodeParams& p, int sms, cudaStream_t st) {
  using namespace kvc;
  const size_t smem = decode_smem_bytes<T, D, G>(p.S, sms);
  DevInfo* di = nullptr;
  if (dev_info(&di) != KVC_OK) return KVC_ERR_CUDA;
  if (smem > (size_t)di->smem_optin)
    return fail(KVC_ERR_UNSUPPORTED, "kvc_decode_attn: %d slots need %zu B of shared memory (> %d)", p.S, smem,
                di->smem_optin);
  kvc_status rc = set_smem(decode_kernel<T, D, G>, smem, "kvc_decode_attn");
  if (rc != KVC_OK) return rc;
  decode_kernel<T, D, G><<<sms, DecCfg<T, D, G>::THREADS, smem, st>>>(p);
  count_launches(1);
  return check_launch("kvc_decode_attn");
}

// How many clusters of k decode CTAs can be resident at once (shared memory per SM, GPC
// sizes: a cluster never spans GPCs, so a GPC whose SM count k does not divide leaves SMs
// idle)? Asked once per (k, device); every decode CTA takes a whole SM's shared memory,
// so the answer does not depend on the exact size.
template <int D, bool PACK>
int max_active_clusters(int k, size_t smem, int sms) {
  static std::mutex mu;
  static std::map<std::pair<int, int>, int> known;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  auto it = known.find({k, dev});
  if (it != known.end()) return it->second;
  int n = 0;
  if (set_smem(kvc::decode_mma_kernel<D, PACK>, smem, "cluster check") == KVC_OK) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((sms / k) * k);
    cfg.blockDim = dim3(kvc::DmCfg<D>::THREADS);
    cfg.dynamicSmemBytes = smem;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = k;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaOccupancyMaxActiveClusters(&n, kvc::decode_mma_kernel<D, PACK>, &cfg) != cudaSuccess) n = 0;
    cudaGetLastError();
  }
  known[{k, dev}] = n;
  return n;
}

// bf16: tensor-core decode (any G <= 8), K/V tiles by TMA through 2-D tensor maps of kp / vp.
// Few slots (2 S <= SMs): clusters of k <= min(8, SMs / S) CTAs, one per slot, when the
// kernel finds the lengths near uniform; otherwise the token-range split over the grid.
template <int D, bool PACK>
kvc_status launch_decode_mma(const kvc::DecodeParams& p, int G, int sms, cudaStream_t st, bool allow_cluster) {
  using namespace kvc;
  DevInfo* di = nullptr;
  if (dev_info(&di) != KVC_OK) return KVC_ERR_CUDA;
  // cluster size for the per-slot mode (the kernel decides from the lengths whether to
  // use it). The grid is the resident clusters, at most SMs / k of them; a size is kept
  // only when the slot-count half of the kernel's test can pass (S k <= grid <= 4/3 S k),
  // otherwise the launch is a plain one CTA per SM.
  if (p.kp_rows > INT32_MAX)   // TMA row coordinates are 32-bit
    return fail(KVC_ERR_UNSUPPORTED, "kvc_decode_attn: %lld cache rows (> 2^31 - 1)", (long long)p.kp_rows);
  int k = p.S > 0 ? sms / p.S : 0;
  if (k > DM_MAX_CLUSTER) k = DM_MAX_CLUSTER;
  if (!allow_cluster || force_token_split()) k = 1;
  const size_t optin = (size_t)di->smem_optin - 2048;   // room for the kernel's static shared memory
  const size_t smem_max = decode_mma_smem_bytes<D>(p.S, G, sms, 4);   // any grid <= SMs, 4 stages
  if (smem_max > optin)
    return fail(KVC_ERR_UNSUPPORTED, "kvc_decode_attn: %d slots need %zu B of shared memory (> %d)", p.S, smem_max,
                di->smem_optin);
  int grid = sms;
  for (; k >= 2; k /= 2) {
    const int n = std::min(sms / k, max_active_clusters<D, PACK>(k, smem_max, sms));
    const long long g = (long long)n * k, sk = (long long)p.S * k;
    if (n >= 1 && sk <= g && 4 * sk >= 3 * g) {
      grid = (int)g;
      break;
    }
  }
  const bool cluster = k >= 2;
  // Four stages of 64 tokens: six measured slower on B200 (137 vs 131 us for 865 MB). The
  // count must be even: the two consumer groups take alternate tiles, so with an even count
  // every stage always serves the same group and each group waits on every phase of its
  // stages' barriers.
  const int nst = 4;
  const size_t smem = decode_mma_smem_bytes<D>(p.S, G, grid, nst);
  encode_tiled_fn enc = get_encode_tiled();
  CUtensorMap mk64, mk16, mv64, mv16;
  const long long rows = p.kp_rows > 0 ? p.kp_rows : 1;
  if (!enc || !make_map_2d_rows(&mk64, enc, p.kp, D, rows, 64) || !make_map_2d_rows(&mk16, enc, p.kp, D, rows, 16) ||
      !make_map_2d_rows(&mv64, enc, p.vp, D, rows, 64) || !make_map_2d_rows(&mv16, enc, p.vp, D, rows, 16))
    return fail(KVC_ERR_CUDA, "kvc_decode_attn: cuTensorMapEncodeTiled failed");
  // programmatic dependent launch: this grid may be scheduled while the previous kernel
  // on the stream finishes; the kernel waits (griddepcontrol.wait) before reading inputs
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(DmCfg<D>::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = cluster ? k : 1;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster ? 2 : 1;
  kvc_status rc = set_smem(decode_mma_kernel<D, PACK>, std::max(smem, smem_max), "kvc_decode_attn");
  if (rc != KVC_OK) return rc;
  cudaError_t e = cudaLaunchKernelEx(&cfg, decode_mma_kernel<D, PACK>, mk64, mk16, mv64, mv16, p, G, cluster ? k : 1, nst);
  if (e != cudaSuccess) return fail(KVC_ERR_CUDA, "kvc_decode_attn: launch: %s", cudaGetErrorString(e));
  count_launches(1);
  return check_launch("kvc_decode_attn");
}

// bf16, d = 128: decode on tcgen05 (decode_tc.cuh), same work split as above; three
// pipeline stages when they fit in shared memory, else two. Returns KVC_ERR_UNSUPPORTED
// (without launching) when not even two fit, and the caller takes the mma.sync kernel.
kvc_status launch_decode_tc(const kvc::DecodeParams& p, int G, int sms, cudaStream_t st, bool allow_cluster) {
  using namespace kvc;
  DevInfo* di = nullptr;
  if (dev_info(&di) != KVC_OK) return KVC_ERR_CUDA;
  int k = p.S > 0 ? sms / p.S : 0;
  if (k > DM_MAX_CLUSTER) k = DM_MAX_CLUSTER;
  if (!allow_cluster || force_token_split()) k = 1;
  auto total = [&](int grid, int ksz, int nst) { return DtLayout::make(p.S, G, grid, ksz, nst).total; };
  // the largest layout any launch below can take (grid <= SMs, records of up to 8 CTAs)
  const size_t smem_max2 = total(sms, DM_MAX_CLUSTER, 2);
  const size_t optin = (size_t)di->smem_optin - 2048;   // room for the kernel's static shared memory
  if (smem_max2 > optin) return KVC_ERR_UNSUPPORTED;
  int grid = sms;
  for (; k >= 2; k /= 2) {
    static std::mutex mu;
    static std::map<std::pair<int, int>, int> known;   // (k, device) -> resident clusters
    int dev = 0, n = 0;
    cudaGetDevice(&dev);
    {
      std::lock_guard<std::mutex> lk(mu);
      auto it = known.find({k, dev});
      if (it != known.end()) {
        n = it->second;
      } else {
        if (set_smem(decode_tc_kernel, smem_max2, "cluster check") == KVC_OK) {
          cudaLaunchConfig_t cfg = {};
          cfg.gridDim = dim3((sms / k) * k);
          cfg.blockDim = dim3(DtCfg::THREADS);
          cfg.dynamicSmemBytes = smem_max2;
          cudaLaunchAttribute attr[1];
          attr[0].id = cudaLaunchAttributeClusterDimension;
          attr[0].val.clusterDim.x = k;
          attr[0].val.clusterDim.y = 1;
          attr[0].val.clusterDim.z = 1;
          cfg.attrs = attr;
          cfg.numAttrs = 1;
          if (cudaOccupancyMaxActiveClusters(&n, decode_tc_kernel, &cfg) != cudaSuccess) n = 0;
          cudaGetLastError();
        }
        known[{k, dev}] = n;
      }
    }
    n = std::min(sms / k, n);
    const long long g = (long long)n * k, sk = (long long)p.S * k;
    if (n >= 1 && sk <= g && 4 * sk >= 3 * g) {
      grid = (int)g;
      break;
    }
  }
  const bool cluster = k >= 2;
  const int ksz = cluster ? k : 1;
  const int nst = total(grid, ksz, 3) <= optin ? 3 : 2;
  const size_t smem = total(grid, ksz, nst);
  encode_tiled_fn enc = get_encode_tiled();
  CUtensorMap mk, mk16, mv, mv16, mq;
  const long long rows = p.kp_rows > 0 ? p.kp_rows : 1;
  if (!enc || !make_map_2d_rows(&mk, enc, p.kp, 128, rows, 128) || !make_map_2d_rows(&mk16, enc, p.kp, 128, rows, 16) ||
      !make_map_2d_rows(&mv, enc, p.vp, 128, rows, 128) || !make_map_2d_rows(&mv16, enc, p.vp, 128, rows, 16) ||
      !make_map_2d_rows(&mq, enc, p.q, 128, (long long)p.S * G, 16))
    return fail(KVC_ERR_CUDA, "kvc_decode_attn: cuTensorMapEncodeTiled failed");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(DtCfg::THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = ksz;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = cluster ? 2 : 1;
  kvc_status rc = set_smem(decode_tc_kernel, std::max(smem, smem_max2), "kvc_decode_attn");
  if (rc != KVC_OK) return rc;
  cudaError_t e = cudaLaunchKernelEx(&cfg, decode_tc_kernel, mk, mk16, mv, mv16, mq, p, G, ksz, nst);
  if (e != cudaSuccess) return fail(KVC_ERR_CUDA, "kvc_decode_attn: launch: %s", cudaGetErrorString(e));
  count_launches(1);
  return check_launch("kvc_decode_attn");
}

template <typename T, int D>
kvc_status decode_by_g(int G, const kvc::DecodeParams& p, int sms, cudaStream_t st) {
  switch (G) {
    case 1: return launch_decode<T, D, 1>(p, sms, st);
    case 2: return launch_decode<T, D, 2>(p, sms, st);
    case 4: return launch_decode<T, D, 4>(p, sms, st);
    default: return fail(KVC_ERR_UNSUPPORTED, "kvc_decode_attn: G = %d (supported: 1, 2, 4)", G);
  }
}

// bf16 with G <= 8 -> tensor-core decode; otherwise the CUDA-core decode (G in {1, 2, 4}).
// allow_cluster = false keeps the token-range split, whose merge uses the scratch.
kvc_status launch_decode_any(const kvc_shape* shape, const kvc::DecodeParams& p, int sms, cudaStream_t stream,
                             bool allow_cluster = true) {
  if (shape->dtype == KVC_BF16 && shape->G <= 8 && !force_simt_decode()) {
    if (shape->d == 128 && force_tc_decode()) {
      const kvc_status rc = launch_decode_tc(p, shape->G, sms, stream, allow_cluster);
      if (rc != KVC_ERR_UNSUPPORTED) return rc;
    }
    const bool pack = shape->G <= 4;   // heads and the bf16 remainder share one MMA
    kvc_status rc;
    if (shape->d == 128)
      rc = pack ? launch_decode_mma<128, true>(p, shape->G, sms, stream, allow_cluster)
                : launch_decode_mma<128, false>(p, shape->G, sms, stream, allow_cluster);
    else
      rc = pack ? launch_decode_mma<64, true>(p, shape->G, sms, stream, allow_cluster)
                : launch_decode_mma<64, false>(p, shape->G, sms, stream, allow_cluster);
    // very many slots can overflow the tensor-core kernel's shared memory; a plain decode
    // (no fused append) then runs on the CUDA-core kernel where G allows
    const bool simt_ok = shape->G == 1 || shape->G == 2 || shape->G == 4;
    if (rc != KVC_ERR_UNSUPPORTED || p.append || !simt_ok) return rc;
  }
  if (shape->dtype == KVC_BF16) {
    if (shape->d == 128) return decode_by_g<__nv_bfloat16, 128>(shape->G, p, sms, stream);
    return decode_by_g<__nv_bfloat16, 64>(shape->G, p, sms, stream);
  }
  if (shape->d == 128) return decode_by_g<float, 128>(shape->G, p, sms, stream);
  return decode_by_g<float, 64>(shape->G, p, sms, stream);
}

}  // namespace

// ---- scratch for kvc_decode_attn_noalloc
// Fixed device-side scratch for callers that cannot allocate device memory. Every
// GPU that loads this library holds these bytes until the process exits. In host
// code `g_noalloc_scratch` is only a stand-in for the symbol, never a device
// address: the address is fetched per device with cudaGetSymbolAddress below.
#define KVC_NOALLOC_SCRATCH_BYTES (4u << 20)
static __device__ __align__(256) unsigned char g_noalloc_scratch[KVC_NOALLOC_SCRATCH_BYTES];

namespace {
void* g_noalloc_ptr[kMaxDevices];
std::mutex g_noalloc_mu;

// Device address of the scratch array on the current device, looked up by the first
// successful call on that device (make it before any stream capture, since the lookup
// may load the module); a failed lookup is not kept, the next call tries again.
kvc_status noalloc_scratch(unsigned char** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(KVC_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(KVC_ERR_UNSUPPORTED, "device index %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();   // not sticky: leave no error for the next check
      return fail(KVC_ERR_CUDA, "scratch address on device %d: %s", dev, cudaGetErrorString(e));
    }
    g_noalloc_ptr[dev] = p;
  }
  *out = static_cast<unsigned char*>(g_noalloc_ptr[dev]);
  return KVC_OK;
}
}  // namespace

extern "C" {

const char* kvc_last_error(void) { return g_last_error.c_str(); }

const char* kvc_version(void) { return "kvc 0.1 (sm_100a)"; }

unsigned long long kvc_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

size_t kvc_workspace_size(int which, const kvc_shape* shape, int32_t C) {
  if (!shape || shape->n_slots <= 0) return 0;
  DevInfo* di = nullptr;
  int sms = 148;
  if (dev_info(&di) == KVC_OK && di->sms > 0) sms = di->sms;
  switch (which) {
    case KVC_WS_SCORE: return score_ws_layout(shape, C, sms).total;
    case KVC_WS_SELECT: return 0;
    case KVC_WS_DECODE: return decode_ws_layout(shape, sms).total;
    default: return 0;
  }
}

kvc_status kvc_get_status(cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return fail(KVC_ERR_CUDA, "stream synchronize: %s", cudaGetErrorString(e));
  unsigned int word = 0, zero = 0;
  e = cudaMemcpyFromSymbol(&word, g_kvc_deverr, sizeof(word));
  if (e != cudaSuccess) return fail(KVC_ERR_CUDA, "read error word: %s", cudaGetErrorString(e));
  if (word == 0) {
    g_last_error.clear();
    return KVC_OK;
  }
  cudaMemcpyToSymbol(g_kvc_deverr, &zero, sizeof(zero));
  return fail(KVC_ERR_DEVICE, "device error word 0x%x:%s%s%s%s", word,
              (word & KVC_DEVERR_APPEND_OVERFLOW) ? " append-overflow" : "",
              (word & KVC_DEVERR_INDEX_RANGE) ? " index-out-of-range" : "",
              (word & KVC_DEVERR_WAIT_TIMEOUT) ? " wait-timeout" : "",
              (word & KVC_DEVERR_WORKSPACE) ? " workspace" : "");
}

kvc_status kvc_score(const kvc_shape* shape, const void* q_win, const void* k, const int32_t* chunk_end, int32_t C,
                     const float* row_lse, float* score, void* ws, size_t ws_bytes, cudaStream_t stream) {
  kvc_status rc = check_shape(shape, true);
  if (rc != KVC_OK) return rc;
  if (!q_win || !k || !score) return fail(KVC_ERR_INVALID_ARG, "kvc_score: q_win, k and score must be non-NULL");
  if (chunk_end && (C <= 0 || C > shape->L))
    return fail(KVC_ERR_SHAPE, "kvc_score: chunk count C = %d must be in [1, L]", C);
  const int R = shape->G * shape->w;
  if (R > 256) return fail(KVC_ERR_UNSUPPORTED, "kvc_score: G*w = %d > 256", R);
  DevInfo* di = nullptr;
  if ((rc = dev_info(&di)) != KVC_OK) return rc;
  const int Cc = chunk_end ? C : 0;
  const ScoreWs w = score_ws_layout(shape, Cc, di->sms);
  if (!ws || ws_bytes < w.total)
    return fail(KVC_ERR_WORKSPACE, "kvc_score: workspace %zu B < required %zu B", ws_bytes, w.total);
  if (!aligned16(q_win) || !aligned16(k) || !aligned16(ws))
    return fail(KVC_ERR_INVALID_ARG, "kvc_score: q_win, k and ws must be 16-byte aligned");
  unsigned char* wsb = static_cast<unsigned char*>(ws);
  float2* part = reinterpret_cast<float2*>(wsb + w.part_off);
  float* lse = reinterpret_cast<float*>(wsb + w.lse_off);
  const int N = chunk_end ? C : shape->L;
  const float scale = 1.0f / sqrtf((float)shape->d);
  const int S = shape->n_slots, d = shape->d;

  if (kvc::tc_supported(shape, di->cc_major, di->cc_minor) && !force_simt()) {
    unsigned nl = 0;
    if (force_two_pass_score() || force_cluster_score() || !kvc::cl_takes(shape, Cc, di->sms, diag_cluster_k()))
      rc = kvc::tc_score(shape, q_win, k, chunk_end, C, row_lse, score, part, lse, wsb + w.keys_off, di->sms, stream,
                         &fail, &nl, force_two_pass_score());
    else
      rc = kvc::tc_score_cl(shape, q_win, k, chunk_end, C, row_lse, score, lse, wsb + w.keys_off, di->sms, stream,
                            &fail, &nl, diag_cluster_k());
    count_launches(nl);
    if (rc != KVC_OK) return rc;
    return check_launch("kvc_score");
  }

  // CUDA-core path: stats + merge + column sums (or column sums alone given row_lse)
  count_launches(row_lse ? 1 : 3);
  const int nblk = (N + kvc::SIMT_TB - 1) / kvc::SIMT_TB;
  const size_t sm1 = ((size_t)R * d + (size_t)kvc::SIMT_TB * (d + 1)) * sizeof(float);
  const size_t sm2 = sm1 + (size_t)R * sizeof(float) + kvc::SIMT_THREADS * sizeof(float);
  dim3 grid(nblk, S);
  if (shape->dtype == KVC_FP32) {
    const float* q = static_cast<const float*>(q_win);
    const float* kk = static_cast<const float*>(k);
    if (!row_lse) {
      if ((rc = set_smem(kvc::score_stats_simt<float>, sm1, "kvc_score")) != KVC_OK) return rc;
      kvc::score_stats_simt<float><<<grid, kvc::SIMT_THREADS, sm1, stream>>>(q, kk, chunk_end, N, shape->L,
                                                                              shape->G, shape->w, d, scale, part);
      kvc::score_lse_merge<<<S, 256, 0, stream>>>(part, nblk, R, lse);
    }
    if ((rc = set_smem(kvc::score_colsum_simt<float>, sm2, "kvc_score")) != KVC_OK) return rc;
    kvc::score_colsum_simt<float><<<grid, kvc::SIMT_THREADS, sm2, stream>>>(
        q, kk, chunk_end, N, shape->L, shape->G, shape->w, d, scale, row_lse ? row_lse : lse, score);
  } else {
    const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(q_win);
    const __nv_bfloat16* kk = static_cast<const __nv_bfloat16*>(k);
    if (!row_lse) {
      if ((rc = set_smem(kvc::score_stats_simt<__nv_bfloat16>, sm1, "kvc_score")) != KVC_OK) return rc;
      kvc::score_stats_simt<__nv_bfloat16><<<grid, kvc::SIMT_THREADS, sm1, stream>>>(
          q, kk, chunk_end, N, shape->L, shape->G, shape->w, d, scale, part);
      kvc::score_lse_merge<<<S, 256, 0, stream>>>(part, nblk, R, lse);
    }
    if ((rc = set_smem(kvc::score_colsum_simt<__nv_bfloat16>, sm2, "kvc_score")) != KVC_OK) return rc;
    kvc::score_colsum_simt<__nv_bfloat16><<<grid, kvc::SIMT_THREADS, sm2, stream>>>(
        q, kk, chunk_end, N, shape->L, shape->G, shape->w, d, scale, row_lse ? row_lse : lse, score);
  }
  return check_launch("kvc_score");
}

// Selection launch. Few slots: a cluster of k CTAs per slot (select_cluster_kernel), k the
// largest power of two <= 16 with all S*k CTAs in one wave, at least 128 keys per CTA and
// each CTA's key range in shared memory; otherwise one CTA per slot (select_kernel).
int select_cluster_size(int S, int N, int sms, int optin, int* cap_out, size_t* smem_out) {
  if (force_cta_select()) return 1;
  for (int k = kvc::SCL_MAX_K; k >= 2; k >>= 1) {
    if ((long long)S * k > sms) continue;
    const int per = (N + k - 1) / k;
    if (per < 128) continue;
    const int cap = (per + 3) & ~3;
    const size_t smem = kvc::select_cluster_smem_bytes(cap);
    if (smem > (size_t)optin) continue;
    static std::mutex mu;
    static std::map<std::tuple<int, int, size_t>, int> known;
    int dev = 0;
    cudaGetDevice(&dev);
    int n = 0;
    {
      std::lock_guard<std::mutex> lk(mu);
      auto it = known.find({k, dev, smem});
      if (it != known.end()) {
        n = it->second;
      } else {
        // (set_smem only ever raises the kernel's limit, which launches of other sizes rely on)
        if (set_smem(kvc::select_cluster_kernel, smem, "kvc_select") != KVC_OK) cudaGetLastError();
        if (k > 8) cudaFuncSetAttribute(kvc::select_cluster_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(k);
        cfg.blockDim = dim3(kvc::SCL_THREADS);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = k;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        if (cudaOccupancyMaxActiveClusters(&n, kvc::select_cluster_kernel, &cfg) != cudaSuccess) n = 0;
        cudaGetLastError();
        known[{k, dev, smem}] = n;
      }
    }
    if (n < S) continue;
    *cap_out = cap;
    *smem_out = smem;
    return k;
  }
  return 1;
}

kvc_status launch_select(kvc::SelectParams p, int S, int N, cudaStream_t stream, const char* what) {
  DevInfo* di = nullptr;
  kvc_status rc = dev_info(&di);
  if (rc != KVC_OK) return rc;
  int cap = 0;
  size_t smem = 0;
  const int k = select_cluster_size(S, N, di->sms, di->smem_optin, &cap, &smem);
  if (k >= 2) {
    p.key_cap = cap;
    if ((rc = set_smem(kvc::select_cluster_kernel, smem, what)) != KVC_OK) return rc;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(S * k);
    cfg.blockDim = dim3(kvc::SCL_THREADS);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = k;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kvc::select_cluster_kernel, p);
    if (e != cudaSuccess) {
      cudaGetLastError();                 // not sticky: leave no error for the next check
      return fail(KVC_ERR_CUDA, "%s: launch: %s", what, cudaGetErrorString(e));
    }
  } else {
    // More slots than SMs: no key cache and 512-thread CTAs, so two share an SM (64
    // registers a thread) and the slots run in one wave, the scores re-read from L2 each
    // pass; otherwise one 1024-thread CTA per slot caches its keys.
    const bool many = S > di->sms;
    p.key_cap = many ? 0 : kvc::select_key_cap(p.L, p.C);
    smem = kvc::select_smem_bytes(p.key_cap);
    if ((rc = set_smem(kvc::select_kernel, smem, what)) != KVC_OK) return rc;
    kvc::select_kernel<<<S, many ? kvc::SEL_THREADS / 2 : kvc::SEL_THREADS, smem, stream>>>(p);
  }
  count_launches(1);
  return check_launch(what);
}

kvc_status kvc_select(const kvc_shape* shape, const float* score, const int8_t* policy, const int32_t* budget,
                      float mass, const uint8_t* special_mask, const int32_t* chunk_end, int32_t C, int32_t* idx,
                      int32_t max_sel, int32_t* count, void* ws, size_t ws_bytes, cudaStream_t stream) {
  (void)ws;
  (void)ws_bytes;
  kvc_status rc = check_shape(shape, false);
  if (rc != KVC_OK) return rc;
  if (!policy || !budget || !count) return fail(KVC_ERR_INVALID_ARG, "kvc_select: policy, budget, count must be non-NULL");
  if (max_sel < 0) return fail(KVC_ERR_SHAPE, "kvc_select: max_sel < 0");
  if (!(mass > 0.f && mass <= 1.f)) return fail(KVC_ERR_INVALID_ARG, "kvc_select: mass %g not in (0, 1]", mass);
  if (chunk_end && (C <= 0 || C > shape->L)) return fail(KVC_ERR_SHAPE, "kvc_select: C = %d not in [1, L]", C);
  // The policy array is on the device; the kernel reads it. Pointers a policy may
  // need are checked for presence here; a slot whose policy needs a missing
  // pointer would read NULL, so the caller states which kinds occur via the pointers.
  kvc::SelectParams p{};
  p.score = score;
  p.policy = policy;
  p.budget = budget;
  p.mass = mass;
  p.special_mask = special_mask;
  p.chunk_end = chunk_end;
  p.C = chunk_end ? C : 0;
  p.L = shape->L;
  p.n_kv_heads = shape->n_kv_heads;
  p.batch = shape->batch;
  p.idx = idx;
  p.max_sel = max_sel;
  p.count = count;
  p.n_local = 0;
  return launch_select(p, shape->n_slots, std::max(shape->L, p.C), stream, "kvc_select");
}

namespace kvc {
// One thread waits on a barrier that nothing arrives on, with the same bounded wait every
// pipeline of the library uses (only the limit differs): it gives up, flags the timeout and
// the kernel returns.
__global__ void wait_limit_probe_kernel(unsigned long long limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait_limit(&bar, 0, limit_ns);
}
}  // namespace kvc

kvc_status kvc_diag_set_path(int32_t knob, int32_t choice) {
  static const int n_choices[KVC_DIAG_KNOBS] = {4, 2, 2, 3, 2, 17};
  if (knob < 0 || knob >= KVC_DIAG_KNOBS) return fail(KVC_ERR_INVALID_ARG, "kvc_diag_set_path: unknown knob %d", knob);
  if (choice < 0 || choice >= n_choices[knob])
    return fail(KVC_ERR_INVALID_ARG, "kvc_diag_set_path: choice %d not in [0, %d) for knob %d", choice,
                n_choices[knob], knob);
  g_diag[knob].store(choice, std::memory_order_relaxed);
  g_last_error.clear();
  return KVC_OK;
}

int32_t kvc_diag_get_path(int32_t knob) {
  if (knob < 0 || knob >= KVC_DIAG_KNOBS) return -1;
  return diag(knob);
}

kvc_status kvc_check_wait_limit(int32_t limit_us, cudaStream_t stream) {
  if (limit_us < 1 || limit_us > 1000000)
    return fail(KVC_ERR_INVALID_ARG, "kvc_check_wait_limit: limit_us = %d not in [1, 1e6]", limit_us);
  kvc::wait_limit_probe_kernel<<<1, 32, 0, stream>>>((unsigned long long)limit_us * 1000ull);
  count_launches(1);
  return check_launch("kvc_check_wait_limit");
}

kvc_status kvc_alloc_budgets(const int32_t* counts, int32_t n_layers, int32_t spl, int32_t L, int32_t avg_B,
                             int32_t floor_B, int32_t* budgets, int32_t* slot_budgets, cudaStream_t stream) {
  if (!counts || !budgets) return fail(KVC_ERR_INVALID_ARG, "kvc_alloc_budgets: counts and budgets must be non-NULL");
  if (n_layers <= 0 || n_layers > 1024 || spl <= 0 || L <= 0)
    return fail(KVC_ERR_SHAPE, "kvc_alloc_budgets: need 1 <= n_layers <= 1024, spl >= 1, L >= 1");
  if (!(0 <= floor_B && floor_B <= avg_B && avg_B <= L))
    return fail(KVC_ERR_SHAPE, "kvc_alloc_budgets: need 0 <= floor_B (%d) <= avg_B (%d) <= L (%d)", floor_B, avg_B, L);
  kvc::alloc_kernel<<<1, 1024, 0, stream>>>(counts, n_layers, spl, L, avg_B, floor_B, budgets, slot_budgets);
  count_launches(1);
  return check_launch("kvc_alloc_budgets");
}

kvc_status kvc_layout(const int32_t* count, int32_t n_slots, int32_t reserve, int64_t* off, int32_t* cap,
                      cudaStream_t stream) {
  if (!count || !off || !cap) return fail(KVC_ERR_INVALID_ARG, "kvc_layout: count, off, cap must be non-NULL");
  if (n_slots <= 0 || reserve < 0) return fail(KVC_ERR_SHAPE, "kvc_layout: n_slots > 0 and reserve >= 0 required");
  kvc::layout_kernel<<<1, 1024, 0, stream>>>(count, n_slots, reserve, off, cap);
  count_launches(1);
  return check_launch("kvc_layout");
}

// Compaction, after the layout (off given) or, with `layout`, computing it in the same launch
// (off_out and cap_out written; S <= CP_MAX_SLOTS on the one-wave kernel).
static kvc_status launch_compact(const char* what, const kvc_shape* shape, const void* k, const void* v,
                                 const int32_t* idx, int32_t max_sel, const int32_t* count, const int64_t* off,
                                 void* kp, void* vp, int64_t kp_rows, int32_t* len, bool layout, int32_t reserve,
                                 int64_t* off_out, int32_t* cap_out, cudaStream_t stream) {
  kvc_status rc = check_shape(shape, false);
  if (rc != KVC_OK) return rc;
  if (!k || !v || !idx || !count || !(layout ? off_out && cap_out : off != nullptr) || !kp || !vp || !len)
    return fail(KVC_ERR_INVALID_ARG, "%s: NULL pointer argument", what);
  if (max_sel <= 0 || kp_rows < 0) return fail(KVC_ERR_SHAPE, "%s: max_sel > 0, kp_rows >= 0 required", what);
  if (layout && reserve < 0) return fail(KVC_ERR_SHAPE, "%s: reserve >= 0 required", what);
  if (!aligned16(k) || !aligned16(v) || !aligned16(kp) || !aligned16(vp))
    return fail(KVC_ERR_INVALID_ARG, "%s: k, v, kp, vp must be 16-byte aligned", what);
  DevInfo* di = nullptr;
  if ((rc = dev_info(&di)) != KVC_OK) return rc;
  const int tpr = (int)(shape->d * esize(shape->dtype) / 16);
  if (tpr != 8 && tpr != 16 && tpr != 32) return fail(KVC_ERR_UNSUPPORTED, "%s: row of %d bytes", what, tpr * 16);
  const uint4* k4 = static_cast<const uint4*>(k);
  const uint4* v4 = static_cast<const uint4*>(v);
  uint4* kp4 = static_cast<uint4*>(kp);
  uint4* vp4 = static_cast<uint4*>(vp);
  const int S = shape->n_slots, L = shape->L;
  if (layout && (S > kvc::CP_MAX_SLOTS || force_old_compact())) {
    // more slots than one CTA stages: the layout kernel first, then the plain compaction
    if ((rc = kvc_layout(count, S, reserve, off_out, cap_out, stream)) != KVC_OK) return rc;
    return launch_compact(what, shape, k, v, idx, max_sel, count, off_out, kp, vp, kp_rows, len, false, 0, nullptr,
                          nullptr, stream);
  }
  if (!force_old_compact()) {
    const int blocks = di->sms * 4;   // one wave at four CTAs per SM
#define KVC_COMPACT_WAVE(T, LY)                                                                                  \
  kvc::compact_wave_kernel<T, LY><<<blocks, kvc::CP_THREADS, 0, stream>>>(k4, v4, idx, max_sel, count, off, S, L, \
                                                                          kp4, vp4, kp_rows, len, reserve, off_out, \
                                                                          cap_out)
    if (layout) {
      if (tpr == 8) KVC_COMPACT_WAVE(8, true);
      else if (tpr == 16) KVC_COMPACT_WAVE(16, true);
      else KVC_COMPACT_WAVE(32, true);
    } else {
      if (tpr == 8) KVC_COMPACT_WAVE(8, false);
      else if (tpr == 16) KVC_COMPACT_WAVE(16, false);
      else KVC_COMPACT_WAVE(32, false);
    }
#undef KVC_COMPACT_WAVE
  } else {
    const int blocks = di->sms * 8;
    switch (tpr) {
      case 8: kvc::compact_kernel<8, 4><<<blocks, 256, 0, stream>>>(k4, v4, idx, max_sel, count, off, S, L, kp4, vp4,
                                                                     kp_rows, len); break;
      case 16: kvc::compact_kernel<16, 4><<<blocks, 256, 0, stream>>>(k4, v4, idx, max_sel, count, off, S, L, kp4,
                                                                       vp4, kp_rows, len); break;
      default: kvc::compact_kernel<32, 4><<<blocks, 256, 0, stream>>>(k4, v4, idx, max_sel, count, off, S, L, kp4,
                                                                       vp4, kp_rows, len); break;
    }
  }
  count_launches(1);
  return check_launch(what);
}

kvc_status kvc_compact(const kvc_shape* shape, const void* k, const void* v, const int32_t* idx, int32_t max_sel,
                       const int32_t* count, const int64_t* off, void* kp, void* vp, int64_t kp_rows, int32_t* len,
                       cudaStream_t stream) {
  return launch_compact("kvc_compact", shape, k, v, idx, max_sel, count, off, kp, vp, kp_rows, len, false, 0, nullptr,
                        nullptr, stream);
}

kvc_status kvc_layout_compact(const kvc_shape* shape, const void* k, const void* v, const int32_t* idx,
                              int32_t max_sel, const int32_t* count, int32_t reserve, int64_t* off, int32_t* cap,
                              void* kp, void* vp, int64_t kp_rows, int32_t* len, cudaStream_t stream) {
  return launch_compact("kvc_layout_compact", shape, k, v, idx, max_sel, count, nullptr, kp, vp, kp_rows, len, true,
                        reserve, off, cap, stream);
}

kvc_status kvc_append_window(const kvc_shape* shape, const void* k_new, const void* v_new, const int64_t* off,
                             const int32_t* cap, int32_t* len, const int32_t* window, int32_t* head, void* kp,
                             void* vp, int64_t kp_rows, cudaStream_t stream) {
  kvc_status rc = check_shape(shape, false);
  if (rc != KVC_OK) return rc;
  if (!k_new || !v_new || !off || !cap || !len || !window || !head || !kp || !vp)
    return fail(KVC_ERR_INVALID_ARG, "kvc_append_window: NULL pointer argument");
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(kp) || !aligned16(vp))
    return fail(KVC_ERR_INVALID_ARG, "kvc_append_window: buffers must be 16-byte aligned");
  const int tpr = (int)(shape->d * esize(shape->dtype) / 16);
  kvc::append_window_kernel<<<shape->n_slots, tpr, 0, stream>>>(
      static_cast<const uint4*>(k_new), static_cast<const uint4*>(v_new), off, cap, len, window, head,
      static_cast<uint4*>(kp), static_cast<uint4*>(vp), kp_rows, tpr);
  count_launches(1);
  return check_launch("kvc_append_window");
}

kvc_status kvc_append(const kvc_shape* shape, const void* k_new, const void* v_new, const int64_t* off,
                      const int32_t* cap, int32_t* len, void* kp, void* vp, int64_t kp_rows, cudaStream_t stream) {
  kvc_status rc = check_shape(shape, false);
  if (rc != KVC_OK) return rc;
  if (!k_new || !v_new || !off || !cap || !len || !kp || !vp)
    return fail(KVC_ERR_INVALID_ARG, "kvc_append: NULL pointer argument");
  if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(kp) || !aligned16(vp))
    return fail(KVC_ERR_INVALID_ARG, "kvc_append: buffers must be 16-byte aligned");
  const int tpr = (int)(shape->d * esize(shape->dtype) / 16);
  kvc::append_kernel<<<shape->n_slots, tpr, 0, stream>>>(static_cast<const uint4*>(k_new),
                                                          static_cast<const uint4*>(v_new), off, cap, len,
                                                          static_cast<uint4*>(kp), static_cast<uint4*>(vp), kp_rows,
                                                          tpr);
  count_launches(1);
  return check_launch("kvc_append");
}

kvc_status kvc_decode_attn(const kvc_shape* shape, const void* q, const void* kp, const void* vp, const int64_t* off,
                           const int32_t* len, int64_t kp_rows, float* out, void* ws, size_t ws_bytes,
                           cudaStream_t stream) {
  kvc_status rc = check_shape(shape, false);
  if (rc != KVC_OK) return rc;
  if (!q || !kp || !vp || !off || !len || !out) return fail(KVC_ERR_INVALID_ARG, "kvc_decode_attn: NULL pointer argument");
  if (shape->n_slots > kvc::DEC_MAX_SLOTS)
    return fail(KVC_ERR_UNSUPPORTED, "kvc_decode_attn: %d slots > %d", shape->n_slots, kvc::DEC_MAX_SLOTS);
  if (!aligned16(q) || !aligned16(kp) || !aligned16(vp) || !aligned16(ws) || !aligned16(out))
    return fail(KVC_ERR_INVALID_ARG, "kvc_decode_attn: q, kp, vp, out, ws must be 16-byte aligned");
  DevInfo* di = nullptr;
  if ((rc = dev_info(&di)) != KVC_OK) return rc;
  const DecodeWs w = decode_ws_layout(shape, di->sms);
  if (!ws || ws_bytes < w.total)
    return fail(KVC_ERR_WORKSPACE, "kvc_decode_attn: workspace %zu B < required %zu B", ws_bytes, w.total);
  unsigned char* wsb = static_cast<unsigned char*>(ws);
  kvc::DecodeParams p{};
  p.q = q;
  p.kp = kp;
  p.vp = vp;
  p.off = off;
  p.len = len;
  p.kp_rows = kp_rows;
  p.S = shape->n_slots;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)shape->d);
  p.out = out;
  p.partial = reinterpret_cast<float*>(wsb + w.part_off);
  p.counters = reinterpret_cast<int*>(wsb + w.cnt_off);
  return launch_decode_any(shape, p, di->sms, stream);
}

// Decode attention without a caller workspace: the kvc_decode_attn kernel in its
// token-range split (whose merge goes through the scratch), with the scratch in the
// fixed array above. Allocates nothing.
kvc_status kvc_decode_attn_noalloc(const kvc_shape* shape, const void* q, const void* kp, const void* vp,
                                   const int64_t* off, const int32_t* len, int64_t kp_rows, float* out,
                                   cudaStream_t stream) {
  kvc_status rc = check_shape(shape, false);
  if (rc != KVC_OK) return rc;
  if (!q || !kp || !vp || !off || !len || !out)
    return fail(KVC_ERR_INVALID_ARG, "kvc_decode_attn_noalloc: NULL pointer argument");
  if (shape->n_slots > kvc::DEC_MAX_SLOTS)
    return fail(KVC_ERR_UNSUPPORTED, "kvc_decode_attn_noalloc: %d slots > %d", shape->n_slots, kvc::DEC_MAX_SLOTS);
  if (!aligned16(q) || !aligned16(kp) || !aligned16(vp) || !aligned16(out))
    return fail(KVC_ERR_INVALID_ARG, "kvc_decode_attn_noalloc: q, kp, vp, out must be 16-byte aligned");
  DevInfo* di = nullptr;
  if ((rc = dev_info(&di)) != KVC_OK) return rc;
  const DecodeWs w = decode_ws_layout(shape, di->sms);
  if (w.total > KVC_NOALLOC_SCRATCH_BYTES)
    return fail(KVC_ERR_WORKSPACE,
                "kvc_decode_attn_noalloc: this shape needs %zu B of scratch; the fixed array holds %u B "
                "(use kvc_decode_attn with a workspace)",
                w.total, (unsigned)KVC_NOALLOC_SCRATCH_BYTES);
  unsigned char* wsb = nullptr;
  if ((rc = noalloc_scratch(&wsb)) != KVC_OK) return rc;
  // the merge tickets must start at zero; the array keeps whatever the last call left
  cudaError_t e = cudaMemsetAsync(wsb + w.cnt_off, 0, w.cnt_bytes, stream);
  if (e != cudaSuccess) return fail(KVC_ERR_CUDA, "kvc_decode_attn_noalloc: clear: %s", cudaGetErrorString(e));
  kvc::DecodeParams p{};
  p.q = q;
  p.kp = kp;
  p.vp = vp;
  p.off = off;
  p.len = len;
  p.kp_rows = kp_rows;
  p.S = shape->n_slots;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)shape->d);
  p.out = out;
  p.partial = reinterpret_cast<float*>(wsb + w.part_off);
  p.counters = reinterpret_cast<int*>(wsb + w.cnt_off);
  return launch_decode_any(shape, p, di->sms, stream, /*allow_cluster=*/false);
}

namespace {
kvc_status append_decode(const char* what, const kvc_shape* shape, const void* k_new, const void* v_new,
                         const void* q, void* kp, void* vp, const int64_t* off, const int32_t* cap,
                         const int32_t* stable, int32_t* len, int64_t kp_rows, float* out, void* ws, size_t ws_bytes,
                         cudaStream_t stream) {
  kvc_status rc = check_shape(shape, false);
  if (rc != KVC_OK) return rc;
  if (!k_new || !v_new || !q || !kp || !vp || !off || !cap || !len || !out)
    return fail(KVC_ERR_INVALID_ARG, "%s: NULL pointer argument", what);
  if (shape->dtype != KVC_BF16 || shape->G > 8 || force_simt_decode()) {
    // the CUDA-core decode has no fused append: the two calls in sequence
    if ((rc = kvc_append(shape, k_new, v_new, off, cap, len, kp, vp, kp_rows, stream)) != KVC_OK) return rc;
    return kvc_decode_attn(shape, q, kp, vp, off, len, kp_rows, out, ws, ws_bytes, stream);
  }
  if (shape->n_slots > kvc::DEC_MAX_SLOTS)
    return fail(KVC_ERR_UNSUPPORTED, "%s: %d slots > %d", what, shape->n_slots, kvc::DEC_MAX_SLOTS);
  if (!aligned16(q) || !aligned16(kp) || !aligned16(vp) || !aligned16(ws) || !aligned16(k_new) || !aligned16(v_new) ||
      !aligned16(out))
    return fail(KVC_ERR_INVALID_ARG, "%s: buffers must be 16-byte aligned", what);
  DevInfo* di = nullptr;
  if ((rc = dev_info(&di)) != KVC_OK) return rc;
  const DecodeWs w = decode_ws_layout(shape, di->sms);
  if (!ws || ws_bytes < w.total)
    return fail(KVC_ERR_WORKSPACE, "%s: workspace %zu B < required %zu B", what, ws_bytes, w.total);
  unsigned char* wsb = static_cast<unsigned char*>(ws);
  kvc::DecodeParams p{};
  p.q = q;
  p.kp = kp;
  p.vp = vp;
  p.off = off;
  p.len = len;
  p.kp_rows = kp_rows;
  p.S = shape->n_slots;
  p.scale_log2 = 1.4426950408889634f / sqrtf((float)shape->d);
  p.out = out;
  p.partial = reinterpret_cast<float*>(wsb + w.part_off);
  p.counters = reinterpret_cast<int*>(wsb + w.cnt_off);
  p.append = 1;
  p.k_new = k_new;
  p.v_new = v_new;
  p.cap = cap;
  p.len_out = len;
  p.stable = stable;
  return launch_decode_any(shape, p, di->sms, stream);
}
}  // namespace

kvc_status kvc_append_decode(const kvc_shape* shape, const void* k_new, const void* v_new, const void* q, void* kp,
                             void* vp, const int64_t* off, const int32_t* cap, int32_t* len, int64_t kp_rows,
                             float* out, void* ws, size_t ws_bytes, cudaStream_t stream) {
  return append_decode("kvc_append_decode", shape, k_new, v_new, q, kp, vp, off, cap, nullptr, len, kp_rows, out, ws,
                       ws_bytes, stream);
}

kvc_status kvc_append_decode_chain(const kvc_shape* shape, const void* k_new, const void* v_new, const void* q,
                                   void* kp, void* vp, const int64_t* off, const int32_t* cap, const int32_t* stable,
                                   int32_t* len, int64_t kp_rows, float* out, void* ws, size_t ws_bytes,
                                   cudaStream_t stream) {
  if (!stable) return fail(KVC_ERR_INVALID_ARG, "kvc_append_decode_chain: stable is NULL");
  return append_decode("kvc_append_decode_chain", shape, k_new, v_new, q, kp, vp, off, cap, stable, len, kp_rows, out,
                       ws, ws_bytes, stream);
}

kvc_status kvc_select_chunks(const kvc_shape* shape, const float* chunk_score, const int32_t* chunk_end, int32_t C,
                             const int32_t* target, int32_t n_local, int32_t* idx, int32_t max_sel, int32_t* count,
                             cudaStream_t stream) {
  kvc_status rc = check_shape(shape, false);
  if (rc != KVC_OK) return rc;
  if (!chunk_score || !chunk_end || !target || !idx || !count)
    return fail(KVC_ERR_INVALID_ARG, "kvc_select_chunks: NULL pointer argument");
  if (C <= 0 || C > shape->L || max_sel <= 0 || n_local < 0)
    return fail(KVC_ERR_SHAPE, "kvc_select_chunks: need 1 <= C <= L, max_sel > 0, n_local >= 0");
  // every slot follows the chunk policy; the policy array is not needed
  kvc::SelectParams p{};
  p.score = chunk_score;
  p.policy = nullptr;
  p.budget = target;
  p.mass = 0.9f;
  p.chunk_end = chunk_end;
  p.C = C;
  p.L = shape->L;
  p.n_kv_heads = shape->n_kv_heads;
  p.batch = shape->batch;
  p.idx = idx;
  p.max_sel = max_sel;
  p.count = count;
  p.n_local = n_local;
  return launch_select(p, shape->n_slots, C, stream, "kvc_select_chunks");
}

kvc_status kvc_retained_mass(const kvc_shape* shape, const float* score, int32_t N, const int32_t* idx,
                             int32_t max_sel, const int32_t* count, float* retained, cudaStream_t stream) {
  kvc_status rc = check_shape(shape, false);
  if (rc != KVC_OK) return rc;
  if (!score || !idx || !count || !retained) return fail(KVC_ERR_INVALID_ARG, "kvc_retained_mass: NULL pointer");
  if (N <= 0 || max_sel <= 0) return fail(KVC_ERR_SHAPE, "kvc_retained_mass: N and max_sel must be positive");
  kvc::retained_mass_kernel<<<shape->n_slots, kvc::PROF_THREADS, 0, stream>>>(score, N, idx, max_sel, count,
                                                                               retained);
  count_launches(1);
  return check_launch("kvc_retained_mass");
}

kvc_status kvc_profile_heads(const kvc_shape* shape, const float* score, const uint8_t* special_mask,
                             int32_t window, float tau, int8_t* policy, float* shares, cudaStream_t stream) {
  kvc_status rc = check_shape(shape, false);
  if (rc != KVC_OK) return rc;
  if (!score || !policy) return fail(KVC_ERR_INVALID_ARG, "kvc_profile_heads: score and policy must be non-NULL");
  if (!(tau > 0.f && tau <= 1.f) || window < 0)
    return fail(KVC_ERR_INVALID_ARG, "kvc_profile_heads: need 0 < tau <= 1 and window >= 0");
  kvc::profile_kernel<<<shape->n_slots, kvc::PROF_THREADS, 0, stream>>>(
      score, shape->L, special_mask, shape->n_kv_heads, shape->batch, window, tau, policy, shares);
  count_launches(1);
  return check_launch("kvc_profile_heads");
}

}  // extern "C"
