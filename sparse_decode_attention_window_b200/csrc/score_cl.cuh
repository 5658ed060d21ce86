// Window scoring in slot clusters: a thread-block cluster of k CTAs per slot; each CTA takes
// one range of the slot's key tiles through both passes, and the rows' normalisers are
// folded across the cluster in shared memory between the passes.
//
// Observation-window importance (ZigZagKV Eq. 7; chunk keys per ChunkLLM Eq. 3): every
// window row's softmax needs its normaliser over all the keys it sees before any key's
// column sum can be formed, so the keys are swept twice:
//   pass 1  D = Q K^T  (rows on TMEM lanes): per row, max and sum of 2^x over the range;
//   exchange every CTA sends its rows' (max, sum) to every CTA of the cluster (st.async,
//           counted on an mbarrier in the receiver); each folds them into lse2 per row;
//   pass 2  D = K Q^T  (keys on TMEM lanes): per key, the sum over rows of 2^(z - lse2).
// Pass 2 re-reads the range pass 1 just read, from L2 while the clusters running at the
// same time hold together less than L2. On B200 TMA re-reads from L2 only approach their
// bandwidth with large boxes (measured: 7.8 TB/s with 128-row boxes, 13.6 with 256-row
// boxes; DRAM 6.6 either way), so a job is a tile of 256 keys, brought as 64-dimension x
// 256-row boxes. Both passes cost one 2^x per logit on the special-function unit, which
// bounds the kernel once the keys cross DRAM only once.
//
// Warp roles (576 threads): warp 0 - TMA (Q once, then the range's boxes for pass 1 and
// again for pass 2, into a four-stage ring); warp 1 - TMEM allocation and one lane issuing
// the MMAs; warps 2..17 - four epilogue groups of four warps. Two TMEM accumulators of 256
// columns: job i goes to accumulator i % 2, which groups 2a and 2a + 1 read, each one
// 128-column half (pass 1: 128 of the tile's keys for every row; pass 2: 128 keys over
// every row), 32 columns per TMEM load, so that 16 epilogue warps fit in the register file
// and keep the 2^x unit busy. Clusters never wait for one another; the hardware starts a
// new cluster whenever one ends.
#pragma once
#include "score_sm100.cuh"

namespace kvc {

constexpr int CL_TILE = 256;                        // keys per job
constexpr int CL_NACC = 2;                          // TMEM accumulators of 256 columns
constexpr int CL_GROUPS = 4;                        // epilogue groups (a half accumulator each)
constexpr int CL_EPI = 32 * 4 * CL_GROUPS;          // 512 epilogue threads
constexpr int CL_THREADS = 64 + CL_EPI;             // 576
constexpr int CL_STAGES = 4;                        // 32 KB boxes in flight (5 measured no faster)
constexpr int CL_BOX = CL_TILE * 128;               // one box: 256 rows x 128 B
constexpr int CL_TMEM_COLS = CL_NACC * CL_TILE;     // 512: the whole TMEM of the SM
constexpr int CL_MAX_K = 16;                        // CTAs per slot (above 8: non-portable cluster size)
constexpr float CL_LAZY = 8.f;                      // pass 1 raises its reference max only past +8

template <int D>
struct ClSmem {
  static constexpr int KB = D / 64;                        // boxes (stages) per job
  static constexpr int Q_BYTES = TC_ROWS * D * 2;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_BYTES;
  static constexpr int LSE_OFF = K_OFF + CL_STAGES * CL_BOX;        // [128] float
  static constexpr int WIN_OFF = LSE_OFF + TC_ROWS * 4;             // [128] int
  static constexpr int ST_OFF = WIN_OFF + TC_ROWS * 4;              // [GROUPS][128] float2
  static constexpr int XALL_OFF = ST_OFF + CL_GROUPS * TC_ROWS * 8; // [MAX_K][128] float2, by sender
  static constexpr int BAR_OFF = XALL_OFF + CL_MAX_K * TC_ROWS * 8;
  // kv_full[ST], kv_empty[ST], q_full, tm_full[2], tm_empty[2], xbar
  static constexpr int NBAR = 2 * CL_STAGES + 1 + 2 * CL_NACC + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;               // tmem slot, abort flag
  static constexpr int TOTAL = MISC_OFF + 64;
  static constexpr int ALLOC = TOTAL + 1024;                        // room to align the base to 1024 B
};

struct ClParams {
  int S, N, L, w, R;
  int tiles;          // key tiles (CL_TILE) per slot
  int k;              // CTAs per slot (the cluster size when p1)
  int p1;             // 1: compute the row normalisers (pass 1 + exchange); 0: lse2 given
  float scale2;       // log2(e) / sqrt(d)
  const int32_t* key_pos;   // chunk mode: position of key n; NULL: key n at position n
  const float* lse2;  // p1 == 0: [S][R] row normalisers, log2 units
  float* score;       // [S][N]
};

// keys n < result are visible to a window row at position rowpos
KVC_DEV int visible_keys_cl(const ClParams& p, int rowpos) {
  if (!p.key_pos) return min(p.N, rowpos + 1);
  int lo = 0, hi = p.N;   // first n with key_pos[n] > rowpos
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (p.key_pos[mid] <= rowpos) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// The epilogue's sweep over its 128 accumulator columns: two 64-column halves of TMEM
// loads (32 columns each into two register buffers); the accumulator half is released
// as soon as its last columns are loaded.
#define CL_TMEM_SWEEP(chunk)                                            \
  do {                                                                  \
    tc_ld32(ta0 + 0, va);                                               \
    tc_ld32(ta0 + 32, vb);                                              \
    tc_wait_ld();                                                       \
    chunk(va, 0);                                                       \
    chunk(vb, 32);                                                      \
    tc_ld32(ta0 + 64, va);                                              \
    tc_ld32(ta0 + 96, vb);                                              \
    tc_wait_ld();                                                       \
    tc_fence_before();                                                  \
    __syncwarp();                                                       \
    if (lane == 0) mbar_arrive(&tm_empty[acc]);                         \
    chunk(va, 64);                                                      \
    chunk(vb, 96);                                                      \
  } while (0)

template <int D>
__global__ void __launch_bounds__(CL_THREADS, 1)
score_cl_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k, ClParams p) {
  using L_ = ClSmem<D>;
  extern __shared__ __align__(1024) unsigned char cl_smem_raw[];
  const uint32_t raw = smem_u32(cl_smem_raw);
  unsigned char* sm = cl_smem_raw + (((raw + 1023u) & ~1023u) - raw);
  unsigned char* q_s = sm + L_::Q_OFF;
  unsigned char* k_s = sm + L_::K_OFF;
  float* lse_s = reinterpret_cast<float*>(sm + L_::LSE_OFF);
  int* win_s = reinterpret_cast<int*>(sm + L_::WIN_OFF);
  float2* stats = reinterpret_cast<float2*>(sm + L_::ST_OFF);
  float2* xall = reinterpret_cast<float2*>(sm + L_::XALL_OFF);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L_::BAR_OFF);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + CL_STAGES;
  uint64_t* q_full = bars + 2 * CL_STAGES;
  uint64_t* tm_full = q_full + 1;
  uint64_t* tm_empty = tm_full + CL_NACC;
  uint64_t* xbar = tm_empty + CL_NACC;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L_::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L_::MISC_OFF + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = p.k;
  const int s = blockIdx.x / k, rank = blockIdx.x - s * k;   // 1-D grid and clusters: rank = cluster rank
  const int j0 = (int)((long long)rank * p.tiles / k), j1 = (int)((long long)(rank + 1) * p.tiles / k);
  const int nj = j1 - j0;
  const int njobs = p.p1 ? 2 * nj : nj;
  const bool exch = p.p1 && k > 1;

  if (threadIdx.x == 0) {
    for (int i = 0; i < CL_STAGES; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(q_full, 1);
    for (int i = 0; i < CL_NACC; ++i) {
      mbar_init(&tm_full[i], 1);
      mbar_init(&tm_empty[i], 8);    // lane 0 of each warp of the two groups reading it
    }
    mbar_init(xbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (threadIdx.x < TC_ROWS) win_s[threadIdx.x] = threadIdx.x < p.R ? threadIdx.x % p.w : 0x40000000;
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&map_q);
    prefetch_tensormap(&map_k);
  }
  if (warp == 1) tc_alloc(tmem_slot, CL_TMEM_COLS);
  // every CTA's barriers are initialised before any CTA of the cluster sends to it (the
  // matching wait precedes the first st.async, or the end of the kernel)
  if (exch) cluster_arrive_relaxed();
  bool cl_waited = false;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int st = 0;
      uint32_t kph = 0;
      long long boxes = 0;
      bool ok = true;
      mbar_arrive_expect_tx(q_full, L_::Q_BYTES);
#pragma unroll
      for (int kb = 0; kb < L_::KB; ++kb) tma_load_3d(q_s + kb * TC_ROWS * 128, &map_q, kb * 64, 0, s, q_full);
      for (int i = 0; i < njobs && ok; ++i) {
        const int j = j0 + (i < nj ? i : i - nj);   // the range, once per pass
#pragma unroll
        for (int kb = 0; kb < L_::KB; ++kb) {
          if (!mbar_wait(&kv_empty[st], kph ^ 1) || *abort_flag) { ok = false; break; }
          mbar_arrive_expect_tx(&kv_full[st], CL_BOX);
          tma_load_3d(k_s + st * CL_BOX, &map_k, kb * 64, j * CL_TILE, s, &kv_full[st]);
          ++boxes;
          if (++st == CL_STAGES) { st = 0; kph ^= 1; }
        }
      }
      if (!ok) *abort_flag = 1;
      // every copy this thread issued has landed before the CTA may exit
      for (long long b = boxes > CL_STAGES ? boxes - CL_STAGES : 0; b < boxes; ++b)
        mbar_wait(&kv_full[b % CL_STAGES], (uint32_t)((b / CL_STAGES) & 1));
      mbar_wait(q_full, 0);
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      int st = 0;
      uint32_t kph = 0, teph = 0;
      long long boxes = 0, done = 0;
      bool ok = mbar_wait(q_full, 0) && !*abort_flag;
      const uint32_t q_addr = smem_u32(q_s);
      for (int i = 0; i < njobs && ok; ++i) {
        const int acc = i & 1;
        const bool pass1 = p.p1 && i < nj;
        if (!mbar_wait(&tm_empty[acc], ((teph >> acc) & 1u) ^ 1u) || *abort_flag) { ok = false; break; }
        teph ^= 1u << acc;
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * CL_TILE);
        for (int kb = 0; kb < L_::KB; ++kb) {
          if (!mbar_wait(&kv_full[st], kph) || *abort_flag) { ok = false; break; }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(k_s + st * CL_BOX);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {   // 4 x K=16 per 64-element box (+32 B each)
            const uint32_t qa = q_addr + kb * TC_ROWS * 128 + kk * 32;
            const uint32_t ka = k_addr + kk * 32;
            const uint32_t accum = (kb | kk) != 0;
            if (pass1) {
              // D[128 rows x 256 keys] = Q K^T
              tc_mma(d_tmem, smem_desc_sw128(qa), smem_desc_sw128(ka), tc_idesc(128, 256), accum);
            } else {
              // D[keys x 128 rows] = K Q^T for the tile's two 128-key halves
              tc_mma(d_tmem, smem_desc_sw128(ka), smem_desc_sw128(qa), tc_idesc(128, 128), accum);
              tc_mma(d_tmem + 128, smem_desc_sw128(ka + 128 * 128), smem_desc_sw128(qa), tc_idesc(128, 128), accum);
            }
          }
          tc_commit(&kv_empty[st]);     // the box is free once these MMAs completed
          ++boxes;
          if (++st == CL_STAGES) { st = 0; kph ^= 1; }
        }
        if (!ok) break;
        tc_commit(&tm_full[acc]);       // the accumulator is ready for its two groups
        ++done;
      }
      if (!ok) *abort_flag = 1;
      // every commit this thread issued has arrived before the CTA may exit
      for (long long b = boxes > CL_STAGES ? boxes - CL_STAGES : 0; b < boxes; ++b)
        mbar_wait(&kv_empty[b % CL_STAGES], (uint32_t)((b / CL_STAGES) & 1));
      for (long long d = done > CL_NACC ? done - CL_NACC : 0; d < done; ++d)
        mbar_wait(&tm_full[d % CL_NACC], (uint32_t)((d / CL_NACC) & 1));
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue: four groups of four warps
    const int ew = warp - 2;                 // 0..15
    const int g = ew >> 2;                   // group
    const int acc = g >> 1, half = g & 1;    // accumulator, 128-column half
    const int quarter = warp & 3;            // TMEM lanes 32*quarter .. +31
    const int t = quarter * 32 + lane;       // pass 1: window row; pass 2: key of the half
    const uint32_t ta0 = tmem_base + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(acc * CL_TILE + half * 128);
    const int Lw = p.L - p.w;
    uint32_t tph = 0;
    bool ok = true;
    float va[32], vb[32];
    int i = acc;                             // this group's next job
    if (p.p1) {
      // ---- pass 1 over this group's jobs of the range: row t's max and sum of 2^x
      const int vis = t < p.R ? visible_keys_cl(p, Lw + (t % p.w)) : 0;
      float m2 = -INFINITY, lsum = 0.f;
      for (; i < nj && ok; i += CL_NACC) {
        if (!mbar_wait(&tm_full[acc], tph)) { ok = false; *abort_flag = 1; break; }
        tph ^= 1;
        tc_fence_after();
        const int n0 = (j0 + i) * CL_TILE + half * 128;
        const int nv = min(max(vis - n0, 0), 128);
        auto chunk = [&](const float* v, int c0) {
          const int cv = min(max(nv - c0, 0), 32);
          if (t >= p.R || cv == 0) return;
          float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
          for (int u = 0; u < 32; ++u) mx[u & 3] = u < cv ? fmaxf(mx[u & 3], v[u]) : mx[u & 3];
          const float mxs = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * p.scale2;
          if (mxs > m2 + CL_LAZY) {   // a new reference only when a logit passes it by > 2^8
            lsum = m2 == -INFINITY ? 0.f : lsum * ex2_ftz(m2 - mxs);
            m2 = mxs;
          }
          float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
          for (int u = 0; u < 32; ++u) a[u & 3] += u < cv ? ex2_ftz(fmaf(v[u], p.scale2, -m2)) : 0.f;
          lsum += (a[0] + a[1]) + (a[2] + a[3]);
        };
        CL_TMEM_SWEEP(chunk);
      }
      // ---- the four groups fold in shared memory, the CTA's rows go to every CTA of the
      // cluster, and each CTA folds the cluster's rows into lse2
      stats[g * TC_ROWS + t] = make_float2(m2, lsum);
      if (named_bar_or(1, CL_EPI, !ok)) ok = false;
      if (g == 0) {
        float M = -INFINITY, l = 0.f;
        if (t < p.R) {
#pragma unroll
          for (int gg = 0; gg < CL_GROUPS; ++gg) M = fmaxf(M, stats[gg * TC_ROWS + t].x);
          if (M != -INFINITY)
#pragma unroll
            for (int gg = 0; gg < CL_GROUPS; ++gg) {
              const float2 e = stats[gg * TC_ROWS + t];
              if (e.x != -INFINITY) l += e.y * ex2_ftz(e.x - M);
            }
        }
        float2* mine = xall + rank * TC_ROWS + t;
        *mine = make_float2(M, l);
        if (exch) {
          // every row goes to every other CTA of the cluster, so each expects a fixed byte count
          cluster_wait();
          cl_waited = true;
          for (int r = 1; r < k; ++r) {
            const uint32_t dst = (uint32_t)((rank + r) % k);
            st_async_f32x2(map_to_rank(mine, dst), M, l, map_to_rank(xbar, dst));
          }
          if (t == 0) mbar_arrive_expect_tx(xbar, (uint32_t)((k - 1) * TC_ROWS * 8));
        }
      }
      if (exch && !mbar_wait_cluster(xbar, 0)) ok = false;
      named_bar_sync(2, CL_EPI);
      if (g == 0) {
        float M = -INFINITY;
        for (int r = 0; r < k; ++r) M = fmaxf(M, xall[r * TC_ROWS + t].x);
        float l = 0.f;
        if (M != -INFINITY)
          for (int r = 0; r < k; ++r) {
            const float2 e = xall[r * TC_ROWS + t];
            if (e.x != -INFINITY) l += e.y * ex2_ftz(e.x - M);
          }
        lse_s[t] = (t < p.R && l > 0.f) ? M + log2f(l) : INFINITY;
      }
    } else if (g == 0) {
      lse_s[t] = t < p.R ? p.lse2[(size_t)s * p.R + t] : INFINITY;
    }
    if (named_bar_or(3, CL_EPI, !ok)) ok = false;
    // ---- pass 2 over this group's jobs: key n0 + t over the 128 window rows
    const int p2first = p.p1 ? nj : 0;
    for (; i < njobs && ok; i += CL_NACC) {
      if (!mbar_wait(&tm_full[acc], tph)) { ok = false; *abort_flag = 1; break; }
      tph ^= 1;
      tc_fence_after();
      const int n = (j0 + i - p2first) * CL_TILE + half * 128 + t;
      const bool live = n < p.N;
      const int pos = live ? (p.key_pos ? p.key_pos[n] : n) : 0;
      const int imin = pos - Lw;              // rows with window index >= imin see the key
      float a[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      auto chunk = [&](const float* v, int r0) {
        if (!live) return;
        if (imin <= 0) {
#pragma unroll
          for (int u = 0; u < 32; u += 4) {
            const float4 l4 = *reinterpret_cast<const float4*>(lse_s + r0 + u);
            a[(u + 0) & 7] += ex2_ftz(fmaf(v[u + 0], p.scale2, -l4.x));
            a[(u + 1) & 7] += ex2_ftz(fmaf(v[u + 1], p.scale2, -l4.y));
            a[(u + 2) & 7] += ex2_ftz(fmaf(v[u + 2], p.scale2, -l4.z));
            a[(u + 3) & 7] += ex2_ftz(fmaf(v[u + 3], p.scale2, -l4.w));
          }
        } else {
#pragma unroll
          for (int u = 0; u < 32; ++u)
            a[u & 7] += win_s[r0 + u] >= imin ? ex2_ftz(fmaf(v[u], p.scale2, -lse_s[r0 + u])) : 0.f;
        }
      };
      CL_TMEM_SWEEP(chunk);
      if (live) p.score[(size_t)s * p.N + n] = ((a[0] + a[1]) + (a[2] + a[3])) + ((a[4] + a[5]) + (a[6] + a[7]));
    }
  }
  // do not leave while another CTA of the cluster may still send into this one
  if (exch && !cl_waited) cluster_wait();

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tc_dealloc(tmem_base, CL_TMEM_COLS);
}

// ---------------------------------------------------------------- host side
// The cluster size k (CTAs per slot): the largest k <= 16 (and <= the slot's tiles) whose
// S clusters can all be resident at once; 0 when even k = 1 needs more than one wave (many
// slots): those shapes take the two-launch form, whose pass 2 streams the keys again
// rather than the short-lived clusters of several waves (measured: 1115 against 801 us
// for 256 slots of 32768 keys).
// The kernel's shared-memory size and cluster-size attributes, set once per device before
// any occupancy query or launch (a query without them answers 0 clusters).
template <int D>
cudaError_t cl_prepare() {
  static std::mutex mu;
  static bool set[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lk(mu);
  if (set[dev]) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(score_cl_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)ClSmem<D>::ALLOC);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(score_cl_kernel<D>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  if (e == cudaSuccess) set[dev] = true;
  return e;
}

template <int D>
int cl_resident_clusters(int k, size_t smem) {
  if (cl_prepare<D>() != cudaSuccess) {
    cudaGetLastError();
    return 0;
  }
  static std::mutex mu;
  static std::map<std::pair<int, int>, int> known;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  auto it = known.find({k, dev});
  if (it != known.end()) return it->second;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(k);
  cfg.blockDim = dim3(CL_THREADS);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = k;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, score_cl_kernel<D>, &cfg) != cudaSuccess) n = 0;
  cudaGetLastError();
  known[{k, dev}] = n;
  return n;
}

template <int D>
int cl_choose_k(int S, int tiles, int sms) {
  const size_t smem = ClSmem<D>::ALLOC;
  for (int k = std::min(CL_MAX_K, tiles); k >= 1; --k) {
    const int n = k == 1 ? sms : cl_resident_clusters<D>(k, smem);
    if (n >= S) return k;
  }
  return 0;
}

// Whether the slot-cluster form takes this shape (every slot's cluster resident at once).
inline bool cl_takes(const kvc_shape* sh, int C, int sms, int k_force) {
  const long long N = C > 0 ? C : sh->L;
  const int tiles = (int)((N + CL_TILE - 1) / CL_TILE);
  if (k_force > 0) return true;
  if (sh->d == 128) return cl_choose_k<128>(sh->n_slots, tiles, sms) > 0;
  return cl_choose_k<64>(sh->n_slots, tiles, sms) > 0;
}

template <int D>
kvc_status tc_score_cl_d(const kvc_shape* sh, const void* q_win, const void* k, const int32_t* chunk_end, int32_t C,
                         const float* row_lse, float* score, float* lse2, void* keys_ws, int sms, cudaStream_t st,
                         fail_fn fail, unsigned* launches, int k_force) {
  const int S = sh->n_slots, R = sh->G * sh->w, L = sh->L;
  const int N = chunk_end ? C : L;
  const void* kbase = k;
  long long krows = L;
  if (chunk_end) {
    const int tpr = D * 2 / 16;
    const long long total = (long long)S * C * tpr;
    const int blocks = (int)std::min<long long>((total + 255) / 256, (long long)sms * 16);
    gather_rows_kernel<<<blocks, 256, 0, st>>>(static_cast<const uint4*>(k), chunk_end, C, L, S, tpr,
                                               static_cast<uint4*>(keys_ws));
    ++*launches;
    kbase = keys_ws;
    krows = C;
  }
  if (row_lse) {
    lse_to_lse2<<<std::max(1, std::min((S * R + 255) / 256, sms * 4)), 256, 0, st>>>(row_lse, S * R, lse2);
    ++*launches;
  }
  CUtensorMap mq, mk;
  if (!make_map_3d(&mq, q_win, D, R, S, TC_ROWS) || !make_map_3d(&mk, kbase, D, krows, S, CL_TILE))
    return fail(KVC_ERR_CUDA, "kvc_score: cuTensorMapEncodeTiled failed");
  const size_t smem = ClSmem<D>::ALLOC;
  cudaError_t e = cl_prepare<D>();
  if (e != cudaSuccess) return fail(KVC_ERR_CUDA, "kvc_score: kernel attribute: %s", cudaGetErrorString(e));
  ClParams p{};
  p.S = S; p.N = N; p.L = L; p.w = sh->w; p.R = R;
  p.tiles = (N + CL_TILE - 1) / CL_TILE;
  p.p1 = row_lse ? 0 : 1;
  p.k = k_force > 0 ? std::min(k_force, std::min(CL_MAX_K, p.tiles)) : cl_choose_k<D>(S, p.tiles, sms);
  p.scale2 = 1.4426950408889634f / sqrtf((float)D);
  p.key_pos = chunk_end;
  p.lse2 = lse2;
  p.score = score;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)S * (unsigned)p.k);
  cfg.blockDim = dim3(CL_THREADS);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = p.p1 ? p.k : 1;   // the normaliser exchange needs the slot's CTAs together
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, score_cl_kernel<D>, mq, mk, p);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return fail(KVC_ERR_CUDA, "kvc_score: launch: %s", cudaGetErrorString(e));
  }
  ++*launches;
  return KVC_OK;
}

inline kvc_status tc_score_cl(const kvc_shape* sh, const void* q_win, const void* k, const int32_t* chunk_end,
                              int32_t C, const float* row_lse, float* score, float* lse2, void* keys_ws, int sms,
                              cudaStream_t st, fail_fn fail, unsigned* launches, int k_force = 0) {
  if (sh->d == 128)
    return tc_score_cl_d<128>(sh, q_win, k, chunk_end, C, row_lse, score, lse2, keys_ws, sms, st, fail, launches,
                              k_force);
  return tc_score_cl_d<64>(sh, q_win, k, chunk_end, C, row_lse, score, lse2, keys_ws, sms, st, fail, launches, k_force);
}

}  // namespace kvc
