// Window scoring on the sm_100a tensor cores: tcgen05.mma (bf16 in, fp32 in
// TMEM), operands staged by TMA, softmax statistics and column sums fused into
// the TMEM epilogue.
//
// Observation-window importance (ZigZagKV Eq. 7, after SnapKV; chunk keys per
// ChunkLLM Eq. 3): the R = G*w window rows of a slot (query head j, window row i
// at position L - w + i) each take a softmax over the keys they see, and a key's
// score is its column sum. Per slot the contraction is [R x d] x [d x N]; with
// R = 128 it runs at 128 flop per key byte, below the B200 ridge, so it is
// HBM-bound and the exp work of the epilogue is the next limit.
//
// Two passes over the keys, both on the tensor cores:
//   pass 1  D[rows x keys]  = Q K^T : a thread owns a TMEM lane = one window row
//           and keeps its running max and sum of exp2 over its key range, so the
//           row statistics need no cross-thread reduction;
//   merge   per row, lse2 = log2 sum over the key-range partials;
//   pass 2  D[keys x rows]  = K Q^T : the transposed product puts one key on each
//           TMEM lane, so the column sum of exp2(z - lse2_r) is a per-thread sum.
// Each pass is a persistent kernel: warp 0 issues TMA (Q once per work item,
// 128-key K tiles into a 4-stage ring), warp 1 owns the TMEM allocation and one
// lane issues the MMAs into two TMEM accumulators (128 columns each) so the
// next tile's MMA overlaps the current tile's epilogue, warps 2-5 run the
// epilogue (warp w reads TMEM lanes 32*(w%4) .. +31).
// Chunk keys are first gathered into a contiguous buffer (one row per chunk).
#pragma once
#include <algorithm>
#include <map>
#include <mutex>
#include "common.cuh"
#include "cache.cuh"

namespace kvc {

typedef kvc_status (*fail_fn)(kvc_status, const char*, ...);

constexpr int TC_TILE = 128;      // keys per tile (MMA N in pass 1, M in pass 2)
constexpr int TC_ROWS = 128;      // window rows per slot, padded (MMA M in pass 1, N in pass 2)
constexpr int TC_STAGES = 4;
constexpr int TC_EPI_WARPS = 8;   // two per SM sub-partition; warp pair (w, w+4) splits the 128 columns
constexpr int TC_THREADS = 32 * (2 + TC_EPI_WARPS);
constexpr int TC_TMEM_COLS = 256; // two 128-column fp32 accumulators
constexpr int TC_MAX_CLUSTER = 16; // fused mode: CTAs per slot (16 needs the non-portable cluster size)

// ---------------------------------------------------------------- PTX wrappers (tcgen05)
KVC_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
KVC_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

KVC_DEV void tc_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
KVC_DEV void tc_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, bf16 -> fp32, shapes from the instruction descriptor.
KVC_DEV void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` once every tcgen05 operation this thread issued so far has completed.
KVC_DEV void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// 32 lanes x 32 consecutive fp32 columns: thread t of the warp gets lane (base lane + t).
KVC_DEV void tc_ld32(uint32_t taddr, float* v) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
KVC_DEV void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 2^x on the special-function unit (approximate, subnormal results flushed to zero:
// a probability below 2^-126 adds nothing to a softmax sum at fp32 precision).
KVC_DEV float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}



// Shared-memory matrix descriptor: K-major operand in the 128-byte swizzle layout
// TMA writes (rows of 128 B, 8-row groups 1024 B apart), start 1024-B aligned.
KVC_DEV uint64_t smem_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);        // start address
  d |= (uint64_t)1u << 16;                          // leading-dimension offset (unused for swizzled K-major)
  d |= (uint64_t)(1024u >> 4) << 32;                // stride between 8-row groups
  d |= (uint64_t)1u << 46;                          // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                          // 128-byte swizzle
  return d;
}

// Instruction descriptor: kind::f16, A = B = bf16, D = fp32, both K-major, M x N.
constexpr uint32_t tc_idesc(int M, int N) {
  return (1u << 4)                     // D format: f32
         | (1u << 7)                   // A format: bf16
         | (1u << 10)                  // B format: bf16
         | ((uint32_t)(N >> 3) << 17)  // N / 8
         | ((uint32_t)(M >> 4) << 24); // M / 16
}

// ---------------------------------------------------------------- shared layout
template <int D>
struct TcSmem {
  static constexpr int KB = D / 64;                       // 64-element (128 B) k-blocks
  static constexpr int Q_BYTES = TC_ROWS * D * 2;         // 16 or 32 KB
  static constexpr int K_BYTES = TC_TILE * D * 2;         // per stage
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_BYTES;
  static constexpr int BAR_OFF = K_OFF + TC_STAGES * K_BYTES;
  // barriers: kv_full[ST], kv_empty[ST], q_full, q_empty, tm_full[2], tm_empty[2]
  static constexpr int NBAR = 2 * TC_STAGES + 2 + 4;
  static constexpr int MISC_OFF = BAR_OFF + NBAR * 8;     // tmem addr, flags
  static constexpr int LSE_OFF = MISC_OFF + 64;           // pass 2: lse2[128], win index [128]
  static constexpr int XCH_OFF = LSE_OFF + 2 * TC_ROWS * 4; // half-to-half exchange [128] float2
  static constexpr int XALL_OFF = XCH_OFF + TC_ROWS * 8;    // fused mode: row stats of every CTA [16][128] float2
  static constexpr int XBAR_OFF = XALL_OFF + TC_MAX_CLUSTER * TC_ROWS * 8;
  static constexpr int TOTAL = XBAR_OFF + 8;
  static constexpr int ALLOC = TOTAL + 1024;              // room to align the base to 1024 B
};

struct TcParams {
  int S, N, L, w, R, G;
  int tiles;          // tiles per slot = ceil(N / 128)
  int tpi;            // tiles per work item
  int nsplit;         // work items per slot = ceil(tiles / tpi) (fused mode: the cluster size)
  float scale2;       // log2(e) / sqrt(d)
  const int32_t* key_pos;  // chunk mode: position of key n (chunk_end); NULL: key n at position n
  float2* part;       // pass 1 out: [S][nsplit][R] (max2, sum)
  const float* lse2;  // pass 2 in: [S][R]
  float* score;       // pass 2 out: [S][N]
};

// keys n < vis are visible to a window row at position rowpos
KVC_DEV int visible_keys(const TcParams& p, int rowpos) {
  if (!p.key_pos) return min(p.N, rowpos + 1);
  int lo = 0, hi = p.N;   // first n with key_pos[n] > rowpos
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (p.key_pos[mid] <= rowpos) lo = mid + 1; else hi = mid;
  }
  return lo;
}

// PASS = 1: row statistics; PASS = 2: column sums; PASS = 3: both, fused - launched in
// clusters of nsplit CTAs, cluster j scores slot j, CTA r its r-th key range: pass 1 over
// the range, every CTA sends its rows' (max, sum) to every CTA of the cluster (st.async,
// counted on an mbarrier in the receiver, so the TMA and MMA warps never wait on the
// exchange), each CTA folds them into the rows' normalisers, and pass 2 re-reads the same
// key tiles while they are still in L2.
template <int D, int PASS>
__global__ void __launch_bounds__(TC_THREADS, 1)
score_tc_kernel(const __grid_constant__ CUtensorMap map_q, const __grid_constant__ CUtensorMap map_k, TcParams p) {
  using L_ = TcSmem<D>;
  extern __shared__ __align__(1024) unsigned char tc_smem_raw[];
  // 1024-byte aligned base for the swizzled operand tiles
  const uint32_t raw = smem_u32(tc_smem_raw);
  unsigned char* sm = tc_smem_raw + (((raw + 1023u) & ~1023u) - raw);
  unsigned char* q_s = sm + L_::Q_OFF;
  unsigned char* k_s = sm + L_::K_OFF;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + L_::BAR_OFF);
  uint64_t* kv_full = bars;
  uint64_t* kv_empty = bars + TC_STAGES;
  uint64_t* q_full = bars + 2 * TC_STAGES;
  uint64_t* q_empty = q_full + 1;
  uint64_t* tm_full = q_full + 2;
  uint64_t* tm_empty = q_full + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(sm + L_::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(sm + L_::MISC_OFF + 4);
  float* lse_s = reinterpret_cast<float*>(sm + L_::LSE_OFF);
  int* win_s = reinterpret_cast<int*>(sm + L_::LSE_OFF + TC_ROWS * 4);
  float2* xch = reinterpret_cast<float2*>(sm + L_::XCH_OFF);
  float2* xall = reinterpret_cast<float2*>(sm + L_::XALL_OFF);   // fused: [rank][row] (max2, sum)
  uint64_t* xbar = reinterpret_cast<uint64_t*>(sm + L_::XBAR_OFF);
  constexpr int NPASS = PASS == 3 ? 2 : 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_items = p.S * p.nsplit;
  long long tiles_before = 0;   // epilogue: tiles of this CTA's earlier items

  if (threadIdx.x == 0) {
    for (int i = 0; i < TC_STAGES; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    mbar_init(xbar, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tm_full[b], 1);
      mbar_init(&tm_empty[b], TC_EPI_WARPS / 2);
    }
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&map_q);
    prefetch_tensormap(&map_k);
  }
  if (warp == 1) tc_alloc(tmem_slot, TC_TMEM_COLS);
  // fused: every CTA's barriers are initialised before any CTA of the cluster sends to it
  // (the matching wait precedes the first st.async, or ends the kernel)
  if (PASS == 3) cluster_arrive_relaxed();
  bool cl_waited = false;
  if (threadIdx.x < TC_ROWS) {
    // window index of pass-2 column r (rows beyond R never match)
    win_s[threadIdx.x] = threadIdx.x < p.R ? threadIdx.x % p.w : 0x40000000;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      int st = 0;
      uint32_t ph = 0, qph = 0;
      long long issued = 0, q_issued = 0;
      bool ok = true;
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const int s = item / p.nsplit, sp = item - s * p.nsplit;
        const int j0 = sp * p.tpi, j1 = min(p.tiles, j0 + p.tpi);
        if (!mbar_wait(q_empty, qph ^ 1)) { ok = false; break; }
        mbar_arrive_expect_tx(q_full, L_::Q_BYTES);
#pragma unroll
        for (int kb = 0; kb < L_::KB; ++kb) tma_load_3d(q_s + kb * TC_ROWS * 128, &map_q, kb * 64, 0, s, q_full);
        qph ^= 1;
        ++q_issued;
        for (int jj = j0; jj < j0 + NPASS * (j1 - j0) && ok; ++jj) {   // fused: the range twice
          const int j = j0 + (jj - j0) % (j1 - j0);
          if (!mbar_wait(&kv_empty[st], ph ^ 1) || *abort_flag) { ok = false; break; }
          mbar_arrive_expect_tx(&kv_full[st], L_::K_BYTES);
          unsigned char* dst = k_s + st * L_::K_BYTES;
#pragma unroll
          for (int kb = 0; kb < L_::KB; ++kb)
            tma_load_3d(dst + kb * TC_TILE * 128, &map_k, kb * 64, j * TC_TILE, s, &kv_full[st]);
          ++issued;
          if (++st == TC_STAGES) { st = 0; ph ^= 1; }
        }
      }
      if (!ok) *abort_flag = 1;
      // every load this thread issued has landed before the CTA may exit
      for (long long k = issued > TC_STAGES ? issued - TC_STAGES : 0; k < issued; ++k)
        mbar_wait(&kv_full[k % TC_STAGES], (uint32_t)((k / TC_STAGES) & 1));
      if (q_issued > 0) mbar_wait(q_full, (uint32_t)((q_issued - 1) & 1));
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = tc_idesc(128, 128);
      int st = 0, b = 0;
      uint32_t ph = 0, qph = 0, tph = 0;
      long long done_tiles = 0, done_items = 0;
      bool ok = true;
      const uint32_t q_addr = smem_u32(q_s);
      for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
        const int s = item / p.nsplit, sp = item - s * p.nsplit;
        const int j0 = sp * p.tpi, j1 = min(p.tiles, j0 + p.tpi);
        if (!mbar_wait(q_full, qph) || *abort_flag) { ok = false; break; }
        qph ^= 1;
        for (int jj = j0; jj < j0 + NPASS * (j1 - j0); ++jj) {   // fused: pass 1, then pass 2
          const bool rows_on_lanes = PASS == 1 || (PASS == 3 && jj < j1);   // D = Q K^T
          if (!mbar_wait(&kv_full[st], ph) || !mbar_wait(&tm_empty[b], tph ^ 1) || *abort_flag) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t k_addr = smem_u32(k_s + st * L_::K_BYTES);
          const uint32_t d_tmem = tmem_base + (uint32_t)(b * 128);
#pragma unroll
          for (int kb = 0; kb < L_::KB; ++kb) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {   // 4 x K=16 per 64-element k-block (+32 B each)
              const uint32_t qa = q_addr + kb * TC_ROWS * 128 + kk * 32;
              const uint32_t ka = k_addr + kb * TC_TILE * 128 + kk * 32;
              const uint64_t a = rows_on_lanes ? smem_desc_sw128(qa) : smem_desc_sw128(ka);
              const uint64_t bb = rows_on_lanes ? smem_desc_sw128(ka) : smem_desc_sw128(qa);
              tc_mma(d_tmem, a, bb, idesc, (kb | kk) != 0);
            }
          }
          tc_commit(&kv_empty[st]);     // K stage free once these MMAs completed
          tc_commit(&tm_full[b]);       // accumulator b ready for the epilogue
          ++done_tiles;
          if (++st == TC_STAGES) { st = 0; ph ^= 1; }
          if (++b == 2) { b = 0; tph ^= 1; }
        }
        tc_commit(q_empty);             // Q free once the item's MMAs completed
        ++done_items;
      }
      if (!ok) *abort_flag = 1;
      // every commit this thread issued has arrived before the CTA may exit
      for (long long k = done_tiles > TC_STAGES ? done_tiles - TC_STAGES : 0; k < done_tiles; ++k)
        mbar_wait(&kv_empty[k % TC_STAGES], (uint32_t)((k / TC_STAGES) & 1));
      for (long long k = done_tiles > 2 ? done_tiles - 2 : 0; k < done_tiles; ++k)
        mbar_wait(&tm_full[k % 2], (uint32_t)((k / 2) & 1));
      if (done_items > 0) mbar_wait(q_empty, (uint32_t)((done_items - 1) & 1));
    }
    __syncwarp();
  } else {
    // ------------------------------------------------ epilogue: warps 2..9
    // Two groups of four warps (one warp per SM sub-partition in each group) take the
    // item's tiles in turn: group 0 the even tiles (TMEM accumulator 0), group 1 the odd
    // ones (accumulator 1), so a thread always reads whole 128-column rows and no tile
    // needs a cross-warp reduction. Warp w reads TMEM lanes 32*(w%4) .. +31.
    const int ew = warp - 2;                      // 0..7
    const int quarter = warp & 3;
    const int grp = ew >> 2;                      // 0 or 1 = the TMEM accumulator this group reads
    const int t = quarter * 32 + lane;            // pass 1: window row; pass 2: key within the tile
    const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
    constexpr int NEPI = 32 * TC_EPI_WARPS;
    uint32_t tph = 0;                             // phase of this group's accumulator barrier
    const int Lw = p.L - p.w;
    bool ok = true;
    bool x_waited = false;                        // fused: the exchange barrier was waited on
    for (int item = blockIdx.x; item < n_items && ok; item += gridDim.x) {
      const int s = item / p.nsplit, sp = item - s * p.nsplit;
      const int j0 = sp * p.tpi, j1 = max(j0, min(p.tiles, j0 + p.tpi));
      for (int ps = 0; ps < NPASS && ok; ++ps) {
      const bool p1 = PASS == 1 || (PASS == 3 && ps == 0);   // this sweep: row statistics
      float m2 = -INFINITY, lsum = 0.f;            // pass 1 running stats of row t over this group's tiles
      int vis = 0;
      if (p1) {
        vis = t < p.R ? visible_keys(p, Lw + (t % p.w)) : 0;
      } else {
        named_bar_sync(1, NEPI);                    // previous item's lse_s reads are done
        if (grp == 0) {
          if (PASS == 2) {
            lse_s[t] = t < p.R ? p.lse2[(size_t)s * p.R + t] : INFINITY;
          } else {
            // fused: every CTA of the cluster sent its rows' (max2, sum); fold them
            x_waited = true;
            if (!mbar_wait_cluster(xbar, 0)) ok = false;
            float M = -INFINITY;
            for (int r = 0; r < p.nsplit; ++r) M = fmaxf(M, xall[r * TC_ROWS + t].x);
            float l = 0.f;
            if (M != -INFINITY)
              for (int r = 0; r < p.nsplit; ++r) {
                const float2 q = xall[r * TC_ROWS + t];
                if (q.x != -INFINITY) l += q.y * ex2_ftz(q.x - M);
              }
            lse_s[t] = (t < p.R && l > 0.f) ? M + log2f(l) : INFINITY;
          }
        }
        named_bar_sync(1, NEPI);
      }
      // the MMA warp alternates accumulators continuously across items: tile k of the
      // CTA's sequence uses accumulator k & 1; this group takes the tiles with k & 1 == grp
      for (int j = j0; j < j1; ++j) {
        const long long k = tiles_before + (j - j0);
        if ((int)(k & 1) != grp || !ok) continue;
        if (!mbar_wait(&tm_full[grp], tph)) { ok = false; continue; }   // skip the rest, still meet below
        tph ^= 1;
        tc_fence_after();
        float v[128];
        const uint32_t ta = tmem_base + lane_base + (uint32_t)(grp * 128);
        tc_ld32(ta + 0, v);
        tc_ld32(ta + 32, v + 32);
        tc_ld32(ta + 64, v + 64);
        tc_ld32(ta + 96, v + 96);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tm_empty[grp]);

        const int n0 = j * TC_TILE;
        if (p1) {
          if (t < p.R) {
            const int nv = min(vis - n0, TC_TILE);      // visible columns of this tile
            if (nv > 0) {
              float mx[8];
#pragma unroll
              for (int c = 0; c < 8; ++c) mx[c] = -INFINITY;
              if (nv == TC_TILE) {
#pragma unroll
                for (int c = 0; c < TC_TILE; ++c) mx[c & 7] = fmaxf(mx[c & 7], v[c]);
              } else {
#pragma unroll
                for (int c = 0; c < TC_TILE; ++c) mx[c & 7] = c < nv ? fmaxf(mx[c & 7], v[c]) : mx[c & 7];
              }
              const float mxa = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                      fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
              const float mnew = fmaxf(m2, mxa * p.scale2);
              float acc[8];
#pragma unroll
              for (int c = 0; c < 8; ++c) acc[c] = 0.f;
              if (nv == TC_TILE) {
#pragma unroll
                for (int c = 0; c < TC_TILE; ++c) acc[c & 7] += ex2_ftz(fmaf(v[c], p.scale2, -mnew));
              } else {
#pragma unroll
                for (int c = 0; c < TC_TILE; ++c) acc[c & 7] += c < nv ? ex2_ftz(fmaf(v[c], p.scale2, -mnew)) : 0.f;
              }
              const float at = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
              lsum = lsum * ex2_ftz(m2 - mnew) + at;
              m2 = mnew;
            }
          }
        } else {
          const int n = n0 + t;
          if (n < p.N) {
            const int pos = p.key_pos ? p.key_pos[n] : n;
            const int imin = pos - Lw;                 // rows with window index >= imin see the key
            float acc[8];
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[c] = 0.f;
            if (imin <= 0) {
#pragma unroll
              for (int c = 0; c < TC_ROWS; c += 4) {
                const float4 l4 = *reinterpret_cast<const float4*>(lse_s + c);
                acc[(c + 0) & 7] += ex2_ftz(fmaf(v[c + 0], p.scale2, -l4.x));
                acc[(c + 1) & 7] += ex2_ftz(fmaf(v[c + 1], p.scale2, -l4.y));
                acc[(c + 2) & 7] += ex2_ftz(fmaf(v[c + 2], p.scale2, -l4.z));
                acc[(c + 3) & 7] += ex2_ftz(fmaf(v[c + 3], p.scale2, -l4.w));
              }
            } else {
#pragma unroll
              for (int c = 0; c < TC_ROWS; ++c)
                acc[c & 7] += win_s[c] >= imin ? ex2_ftz(fmaf(v[c], p.scale2, -lse_s[c])) : 0.f;
            }
            p.score[(size_t)s * p.N + n] =
                ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
          }
        }
      }
      tiles_before += j1 - j0;
      // both groups meet here whatever happened; any failed wait stops every epilogue warp
      if (named_bar_or(2, NEPI, !ok)) { ok = false; break; }
      if (p1) {
        // merge the two groups' running stats of row t, then write the item's partial
        if (grp == 1) xch[t] = make_float2(m2, lsum);
        named_bar_sync(2, NEPI);
        if (grp == 0) {
          const float2 o = xch[t];
          const float M = fmaxf(m2, o.x);
          float l = 0.f;
          if (M != -INFINITY)
            l = (m2 == -INFINITY ? 0.f : lsum * ex2_ftz(m2 - M)) + (o.x == -INFINITY ? 0.f : o.y * ex2_ftz(o.x - M));
          if (PASS == 1) {
            if (t < p.R) p.part[((size_t)s * p.nsplit + sp) * p.R + t] = make_float2(M, l);
          } else {
            // fused: this CTA's stats of row t go to slot `me` of every CTA in the cluster
            // (every row, so the byte count each CTA expects is fixed)
            if (!cl_waited) { cluster_wait(); cl_waited = true; }
            const uint32_t me = cluster_rank();
            float2* mine = xall + me * TC_ROWS + t;
            for (int r = 0; r < p.nsplit; ++r) {
              if (r == (int)me) *mine = make_float2(M, l);
              else st_async_f32x2(map_to_rank(mine, (uint32_t)r), M, l, map_to_rank(xbar, (uint32_t)r));
            }
            if (t == 0) mbar_arrive_expect_tx(xbar, (uint32_t)((p.nsplit - 1) * TC_ROWS * 8));
          }
        }
      }
      }   // sweeps
    }
    // fused: do not leave while other CTAs may still be sending into this one
    if (PASS == 3 && grp == 0 && !x_waited) mbar_wait_cluster(xbar, 0);
  }
  if (PASS == 3 && !cl_waited) cluster_wait();

  // the producer and MMA lanes drained their own operations above
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tc_dealloc(tmem_base, TC_TMEM_COLS);
}

// lse2[s][r] = M + log2(sum over splits of l * 2^(m - M))
__global__ void score_lse2_merge(const float2* __restrict__ part, int nsplit, int R, float* __restrict__ lse2) {
  const int s = blockIdx.x;
  for (int r = threadIdx.x; r < R; r += blockDim.x) {
    float M = -INFINITY;
    for (int b = 0; b < nsplit; ++b) M = fmaxf(M, part[((size_t)s * nsplit + b) * R + r].x);
    float l = 0.f;
    if (M != -INFINITY)
      for (int b = 0; b < nsplit; ++b) {
        const float2 q = part[((size_t)s * nsplit + b) * R + r];
        if (q.x != -INFINITY) l += q.y * exp2f(q.x - M);
      }
    lse2[(size_t)s * R + r] = l > 0.f ? M + log2f(l) : INFINITY;
  }
}

// natural-log row normalisers supplied by the caller -> log2 domain
__global__ void lse_to_lse2(const float* __restrict__ lse, int n, float* __restrict__ lse2) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x)
    lse2[i] = lse[i] * 1.4426950408889634f;
}

// ---------------------------------------------------------------- host side
inline int tc_tiles_per_item(int S, long long N, int sms) {
  const long long tiles = (N + TC_TILE - 1) / TC_TILE;
  int best = 1;
  double best_cost = 1e300;
  for (int tpi = 1; tpi <= 64 && tpi <= tiles; ++tpi) {
    const long long items = (long long)S * ((tiles + tpi - 1) / tpi);
    const long long rounds = (items + sms - 1) / sms;
    const double cost = (double)rounds * (tpi + 1.0);   // +1: per-item Q load and pipeline ramp
    if (cost < best_cost - 1e-9) { best_cost = cost; best = tpi; }
  }
  return best;
}

inline long long tc_num_splits(int S, long long N, int sms) {
  const long long tiles = (N + TC_TILE - 1) / TC_TILE;
  const int tpi = tc_tiles_per_item(S, N, sms);
  return (tiles + tpi - 1) / tpi;
}

inline bool tc_supported(const kvc_shape* sh, int cc_major, int cc_minor) {
  (void)cc_minor;
  return cc_major == 10 && sh->dtype == KVC_BF16 && (sh->d == 64 || sh->d == 128) && sh->G * sh->w <= TC_ROWS;
}

typedef CUresult (*encode_tiled_fn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                    const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                    CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline encode_tiled_fn get_encode_tiled() {
  static encode_tiled_fn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<encode_tiled_fn>(ptr);
  }
  return fn;
}

// bf16 tensor [slots][rows][d] with a box of 64 elements x box_rows rows x 1 slot, 128-byte swizzle.
inline bool make_map_3d(CUtensorMap* m, const void* base, int d, long long rows, int slots, int box_rows) {
  encode_tiled_fn enc = get_encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)slots};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)rows * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Can one cluster of k fused scoring CTAs be resident (k up to 16 needs a GPC that large)?
template <int D>
bool tc_cluster_fits(int k, size_t smem) {
  static std::mutex mu;
  static std::map<std::pair<int, int>, bool> known;
  int dev = 0;
  cudaGetDevice(&dev);
  std::lock_guard<std::mutex> lk(mu);
  auto it = known.find({k, dev});
  if (it != known.end()) return it->second;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(k);
  cfg.blockDim = dim3(TC_THREADS);
  cfg.dynamicSmemBytes = smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = k;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int n = 0;
  const bool ok = cudaOccupancyMaxActiveClusters(&n, score_tc_kernel<D, 3>, &cfg) == cudaSuccess && n >= 1;
  cudaGetLastError();
  known[{k, dev}] = ok;
  return ok;
}

template <int D>
kvc_status tc_score_d(const kvc_shape* sh, const void* q_win, const void* k, const int32_t* chunk_end, int32_t C,
                      const float* row_lse, float* score, float2* part, float* lse2, void* keys_ws, int sms,
                      cudaStream_t st, fail_fn fail, unsigned* launches, bool force_two_pass) {
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
  CUtensorMap mq, mk;
  if (!make_map_3d(&mq, q_win, D, R, S, TC_ROWS) || !make_map_3d(&mk, kbase, D, krows, S, TC_TILE))
    return fail(KVC_ERR_CUDA, "kvc_score: cuTensorMapEncodeTiled failed");
  TcParams p{};
  p.S = S; p.N = N; p.L = L; p.w = sh->w; p.R = R; p.G = sh->G;
  p.tiles = (N + TC_TILE - 1) / TC_TILE;
  p.tpi = tc_tiles_per_item(S, N, sms);
  p.nsplit = (p.tiles + p.tpi - 1) / p.tpi;
  p.scale2 = 1.4426950408889634f / sqrtf((float)D);
  p.key_pos = chunk_end;
  p.part = part;
  p.lse2 = lse2;
  p.score = score;
  const size_t smem = TcSmem<D>::ALLOC;
  static bool attr_set[2][64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  const int di = D == 128 ? 1 : 0;
  if (dev >= 0 && dev < 64 && !attr_set[di][dev]) {
    cudaError_t e = cudaFuncSetAttribute(score_tc_kernel<D, 1>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(score_tc_kernel<D, 2>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(score_tc_kernel<D, 3>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(score_tc_kernel<D, 3>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return fail(KVC_ERR_CUDA, "kvc_score: kernel attribute: %s", cudaGetErrorString(e));
    attr_set[di][dev] = true;
  }
  // Fused (one launch: both passes and the row-normaliser merge inside slot clusters) when
  // the clusters of k = SMs / S CTAs keep >= 3/4 of the SMs busy and every CTA has at least
  // 8 key tiles per pass to amortise its setup and the exchange; pass 2 then re-reads keys
  // that pass 1 just brought into L2.
  if (!row_lse && !force_two_pass) {
    int k = std::min(TC_MAX_CLUSTER, sms / std::max(S, 1));
    k = std::min(k, p.tiles);
    if (k >= 1) {
      const int tpi = (p.tiles + k - 1) / k;
      k = (p.tiles + tpi - 1) / tpi;               // no empty key range
      if (4LL * S * k >= 3LL * sms && tpi >= 8 && tc_cluster_fits<D>(k, smem)) {
        TcParams pf = p;
        pf.tpi = tpi;
        pf.nsplit = k;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(S * k);
        cfg.blockDim = dim3(TC_THREADS);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = k;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        cudaError_t e = cudaLaunchKernelEx(&cfg, score_tc_kernel<D, 3>, mq, mk, pf);
        if (e != cudaSuccess) return fail(KVC_ERR_CUDA, "kvc_score: fused launch: %s", cudaGetErrorString(e));
        ++*launches;
        return KVC_OK;
      }
    }
  }
  const int items = S * p.nsplit;
  const int grid = std::min(items, sms);
  if (!row_lse) {
    score_tc_kernel<D, 1><<<grid, TC_THREADS, smem, st>>>(mq, mk, p);
    score_lse2_merge<<<S, 128, 0, st>>>(part, p.nsplit, R, lse2);
    *launches += 2;
  } else {
    lse_to_lse2<<<std::max(1, std::min((S * R + 255) / 256, sms * 4)), 256, 0, st>>>(row_lse, S * R, lse2);
    ++*launches;
  }
  score_tc_kernel<D, 2><<<grid, TC_THREADS, smem, st>>>(mq, mk, p);
  ++*launches;
  return KVC_OK;
}

inline kvc_status tc_score(const kvc_shape* sh, const void* q_win, const void* k, const int32_t* chunk_end, int32_t C,
                           const float* row_lse, float* score, float2* part, float* lse2, void* keys_ws, int sms,
                           cudaStream_t st, fail_fn fail, unsigned* launches, bool force_two_pass) {
  if (sh->d == 128)
    return tc_score_d<128>(sh, q_win, k, chunk_end, C, row_lse, score, part, lse2, keys_ws, sms, st, fail, launches,
                           force_two_pass);
  return tc_score_d<64>(sh, q_win, k, chunk_end, C, row_lse, score, part, lse2, keys_ws, sms, st, fail, launches,
                        force_two_pass);
}

}  // namespace kvc
