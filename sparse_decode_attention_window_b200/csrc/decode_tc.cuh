// Split-K GQA decode attention on the sm_100a tensor cores (tcgen05.mma, fp32 in TMEM),
// bf16 cache, d = 128.
//
// For query head h of slot s = h / G (ZigZagKV / FastGen / ChunkLLM decode over the
// compacted cache):
//   out[h] = sum_{r < len[s]} softmax_r(q_h . K[off_s + r] / sqrt(d)) V[off_s + r].
//
// Per 128-token tile of one slot, two MMAs with the tokens on the 128 TMEM lanes or
// in the reduction:
//   S^T [128 tokens x 16] = K_tile [128 x d] . Q^T [d x 16]     (heads in columns 0..G-1)
//   O^T [d x 16]         += V^T [d x 128 tokens] . P^T [128 x 16]
// K is the K-major A operand exactly as TMA lands it (128-byte swizzle); V^T is the same
// V tile read as an MN-major operand; Q^T and P^T are K-major B operands. Columns 0-7 of
// P^T carry the bf16 high part of each probability and columns 8-15 its bf16 remainder,
// so one MMA accumulates both and p keeps ~16 mantissa bits (m, l, O stay fp32).
//
// Warp roles (192 threads): warps 0-3 own TMEM lane quadrants - during a tile thread t is
// token t (softmax of its S^T row, its column of P^T), at a segment end it is output
// dimension t (its row of O^T); warp 4 issues the TMA loads (K, V and the 16 rows of q
// from the slot on, per stage); warp 5 owns the TMEM allocation and issues the MMAs,
// S of tile i+1 before O of tile i so the softmax of one tile overlaps the next product.
//
// The online softmax keeps one running maximum per head for the whole CTA and raises it
// only when a logit exceeds it by more than 2^8 (DM_LAZY_LOG2); a raise rescales the
// O^T accumulator in TMEM, which is rare after the first tile of a segment.
//
// The work split (per-slot clusters or token ranges) and the merges follow the
// mma.sync kernel in decode_mma.cuh; a cluster CTA sends its record to rank 0 with
// st.async, counted on an mbarrier there, so no cluster-wide barrier sits on the path.
//
// Measured on B200 this kernel is 10-20 % slower than the mma.sync one, which is why it
// is only a cross-check path (KVC_DECODE_PATH=tc): with N = 16 each group of eight MMAs
// takes ~0.5 us from issue to completion, and a stage stays busy from landing through
// S, the softmax and O, so at three 64 KB stages fewer bytes are in flight per SM than
// with the mma.sync kernel's four 32 KB stages that free as soon as a warp is done.
#pragma once
#include "common.cuh"
#include "decode.cuh"
#include "score_sm100.cuh"
#include "decode_mma.cuh"

namespace kvc {

struct DtCfg {
  static constexpr int D = 128;
  static constexpr int KB = D / 64;                  // 64-element (128-byte) k-blocks of a row
  static constexpr int TILE = 128;                   // tokens per stage
  static constexpr int NCOL = 16;                    // MMA N: 8 head columns + 8 remainder columns
  static constexpr int KREG = TILE * 128;            // one k-block of a K or V tile (16 KB)
  static constexpr int QREG = NCOL * 128;            // one k-block of the q tile (2 KB)
  static constexpr int STAGE_BYTES = 2 * KB * KREG + KB * QREG;   // K, V, q
  static constexpr int PREG = NCOL * 128;            // one 64-token block of P^T (2 KB)
  static constexpr int PBUF = (TILE / 64) * PREG;    // one P^T buffer (4 KB)
  static constexpr int CONS_WARPS = 4, PROD_WARP = 4, MMA_WARP = 5;
  static constexpr int CONS_THREADS = 32 * CONS_WARPS;
  static constexpr int THREADS = 32 * 6;
  static constexpr int TMEM_COLS = 64;               // S^T buffers at 0 and 16, O^T buffers at 32 and 48
  static constexpr int MIN_TOKENS_PER_CTA = TILE;    // token split: no CTA gets less than a tile
  static constexpr uint32_t IDESC_S = tc_idesc(128, NCOL);               // A, B K-major
  static constexpr uint32_t IDESC_O = tc_idesc(128, NCOL) | (1u << 15);  // A (V^T) MN-major
};

// Shared-memory layout of decode_tc_kernel (host and device agree on it).
struct DtLayout {
  int nst;                                           // pipeline stages (2 or 3)
  size_t stages, pbuf, bars, P, offs, red, xr, app, total;
  KVC_HD static DtLayout make(int S, int G, int /* grid: unused, kept for the callers */, int ksz, int nst) {
    using C = DtCfg;
    DtLayout l{};
    l.nst = nst;
    size_t o = 0;
    l.stages = o; o += (size_t)nst * C::STAGE_BYTES;       // 1024-byte aligned pieces
    l.pbuf = o;   o += 2 * (size_t)C::PBUF;
    l.bars = o;   o += 32 * sizeof(uint64_t);
    l.P = o;      o += (size_t)(S + 1) * sizeof(long long);
    l.offs = o;   o += (size_t)S * sizeof(long long);
    l.red = o;    o += 6 * C::CONS_WARPS * 8 * sizeof(float);     // maxima, sums [warp][8]; merge weights [8][8], 1/sum [8]
    // per-slot clusters: the ksz records that rank 0 merges, 16-byte aligned
    const size_t clu = ksz >= 2 ? (size_t)ksz * partial_stride(G, C::D) * sizeof(float) : 0;
    o = (o + 15) & ~(size_t)15;
    l.xr = o;     o += clu;
    l.app = o;    o += (size_t)S;
    l.total = o + 1024 + 16;                                // base alignment slack
    return l;
  }
};

// ---------------------------------------------------------------- PTX wrappers
// Shared-memory descriptor, 128-byte swizzle, with an explicit leading-dimension byte
// offset (the stride between 64-element atoms of an MN-major operand).
KVC_DEV uint64_t smem_desc_sw128_lbo(uint32_t saddr, uint32_t lbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)(1024u >> 4) << 32;                // 8-row groups 1024 bytes apart
  d |= (uint64_t)1u << 46;                          // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                          // 128-byte swizzle
  return d;
}

// 32 lanes x 8 consecutive fp32 columns.
KVC_DEV void tc_ld8(uint32_t taddr, float* v) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}
// 32 lanes x 16 consecutive fp32 columns.
KVC_DEV void tc_ld16(uint32_t taddr, float* v) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}
KVC_DEV void tc_st16(uint32_t taddr, const float* v) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, "
      "%15, %16};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])), "r"(__float_as_uint(v[3])),
      "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])), "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])),
      "r"(__float_as_uint(v[8])), "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])),
      "r"(__float_as_uint(v[11])), "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])),
      "r"(__float_as_uint(v[14])), "r"(__float_as_uint(v[15]))
      : "memory");
}
KVC_DEV void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Per-tile bookkeeping shared by the three roles: the CTA walks its token range
// [b0, b1) slot segment by slot segment in 128-token tiles; tile i (counted over the
// whole CTA) uses stage i % nst, S^T / P^T buffer i & 1, and the O^T buffer of its
// segment's parity.
__global__ void __launch_bounds__(DtCfg::THREADS, 1)
decode_tc_kernel(const __grid_constant__ CUtensorMap mk, const __grid_constant__ CUtensorMap mk16,
                 const __grid_constant__ CUtensorMap mv, const __grid_constant__ CUtensorMap mv16,
                 const __grid_constant__ CUtensorMap mq, DecodeParams a, int G, int ksz, int nst) {
  using C = DtCfg;
  constexpr int D = C::D;
  extern __shared__ __align__(1024) unsigned char dt_raw[];
  const uint32_t raw = smem_u32(dt_raw);
  unsigned char* sm = dt_raw + (((raw + 1023u) & ~1023u) - raw);
  const int S = a.S;
  const DtLayout lay = DtLayout::make(S, G, gridDim.x, ksz, nst);
  unsigned char* stages = sm + lay.stages;
  unsigned char* pbuf = sm + lay.pbuf;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + lay.bars);
  uint64_t* kv_full = bars;             // [nst]   TMA bytes
  uint64_t* kv_empty = bars + 3;        // [nst]   MMA commit after O of the stage's tile
  uint64_t* s_full = bars + 6;          // [2]     MMA commit after S
  uint64_t* s_empty = bars + 8;         // [2]     4 consumer warps have read S
  uint64_t* p_full = bars + 10;         // [2]     4 consumer warps have written P
  uint64_t* p_empty = bars + 12;        // [2]     MMA commit after O
  uint64_t* mma_done = bars + 14;       //         MMA commit after the last O (before the TMEM release)
  uint64_t* rec_bar = bars + 15;        //         rank 0: the other CTAs' records (st.async bytes)
  long long* P = reinterpret_cast<long long*>(sm + lay.P);
  long long* offs = reinterpret_cast<long long*>(sm + lay.offs);
  float* red = reinterpret_cast<float*>(sm + lay.red);   // see DtLayout
  float* xr = reinterpret_cast<float*>(sm + lay.xr);
  unsigned char* app = sm + lay.app;
  __shared__ unsigned long long scan_sh[33];
  __shared__ int last_flag;
  __shared__ int abort_flag;
  __shared__ unsigned long long max_len_sh;
  __shared__ uint32_t tmem_slot;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // Nothing before the dependency wait reads global memory that an earlier kernel writes.
  if (tid == 0) {
    max_len_sh = 0;
    abort_flag = 0;
    for (int i = 0; i < nst; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s_full[b], 1);
      mbar_init(&s_empty[b], C::CONS_WARPS);
      mbar_init(&p_full[b], C::CONS_WARPS);
      mbar_init(&p_empty[b], 1);
    }
    mbar_init(mma_done, 1);
    mbar_init(rec_bar, 1);
    fence_mbar_init();
  }
  if (warp == C::PROD_WARP && lane == 0) {
    prefetch_tensormap(&mk);
    prefetch_tensormap(&mv);
    prefetch_tensormap(&mq);
    prefetch_tensormap(&mk16);
    prefetch_tensormap(&mv16);
  }
  if (warp == C::MMA_WARP) tc_alloc(&tmem_slot, C::TMEM_COLS);
  // cluster launch: every CTA's barrier initialisation is visible cluster-wide before
  // any CTA sends to another (the matching wait comes before the first st.async)
  if (ksz >= 2) cluster_arrive_relaxed();
  bool cl_waited = false;
  // Launched with programmatic stream serialization: wait until the previous kernel on
  // the stream has completed and its writes are visible, then let the next one launch.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // ---- prologue: lengths (with the fused append's new token), their prefix, the maximum
  unsigned long long carry = 0, mxl = 0;
  for (int base = 0; base < S; base += blockDim.x) {
    const int s = base + tid;
    unsigned long long x = 0;
    if (s < S) {
      const int ln = a.len[s];
      const long long os = a.off[s];
      const int cp = a.append ? a.cap[s] : 0;
      long long n = max(ln, 0);
      offs[s] = os;
      const long long room = a.kp_rows - os;
      if (n > room) { kvc_flag(KVC_DEVERR_INDEX_RANGE); n = room > 0 ? room : 0; }
      unsigned char ap = 0;
      if (a.append) {
        if (ln >= 0 && n < cp && n < room) { ap = 1; ++n; }
        else if (blockIdx.x == 0) kvc_flag(KVC_DEVERR_APPEND_OVERFLOW);
      }
      app[s] = ap;
      x = (unsigned long long)n;
      mxl = x > mxl ? x : mxl;
    }
    unsigned long long tot;
    const unsigned long long before = carry + block_exclusive_scan<unsigned long long>(x, scan_sh, &tot);
    if (s < S) P[s] = (long long)before;
    carry += tot;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long y = __shfl_xor_sync(0xffffffffu, mxl, o);
    mxl = y > mxl ? y : mxl;
  }
  if (lane == 0) atomicMax(&max_len_sh, mxl);
  if (tid == 0) P[S] = (long long)carry;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_slot;

  // Fused append: every CTA has read len once it gets here. Its ticket is taken now but
  // only looked at when the CTA ends; the CTA that drew the last ticket then publishes
  // the new lengths (nothing in this launch reads len after its prologue).
  int ticket = -1;
  if (a.append && tid == 0)
    asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(ticket) : "l"(&a.counters[S]), "r"(1) : "memory");

  const long long N = P[S];
  const int nC = gridDim.x, c = blockIdx.x;
  const bool per_slot = ksz >= 2 && (long long)S * ksz <= nC && 4LL * S * ksz >= 3LL * nC &&
                        4LL * (long long)max_len_sh * S <= 5LL * N;
  const int my_cluster = c / (ksz > 0 ? ksz : 1);
  const bool in_slot_cluster = per_slot && my_cluster < S;
  int nE = 0;
  bool active = false;
  long long b0 = 0, b1 = 0;
  if (!per_slot) {
    for (int s = c; s < S; s += nC)
      if (P[s + 1] == P[s])
        for (int e = tid; e < G * D; e += blockDim.x) a.out[(size_t)s * G * D + e] = 0.f;
    nE = (int)min((long long)nC, (N + C::MIN_TOKENS_PER_CTA - 1) / C::MIN_TOKENS_PER_CTA);
    active = N > 0 && c < nE;
    b0 = active ? (long long)c * N / nE : 0;
    b1 = active ? (long long)(c + 1) * N / nE : 0;
  } else if (in_slot_cluster) {
    const long long r = (long long)cluster_rank(), ns = P[my_cluster + 1] - P[my_cluster];
    b0 = P[my_cluster] + r * ns / ksz;
    b1 = P[my_cluster] + (r + 1) * ns / ksz;
    active = b1 > b0;
  }
  auto slot_of = [&](long long t) {
    if (per_slot) return my_cluster;
    int lo = 0, hi = S - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (P[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  auto cta_of = [&](long long t) { return (int)(((t + 1) * nE - 1) / N); };

  if (warp == C::PROD_WARP) {
    // ---------------- producer: K and V tiles (16-row boxes for a partial tile) and the
    // 16 rows of q from the slot's first head on, into stage i % nst
    if (lane == 0 && active) {
      long long i = 0;
      bool ok = true;
      for (long long t = b0; t < b1 && ok;) {
        const int s = slot_of(t);
        const long long seg_end = min(b1, P[s + 1]);
        for (long long u = t; u < seg_end; u += C::TILE, ++i) {
          const int st = (int)(i % nst);
          const long long n = i / nst;
          if ((n > 0 && !mbar_wait(&kv_empty[st], (uint32_t)((n - 1) & 1))) || *(volatile int*)&abort_flag) {
            ok = false;
            break;
          }
          const int rows = (int)min((long long)C::TILE, seg_end - u);
          const int row0 = (int)(offs[s] + (u - P[s]));
          unsigned char* kdst = stages + (size_t)st * C::STAGE_BYTES;
          unsigned char* vdst = kdst + C::KB * C::KREG;
          unsigned char* qdst = vdst + C::KB * C::KREG;
          const int nbox = (rows + 15) / 16;
          const uint32_t kv_bytes = rows == C::TILE ? 2u * C::KB * C::KREG : 2u * C::KB * nbox * 16 * 128;
          mbar_arrive_expect_tx(&kv_full[st], kv_bytes + C::KB * C::QREG);
          if (rows == C::TILE) {
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb) {
              tma_load_2d(kdst + kb * C::KREG, &mk, kb * 64, row0, &kv_full[st]);
              tma_load_2d(vdst + kb * C::KREG, &mv, kb * 64, row0, &kv_full[st]);
            }
          } else {
            for (int bx = 0; bx < nbox; ++bx)
#pragma unroll
              for (int kb = 0; kb < C::KB; ++kb) {
                tma_load_2d(kdst + kb * C::KREG + bx * 2048, &mk16, kb * 64, row0 + bx * 16, &kv_full[st]);
                tma_load_2d(vdst + kb * C::KREG + bx * 2048, &mv16, kb * 64, row0 + bx * 16, &kv_full[st]);
              }
          }
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb) tma_load_2d(qdst + kb * C::QREG, &mq, kb * 64, s * G, &kv_full[st]);
        }
        t = seg_end;
      }
      if (!ok) *(volatile int*)&abort_flag = 1;
      // every load issued has landed before the CTA may exit
      for (long long k = i > nst ? i - nst : 0; k < i; ++k)
        mbar_wait(&kv_full[k % nst], (uint32_t)((k / nst) & 1));
    }
    __syncwarp();
  } else if (warp == C::MMA_WARP) {
    // ---------------- MMA issuer: S^T of tile i, then O^T of tile i - 1 (once its P^T is in)
    if (active) {
      long long i = 0, issued_o = 0;
      int seg = 0;
      bool ok = true;
      int pend_seg = 0;           // segment parity of the tile whose O^T is pending
      bool pend_first = false;    // ... and whether it starts its segment
      auto issue_o = [&](long long j) -> bool {
        const int bj = (int)(j & 1), stj = (int)(j % nst);
        if (!mbar_wait(&p_full[bj], (uint32_t)((j >> 1) & 1)) || *(volatile int*)&abort_flag) return false;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t d_tmem = tmem_base + 32u + 16u * (uint32_t)pend_seg;
          const uint32_t v_addr = smem_u32(stages + (size_t)stj * C::STAGE_BYTES + C::KB * C::KREG);
          const uint32_t p_addr = smem_u32(pbuf + bj * C::PBUF);
#pragma unroll
          for (int kt = 0; kt < C::TILE / 16; ++kt) {
            const uint64_t adesc = smem_desc_sw128_lbo(v_addr + kt * 2048, C::KREG);   // 16 tokens = 2 row groups
            const uint64_t bdesc = smem_desc_sw128(p_addr + (kt >> 2) * C::PREG + (kt & 3) * 32);
            tc_mma(d_tmem, adesc, bdesc, C::IDESC_O, (pend_first && kt == 0) ? 0u : 1u);
          }
          tc_commit(&kv_empty[stj]);   // K, V and q of the stage read
          tc_commit(&p_empty[bj]);     // P^T buffer read and O^T up to date with tile j
        }
        __syncwarp();
        ++issued_o;
        return true;
      };
      for (long long t = b0; t < b1 && ok; ++seg) {
        const int s = slot_of(t);
        const long long seg_end = min(b1, P[s + 1]);
        for (long long u = t; u < seg_end && ok; u += C::TILE, ++i) {
          const int st = (int)(i % nst), b = (int)(i & 1);
          const int rows = (int)min((long long)C::TILE, seg_end - u);
          unsigned char* kdst = stages + (size_t)st * C::STAGE_BYTES;
          unsigned char* vdst = kdst + C::KB * C::KREG;
          // fused append: the slot's new token is its last row; its K and V rows come from
          // k_new / v_new (loaded before the wait) into the staged tile and the cache
          const long long last = P[s + 1] - 1;
          const bool patch = app[s] && last >= u && last < u + rows;
          uint4 nv = make_uint4(0, 0, 0, 0);
          if (patch) {
            const uint4* src = static_cast<const uint4*>(lane < 16 ? a.k_new : a.v_new) + (size_t)s * (D / 8);
            nv = src[lane & 15];
          }
          if (!mbar_wait(&kv_full[st], (uint32_t)((i / nst) & 1)) || *(volatile int*)&abort_flag) { ok = false; break; }
          if (patch) {
            const int tr = (int)(last - u), ch = lane & 15;
            unsigned char* dst = (lane < 16 ? kdst : vdst) + (ch >> 3) * C::KREG + swz(tr, ch & 7);
            *reinterpret_cast<uint4*>(dst) = nv;
            void* cache = const_cast<void*>(lane < 16 ? a.kp : a.vp);
            reinterpret_cast<uint4*>(cache)[(size_t)(offs[s] + (last - P[s])) * (D / 8) + ch] = nv;
            fence_proxy_async();     // the generic writes precede the tensor core's reads
          }
          __syncwarp();
          if (i >= 2 && !mbar_wait(&s_empty[b], (uint32_t)(((i >> 1) - 1) & 1))) { ok = false; break; }
          tc_fence_after();
          if (lane == 0) {
            const uint32_t d_tmem = tmem_base + 16u * (uint32_t)b;
            const uint32_t k_addr = smem_u32(kdst);
            const uint32_t q_addr = smem_u32(vdst + C::KB * C::KREG);
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk)
                tc_mma(d_tmem, smem_desc_sw128(k_addr + kb * C::KREG + kk * 32),
                       smem_desc_sw128(q_addr + kb * C::QREG + kk * 32), C::IDESC_S, (kb | kk) != 0);
            tc_commit(&s_full[b]);
          }
          __syncwarp();
          if (i >= 1 && !issue_o(i - 1)) { ok = false; break; }
          pend_seg = seg & 1;
          pend_first = u == t;
        }
        t = seg_end;
      }
      if (ok && i >= 1) ok = issue_o(i - 1);
      if (!ok) *(volatile int*)&abort_flag = 1;
      // every MMA this warp issued has completed before the TMEM is released
      if (lane == 0 && (issued_o > 0 || i > 0)) {
        tc_commit(mma_done);
        mbar_wait(mma_done, 0);
      }
      __syncwarp();
    }
  } else if (active || in_slot_cluster) {
    // ---------------- consumers: thread t is token t of each tile, output dimension t at a
    // segment end (warp w reads TMEM lanes 32w .. 32w + 31)
    const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
    float* rmax = red;                          // [warp][8] tile maxima
    float* rsum = red + C::CONS_WARPS * 8;      // [warp][8] sums
    long long i = 0;
    int seg = 0;
    bool aborted = false;
    bool pending_empty = in_slot_cluster && !active;   // a cluster CTA without tokens: one empty record
    for (long long t = b0; (t < b1 && !aborted) || pending_empty; ++seg) {
      pending_empty = false;
      const int s = slot_of(t);
      const long long seg_end = active ? min(b1, P[s + 1]) : t;
      float m[8], l[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) { m[h] = -INFINITY; l[h] = 0.f; }
      long long last_i = -1;
      const uint32_t o_col = 32u + 16u * (uint32_t)(seg & 1);

      for (long long u = t; u < seg_end; u += C::TILE, ++i) {
        const int b = (int)(i & 1), st = (int)(i % nst);
        const int rows = (int)min((long long)C::TILE, seg_end - u);
        if (!mbar_wait(&s_full[b], (uint32_t)((i >> 1) & 1))) { aborted = true; break; }
        tc_fence_after();
        float sv[8];
        tc_ld8(tmem_base + lane_off + 16u * (uint32_t)b, sv);
        tc_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[b]);
        const bool valid = tid < rows;
        float z[8];
        bool need = false;
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          z[h] = (valid && h < G) ? sv[h] * a.scale_log2 : -INFINITY;
          need |= z[h] > m[h] + DM_LAZY_LOG2;
        }
        if (named_bar_or(2, C::CONS_THREADS, need)) {
          // raise the running maxima to this tile's (the same values in every thread)
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            float x = z[h];
#pragma unroll
            for (int o_ = 16; o_ > 0; o_ >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o_));
            if (lane == 0) rmax[warp * 8 + h] = x;
          }
          named_bar_sync(2, C::CONS_THREADS);
          float al[8];
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            float mx = m[h];
#pragma unroll
            for (int w = 0; w < C::CONS_WARPS; ++w) mx = fmaxf(mx, rmax[w * 8 + h]);
            al[h] = mx == -INFINITY ? 1.f : ex2_ftz(m[h] - mx);   // 0 while m was -inf
            m[h] = mx;
            l[h] *= al[h];
          }
          if (last_i >= 0) {
            // O^T holds this segment's earlier tiles: rescale it in TMEM once they are in
            // (p_empty of tile i - 1's buffer: this thread last waited on it one phase earlier)
            if (!mbar_wait(&p_empty[(i - 1) & 1], (uint32_t)(((i - 1) >> 1) & 1))) { aborted = true; break; }
            tc_fence_after();
            float ov[16];
            tc_ld16(tmem_base + lane_off + o_col, ov);
            tc_wait_ld();
#pragma unroll
            for (int h = 0; h < 8; ++h) {
              ov[h] *= al[h];
              ov[8 + h] *= al[h];
            }
            tc_st16(tmem_base + lane_off + o_col, ov);
            tc_wait_st();
            tc_fence_before();
          }
          named_bar_sync(2, C::CONS_THREADS);   // every thread has read rmax
        }
        float p[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          p[h] = z[h] == -INFINITY ? 0.f : ex2_ftz(z[h] - m[h]);
          l[h] += p[h];
        }
        if (i >= 2 && !mbar_wait(&p_empty[b], (uint32_t)(((i >> 1) - 1) & 1))) { aborted = true; break; }
        // P^T (K-major B operand, 128-byte swizzle): row h the bf16 high part, row 8 + h the
        // remainder, column = token
        {
          unsigned char* pb = pbuf + b * C::PBUF + (tid >> 6) * C::PREG;
          const int ch = (tid & 63) >> 3, within = (tid & 7) * 2;
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            if (h < G) {
              const __nv_bfloat16 hi = __float2bfloat16_rn(p[h]);
              const __nv_bfloat16 lo = __float2bfloat16_rn(p[h] - __bfloat162float(hi));
              *reinterpret_cast<__nv_bfloat16*>(pb + h * 128 + ((ch ^ h) << 4) + within) = hi;
              *reinterpret_cast<__nv_bfloat16*>(pb + (8 + h) * 128 + ((ch ^ h) << 4) + within) = lo;
            }
          }
        }
        if (!valid) {
          // rows past the segment may hold anything (another slot, unwritten capacity,
          // earlier tiles): zero this token's V row so 0 * V stays 0 in the MMA
          unsigned char* vrow = stages + (size_t)st * C::STAGE_BYTES + C::KB * C::KREG;
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb)
#pragma unroll
            for (int c8 = 0; c8 < 8; ++c8)
              *reinterpret_cast<uint4*>(vrow + kb * C::KREG + swz(tid, c8)) = make_uint4(0, 0, 0, 0);
        }
        fence_proxy_async();     // P^T and the zeroed rows precede the tensor core's reads
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[b]);
        last_i = i;
      }
      if (aborted) break;

      // ---- segment end: O^T row tid = output dimension tid of every head
      float o[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) o[h] = 0.f;
      if (last_i >= 0) {
        if (!mbar_wait(&p_empty[last_i & 1], (uint32_t)((last_i >> 1) & 1))) { aborted = true; break; }
        tc_fence_after();
        float ov[16];
        tc_ld16(tmem_base + lane_off + o_col, ov);
        tc_wait_ld();
        tc_fence_before();
#pragma unroll
        for (int h = 0; h < 8; ++h) o[h] = ov[h] + ov[8 + h];
      }
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        float x = l[h];
#pragma unroll
        for (int o_ = 16; o_ > 0; o_ >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o_);
        if (lane == 0) rsum[warp * 8 + h] = x;
      }
      named_bar_sync(2, C::CONS_THREADS);
      float L[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        L[h] = 0.f;
#pragma unroll
        for (int w = 0; w < C::CONS_WARPS; ++w) L[h] += rsum[w * 8 + h];
      }
      const int d = tid;
      const int rs = partial_stride(G, D);
      if (per_slot) {
        // send this CTA's record (outputs, maxima, sums) to rank 0; rank 0 merges
        cluster_wait();
        cl_waited = true;
        const uint32_t rank = cluster_rank();
        float* rec = xr + (size_t)rank * rs;
        if (rank == 0) {
#pragma unroll
          for (int h = 0; h < 8; ++h)
            if (h < G) {
              rec[h * D + d] = o[h];
              if (d == h) {
                rec[G * D + h] = m[h];
                rec[G * D + G + h] = L[h];
              }
            }
        } else {
          const uint32_t rb = map_to_rank(rec_bar, 0);
#pragma unroll
          for (int h = 0; h < 8; ++h)
            if (h < G) {
              st_async_f32(map_to_rank(rec + h * D + d, 0), o[h], rb);
              if (d == h) {
                st_async_f32(map_to_rank(rec + G * D + h, 0), m[h], rb);
                st_async_f32(map_to_rank(rec + G * D + G + h, 0), L[h], rb);
              }
            }
        }
      } else {
        const int cfirst = cta_of(P[s]), clast = cta_of(P[s + 1] - 1);
        if (cfirst == clast) {
#pragma unroll
          for (int h = 0; h < 8; ++h)
            if (h < G) a.out[((size_t)s * G + h) * D + d] = L[h] > 0.f ? o[h] / L[h] : 0.f;
        } else {
          float* mypart = a.partial + (size_t)(c + s) * rs;
#pragma unroll
          for (int h = 0; h < 8; ++h)
            if (h < G) {
              mypart[h * D + d] = o[h];
              if (d == h) {
                mypart[G * D + h] = m[h];
                mypart[G * D + G + h] = L[h];
              }
            }
          // the CTA's partial writes, then one fenced ticket (the barrier + one-thread fence
          // orders every thread's writes before the atomic)
          named_bar_sync(2, C::CONS_THREADS);
          if (tid == 0) last_flag = slot_ticket(&a.counters[s], clast - cfirst);
          named_bar_sync(2, C::CONS_THREADS);
          if (last_flag) {
            merge_partials_par(a, s, G, D, cfirst, clast, tid, C::CONS_THREADS);
            if (tid == 0) a.counters[s] = 0;
          }
        }
      }
      named_bar_sync(2, C::CONS_THREADS);   // rsum / xr are reused by the next segment
      t = seg_end;
    }
    if (aborted) *(volatile int*)&abort_flag = 1;

    if (in_slot_cluster && cluster_rank() == 0 && !aborted) {
      // rank 0: its own record is in place; wait for the other ksz - 1, then merge
      named_bar_sync(2, C::CONS_THREADS);
      const int rs = partial_stride(G, D);
      if (tid == 0) mbar_arrive_expect_tx(rec_bar, (uint32_t)((ksz - 1) * (G * D + 2 * G) * 4));
      if (mbar_wait_cluster(rec_bar, 0)) {
        float* sc = red + 2 * C::CONS_WARPS * 8;   // [ksz][8] weights, then 1 / sum [8]
        float* linv = sc + 8 * 8;
        if (tid < G) {
          float M = -INFINITY;
          for (int r = 0; r < ksz; ++r) M = fmaxf(M, xr[r * rs + G * D + tid]);
          float Lt = 0.f;
          for (int r = 0; r < ksz; ++r) {
            const float mr = xr[r * rs + G * D + tid];
            const float w = mr == -INFINITY ? 0.f : ex2_ftz(mr - M);
            sc[r * 8 + tid] = w;
            Lt += xr[r * rs + G * D + G + tid] * w;
          }
          linv[tid] = Lt > 0.f ? 1.f / Lt : 0.f;
        }
        named_bar_sync(2, C::CONS_THREADS);
        for (int h = 0; h < G; ++h) {
          float acc = 0.f;
          for (int r = 0; r < ksz; ++r) acc += sc[r * 8 + h] * xr[r * rs + h * D + tid];
          a.out[((size_t)my_cluster * G + h) * D + tid] = acc * linv[h];
        }
      }
    }
  }

  // ---- end: the cluster barrier pair, the fused append's length update, TMEM release
  if (ksz >= 2 && !cl_waited) cluster_wait();
  if (a.append) {
    if (tid == 0) last_flag = ticket == (int)gridDim.x - 1;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (a.append && last_flag) {
    for (int s = tid; s < S; s += blockDim.x)
      if (app[s]) a.len_out[s] = a.len[s] + 1;
    if (tid == 0) a.counters[S] = 0;
  }
  if (warp == C::MMA_WARP) tc_dealloc(tmem_base, C::TMEM_COLS);
}

}  // namespace kvc
