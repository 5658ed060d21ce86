// Split-K GQA decode attention over the ragged packed cache, bf16, on the tensor
// cores through warp-level mma.sync (m16n8k16, fp32 accumulation).
//
// For query head h of slot s = h / G (ZigZagKV / FastGen / ChunkLLM decode over
// the compacted cache):
//   out[h] = sum_{r < len[s]} softmax_r(q_h . K[off_s + r] / sqrt(d)) V[off_s + r].
//
// Two work splits, chosen on the device from the plan lengths:
//  - token ranges (as the CUDA-core decode, decode.cuh): the tokens of all slots are
//    cut into ranges of equal cost, one per CTA, ranges may cross slot boundaries,
//    and the last CTA to finish a slot merges the partials through global memory;
//  - per-slot clusters, for few near-uniform slots: slot j gets cluster j of k CTAs,
//    each sends its record (outputs, maxima, sums) into rank 0's shared memory by
//    st.async and rank 0 merges them.
// Inside a CTA, eight consumer warps (two groups of four, alternate 64-token tiles)
// each keep an online-softmax partial; one barrier publishes the unscaled partials
// and the combining threads rescale them to the common maximum.
//
// Why tensor cores here: the kernel is HBM-bound (4 flop per byte at G = 4), but
// on the CUDA cores it needed ~67 warp instructions per cached token and stayed
// issue-latency bound near 3 TB/s. As tiny MMAs the dot products cost a few
// instructions per token:
//   S^T [16 tokens x 8 heads] = K_tile [16 x d] . Q^T [d x 8]   (heads padded to 8)
//   O^T [d x 8 heads]        += V^T [d x 16 tokens] . P^T [16 x 8]
// K and V tiles arrive by TMA with the 128-byte swizzle so ldmatrix (and
// ldmatrix.trans for V^T) reads them without bank conflicts; the probabilities
// move from the S^T accumulator layout to the P^T operand layout with movmatrix,
// split into bf16 hi + lo parts so P keeps ~16 mantissa bits; m, l and O stay fp32.
#pragma once
#include "common.cuh"
#include "decode.cuh"
#include "score_sm100.cuh"

namespace kvc {

template <int D>
struct DmCfg {
  static constexpr int KB = D / 64;                  // 128-byte k-blocks per row
  static constexpr int TILE = 64;                    // tokens per stage
  static constexpr int REGION = TILE * 128;          // one k-block of one tile (8 KB)
  static constexpr int STAGE_BYTES = 2 * KB * REGION;
  static constexpr int MAX_STAGES = 6;              // pipeline depth chosen at launch: 4 or 6 (even, see the launcher)
  static constexpr int GROUP_WARPS = 4;              // a group takes a tile: one 16-token m-tile per warp
  static constexpr int CONS_WARPS = 2 * GROUP_WARPS; // two groups take alternate tiles
  static constexpr int CONS_THREADS = CONS_WARPS * 32;
  static constexpr int THREADS = CONS_THREADS + 32;
  static constexpr int KSTEPS = D / 16;
  static constexpr int DTILES = D / 16;
  static constexpr int WO_STRIDE = D + 4;            // padded head row of the in-CTA combine buffer
};

// Online-softmax rescale threshold (log2 units): a warp keeps its running maximum until
// a logit exceeds it by more than this, so most tiles skip the max reduction and the
// rescale; probabilities then stay below 2^8, far inside fp32 and the bf16 hi/lo split.
constexpr float DM_LAZY_LOG2 = 8.f;
constexpr int DM_MIN_TOKENS_PER_CTA = 64;            // token split: no CTA gets less than a tile
constexpr long long DM_SEG_COST = 256;               // token split: fixed work of one slot segment, in tokens
constexpr int DM_MAX_CLUSTER = 8;
constexpr int DM_APPENDS = 1 << 30;                  // flag in the per-slot row count: the last row is appended

// Shared-memory layout of decode_mma_kernel (host and device agree on it).
struct DmLayout {
  size_t stages, qbuf, bars, P, offs, wm, wo, xr, vl, total;
  template <int D>
  KVC_HD static DmLayout make(int S, int G, int grid, int nst) {
    using C = DmCfg<D>;
    DmLayout l{};
    size_t o = 0;
    l.stages = o;  o += (size_t)nst * C::STAGE_BYTES;                // 1024-byte aligned base
    l.qbuf = o;    o += (size_t)nst * G * D * 2;                     // the slot's q, one per stage
    l.bars = o;    o += (2 * C::MAX_STAGES + 1) * sizeof(uint64_t);  // full, empty, rank 0's record barrier
    l.P = o;       o += (size_t)(S + 1) * sizeof(long long);
    l.offs = o;    o += (size_t)S * sizeof(int);                      // row offsets (< 2^31, as TMA rows)
    l.wm = o;      o += 2 * C::CONS_WARPS * 8 * sizeof(float);       // per-warp max and sum, 8 heads
    l.wo = o;      o += (size_t)C::CONS_WARPS * G * C::WO_STRIDE * sizeof(float);
    // per-slot clusters: the k CTA records [k][G*D + 2G, padded] that rank 0 merges
    const size_t clu = 2 * S <= grid ? (size_t)DM_MAX_CLUSTER * partial_stride(G, D) * sizeof(float) : 0;
    l.xr = o;      o += clu;
    l.vl = o;      o += (size_t)S * sizeof(int);                      // rows attended per slot | DM_APPENDS
    l.total = o + 1024 + 16;                                          // base alignment slack
    return l;
  }
};

template <int D>
inline size_t decode_mma_smem_bytes(int S, int G, int grid, int nst) {
  return DmLayout::make<D>(S, G, grid, nst).total;
}

KVC_DEV void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
KVC_DEV void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
KVC_DEV void mma_bf16(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                      uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
KVC_DEV uint32_t movmatrix_t(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
KVC_DEV uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}
KVC_DEV float bf16_round(float x) { return __bfloat162float(__float2bfloat16_rn(x)); }

// Byte offset of (row, 16-byte chunk) in a 128-byte-swizzled region of 128-byte rows.
KVC_DEV uint32_t swz(int row, int chunk) { return (uint32_t)(row * 128 + ((chunk ^ (row & 7)) << 4)); }

// 2-D bf16 tensor [rows][d] with a box of 64 elements x box_rows rows, 128-byte swizzle.
inline bool make_map_2d_rows(CUtensorMap* m, encode_tiled_fn enc, const void* base, int d, long long rows,
                             int box_rows) {
  cuuint64_t dims[2] = {(cuuint64_t)d, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)d * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

KVC_DEV void tma_load_2d(void* smem_dst, const CUtensorMap* map, int c0, int c1, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], "
      "[%4];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// The last CTA to finish slot s in the token split merges the slot's CTA partials
// (CTAs cfirst..clast, stored consecutively at index c + s). Each thread owns one float4
// column of the outputs and folds the partials in groups of 8 whose (max, sum, column)
// loads are issued together, so up to 8 partials cost one round trip to L2.
KVC_DEV void merge_partials_par(const DecodeParams& a, int s, int G, int D, int cfirst, int clast, int tid,
                                int nthr) {
  const int np = clast - cfirst + 1;
  const size_t stride = (size_t)partial_stride(G, D);
  const float* base = a.partial + (size_t)(cfirst + s) * stride;
  const int nq = G * D / 4;
  for (int c4 = tid; c4 < nq; c4 += nthr) {
    const int h = (c4 * 4) / D;
    float M = -INFINITY, Lt = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int p0 = 0; p0 < np; p0 += 8) {
      float m[8], l[8];
      float4 v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const bool in = p0 + k < np;
        const float* pp = base + (size_t)(p0 + k) * stride;
        m[k] = in ? __ldcg(pp + (size_t)G * D + h) : -INFINITY;
        l[k] = in ? __ldcg(pp + (size_t)G * D + G + h) : 0.f;
        v[k] = in ? __ldcg(reinterpret_cast<const float4*>(pp) + c4) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float Mn = M;
#pragma unroll
      for (int k = 0; k < 8; ++k) Mn = fmaxf(Mn, m[k]);
      if (Mn == -INFINITY) continue;
      const float sc = M == -INFINITY ? 0.f : ex2_ftz(M - Mn);
      Lt *= sc;
      acc.x *= sc; acc.y *= sc; acc.z *= sc; acc.w *= sc;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float w = m[k] == -INFINITY ? 0.f : ex2_ftz(m[k] - Mn);
        Lt += l[k] * w;
        acc.x += v[k].x * w; acc.y += v[k].y * w; acc.z += v[k].z * w; acc.w += v[k].w * w;
      }
      M = Mn;
    }
    const float li = Lt > 0.f ? 1.f / Lt : 0.f;
    reinterpret_cast<float4*>(a.out + (size_t)s * G * D)[c4] = make_float4(acc.x * li, acc.y * li, acc.z * li, acc.w * li);
  }
}

// Two ways to split the work, chosen on the device from the lengths (every CTA reads
// all of them and reaches the same choice):
//  * per-slot clusters - when the grid was launched in clusters of k CTAs, every slot
//    fits one cluster, the clusters cover >= 3/4 of the grid and the lengths are near
//    uniform (max * S <= 1.25 * total): slot j gets cluster j, whose k CTAs split its
//    tokens evenly; each CTA pushes its record (outputs, max, sum) into rank 0's shared
//    memory and rank 0 merges the k records after one cluster barrier;
//  * token ranges - otherwise: the valid tokens of all slots are cut into equal ranges
//    of at least DM_MIN_TOKENS_PER_CTA (ranges may cross slots); a slot covered by one
//    CTA is written directly, otherwise partials merge through global tickets.
// Inside a CTA, warp 4 issues the TMA loads (K and V tiles, and the slot's q with the
// first tile of a segment) and warps 0-3 each take 16 tokens of every 64-token tile.
// PACK (G <= 4): the Q^T operand repeats heads 0-3 in columns 4-7, so the same S^T
// columns 4-7 let the P^T operand carry the bf16 remainder of p next to its bf16 high
// part, and one O MMA per d-tile accumulates both (summed once per segment).
template <int D, bool PACK>
__global__ void __launch_bounds__(DmCfg<D>::THREADS, 1)
decode_mma_kernel(const __grid_constant__ CUtensorMap mk64, const __grid_constant__ CUtensorMap mk16,
                  const __grid_constant__ CUtensorMap mv64, const __grid_constant__ CUtensorMap mv16,
                  DecodeParams a, int G, int ksz, int nst) {
  using C = DmCfg<D>;
  extern __shared__ __align__(1024) unsigned char dm_raw[];
  const uint32_t raw = smem_u32(dm_raw);
  unsigned char* sm = dm_raw + (((raw + 1023u) & ~1023u) - raw);
  const int S = a.S;
  const DmLayout lay = DmLayout::make<D>(S, G, gridDim.x, nst);
  unsigned char* stages = sm + lay.stages;
  unsigned char* qbuf = sm + lay.qbuf;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + lay.bars);
  uint64_t* empty = full + C::MAX_STAGES;
  uint64_t* rec_bar = empty + C::MAX_STAGES;   // rank 0 of a slot cluster: the other CTAs' records (st.async bytes)
  long long* P = reinterpret_cast<long long*>(sm + lay.P);
  int* offs = reinterpret_cast<int*>(sm + lay.offs);
  float* wm = reinterpret_cast<float*>(sm + lay.wm);        // [warp][8] maxima
  float* wl = wm + C::CONS_WARPS * 8;                        // [warp][8] sums
  float* wo = reinterpret_cast<float*>(sm + lay.wo);        // [warp][G][WO_STRIDE]
  float* xr = reinterpret_cast<float*>(sm + lay.xr);
  int* vlen_sh = reinterpret_cast<int*>(sm + lay.vl);
  // rows attended in slot s; with the fused append the last of them is the new token
  auto vlen = [&](int s) { return vlen_sh[s] & ~DM_APPENDS; };
  auto appends = [&](int s) { return (vlen_sh[s] & DM_APPENDS) != 0; };
  __shared__ unsigned long long scan_sh[33];
  __shared__ int last_flag;
  __shared__ int abort_flag;
  __shared__ unsigned long long max_len_sh;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) {
    max_len_sh = 0;
    abort_flag = 0;
    for (int i = 0; i < nst; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], C::GROUP_WARPS);
    }
    mbar_init(rec_bar, 1);
    fence_mbar_init();
  }
  if (warp == C::CONS_WARPS && lane == 0) {
    prefetch_tensormap(&mk64);
    prefetch_tensormap(&mv64);
    prefetch_tensormap(&mk16);
    prefetch_tensormap(&mv16);
  }
  // cluster launch: every CTA's barrier initialisation is visible cluster-wide before
  // any CTA sends to another (the matching wait comes before the first st.async)
  if (ksz >= 2) cluster_arrive_relaxed();
  bool cl_waited = false;
  // The work is planned on the slots' capacities when the call appends (the decode loop
  // never writes cap), otherwise on the lengths. `early`: the caller promises that the
  // previous kernel on the stream wrote none of off, cap, stable and no K/V row below
  // stable[s]; the plan, and the loads of the first tiles below stable[s], then run before
  // the dependency wait (programmatic dependent launch). Otherwise nothing before the wait
  // reads global memory that an earlier kernel writes.
  const bool plan_cap = a.append != 0;
  const bool early = plan_cap && a.stable != nullptr;
  if (!early) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }

  // Fused append, slot s of plan length n: the rows attended (*vl) and whether the new
  // token is the last of them (*ap) - the slot has room below cap and the buffer. The same
  // test decides, in the CTA that ends last, which lengths grow.
  auto append_rows = [&](int s, int ln, int cp, long long n, long long* vl_out, bool* ap_out) {
    const long long room = a.kp_rows - offs[s];
    long long vl = max(ln, 0);
    bool bad = false;
    if (vl > room) {
      bad = true;
      vl = room > 0 ? room : 0;
    }
    bool ap = ln >= 0 && vl < cp && vl < room && vl < n;
    if (ap) ++vl;
    if (vl > n) {                      // a length beyond the capacity
      bad = true;
      vl = n;
    }
    if (early) {
      const long long st = min((long long)max(a.stable[s], 0), n);
      if (vl < st) {
        bad = true;
        ap = false;
        vl = st;
      }
    }
    *vl_out = vl;
    *ap_out = ap;
    return bad;
  };
  // plan lengths (clipped to the buffer), their prefix over the slots, and the largest one
  unsigned long long carry = 0, mxl = 0;
  for (int base = 0; base < S; base += blockDim.x) {
    const int s = base + tid;
    unsigned long long x = 0;
    if (s < S) {
      // every global read of the slot first, so that their latencies overlap
      long long os = a.off[s];
      const int cp = plan_cap ? a.cap[s] : 0;   // cap is NULL for a plain decode
      const int ln = (!plan_cap || !early) ? a.len[s] : 0;
      if (os < 0 || os > a.kp_rows) {   // an offset outside the buffer: nothing of the slot is read or written
        kvc_flag(KVC_DEVERR_INDEX_RANGE);
        os = a.kp_rows;
      }
      offs[s] = (int)os;                // kp_rows < 2^31 (checked at launch)
      const long long room = a.kp_rows - os;
      long long n = max(plan_cap ? cp : ln, 0);
      if (n > room) {
        if (!plan_cap) kvc_flag(KVC_DEVERR_INDEX_RANGE);
        n = room > 0 ? room : 0;
      }
      x = (unsigned long long)n;
      mxl = x > mxl ? x : mxl;
      if (!early) {                     // the lengths are readable already: rows attended, in the same pass
        int v = (int)n;
        if (plan_cap) {
          long long vl;
          bool ap;
          append_rows(s, ln, cp, n, &vl, &ap);
          v = (int)vl | (ap ? DM_APPENDS : 0);
        }
        vlen_sh[s] = v;
      }
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
  __syncthreads();

  const long long N = P[S];
  const int nC = gridDim.x, c = blockIdx.x;
  // Token split by cost: every slot segment a CTA touches costs DM_SEG_COST tokens' worth
  // of fixed work (its last partial tile, the combine, the output or partial), so token t
  // of slot s sits at cost t + (s + 1) DM_SEG_COST and CTAs get equal cost ranges; a CTA
  // that crosses many short slots gets fewer tokens.
  const long long T = N + (long long)S * DM_SEG_COST;
  auto token_at_cost = [&](long long x) -> long long {   // first token whose cost is >= x
    if (x >= T) return N;
    int lo = 0, hi = S - 1;                                // last slot whose cost range starts <= x
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (P[mid] + (long long)mid * DM_SEG_COST <= x) lo = mid; else hi = mid - 1;
    }
    return max(P[lo], x - (long long)(lo + 1) * DM_SEG_COST);
  };
  // per-slot clusters: launched in clusters, every slot has one, they fill >= 3/4 of
  // the grid, and the plan lengths are near uniform (the same test in every CTA)
  const bool per_slot = ksz >= 2 && (long long)S * ksz <= nC && 4LL * S * ksz >= 3LL * nC &&
                        4LL * (long long)max_len_sh * S <= 5LL * N;
  const int my_cluster = per_slot ? (int)((unsigned)c / (unsigned)ksz) : c;
  const bool in_slot_cluster = per_slot && my_cluster < S;
  int nE = 0;
  bool active = false;
  long long b0 = 0, b1 = 0;
  if (!per_slot) {
    for (int s = c; s < S; s += nC)
      if (P[s + 1] == P[s])
        for (int e = tid; e < G * D; e += blockDim.x) a.out[(size_t)s * G * D + e] = 0.f;
    nE = (int)min((long long)nC, (N + DM_MIN_TOKENS_PER_CTA - 1) / DM_MIN_TOKENS_PER_CTA);
    if (N > 0 && c < nE) {
      b0 = token_at_cost((long long)c * T / nE);
      b1 = token_at_cost((long long)(c + 1) * T / nE);
    }
    active = b1 > b0;
  } else if (in_slot_cluster) {
    const long long ns = P[my_cluster + 1] - P[my_cluster];
    const unsigned r = cluster_rank(), k = (unsigned)ksz;
    if (ns < (1LL << 27)) {            // 32-bit arithmetic (a 64-bit division costs hundreds of cycles)
      const unsigned n32 = (unsigned)ns;
      b0 = P[my_cluster] + r * n32 / k;
      b1 = P[my_cluster] + (r + 1) * n32 / k;
    } else {
      b0 = P[my_cluster] + (long long)r * ns / ksz;
      b1 = P[my_cluster] + (long long)(r + 1) * ns / ksz;
    }
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
  // the CTA whose cost range holds token t of slot s
  auto cta_of = [&](long long t, int s) {
    const long long x = t + (long long)(s + 1) * DM_SEG_COST;
    return (int)(((x + 1) * nE - 1) / T);
  };
  const uint32_t q_bytes = (uint32_t)(G * D * 2);

  // Early: the producer starts the K/V loads of the first full tiles of the CTA's first
  // segment that lie below stable[s] - the same tiles, in the same order and stages, that
  // its main loop takes first. They carry no q: the consumers read the first segment's q
  // themselves after the wait.
  int nspec = 0;
  if (early && warp == C::CONS_WARPS && lane == 0 && active) {
    const int s = slot_of(b0);
    const long long seg_end = min(b1, P[s + 1]);
    const long long st_end = min(seg_end, P[s] + (long long)max(a.stable[s], 0));
    for (long long u = b0; u + C::TILE <= st_end && nspec < nst; u += C::TILE) {
      const int row0 = (int)(offs[s] + (u - P[s]));
      unsigned char* kdst = stages + nspec * C::STAGE_BYTES;
      unsigned char* vdst = kdst + C::KB * C::REGION;
      mbar_arrive_expect_tx(&full[nspec], 2 * C::KB * C::REGION);
#pragma unroll
      for (int kb = 0; kb < C::KB; ++kb) {
        tma_load_2d(kdst + kb * C::REGION, &mk64, kb * 64, row0, &full[nspec]);
        tma_load_2d(vdst + kb * C::REGION, &mv64, kb * 64, row0, &full[nspec]);
      }
      ++nspec;
    }
  }
  if (early) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  }
  // Early: the consumers' Q^T operand of the first segment, straight from global memory
  // (q is written by the previous kernel; its tiles carry none), overlapping the reads below
  const int g_ = (tid & 31) >> 2, qd_ = tid & 3;
  const int qhead0 = PACK ? (g_ & 3) : g_;
  uint32_t q0[C::KSTEPS][2];
  if (early && warp < C::CONS_WARPS && active) {
    const unsigned char* qg = static_cast<const unsigned char*>(a.q) + (size_t)slot_of(b0) * q_bytes;
#pragma unroll
    for (int ks = 0; ks < C::KSTEPS; ++ks) {
      uint32_t v0 = 0, v1 = 0;
      if (qhead0 < G) {
        const unsigned char* qr = qg + ((size_t)qhead0 * D + ks * 16 + 2 * qd_) * 2;
        v0 = __ldg(reinterpret_cast<const unsigned int*>(qr));
        v1 = __ldg(reinterpret_cast<const unsigned int*>(qr + 16));
      }
      q0[ks][0] = v0;
      q0[ks][1] = v1;
    }
  }

  // Early: rows attended in each slot this CTA touches, now that the lengths (written by
  // the previous launch) can be read: the length plus the new token as the last row where
  // the slot has room. A slot is never attended over fewer than its stable rows; a shorter
  // length breaks the caller's promise: flagged, and the slot gets no new token.
  // The producer, maybe still issuing those loads, takes no part: the consumers read the
  // lengths, sync among themselves and release the producer through barrier 2.
  if (early && warp < C::CONS_WARPS) {
    int s_lo = 0, s_hi = -1;
    if (per_slot) {
      if (in_slot_cluster) s_lo = s_hi = my_cluster;
    } else if (active) {
      s_lo = slot_of(b0);
      s_hi = slot_of(b1 - 1);
    }
    for (int s = s_lo + tid; s <= s_hi; s += C::CONS_THREADS) {
      const long long n = P[s + 1] - P[s];
      int v = (int)n;
      if (plan_cap) {
        long long vl;
        bool ap;
        append_rows(s, a.len[s], a.cap[s], n, &vl, &ap);
        v = (int)vl | (ap ? DM_APPENDS : 0);
      }
      vlen_sh[s] = v;
    }
    named_bar_sync(3, C::CONS_THREADS);
    named_bar_arrive(2, C::THREADS);
  } else if (early) {
    __syncwarp();
    named_bar_sync(2, C::THREADS);     // the consumers have written the rows attended
  }

  // Fused append: every CTA has read len once it gets here. Its ticket is taken now (a
  // release: the CTA's reads of len come first; no acquire, so warp 0 does not wait for
  // it) but only looked at when the CTA ends; the CTA that drew the last ticket then
  // publishes the new lengths (nothing in this launch reads len after this point). The
  // ticket stays on a consumer thread: drawn in the producer warp, chained steps measured
  // wrong lengths (cause not found).
  int ticket = -1;
  if (a.append && tid == 0)
    asm volatile("atom.release.gpu.global.add.s32 %0, [%1], 1;" : "=r"(ticket) : "l"(&a.counters[S]), "r"(1) : "memory");

  if (warp == C::CONS_WARPS) {
    // ---------------- producer: TMA of 64-token K and V tiles (16-row boxes for a partial
    // tile); the first tile of a segment also brings the slot's q
    if (lane == 0 && active) {
      int stage = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      for (long long t = b0; t < b1 && ok;) {
        const int s = slot_of(t);
        const long long seg_end = min(b1, P[s + 1]);
        const long long vend = min(seg_end, P[s] + (long long)vlen(s));   // attended rows of the segment
        for (long long u = t; u < vend; u += C::TILE) {
          const int rows = (int)min((long long)C::TILE, vend - u);
          if (issued < nspec) {            // on its way since before the wait
            ++issued;
            if (++stage == nst) { stage = 0; ph ^= 1; }
            continue;
          }
          // the first nst tiles find their stages free
          if ((issued >= nst && !mbar_wait(&empty[stage], ph ^ 1)) || *(volatile int*)&abort_flag) {
            ok = false;
            break;
          }
          const int row0 = (int)(offs[s] + (u - P[s]));
          unsigned char* kdst = stages + stage * C::STAGE_BYTES;
          unsigned char* vdst = kdst + C::KB * C::REGION;
          const uint32_t qb = q_bytes;   // q rides with every tile: either group may start the segment
          if (rows == C::TILE) {
            mbar_arrive_expect_tx(&full[stage], 2 * C::KB * C::REGION + qb);
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb) {
              tma_load_2d(kdst + kb * C::REGION, &mk64, kb * 64, row0, &full[stage]);
              tma_load_2d(vdst + kb * C::REGION, &mv64, kb * 64, row0, &full[stage]);
            }
          } else {
            const int nbox = (rows + 15) / 16;
            mbar_arrive_expect_tx(&full[stage], 2 * C::KB * nbox * 16 * 128 + qb);
            for (int bx = 0; bx < nbox; ++bx)
#pragma unroll
              for (int kb = 0; kb < C::KB; ++kb) {
                tma_load_2d(kdst + kb * C::REGION + bx * 16 * 128, &mk16, kb * 64, row0 + bx * 16, &full[stage]);
                tma_load_2d(vdst + kb * C::REGION + bx * 16 * 128, &mv16, kb * 64, row0 + bx * 16, &full[stage]);
              }
          }
          if (qb)
            bulk_g2s(qbuf + (size_t)stage * q_bytes, static_cast<const unsigned char*>(a.q) + (size_t)s * q_bytes,
                     q_bytes, &full[stage]);
          ++issued;
          if (++stage == nst) { stage = 0; ph ^= 1; }
        }
        t = seg_end;
      }
      if (!ok) *(volatile int*)&abort_flag = 1;
      // every load issued has landed before the CTA may exit
      for (long long k = issued > nst ? issued - nst : 0; k < issued; ++k)
        mbar_wait(&full[k % nst], (uint32_t)((k / nst) & 1));
    }
    __syncwarp();
  } else if (active || in_slot_cluster) {
    // ---------------- consumers: group cw / 4 takes the tiles of its parity (counted over the
    // CTA), and warp cw owns rows [16 (cw % 4), + 16) of each of them; two groups keep two
    // tiles' dependency chains in flight on every SM sub-partition
    const int cw = warp;
    const int grp = cw / C::GROUP_WARPS;
    const int g = lane >> 2, qd = lane & 3;                 // fragment row group, column pair
    const int mrow0 = 16 * (cw % C::GROUP_WARPS);
    const int lm_j = lane >> 3, lm_r = lane & 7;            // ldmatrix lane roles
    // heads of this thread's S^T / O^T columns 2qd and 2qd + 1
    const int hc0 = PACK ? 2 * (qd & 1) : 2 * qd, hc1 = hc0 + 1;
    const bool lo_cols = PACK && qd >= 2;                   // columns carrying the bf16 remainder
    const bool own = PACK ? qd < 2 : true;                  // lanes that hold final head values
    const bool hv0 = own && hc0 < G, hv1 = own && hc1 < G;
    const int qhead = PACK ? (g & 3) : g;                   // head of Q^T column g
    int stage = 0;
    uint32_t ph = 0;
    long long tile_k = 0;                                   // tiles of this CTA so far
    bool aborted = false;
    bool pending_empty = in_slot_cluster && !active;       // a cluster CTA without tokens: one empty record
    for (long long t = b0; (t < b1 && !aborted) || pending_empty;) {
      pending_empty = false;
      const int s = slot_of(t);
      const long long seg_end = active ? min(b1, P[s + 1]) : t;
      const long long vend = min(seg_end, P[s] + (long long)vlen(s));   // attended rows of the segment

      uint32_t qb[C::KSTEPS][2];
      float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
      float o[C::DTILES][4];
#pragma unroll
      for (int dt = 0; dt < C::DTILES; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;

      bool have_q = false;
      for (long long u = t; u < vend; u += C::TILE, ++tile_k) {
        if ((int)(tile_k & 1) != grp) {      // the other group's tile
          if (++stage == nst) { stage = 0; ph ^= 1; }
          continue;
        }
        const int rows = (int)min((long long)C::TILE, vend - u);
        if (!mbar_wait(&full[stage], ph)) {   // the group's warps wait on this barrier: all stop here
          *(volatile int*)&abort_flag = 1;
          aborted = true;
          break;
        }
        if (!have_q && early && t == b0) {   // the first segment's q, read after the wait
          have_q = true;
#pragma unroll
          for (int ks = 0; ks < C::KSTEPS; ++ks) {
            qb[ks][0] = q0[ks][0];
            qb[ks][1] = q0[ks][1];
          }
        }
        if (!have_q) {
          have_q = true;
          // Q^T operand (k = d, n = head) from the copy that came with this tile
          const unsigned char* qs = qbuf + (size_t)stage * q_bytes;
#pragma unroll
          for (int ks = 0; ks < C::KSTEPS; ++ks) {
            uint32_t v0 = 0, v1 = 0;
            if (qhead < G) {
              const unsigned char* qr = qs + ((size_t)qhead * D + ks * 16 + 2 * qd) * 2;
              v0 = *reinterpret_cast<const uint32_t*>(qr);
              v1 = *reinterpret_cast<const uint32_t*>(qr + 16);
            }
            qb[ks][0] = v0;
            qb[ks][1] = v1;
          }
        }
        unsigned char* Ks = stages + stage * C::STAGE_BYTES;
        unsigned char* Vs = Ks + C::KB * C::REGION;
        const int mv = rows - mrow0;                       // valid rows of this warp's m-tile
        // fused append: the slot's new token is its last valid row; if it falls in this
        // warp's m-tile, put it into the staged tile (the cache row is stale) and the cache
        bool patched = false;
        const long long arow_t = appends(s) ? P[s] + vlen(s) - 1 : -1;   // the appended token, in plan space
        if (arow_t >= u && arow_t < u + rows) {
          const int tr = (int)(arow_t - u);
          if (tr >= mrow0 && tr < mrow0 + 16) {
            const uint4* kn = static_cast<const uint4*>(a.k_new) + (size_t)s * (D / 8);
            const uint4* vn = static_cast<const uint4*>(a.v_new) + (size_t)s * (D / 8);
            const size_t dst_row = (size_t)(offs[s] + vlen(s) - 1) * (D / 8);
            for (int ch = lane; ch < D / 8; ch += 32) {
              const uint4 kv = kn[ch], vv = vn[ch];
              *reinterpret_cast<uint4*>(Ks + (ch >> 3) * C::REGION + swz(tr, ch & 7)) = kv;
              *reinterpret_cast<uint4*>(Vs + (ch >> 3) * C::REGION + swz(tr, ch & 7)) = vv;
              reinterpret_cast<uint4*>(const_cast<void*>(a.kp))[dst_row + ch] = kv;
              reinterpret_cast<uint4*>(const_cast<void*>(a.vp))[dst_row + ch] = vv;
            }
            patched = true;
            __syncwarp();
          }
        }
        if (mv > 0) {
          if (mv < 16) {
            // rows past the segment may hold anything (another slot, unwritten capacity):
            // zero those V rows so 0 * V stays 0 in the MMA
            for (int e = lane; e < (16 - mv) * 8 * C::KB; e += 32) {
              const int rr = mrow0 + mv + e / (8 * C::KB);
              const int rest = e % (8 * C::KB);
              *reinterpret_cast<uint4*>(Vs + (rest / 8) * C::REGION + rr * 128 + (rest % 8) * 16) =
                  make_uint4(0, 0, 0, 0);
            }
            __syncwarp();
          }
          // S^T = K_tile . Q^T in four independent accumulators (short dependency chains)
          float c4[4][4];
#pragma unroll
          for (int i = 0; i < 4; ++i) c4[i][0] = c4[i][1] = c4[i][2] = c4[i][3] = 0.f;
          const int arow = mrow0 + lm_r + 8 * (lm_j & 1);
#pragma unroll
          for (int ks = 0; ks < C::KSTEPS; ++ks) {
            const int kb = ks >> 2;
            const int chunk = (ks & 3) * 2 + (lm_j >> 1);
            uint32_t a0, a1, a2, a3;
            ldsm_x4(smem_u32(Ks + kb * C::REGION + swz(arow, chunk)), a0, a1, a2, a3);
            mma_bf16(c4[ks & 3], a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
          }
          float cs[4];
#pragma unroll
          for (int i = 0; i < 4; ++i) cs[i] = (c4[0][i] + c4[1][i]) + (c4[2][i] + c4[3][i]);
          // tokens t0 = g, t1 = g + 8 of the m-tile; columns 2qd, 2qd + 1
          const bool v0 = g < mv, v1 = g + 8 < mv;
          const float s00 = v0 ? cs[0] * a.scale_log2 : -INFINITY;
          const float s01 = v0 ? cs[1] * a.scale_log2 : -INFINITY;
          const float s10 = v1 ? cs[2] * a.scale_log2 : -INFINITY;
          const float s11 = v1 ? cs[3] * a.scale_log2 : -INFINITY;
          const bool need = s00 > m0 + DM_LAZY_LOG2 || s10 > m0 + DM_LAZY_LOG2 || s01 > m1 + DM_LAZY_LOG2 ||
                            s11 > m1 + DM_LAZY_LOG2;
          if (__any_sync(0xffffffffu, need)) {
            float mx0 = fmaxf(s00, s10), mx1 = fmaxf(s01, s11);
#pragma unroll
            for (int o_ = 4; o_ < 32; o_ <<= 1) {
              mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o_));
              mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o_));
            }
            // row g = 0 of the m-tile is valid, so both maxima are finite here
            const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
            const float al0 = ex2_ftz(m0 - n0), al1 = ex2_ftz(m1 - n1);   // 0 while m was -inf
            m0 = n0;
            m1 = n1;
            l0 *= al0;
            l1 *= al1;
#pragma unroll
            for (int dt = 0; dt < C::DTILES; ++dt) {
              o[dt][0] *= al0;
              o[dt][1] *= al1;
              o[dt][2] *= al0;
              o[dt][3] *= al1;
            }
          }
          const float p00 = ex2_ftz(s00 - m0), p01 = ex2_ftz(s01 - m1);   // exp2(-inf) = 0
          const float p10 = ex2_ftz(s10 - m0), p11 = ex2_ftz(s11 - m1);
          l0 += p00 + p10;
          l1 += p01 + p11;
          // P^T operand (k = token, n = column): transpose the 8x8 blocks with movmatrix
          const float r00 = bf16_round(p00), r01 = bf16_round(p01), r10 = bf16_round(p10), r11 = bf16_round(p11);
          const int vrow = mrow0 + lm_r + 8 * (lm_j >> 1);
          if (PACK) {
            // pick each lane's values first: movmatrix is a warp-wide .aligned instruction,
            // so every lane must execute the same one
            const uint32_t x0 = lo_cols ? pack_bf16(p00 - r00, p01 - r01) : pack_bf16(r00, r01);
            const uint32_t x1 = lo_cols ? pack_bf16(p10 - r10, p11 - r11) : pack_bf16(r10, r11);
            const uint32_t b0 = movmatrix_t(x0);
            const uint32_t b1 = movmatrix_t(x1);
#pragma unroll
            for (int dt = 0; dt < C::DTILES; ++dt) {
              const int dcol = dt * 16 + 8 * (lm_j & 1);
              uint32_t a0, a1, a2, a3;
              ldsm_x4_t(smem_u32(Vs + (dcol >> 6) * C::REGION + swz(vrow, (dcol & 63) >> 3)), a0, a1, a2, a3);
              mma_bf16(o[dt], a0, a1, a2, a3, b0, b1);
            }
          } else {
            const uint32_t bh0 = movmatrix_t(pack_bf16(r00, r01));
            const uint32_t bh1 = movmatrix_t(pack_bf16(r10, r11));
            const uint32_t bl0 = movmatrix_t(pack_bf16(p00 - r00, p01 - r01));
            const uint32_t bl1 = movmatrix_t(pack_bf16(p10 - r10, p11 - r11));
#pragma unroll
            for (int dt = 0; dt < C::DTILES; ++dt) {
              const int dcol = dt * 16 + 8 * (lm_j & 1);
              uint32_t a0, a1, a2, a3;
              ldsm_x4_t(smem_u32(Vs + (dcol >> 6) * C::REGION + swz(vrow, (dcol & 63) >> 3)), a0, a1, a2, a3);
              mma_bf16(o[dt], a0, a1, a2, a3, bh0, bh1);
              mma_bf16(o[dt], a0, a1, a2, a3, bl0, bl1);
            }
          }
          if (mv < 16) fence_proxy_async();      // our generic writes precede the next TMA into this stage
        }
        if (patched) fence_proxy_async();
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[stage]);
        if (++stage == nst) { stage = 0; ph ^= 1; }
      }
      // ---- the warp's totals: l over its 8 row groups; PACK adds the remainder columns
#pragma unroll
      for (int o_ = 4; o_ < 32; o_ <<= 1) {
        l0 += __shfl_xor_sync(0xffffffffu, l0, o_);
        l1 += __shfl_xor_sync(0xffffffffu, l1, o_);
      }
      if (PACK) {
#pragma unroll
        for (int dt = 0; dt < C::DTILES; ++dt)
#pragma unroll
          for (int j = 0; j < 4; ++j) o[dt][j] += __shfl_down_sync(0xffffffffu, o[dt][j], 2, 4);
      }
      // ---- the warp's partial, unscaled (its own maximum m, sum l and output O); the combine
      // below rescales each to the heads' common maximum
      if (g == 0) {
        if (hv0) {
          wm[cw * 8 + hc0] = m0;
          wl[cw * 8 + hc0] = l0;
        }
        if (hv1) {
          wm[cw * 8 + hc1] = m1;
          wl[cw * 8 + hc1] = l1;
        }
      }
      float* wow = wo + (size_t)cw * G * C::WO_STRIDE;
#pragma unroll
      for (int dt = 0; dt < C::DTILES; ++dt) {
        const int d0 = dt * 16 + g;
        if (hv0) {
          wow[hc0 * C::WO_STRIDE + d0] = o[dt][0];
          wow[hc0 * C::WO_STRIDE + d0 + 8] = o[dt][2];
        }
        if (hv1) {
          wow[hc1 * C::WO_STRIDE + d0] = o[dt][1];
          wow[hc1 * C::WO_STRIDE + d0 + 8] = o[dt][3];
        }
      }
      // one barrier for both: the partials are visible to every consumer thread, and the two
      // groups (which wait on different stage barriers) agree on an abort
      if (named_bar_or(1, C::CONS_THREADS, aborted)) {
        aborted = true;
        break;
      }

      const int cfirst = per_slot ? 0 : cta_of(P[s], s), clast = per_slot ? 0 : cta_of(P[s + 1] - 1, s);
      const bool single = !per_slot && cfirst == clast;
      float* mypart = a.partial + (size_t)(c + s) * partial_stride(G, D);
      const uint32_t my_rank = per_slot ? cluster_rank() : 0u;
      float* rec = xr + (size_t)my_rank * partial_stride(G, D);   // this CTA's record in rank 0's memory
      uint32_t rec_remote = 0, bar_remote = 0;
      if (per_slot) {
        // rank 0's barrier is initialised (cluster-wide arrive at the start); the record goes
        // there by st.async, counted on rank 0's record barrier
        cluster_wait();
        cl_waited = true;
        if (my_rank != 0) {
          rec_remote = map_to_rank(rec, 0);
          bar_remote = map_to_rank(rec_bar, 0);
        }
      }
      for (int e = tid; e < G * D; e += C::CONS_THREADS) {
        const int h = e / D, d = e - h * D;
        float Mh = -INFINITY;
#pragma unroll
        for (int w = 0; w < C::CONS_WARPS; ++w) Mh = fmaxf(Mh, wm[w * 8 + h]);
        // each warp's share scaled by 2^(m_w - M): rounded products, then a sum in warp order
        float A = 0.f, Lh = 0.f;
#pragma unroll
        for (int w = 0; w < C::CONS_WARPS; ++w) {
          const float mw = wm[w * 8 + h];
          const float f = mw == -INFINITY ? 0.f : ex2_ftz(mw - Mh);
          A += __fmul_rn(wo[((size_t)w * G + h) * C::WO_STRIDE + d], f);
          Lh += __fmul_rn(wl[w * 8 + h], f);
        }
        if (per_slot && my_rank == 0) {
          rec[e] = A;
          if (d == 0) {
            rec[G * D + h] = Mh;
            rec[G * D + G + h] = Lh;
          }
        } else if (per_slot) {
          st_async_f32(rec_remote + 4u * (uint32_t)e, A, bar_remote);
          if (d == 0) {
            st_async_f32(rec_remote + 4u * (uint32_t)(G * D + h), Mh, bar_remote);
            st_async_f32(rec_remote + 4u * (uint32_t)(G * D + G + h), Lh, bar_remote);
          }
        } else if (single) {
          a.out[(size_t)s * G * D + e] = Lh > 0.f ? A / Lh : 0.f;
        } else {
          mypart[e] = A;
          if (d == 0) {
            mypart[G * D + h] = Mh;
            mypart[G * D + G + h] = Lh;
          }
        }
      }
      if (!per_slot && !single) {
        // the CTA's partial writes, then one fenced ticket (the barrier + one-thread fence
        // orders every thread's writes before the atomic)
        named_bar_sync(1, C::CONS_THREADS);
        if (tid == 0) last_flag = slot_ticket(&a.counters[s], clast - cfirst);
        named_bar_sync(1, C::CONS_THREADS);
        if (last_flag) {
          merge_partials_par(a, s, G, D, cfirst, clast, tid, C::CONS_THREADS);
          if (tid == 0) a.counters[s] = 0;
        }
      }
      named_bar_sync(1, C::CONS_THREADS);   // wm / wo / xr are reused by the next segment
      t = seg_end;
    }

    if (in_slot_cluster && !aborted && cluster_rank() == 0) {
      // rank 0: its own record is in place; wait for the other ksz - 1, then merge
      const int rs = partial_stride(G, D);
      if (tid == 0) mbar_arrive_expect_tx(rec_bar, (uint32_t)((ksz - 1) * (G * D + 2 * G) * 4));
      if (mbar_wait_cluster(rec_bar, 0)) {
        // each thread weighs the records for its own outputs' head (no barrier)
        for (int e = tid; e < G * D; e += C::CONS_THREADS) {
          const int h = e / D;
          float M = -INFINITY;
          for (int r = 0; r < ksz; ++r) M = fmaxf(M, xr[r * rs + G * D + h]);
          float acc = 0.f, Lt = 0.f;
          for (int r = 0; r < ksz; ++r) {
            const float mr = xr[r * rs + G * D + h];
            const float w = mr == -INFINITY ? 0.f : ex2_ftz(mr - M);
            Lt += xr[r * rs + G * D + G + h] * w;
            acc += w * xr[r * rs + e];
          }
          const float linv = Lt > 0.f ? 1.f / Lt : 0.f;
          a.out[(size_t)my_cluster * G * D + e] = acc * linv;
        }
      }
    }
  }

  if (ksz >= 2 && !cl_waited) cluster_wait();

  if (a.append) {
    if (tid == 0) {
      last_flag = ticket == (int)gridDim.x - 1;
      if (last_flag) asm volatile("fence.acq_rel.gpu;" ::: "memory");   // after every CTA's reads of len
    }
    __syncthreads();
    if (last_flag) {
      // the same test as the rows pass above, for every slot
      for (int s = tid; s < S; s += blockDim.x) {
        long long vl;
        bool ap;
        if (append_rows(s, a.len[s], a.cap[s], P[s + 1] - P[s], &vl, &ap)) kvc_flag(KVC_DEVERR_INDEX_RANGE);
        if (ap) a.len_out[s] = a.len[s] + 1;
        else kvc_flag(KVC_DEVERR_APPEND_OVERFLOW);
      }
      if (tid == 0) a.counters[S] = 0;
    }
  }
}

}  // namespace kvc
