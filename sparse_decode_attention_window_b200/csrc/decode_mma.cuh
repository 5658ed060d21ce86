// Split-K GQA decode attention over the ragged packed cache, bf16, on the tensor
// cores through warp-level mma.sync (m16n8k16, fp32 accumulation).
//
// For query head h of slot s = h / G (ZigZagKV / FastGen / ChunkLLM decode over
// the compacted cache):
//   out[h] = sum_{r < len[s]} softmax_r(q_h . K[off_s + r] / sqrt(d)) V[off_s + r].
//
// The work split and the merge are those of the CUDA-core decode (decode.cuh):
// the valid tokens of all slots are cut into equal ranges, one per CTA, ranges may
// cross slot boundaries, and the last CTA to finish a slot merges its partials.
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
  static constexpr int STAGES = 4;
  static constexpr int CONS_WARPS = 4;               // each consumes one 16-token m-tile per stage
  static constexpr int THREADS = (CONS_WARPS + 1) * 32;
  static constexpr int KSTEPS = D / 16;
  static constexpr int DTILES = D / 16;
};

template <int D>
constexpr size_t decode_mma_smem_bytes(int S, int G, int grid) {
  using C = DmCfg<D>;
  return 1024 + (size_t)C::STAGES * C::STAGE_BYTES + 2 * C::STAGES * sizeof(uint64_t) +
         (size_t)(2 * S + 1) * sizeof(long long) + (size_t)C::CONS_WARPS * (2 * G + G * D) * sizeof(float) +
         (size_t)2 * grid * G * sizeof(float) + (size_t)G * (D + 2) * sizeof(float) + (size_t)S + 16;
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

KVC_DEV void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
KVC_DEV uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Read a float from the same shared-memory offset in CTA `rank` of this cluster.
KVC_DEV float ld_dsmem(const float* local, uint32_t rank) {
  uint32_t ra;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
  return v;
}

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

// Two ways to split the work, chosen on the device from the lengths (every CTA reads
// all of them and reaches the same choice):
//  * per-slot clusters - when the grid was launched in clusters of k CTAs, every slot
//    fits one cluster, the clusters cover >= 3/4 of the grid and the lengths are near
//    uniform (max * S <= 1.25 * total): slot j gets cluster j, whose k CTAs split its
//    tokens evenly and merge their k partials through distributed shared memory;
//  * token ranges - otherwise: the valid tokens of all slots are cut into gridDim.x
//    equal ranges (ranges may cross slots) and partials merge through global tickets.
template <int D>
__global__ void __launch_bounds__(DmCfg<D>::THREADS, 1)
decode_mma_kernel(const __grid_constant__ CUtensorMap mk64, const __grid_constant__ CUtensorMap mk16,
                  const __grid_constant__ CUtensorMap mv64, const __grid_constant__ CUtensorMap mv16,
                  DecodeParams a, int G, int ksz) {
  using C = DmCfg<D>;
  extern __shared__ __align__(1024) unsigned char dm_raw[];
  const uint32_t raw = smem_u32(dm_raw);
  unsigned char* sm = dm_raw + (((raw + 1023u) & ~1023u) - raw);
  unsigned char* stages = sm;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  long long* P = reinterpret_cast<long long*>(empty + C::STAGES);
  long long* offs = P + a.S + 1;                          // off[] of the slots
  float* comb = reinterpret_cast<float*>(offs + a.S);    // [warps][2G + G*D]
  float* cres = comb + C::CONS_WARPS * (2 * G + G * D) + 2 * gridDim.x * G;   // cluster mode: acc[G*D], m[G], l[G]
  unsigned char* app = reinterpret_cast<unsigned char*>(cres + G * (D + 2));
  __shared__ unsigned long long scan_sh[33];
  __shared__ int last_flag;
  __shared__ int abort_flag;
  __shared__ unsigned long long max_len_sh;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (tid == 0) max_len_sh = 0;
  __syncthreads();
  const int S = a.S;
  const __nv_bfloat16* q = static_cast<const __nv_bfloat16*>(a.q);

  // Launched with programmatic stream serialization: wait here until the previous
  // kernel on the stream has completed and its writes are visible (nothing above
  // reads global memory), then let the next kernel start its own launch.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // One slot's length (clipped to the buffer); with the fused append, a slot that has
  // room gets its new token as its last row.
  auto slot_len = [&](int s, unsigned char* ap_out, bool flag_overflow) -> long long {
    long long n = max(a.len[s], 0);
    const long long os = a.off[s];
    offs[s] = os;
    const long long room = a.kp_rows - os;
    if (n > room) { kvc_flag(KVC_DEVERR_INDEX_RANGE); n = room > 0 ? room : 0; }
    unsigned char ap = 0;
    if (a.append) {
      if (a.len[s] >= 0 && n < a.cap[s] && n < room) { ap = 1; ++n; }
      else if (flag_overflow) kvc_flag(KVC_DEVERR_APPEND_OVERFLOW);
    }
    *ap_out = ap;
    return n;
  };
  // prefix of the lengths over all slots, and the largest one
  unsigned long long carry = 0, mxl = 0;
  for (int base = 0; base < S; base += blockDim.x) {
    const int s = base + tid;
    unsigned long long x = 0;
    if (s < S) {
      unsigned char ap;
      x = (unsigned long long)slot_len(s, &ap, blockIdx.x == 0);
      app[s] = ap;
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
  if (tid == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], C::CONS_WARPS);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (a.append) {
    // every CTA has read len once its prologue is done; the last CTA to get here
    // publishes the new lengths (nothing in this launch reads len again)
    if (tid == 0) {
      int old;
      asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(&a.counters[S]), "r"(1) : "memory");
      last_flag = old == (int)gridDim.x - 1;
    }
    __syncthreads();
    if (last_flag) {
      for (int s = tid; s < S; s += blockDim.x)
        if (app[s]) a.len_out[s] = a.len[s] + 1;
      if (tid == 0) a.counters[S] = 0;
    }
  }

  const long long N = P[S];
  const int nC = gridDim.x, c = blockIdx.x;
  // per-slot clusters: launched in clusters, every slot has one, they fill >= 3/4 of
  // the grid, and the lengths are near uniform (the same test in every CTA)
  const bool per_slot = ksz >= 2 && (long long)S * ksz <= nC && 4LL * S * ksz >= 3LL * nC &&
                       4LL * (long long)max_len_sh * S <= 5LL * N;
  int nE = 0;
  bool active = false;
  long long b0 = 0, b1 = 0;
  const int my_cluster = c / (ksz > 0 ? ksz : 1);
  if (!per_slot) {
    for (int s = c; s < S; s += nC)
      if (P[s + 1] == P[s])
        for (int e = tid; e < G * D; e += blockDim.x) a.out[(size_t)s * G * D + e] = 0.f;
    nE = (int)min((long long)nC, N);
    active = N > 0 && c < nE;
    b0 = active ? (long long)c * N / nE : 0;
    b1 = active ? (long long)(c + 1) * N / nE : 0;
  } else if (my_cluster < S) {
    const int sl = my_cluster;
    const long long r = (long long)cluster_rank(), ns = P[sl + 1] - P[sl];
    b0 = P[sl] + r * ns / ksz;
    b1 = P[sl] + (r + 1) * ns / ksz;
    active = b1 > b0;
  }
  if (per_slot)
    for (int e = tid; e < G * (D + 2); e += blockDim.x) cres[e] = e >= G * D && e < G * D + G ? -INFINITY : 0.f;

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

  if (!active) {
    // nothing to stream
  } else if (warp == C::CONS_WARPS) {
    // ---------------- producer: TMA of 64-token K and V tiles (16-row boxes for a partial tile)
    if (lane == 0) {
      prefetch_tensormap(&mk64);
      prefetch_tensormap(&mv64);
      int stage = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      for (long long t = b0; t < b1 && ok;) {
        const int s = slot_of(t);
        const long long seg_end = min(b1, P[s + 1]);
        for (long long u = t; u < seg_end; u += C::TILE) {
          const int rows = (int)min((long long)C::TILE, seg_end - u);
          if (!mbar_wait(&empty[stage], ph ^ 1) || *(volatile int*)&abort_flag) { ok = false; break; }
          const int row0 = (int)(offs[s] + (u - P[s]));
          unsigned char* kdst = stages + stage * C::STAGE_BYTES;
          unsigned char* vdst = kdst + C::KB * C::REGION;
          if (rows == C::TILE) {
            mbar_arrive_expect_tx(&full[stage], 2 * C::KB * C::REGION);
#pragma unroll
            for (int kb = 0; kb < C::KB; ++kb) {
              tma_load_2d(kdst + kb * C::REGION, &mk64, kb * 64, row0, &full[stage]);
              tma_load_2d(vdst + kb * C::REGION, &mv64, kb * 64, row0, &full[stage]);
            }
          } else {
            const int nbox = (rows + 15) / 16;
            mbar_arrive_expect_tx(&full[stage], 2 * C::KB * nbox * 16 * 128);
            for (int bx = 0; bx < nbox; ++bx)
#pragma unroll
              for (int kb = 0; kb < C::KB; ++kb) {
                tma_load_2d(kdst + kb * C::REGION + bx * 16 * 128, &mk16, kb * 64, row0 + bx * 16, &full[stage]);
                tma_load_2d(vdst + kb * C::REGION + bx * 16 * 128, &mv16, kb * 64, row0 + bx * 16, &full[stage]);
              }
          }
          ++issued;
          if (++stage == C::STAGES) { stage = 0; ph ^= 1; }
        }
        t = seg_end;
      }
      if (!ok) *(volatile int*)&abort_flag = 1;
      // every load issued has landed before the CTA may exit
      for (long long k = issued > C::STAGES ? issued - C::STAGES : 0; k < issued; ++k)
        mbar_wait(&full[k % C::STAGES], (uint32_t)((k / C::STAGES) & 1));
    }
    __syncwarp();
  } else {
  // ---------------- consumers: warp cw owns rows [16 cw, 16 cw + 16) of every tile
  const int cw = warp;
  const int g = lane >> 2, qd = lane & 3;                 // fragment row group, column pair
  const int h0 = 2 * qd, h1 = 2 * qd + 1;                 // heads of this thread's S^T / O^T columns
  const int mrow0 = 16 * cw;
  // ldmatrix lane roles
  const int lm_j = lane >> 3, lm_r = lane & 7;
  int stage = 0;
  uint32_t ph = 0;
  bool aborted = false;
  for (long long t = b0; t < b1 && !aborted;) {
    const int s = slot_of(t);
    const long long seg_end = min(b1, P[s + 1]);

    // Q^T operand (k = d, n = head), heads >= G are zero
    uint32_t qb[C::KSTEPS][2];
    {
      const int head = g;
#pragma unroll
      for (int ks = 0; ks < C::KSTEPS; ++ks) {
        uint32_t v0 = 0, v1 = 0;
        if (head < G) {
          const __nv_bfloat16* qr = q + ((size_t)s * G + head) * D + ks * 16 + 2 * qd;
          v0 = *reinterpret_cast<const uint32_t*>(qr);
          v1 = *reinterpret_cast<const uint32_t*>(qr + 8);
        }
        qb[ks][0] = v0;
        qb[ks][1] = v1;
      }
    }
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float o[C::DTILES][4];
#pragma unroll
    for (int dt = 0; dt < C::DTILES; ++dt) o[dt][0] = o[dt][1] = o[dt][2] = o[dt][3] = 0.f;

    for (long long u = t; u < seg_end; u += C::TILE) {
      const int rows = (int)min((long long)C::TILE, seg_end - u);
      if (!mbar_wait(&full[stage], ph)) {   // every consumer warp waits on this barrier: all stop here
        *(volatile int*)&abort_flag = 1;
        aborted = true;
        break;
      }
      unsigned char* Ks = stages + stage * C::STAGE_BYTES;
      unsigned char* Vs = Ks + C::KB * C::REGION;
      const int mv = rows - mrow0;                       // valid rows of this warp's m-tile
      // fused append: the slot's new token is its last valid row; if it falls in this
      // warp's m-tile, put it into the staged tile (the cache row is stale) and the cache
      bool patched = false;
      if (app[s] && P[s + 1] - 1 >= u && P[s + 1] - 1 < u + rows) {
        const int tr = (int)(P[s + 1] - 1 - u);
        if (tr >= mrow0 && tr < mrow0 + 16) {
          const uint4* kn = static_cast<const uint4*>(a.k_new) + (size_t)s * (D / 8);
          const uint4* vn = static_cast<const uint4*>(a.v_new) + (size_t)s * (D / 8);
          const size_t dst_row = (size_t)(offs[s] + (P[s + 1] - 1 - P[s])) * (D / 8);
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
        // S^T = K_tile . Q^T
        float cs[4] = {0.f, 0.f, 0.f, 0.f};
        const int arow = mrow0 + lm_r + 8 * (lm_j & 1);
#pragma unroll
        for (int ks = 0; ks < C::KSTEPS; ++ks) {
          const int kb = ks >> 2;
          const int chunk = (ks & 3) * 2 + (lm_j >> 1);
          uint32_t a0, a1, a2, a3;
          ldsm_x4(smem_u32(Ks + kb * C::REGION + swz(arow, chunk)), a0, a1, a2, a3);
          mma_bf16(cs, a0, a1, a2, a3, qb[ks][0], qb[ks][1]);
        }
        // tokens t0 = g, t1 = g + 8 of the m-tile; heads h0, h1
        const bool v0 = g < mv, v1 = g + 8 < mv;
        const float s00 = v0 ? cs[0] * a.scale_log2 : -INFINITY;   // (t0, h0)
        const float s01 = v0 ? cs[1] * a.scale_log2 : -INFINITY;   // (t0, h1)
        const float s10 = v1 ? cs[2] * a.scale_log2 : -INFINITY;   // (t1, h0)
        const float s11 = v1 ? cs[3] * a.scale_log2 : -INFINITY;   // (t1, h1)
        float mx0 = fmaxf(s00, s10), mx1 = fmaxf(s01, s11);
#pragma unroll
        for (int o_ = 4; o_ < 32; o_ <<= 1) {
          mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o_));
          mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o_));
        }
        const float n0 = fmaxf(m0, mx0), n1 = fmaxf(m1, mx1);
        const float al0 = n0 == -INFINITY ? 1.f : exp2f(m0 - n0);
        const float al1 = n1 == -INFINITY ? 1.f : exp2f(m1 - n1);
        m0 = n0;
        m1 = n1;
        const float p00 = s00 == -INFINITY ? 0.f : exp2f(s00 - n0);
        const float p01 = s01 == -INFINITY ? 0.f : exp2f(s01 - n1);
        const float p10 = s10 == -INFINITY ? 0.f : exp2f(s10 - n0);
        const float p11 = s11 == -INFINITY ? 0.f : exp2f(s11 - n1);
        l0 = l0 * al0 + p00 + p10;
        l1 = l1 * al1 + p01 + p11;
        if (al0 != 1.f || al1 != 1.f) {
#pragma unroll
          for (int dt = 0; dt < C::DTILES; ++dt) {
            o[dt][0] *= al0;
            o[dt][1] *= al1;
            o[dt][2] *= al0;
            o[dt][3] *= al1;
          }
        }
        // P^T operand (k = token, n = head): transpose the 8x8 blocks, hi + lo bf16 parts
        const float r00 = bf16_round(p00), r01 = bf16_round(p01), r10 = bf16_round(p10), r11 = bf16_round(p11);
        const uint32_t bh0 = movmatrix_t(pack_bf16(r00, r01));
        const uint32_t bh1 = movmatrix_t(pack_bf16(r10, r11));
        const uint32_t bl0 = movmatrix_t(pack_bf16(p00 - r00, p01 - r01));
        const uint32_t bl1 = movmatrix_t(pack_bf16(p10 - r10, p11 - r11));
        // O^T += V^T . P^T
        const int vrow = mrow0 + lm_r + 8 * (lm_j >> 1);
#pragma unroll
        for (int dt = 0; dt < C::DTILES; ++dt) {
          const int dcol = dt * 16 + 8 * (lm_j & 1);      // first d of this lane's 8x8 block
          const int kb = dcol >> 6;
          const int chunk = (dcol & 63) >> 3;
          uint32_t a0, a1, a2, a3;
          ldsm_x4_t(smem_u32(Vs + kb * C::REGION + swz(vrow, chunk)), a0, a1, a2, a3);
          mma_bf16(o[dt], a0, a1, a2, a3, bh0, bh1);
          mma_bf16(o[dt], a0, a1, a2, a3, bl0, bl1);
        }
        if (mv < 16) fence_proxy_async();      // our generic writes precede the next TMA into this stage
      }
      if (patched) fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (++stage == C::STAGES) { stage = 0; ph ^= 1; }
    }

    if (aborted) break;
    // ---- per-warp totals: l over the 8 token rows of the fragment
#pragma unroll
    for (int o_ = 4; o_ < 32; o_ <<= 1) {
      l0 += __shfl_xor_sync(0xffffffffu, l0, o_);
      l1 += __shfl_xor_sync(0xffffffffu, l1, o_);
    }
    float* cm = comb + cw * (2 * G + G * D);   // m[G], l[G], acc[G][D]
    if (g == 0) {
      if (h0 < G) { cm[h0] = m0; cm[G + h0] = l0; }
      if (h1 < G) { cm[h1] = m1; cm[G + h1] = l1; }
    }
#pragma unroll
    for (int dt = 0; dt < C::DTILES; ++dt) {
      const int d0 = dt * 16 + g;
      if (h0 < G) {
        cm[2 * G + h0 * D + d0] = o[dt][0];
        cm[2 * G + h0 * D + d0 + 8] = o[dt][2];
      }
      if (h1 < G) {
        cm[2 * G + h1 * D + d0] = o[dt][1];
        cm[2 * G + h1 * D + d0 + 8] = o[dt][3];
      }
    }
    named_bar_sync(1, C::CONS_WARPS * 32);

    const int cfirst = per_slot ? 0 : cta_of(P[s]), clast = per_slot ? 0 : cta_of(P[s + 1] - 1);
    const bool single = cfirst == clast;
    float* mypart = a.partial + (size_t)(c + s) * G * (D + 2);
    for (int e = tid; e < G * D; e += C::CONS_WARPS * 32) {
      const int h = e / D;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < C::CONS_WARPS; ++w) M = fmaxf(M, comb[w * (2 * G + G * D) + h]);
      float Lt = 0.f, A = 0.f;
#pragma unroll
      for (int w = 0; w < C::CONS_WARPS; ++w) {
        const float* cmw = comb + w * (2 * G + G * D);
        const float mw = cmw[h];
        if (mw == -INFINITY) continue;
        const float sc = exp2f(mw - M);
        Lt += cmw[G + h] * sc;
        A += cmw[2 * G + e] * sc;
      }
      if (per_slot) {
        cres[e] = A;
        if (e % D == 0) {
          cres[G * D + h] = M;
          cres[G * D + G + h] = Lt;
        }
      } else if (single) {
        a.out[(size_t)s * G * D + e] = Lt > 0.f ? A / Lt : 0.f;
      } else {
        mypart[e] = A;
        if (e % D == 0) {
          mypart[G * D + h] = M;
          mypart[G * D + G + h] = Lt;
        }
      }
    }
    if (!per_slot && !single) {
      // the CTA's partial writes, then one fenced ticket (the barrier + one-thread fence
      // orders every thread's writes before the atomic)
      named_bar_sync(1, C::CONS_WARPS * 32);
      if (tid == 0) last_flag = slot_ticket(&a.counters[s], clast - cfirst);
      named_bar_sync(1, C::CONS_WARPS * 32);
      if (last_flag) {
        merge_partials(a, s, G, D, cfirst, clast, tid, C::CONS_WARPS * 32);
        if (tid == 0) a.counters[s] = 0;
      }
    }
    named_bar_sync(1, C::CONS_WARPS * 32);
    t = seg_end;
  }
  }

  if (per_slot) {
    // every CTA of the slot's cluster has its partial in cres; rank 0 merges them
    cluster_sync_all();
    const int k = ksz, sl = my_cluster;
    if (cluster_rank() == 0 && sl < S) {
      for (int e = tid; e < G * D; e += blockDim.x) {
        const int h = e / D;
        float M = -INFINITY;
        for (int r = 0; r < k; ++r) M = fmaxf(M, ld_dsmem(cres + G * D + h, r));
        float Lt = 0.f, A = 0.f;
        if (M != -INFINITY)
          for (int r = 0; r < k; ++r) {
            const float m = ld_dsmem(cres + G * D + h, r);
            if (m == -INFINITY) continue;
            const float sc = exp2f(m - M);
            Lt += ld_dsmem(cres + G * D + G + h, r) * sc;
            A += ld_dsmem(cres + e, r) * sc;
          }
        a.out[(size_t)sl * G * D + e] = Lt > 0.f ? A / Lt : 0.f;
      }
    }
    cluster_sync_all();   // keep every CTA's shared memory alive until rank 0 has read it
  }
}

}  // namespace kvc
