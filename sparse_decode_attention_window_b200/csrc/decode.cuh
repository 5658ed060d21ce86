// Split-K GQA decode attention over the ragged packed cache.
//
// For query head h of slot s = h / G:
//   out[h] = sum_{r < len[s]} softmax_r(q_h . K[off_s + r] / sqrt(d)) V[off_s + r].
//
// Work split: the valid tokens of all slots, taken in slot order, are cut into
// gridDim.x equal ranges, one per CTA (persistent, one CTA per SM); a range may
// cross slot boundaries, so every CTA streams the same number of bytes whatever
// the mix of lengths. A CTA emits one (max, sum, unnormalised output) partial per
// slot segment it touched; a slot covered by one CTA is written directly,
// otherwise the last CTA to finish the slot (atomic ticket, no waiting) merges
// the partials. Partial (c, s) lives at index c + s, which is unique because the
// (CTA, slot) pairs form a monotone staircase.
//
// Inside a CTA: warp 4 is the producer - one lane issues plain bulk copies
// (cp.async.bulk) of 64-token K and V tiles into a ring of shared-memory stages
// guarded by mbarriers; warps 0-3 consume. The work is HBM-bound (G = 4 flop per
// byte), so the dot products run on the CUDA cores: 8 lanes share a token row
// (each owns d/8 contiguous elements, read as 16-byte chunks in a lane-rotated
// order so the 8 lanes of a row hit 8 distinct bank groups), the G per-head
// partial sums are reduced across the 8 lanes by a transposing butterfly that
// leaves each lane holding one head's logit, and the online softmax runs per
// 16-token warp tile in the exp2 domain.
#pragma once
#include "common.cuh"

namespace kvc {

template <typename T, int D, int G>
struct DecCfg {
  static constexpr int ES = sizeof(T);
  static constexpr int ROWB = D * ES;             // bytes per cache row
  static constexpr int EPL = D / 8;               // elements per lane (8 lanes per row)
  static constexpr int CE = 16 / ES;              // elements per 16-byte chunk
  static constexpr int NCH = EPL / CE;            // chunks per lane: 1, 2 or 4
  static constexpr int TILE = 64;                 // tokens per stage
  static constexpr int STAGE_BYTES = 2 * TILE * ROWB;
  static constexpr int STAGES = STAGE_BYTES <= 32768 ? 4 : 3;
  static constexpr int LG = G == 1 ? 0 : G == 2 ? 1 : G == 4 ? 2 : 3;
  static constexpr int CONS_WARPS = 4;
  static constexpr int THREADS = (CONS_WARPS + 1) * 32;
  static constexpr int REDUND = 8 >> LG;          // lanes holding the same (token, head) logit
  static_assert(G == 1 || G == 2 || G == 4, "decode supports G in {1, 2, 4}");
  static_assert(NCH >= 1 && NCH <= 4, "row part must be 1..4 chunks");
};

constexpr int DEC_MAX_SLOTS = 4096;

template <typename T, int D, int G>
constexpr size_t decode_smem_bytes(int S, int grid) {
  using C = DecCfg<T, D, G>;
  return (size_t)C::STAGES * C::STAGE_BYTES + 2 * C::STAGES * sizeof(uint64_t) + (size_t)(S + 1) * sizeof(long long) +
         (size_t)C::CONS_WARPS * (2 * G + G * D) * sizeof(float) + (size_t)2 * grid * G * sizeof(float) + 16;
}

template <int G>
KVC_DEV float pick(const float (&a)[G], int i) {
  float r = a[0];
#pragma unroll
  for (int h = 1; h < G; ++h) r = (i == h) ? a[h] : r;
  return r;
}

// Sum of the G per-head values over the 8 lanes of a row; afterwards the lane
// holds head (p >> (3 - LG)) & (G - 1).
template <int G>
KVC_DEV float row_reduce(float (&v)[G], int p) {
  int n = G;
#pragma unroll
  for (int mask = 4; mask >= 1; mask >>= 1) {
    if (n > 1) {
      const bool upper = (p & mask) != 0;
      const int half = n / 2;
#pragma unroll
      for (int i = 0; i < G / 2; ++i) {
        if (i < half) {
          const float keep = upper ? v[half + i] : v[i];
          const float send = upper ? v[i] : v[half + i];
          v[i] = keep + __shfl_xor_sync(0xffffffffu, send, mask);
        }
      }
      n = half;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], mask);
    }
  }
  return v[0];
}

template <typename T, int D, int G>
KVC_DEV void load_part(const unsigned char* row, int p, int rot, float (&f)[D / 8]) {
  using C = DecCfg<T, D, G>;
  const uint4* base = reinterpret_cast<const uint4*>(row + p * C::EPL * C::ES);
#pragma unroll
  for (int c = 0; c < C::NCH; ++c) {
    const int cc = (c + rot) & (C::NCH - 1);
    const uint4 u = base[cc];
    Chunk16<T>::unpack(u, &f[c * C::CE]);
  }
}

// Floats per (CTA, slot) partial: G*D unnormalised outputs, G maxima, G sums, padded
// to a multiple of 4 floats so every partial starts 16-byte aligned.
KVC_HD constexpr int partial_stride(int G, int D) { return (G * (D + 2) + 3) & ~3; }

struct DecodeParams {
  const void* q;
  const void* kp;
  const void* vp;
  const int64_t* off;
  const int32_t* len;
  long long kp_rows;
  int S;
  float scale_log2;
  float* out;
  float* partial;   // [(gridDim.x + S) * partial_stride(G, D)]
  int* counters;    // [S + 1], zero on entry and on exit ([S]: grid-wide ticket of the fused append)
  // fused append (tensor-core kernel only): the new token of slot s is k_new[s], v_new[s]
  int append;
  const void* k_new;
  const void* v_new;
  const int32_t* cap;
  int32_t* len_out;  // = len; incremented by the last CTA to finish
  // optional (fused append, tensor-core kernel): rows [0, stable[s]) of slot s are written
  // neither by the previous kernel on the stream nor by this launch, and off, cap, stable
  // are not written by the previous kernel either; the launch may then plan and load those
  // rows before the previous kernel has finished
  const int32_t* stable;
};

// The last CTA to finish slot s merges the slot's partials (CTAs cfirst..clast, stored
// consecutively at index c + s) in one online pass: each thread owns output elements
// e and folds the partials in groups of 8 whose (max, sum, value) loads are issued
// together, so a merge of up to 8 partials costs one round trip to L2.
KVC_DEV void merge_partials(const DecodeParams& a, int s, int G, int D, int cfirst, int clast, int tid, int nthr) {
  const int np = clast - cfirst + 1;
  const size_t stride = (size_t)partial_stride(G, D);
  const float* base = a.partial + (size_t)(cfirst + s) * stride;
  for (int e = tid; e < G * D; e += nthr) {
    const int h = e / D;
    float M = -INFINITY, Lt = 0.f, A = 0.f;
    for (int i0 = 0; i0 < np; i0 += 8) {
      float m[8], l[8], v[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const bool in = i0 + k < np;
        const float* pp = base + (size_t)(i0 + k) * stride;
        m[k] = in ? __ldcg(pp + (size_t)G * D + h) : -INFINITY;
        l[k] = in ? __ldcg(pp + (size_t)G * D + G + h) : 0.f;
        v[k] = in ? __ldcg(pp + e) : 0.f;
      }
      float Mn = M;
#pragma unroll
      for (int k = 0; k < 8; ++k) Mn = fmaxf(Mn, m[k]);
      if (Mn == -INFINITY) continue;
      const float sc = M == -INFINITY ? 0.f : exp2f(M - Mn);
      Lt *= sc;
      A *= sc;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float w = m[k] == -INFINITY ? 0.f : exp2f(m[k] - Mn);
        Lt += l[k] * w;
        A += v[k] * w;
      }
      M = Mn;
    }
    a.out[(size_t)s * G * D + e] = Lt > 0.f ? A / Lt : 0.f;
  }
}

// Ticket of slot s: returns true in the CTA that finishes the slot last. Called by one
// thread after a CTA barrier that follows the CTA's partial writes; the acq_rel atomic
// publishes them (release is cumulative over the barrier) and, in the last CTA, makes
// the other CTAs' partials visible (acquire).
KVC_DEV bool slot_ticket(int* counter, int last_value) {
  int old;
  asm volatile("atom.acq_rel.gpu.global.add.s32 %0, [%1], 1;" : "=r"(old) : "l"(counter), "r"(1) : "memory");
  return old == last_value;
}

template <typename T, int D, int G>
__global__ void __launch_bounds__(DecCfg<T, D, G>::THREADS, 1) decode_kernel(DecodeParams a) {
  using C = DecCfg<T, D, G>;
  extern __shared__ __align__(128) unsigned char dsm[];
  unsigned char* stages = dsm;
  uint64_t* full = reinterpret_cast<uint64_t*>(dsm + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  long long* P = reinterpret_cast<long long*>(empty + C::STAGES);
  float* comb = reinterpret_cast<float*>(P + a.S + 1);   // [warps][2G + G*D]
  __shared__ unsigned long long scan_sh[33];
  __shared__ int last_flag;
  __shared__ int abort_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = a.S;
  const T* q = static_cast<const T*>(a.q);
  const T* kp = static_cast<const T*>(a.kp);
  const T* vp = static_cast<const T*>(a.vp);

  // prefix of the valid lengths over slots
  unsigned long long carry = 0;
  for (int base = 0; base < S; base += blockDim.x) {
    const int s = base + tid;
    unsigned long long x = 0;
    if (s < S) {
      long long n = max(a.len[s], 0);
      const long long room = a.kp_rows - a.off[s];        // rows of the buffer from the slot's start
      if (n > room) { kvc_flag(KVC_DEVERR_INDEX_RANGE); n = room > 0 ? room : 0; }
      x = (unsigned long long)n;
    }
    unsigned long long tot;
    const unsigned long long before = carry + block_exclusive_scan<unsigned long long>(x, scan_sh, &tot);
    if (s < S) P[s] = (long long)before;
    carry += tot;
  }
  if (tid == 0) {
    P[S] = (long long)carry;
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], C::CONS_WARPS);
    }
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  const long long N = P[S];
  const int nC = gridDim.x, c = blockIdx.x;
  // empty slots: zero output rows (split over CTAs)
  for (int s = c; s < S; s += nC)
    if (P[s + 1] == P[s])
      for (int e = tid; e < G * D; e += blockDim.x) a.out[(size_t)s * G * D + e] = 0.f;
  if (N == 0) return;
  // nE <= N CTAs take part, so every range is non-empty and the per-slot ticket
  // count (CTAs whose range meets the slot) is exact
  const int nE = (int)min((long long)nC, N);
  if (c >= nE) return;
  const long long b0 = (long long)c * N / nE, b1 = (long long)(c + 1) * N / nE;

  auto slot_of = [&](long long t) {          // the non-empty slot holding valid token t
    int lo = 0, hi = S - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (P[mid] <= t) lo = mid; else hi = mid - 1;
    }
    return lo;
  };
  auto cta_of = [&](long long t) { return (int)(((t + 1) * nE - 1) / N); };

  if (warp == C::CONS_WARPS) {
    // ---------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      for (long long t = b0; t < b1 && ok;) {
        const int s = slot_of(t);
        const long long seg_end = min(b1, P[s + 1]);
        for (long long u = t; u < seg_end; u += C::TILE) {
          const int rows = (int)min((long long)C::TILE, seg_end - u);
          if (!mbar_wait(&empty[stage], ph ^ 1)) { ok = false; break; }
          if (*(volatile int*)&abort_flag) { ok = false; break; }
          const uint32_t bytes = (uint32_t)rows * C::ROWB;
          mbar_arrive_expect_tx(&full[stage], 2 * bytes);
          const long long row0 = a.off[s] + (u - P[s]);
          unsigned char* dst = stages + stage * C::STAGE_BYTES;
          bulk_g2s(dst, kp + row0 * D, bytes, &full[stage]);
          bulk_g2s(dst + C::TILE * C::ROWB, vp + row0 * D, bytes, &full[stage]);
          ++issued;
          if (++stage == C::STAGES) { stage = 0; ph ^= 1; }
        }
        t = seg_end;
      }
      if (!ok) {
        // unwind: wait (bounded) for the copies still in flight into our stages
        const long long n = min(issued, (long long)C::STAGES);
        for (long long i = 1; i <= n; ++i) {
          const long long k = issued - i;
          mbar_wait(&full[k % C::STAGES], (uint32_t)((k / C::STAGES) & 1));
        }
      }
    }
    return;
  }

  // ---------------- consumers (warps 0..3)
  const int cw = warp, t_in = lane >> 3, p = lane & 7;
  const int rot = (p * C::NCH / 8) & (C::NCH - 1);
  const int hh = (p >> (3 - C::LG)) & (G - 1);           // head this lane's reduced logit belongs to
  const bool canon = (p & (C::REDUND - 1)) == 0;           // one lane per (token, head) counts the sum
  int stage = 0;
  uint32_t ph = 0;
  for (long long t = b0; t < b1;) {
    const int s = slot_of(t);
    const long long seg_end = min(b1, P[s + 1]);

    float qf[G][C::EPL];
#pragma unroll
    for (int h = 0; h < G; ++h)
      load_part<T, D, G>(reinterpret_cast<const unsigned char*>(q + ((size_t)s * G + h) * D), p, rot, qf[h]);
    float m_all[G], acc[G][C::EPL];
    float lown = 0.f;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      m_all[h] = -INFINITY;
#pragma unroll
      for (int e = 0; e < C::EPL; ++e) acc[h][e] = 0.f;
    }

    for (long long u = t; u < seg_end; u += C::TILE) {
      const int rows = (int)min((long long)C::TILE, seg_end - u);
      if (!mbar_wait(&full[stage], ph)) { *(volatile int*)&abort_flag = 1; return; }
      const unsigned char* Ks = stages + stage * C::STAGE_BYTES;
      const unsigned char* Vs = Ks + C::TILE * C::ROWB;
      float z[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int tk = cw * 16 + g * 4 + t_in;
        float kf[C::EPL];
        load_part<T, D, G>(Ks + tk * C::ROWB, p, rot, kf);
        float v[G];
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float s0 = 0.f;
#pragma unroll
          for (int e = 0; e < C::EPL; ++e) s0 = fmaf(qf[h][e], kf[e], s0);
          v[h] = s0;
        }
        const float zz = row_reduce<G>(v, p);
        z[g] = tk < rows ? zz * a.scale_log2 : -INFINITY;
      }
      // running max per head over this warp's tokens
      float mx = fmaxf(fmaxf(z[0], z[1]), fmaxf(z[2], z[3]));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 8));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
      float alpha[G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float tm = __shfl_sync(0xffffffffu, mx, h << (3 - C::LG));
        const float mn = fmaxf(m_all[h], tm);
        alpha[h] = (mn == -INFINITY) ? 1.f : exp2f(m_all[h] - mn);
        m_all[h] = mn;
      }
      lown *= pick<G>(alpha, hh);
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < C::EPL; ++e) acc[h][e] *= alpha[h];
      const float mh = pick<G>(m_all, hh);
      float pr[4];
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        pr[g] = (z[g] == -INFINITY) ? 0.f : exp2f(z[g] - mh);
        if (canon) lown += pr[g];
      }
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int tk = cw * 16 + g * 4 + t_in;
        float vf[C::EPL];
        load_part<T, D, G>(Vs + tk * C::ROWB, p, rot, vf);
        float pw[G];
#pragma unroll
        for (int h = 0; h < G; ++h) pw[h] = __shfl_sync(0xffffffffu, pr[g], (t_in << 3) | (h << (3 - C::LG)));
        if (tk < rows) {
#pragma unroll
          for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < C::EPL; ++e) acc[h][e] = fmaf(pw[h], vf[e], acc[h][e]);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[stage]);
      if (++stage == C::STAGES) { stage = 0; ph ^= 1; }
    }

    // ---- merge the warp's 4 token lanes, then the 4 warps
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
      for (int e = 0; e < C::EPL; ++e) {
        float x = acc[h][e];
        x += __shfl_xor_sync(0xffffffffu, x, 8);
        x += __shfl_xor_sync(0xffffffffu, x, 16);
        acc[h][e] = x;
      }
#pragma unroll
    for (int o = 1; o < C::REDUND; o <<= 1) lown += __shfl_xor_sync(0xffffffffu, lown, o);
    lown += __shfl_xor_sync(0xffffffffu, lown, 8);
    lown += __shfl_xor_sync(0xffffffffu, lown, 16);
    float* cm = comb + cw * (2 * G + G * D);   // m[G], l[G], acc[G][D]
    if (lane == 0)
#pragma unroll
      for (int h = 0; h < G; ++h) cm[h] = m_all[h];
    if (t_in == 0 && (p & (C::REDUND - 1)) == 0) cm[G + hh] = lown;
    if (t_in == 0) {
#pragma unroll
      for (int h = 0; h < G; ++h)
#pragma unroll
        for (int cix = 0; cix < C::NCH; ++cix) {
          const int cc = (cix + rot) & (C::NCH - 1);
#pragma unroll
          for (int i = 0; i < C::CE; ++i) cm[2 * G + h * D + p * C::EPL + cc * C::CE + i] = acc[h][cix * C::CE + i];
        }
    }
    named_bar_sync(1, C::CONS_WARPS * 32);

    const int cfirst = cta_of(P[s]), clast = cta_of(P[s + 1] - 1);
    const bool single = cfirst == clast;
    float* mypart = a.partial + (size_t)(c + s) * partial_stride(G, D);
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
      if (single) {
        a.out[(size_t)s * G * D + e] = Lt > 0.f ? A / Lt : 0.f;
      } else {
        mypart[e] = A;
        if (e % D == 0) {
          mypart[G * D + h] = M;
          mypart[G * D + G + h] = Lt;
        }
      }
    }
    if (!single) {
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
    named_bar_sync(1, C::CONS_WARPS * 32);   // comb is reused by the next segment
    t = seg_end;
  }
}

}  // namespace kvc
