// The packed per-head cache: layout (offsets by an exclusive scan of the
// capacities), compaction (128-bit gathers of the kept K and V rows), the
// per-step append, the gather of chunk keys, and the ZigZagKV per-layer budget
// allocation (Eq. 4-6) that decides how many rows each layer keeps.
#pragma once
#include "common.cuh"

namespace kvc {

// ---------------------------------------------------------------- layout
// One CTA: cap[s] = round_up(count[s] + reserve, 16); off = exclusive scan (int64).
__global__ void __launch_bounds__(1024) layout_kernel(const int32_t* __restrict__ count, int S, int reserve,
                                                      int64_t* __restrict__ off, int32_t* __restrict__ cap) {
  __shared__ unsigned long long sh[33];
  unsigned long long carry = 0;
  for (int base = 0; base < S; base += blockDim.x) {
    const int s = base + threadIdx.x;
    unsigned long long c = 0;
    if (s < S) {
      long long want = (long long)max(count[s], 0) + reserve;
      c = (unsigned long long)((want + 15) / 16 * 16);
      cap[s] = (int32_t)c;
    }
    unsigned long long tot;
    unsigned long long before = carry + block_exclusive_scan<unsigned long long>(c, sh, &tot);
    if (s < S) off[s] = (int64_t)before;
    carry += tot;
  }
  if (threadIdx.x == 0) off[S] = (int64_t)carry;
}

// ---------------------------------------------------------------- compaction
// Persistent grid; CTA c owns the contiguous packed rows [c*R/grid, (c+1)*R/grid) of the
// R = off[S] rows, so consecutive rows mostly share a slot: each row group finds the
// slot of its first row by binary search once and then walks forward. A group of
// TPR = row_bytes / 16 threads moves one K row and one V row with 16-byte accesses;
// each group keeps UNROLL rows in flight.
template <int TPR, int UNROLL>
__global__ void __launch_bounds__(256, 4) compact_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                                      const int32_t* __restrict__ idx, int max_sel,
                                                      const int32_t* __restrict__ count,
                                                      const int64_t* __restrict__ off, int S, int L,
                                                      uint4* __restrict__ kp, uint4* __restrict__ vp,
                                                      int64_t kp_rows, int32_t* __restrict__ len) {
  const long long gtid = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (gtid < S) len[gtid] = min(max(count[gtid], 0), max_sel);
  constexpr int GROUPS = 256 / TPR;                 // row groups per CTA
  const int part = threadIdx.x % TPR, grp = threadIdx.x / TPR;
  const long long total = off[S];
  const long long r0 = total * blockIdx.x / gridDim.x, r1 = total * (blockIdx.x + 1) / gridDim.x;
  if (r0 >= r1) return;
  // slot of row r0: last s with off[s] <= r0
  int s = 0;
  {
    int lo = 0, hi = S - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (off[mid] <= r0) lo = mid; else hi = mid - 1;
    }
    s = lo;
  }
  long long s_end = off[s + 1];
  for (long long g0 = r0 + grp; g0 < r1; g0 += (long long)GROUPS * UNROLL) {
    uint4 kr[UNROLL], vr[UNROLL];
    long long dst[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      dst[u] = -1;
      const long long g = g0 + (long long)u * GROUPS;
      if (g >= r1) continue;
      while (g >= s_end && s < S - 1) {          // rows only increase: walk the slots forward
        ++s;
        s_end = off[s + 1];
      }
      const long long r = g - off[s];
      const int cnt = min(count[s], max_sel);
      if (r >= cnt) continue;                      // capacity padding: not written
      const int j = idx[(size_t)s * max_sel + r];
      if (j < 0 || j >= L || g >= kp_rows) {
        kvc_flag(KVC_DEVERR_INDEX_RANGE);
        continue;
      }
      const size_t src = ((size_t)s * L + j) * TPR + part;
      kr[u] = __ldg(k + src);
      vr[u] = __ldg(v + src);
      dst[u] = g * TPR + part;
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u)
      if (dst[u] >= 0) {
        kp[dst[u]] = kr[u];
        vp[dst[u]] = vr[u];
      }
  }
}

// ---------------------------------------------------------------- compaction, one wave
// One CTA per (SM x 4), each owning the contiguous packed rows [r0, r1). Its dependent
// round trips to memory are few and fixed: warp 0 finds the slots of r0 and r1 - 1 with
// two 32-wide probes of off[]; the CTA stages those slots' offsets and counts in shared
// memory (up to CP_MAX_SLOTS, else a chunk-local binary search in global memory); then,
// 256 rows at a time, every thread resolves one row's source (one coalesced idx load)
// and the CTA copies the chunk's K and V rows with 16-byte accesses, CP_UNROLL rows in
// flight per row group.
constexpr int CP_THREADS = 256;
constexpr int CP_MAX_SLOTS = 512;
constexpr int CP_UNROLL = 4;

// last s in [0, S) with off[s] <= x, by two rounds of 32 probes (one warp)
KVC_DEV int warp_slot_search(const int64_t* __restrict__ off, int S, long long x) {
  const int lane = threadIdx.x & 31;
  int lo = 0, n = S;
  while (n > 1) {
    const int step = (n + 31) / 32;
    const int i = lo + lane * step;
    const bool le = i < lo + n && off[i] <= x;
    const unsigned m = __ballot_sync(0xffffffffu, le);
    const int best = m ? 31 - __clz(m) : 0;
    lo = lo + best * step;
    n = min(step, S - lo);
  }
  return lo;
}

//
// LAYOUT (S <= CP_MAX_SLOTS): the layout is computed here as well, in one launch: every CTA
// scans the capacities round_up(count + reserve, 16) into shared memory itself, and CTA 0
// also writes them out (off_out, cap_out), so the copy no longer waits for a layout kernel.
template <int TPR, bool LAYOUT>
__global__ void __launch_bounds__(CP_THREADS, 4) compact_wave_kernel(
    const uint4* __restrict__ k, const uint4* __restrict__ v, const int32_t* __restrict__ idx, int max_sel,
    const int32_t* __restrict__ count, const int64_t* __restrict__ off, int S, int L, uint4* __restrict__ kp,
    uint4* __restrict__ vp, int64_t kp_rows, int32_t* __restrict__ len, int reserve, int64_t* __restrict__ off_out,
    int32_t* __restrict__ cap_out) {
  __shared__ long long s_off[CP_MAX_SLOTS + 1];
  __shared__ int s_cnt[CP_MAX_SLOTS];
  __shared__ long long src_row[CP_THREADS];   // source row s * L + j, or -1: not written
  __shared__ int s_first_sh, s_last_sh;
  __shared__ unsigned long long scan_sh[32];
  const int tid = threadIdx.x;
  for (long long s = (long long)blockIdx.x * blockDim.x + tid; s < S; s += (long long)gridDim.x * blockDim.x)
    len[s] = min(max(count[s], 0), max_sel);
  long long total;
  int s_first, ns;
  bool staged;
  if (LAYOUT) {
    // the same arithmetic as layout_kernel, over all S slots
    const bool writer = blockIdx.x == 0;
    unsigned long long carry = 0;
    for (int base = 0; base < S; base += CP_THREADS) {
      const int s = base + tid;
      unsigned long long c = 0;
      if (s < S) {
        const int cs = count[s];
        c = (unsigned long long)(((long long)max(cs, 0) + reserve + 15) / 16 * 16);
        s_cnt[s] = min(cs, max_sel);
        if (writer) cap_out[s] = (int32_t)c;
      }
      unsigned long long tot;
      const unsigned long long before = carry + block_exclusive_scan<unsigned long long>(c, scan_sh, &tot);
      if (s < S) {
        s_off[s] = (long long)before;
        if (writer) off_out[s] = (int64_t)before;
      }
      carry += tot;
    }
    if (tid == 0) {
      s_off[S] = (long long)carry;
      if (writer) off_out[S] = (int64_t)carry;
    }
    __syncthreads();
    total = s_off[S];
    s_first = 0;
    ns = S;
    staged = true;
  } else {
    total = off[S];
  }
  const long long r0 = total * blockIdx.x / gridDim.x, r1 = total * (blockIdx.x + 1) / gridDim.x;
  if (r0 >= r1) return;
  if (!LAYOUT) {
    if (tid < 32) {
      const int a = warp_slot_search(off, S, r0);
      const int b = warp_slot_search(off, S, r1 - 1);
      if (tid == 0) { s_first_sh = a; s_last_sh = b; }
    }
    __syncthreads();
    s_first = s_first_sh;
    ns = s_last_sh - s_first_sh + 1;
    staged = ns <= CP_MAX_SLOTS;
    if (staged) {
      for (int i = tid; i <= ns; i += blockDim.x) s_off[i] = off[s_first + i];
      for (int i = tid; i < ns; i += blockDim.x) s_cnt[i] = min(count[s_first + i], max_sel);
    }
    __syncthreads();
  }
  constexpr int GROUPS = CP_THREADS / TPR;
  const int part = tid % TPR, grp = tid / TPR;
  for (long long base = r0; base < r1; base += CP_THREADS) {
    // resolve one row per thread
    const long long g = base + tid;
    long long src = -1;
    if (g < r1) {
      int lo, hi;
      if (staged) { lo = 0; hi = ns - 1; } else { lo = s_first; hi = s_first + ns - 1; }
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        const long long om = staged ? s_off[mid] : off[mid];
        if (om <= g) lo = mid; else hi = mid - 1;
      }
      const int s = staged ? s_first + lo : lo;
      const long long r = g - (staged ? s_off[lo] : off[s]);
      const int cnt = staged ? s_cnt[lo] : min(count[s], max_sel);
      if (r < cnt) {
        const int j = idx[(size_t)s * max_sel + r];
        if (j < 0 || j >= L || g >= kp_rows) kvc_flag(KVC_DEVERR_INDEX_RANGE);
        else src = (long long)s * L + j;
      }
    }
    src_row[tid] = src;
    __syncthreads();
    const int nrows = (int)min((long long)CP_THREADS, r1 - base);
    for (int i0 = grp; i0 < nrows; i0 += GROUPS * CP_UNROLL) {
      uint4 kr[CP_UNROLL], vr[CP_UNROLL];
      long long dst[CP_UNROLL];
#pragma unroll
      for (int u = 0; u < CP_UNROLL; ++u) {
        const int i = i0 + u * GROUPS;
        dst[u] = -1;
        if (i < nrows) {
          const long long sr = src_row[i];
          if (sr >= 0) {
            kr[u] = __ldg(k + (size_t)sr * TPR + part);
            vr[u] = __ldg(v + (size_t)sr * TPR + part);
            dst[u] = (base + i) * TPR + part;
          }
        }
      }
#pragma unroll
      for (int u = 0; u < CP_UNROLL; ++u)
        if (dst[u] >= 0) {
          kp[dst[u]] = kr[u];
          vp[dst[u]] = vr[u];
        }
    }
    __syncthreads();   // src_row is reused by the next chunk
  }
}

// ---------------------------------------------------------------- append
// grid S, block TPR: row off[s] + len[s] <- the new token; len[s] += 1.
__global__ void append_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                              const int64_t* __restrict__ off, const int32_t* __restrict__ cap,
                              int32_t* __restrict__ len, uint4* __restrict__ kp, uint4* __restrict__ vp,
                              int64_t kp_rows, int tpr) {
  const int s = blockIdx.x;
  const int n = len[s];
  const bool ok = n >= 0 && n < cap[s] && off[s] + n < kp_rows;
  if (ok) {
    const size_t dst = ((size_t)off[s] + n) * tpr + threadIdx.x;
    kp[dst] = k_new[(size_t)s * tpr + threadIdx.x];
    vp[dst] = v_new[(size_t)s * tpr + threadIdx.x];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (ok) len[s] = n + 1;
    else kvc_flag(KVC_DEVERR_APPEND_OVERFLOW);
  }
}

// ---------------------------------------------------------------- append with a sliding window
// grid S, block TPR. A slot with window[s] > 0 that already holds window[s] rows keeps
// holding them: the new token overwrites row head[s] (the oldest) and head[s] advances
// cyclically. Any other slot appends as append_kernel. Attention over a slot's rows does
// not depend on their order, so the window's rows can stay a ring.
__global__ void append_window_kernel(const uint4* __restrict__ k_new, const uint4* __restrict__ v_new,
                                     const int64_t* __restrict__ off, const int32_t* __restrict__ cap,
                                     int32_t* __restrict__ len, const int32_t* __restrict__ window,
                                     int32_t* __restrict__ head, uint4* __restrict__ kp, uint4* __restrict__ vp,
                                     int64_t kp_rows, int tpr) {
  const int s = blockIdx.x;
  const int n = len[s], w = window[s];
  const bool ring = w > 0 && n >= w;
  const int h = ring ? head[s] : 0;
  const int row = ring ? h : n;
  const bool ok = n >= 0 && row >= 0 && row < cap[s] && (!ring || h < w) && off[s] + row < kp_rows;
  if (ok) {
    const size_t dst = ((size_t)off[s] + row) * tpr + threadIdx.x;
    kp[dst] = k_new[(size_t)s * tpr + threadIdx.x];
    vp[dst] = v_new[(size_t)s * tpr + threadIdx.x];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (!ok) kvc_flag(KVC_DEVERR_APPEND_OVERFLOW);
    else if (ring) head[s] = h + 1 == w ? 0 : h + 1;
    else len[s] = n + 1;
  }
}

// ---------------------------------------------------------------- chunk keys
// kc[s][c] = k[s][chunk_end[c]] (ChunkLLM Eq. 3: a chunk is keyed by its last token).
__global__ void gather_rows_kernel(const uint4* __restrict__ k, const int32_t* __restrict__ rows, int C, int L,
                                   int S, int tpr, uint4* __restrict__ out) {
  const long long total = (long long)S * C * tpr;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < total;
       e += (long long)gridDim.x * blockDim.x) {
    const long long row = e / tpr;
    const int part = (int)(e - row * tpr);
    const int s = (int)(row / C), c = (int)(row - (long long)s * C);
    const int j = rows[c];
    if (j < 0 || j >= L) { kvc_flag(KVC_DEVERR_INDEX_RANGE); continue; }
    out[e] = k[((size_t)s * L + j) * tpr + part];
  }
}

// ---------------------------------------------------------------- ZigZagKV allocation
// One CTA of 1024 threads; n_layers <= 1024. Exact integer arithmetic.
__global__ void __launch_bounds__(1024) alloc_kernel(const int32_t* __restrict__ counts, int nL, int spl, int L,
                                                     int avg_B, int floor_B, int32_t* __restrict__ budgets,
                                                     int32_t* __restrict__ slot_budgets) {
  __shared__ long long Cl[1024];
  __shared__ unsigned char capped[1024];
  __shared__ long long rem[1024];
  __shared__ long long base_[1024];
  __shared__ unsigned long long red[33];
  __shared__ int any_new;
  const int tid = threadIdx.x;
  for (int l = tid; l < nL; l += blockDim.x) {
    long long c = 0;
    for (int i = 0; i < spl; ++i) c += max(counts[(size_t)l * spl + i], 0);
    Cl[l] = c;
    capped[l] = 0;
  }
  __syncthreads();
  const long long T = (long long)nL * avg_B;
  const long long f = min(floor_B, L);
  long long R = 0, E = 0, den = 0;
  bool uniform = false;
  int nU = 0;
  while (true) {
    // sums over the uncapped layers
    unsigned long long my_c = 0, my_u = 0;
    for (int l = tid; l < nL; l += blockDim.x)
      if (!capped[l]) { my_c += (unsigned long long)Cl[l]; my_u += 1; }
    const unsigned long long sumC = block_sum<unsigned long long>(my_c, red);
    nU = (int)block_sum<unsigned long long>(my_u, red);
    if (nU == 0) break;
    R = T - (long long)(nL - nU) * L;
    E = R - (long long)nU * f;
    uniform = sumC == 0;
    den = uniform ? nU : (long long)sumC;
    if (tid == 0) any_new = 0;
    __syncthreads();
    for (int l = tid; l < nL; l += blockDim.x) {
      if (capped[l]) continue;
      const __int128 wl = uniform ? 1 : Cl[l];
      // ideal = f + E * wl / den > L  <=>  f*den + E*wl > L*den
      if ((__int128)f * den + (__int128)E * wl > (__int128)L * den) { capped[l] = 2; any_new = 1; }
    }
    __syncthreads();
    const int again = any_new;
    for (int l = tid; l < nL; l += blockDim.x)
      if (capped[l] == 2) capped[l] = 1;
    __syncthreads();
    if (!again) break;
  }
  // floor + largest remainder over the uncapped layers (ties: lower layer)
  unsigned long long my_b = 0;
  for (int l = tid; l < nL; l += blockDim.x) {
    if (capped[l]) continue;
    const __int128 wl = uniform ? 1 : Cl[l];
    const __int128 num = (__int128)f * den + (__int128)E * wl;
    base_[l] = (long long)(num / den);
    rem[l] = (long long)(num % den);
    my_b += (unsigned long long)base_[l];
  }
  const long long sum_base = nU > 0 ? (long long)block_sum<unsigned long long>(my_b, red) : 0;
  const long long left = R - sum_base;
  for (int l = tid; l < nL; l += blockDim.x) {
    long long b;
    if (capped[l]) {
      b = L;
    } else {
      long long rank = 0;
      for (int m = 0; m < nL; ++m)
        if (!capped[m] && (rem[m] > rem[l] || (rem[m] == rem[l] && m < l))) ++rank;
      b = base_[l] + (rank < left ? 1 : 0);
    }
    budgets[l] = (int32_t)b;
    if (slot_budgets)
      for (int i = 0; i < spl; ++i) slot_budgets[(size_t)l * spl + i] = (int32_t)b;
  }
}

}  // namespace kvc
