// Per-slot budget selection: one CTA per slot, policy chosen per slot.
//
// TOPB, MASS_COUNT and CHUNK are one algorithm: walk the keys in descending
// score order (ties: ascending index) and stop at the shortest prefix whose
// weight reaches a target -
//   TOPB        weight 1,                 target B          (per-head top-B eviction)
//   MASS_COUNT  weight = score,           target mass * sum (ZigZagKV Eq. 3, LMBA)
//   CHUNK       weight = chunk length,    target token count (ChunkLLM top chunks)
// The prefix is found without sorting, by a 3-digit MSB radix select on the
// order-preserving integer image of the fp32 score (11 + 11 + 10 bits) with a
// per-bin count and weight histogram. Score weights are summed as 64-bit fixed
// point (exact and order-independent); the scale is chosen per slot from the
// slot's largest score so the total cannot overflow.
// Kept indices are emitted in ascending position order by a block scan.
// LOCAL / SPECIAL / FULL (FastGen head policies) need no scores.
#pragma once
#include "common.cuh"

namespace kvc {

constexpr int SEL_THREADS = 1024;
constexpr int SEL_MAX_BINS = 2048;
constexpr int SEL_SMEM_KEYS = 32768;   // keys cached in shared memory up to this many

struct SelectParams {
  const float* score;
  const int8_t* policy;
  const int32_t* budget;
  float mass;
  const uint8_t* special_mask;
  const int32_t* chunk_end;
  int C;
  int L;
  int n_kv_heads;
  int batch;
  int32_t* idx;
  int max_sel;
  int32_t* count;
  int key_cap;      // keys the shared-memory cache holds (<= SEL_SMEM_KEYS)
  int n_local;      // CHUNK: the last n_local chunks are always kept (ChunkLLM local chunks)
};

KVC_DEV uint32_t order_key(float f) {
  uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
// The score whose order_key is k (the mapping is a bijection on bit patterns).
KVC_DEV float key_score(uint32_t k) { return __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k); }

// floor(max(v, 0) * 2^fx) as an integer, exactly: the fp32 significand shifted by the
// scaled exponent (no floating-point rounding). The scale is chosen from the slot's
// largest score, so every finite weight stays below 2^62 (shift <= 39); larger
// shifts (an infinite score) saturate.
KVC_DEV unsigned long long fixed_weight(float v, int fx) {
  if (!(v > 0.f)) return 0ull;
  const uint32_t b = __float_as_uint(v);
  const int e = (int)(b >> 23);                                     // sign bit is 0
  const unsigned long long m = e ? (unsigned long long)((b & 0x7fffffu) | 0x800000u) : (b & 0x7fffffu);
  const int sh = (e ? e - 150 : -149) + fx;                          // v = m * 2^(sh - fx)
  if (sh >= 0) return sh <= 40 ? m << sh : ~0ull;
  return sh > -64 ? m >> -sh : 0ull;
}

// Adds a 64-bit weight to a bin kept as two 32-bit words, with one shared atomic per
// word: the low word's atomic returns its old value, so the addition that wraps it is
// known and carries one into the high word. Exact for any number of keys (the low word
// wraps as often as the true sum crosses a multiple of 2^32, and each wrap is counted
// once). Per key, so no grouping of a warp's keys by bin is needed.
KVC_DEV void bin_add_u64(uint32_t* lo, uint32_t* hi, unsigned long long w) {
  const uint32_t wl = (uint32_t)w, wh = (uint32_t)(w >> 32);
  const uint32_t old = atomicAdd(lo, wl);
  const uint32_t up = wh + (old + wl < old ? 1u : 0u);
  if (up) atomicAdd(hi, up);
}

struct SelShared {
  uint32_t hcnt[SEL_MAX_BINS];
  uint32_t hwl[SEL_MAX_BINS], hwh[SEL_MAX_BINS];   // bin weights, low and high 32 bits
  unsigned long long scan64[33];
  uint32_t scan32[33];
  // results of the bin search
  uint32_t sel_bin;
  uint32_t cnt_above_bin;
  unsigned long long w_above_bin;
  unsigned long long s_sel;
  int fixed_exp;
};

// Emit positions [lo, lo + n) to idx row (clipped to max_sel).
KVC_DEV void emit_range(int32_t* idx_row, int max_sel, int lo, int n) {
  for (int r = threadIdx.x; r < n; r += blockDim.x)
    if (r < max_sel) idx_row[r] = lo + r;
}

__global__ void __launch_bounds__(SEL_THREADS) select_kernel(SelectParams a) {
  extern __shared__ __align__(16) unsigned char sel_smem_raw[];
  SelShared& sh = *reinterpret_cast<SelShared*>(sel_smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(sel_smem_raw + sizeof(SelShared));

  const int s = blockIdx.x;
  const int pol = a.policy ? a.policy[s] : KVC_POL_CHUNK;   // no policy array: every slot selects chunks
  const int L = a.L;
  int32_t* idx_row = a.idx ? a.idx + (size_t)s * a.max_sel : nullptr;
  const int tid = threadIdx.x;

  if (pol == KVC_POL_LOCAL || pol == KVC_POL_FULL) {
    if (!idx_row) {
      if (tid == 0) { kvc_flag(KVC_DEVERR_INDEX_RANGE); a.count[s] = 0; }
      return;
    }
    int W = pol == KVC_POL_FULL ? L : min(max(a.budget[s], 0), L);
    emit_range(idx_row, a.max_sel, L - W, W);
    if (tid == 0) {
      if (W > a.max_sel) kvc_flag(KVC_DEVERR_INDEX_RANGE);
      a.count[s] = min(W, a.max_sel);
    }
    return;
  }
  if (pol == KVC_POL_SPECIAL) {
    if (!a.special_mask || !idx_row) {
      if (tid == 0) { kvc_flag(KVC_DEVERR_INDEX_RANGE); a.count[s] = 0; }
      return;
    }
    const int b = (s / a.n_kv_heads) % a.batch;
    const uint8_t* m = a.special_mask + (size_t)b * L;
    uint32_t carry = 0;
    for (int base = 0; base < L; base += blockDim.x) {
      int n = base + tid;
      uint32_t f = (n < L && m[n]) ? 1u : 0u, tot;
      uint32_t pos = carry + block_exclusive_scan<uint32_t>(f, sh.scan32, &tot);
      if (f && pos < (uint32_t)a.max_sel) idx_row[pos] = n;
      carry += tot;
    }
    if (tid == 0) {
      if (carry > (uint32_t)a.max_sel) kvc_flag(KVC_DEVERR_INDEX_RANGE);
      a.count[s] = min((int)carry, a.max_sel);
    }
    return;
  }

  // ------------------------------------------------ weighted selection
  const bool chunk = pol == KVC_POL_CHUNK;
  const bool massc = pol == KVC_POL_MASS_COUNT;
  const int N = chunk ? a.C : L;
  const float* sc = a.score + (size_t)s * N;
  const int32_t* ce = a.chunk_end;
  const bool cached = N <= a.key_cap;
  const bool unit = !chunk && !massc;      // top-B: unit weights
  if (!a.score || (chunk && !ce) || (!massc && !idx_row) || (pol != KVC_POL_TOPB && !massc && !chunk)) {
    // a policy whose inputs are missing (or an unknown policy code): keep nothing, report it
    if (tid == 0) { kvc_flag(KVC_DEVERR_INDEX_RANGE); a.count[s] = 0; }
    return;
  }

  // CHUNK with local chunks: the last n_local chunks are kept before any other; giving
  // them the largest key makes the selection take them first. If they alone reach the
  // token target, they are the whole selection.
  const int n_local = chunk ? min(max(a.n_local, 0), N) : 0;
  if (n_local > 0) {
    const int first_local_tok = N - n_local > 0 ? ce[N - n_local - 1] + 1 : 0;
    if ((long long)(L - first_local_tok) >= (long long)a.budget[s]) {
      emit_range(idx_row, a.max_sel, first_local_tok, L - first_local_tok);
      if (tid == 0) {
        if (L - first_local_tok > a.max_sel) kvc_flag(KVC_DEVERR_INDEX_RANGE);
        a.count[s] = min(L - first_local_tok, a.max_sel);
      }
      return;
    }
  }
  auto raw_key = [&](int n) -> uint32_t { return n >= N - n_local ? 0xffffffffu : order_key(sc[n]); };
  // Keys are read four consecutive ones per thread with one 16-byte load where the slot's
  // scores are 16-byte aligned (the passes are bound by the latency of these loads when the
  // keys are not cached in shared memory).
  const bool vec = ((reinterpret_cast<uintptr_t>(sc) & 15u) == 0);
  auto keys4 = [&](int n0, uint32_t* k4) {
    if (cached) {
#pragma unroll
      for (int i = 0; i < 4; ++i) k4[i] = n0 + i < N ? keys[n0 + i] : 0u;
    } else if (vec && n0 + 3 < N && n0 + 3 < N - n_local) {
      const float4 f = __ldg(reinterpret_cast<const float4*>(sc + n0));
      k4[0] = order_key(f.x);
      k4[1] = order_key(f.y);
      k4[2] = order_key(f.z);
      k4[3] = order_key(f.w);
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i) k4[i] = n0 + i < N ? raw_key(n0 + i) : 0u;
    }
  };
  if (cached)
    for (int n = tid; n < N; n += blockDim.x) keys[n] = raw_key(n);
  // weights
  int fx = 0;
  if (massc) {
    float mx = 0.f;
    for (int n0 = tid * 4; n0 < N; n0 += blockDim.x * 4) {
      uint32_t k4[4];
      keys4(n0, k4);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        if (n0 + i < N) mx = fmaxf(mx, key_score(k4[i]));
    }
    mx = warp_max(mx);
    if ((tid & 31) == 0) sh.scan32[tid >> 5] = __float_as_uint(mx);
    __syncthreads();
    if (tid == 0) {
      float m = 0.f;
      for (int i = 0; i < (int)(blockDim.x >> 5); ++i) m = fmaxf(m, __uint_as_float(sh.scan32[i]));
      int ex = 0;
      frexpf(m > 0.f ? m : 1.f, &ex);             // m < 2^ex
      int lg = 32 - __clz(max(N - 1, 1));         // 2^lg >= N
      sh.fixed_exp = 62 - lg - ex;
    }
    __syncthreads();
    fx = sh.fixed_exp;
  }
  auto key_of = [&](int n) -> uint32_t { return cached ? keys[n] : raw_key(n); };
  // the weight of key n (MASS_COUNT: its score, recovered from the key)
  auto weight_of = [&](int n, uint32_t key) -> unsigned long long {
    if (chunk) return (unsigned long long)(ce[n] - (n > 0 ? ce[n - 1] : -1));
    if (massc) return fixed_weight(key_score(key), fx);
    return 1ull;
  };

  // target (MASS_COUNT: from the total weight, which the first radix pass sums)
  unsigned long long target = 0;
  if (!massc) {
    long long want = a.budget[s];
    long long full = chunk ? (long long)L : (long long)N;
    if (want >= full || want <= 0) {
      // keep everything (or nothing)
      int n_out = want <= 0 ? 0 : (int)full;
      emit_range(idx_row, a.max_sel, 0, n_out);
      if (tid == 0) {
        if (n_out > a.max_sel) kvc_flag(KVC_DEVERR_INDEX_RANGE);
        a.count[s] = min(n_out, a.max_sel);
      }
      return;
    }
    target = (unsigned long long)want;
  }

  // radix passes: digits [31:21], [20:10], [9:0]
  uint32_t prefix = 0, pmask = 0, cnt_above = 0;
  unsigned long long w_above = 0;
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nb = pass == 2 ? 1024 : 2048;
    for (int b = tid; b < nb; b += blockDim.x) { sh.hcnt[b] = 0; sh.hwl[b] = 0; sh.hwh[b] = 0; }
    __syncthreads();
    for (int n0 = tid * 4; n0 < N; n0 += blockDim.x * 4) {
      uint32_t k4[4];
      keys4(n0, k4);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int n = n0 + i;
        const uint32_t key = k4[i];
        // one shared atomic per key and word (grouping a warp's keys by bin with match.any
        // costs more when they spread over many bins); top-B: every weight is 1, the count
        // is the weight
        if (n < N && (key & pmask) == prefix) {
          const uint32_t bin = (key >> shift) & (nb - 1);
          atomicAdd(&sh.hcnt[bin], 1u);
          if (!unit) bin_add_u64(&sh.hwl[bin], &sh.hwh[bin], weight_of(n, key));
        }
      }
    }
    __syncthreads();
    // descending walk over the bins: thread t owns bins [nb - (t+1)*per, nb - t*per)
    const int per = (nb + blockDim.x - 1) / blockDim.x;
    const int hi = nb - tid * per;           // exclusive
    const int lo = max(hi - per, 0);
    unsigned long long my_w = 0;
    uint32_t my_c = 0;
    auto bin_w = [&](int b) -> unsigned long long {
      return unit ? (unsigned long long)sh.hcnt[b] : ((unsigned long long)sh.hwh[b] << 32) | sh.hwl[b];
    };
    for (int b = hi - 1; b >= lo; --b) { my_w += bin_w(b); my_c += sh.hcnt[b]; }
    unsigned long long tot_w;
    uint32_t tot_c;
    unsigned long long before_w = block_exclusive_scan<unsigned long long>(hi > lo ? my_w : 0ull, sh.scan64, &tot_w);
    uint32_t before_c = block_exclusive_scan<uint32_t>(hi > lo ? my_c : 0u, sh.scan32, &tot_c);
    if (massc && pass == 0) {
      // every key is in the first pass's histogram: tot_w is the slot's total weight
      if (tot_w == 0) {           // no mass at all: the first key alone reaches 0.9 * 0
        if (tid == 0) a.count[s] = 1;
        return;
      }
      target = (unsigned long long)ceil((double)a.mass * (double)tot_w);
      if (target == 0) target = 1;
      if (target > tot_w) target = tot_w;
    }
    {
      unsigned long long run = w_above + before_w;
      uint32_t runc = before_c;
      for (int b = hi - 1; b >= lo; --b) {
        const uint32_t cb = sh.hcnt[b];
        const unsigned long long wb = bin_w(b);
        if (cb > 0 && run < target && run + wb >= target) {
          sh.sel_bin = b;
          sh.w_above_bin = run;
          sh.cnt_above_bin = runc;
        }
        run += wb;
        runc += cb;
      }
    }
    __syncthreads();
    prefix |= sh.sel_bin << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
    w_above = sh.w_above_bin;
    cnt_above += sh.cnt_above_bin;
    __syncthreads();
  }
  const uint32_t T = prefix;
  const unsigned long long need = target - w_above;     // > 0, reached inside the tie group

  if (massc) {
    if (tid == 0) {
      // every tied key has the same weight
      const unsigned long long bw = ((unsigned long long)sh.hwh[sh.sel_bin] << 32) | sh.hwl[sh.sel_bin];
      unsigned long long wt = bw / sh.hcnt[sh.sel_bin];
      unsigned long long take = (need + wt - 1) / wt;
      a.count[s] = (int)(cnt_above + take);
    }
    return;
  }

  // weight of the kept part of the tie group: TOPB -> need; CHUNK -> the shortest
  // index-ordered prefix of tied chunks whose lengths reach `need`
  if (tid == 0) sh.s_sel = chunk ? 0ull : need;
  __syncthreads();
  if (chunk) {
    unsigned long long carry = 0;
    for (int base = 0; base < N; base += blockDim.x) {
      const int n = base + tid;
      const uint32_t key = n < N ? key_of(n) : 0u;
      unsigned long long wt = (n < N && key == T) ? weight_of(n, key) : 0ull, tot;
      unsigned long long before = carry + block_exclusive_scan<unsigned long long>(wt, sh.scan64, &tot);
      if (wt > 0 && before < need && before + wt >= need) sh.s_sel = before + wt;
      carry += tot;
      if (carry >= need) break;           // uniform across the block
    }
    __syncthreads();
  }
  const unsigned long long s_sel = sh.s_sel;

  // emission in ascending position order: each thread takes SEL_IT consecutive
  // keys; one block scan per tile of the packed (weight above T, tied weight)
  // pair - both sums are < 2^31, so the two 32-bit halves never carry.
  constexpr int SEL_IT = 8;
  unsigned long long carry = 0;
  const uint32_t s_sel32 = (uint32_t)s_sel;
  for (int base = 0; base < N; base += blockDim.x * SEL_IT) {
    const int n0 = base + tid * SEL_IT;
    uint32_t kk[SEL_IT], ww[SEL_IT];
    uint32_t g_loc = 0, t_loc = 0;
#pragma unroll
    for (int i = 0; i < SEL_IT; i += 4) keys4(n0 + i, kk + i);
#pragma unroll
    for (int i = 0; i < SEL_IT; ++i) {
      const int n = n0 + i;
      ww[i] = (n < N && kk[i] >= T) ? (uint32_t)weight_of(n, kk[i]) : 0u;
      if (kk[i] > T) g_loc += ww[i];
      else if (kk[i] == T) t_loc += ww[i];
    }
    unsigned long long tot;
    const unsigned long long before =
        carry + block_exclusive_scan<unsigned long long>(((unsigned long long)g_loc << 32) | t_loc, sh.scan64, &tot);
    uint32_t bg = (uint32_t)(before >> 32), bt = (uint32_t)before;
#pragma unroll
    for (int i = 0; i < SEL_IT; ++i) {
      const int n = n0 + i;
      if (ww[i] == 0) continue;
      const bool gt = kk[i] > T;
      if (gt || bt < s_sel32) {
        const uint32_t pos = bg + (bt < s_sel32 ? bt : s_sel32);
        if (!chunk) {
          if (pos < (uint32_t)a.max_sel) idx_row[pos] = n;
        } else {
          const int start = n > 0 ? ce[n - 1] + 1 : 0;
          for (uint32_t t = 0; t < ww[i]; ++t)
            if (pos + t < (uint32_t)a.max_sel) idx_row[pos + t] = start + (int)t;
        }
      }
      if (gt) bg += ww[i];
      else bt += ww[i];
    }
    carry += tot;
  }
  if (tid == 0) {
    const unsigned long long total = (carry >> 32) + s_sel;
    if (total > (unsigned long long)a.max_sel) kvc_flag(KVC_DEVERR_INDEX_RANGE);
    a.count[s] = (int)min(total, (unsigned long long)a.max_sel);
  }
}

// ---------------------------------------------------------------- cluster form
// The same selection spread over a cluster of K CTAs per slot (2 <= K <= 16, the cluster
// size). Rank r owns the contiguous key range [r*per, min(N, (r+1)*per)) and caches its
// keys in shared memory. Each radix pass:
//   1. every CTA builds the histogram of its own range;                 cluster barrier
//   2. rank r sums the bins of its slice [r*nb/K, (r+1)*nb/K) over the cluster through
//      distributed shared memory and keeps them with their descending inclusive prefix
//      sums and the slice totals;                                       cluster barrier
//   3. every CTA finds the slice holding the target from the K slice totals and the bin
//      inside it from that slice's prefixes: the same answer on every rank, no third
//      exchange.
// Emission exchanges each range's (weight above T, tied weight) pair once, after which
// each rank writes the output positions of its own range (CHUNK also shares s_sel, which
// the rank holding the crossing chunk computes). Keys, weights, histograms and every sum
// are those of select_kernel, so both forms return the same selection.
constexpr int SCL_THREADS = 512;
constexpr int SCL_MAX_K = 16;
constexpr int SCL_IT = 4;       // consecutive keys per thread in an emission tile

struct SelClShared {
  uint32_t hcnt[SEL_MAX_BINS];                 // histogram of this CTA's key range
  uint32_t hwl[SEL_MAX_BINS], hwh[SEL_MAX_BINS];   // bin weights, low and high 32 bits
  // the owned bin slice summed over the cluster, in descending bin order (t = 0: highest)
  uint32_t mc[SEL_MAX_BINS / 2], pc[SEL_MAX_BINS / 2];
  unsigned long long mw[SEL_MAX_BINS / 2], pw[SEL_MAX_BINS / 2];
  unsigned long long scan64[33];
  uint32_t scan32[33];
  // values the other ranks read
  unsigned long long st_w;     // owned slice: total weight
  uint32_t st_c;               //              total count
  uint32_t xmax;               // MASS_COUNT: bits of this range's largest score
  uint32_t xspec;              // SPECIAL: marked positions in this range
  unsigned long long xgt;      // emission: (weight above T) << 32 | tied weight, this range
  unsigned long long xssel;    // CHUNK: s_sel, written by the rank holding the crossing chunk
  // the crossing bin of the current pass
  uint32_t sel_bin, cnt_above_bin, bin_c;
  unsigned long long w_above_bin, bin_w;
};

KVC_DEV void cluster_arrive() { asm volatile("barrier.cluster.arrive.aligned;" ::: "memory"); }

__global__ void __launch_bounds__(SCL_THREADS) select_cluster_kernel(SelectParams a) {
  extern __shared__ __align__(16) unsigned char scl_smem_raw[];
  SelClShared& sh = *reinterpret_cast<SelClShared*>(scl_smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(scl_smem_raw + sizeof(SelClShared));
  uint32_t* wts = keys + a.key_cap;            // CHUNK: chunk lengths, then output positions

  const int K = (int)cluster_nctas();
  const int r = (int)cluster_rank();
  const int s = blockIdx.x / K;
  const int tid = threadIdx.x, nthr = blockDim.x, lane = tid & 31;
  const int pol = a.policy ? a.policy[s] : KVC_POL_CHUNK;
  const int L = a.L;
  int32_t* idx_row = a.idx ? a.idx + (size_t)s * a.max_sel : nullptr;
  const bool lead = r == 0 && tid == 0;
  constexpr unsigned FULL = 0xffffffffu;
  if (K < 2 || K > SCL_MAX_K) {                 // launched without a cluster of 2..16
    if (tid == 0) kvc_flag(KVC_DEVERR_INDEX_RANGE);
    return;
  }

  // this rank's share [lo, hi) of n items
  auto share = [&](int n, int* lo, int* hi) {
    const int per = (n + K - 1) / K;
    *lo = min(r * per, n);
    *hi = min(*lo + per, n);
  };
  // positions [first, first + n) to the row, this rank's share of them
  auto emit_share = [&](int first, int n) {
    int lo, hi;
    share(n, &lo, &hi);
    for (int i = lo + tid; i < hi; i += nthr)
      if (i < a.max_sel) idx_row[i] = first + i;
  };
  auto set_count = [&](long long n) {
    if (n > a.max_sel) kvc_flag(KVC_DEVERR_INDEX_RANGE);
    a.count[s] = (int)min(n, (long long)a.max_sel);
  };

  if (pol == KVC_POL_LOCAL || pol == KVC_POL_FULL) {
    if (!idx_row) {
      if (lead) { kvc_flag(KVC_DEVERR_INDEX_RANGE); a.count[s] = 0; }
      return;
    }
    const int W = pol == KVC_POL_FULL ? L : min(max(a.budget[s], 0), L);
    emit_share(L - W, W);
    if (lead) set_count(W);
    return;
  }
  if (pol == KVC_POL_SPECIAL) {
    if (!a.special_mask || !idx_row) {
      if (lead) { kvc_flag(KVC_DEVERR_INDEX_RANGE); a.count[s] = 0; }
      return;
    }
    const int b = (s / a.n_kv_heads) % a.batch;
    const uint8_t* m = a.special_mask + (size_t)b * L;
    int lo, hi;
    share(L, &lo, &hi);
    uint32_t mine = 0;
    for (int n = lo + tid; n < hi; n += nthr) mine += m[n] ? 1u : 0u;
    mine = block_sum<uint32_t>(mine, sh.scan32);
    if (tid == 0) sh.xspec = mine;
    cluster_sync();
    const uint32_t v = lane < K ? ld_cluster_u32(map_to_rank(&sh.xspec, lane)) : 0u;
    uint32_t carry = lane < r ? v : 0u, total = v;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      carry += __shfl_xor_sync(FULL, carry, o);
      total += __shfl_xor_sync(FULL, total, o);
    }
    cluster_arrive();                 // last read of another CTA's shared memory
    for (int base = lo; base < hi; base += nthr) {
      const int n = base + tid;
      uint32_t f = (n < hi && m[n]) ? 1u : 0u, tot;
      const uint32_t pos = carry + block_exclusive_scan<uint32_t>(f, sh.scan32, &tot);
      if (f && pos < (uint32_t)a.max_sel) idx_row[pos] = n;
      carry += tot;
    }
    if (lead) set_count(total);
    cluster_wait();                   // no CTA leaves while another may still read it
    return;
  }

  // ------------------------------------------------ weighted selection
  const bool chunk = pol == KVC_POL_CHUNK;
  const bool massc = pol == KVC_POL_MASS_COUNT;
  const bool unit = !chunk && !massc;
  const int N = chunk ? a.C : L;
  const float* sc = a.score + (size_t)s * N;
  const int32_t* ce = a.chunk_end;
  if (!a.score || (chunk && !ce) || (!massc && !idx_row) || (pol != KVC_POL_TOPB && !massc && !chunk)) {
    if (lead) { kvc_flag(KVC_DEVERR_INDEX_RANGE); a.count[s] = 0; }
    return;
  }
  const int n_local = chunk ? min(max(a.n_local, 0), N) : 0;
  if (n_local > 0) {
    const int first_local_tok = N - n_local > 0 ? ce[N - n_local - 1] + 1 : 0;
    if ((long long)(L - first_local_tok) >= (long long)a.budget[s]) {
      emit_share(first_local_tok, L - first_local_tok);
      if (lead) set_count(L - first_local_tok);
      return;
    }
  }
  unsigned long long target = 0;
  if (!massc) {
    const long long want = a.budget[s];
    const long long full = chunk ? (long long)L : (long long)N;
    if (want >= full || want <= 0) {
      const int n_out = want <= 0 ? 0 : (int)full;
      emit_share(0, n_out);
      if (lead) set_count(n_out);
      return;
    }
    target = (unsigned long long)want;
  }

  if ((N + K - 1) / K > a.key_cap) {             // the range does not fit the key cache
    if (lead) { kvc_flag(KVC_DEVERR_INDEX_RANGE); a.count[s] = 0; }
    return;
  }
  int lo, hi;
  share(N, &lo, &hi);
  const int nr = hi - lo;
  float mx = 0.f;
  for (int i = tid; i < nr; i += nthr) {
    const int n = lo + i;
    const float f = sc[n];
    keys[i] = n >= N - n_local ? 0xffffffffu : order_key(f);
    if (chunk) wts[i] = (uint32_t)(ce[n] - (n > 0 ? ce[n - 1] : -1));
    if (massc) mx = fmaxf(mx, f);
  }
  int fx = 0;
  if (massc) {
    // fixed-point scale from the slot's largest score: every rank derives the same one
    mx = warp_max(mx);
    if (lane == 0) sh.scan32[tid >> 5] = __float_as_uint(mx);
    __syncthreads();
    if (tid == 0) {
      float m = 0.f;
      for (int w = 0; w < (nthr >> 5); ++w) m = fmaxf(m, __uint_as_float(sh.scan32[w]));
      sh.xmax = __float_as_uint(m);
    }
    cluster_sync();
    float m = lane < K ? __uint_as_float(ld_cluster_u32(map_to_rank(&sh.xmax, lane))) : 0.f;
    m = warp_max(m);
    int ex = 0;
    frexpf(m > 0.f ? m : 1.f, &ex);             // m < 2^ex
    const int lg = 32 - __clz(max(N - 1, 1));   // 2^lg >= N
    fx = 62 - lg - ex;
  }
  __syncthreads();
  auto weight_of = [&](int i) -> unsigned long long {
    if (chunk) return wts[i];
    if (massc) {
      return fixed_weight(key_score(keys[i]), fx);
    }
    return 1ull;
  };

  // radix passes: digits [31:21], [20:10], [9:0]
  uint32_t prefix = 0, pmask = 0, cnt_above = 0;
  unsigned long long w_above = 0;
  bool no_mass = false;
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
    const int nb = pass == 2 ? 1024 : 2048;
    const int sl = nb / K;                      // bins per slice (>= 64)
    for (int b = tid; b < nb; b += nthr) {
      sh.hcnt[b] = 0;
      sh.hwl[b] = 0;
      sh.hwh[b] = 0;
    }
    __syncthreads();
    // 1. histogram of this range
    for (int base = 0; base < nr; base += nthr) {
      const int i = base + tid;
      bool match = false;
      uint32_t bin = 0;
      unsigned long long wt = 0;
      if (i < nr) {
        const uint32_t key = keys[i];
        match = (key & pmask) == prefix;
        bin = (key >> shift) & (nb - 1);
        if (match) wt = weight_of(i);
      }
      if (match) {                     // one shared atomic per key and word (as select_kernel)
        atomicAdd(&sh.hcnt[bin], 1u);
        if (!unit) bin_add_u64(&sh.hwl[bin], &sh.hwh[bin], wt);
      }
    }
    cluster_sync();
    // 2. the owned slice over the cluster: thread tid takes the bins t in [tid*per_t, +per_t)
    {
      const int per_t = (sl + nthr - 1) / nthr;     // 1 or 2
      const int t0 = tid * per_t;
      uint32_t c[2] = {0u, 0u};
      unsigned long long w[2] = {0ull, 0ull};
      uint32_t my_c = 0;
      unsigned long long my_w = 0;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int t = t0 + j;
        if (j >= per_t || t >= sl) continue;
        const int b = (r + 1) * sl - 1 - t;
        for (int q = 0; q < K; ++q) {
          c[j] += ld_cluster_u32(map_to_rank(&sh.hcnt[b], q));
          if (!unit)
            w[j] += ((unsigned long long)ld_cluster_u32(map_to_rank(&sh.hwh[b], q)) << 32) |
                    ld_cluster_u32(map_to_rank(&sh.hwl[b], q));
        }
        if (unit) w[j] = c[j];
        my_c += c[j];
        my_w += w[j];
      }
      unsigned long long tot_w;
      unsigned long long ex_w = block_exclusive_scan<unsigned long long>(my_w, sh.scan64, &tot_w);
      uint32_t tot_c = 0, ex_c = 0;
      if (massc) ex_c = block_exclusive_scan<uint32_t>(my_c, sh.scan32, &tot_c);
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int t = t0 + j;
        if (j >= per_t || t >= sl) continue;
        ex_w += w[j];
        ex_c += c[j];
        sh.mw[t] = w[j];
        sh.pw[t] = ex_w;
        sh.mc[t] = c[j];
        sh.pc[t] = ex_c;
      }
      if (tid == 0) {
        sh.st_w = tot_w;
        sh.st_c = tot_c;
      }
    }
    cluster_sync();
    // 3. the crossing slice from the K slice totals (every warp alike), then its bin
    unsigned long long qw = 0;
    uint32_t qc = 0;
    if (lane < K) {
      qw = ld_cluster_u64(map_to_rank(&sh.st_w, lane));
      if (massc) qc = ld_cluster_u32(map_to_rank(&sh.st_c, lane));
    }
    unsigned long long suf_w = qw;             // slices lane..K-1 (higher slices hold higher bins)
    uint32_t suf_c = qc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long yw = __shfl_down_sync(FULL, suf_w, o);
      const uint32_t yc = __shfl_down_sync(FULL, suf_c, o);
      if (lane + o < 32) {
        suf_w += yw;
        suf_c += yc;
      }
    }
    if (massc && pass == 0) {
      const unsigned long long total = __shfl_sync(FULL, suf_w, 0);
      if (total == 0) {                         // no mass at all: the first key alone reaches 0.9 * 0
        no_mass = true;
        break;
      }
      target = (unsigned long long)ceil((double)a.mass * (double)total);
      if (target == 0) target = 1;
      if (target > total) target = total;
    }
    const unsigned long long above_w = w_above + suf_w - qw;
    const unsigned cm = __ballot_sync(FULL, lane < K && above_w < target && target <= above_w + qw);
    if (cm == 0 && tid == 0) kvc_flag(KVC_DEVERR_INDEX_RANGE);   // cannot happen: target <= total weight
    const int qs = cm ? __ffs(cm) - 1 : 0;
    const unsigned long long rb = __shfl_sync(FULL, above_w, qs);
    const uint32_t cb = __shfl_sync(FULL, suf_c - qc, qs);
    for (int t = tid; t < sl; t += nthr) {
      const unsigned long long wb = ld_cluster_u64(map_to_rank(&sh.mw[t], qs));
      const unsigned long long run = rb + ld_cluster_u64(map_to_rank(&sh.pw[t], qs)) - wb;
      if (run < target && target <= run + wb) {
        sh.sel_bin = (uint32_t)((qs + 1) * sl - 1 - t);
        sh.w_above_bin = run;
        sh.bin_w = wb;
        if (massc) {
          const uint32_t mcb = ld_cluster_u32(map_to_rank(&sh.mc[t], qs));
          sh.bin_c = mcb;
          sh.cnt_above_bin = cb + ld_cluster_u32(map_to_rank(&sh.pc[t], qs)) - mcb;
        }
      }
    }
    __syncthreads();
    // (sel_bin and the slice arrays are rewritten only after the next pass's two barriers)
    prefix |= sh.sel_bin << shift;
    pmask |= (uint32_t)(nb - 1) << shift;
    w_above = sh.w_above_bin;
    if (massc) cnt_above += sh.cnt_above_bin;
  }

  if (massc) {
    cluster_arrive();                           // last read of another CTA's shared memory
    if (lead) {
      if (no_mass) {
        a.count[s] = 1;
      } else {
        const unsigned long long need = target - w_above;
        const unsigned long long wt = sh.bin_w / max(sh.bin_c, 1u);   // every tied key weighs the same
        const unsigned long long take = wt ? (need + wt - 1) / wt : 1ull;
        a.count[s] = (int)(cnt_above + take);
      }
    }
    cluster_wait();
    return;
  }

  const uint32_t T = prefix;
  const unsigned long long need = target - w_above;     // > 0, reached inside the tie group
  // E1: each range's weight above T and tied weight (each sum < 2^31: no carry between halves)
  uint32_t g_loc = 0, t_loc = 0;
  for (int i = tid; i < nr; i += nthr) {
    const uint32_t k = keys[i];
    if (k >= T) {
      const uint32_t w = (uint32_t)weight_of(i);
      if (k > T) g_loc += w;
      else t_loc += w;
    }
  }
  const unsigned long long mine = block_sum<unsigned long long>(((unsigned long long)g_loc << 32) | t_loc, sh.scan64);
  if (tid == 0) sh.xgt = mine;
  cluster_sync();
  const unsigned long long v = lane < K ? ld_cluster_u64(map_to_rank(&sh.xgt, lane)) : 0ull;
  unsigned long long below = lane < r ? v : 0ull, all = v;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    below += __shfl_xor_sync(FULL, below, o);
    all += __shfl_xor_sync(FULL, all, o);
  }
  unsigned long long s_sel = need;
  if (chunk) {
    // the rank whose range holds the crossing tied chunk: its tied weight prefix < need <= + its own
    uint32_t ex_t = (uint32_t)v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(FULL, ex_t, o);
      if (lane >= o) ex_t += y;
    }
    ex_t -= (uint32_t)v;
    const unsigned cm = __ballot_sync(FULL, lane < K && ex_t < need && need <= (unsigned long long)ex_t + (uint32_t)v);
    const int rc = cm ? __ffs(cm) - 1 : 0;
    if (r == rc) {
      // s_sel: the running tied weight, in index order, at the chunk that reaches `need`
      unsigned long long carry = (uint32_t)below;
      for (int base = 0; base < nr; base += nthr) {
        const int i = base + tid;
        unsigned long long wt = (i < nr && keys[i] == T) ? (unsigned long long)wts[i] : 0ull, tot;
        const unsigned long long before = carry + block_exclusive_scan<unsigned long long>(wt, sh.scan64, &tot);
        if (wt > 0 && before < need && before + wt >= need) sh.xssel = before + wt;
        carry += tot;
        if (carry >= need) break;               // uniform across the block
      }
    }
    cluster_sync();
    unsigned long long x = lane == 0 ? ld_cluster_u64(map_to_rank(&sh.xssel, rc)) : 0ull;
    s_sel = __shfl_sync(FULL, x, 0);
  }
  cluster_arrive();                             // last read of another CTA's shared memory

  // emission in ascending position order over this range (see select_kernel)
  unsigned long long carry = below;
  const uint32_t s_sel32 = (uint32_t)s_sel;
  for (int base = 0; base < nr; base += nthr * SCL_IT) {
    const int i0 = base + tid * SCL_IT;
    uint32_t kk[SCL_IT], ww[SCL_IT];
    uint32_t g = 0, t = 0;
#pragma unroll
    for (int j = 0; j < SCL_IT; ++j) {
      const int i = i0 + j;
      kk[j] = i < nr ? keys[i] : 0u;
      ww[j] = (i < nr && kk[j] >= T) ? (uint32_t)weight_of(i) : 0u;
      if (kk[j] > T) g += ww[j];
      else t += ww[j];
    }
    unsigned long long tot;
    const unsigned long long before =
        carry + block_exclusive_scan<unsigned long long>(((unsigned long long)g << 32) | t, sh.scan64, &tot);
    uint32_t bg = (uint32_t)(before >> 32), bt = (uint32_t)before;
#pragma unroll
    for (int j = 0; j < SCL_IT; ++j) {
      const int i = i0 + j;
      const uint32_t pos = bg + (bt < s_sel32 ? bt : s_sel32);
      if (chunk) {
        if (i < nr) wts[i] = pos;               // where chunk i's tokens start (length 0 if not kept)
      } else if (ww[j] != 0 && (kk[j] > T || bt < s_sel32)) {
        if (pos < (uint32_t)a.max_sel) idx_row[pos] = lo + i;
      }
      if (kk[j] > T) bg += ww[j];
      else bt += ww[j];
    }
    carry += tot;
  }
  if (chunk) {
    __syncthreads();
    // output position p belongs to the last chunk of the range that starts at or before p
    const uint32_t cg = (uint32_t)(carry >> 32), ct = (uint32_t)carry;
    const uint32_t out_lo = (uint32_t)(below >> 32) + min((uint32_t)below, s_sel32);
    const uint32_t out_hi = cg + min(ct, s_sel32);
    for (uint32_t p = out_lo + tid; p < out_hi; p += nthr) {
      int l = 0, h = nr;
      while (l < h) {
        const int mid = (l + h) >> 1;
        if (wts[mid] <= p) l = mid + 1;
        else h = mid;
      }
      if (l == 0) continue;                     // not reached: wts[0] == out_lo <= p
      const int n = lo + l - 1;
      const int start = n > 0 ? ce[n - 1] + 1 : 0;
      if (p < (uint32_t)a.max_sel) idx_row[p] = start + (int)(p - wts[l - 1]);
    }
  }
  if (lead) set_count((long long)(all >> 32) + (long long)s_sel);
  cluster_wait();
}

inline size_t select_cluster_smem_bytes(int key_cap) { return sizeof(SelClShared) + (size_t)key_cap * 8; }

inline int select_key_cap(int L, int C) {
  const int n = L > C ? L : C;
  return n < SEL_SMEM_KEYS ? n : SEL_SMEM_KEYS;
}
inline size_t select_smem_bytes(int key_cap) { return sizeof(SelShared) + (size_t)key_cap * 4; }

}  // namespace kvc
