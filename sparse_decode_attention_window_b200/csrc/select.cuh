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

struct SelShared {
  uint32_t hcnt[SEL_MAX_BINS];
  unsigned long long hw[SEL_MAX_BINS];
  unsigned long long wstage[SEL_THREADS];
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
  if (cached)
    for (int n = tid; n < N; n += blockDim.x) keys[n] = raw_key(n);
  // weights
  int fx = 0;
  if (massc) {
    float mx = 0.f;
    for (int n = tid; n < N; n += blockDim.x) mx = fmaxf(mx, sc[n]);
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
  auto weight_of = [&](int n) -> unsigned long long {
    if (chunk) return (unsigned long long)(ce[n] - (n > 0 ? ce[n - 1] : -1));
    if (massc) {
      float v = fmaxf(sc[n], 0.f);
      return (unsigned long long)__double2ull_rz(ldexp((double)v, fx));
    }
    return 1ull;
  };

  // target
  unsigned long long target;
  if (massc) {
    unsigned long long tw = 0;
    for (int n = tid; n < N; n += blockDim.x) tw += weight_of(n);
    unsigned long long total = block_sum<unsigned long long>(tw, sh.scan64);
    if (total == 0) {           // no mass at all: the first key alone reaches 0.9 * 0
      if (tid == 0) a.count[s] = 1;
      return;
    }
    double t = ceil((double)a.mass * (double)total);
    target = (unsigned long long)t;
    if (target == 0) target = 1;
    if (target > total) target = total;
  } else {
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
  const int shifts[3] = {21, 10, 0};
  const int bitsz[3] = {11, 11, 10};
  const int lane = tid & 31;
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = shifts[pass], nb = 1 << bitsz[pass];
    for (int b = tid; b < nb; b += blockDim.x) { sh.hcnt[b] = 0; sh.hw[b] = 0; }
    __syncthreads();
    for (int base = 0; base < N; base += blockDim.x) {
      const int n = base + tid;
      bool match = false;
      uint32_t bin = 0;
      unsigned long long wt = 0;
      if (n < N) {
        uint32_t key = key_of(n);
        match = (key & pmask) == prefix;
        bin = (key >> shift) & (nb - 1);
        if (match) wt = weight_of(n);
      }
      const unsigned mm = __ballot_sync(0xffffffffu, match);
      if (match) {
        const unsigned peers = __match_any_sync(mm, bin);
        const int leader = __ffs(peers) - 1;
        if (unit) {
          // top-B: every weight is 1, the count is the weight
          if (lane == leader) atomicAdd(&sh.hcnt[bin], (uint32_t)__popc(peers));
        } else {
          sh.wstage[tid] = wt;
          __syncwarp(mm);
          if (lane == leader) {
            unsigned long long sum = 0;
            unsigned rest = peers;
            while (rest) {
              int l = __ffs(rest) - 1;
              rest &= rest - 1;
              sum += sh.wstage[(tid & ~31) + l];
            }
            atomicAdd(&sh.hcnt[bin], (uint32_t)__popc(peers));
            atomicAdd(&sh.hw[bin], sum);
          }
          __syncwarp(mm);
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
    for (int b = hi - 1; b >= lo; --b) { my_w += unit ? sh.hcnt[b] : sh.hw[b]; my_c += sh.hcnt[b]; }
    unsigned long long tot_w;
    uint32_t tot_c;
    unsigned long long before_w = block_exclusive_scan<unsigned long long>(hi > lo ? my_w : 0ull, sh.scan64, &tot_w);
    uint32_t before_c = block_exclusive_scan<uint32_t>(hi > lo ? my_c : 0u, sh.scan32, &tot_c);
    {
      unsigned long long run = w_above + before_w;
      uint32_t runc = before_c;
      for (int b = hi - 1; b >= lo; --b) {
        const uint32_t cb = sh.hcnt[b];
        const unsigned long long wb = unit ? (unsigned long long)cb : sh.hw[b];
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
      unsigned long long wt = sh.hw[sh.sel_bin] / sh.hcnt[sh.sel_bin];
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
      unsigned long long wt = (n < N && key_of(n) == T) ? weight_of(n) : 0ull, tot;
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
    for (int i = 0; i < SEL_IT; ++i) {
      const int n = n0 + i;
      kk[i] = n < N ? key_of(n) : 0u;
      ww[i] = (n < N && kk[i] >= T) ? (uint32_t)weight_of(n) : 0u;
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

inline int select_key_cap(int L, int C) {
  const int n = L > C ? L : C;
  return n < SEL_SMEM_KEYS ? n : SEL_SMEM_KEYS;
}
inline size_t select_smem_bytes(int key_cap) { return sizeof(SelShared) + (size_t)key_cap * 4; }

}  // namespace kvc
