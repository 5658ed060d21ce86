// Measurements over the window scores that drive the selection:
//  * retained_mass_kernel - share of each head's window-attention mass its kept tokens
//    hold (the quantity behind ZigZagKV's attention loss, Section 5.5 / Table 3);
//  * profile_kernel - FastGen-style head profiling: the cheapest of the local, special
//    and full policies that retains at least tau of the head's mass.
// One CTA per slot; sums in fp64 (order-independent enough for the 1e-5 comparisons).
#pragma once
#include "common.cuh"

namespace kvc {

constexpr int PROF_THREADS = 512;

KVC_DEV double block_sum_f64(double x, double* sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  if (lane == 0) sh[warp] = x;
  __syncthreads();
  double t = 0.0;
  if (threadIdx.x == 0) {
    for (int w = 0; w < nw; ++w) t += sh[w];
    sh[32] = t;
  }
  __syncthreads();
  t = sh[32];
  __syncthreads();
  return t;
}

// retained[s] = sum_{r < count[s]} score[s][idx[s][r]] / sum_n score[s][n]  (0 if no mass)
__global__ void __launch_bounds__(PROF_THREADS) retained_mass_kernel(const float* __restrict__ score, int N,
                                                                     const int32_t* __restrict__ idx, int max_sel,
                                                                     const int32_t* __restrict__ count,
                                                                     float* __restrict__ retained) {
  __shared__ double sh[33];
  const int s = blockIdx.x;
  const float* sc = score + (size_t)s * N;
  double tot = 0.0, kept = 0.0;
  for (int n = threadIdx.x; n < N; n += blockDim.x) tot += (double)sc[n];
  const int cnt = min(max(count[s], 0), max_sel);
  for (int r = threadIdx.x; r < cnt; r += blockDim.x) {
    const int j = idx[(size_t)s * max_sel + r];
    if (j >= 0 && j < N) kept += (double)sc[j];
    else kvc_flag(KVC_DEVERR_INDEX_RANGE);
  }
  tot = block_sum_f64(tot, sh);
  kept = block_sum_f64(kept, sh);
  if (threadIdx.x == 0) retained[s] = tot > 0.0 ? (float)(kept / tot) : 0.f;
}

// policy[s]: among LOCAL (last W tokens) and SPECIAL (the batch row's special tokens),
// the one keeping fewer tokens (ties: LOCAL) whose mass share reaches tau, tried in that
// order; FULL if neither does.
__global__ void __launch_bounds__(PROF_THREADS) profile_kernel(const float* __restrict__ score, int L,
                                                               const uint8_t* __restrict__ special_mask,
                                                               int n_kv_heads, int batch, int W, float tau,
                                                               int8_t* __restrict__ policy,
                                                               float* __restrict__ shares /* [S][2] or NULL */) {
  __shared__ double sh[33];
  const int s = blockIdx.x;
  const int b = (s / n_kv_heads) % batch;
  const float* sc = score + (size_t)s * L;
  const uint8_t* m = special_mask ? special_mask + (size_t)b * L : nullptr;
  const int wl = min(max(W, 0), L);
  double tot = 0.0, loc = 0.0, spc = 0.0, nspec = 0.0;
  for (int n = threadIdx.x; n < L; n += blockDim.x) {
    const double v = (double)sc[n];
    tot += v;
    if (n >= L - wl) loc += v;
    if (m && m[n]) { spc += v; nspec += 1.0; }
  }
  tot = block_sum_f64(tot, sh);
  loc = block_sum_f64(loc, sh);
  spc = block_sum_f64(spc, sh);
  nspec = block_sum_f64(nspec, sh);
  if (threadIdx.x == 0) {
    const double fl = tot > 0.0 ? loc / tot : 0.0, fs = tot > 0.0 ? spc / tot : 0.0;
    const bool ok_l = fl >= (double)tau, ok_s = m && fs >= (double)tau;
    int8_t pol = KVC_POL_FULL;
    if ((double)wl <= nspec) {
      pol = ok_l ? KVC_POL_LOCAL : (ok_s ? KVC_POL_SPECIAL : KVC_POL_FULL);
    } else {
      pol = ok_s ? KVC_POL_SPECIAL : (ok_l ? KVC_POL_LOCAL : KVC_POL_FULL);
    }
    policy[s] = pol;
    if (shares) {
      shares[2 * s] = (float)fl;
      shares[2 * s + 1] = (float)fs;
    }
  }
}

}  // namespace kvc
