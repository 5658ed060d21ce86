// Window scoring on the CUDA cores (fp32 arithmetic), for fp32 inputs and for any
// shape the tensor-core path does not take.
//
// Observation-window importance (ZigZagKV, Eq. 7, after SnapKV): for each slot,
// every window row r = j*w + i (query head j of the group, window row i, at
// position L - w + i) takes a softmax over the keys it sees, and the score of key
// n is the sum over rows of p_{r,n}. Two passes over the keys:
//   1. per key block, each row's max and sum of exp (partial softmax statistics);
//   2. (after a tiny merge kernel) each key's column sum of exp(z - lse_r).
// Chunk scoring (ChunkLLM Eq. 3) is the same with key n read from row
// chunk_end[n] and placed at that position.
#pragma once
#include "common.cuh"

namespace kvc {

constexpr int SIMT_TB = 64;        // keys per block
constexpr int SIMT_THREADS = 256;

// Keys of the block in shared memory as fp32 rows of stride d+1 (conflict-free
// when lanes read different keys at the same column).
template <typename T>
KVC_DEV void simt_load_keys(float* ks, const T* k_slot, const int32_t* key_idx, int n0, int N, int L, int d) {
  for (int e = threadIdx.x; e < SIMT_TB * d; e += blockDim.x) {
    int j = e / d, c = e - j * d;
    int n = n0 + j;
    float v = 0.f;
    if (n < N) {
      const int row = key_idx ? key_idx[n] : n;
      if (row >= 0 && row < L) v = to_f(k_slot[(size_t)row * d + c]);
      else if (c == 0) kvc_flag(KVC_DEVERR_INDEX_RANGE);
    }
    ks[j * (d + 1) + c] = v;
  }
}

template <typename T>
KVC_DEV void simt_load_q(float* qs, const T* q_slot, int R, int d) {
  for (int e = threadIdx.x; e < R * d; e += blockDim.x) qs[e] = to_f(q_slot[e]);
}

// grid (nblk, S); part[(s*nblk + blk)*R + r] = (row max, row sum of exp(z - max)) over the block.
template <typename T>
__global__ void __launch_bounds__(SIMT_THREADS)
score_stats_simt(const T* __restrict__ q_win, const T* __restrict__ k, const int32_t* __restrict__ key_idx,
                 int N, int L, int G, int w, int d, float scale, float2* __restrict__ part) {
  extern __shared__ float sm_simt[];
  const int R = G * w;
  const int s = blockIdx.y, blk = blockIdx.x, nblk = gridDim.x;
  float* qs = sm_simt;                 // [R][d]
  float* ks = qs + R * d;              // [TB][d+1]
  const int n0 = blk * SIMT_TB;
  simt_load_q(qs, q_win + (size_t)s * R * d, R, d);
  simt_load_keys(ks, k + (size_t)s * L * d, key_idx, n0, N, L, d);
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int r = warp; r < R; r += nw) {
    const int rowpos = L - w + (r % w);
    float z[SIMT_TB / 32];
    float m = -INFINITY;
#pragma unroll
    for (int u = 0; u < SIMT_TB / 32; ++u) {
      int j = lane + 32 * u, n = n0 + j;
      bool vis = n < N && (key_idx ? key_idx[n] : n) <= rowpos;
      float acc = 0.f;
      for (int c = 0; c < d; ++c) acc = fmaf(qs[r * d + c], ks[j * (d + 1) + c], acc);
      z[u] = vis ? acc * scale : -INFINITY;
      m = fmaxf(m, z[u]);
    }
    m = warp_max(m);
    float l = 0.f;
#pragma unroll
    for (int u = 0; u < SIMT_TB / 32; ++u) l += (z[u] == -INFINITY) ? 0.f : expf(z[u] - m);
    l = warp_sum(l);
    if (lane == 0) part[((size_t)s * nblk + blk) * R + r] = make_float2(m, l);
  }
}

// grid S, block >= R: lse[s*R + r] = max + log(sum of exp) over all blocks (natural log).
__global__ void score_lse_merge(const float2* __restrict__ part, int nblk, int R, float* __restrict__ lse) {
  const int s = blockIdx.x;
  for (int r = threadIdx.x; r < R; r += blockDim.x) {
    float M = -INFINITY;
    for (int b = 0; b < nblk; ++b) M = fmaxf(M, part[((size_t)s * nblk + b) * R + r].x);
    float l = 0.f;
    if (M != -INFINITY)
      for (int b = 0; b < nblk; ++b) {
        float2 p = part[((size_t)s * nblk + b) * R + r];
        if (p.x != -INFINITY) l += p.y * expf(p.x - M);
      }
    lse[(size_t)s * R + r] = (l > 0.f) ? M + logf(l) : INFINITY;   // +inf: row sees nothing
  }
}

// grid (nblk, S): score[s][n] = sum_r exp(z_{r,n} - lse_r) over the rows that see key n.
template <typename T>
__global__ void __launch_bounds__(SIMT_THREADS)
score_colsum_simt(const T* __restrict__ q_win, const T* __restrict__ k, const int32_t* __restrict__ key_idx,
                  int N, int L, int G, int w, int d, float scale, const float* __restrict__ lse,
                  float* __restrict__ score) {
  extern __shared__ float sm_simt[];
  const int R = G * w;
  const int s = blockIdx.y, blk = blockIdx.x;
  float* qs = sm_simt;                 // [R][d]
  float* ls = qs + R * d;              // [R]
  float* ks = ls + R;                  // [TB][d+1]
  float* red = ks + SIMT_TB * (d + 1); // [threads]
  const int n0 = blk * SIMT_TB;
  simt_load_q(qs, q_win + (size_t)s * R * d, R, d);
  for (int r = threadIdx.x; r < R; r += blockDim.x) ls[r] = lse[(size_t)s * R + r];
  simt_load_keys(ks, k + (size_t)s * L * d, key_idx, n0, N, L, d);
  __syncthreads();
  const int j = threadIdx.x % SIMT_TB, part = threadIdx.x / SIMT_TB, nparts = blockDim.x / SIMT_TB;
  const int n = n0 + j;
  float acc = 0.f;
  if (n < N) {
    const int pos = key_idx ? key_idx[n] : n;
    for (int r = part; r < R; r += nparts) {
      if (pos > L - w + (r % w)) continue;
      float z = 0.f;
      for (int c = 0; c < d; ++c) z = fmaf(qs[r * d + c], ks[j * (d + 1) + c], z);
      acc += expf(z * scale - ls[r]);
    }
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  if (part == 0 && n < N) {
    float t = 0.f;
    for (int p = 0; p < nparts; ++p) t += red[p * SIMT_TB + j];
    score[(size_t)s * N + n] = t;
  }
}

}  // namespace kvc
