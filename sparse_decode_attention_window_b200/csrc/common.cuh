// Device-side helpers shared by the kernels of libkvc: the error word, block
// scans, mbarrier / bulk-copy / TMA wrappers (inline PTX for sm_100a) with
// bounded waits.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda.h>
#include <stdint.h>

#include "../../include/kvc.h"

#define KVC_DEV __device__ __forceinline__
#define KVC_HD __host__ __device__ __forceinline__

// One error word per device (this library is built as a single translation unit).
__device__ unsigned int g_kvc_deverr;

KVC_DEV void kvc_flag(unsigned bits) { atomicOr(&g_kvc_deverr, bits); }

// ---------------------------------------------------------------- conversions
template <typename T> KVC_DEV float to_f(T x);
template <> KVC_DEV float to_f<float>(float x) { return x; }
template <> KVC_DEV float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }

// Unpack one 16-byte chunk into fp32 values (8 bf16 or 4 fp32).
template <typename T> struct Chunk16;
template <> struct Chunk16<float> {
  static constexpr int N = 4;
  KVC_DEV static void unpack(const uint4& u, float* f) {
    f[0] = __uint_as_float(u.x); f[1] = __uint_as_float(u.y);
    f[2] = __uint_as_float(u.z); f[3] = __uint_as_float(u.w);
  }
};
template <> struct Chunk16<__nv_bfloat16> {
  static constexpr int N = 8;
  KVC_DEV static void unpack(const uint4& u, float* f) {
    // bf16 -> fp32 is exact: the bf16 bits are the top half of the fp32 bits
    f[0] = __uint_as_float(u.x << 16); f[1] = __uint_as_float(u.x & 0xffff0000u);
    f[2] = __uint_as_float(u.y << 16); f[3] = __uint_as_float(u.y & 0xffff0000u);
    f[4] = __uint_as_float(u.z << 16); f[5] = __uint_as_float(u.z & 0xffff0000u);
    f[6] = __uint_as_float(u.w << 16); f[7] = __uint_as_float(u.w & 0xffff0000u);
  }
};

// ---------------------------------------------------------------- block scans
// Exclusive scan over the whole block (blockDim.x a multiple of 32, <= 1024).
// `sh` must hold 33 values of V. Returns the exclusive prefix; *total the block sum.
template <typename V>
KVC_DEV V block_exclusive_scan(V x, V* sh, V* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  V inc = x;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    V y = __shfl_up_sync(0xffffffffu, inc, o);
    if (lane >= o) inc += y;
  }
  if (lane == 31) sh[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    V v = lane < nw ? sh[lane] : V(0);
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      V y = __shfl_up_sync(0xffffffffu, v, o);
      if (lane >= o) v += y;
    }
    sh[lane] = v;
  }
  __syncthreads();
  V before = warp > 0 ? sh[warp - 1] : V(0);
  *total = sh[nw - 1];
  __syncthreads();
  return before + inc - x;
}

template <typename V>
KVC_DEV V block_sum(V x, V* sh) {
  V t;
  block_exclusive_scan(x, sh, &t);
  return t;
}

KVC_DEV float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
KVC_DEV float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// ---------------------------------------------------------------- PTX: mbarrier, bulk copies
KVC_DEV uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

KVC_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
KVC_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }
KVC_DEV void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

KVC_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
KVC_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
KVC_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

KVC_DEV uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Every wait in this library gives up after this long, flags KVC_DEVERR_WAIT_TIMEOUT
// and lets the caller unwind; no kernel can spin forever.
#ifndef KVC_WAIT_LIMIT_NS
#define KVC_WAIT_LIMIT_NS 2000000000ull
#endif

KVC_DEV bool mbar_wait_limit(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_timer_ns() - t0 > limit_ns) {
      kvc_flag(KVC_DEVERR_WAIT_TIMEOUT);
      return false;
    }
  }
}
KVC_DEV bool mbar_wait(uint64_t* bar, uint32_t parity) { return mbar_wait_limit(bar, parity, KVC_WAIT_LIMIT_NS); }

// ---------------------------------------------------------------- thread-block clusters
KVC_DEV uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}


// Map a local shared-memory address to the same offset in CTA `rank` of the cluster.
KVC_DEV uint32_t map_to_rank(const void* local, uint32_t rank) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_u32(local)), "r"(rank));
  return ra;
}
// Asynchronous 4-byte store into another CTA's shared memory; its completion counts 4
// bytes on that CTA's mbarrier.
KVC_DEV void st_async_f32(uint32_t remote_addr, float v, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(remote_addr),
               "r"(__float_as_uint(v)), "r"(remote_bar)
               : "memory");
}
KVC_DEV void cluster_arrive_relaxed() { asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory"); }
KVC_DEV void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }
KVC_DEV uint32_t cluster_nctas() {
  uint32_t n;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(n));
  return n;
}
// Every thread of every CTA in the cluster: shared-memory writes made before it (release)
// are visible to every CTA of the cluster after it (acquire).
KVC_DEV void cluster_sync() {
  asm volatile("barrier.cluster.arrive.aligned;\n\tbarrier.cluster.wait.aligned;" ::: "memory");
}
// Loads from another CTA's shared memory (an address from map_to_rank).
KVC_DEV uint32_t ld_cluster_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
KVC_DEV unsigned long long ld_cluster_u64(uint32_t addr) {
  unsigned long long v;
  asm volatile("ld.shared::cluster.u64 %0, [%1];" : "=l"(v) : "r"(addr) : "memory");
  return v;
}

// Bounded wait with cluster-scope acquire (data that other CTAs sent with st.async).
KVC_DEV bool mbar_wait_cluster(uint64_t* bar, uint32_t parity) {
  auto try_once = [&]() {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
  };
  if (try_once()) return true;
  const uint64_t t0 = global_timer_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 64; ++i)
      if (try_once()) return true;
    if (global_timer_ns() - t0 > KVC_WAIT_LIMIT_NS) {
      kvc_flag(KVC_DEVERR_WAIT_TIMEOUT);
      return false;
    }
  }
}

// Asynchronous 8-byte store into another CTA's shared memory; its completion counts 8
// bytes on that CTA's mbarrier.
KVC_DEV void st_async_f32x2(uint32_t remote_addr, float x, float y, uint32_t remote_bar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.b32 [%0], {%1, %2}, [%3];" ::"r"(remote_addr),
               "r"(__float_as_uint(x)), "r"(__float_as_uint(y)), "r"(remote_bar)
               : "memory");
}

// Plain (untiled) bulk copy global -> shared, completion counted on `bar`.
// Both addresses 16-byte aligned, bytes a multiple of 16.
KVC_DEV void bulk_g2s(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Tiled TMA load of a 3-D box into this CTA's shared memory. c0 is the innermost coordinate.
KVC_DEV void tma_load_3d(void* smem_dst, const CUtensorMap* map, int c0, int c1, int c2, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, "
      "%4}], [%5];" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
      : "memory");
}

KVC_DEV void prefetch_tensormap(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Arrive on named barrier `id` without waiting (the threads that sync on it wait for these).
KVC_DEV void named_bar_arrive(int id, int nthreads) {
  asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier among `nthreads` threads (a multiple of 32) with id `id` (1..15).
KVC_DEV void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Named barrier that also ORs a predicate over the participating threads.
KVC_DEV bool named_bar_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

KVC_DEV int elect_lane0() { return (threadIdx.x & 31) == 0; }
