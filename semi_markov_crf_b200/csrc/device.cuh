// device.cuh -- sm_100a device helpers shared by the semi-CRF kernels.
//
// Everything here is plain CUDA C++ or inline PTX written for this library:
// base-2 transcendental instructions, group reductions over aligned lane
// groups, shared-memory float max through an order-preserving integer map,
// and TMA bulk copies (cp.async.bulk, no multicast) completed on an mbarrier
// whose wait is bounded.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace semicrf {

constexpr unsigned FULL_MASK = 0xffffffffu;
constexpr double LOG2E_D = 1.4426950408889634073599246810019;
constexpr double LN2_D = 0.69314718055994530941723212145818;
constexpr float NEG_INF = -__builtin_huge_valf();

// Status codes written to the workspace status word (mirror semicrf.h).
constexpr int ST_DEVICE_TIMEOUT = 5;
constexpr int ST_BAD_LENGTH = 6;

// Bounds-checking debug build (-DSEMICRF_BOUNDS_CHECK; libsemicrf_b200_check.so).
// SEMICRF_INB(status, cond, site) is true in the release build; in the
// debug build a false `cond` records ST_BOUNDS | site << 8 in the status
// word (the first failure wins) and the caller skips the access it guards.
// Sites are numbered per file (see the SITE_* constants at each use); no
// trap, no fault: the kernel carries on and the host reads the status.
constexpr int ST_BOUNDS = 7;
#ifdef SEMICRF_BOUNDS_CHECK
__device__ __noinline__ inline void bounds_fail(int* status, int site) {
  if (status) atomicCAS(status, 0, ST_BOUNDS | (site << 8));
}
#define SEMICRF_INB(status, cond, site) \
  ((cond) ? true : (::semicrf::bounds_fail((status), (site)), false))
#else
#define SEMICRF_INB(status, cond, site) true
#endif

// Polls of an mbarrier before a wait gives up (each try_wait may itself
// suspend for a bounded, hardware-defined time).
constexpr int WAIT_SPIN_LIMIT = 1 << 22;

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float lg2(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// All-reduce over aligned groups of G lanes (G a power of two <= 32).  Every
// lane of the warp must execute the call.
__device__ __forceinline__ float group_max(float v, int G) {
  for (int o = G >> 1; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL_MASK, v, o));
  return v;
}
__device__ __forceinline__ float group_sum(float v, int G) {
  for (int o = G >> 1; o > 0; o >>= 1) v += __shfl_xor_sync(FULL_MASK, v, o);
  return v;
}

// Order-preserving float <-> int map, so shared-memory atomicMax on int gives
// a float max.
__device__ __forceinline__ int f2ord(float f) {
  int i = __float_as_int(f);
  return i >= 0 ? i : (i ^ 0x7fffffff);
}
__device__ __forceinline__ float ord2f(int i) {
  return __int_as_float(i >= 0 ? i : (i ^ 0x7fffffff));
}

__device__ __forceinline__ uint32_t smem_addr(const void* p);

// Contributes `key` (an f2ord value; pass INT_MIN for "no value") to the
// shared-memory max at `slot`: a warp-level max first, then one native
// shared-memory reduction per warp.  Every lane of the warp must call it.
__device__ __forceinline__ void warp_max_to_shared(int* slot, int key) {
  const int m = __reduce_max_sync(FULL_MASK, key);
  if ((threadIdx.x & 31) == 0)
    asm volatile("red.shared.max.s32 [%0], %1;" ::"r"(smem_addr(slot)), "r"(m) : "memory");
}

__device__ __forceinline__ void set_status(int* status, int code) {
  atomicCAS(status, 0, code);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Orders this thread's earlier generic-proxy shared-memory accesses before
// later async-proxy (TMA) accesses.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}

// One-dimensional TMA bulk copy global -> shared, completing on `bar`.
// dst, src 16-byte aligned; bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

// ----------------------------------------------------------------------------- clusters
// Rank of this CTA in its thread-block cluster.
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Cluster-wide barrier: every thread of every CTA of the cluster arrives
// (release: its earlier shared-memory stores, local or remote, are ordered
// before) and waits (acquire).  All threads of a warp execute it together.
__device__ __forceinline__ void cluster_sync() {
  asm volatile(
      "barrier.cluster.arrive.release.aligned;\n\t"
      "barrier.cluster.wait.acquire.aligned;" ::
          : "memory");
}

// Plain store of one float into the shared memory of CTA `rank` of this
// cluster, at the offset `local` has in this CTA's shared memory (the same
// carve in every CTA).  No multicast.
__device__ __forceinline__ void st_cluster(const float* local, uint32_t rank, float v) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_addr(local)), "r"(rank));
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(ra), "f"(v) : "memory");
}

// Asynchronous store of one float into the shared memory of CTA `rank` of
// this cluster (the offset `local` has here), completing `bytes` = 4 of the
// transaction count of that CTA's mbarrier at the offset of `bar`.  The
// receiver learns of the data by waiting on its own mbarrier; no memory
// fence is involved on either side.  No multicast.
__device__ __forceinline__ void st_async_cluster(const float* local, const uint64_t* bar,
                                                 uint32_t rank, float v) {
  uint32_t ra, rb;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_addr(local)), "r"(rank));
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(rb) : "r"(smem_addr(bar)), "r"(rank));
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(ra),
               "r"(__float_as_uint(v)), "r"(rb)
               : "memory");
}

// The address of `local` (a shared-memory location of this CTA) in the
// shared memory of cluster CTA `rank`.  A CTA's window is linear, so the
// address of local + off there is this plus off.
__device__ __forceinline__ uint32_t cluster_addr(const void* local, uint32_t rank) {
  uint32_t ra;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(smem_addr(local)), "r"(rank));
  return ra;
}

// st_async_cluster with the remote addresses already mapped (cluster_addr):
// v to ra, completing 4 bytes on the mbarrier at rb.
__device__ __forceinline__ void st_async_mapped(uint32_t ra, uint32_t rb, float v) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b32 [%0], %1, [%2];" ::"r"(ra),
               "r"(__float_as_uint(v)), "r"(rb)
               : "memory");
}

// Bounded wait, with cluster-scope acquire, for phase `parity` of `bar`
// (data delivered by st_async_cluster from any CTA of the cluster).
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, int spins) {
  const uint32_t a = smem_addr(bar);
  for (int i = 0; i < spins; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}

// Bounded wait for phase `parity` of `bar`.  Returns false if it gave up.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int spins) {
  const uint32_t a = smem_addr(bar);
  for (int i = 0; i < spins; ++i) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    if (ok) return true;
  }
  return false;
}

}  // namespace semicrf
