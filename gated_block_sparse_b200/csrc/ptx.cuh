// Inline-PTX wrappers for sm_100a: mbarriers, bulk (TMA) copies, fences.
// Every wait is bounded in time: it records an error code in a device flag
// and returns false, so a lost arrival cannot hang the GPU.
#pragma once

#include <stdint.h>

namespace sas {

// Device-side error word, read back by the host API after a kernel (0 = ok).
// Kernels OR in one of these bits when a bounded wait gives up.
enum : uint32_t { kErrWaitTimeout = 1u, kErrBadIndex = 2u };

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Makes mbarrier initialisation visible to the async proxy (TMA, tensor core).
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
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

__device__ __forceinline__ uint64_t global_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wall-clock bound of one wait. A try_wait may suspend the thread for a
// hardware-chosen time, so the bound is on time, not on the poll count.
constexpr uint64_t kWaitLimitNs = 200ull * 1000 * 1000;  // 200 ms

// Bounded wait for the phase with the given parity to complete, for phases
// completed by other threads' arrivals. Returns false if it gives up: after
// kWaitLimitNs, or at once when *err already carries kErrWaitTimeout (a wait
// elsewhere timed out: the launch is aborting, so no further wait may stall).
// A timeout sets kErrWaitTimeout in *err.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 15u) == 0) {
      if (err && (*reinterpret_cast<volatile uint32_t*>(err) & kErrWaitTimeout)) return false;
      if (global_ns() - t0 > kWaitLimitNs) break;
    }
  }
  if (err) atomicOr(err, kErrWaitTimeout);
  return false;
}

// Bounded wait for a phase completed by data this CTA has in flight (its own
// TMA or bulk copies, its tensor-core operations through tcgen05.commit).
// Bounded by kWaitLimitNs only: even when the launch is aborting it keeps
// waiting, so that no copy or MMA still writes into this CTA's shared memory
// or TMEM when the CTA frees them or exits. Every such operation is issued
// on the abort path too, so these waits end promptly there.
__device__ __forceinline__ bool mbar_wait_data(uint64_t* bar, uint32_t parity, uint32_t* err) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 15u) == 0 && global_ns() - t0 > kWaitLimitNs) break;
  }
  if (err) atomicOr(err, kErrWaitTimeout);
  return false;
}

// Asynchronous hint to bring `bytes` (multiple of 16, address 16-byte
// aligned) of global memory into L2; no completion to wait for.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Bulk copy of `bytes` (multiple of 16, both addresses 16-byte aligned) from
// global to this CTA's shared memory, completing on `bar`.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// ---------------------------------------------------------------- cluster
// Address of the same shared-memory location in CTA `rank` of the cluster
// (a shared::cluster address).
__device__ __forceinline__ uint32_t mapa(uint32_t local, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(local), "r"(rank));
  return r;
}

// Asynchronous stores into another CTA's shared memory (shared::cluster
// addresses from mapa); each completes `bytes` on the destination CTA's
// mbarrier `rbar` (also a shared::cluster address in that CTA).
__device__ __forceinline__ void st_async_u64(uint32_t raddr, unsigned long long v, uint32_t rbar) {
  asm volatile("st.async.shared::cluster.mbarrier::complete_tx::bytes.b64 [%0], %1, [%2];" ::"r"(
                   raddr),
               "l"(v), "r"(rbar)
               : "memory");
}
__device__ __forceinline__ void st_async_f32x2(uint32_t raddr, float a, float b, uint32_t rbar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v2.f32 [%0], {%1, %2}, [%3];" ::"r"(
          raddr),
      "f"(a), "f"(b), "r"(rbar)
      : "memory");
}
__device__ __forceinline__ void st_async_f32x4(uint32_t raddr, float a, float b, float c, float d,
                                               uint32_t rbar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.f32 [%0], {%1, %2, %3, %4}, "
      "[%5];" ::"r"(raddr),
      "f"(a), "f"(b), "f"(c), "f"(d), "r"(rbar)
      : "memory");
}

// try_wait with cluster-scope acquire: for barriers completed by other CTAs'
// st.async, so that their data is visible once the phase is seen complete.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait (as mbar_wait_data) on a barrier completed by other CTAs'
// remote stores into this CTA: it keeps waiting while the launch aborts, so
// the CTA does not leave while those stores may still land.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, uint32_t* err) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((i & 15u) == 0 && global_ns() - t0 > kWaitLimitNs) break;
  }
  if (err) atomicOr(err, kErrWaitTimeout);
  return false;
}

__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

}  // namespace sas
