// Device-side helpers shared by the sparse-decode kernels (sm_100a only).
//
// bf16 unpacking, order-preserving float keys, the bulk-copy (TMA engine) and mbarrier
// primitives as inline PTX, and the bounded waits every kernel uses.  No wait in this
// library spins without a limit: when a limit runs out the kernel records an error code
// in the caller's workspace and skips the rest of its work.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

namespace sas {

// Error codes recorded in the workspace error word (first one wins).
enum DeviceError : uint32_t {
  kDevOk = 0,
  kDevBadSeqlen = 1,     // seqlens[b] outside [0, capacity]
  kDevBadPage = 2,       // page id outside [0, num_pages)
  kDevBadIndex = 3,      // an index list entry outside [0, N_b)
  kDevKOverMax = 4,      // k[b] > k_max (clamped to k_max)
  kDevWaitTimeout = 5,   // a bounded mbarrier wait ran out
};

__device__ __forceinline__ void record_error(uint32_t* err, uint32_t code, uint32_t where) {
  if (err != nullptr) {
    if (atomicCAS(err, 0u, code) == 0u) err[1] = where;
  }
}

// ----------------------------------------------------------------------------- numbers
// Two bf16 values packed in a 32-bit word (element 2i in the low half) -> two floats.
__device__ __forceinline__ float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16hi(uint32_t w) { return __uint_as_float(w & 0xffff0000u); }

// Order-preserving map of an fp32 value to uint32: a > b  <=>  key(a) > key(b).
// -0.0 maps like +0.0, so equal floats give equal keys.
__device__ __forceinline__ uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  if ((u << 1) == 0u) return 0x80000000u;  // +0.0 and -0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }

// Size of the selection, min(k_b, N_b) clamped at 0, and whether it needs ranking (neither
// empty nor every position).  The ranking test is written on the inputs (0 < k < n), which
// means the same as (k_eff == 0 || k_eff == n) negated.  A build that used the latter form once
// returned every position at k = 64, n = 512; no race or uninitialised value was found in that
// code and the cause was not established.  The selection's parity tests cover n = 512 with k
// around 64 and around n.
struct SeqSelection {
  int k_eff;
  bool ranked;
};
__device__ __forceinline__ SeqSelection seq_selection(int kb, int n) {
  SeqSelection s;
  s.k_eff = max(0, min(kb, n));
  s.ranked = (kb > 0) && (n > 0) && (kb < n);
  return s;
}

// ----------------------------------------------------------------------------- PTX
// Programmatic dependent launch.  Every kernel of the library calls pdl_wait() before it touches
// any buffer an earlier kernel on the stream reads or writes, and pdl_trigger() right after, so
// the next kernel may start its independent prologue while this one runs.  Once a kernel has
// passed pdl_wait() every earlier kernel on the stream has completed (each of them waited for
// its own predecessor before triggering).  Both are no-ops for a launch without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

// Make barrier initialisation visible to the bulk-copy (async) proxy and to the cluster.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
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
  return ok != 0u;
}

// Each try_wait blocks for a hardware-defined slice of time before it gives up; this many
// attempts is far beyond any copy's latency (seconds) and still ends.
constexpr uint32_t kWaitLimit = 1u << 22;

__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  for (uint32_t i = 0; i < kWaitLimit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// Global -> this CTA's shared memory bulk copy on the TMA engine; completion is signalled
// on `bar` as transaction bytes.  dst/src 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// L2 eviction-priority policy for cache-hinted stores.
__device__ __forceinline__ uint64_t l2_evict_last() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// Hint the L2 to fetch a global range ahead of use (no shared memory involved).
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Streaming global loads that should not displace reused lines.
__device__ __forceinline__ uint4 ldg_stream128(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

}  // namespace sas
