// ep_device.cuh -- device helpers shared by the kernels of libeplayout.so:
// status reporting, bounded waits, mbarrier + 1-D bulk-copy (TMA) wrappers,
// cache-hinted vector loads and stores, bf16 / e4m3 conversions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp8.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/eplayout.h"

namespace ep {

// ---------------------------------------------------------------------------
// status and bounded waits
// ---------------------------------------------------------------------------

__device__ __forceinline__ void report(int32_t* status, int bits) {
  if (status) atomicOr(status, bits);
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Give-up budget for every device-side wait in this library: a wait that has
// not been satisfied after this long reports EP_DEV_TIMEOUT and returns.
constexpr uint64_t kWaitBudgetNs = 2000000000ull;  // 2 s

// Forced give-ups (ep_debug_force_timeouts). A wait at a listed site
// (EP_WAIT_SITE_* bits) ignores its condition, as if nothing ever set it,
// and gives up after `budget_ns`; the kernel then takes the same give-up
// path a real stall would. Waits for copies already in flight (the drains
// before a CTA exits) are never forced. Each translation unit holds its own
// copy of this word (it is static), set for the current device by that
// unit's wait-debug setter; zero by default: nothing forced.
struct WaitDebug {
  uint32_t sites;
  uint32_t reserved;
  uint64_t budget_ns;
};
static __device__ WaitDebug g_wait_debug;

// Read once at kernel entry by the kernels that wait at `site`.
__device__ __forceinline__ bool wait_forced(uint32_t site) {
  return (*reinterpret_cast<volatile const uint32_t*>(&g_wait_debug.sites) & site) != 0u;
}

__device__ __forceinline__ uint64_t forced_budget_ns() {
  return *reinterpret_cast<volatile const uint64_t*>(&g_wait_debug.budget_ns);
}

// Spin until the forced budget runs out (the condition is never looked at).
__device__ __forceinline__ void forced_stall() {
  const uint64_t budget = forced_budget_ns();
  const uint64_t t0 = globaltimer_ns();
  while (globaltimer_ns() - t0 <= budget) {
  }
}

// Host side: set this translation unit's copy on the current device.
static inline cudaError_t set_wait_debug_here(uint32_t sites, uint64_t budget_ns) {
  const WaitDebug c{sites, 0u, budget_ns};
  return cudaMemcpyToSymbol(g_wait_debug, &c, sizeof(c));
}

// ---------------------------------------------------------------------------
// relaxed / acquire global accesses for inter-CTA flags
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t ld_relaxed_gpu(const uint32_t* p) {
  uint32_t v;
  asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void st_relaxed_gpu(uint32_t* p, uint32_t v) {
  asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ int32_t ld_acquire_gpu(const int32_t* p) {
  int32_t v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// ---------------------------------------------------------------------------
// 16-byte global accesses with cache hints
// ---------------------------------------------------------------------------

// Streaming read-only load: no L1 allocation (data is touched once).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

__device__ __forceinline__ void st_v4(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// 32-byte forms (256-bit global accesses, sm_100): p must be 32-byte aligned.
__device__ __forceinline__ void ld_stream_v8(const void* p, uint4& lo,
                                             uint4& hi) {
  asm volatile(
      "ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(lo.x), "=r"(lo.y), "=r"(lo.z), "=r"(lo.w), "=r"(hi.x),
        "=r"(hi.y), "=r"(hi.z), "=r"(hi.w)
      : "l"(p));
}

__device__ __forceinline__ void st_v8(void* p, uint4 lo, uint4 hi) {
  asm volatile("st.global.v8.u32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p),
               "r"(lo.x), "r"(lo.y), "r"(lo.z), "r"(lo.w), "r"(hi.x),
               "r"(hi.y), "r"(hi.z), "r"(hi.w)
               : "memory");
}

// Streaming store (evict-first): the receive buffer is far larger than L2.
__device__ __forceinline__ void st_cs_v4(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x),
               "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

// ---------------------------------------------------------------------------
// mbarrier and 1-D bulk async copies (sm_90+ TMA engine, no tensor map)
// ---------------------------------------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(count)
               : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar,
                                                      uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\t"
      "mbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
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
  return ok != 0;
}

// Wait for the phase with `parity` to complete; false after the budget.
// `forced`: a forced give-up (see WaitDebug), false after the forced budget.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar,
                                                  uint32_t parity,
                                                  bool forced = false) {
  if (forced) {
    forced_stall();
    return false;
  }
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if (globaltimer_ns() - t0 > kWaitBudgetNs) return false;
  }
}

// Bulk copy global -> shared, completion counted on `bar` (complete_tx).
// Both addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gmem_src,
                                         uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes "
      "[%0], [%1], %2, [%3];" ::"r"(smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Bulk copy shared -> global, tracked by the issuing thread's bulk groups.
__device__ __forceinline__ void bulk_s2g(void* gmem_dst, const void* smem_src,
                                         uint32_t bytes) {
  asm volatile(
      "cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(
          gmem_dst),
      "r"(smem_u32(smem_src)), "r"(bytes)
      : "memory");
}

__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}

// Wait until at most N committed groups still read their shared source.
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}

template <int N>
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}

// Programmatic dependent launch: a kernel launched with the programmatic
// stream-serialization attribute may start before the kernel ahead of it
// finishes; grid_dependency_wait blocks until that kernel has completed and
// its writes are visible (at once when there is no such dependency).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
// Lets the kernel queued behind this one start launching its CTAs.
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Named barrier `id` over `nthreads` threads that also ORs `pred` over them:
// every participant gets the same answer, so a decision taken on it (such
// as leaving a loop that holds this barrier) is the same in every warp.
__device__ __forceinline__ bool named_barrier_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(uint32_t(pred)), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0u;
}

// Make generic-proxy shared-memory writes visible to the async proxy.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------------------
// conversions
// ---------------------------------------------------------------------------

// bf16 pair packed in a 32-bit word -> two fp32 (exact).
__device__ __forceinline__ float bf16_lo(uint32_t w) {
  return __uint_as_float(w << 16);
}
__device__ __forceinline__ float bf16_hi(uint32_t w) {
  return __uint_as_float(w & 0xFFFF0000u);
}

// two fp32 -> packed bf16 pair, round to nearest even (lo in the low half).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

// two fp32 -> two e4m3 codes (lo in the low byte): round to nearest even,
// saturate finite values to +-448.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  return static_cast<uint32_t>(
      __nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

}  // namespace ep
