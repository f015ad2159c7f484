// ep_block.cuh -- CTA-wide scans and warp ballots shared by the layout
// kernels: exclusive scans of shared-memory arrays and the same-expert lane
// masks used to rank entries stably inside a warp.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace ep {
namespace {

// Barrier over the first THREADS threads of the CTA: __syncthreads() for
// BAR 0, else the named barrier BAR (THREADS a multiple of 32).
template <int THREADS, int BAR>
__device__ __forceinline__ void group_sync() {
  if constexpr (BAR == 0)
    __syncthreads();
  else
    asm volatile("bar.sync %0, %1;" ::"n"(BAR), "n"(THREADS) : "memory");
}

// In-place exclusive scan of buf[0..n) (shared memory) by threads
// [0, THREADS) of the CTA (all of it with BAR 0, else synchronised on the
// named barrier BAR); each thread owns a contiguous run. Returns the total.
template <int THREADS, int BAR = 0>
__device__ int32_t block_exclusive_scan(int32_t* buf, int n, int32_t* warp_tmp) {
  static_assert(THREADS / 32 <= 32, "one warp scans the warp sums");
  const int per = (n + THREADS - 1) / THREADS;
  const int lo = min(n, int(threadIdx.x) * per);
  const int hi = min(lo + per, n);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int32_t local = 0;
  for (int i = lo; i < hi; ++i) local += buf[i];
  int32_t x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_tmp[wid] = x;
  group_sync<THREADS, BAR>();
  if (wid == 0) {
    int32_t s = lane < THREADS / 32 ? warp_tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < THREADS / 32) warp_tmp[lane] = s;
  }
  group_sync<THREADS, BAR>();
  int32_t run = x - local + (wid > 0 ? warp_tmp[wid - 1] : 0);
  const int32_t total = warp_tmp[THREADS / 32 - 1];
  for (int i = lo; i < hi; ++i) {
    const int32_t v = buf[i];
    buf[i] = run;
    run += v;
  }
  group_sync<THREADS, BAR>();
  return total;
}

// Two in-place exclusive scans at once (a and b, n values each, shared
// memory); totals returned through ta / tb.
template <int THREADS>
__device__ void block_exclusive_scan2(int32_t* a, int32_t* b, int n,
                                      int32_t* warp_tmp /* [2*THREADS/32] */,
                                      int32_t& ta, int32_t& tb) {
  constexpr int W = THREADS / 32;
  const int per = (n + THREADS - 1) / THREADS;
  const int lo = min(n, int(threadIdx.x) * per);
  const int hi = min(lo + per, n);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int32_t la = 0, lb = 0;
  for (int i = lo; i < hi; ++i) {
    la += a[i];
    lb += b[i];
  }
  int32_t xa = la, xb = lb;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t ya = __shfl_up_sync(0xffffffffu, xa, o);
    const int32_t yb = __shfl_up_sync(0xffffffffu, xb, o);
    if (lane >= o) {
      xa += ya;
      xb += yb;
    }
  }
  if (lane == 31) {
    warp_tmp[wid] = xa;
    warp_tmp[W + wid] = xb;
  }
  __syncthreads();
  if (wid == 0) {
    int32_t sa = lane < W ? warp_tmp[lane] : 0;
    int32_t sb = lane < W ? warp_tmp[W + lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t ya = __shfl_up_sync(0xffffffffu, sa, o);
      const int32_t yb = __shfl_up_sync(0xffffffffu, sb, o);
      if (lane >= o) {
        sa += ya;
        sb += yb;
      }
    }
    if (lane < W) {
      warp_tmp[lane] = sa;
      warp_tmp[W + lane] = sb;
    }
  }
  __syncthreads();
  int32_t ra = xa - la + (wid > 0 ? warp_tmp[wid - 1] : 0);
  int32_t rb = xb - lb + (wid > 0 ? warp_tmp[W + wid - 1] : 0);
  ta = warp_tmp[W - 1];
  tb = warp_tmp[2 * W - 1];
  for (int i = lo; i < hi; ++i) {
    const int32_t va = a[i], vb = b[i];
    a[i] = ra;
    b[i] = rb;
    ra += va;
    rb += vb;
  }
  __syncthreads();
}

// Bits that tell the experts [0, E) apart.
__device__ __forceinline__ int expert_bits(int E) {
  return E <= 1 ? 0 : 32 - __clz(E - 1);
}

// Lanes of the warp whose key equals this lane's key (valid keys >= 0 only;
// the result is meaningless for invalid lanes). One ballot per key bit.
__device__ __forceinline__ unsigned same_key_lanes(int key, int nbits) {
  unsigned peers = __ballot_sync(0xffffffffu, key >= 0);
  for (int b = 0; b < nbits; ++b) {
    const bool bit = (key >> b) & 1;
    const unsigned bal = __ballot_sync(0xffffffffu, bit);
    peers &= bit ? bal : ~bal;
  }
  return peers;
}

}  // namespace
}  // namespace ep
