// plan.cu -- the perfectly balanced plan, the redundant-expert weight
// prefetch, and two diagnostic kernels.
//
// "MoonEP核心功能深度剖析", section "1. 完美负载平衡": every rank receives
// exactly S*K rows, however skewed the routing, through a few redundant
// experts planned online and prefetched before the expert computation.
// Section "3. 智能内存管理" (图3): each expert projection is one contiguous
// buffer whose rows [0, E) are all experts and whose later rows are the
// local prefetch slots filled by prefetch_weight.
//
// Prefetch: k_prefetch_tma streams the used slots through bulk copies (one
// 16 KB chunk per unit); k_prefetch (16-byte vector copies) serves slot
// tables too large to compact in shared memory.
//
// Plan: the unpadded expert-grouped rows (experts in order) are cut into R
// chunks of T = S*K rows. Expert e holds rows [C_e, C_e + c_e); it meets
// chunks p = floor(C_e/T) .. q = floor((C_e + c_e - 1)/T). Chunk p reads
// weight row e; each later chunk d in (p, q] contains row d*T inside e, so e
// is the one expert entering chunk d from the previous chunk, and it takes
// slot 0 of rank d (weight row E + d*B). A segment's index inside chunk d is
// the number of non-empty experts between the chunk's first expert and e.
#include <algorithm>

#include "ep_device.cuh"
#include "ep_launch.h"

namespace ep {
namespace {

constexpr int kPlanThreads = 1024;

__device__ int32_t block_scan_excl_1024(int32_t* buf, int n, int32_t* warp_tmp) {
  // contiguous runs per thread, warp scan, scan of warp sums
  const int per = (n + kPlanThreads - 1) / kPlanThreads;
  const int lo = min(n, int(threadIdx.x) * per);
  const int hi = min(lo + per, n);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  int32_t local = 0;
  for (int i = lo; i < hi; ++i) local += buf[i];
  int32_t x = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int32_t yv = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += yv;
  }
  if (lane == 31) warp_tmp[wid] = x;
  __syncthreads();
  if (wid == 0) {
    int32_t s = warp_tmp[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t yv = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += yv;
    }
    warp_tmp[lane] = s;
  }
  __syncthreads();
  int32_t run = x - local + (wid > 0 ? warp_tmp[wid - 1] : 0);
  const int32_t total = warp_tmp[31];
  for (int i = lo; i < hi; ++i) {
    const int32_t v = buf[i];
    buf[i] = run;
    run += v;
  }
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(kPlanThreads)
    k_plan_balanced(const int32_t* __restrict__ counts, int R, int S, int K,
                    int E, int B, int32_t* __restrict__ plan_cu,
                    int32_t* __restrict__ plan_expert,
                    int32_t* __restrict__ plan_wrow,
                    int32_t* __restrict__ plan_nseg,
                    int32_t* __restrict__ slot_expert,
                    int32_t* __restrict__ status) {
  extern __shared__ int32_t sm[];
  int32_t* C = sm;              // [E] exclusive row prefix
  int32_t* nz = sm + E;         // [E] exclusive count of non-empty experts
  int32_t* first = sm + 2 * E;  // [R] expert holding row d*T
  __shared__ int32_t warp_tmp[32];
  const int tid = threadIdx.x;
  const int64_t T = int64_t(S) * K;

  for (int e = tid; e < E; e += kPlanThreads) {
    const int32_t c = __ldg(counts + e);
    C[e] = c;
    nz[e] = c > 0 ? 1 : 0;
  }
  for (int j = tid; j < R * B; j += kPlanThreads) slot_expert[j] = -1;
  __syncthreads();
  const int32_t total = block_scan_excl_1024(C, E, warp_tmp);
  block_scan_excl_1024(nz, E, warp_tmp);
  if (int64_t(total) != int64_t(R) * T) {
    if (tid == 0) report(status, EP_DEV_PLAN_TOTAL);
    return;
  }

  // the expert holding the first row of each chunk
  for (int e = tid; e < E; e += kPlanThreads) {
    const int64_t c = __ldg(counts + e);
    if (c == 0) continue;
    const int64_t a = C[e];
    for (int64_t d = (a + T - 1) / T; d * T < a + c && d < R; ++d) first[d] = e;
  }
  __syncthreads();

  for (int e = tid; e < E; e += kPlanThreads) {
    const int64_t c = __ldg(counts + e);
    if (c == 0) continue;
    const int64_t a = C[e], z = a + c;
    const int64_t p = a / T, q = (z - 1) / T;
    for (int64_t d = p; d <= q; ++d) {
      const int64_t lo = d * T;
      const int64_t s = max(a, lo) - lo;
      const int64_t f = min(z, lo + T) - lo;
      const int j = nz[e] - nz[first[d]];
      int32_t* cu = plan_cu + d * (E + 1);
      int32_t* ex = plan_expert + d * E;
      int32_t* wr = plan_wrow + d * E;
      cu[j] = int32_t(s);
      ex[j] = e;
      if (d == p) {
        wr[j] = e;
      } else if (B > 0) {
        slot_expert[d * B] = e;
        wr[j] = int32_t(E + d * B);
      } else {
        wr[j] = -1;
        report(status, EP_DEV_SLOTS);
      }
      if (f == T) {  // the segment that closes chunk d
        plan_nseg[d] = j + 1;
        for (int jj = j + 1; jj <= E; ++jj) cu[jj] = int32_t(T);
        for (int jj = j + 1; jj < E; ++jj) {
          ex[jj] = -1;
          wr[jj] = -1;
        }
      }
    }
  }
}

// Copy slot rows: units are (slot, projection, chunk of kCopyVec vectors).
constexpr int kCopyThreads = 256;
constexpr int64_t kCopyVec = 8192;  // 16-byte vectors per unit (128 KiB)

__global__ void __launch_bounds__(kCopyThreads)
    k_prefetch(const int32_t* __restrict__ slot_expert, int RB, int E,
               int64_t vecs, uint4* __restrict__ gate, uint4* __restrict__ up,
               uint4* __restrict__ down) {
  const int64_t nchunk = (vecs + kCopyVec - 1) / kCopyVec;
  const int64_t units = int64_t(RB) * 3 * nchunk;
  for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
    const int64_t slot = u / (3 * nchunk);
    const int64_t rem = u - slot * 3 * nchunk;
    const int proj = int(rem / nchunk);
    const int64_t ch = rem - int64_t(proj) * nchunk;
    const int32_t e = __ldg(slot_expert + slot);
    if (e < 0 || e >= E) continue;
    uint4* W = proj == 0 ? gate : (proj == 1 ? up : down);
    const uint4* src = W + int64_t(e) * vecs;
    uint4* dst = W + (int64_t(E) + slot) * vecs;
    const int64_t lo = ch * kCopyVec, hi = min(vecs, lo + kCopyVec);
    for (int64_t i = lo + threadIdx.x; i < hi; i += 4 * kCopyThreads) {
      uint4 v[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t ii = i + int64_t(j) * kCopyThreads;
        if (ii < hi) v[j] = ld_stream_v4(src + ii);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t ii = i + int64_t(j) * kCopyThreads;
        if (ii < hi) st_v4(dst + ii, v[j]);
      }
    }
  }
}

// TMA form of the slot copy: one-warp CTAs first compact the used slots into
// shared memory, then stream their (slot, projection, chunk) units through a
// ring of bulk loads and bulk stores (no data passes through registers).
constexpr int kTmaChunk = 16384;   // bytes per unit
constexpr int kTmaCopyStages = 4;
constexpr int kMaxSlotList = 1024;

__global__ void __launch_bounds__(32)
    k_prefetch_tma(const int32_t* __restrict__ slot_expert, int RB, int E,
                   int64_t row_bytes, uint8_t* __restrict__ gate,
                   uint8_t* __restrict__ up, uint8_t* __restrict__ down,
                   int32_t* __restrict__ status) {
  extern __shared__ __align__(128) uint8_t smb[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smb + kTmaCopyStages * kTmaChunk);
  int32_t* list = reinterpret_cast<int32_t*>(full + kTmaCopyStages);  // (slot, e)
  __shared__ int s_n;
  const int lane = threadIdx.x;
  // compact the used slots, in slot order
  int n = 0;
  for (int b = 0; b < RB; b += 32) {
    const int slot = b + lane;
    const int32_t e = slot < RB ? __ldg(slot_expert + slot) : -1;
    const bool used = e >= 0 && e < E;
    const unsigned m = __ballot_sync(0xffffffffu, used);
    if (used) {
      const int at = n + __popc(m & ((1u << lane) - 1u));
      list[2 * at] = slot;
      list[2 * at + 1] = e;
    }
    n += __popc(m);
  }
  if (lane == 0) s_n = n;
  __syncwarp();
  const int64_t nchunk = (row_bytes + kTmaChunk - 1) / kTmaChunk;
  const int64_t units = int64_t(s_n) * 3 * nchunk;
  const int64_t first = blockIdx.x, stride = gridDim.x;
  const int64_t n_mine = first < units ? (units - 1 - first) / stride + 1 : 0;
  if (lane != 0 || n_mine == 0) return;

  auto unit = [&](int64_t i, const uint8_t** src, uint8_t** dst, uint32_t* bytes) {
    const int64_t u = first + i * stride;
    const int64_t j = u / (3 * nchunk);
    const int64_t rem = u - j * 3 * nchunk;
    const int proj = int(rem / nchunk);
    const int64_t ch = rem - int64_t(proj) * nchunk;
    uint8_t* W = proj == 0 ? gate : (proj == 1 ? up : down);
    const int64_t off = ch * kTmaChunk;
    *bytes = uint32_t(min(int64_t(kTmaChunk), row_bytes - off));
    *src = W + int64_t(list[2 * j + 1]) * row_bytes + off;
    *dst = W + (int64_t(E) + list[2 * j]) * row_bytes + off;
  };
  const bool forced = wait_forced(EP_WAIT_SITE_PREFETCH);
  int64_t issued = 0;  // units whose load has been requested, in order
  for (int s = 0; s < kTmaCopyStages; ++s) mbar_init(&full[s], 1);
  fence_mbar_init();
  for (int64_t i = 0; i < kTmaCopyStages && i < n_mine; ++i, ++issued) {
    const uint8_t* src;
    uint8_t* dst;
    uint32_t bytes;
    unit(i, &src, &dst, &bytes);
    mbar_arrive_expect_tx(&full[i], bytes);
    bulk_g2s(smb + size_t(i) * kTmaChunk, src, bytes, &full[i]);
  }
  for (int64_t i = 0; i < n_mine; ++i) {
    const int s = int(i % kTmaCopyStages);
    const uint8_t* src;
    uint8_t* dst;
    uint32_t bytes;
    unit(i, &src, &dst, &bytes);
    if (!mbar_wait_bounded(&full[s], uint32_t(i / kTmaCopyStages) & 1u, forced)) {
      report(status, EP_DEV_TIMEOUT);
      break;
    }
    bulk_s2g(dst, smb + size_t(s) * kTmaChunk, bytes);
    bulk_commit();
    const int64_t nxt = i - 1 + kTmaCopyStages;
    if (i >= 1 && nxt < n_mine) {
      const int sp = int((i - 1) % kTmaCopyStages);
      bulk_wait_read<1>();
      unit(nxt, &src, &dst, &bytes);
      mbar_arrive_expect_tx(&full[sp], bytes);
      bulk_g2s(smb + size_t(sp) * kTmaChunk, src, bytes, &full[sp]);
      ++issued;
    }
  }
  // drain: the last load requested into each stage (still in flight after a
  // give-up), then every store
  for (int64_t i = 0; i < kTmaCopyStages && i < issued; ++i) {
    const int64_t last = issued - 1 - ((issued - 1 - i) % kTmaCopyStages);
    mbar_wait_bounded(&full[i], uint32_t(last / kTmaCopyStages) & 1u);
  }
  bulk_wait_all<0>();
}

// Slot-gradient reduce ("MoonEP核心功能深度剖析", "3. 智能内存管理", 图4: the
// gradient buffer mirrors the weight buffer and the prefetched copies'
// gradients are reduced into the owners' rows). Each CTA compacts the used
// slots in (d, b) order; the first slot of each expert heads its group.
// Units are (group, projection, chunk of float4 vectors): the expert's row
// plus its slots' rows, added in (d, b) order in fp32, as the definition
// states; slot rows are left as they are.
constexpr int kRedThreads = 256;
constexpr int64_t kRedVec = 4096;  // float4 vectors per unit (64 KB)

__global__ void __launch_bounds__(kRedThreads)
    k_reduce_slot_grads(const int32_t* __restrict__ slot_expert, int RB, int E,
                        int64_t vecs, float4* __restrict__ g0,
                        float4* __restrict__ g1, float4* __restrict__ g2) {
  __shared__ int s_slot[kMaxSlotList], s_exp[kMaxSlotList], s_head[kMaxSlotList];
  __shared__ int s_n, s_nh;
  const int tid = threadIdx.x, lane = tid & 31;
  if (tid < 32) {
    int n = 0;
    for (int b = 0; b < RB; b += 32) {
      const int slot = b + lane;
      const int32_t e = slot < RB ? __ldg(slot_expert + slot) : -1;
      const bool used = e >= 0 && e < E;
      const unsigned m = __ballot_sync(0xffffffffu, used);
      if (used) {
        const int at = n + __popc(m & ((1u << lane) - 1u));
        s_slot[at] = slot;
        s_exp[at] = e;
      }
      n += __popc(m);
    }
    if (lane == 0) s_n = n;
  }
  __syncthreads();
  if (tid == 0) {
    int nh = 0;
    for (int j = 0; j < s_n; ++j) {
      bool first = true;
      for (int jj = 0; jj < j && first; ++jj) first = s_exp[jj] != s_exp[j];
      if (first) s_head[nh++] = j;
    }
    s_nh = nh;
  }
  __syncthreads();
  const int n = s_n;
  const int64_t nchunk = (vecs + kRedVec - 1) / kRedVec;
  const int64_t units = int64_t(s_nh) * 3 * nchunk;
  for (int64_t u = blockIdx.x; u < units; u += gridDim.x) {
    const int64_t f = u / (3 * nchunk);
    const int64_t rem = u - f * 3 * nchunk;
    const int proj = int(rem / nchunk);
    const int64_t ch = rem - int64_t(proj) * nchunk;
    const int j0 = s_head[f];
    const int e = s_exp[j0];
    float4* G = proj == 0 ? g0 : (proj == 1 ? g1 : g2);
    const int64_t lo = ch * kRedVec, hi = min(vecs, lo + kRedVec);
    // four vectors per thread per round: their loads go out together
    for (int64_t vb = lo + tid; vb < hi; vb += 4 * kRedThreads) {
      float4 acc[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int64_t v = vb + int64_t(q) * kRedThreads;
        if (v < hi) acc[q] = G[int64_t(e) * vecs + v];
      }
      for (int j = j0; j < n; ++j) {
        if (s_exp[j] != e) continue;
        float4 x[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int64_t v = vb + int64_t(q) * kRedThreads;
          if (v < hi) x[q] = G[(int64_t(E) + s_slot[j]) * vecs + v];
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int64_t v = vb + int64_t(q) * kRedThreads;
          if (v < hi) {
            acc[q].x = acc[q].x + x[q].x;
            acc[q].y = acc[q].y + x[q].y;
            acc[q].z = acc[q].z + x[q].z;
            acc[q].w = acc[q].w + x[q].w;
          }
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int64_t v = vb + int64_t(q) * kRedThreads;
        if (v < hi) G[int64_t(e) * vecs + v] = acc[q];
      }
    }
  }
}

__global__ void k_debug_e4m3(const float* __restrict__ x, uint8_t* __restrict__ out,
                             int64_t n) {
  const int64_t pairs = (n + 1) / 2;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < pairs;
       i += int64_t(gridDim.x) * blockDim.x) {
    const float lo = x[2 * i];
    const float hi = (2 * i + 1 < n) ? x[2 * i + 1] : 0.0f;
    const uint32_t q = e4m3x2(lo, hi);
    out[2 * i] = uint8_t(q & 0xFFu);
    if (2 * i + 1 < n) out[2 * i + 1] = uint8_t(q >> 8);
  }
}

__global__ void k_debug_wait(const int32_t* flag, int64_t max_polls,
                             int32_t* status) {
  if (threadIdx.x != 0 || blockIdx.x != 0) return;
  for (int64_t i = 0; i < max_polls; ++i) {
    if (ld_acquire_gpu(flag) != 0) return;
    __nanosleep(100);
  }
  report(status, EP_DEV_TIMEOUT);
}

// Streaming read of `bytes` bytes (a multiple of 32, 32-byte aligned) with
// 256-bit loads from every thread; the XOR of all 32-bit words goes to
// *sink so that nothing can be skipped.
__global__ void __launch_bounds__(512)
    k_debug_stream_read(const uint8_t* __restrict__ src, int64_t bytes,
                        uint32_t* __restrict__ sink) {
  uint32_t acc = 0;
  for (int64_t i = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) * 32; i < bytes;
       i += int64_t(gridDim.x) * blockDim.x * 32) {
    uint4 lo, hi;
    ld_stream_v8(src + i, lo, hi);
    acc ^= lo.x ^ lo.y ^ lo.z ^ lo.w ^ hi.x ^ hi.y ^ hi.z ^ hi.w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc ^= __shfl_xor_sync(0xffffffffu, acc, o);
  if ((threadIdx.x & 31) == 0) atomicXor(sink, acc);
}

}  // namespace

cudaError_t launch_plan_balanced(const int32_t* counts, int R, int S, int K,
                                 int E, int B, int32_t* plan_cu,
                                 int32_t* plan_expert, int32_t* plan_wrow,
                                 int32_t* plan_nseg, int32_t* slot_expert,
                                 int32_t* status, cudaStream_t stream) {
  const size_t smem = (size_t(2) * E + R) * sizeof(int32_t);
  if (smem > 48 * 1024) {
    cudaError_t err = cudaFuncSetAttribute(
        k_plan_balanced, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err != cudaSuccess) return err;
  }
  k_plan_balanced<<<1, kPlanThreads, smem, stream>>>(counts, R, S, K, E, B,
                                                     plan_cu, plan_expert,
                                                     plan_wrow, plan_nseg,
                                                     slot_expert, status);
  return cudaGetLastError();
}

cudaError_t set_wait_debug_plan(uint32_t sites, uint64_t budget_ns) {
  return set_wait_debug_here(sites, budget_ns);
}

cudaError_t launch_prefetch(const int32_t* slot_expert, int R, int E, int B,
                            int64_t elems, void* gate, void* up, void* down,
                            int num_sms, int32_t* status, cudaStream_t stream) {
  const int64_t RB = int64_t(R) * B;
  if (RB == 0 || elems == 0) return cudaSuccess;
  if (RB <= kMaxSlotList) {
    const size_t smem = size_t(kTmaCopyStages) * kTmaChunk +
                        kTmaCopyStages * sizeof(uint64_t) + 2 * kMaxSlotList * 4;
    cudaError_t err = cudaFuncSetAttribute(
        k_prefetch_tma, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (err != cudaSuccess) return err;
    int per_sm = 0;
    err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_prefetch_tma, 32,
                                                        smem);
    if (err != cudaSuccess) return err;
    const int grid = num_sms * std::max(1, per_sm);
    k_prefetch_tma<<<grid, 32, smem, stream>>>(
        slot_expert, int(RB), E, elems * 2, static_cast<uint8_t*>(gate),
        static_cast<uint8_t*>(up), static_cast<uint8_t*>(down), status);
    return cudaGetLastError();
  }
  const int64_t vecs = elems * 2 / 16;
  const int64_t nchunk = (vecs + kCopyVec - 1) / kCopyVec;
  const int64_t units = RB * 3 * nchunk;
  int per_sm = 0;
  cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
      &per_sm, k_prefetch, kCopyThreads, 0);
  if (err != cudaSuccess) return err;
  const int64_t grid = std::max<int64_t>(
      1, std::min<int64_t>(units, int64_t(num_sms) * std::max(1, per_sm)));
  k_prefetch<<<int(grid), kCopyThreads, 0, stream>>>(
      slot_expert, int(RB), E, vecs, static_cast<uint4*>(gate),
      static_cast<uint4*>(up), static_cast<uint4*>(down));
  return cudaGetLastError();
}

cudaError_t launch_reduce_slot_grads(const int32_t* slot_expert, int R, int E,
                                     int B, int64_t elems, float* g0, float* g1,
                                     float* g2, int num_sms,
                                     cudaStream_t stream) {
  const int64_t RB = int64_t(R) * B;
  if (RB == 0 || elems == 0) return cudaSuccess;
  const int64_t vecs = elems / 4;
  const int64_t nchunk = (vecs + kRedVec - 1) / kRedVec;
  const int64_t grid = std::max<int64_t>(
      1, std::min<int64_t>(RB * 3 * nchunk, int64_t(num_sms) * 8));
  k_reduce_slot_grads<<<int(grid), kRedThreads, 0, stream>>>(
      slot_expert, int(RB), E, vecs, reinterpret_cast<float4*>(g0),
      reinterpret_cast<float4*>(g1), reinterpret_cast<float4*>(g2));
  return cudaGetLastError();
}

cudaError_t launch_debug_e4m3(const float* x, uint8_t* out, int64_t n,
                             cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const int64_t pairs = (n + 1) / 2;
  const int grid = int(std::min<int64_t>((pairs + 255) / 256, 148 * 16));
  k_debug_e4m3<<<grid, 256, 0, stream>>>(x, out, n);
  return cudaGetLastError();
}

cudaError_t launch_debug_wait(const int32_t* flag, int64_t max_polls,
                              int32_t* status, cudaStream_t stream) {
  k_debug_wait<<<1, 32, 0, stream>>>(flag, max_polls, status);
  return cudaGetLastError();
}

cudaError_t launch_debug_stream_read(const void* src, int64_t bytes,
                                     uint32_t* sink, cudaStream_t stream) {
  if (bytes == 0) return cudaSuccess;
  // four 512-thread CTAs per SM: the fastest of 1, 2 and 4 in a probe
  const int64_t grid = std::max<int64_t>(
      1, std::min<int64_t>(int64_t(device_sm_count()) * 4, (bytes + 16383) / 16384));
  k_debug_stream_read<<<int(grid), 512, 0, stream>>>(
      static_cast<const uint8_t*>(src), bytes, sink);
  return cudaGetLastError();
}

}  // namespace ep
