// layout.cu -- dispatch steps 1-3: per-expert histogram, padded expert
// offsets, and stable expert-grouped positions.
//
// "MoonEP核心功能深度剖析", section "2. 高效通信机制": every token is written
// straight to its final expert-grouped position, so the position of entry
// (t,k) must be known before the copy: expert base (padded, section
// "快速上手" token_padding) plus the number of earlier entries, in (t,k)
// order, routed to the same expert.
//
// Two kernels after one small memset:
//   k_histogram       warp-aggregated (match_any + popc) shared-memory counts,
//                     one global add per (CTA, expert); the last CTA to finish
//                     pads the totals and scans them into expert_offsets.
//   k_scan_positions  single-pass multi-bucket scan with decoupled look-back
//                     (Merrill & Garland, "Single-pass Parallel Prefix Scan with
//                     Decoupled Look-back", 2016; one look-back lane per expert
//                     as in Adinets & Merrill, "Onesweep", 2022): each tile
//                     ranks its entries per expert in (t,k) order, publishes
//                     its per-expert aggregate, then reads its predecessors'.
#include <algorithm>

#include "ep_device.cuh"
#include "ep_launch.h"

namespace ep {
namespace {

constexpr int kHistThreads = 512;
constexpr int kHistUnroll = 4;

constexpr int kScanThreads = 512;
constexpr int kScanWarps = kScanThreads / 32;
constexpr int kScanItems = kScanTile / kScanThreads;  // entries per lane
constexpr int kWarpItems = 32 * kScanItems;           // consecutive per warp
constexpr int kLookbackWindow = 16;
static_assert(kScanItems * kScanThreads == kScanTile, "tile shape");

// Look-back descriptor: 2 flag bits over a 30-bit count (N*K < 2^30).
constexpr uint32_t kFlagAggregate = 1u << 30;
constexpr uint32_t kFlagInclusive = 2u << 30;
constexpr uint32_t kValueMask = (1u << 30) - 1u;

struct WsHeader {
  uint32_t hist_done;    // CTAs of k_histogram that have finished
  uint32_t tile_ticket;  // next tile id of k_scan_positions
  uint32_t reserved[62];
};
static_assert(sizeof(WsHeader) == 256, "header size");

constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// In-place exclusive scan of buf[0..n) (shared memory) by a CTA of THREADS
// threads; each thread owns a contiguous run. Returns the total.
template <int THREADS>
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
  __syncthreads();
  if (wid == 0) {
    int32_t s = lane < THREADS / 32 ? warp_tmp[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int32_t y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    if (lane < THREADS / 32) warp_tmp[lane] = s;
  }
  __syncthreads();
  int32_t run = x - local + (wid > 0 ? warp_tmp[wid - 1] : 0);
  const int32_t total = warp_tmp[THREADS / 32 - 1];
  for (int i = lo; i < hi; ++i) {
    const int32_t v = buf[i];
    buf[i] = run;
    run += v;
  }
  __syncthreads();
  return total;
}

__global__ void __launch_bounds__(kHistThreads)
    k_histogram(const int32_t* __restrict__ topk, int64_t M, int E, int pad,
                WsHeader* __restrict__ hdr, int32_t* __restrict__ acc,
                uint32_t* __restrict__ desc, int64_t desc_words,
                int32_t* __restrict__ tokens_per_expert,
                int32_t* __restrict__ expert_offsets,
                int32_t* __restrict__ status) {
  __shared__ int32_t s_hist[kMaxExperts];
  __shared__ int32_t s_warp[kHistThreads / 32];
  __shared__ int s_last;
  const int tid = threadIdx.x, lane = tid & 31;
  for (int e = tid; e < E; e += kHistThreads) s_hist[e] = 0;
  __syncthreads();

  bool bad = false;
  const int64_t per_iter = int64_t(kHistThreads) * kHistUnroll;
  // `base` is uniform over the CTA, so every lane takes part in match_any.
  for (int64_t base = int64_t(blockIdx.x) * per_iter; base < M;
       base += int64_t(gridDim.x) * per_iter) {
    int key[kHistUnroll];
#pragma unroll
    for (int u = 0; u < kHistUnroll; ++u) {
      const int64_t i = base + int64_t(u) * kHistThreads + tid;
      key[u] = -2;  // past the end
      if (i < M) {
        const int e = __ldg(topk + i);
        if (unsigned(e) < unsigned(E)) {
          key[u] = e;
        } else {
          key[u] = -1;
          bad = true;
        }
      }
    }
#pragma unroll
    for (int u = 0; u < kHistUnroll; ++u) {
      const unsigned peers = __match_any_sync(0xffffffffu, key[u]);
      if (key[u] >= 0 && lane == __ffs(peers) - 1)
        atomicAdd(&s_hist[key[u]], __popc(peers));
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) report(status, EP_DEV_BAD_EXPERT);

  // Clear the look-back descriptors of the scan that follows on the stream.
  for (int64_t j = int64_t(blockIdx.x) * kHistThreads + tid; j < desc_words;
       j += int64_t(gridDim.x) * kHistThreads)
    desc[j] = 0u;

  __syncthreads();
  for (int e = tid; e < E; e += kHistThreads)
    if (s_hist[e]) atomicAdd(&acc[e], s_hist[e]);
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = (atomicAdd(&hdr->hist_done, 1u) == gridDim.x - 1);
  __syncthreads();
  if (!s_last) return;
  __threadfence();

  // Last CTA: totals, padded to multiples of token_padding, exclusive scan.
  for (int e = tid; e < E; e += kHistThreads) {
    const int32_t c = __ldcg(acc + e);
    tokens_per_expert[e] = c;
    s_hist[e] = int32_t(((int64_t(c) + pad - 1) / pad) * pad);
  }
  __syncthreads();
  const int32_t total = block_exclusive_scan<kHistThreads>(s_hist, E, s_warp);
  for (int e = tid; e < E; e += kHistThreads) expert_offsets[e] = s_hist[e];
  if (tid == 0) expert_offsets[E] = total;
}

// Sum of expert e's counts over tiles [0, tile): walk the predecessors'
// descriptors from the nearest one back, kLookbackWindow loads in flight,
// until an inclusive prefix is found. Bounded: reports EP_DEV_TIMEOUT and
// returns what it has after kWaitBudgetNs without progress.
__device__ __forceinline__ uint32_t lookback(const uint32_t* desc, int E, int e,
                                             int tile, int32_t* status) {
  uint32_t excl = 0;
  int j = tile - 1;
  uint64_t t0 = 0;
  bool waiting = false;
  while (j >= 0) {
    const int lo = max(0, j - kLookbackWindow + 1);
    uint32_t v[kLookbackWindow];
#pragma unroll
    for (int q = 0; q < kLookbackWindow; ++q)
      v[q] = (j - q >= lo) ? ld_relaxed_gpu(desc + int64_t(j - q) * E + e) : 0u;
    int q = 0;
    for (; q < kLookbackWindow && j - q >= lo; ++q) {
      const uint32_t flag = v[q] & ~kValueMask;
      if (flag == 0u) break;  // not published yet
      excl += v[q] & kValueMask;
      if (flag == kFlagInclusive) return excl;
    }
    const bool consumed_window = (j - q < lo);
    j -= q;
    if (!consumed_window) {
      if (!waiting) {
        waiting = true;
        t0 = globaltimer_ns();
      } else if (globaltimer_ns() - t0 > kWaitBudgetNs) {
        report(status, EP_DEV_TIMEOUT);
        return excl;
      }
      __nanosleep(32);
    } else {
      waiting = false;
    }
  }
  return excl;
}

__global__ void __launch_bounds__(kScanThreads)
    k_scan_positions(const int32_t* __restrict__ topk, int64_t M, int E,
                     const int32_t* __restrict__ counts,
                     const int32_t* __restrict__ offsets,
                     WsHeader* __restrict__ hdr, uint32_t* __restrict__ desc,
                     int num_tiles, int32_t* __restrict__ pos,
                     int32_t* __restrict__ row_src, int64_t cap,
                     int32_t* __restrict__ status) {
  extern __shared__ int32_t smem[];
  int32_t* whist = smem;                    // [kScanWarps][E]
  int32_t* tbase = smem + kScanWarps * E;   // [E]
  __shared__ int s_tile;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  // Tiles are claimed in launch order of arrival, so every predecessor of a
  // tile belongs to a CTA that is already running: the look-back progresses.
  if (tid == 0) s_tile = int(atomicAdd(&hdr->tile_ticket, 1u));
  for (int j = tid; j < kScanWarps * E; j += kScanThreads) whist[j] = 0;
  __syncthreads();
  const int tile = s_tile;
  const int64_t wbase = int64_t(tile) * kScanTile + int64_t(warp) * kWarpItems;

  int key[kScanItems];
  int rank[kScanItems];
#pragma unroll
  for (int r = 0; r < kScanItems; ++r) {
    const int64_t i = wbase + r * 32 + lane;
    key[r] = -2;
    if (i < M) {
      const int e = __ldg(topk + i);
      key[r] = (unsigned(e) < unsigned(E)) ? e : -1;
    }
  }
  // Rank inside the warp, in entry order: 32 entries per round.
  int32_t* my = whist + warp * E;
#pragma unroll
  for (int r = 0; r < kScanItems; ++r) {
    const int k = key[r];
    const unsigned peers = __match_any_sync(0xffffffffu, k);
    int cur = 0;
    if (k >= 0) cur = my[k];
    __syncwarp();
    if (k >= 0 && lane == __ffs(peers) - 1) my[k] = cur + __popc(peers);
    __syncwarp();
    rank[r] = cur + __popc(peers & ((1u << lane) - 1u));
  }
  __syncthreads();

  // Per expert: exclusive scan over the warps (warps hold consecutive
  // entries), the tile's total, and its descriptor.
  for (int e = tid; e < E; e += kScanThreads) {
    int32_t run = 0;
    for (int w = 0; w < kScanWarps; ++w) {
      const int32_t c = whist[w * E + e];
      whist[w * E + e] = run;
      run += c;
    }
    tbase[e] = run;
    st_relaxed_gpu(desc + int64_t(tile) * E + e,
                   (tile == 0 ? kFlagInclusive : kFlagAggregate) | uint32_t(run));
  }
  for (int e = tid; e < E; e += kScanThreads) {
    uint32_t excl = 0;
    if (tile > 0) {
      excl = lookback(desc, E, e, tile, status);
      st_relaxed_gpu(desc + int64_t(tile) * E + e,
                     kFlagInclusive | ((excl + uint32_t(tbase[e])) & kValueMask));
    }
    tbase[e] = __ldg(offsets + e) + int32_t(excl);
  }
  __syncthreads();

#pragma unroll
  for (int r = 0; r < kScanItems; ++r) {
    const int64_t i = wbase + r * 32 + lane;
    const int k = key[r];
    if (k == -2) continue;
    if (k < 0) {
      pos[i] = -1;
      continue;
    }
    const int64_t p = int64_t(tbase[k]) + my[k] + rank[r];
    pos[i] = int32_t(p);
    if (p < cap)
      row_src[p] = int32_t(i);
    else
      report(status, EP_DEV_CAPACITY);
  }

  // Padding rows of the experts this CTA covers: row_src = -1.
  for (int e = tile; e < E; e += num_tiles) {
    const int64_t lo = int64_t(__ldg(offsets + e)) + __ldg(counts + e);
    const int64_t hi = min(int64_t(__ldg(offsets + e + 1)), cap);
    for (int64_t r = lo + tid; r < hi; r += kScanThreads) row_src[r] = -1;
  }
}

}  // namespace

size_t layout_workspace_bytes(int64_t entries, int E) {
  const int64_t tiles = (entries + kScanTile - 1) / kScanTile;
  return sizeof(WsHeader) + align256(size_t(E) * 4) + size_t(tiles) * E * 4;
}

cudaError_t launch_layout(const int32_t* topk, int64_t entries, int E, int pad,
                          int32_t* tokens_per_expert, int32_t* expert_offsets,
                          int32_t* pos, int32_t* row_src, int64_t cap,
                          void* workspace, int32_t* status, int num_sms,
                          cudaStream_t stream) {
  char* ws = static_cast<char*>(workspace);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
  int32_t* acc = reinterpret_cast<int32_t*>(ws + sizeof(WsHeader));
  uint32_t* desc =
      reinterpret_cast<uint32_t*>(ws + sizeof(WsHeader) + align256(size_t(E) * 4));
  const int64_t tiles = (entries + kScanTile - 1) / kScanTile;

  cudaError_t err = cudaMemsetAsync(
      ws, 0, sizeof(WsHeader) + align256(size_t(E) * 4), stream);
  if (err != cudaSuccess) return err;

  const int64_t want = (entries + int64_t(kHistThreads) * kHistUnroll - 1) /
                       (int64_t(kHistThreads) * kHistUnroll);
  const int hist_blocks =
      int(std::max<int64_t>(1, std::min<int64_t>(want, int64_t(num_sms) * 2)));
  k_histogram<<<hist_blocks, kHistThreads, 0, stream>>>(
      topk, entries, E, pad, hdr, acc, desc, tiles * E, tokens_per_expert,
      expert_offsets, status);
  err = cudaGetLastError();
  if (err != cudaSuccess || tiles == 0) return err;

  const size_t smem = size_t(kScanWarps + 1) * E * sizeof(int32_t);
  if (smem > 48 * 1024) {
    err = cudaFuncSetAttribute(k_scan_positions,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               int(smem));
    if (err != cudaSuccess) return err;
  }
  k_scan_positions<<<int(tiles), kScanThreads, smem, stream>>>(
      topk, entries, E, tokens_per_expert, expert_offsets, hdr, desc, int(tiles),
      pos, row_src, cap, status);
  return cudaGetLastError();
}

}  // namespace ep
