// layout.cu -- dispatch steps 1-3: per-expert histogram, padded expert
// offsets, and stable expert-grouped positions.
//
// "MoonEP核心功能深度剖析", section "2. 高效通信机制": every token is written
// straight to its final expert-grouped position, so the position of entry
// (t,k) must be known before the copy: expert base (padded, section
// "快速上手" token_padding) plus the number of earlier entries, in (t,k)
// order, routed to the same expert.
//
// The entries are cut into tiles of kScanTile. A tile ranks each entry among
// the earlier entries of its tile with the same expert (stable: warps hold
// consecutive entries, lanes in order), publishes its per-expert counts, and
// takes the counts of all earlier tiles with a single-pass decoupled
// look-back (Merrill & Garland, "Single-pass Parallel Prefix Scan with
// Decoupled Look-back", 2016; one look-back lane per expert, as in the
// multi-bucket scan of Adinets & Merrill, "Onesweep", 2022).
//
// Inside a warp, the lanes holding the same expert are found with one ballot
// per bit of the expert id (log2 E ballots): each lane keeps the lanes that
// agree with it on every bit. The cost is the same whatever the keys, unlike
// a hardware match whose cost grows with the number of distinct keys.
//
// Two paths here (small batches, N*K <= 32768, take layout_small.cu instead):
//   fused      (tiles fit co-resident) one cooperative launch: every tile
//              publishes its per-expert counts once; once all have, each
//              tile sums them (reduce-then-scan: the counts of the tiles
//              before it, and the totals), scans the padded totals into the
//              expert offsets itself, and writes final positions from the
//              ranks kept in registers. No look-back chain.
//   two-kernel (any size) k_histogram counts with warp-aggregated shared-memory
//              atomics and its last CTA writes the offsets; k_scan_positions
//              then ranks, looks back and writes positions, tile ids claimed
//              in arrival order.
#include <algorithm>

#include "ep_block.cuh"
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
constexpr int kLookbackWindow = 32;  // predecessors per thread per round
constexpr int kLookbackPair = 2;     // threads sharing one expert's look-back
static_assert(kScanItems * kScanThreads == kScanTile, "tile shape");
static_assert(kWarpItems < (1 << 16), "rank packs into 16 bits");
static_assert(kScanTile <= 4096 && kMaxExperts <= (1 << 20), "sort key packs");

// Look-back descriptor: 2 flag bits over a 30-bit count (N*K < 2^30).
constexpr uint32_t kFlagAggregate = 1u << 30;
constexpr uint32_t kFlagInclusive = 2u << 30;
constexpr uint32_t kValueMask = (1u << 30) - 1u;

struct WsHeader {
  uint32_t hist_done;      // CTAs of k_histogram that have finished
  uint32_t tile_ticket;    // next tile id of k_scan_positions
  uint32_t reserved[62];
};
static_assert(sizeof(WsHeader) == 256, "header size");

constexpr size_t align256(size_t x) { return (x + 255) & ~size_t(255); }


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
  const int nbits = expert_bits(E);
  for (int e = tid; e < E; e += kHistThreads) s_hist[e] = 0;
  __syncthreads();

  bool bad = false;
  const int64_t per_iter = int64_t(kHistThreads) * kHistUnroll;
  // `base` is uniform over the CTA, so every lane takes part in the ballots.
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
      const unsigned peers = same_key_lanes(key[u], nbits);
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

// Exclusive prefix of one expert over the tiles before `tile`, found by two
// threads of a warp (h = 0, 1) that look back together. Each round, thread
// h loads the descriptors of kLookbackWindow predecessors, h = 0 the nearest
// ones. Each walks its window from the near end, summing until it meets a
// descriptor that is not yet published or an inclusive prefix (which ends
// the look-back). The pair then merges its two walks with shuffles, so
// 2 * kLookbackWindow predecessors are covered per round of loads. Every
// lane of the warp calls this (shuffles); `active` lanes own an expert.
// Bounded: reports EP_DEV_TIMEOUT and returns what it has after
// kWaitBudgetNs without progress. `forced`: every descriptor reads as not
// yet published, so the look-back gives up after the forced budget.
__device__ __forceinline__ uint32_t lookback_pair(const uint32_t* desc, int E,
                                                  int e, bool active, int h,
                                                  int tile, int32_t* status,
                                                  bool forced) {
  const uint64_t budget = forced ? forced_budget_ns() : kWaitBudgetNs;
  uint32_t excl = 0;
  int j = tile - 1;               // nearest predecessor not yet consumed
  bool done = !active || j < 0;
  uint64_t t0 = 0;
  bool waiting = false;
  while (__any_sync(0xffffffffu, !done)) {
    const int hi = j - h * kLookbackWindow;   // nearest of my window
    uint32_t v[kLookbackWindow];
#pragma unroll
    for (int q = 0; q < kLookbackWindow; ++q)
      v[q] = (!done && !forced && hi - q >= 0)
                 ? ld_relaxed_gpu(desc + int64_t(hi - q) * E + e)
                 : 0u;
    uint32_t sum = 0;
    int used = 0;
    bool stop = false, found = false;
#pragma unroll
    for (int q = 0; q < kLookbackWindow; ++q) {
      if (!stop && hi - q >= 0) {
        const uint32_t flag = v[q] & ~kValueMask;
        if (flag == 0u) {
          stop = true;  // not published yet
        } else {
          sum += v[q] & kValueMask;
          ++used;
          if (flag == kFlagInclusive) stop = found = true;
        }
      }
    }
    // the partner's walk (lanes 2m and 2m+1 share an expert)
    const uint32_t sum_o = __shfl_xor_sync(0xffffffffu, sum, 1);
    const int used_o = __shfl_xor_sync(0xffffffffu, used, 1);
    const bool found_o = __shfl_xor_sync(0xffffffffu, found, 1);
    const uint32_t s0 = h ? sum_o : sum, s1 = h ? sum : sum_o;
    const int u0 = h ? used_o : used, u1 = h ? used : used_o;
    const bool f0 = h ? found_o : found, f1 = h ? found : found_o;
    if (!done) {
      bool progress = true;
      if (f0) {
        excl += s0;
        done = true;
      } else if (u0 < min(kLookbackWindow, j + 1)) {
        excl += s0;  // window 0 stopped at an unpublished descriptor
        j -= u0;
        progress = u0 > 0;
      } else {
        excl += s0 + s1;
        j -= u0 + u1;
        if (f1) done = true;
        else if (u1 < min(kLookbackWindow, j + u1 + 1)) progress = (u0 + u1) > 0;
      }
      if (!done && j < 0) done = true;
      if (!done) {
        if (progress) {
          waiting = false;
        } else if (!waiting) {
          waiting = true;
          t0 = globaltimer_ns();
        } else if (globaltimer_ns() - t0 > budget) {
          report(status, EP_DEV_TIMEOUT);
          done = true;
        }
      }
    }
  }
  return excl;
}

// ---- the phases of one tile, shared by both scan kernels -----------------

// key/rank of one entry packed in 32 bits: (key + 2) << 16 | rank, key = -2
// past the end, -1 invalid id.
__device__ __forceinline__ int packed_key(uint32_t v) { return int(v >> 16) - 2; }
__device__ __forceinline__ int packed_rank(uint32_t v) { return int(v & 0xFFFFu); }

// Loads the tile's entries (warp w holds the consecutive entries
// [w*kWarpItems, (w+1)*kWarpItems) of the tile, 32 per round) and ranks each
// entry among the earlier entries of its warp with the same expert. Leaves
// per-warp expert counts in my[e]. Returns whether an invalid id was seen.
__device__ __forceinline__ bool rank_in_warps(const int32_t* __restrict__ topk,
                                              int64_t M, int E, int64_t wbase,
                                              int32_t* my,
                                              uint32_t (&kr)[kScanItems]) {
  const int lane = threadIdx.x & 31;
  const int nbits = expert_bits(E);
  int key[kScanItems];
#pragma unroll
  for (int r = 0; r < kScanItems; ++r) {
    const int64_t i = wbase + r * 32 + lane;
    key[r] = -2;
    if (i < M) {
      const int e = __ldg(topk + i);
      key[r] = (unsigned(e) < unsigned(E)) ? e : -1;
    }
  }
  // same-key lane masks of all rounds, bit by bit: the rounds' ballots are
  // independent, so they overlap
  bool bad = false;
  unsigned peers[kScanItems];
#pragma unroll
  for (int r = 0; r < kScanItems; ++r) {
    bad |= (key[r] == -1);
    peers[r] = __ballot_sync(0xffffffffu, key[r] >= 0);
  }
  for (int b = 0; b < nbits; ++b) {
#pragma unroll
    for (int r = 0; r < kScanItems; ++r) {
      const bool bit = (key[r] >> b) & 1;
      const unsigned bal = __ballot_sync(0xffffffffu, bit);
      peers[r] &= bit ? bal : ~bal;
    }
  }
#pragma unroll
  for (int r = 0; r < kScanItems; ++r) {
    const int k = key[r];
    int cur = 0;
    if (k >= 0) cur = my[k];
    __syncwarp();
    if (k >= 0 && lane == __ffs(peers[r]) - 1) my[k] = cur + __popc(peers[r]);
    __syncwarp();
    const int rank = k >= 0 ? cur + __popc(peers[r] & ((1u << lane) - 1u)) : 0;
    kr[r] = (uint32_t(k + 2) << 16) | uint32_t(rank);
  }
  return bad;
}

// Per expert: exclusive scan of the warp counts (warps hold consecutive
// entries) into warp bases, the tile total into tcount[e], and the tile's
// descriptor (tile 0 publishes its total as an inclusive prefix). Threads
// are spread over (expert, chunk of warps) so the serial part stays short;
// part[chunk][e] holds the per-chunk totals.
__device__ __forceinline__ void tile_totals_publish(int32_t* whist,
                                                    int32_t* tcount,
                                                    int32_t* part, int E,
                                                    int tile, uint32_t* desc,
                                                    bool first_inclusive = true) {
  const int tpe = max(1, min(kScanWarps, kScanThreads / E));  // threads / expert
  const int chunk = (kScanWarps + tpe - 1) / tpe;             // warps / thread
  for (int j = threadIdx.x; j < E * tpe; j += kScanThreads) {
    const int e = j % E, c = j / E;
    int32_t run = 0;
    for (int w = c * chunk; w < min(kScanWarps, (c + 1) * chunk); ++w) {
      const int32_t v = whist[w * E + e];
      whist[w * E + e] = run;
      run += v;
    }
    part[c * E + e] = run;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kScanThreads) {
    int32_t run = 0;
    for (int c = 0; c < tpe; ++c) {
      const int32_t v = part[c * E + e];
      part[c * E + e] = run;
      run += v;
    }
    tcount[e] = run;
    st_relaxed_gpu(desc + int64_t(tile) * E + e,
                   (tile == 0 && first_inclusive ? kFlagInclusive : kFlagAggregate) |
                       uint32_t(run));
  }
  __syncthreads();
  for (int j = threadIdx.x; j < E * tpe; j += kScanThreads) {
    const int e = j % E, c = j / E;
    const int32_t add = part[c * E + e];
    if (add)
      for (int w = c * chunk; w < min(kScanWarps, (c + 1) * chunk); ++w)
        whist[w * E + e] += add;
  }
}

// Look back for every expert: excl[e] = entries of expert e in tiles before
// this one; publishes this tile's inclusive prefix. Two threads per expert.
__device__ __forceinline__ void tile_lookback(const int32_t* tcount,
                                              int32_t* excl, int E, int tile,
                                              uint32_t* desc, int32_t* status,
                                              bool forced) {
  const int h = threadIdx.x & 1;
  for (int e0 = 0; e0 < E; e0 += kScanThreads / kLookbackPair) {
    const int e = e0 + int(threadIdx.x) / kLookbackPair;
    const bool active = e < E;
    const uint32_t x =
        lookback_pair(desc, E, active ? e : 0, active, h, tile, status, forced);
    if (active && h == 0) {
      if (tile > 0)
        st_relaxed_gpu(desc + int64_t(tile) * E + e,
                       kFlagInclusive | ((x + uint32_t(tcount[e])) & kValueMask));
      excl[e] = int32_t(x);
    }
  }
  __syncthreads();  // excl[e] was written by thread 2e, not by thread e
}

// Fused path: every tile's counts are published once (never overwritten),
// so each tile reads them all once every tile has published: excl[e] =
// entries of e in the tiles before this one, tot[e] = in all tiles. P
// threads share an expert, each summing tiles j = p, p+P, ... with
// kReduceBatch loads in flight; the P partial sums meet in `scratch`
// ([2][P][E] ints). `forced`: every descriptor stays pending, so the wait
// gives up after the forced budget.
constexpr int kReduceBatch = 16;
__device__ __forceinline__ void tile_reduce(const uint32_t* desc, int E, int tile,
                                            int num_tiles, int32_t* excl,
                                            int32_t* tot, int32_t* scratch,
                                            int32_t* status, bool forced) {
  const uint64_t budget = forced ? forced_budget_ns() : kWaitBudgetNs;
  const int P = max(1, min(32, kScanThreads / E));
  for (int idx = threadIdx.x; idx < E * P; idx += kScanThreads) {
    const int e = idx % E, p = idx / E;
    uint32_t sx = 0, st = 0;
    for (int j0 = p; j0 < num_tiles; j0 += P * kReduceBatch) {
      uint32_t v[kReduceBatch];
      unsigned pending = 0;
#pragma unroll
      for (int q = 0; q < kReduceBatch; ++q) {
        const int j = j0 + q * P;
        v[q] = kFlagAggregate;
        if (j < num_tiles) {
          v[q] = ld_relaxed_gpu(desc + int64_t(j) * E + e);
          if ((v[q] & ~kValueMask) == 0u || forced) pending |= 1u << q;
        }
      }
      if (pending) {  // some tile has not published yet: poll those
        const uint64_t t0 = globaltimer_ns();
        while (pending) {
#pragma unroll
          for (int q = 0; q < kReduceBatch; ++q)
            if ((pending >> q) & 1u) {
              v[q] = ld_relaxed_gpu(desc + int64_t(j0 + q * P) * E + e);
              if ((v[q] & ~kValueMask) != 0u && !forced) pending &= ~(1u << q);
            }
          if (pending && globaltimer_ns() - t0 > budget) {
            report(status, EP_DEV_TIMEOUT);
            break;
          }
        }
      }
#pragma unroll
      for (int q = 0; q < kReduceBatch; ++q) {
        const int j = j0 + q * P;
        const uint32_t c = v[q] & kValueMask;
        st += c;
        if (j < tile) sx += c;
      }
    }
    scratch[p * E + e] = int32_t(sx);
    scratch[(P + p) * E + e] = int32_t(st);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kScanThreads) {
    int32_t a = 0, b = 0;
    for (int p = 0; p < P; ++p) {
      a += scratch[p * E + e];
      b += scratch[(P + p) * E + e];
    }
    excl[e] = a;
    tot[e] = b;
  }
  __syncthreads();
}

// pos and row_src of the tile's entries. base[e] = first row of expert e
// for this tile (expert offset + earlier tiles), my[e] = this warp's base.
// pos is written in entry order. For row_src the tile is first counting-
// sorted in shared memory (tpre = exclusive prefix of the tile's counts over
// experts), so that each expert's rows are written as one contiguous run.
__device__ __forceinline__ void scatter_positions(
    int64_t tbase, int64_t wbase, const uint32_t (&kr)[kScanItems],
    const int32_t* base, const int32_t* my, const int32_t* tpre, int E,
    int32_t* sorted, int32_t* __restrict__ pos, int32_t* __restrict__ row_src,
    int64_t cap, int32_t* status) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int r = 0; r < kScanItems; ++r) {
    const int64_t i = wbase + r * 32 + lane;
    const int k = packed_key(kr[r]);
    if (k == -2) continue;
    if (k < 0) {
      pos[i] = -1;
      continue;
    }
    const int within = my[k] + packed_rank(kr[r]);
    pos[i] = int32_t(int64_t(base[k]) + within);
    sorted[tpre[k] + within] = (k << 12) | int(i - tbase);
  }
  __syncthreads();
  const int n = tpre[E];
  for (int t = threadIdx.x; t < n; t += kScanThreads) {
    const int v = sorted[t];
    const int k = v >> 12;
    const int64_t row = int64_t(base[k]) + (t - tpre[k]);
    if (row < cap)
      row_src[row] = int32_t(tbase + (v & 0xFFF));
    else
      report(status, EP_DEV_CAPACITY);
  }
}

// row_src = -1 on the padding rows of experts tile, tile+num_tiles, ...:
// one expert per warp, its rows over the lanes.
__device__ __forceinline__ void padding_row_src(const int32_t* off,
                                                const int32_t* cnt, int E,
                                                int tile, int num_tiles,
                                                int32_t* __restrict__ row_src,
                                                int64_t cap) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int64_t e = tile + int64_t(warp) * num_tiles; e < E;
       e += int64_t(kScanWarps) * num_tiles) {
    const int64_t lo = int64_t(off[e]) + cnt[e];
    const int64_t hi = min(int64_t(off[e + 1]), cap);
    for (int64_t r = lo + lane; r < hi; r += 32) row_src[r] = -1;
  }
}

// Shared memory of a scan CTA, in ints: per-warp counts [warps][E], tile
// counts [E], bases [E], offsets [E+1], totals [E], chunk totals
// [max(E, threads)], tile prefix over experts [E+1], sorted tile [kScanTile].
struct ScanSmem {
  int32_t *whist, *tcnt, *base, *offs, *tot, *part, *tpre, *sorted;
  __device__ ScanSmem(int32_t* s, int E)
      : whist(s),
        tcnt(s + kScanWarps * E),
        base(tcnt + E),
        offs(base + E),
        tot(offs + E + 1),
        part(tot + E),
        tpre(part + max(E, kScanThreads)),
        sorted(tpre + E + 1) {}
};
size_t scan_smem_bytes(int E) {
  return (size_t(kScanWarps) * E + 5 * size_t(E) + 2 +
          std::max<size_t>(E, kScanThreads) + kScanTile) * sizeof(int32_t);
}

// Tile prefix over experts of the tile counts (tpre[E] = valid entries).
__device__ __forceinline__ void tile_prefix(const int32_t* tcnt, int32_t* tpre,
                                            int E, int32_t* warp_tmp);

__device__ __forceinline__ void tile_prefix(const int32_t* tcnt, int32_t* tpre,
                                            int E, int32_t* warp_tmp) {
  for (int e = threadIdx.x; e < E; e += kScanThreads) tpre[e] = tcnt[e];
  __syncthreads();
  const int32_t n = block_exclusive_scan<kScanThreads>(tpre, E, warp_tmp);
  if (threadIdx.x == 0) tpre[E] = n;
  __syncthreads();
}

// ---- two-kernel path (any size): histogram, then the position scan --------

__global__ void __launch_bounds__(kScanThreads, 1)
    k_scan_positions(const int32_t* __restrict__ topk, int64_t M, int E,
                     const int32_t* __restrict__ counts,
                     const int32_t* __restrict__ offsets,
                     WsHeader* __restrict__ hdr, uint32_t* __restrict__ desc,
                     int num_tiles, int32_t* __restrict__ pos,
                     int32_t* __restrict__ row_src, int64_t cap,
                     int32_t* __restrict__ status) {
  grid_launch_dependents();
  extern __shared__ int32_t smem[];
  ScanSmem sm(smem, E);
  __shared__ int s_tile;
  __shared__ int32_t s_warp[kScanThreads / 32];
  const int tid = threadIdx.x, warp = tid >> 5;
  const bool forced = wait_forced(EP_WAIT_SITE_LOOKBACK);

  // Tiles are claimed in order of arrival, so every predecessor of a tile
  // belongs to a CTA that is already running: the look-back progresses.
  if (tid == 0) s_tile = int(atomicAdd(&hdr->tile_ticket, 1u));
  for (int j = tid; j < kScanWarps * E; j += kScanThreads) sm.whist[j] = 0;
  __syncthreads();
  const int tile = s_tile;
  const int64_t wbase = int64_t(tile) * kScanTile + int64_t(warp) * kWarpItems;
  uint32_t kr[kScanItems];
  int32_t* my = sm.whist + warp * E;
  rank_in_warps(topk, M, E, wbase, my, kr);
  __syncthreads();
  tile_totals_publish(sm.whist, sm.tcnt, sm.part, E, tile, desc);
  tile_lookback(sm.tcnt, sm.base, E, tile, desc, status, forced);
  tile_prefix(sm.tcnt, sm.tpre, E, s_warp);
  for (int e = tid; e < E; e += kScanThreads) sm.base[e] += __ldg(offsets + e);
  __syncthreads();
  scatter_positions(int64_t(tile) * kScanTile, wbase, kr, sm.base, my, sm.tpre,
                    E, sm.sorted, pos, row_src, cap, status);
  padding_row_src(offsets, counts, E, tile, num_tiles, row_src, cap);
}

// ---- fused path: one cooperative launch when every tile is co-resident ----

__global__ void __launch_bounds__(kScanThreads, 1)
    k_layout_fused(const int32_t* __restrict__ topk, int64_t M, int E, int pad,
                   WsHeader* __restrict__ hdr, uint32_t* __restrict__ desc,
                   int num_tiles, int32_t* __restrict__ tokens_per_expert,
                   int32_t* __restrict__ expert_offsets,
                   int32_t* __restrict__ pos, int32_t* __restrict__ row_src,
                   int64_t cap, int32_t* __restrict__ status) {
  grid_launch_dependents();
  extern __shared__ int32_t smem[];
  ScanSmem sm(smem, E);
  __shared__ int32_t s_warp2[2 * kScanThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int tile = blockIdx.x;
  const bool forced = wait_forced(EP_WAIT_SITE_TILE_REDUCE);

  for (int j = tid; j < kScanWarps * E; j += kScanThreads) sm.whist[j] = 0;
  __syncthreads();
  const int64_t wbase = int64_t(tile) * kScanTile + int64_t(warp) * kWarpItems;
  uint32_t kr[kScanItems];
  int32_t* my = sm.whist + warp * E;
  const bool bad = rank_in_warps(topk, M, E, wbase, my, kr);
  if (__any_sync(0xffffffffu, bad) && lane == 0) report(status, EP_DEV_BAD_EXPERT);
  __syncthreads();
  // counts published as aggregates only; every tile then reads all of them
  tile_totals_publish(sm.whist, sm.tcnt, sm.part, E, tile, desc, false);
  tile_reduce(desc, E, tile, num_tiles, sm.base, sm.tot, sm.sorted, status, forced);
  // each tile scans the padded totals into expert offsets and its own counts
  // into its counting-sort prefix, in one pass
  for (int e = tid; e < E; e += kScanThreads) {
    const int32_t total = sm.tot[e];
    sm.offs[e] = int32_t(((int64_t(total) + pad - 1) / pad) * pad);
    sm.tpre[e] = sm.tcnt[e];
  }
  __syncthreads();
  int32_t rows_used, tile_n;
  block_exclusive_scan2<kScanThreads>(sm.offs, sm.tpre, E, s_warp2, rows_used, tile_n);
  if (tid == 0) {
    sm.offs[E] = rows_used;
    sm.tpre[E] = tile_n;
  }
  if (tile == num_tiles - 1) {
    for (int e = tid; e < E; e += kScanThreads) {
      tokens_per_expert[e] = sm.tot[e];
      expert_offsets[e] = sm.offs[e];
    }
    if (tid == 0) expert_offsets[E] = rows_used;
  }
  for (int e = tid; e < E; e += kScanThreads) sm.base[e] += sm.offs[e];
  __syncthreads();
  scatter_positions(int64_t(tile) * kScanTile, wbase, kr, sm.base, my, sm.tpre,
                    E, sm.sorted, pos, row_src, cap, status);
  padding_row_src(sm.offs, sm.tot, E, tile, num_tiles, row_src, cap);
}

struct FusedCache {
  int device = -1;
  int E = -1;
  int capacity = 0;  // co-resident CTAs of k_layout_fused
};

cudaError_t set_smem(const void* kern, size_t smem) {
  if (smem <= 48 * 1024) return cudaSuccess;
  return cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              int(smem));
}

// Co-resident CTA capacity of the fused kernel for this device and E
// (0 when cooperative launch is unavailable); cached per (device, E).
int fused_capacity(int E) {
  static FusedCache cache[32];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  for (auto& c : cache)
    if (c.device == dev && c.E == E) return c.capacity;
  int coop = 0, sms = 0, per_sm = 0;
  if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
    return 0;
  const size_t smem = scan_smem_bytes(E);
  if (set_smem(reinterpret_cast<const void*>(k_layout_fused), smem) != cudaSuccess)
    return 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, k_layout_fused,
                                                    kScanThreads, smem) != cudaSuccess)
    return 0;
  const int capacity = coop ? per_sm * sms : 0;
  for (auto& c : cache)
    if (c.device < 0) {
      c = FusedCache{dev, E, capacity};
      break;
    }
  return capacity;
}

}  // namespace

cudaError_t set_wait_debug_layout(uint32_t sites, uint64_t budget_ns) {
  return set_wait_debug_here(sites, budget_ns);
}

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

  const int capacity = (tiles > 0) ? fused_capacity(E) : 0;
  if (tiles > 0 && tiles <= capacity) {
    // one cooperative launch; its descriptors must start at zero
    cudaError_t err = cudaMemsetAsync(ws, 0, layout_workspace_bytes(entries, E), stream);
    if (err != cudaSuccess) return err;
    int n_tiles = int(tiles);
    int64_t M = entries;
    int Ev = E, padv = pad;
    int64_t capv = cap;
    void* args[] = {(void*)&topk, &M, &Ev, &padv, &hdr, &desc, &n_tiles,
                    &tokens_per_expert, &expert_offsets, &pos, &row_src, &capv,
                    &status};
    return cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(k_layout_fused),
                                       dim3(n_tiles), dim3(kScanThreads), args,
                                       scan_smem_bytes(E), stream);
  }

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

  const size_t smem = scan_smem_bytes(E);
  err = set_smem(reinterpret_cast<const void*>(k_scan_positions), smem);
  if (err != cudaSuccess) return err;
  k_scan_positions<<<int(tiles), kScanThreads, smem, stream>>>(
      topk, entries, E, tokens_per_expert, expert_offsets, hdr, desc, int(tiles),
      pos, row_src, cap, status);
  return cudaGetLastError();
}

}  // namespace ep
