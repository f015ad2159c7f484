// layout_small.cu -- the layout of a small batch, alone or together with the
// dispatch copy, in ONE launch with no inter-CTA communication.
//
// "DeepSeek开源周第二天：DeepEP深度分析", section "DeepEP介绍": decoding is
// served by separate low-latency kernels, since a decode batch is small and
// its dispatch is latency-bound. Section "代码解读" (双缓冲区) is the
// double-buffered receive side that goes with it (EPBuffer).
//
// For a small batch, the look-back scan of layout.cu is a chain of
// dependent steps across CTAs (publish, look back, read the last tile's
// totals), each a few hundred ns of memory latency, and a separate dispatch
// launch then adds its own ramp. Here every CTA instead counts ALL N*K
// entries itself in shared memory. The router's top-k array of a decode
// batch is a few tens of KB and stays in L2, so the redundant reads cost
// little. Counting gives each CTA every expert's total (hence the padded
// expert offsets) and, for its own contiguous chunk of tokens, the number of
// earlier entries of each expert. The CTA then ranks its own entries in
// (t, k) order and knows their final rows without hearing from any other
// CTA: no workspace, no memset, no cooperative launch, no wait on another
// CTA.
//
// With a copy mode the same CTA also moves its tokens. Their rows are
// requested by TMA bulk loads at kernel entry, so the loads overlap the
// counting. bf16: once the rows are placed, every warp bulk-stores rows to
// their K receive rows. FP8 is warp-specialised: right after the count,
// warps 4-15 start quantising (token, 512-channel unit) pairs in token
// order into shared-memory output stages (the quantiser of ep_quant.cuh),
// while warps 0-3 compute the offsets and ranks and then join them; warp 0
// then bulk-stores each token as soon as its last unit is quantised. Stage
// reuse is ordered by mbarriers (row landed / token quantised / output
// read), so a chunk longer than the stages streams through them.
// The results are bit-identical to ep_layout followed by ep_dispatch.
//
// The counting costs O(N*K) per CTA, so the host takes this path only for
// small batches (small_layout_fits).
#include <algorithm>

#include "ep_block.cuh"
#include "ep_device.cuh"
#include "ep_launch.h"
#include "ep_quant.cuh"

namespace ep {
namespace {

constexpr int kSmallThreads = 512;
constexpr int kSmallWarps = kSmallThreads / 32;
constexpr int kQuantUnit = 512;  // channels one warp quantises per pass
constexpr int kRankWarps = 4;    // FP8: warps that rank while the rest quantise
constexpr size_t kStageBudget = 192 * 1024;  // staged rows per CTA

enum class Copy { kNone, kBf16, kFp8 };

__host__ __device__ constexpr uint32_t round128(uint32_t x) {
  return (x + 127u) & ~127u;
}

// Shared-memory plan of one CTA, computed identically on host and device:
// `batch` stages, each one staged bf16 token row and, for FP8, its output
// (codes then scales); three barriers per stage; then the int arrays.
struct SmallPlan {
  int chunk;           // tokens per CTA (contiguous)
  int grid;            // CTAs
  int batch;           // stages: token rows staged at once
  uint32_t in_bytes;   // one staged row
  uint32_t out_bytes;  // one FP8 output stage
  size_t bar_off;      // barriers: full[batch] qdone[batch] ofree[batch]
  size_t int_off;      // before[E] after[E] offs[E+1] run[E] spos[] skey[] swt[]
  size_t smem;
};

__host__ __device__ inline SmallPlan small_plan(int64_t N, int K, int E, int H,
                                                Copy mode, int num_sms) {
  SmallPlan p;
  const int64_t sms = num_sms > 0 ? num_sms : 1;
  const int64_t chunk = N > 0 ? (N + sms - 1) / sms : 1;
  p.chunk = int(chunk);
  p.grid = int(N > 0 ? (N + chunk - 1) / chunk : 1);
  p.in_bytes = mode == Copy::kNone ? 0u : round128(uint32_t(H) * 2u);
  p.out_bytes =
      mode == Copy::kFp8 ? round128(uint32_t(H) + uint32_t(H / 128) * 4u) : 0u;
  p.batch = 0;
  if (mode != Copy::kNone) {
    const int64_t b = int64_t(kStageBudget / (p.in_bytes + p.out_bytes));
    p.batch = int(b < 1 ? 1 : (b > chunk ? chunk : b));
  }
  p.bar_off = size_t(p.batch) * (p.in_bytes + p.out_bytes);
  p.int_off = p.bar_off + 3 * 8 * size_t(p.batch > 0 ? p.batch : 1);
  p.smem = p.int_off + 4 * (4 * size_t(E) + 1 + 3 * size_t(p.chunk) * size_t(K));
  return p;
}

// Bounded wait of lane 0 on `bar`, the outcome shared by the warp.
__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity,
                                          int32_t* status, bool forced) {
  bool ok = true;
  if ((threadIdx.x & 31) == 0) ok = mbar_wait_bounded(bar, parity, forced);
  ok = __shfl_sync(0xffffffffu, ok, 0);
  if (!ok && (threadIdx.x & 31) == 0) report(status, EP_DEV_TIMEOUT);
  return ok;
}


// The count's loads: round i0 of the int4 loads over the top-k array
// (topk is 16-byte aligned), kCountUnroll loads per thread per round.
constexpr int kCountUnroll = 4;

template <int NT>
__device__ __forceinline__ void count_loads(const int32_t* __restrict__ topk,
                                            int64_t M4, int64_t i0,
                                            int4 (&v)[kCountUnroll]) {
#pragma unroll
  for (int u = 0; u < kCountUnroll; ++u) {
    const int64_t i = i0 + int64_t(u) * NT * 4;
    v[u] = i < M4 ? __ldg(reinterpret_cast<const int4*>(topk + i))
                  : make_int4(-1, -1, -1, -1);
  }
}

// Counts: every entry of the batch into before[e] (entries ahead of the
// chunk) or after[e] (the chunk and later), and the chunk's own expert ids
// into skey. Threads [0, NT). v holds the first round's loads, issued by the
// caller before the shared memory was set up.
template <int NT>
__device__ __forceinline__ void count_entries(const int32_t* __restrict__ topk,
                                              int64_t M, int E, int64_t split,
                                              int n_ent, int32_t* before,
                                              int32_t* after, int32_t* skey,
                                              int4 (&v)[kCountUnroll]) {
  auto count = [&](int e, int64_t i) {
    if (unsigned(e) < unsigned(E)) atomicAdd(i < split ? &before[e] : &after[e], 1);
    const int64_t r = i - split;
    if (r >= 0 && r < n_ent) skey[r] = e;
  };
  const int64_t M4 = M & ~int64_t(3);
  for (int64_t i0 = int64_t(threadIdx.x) * 4; i0 < M4;
       i0 += int64_t(NT) * 4 * kCountUnroll) {
    if (i0 != int64_t(threadIdx.x) * 4) count_loads<NT>(topk, M4, i0, v);
#pragma unroll
    for (int u = 0; u < kCountUnroll; ++u) {
      const int64_t i = i0 + int64_t(u) * NT * 4;
      if (i < M4) {
        count(v[u].x, i);
        count(v[u].y, i + 1);
        count(v[u].z, i + 2);
        count(v[u].w, i + 3);
      }
    }
  }
  for (int64_t i = M4 + threadIdx.x; i < M; i += NT) count(__ldg(topk + i), i);
}

// Expert totals, padded exclusive offsets, and the chunk's base row per
// expert (before[e] becomes offs[e] + entries ahead of the chunk); CTA 0
// also writes the counts and offsets out. Threads [0, NT).
template <int NT, int BAR>
__device__ __forceinline__ void group_offsets(int32_t* before, int32_t* after,
                                              int32_t* offs, int E, int pad,
                                              int32_t* s_warp,
                                              int32_t* __restrict__ tokens_per_expert,
                                              int32_t* __restrict__ expert_offsets) {
  for (int e = threadIdx.x; e < E; e += NT) {
    const int32_t total = before[e] + after[e];
    after[e] = total;
    // total < 2^30 and pad < 2^31: the rounded-up sum stays below 2^32
    const uint32_t up = uint32_t(total) + uint32_t(pad) - 1u;
    offs[e] = pad == 1 ? total : int32_t((up / uint32_t(pad)) * uint32_t(pad));
  }
  group_sync<NT, BAR>();
  const int32_t used = block_exclusive_scan<NT, BAR>(offs, E, s_warp);
  if (threadIdx.x == 0) offs[E] = used;
  for (int e = threadIdx.x; e < E; e += NT) {
    before[e] += offs[e];
    if (blockIdx.x == 0) {
      tokens_per_expert[e] = after[e];
      expert_offsets[e] = offs[e];
    }
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) expert_offsets[E] = used;
  group_sync<NT, BAR>();
}

// Rank each of the chunk's entries among the chunk's earlier entries of the
// same expert (a count over the earlier ids in shared memory: the threads
// of a warp read the same id at once) and write pos, row_src, the receive
// weight of each row and the rows into spos (-1: none). Threads [0, NT).
template <int NT>
__device__ __forceinline__ void group_rank(const int32_t* skey, const float* swt,
                                          const int32_t* base, int E,
                                          int64_t split, int n_ent, int64_t cap,
                                          int32_t* spos, int32_t* __restrict__ pos,
                                          int32_t* __restrict__ row_src,
                                          float* __restrict__ recv_w,
                                          int32_t* __restrict__ status) {
  bool bad = false;
  for (int j = threadIdx.x; j < n_ent; j += NT) {
    const int key = skey[j];
    int32_t p = -1, keep = -1;
    if (unsigned(key) < unsigned(E)) {
      int earlier = 0;
      for (int i = 0; i < j; ++i) earlier += (skey[i] == key);
      const int64_t row = int64_t(base[key]) + earlier;
      p = int32_t(row);
      if (row < cap) {
        row_src[row] = int32_t(split + j);
        if (recv_w) recv_w[row] = swt[j];
        keep = p;
      } else {
        report(status, EP_DEV_CAPACITY);
      }
    } else {
      bad = true;
    }
    pos[split + j] = p;
    spos[j] = keep;
  }
  if (__any_sync(0xffffffffu, bad) && (threadIdx.x & 31) == 0)
    report(status, EP_DEV_BAD_EXPERT);
}

// Warp 0 alone: rank the chunk's entries in (t, k) order, 32 per round, the lanes of one expert found with one
// ballot per id bit; same outputs as group_rank. run[] must start at zero.
__device__ __forceinline__ void warp_rank(const int32_t* skey, const float* swt,
                                          const int32_t* base, int32_t* run,
                                          int E, int64_t split, int n_ent,
                                          int64_t cap, int32_t* spos,
                                          int32_t* __restrict__ pos,
                                          int32_t* __restrict__ row_src,
                                          float* __restrict__ recv_w,
                                          int32_t* __restrict__ status) {
  const int lane = threadIdx.x & 31;
  const int nbits = expert_bits(E);
  bool bad = false;
  for (int r0 = 0; r0 < n_ent; r0 += 32) {
    const int j = r0 + lane;
    int key = -2;
    if (j < n_ent) {
      const int e = skey[j];
      key = unsigned(e) < unsigned(E) ? e : -1;
    }
    bad |= (key == -1);
    const unsigned peers = same_key_lanes(key, nbits);
    int cur = 0;
    if (key >= 0) cur = run[key];
    __syncwarp();
    if (key >= 0 && lane == __ffs(peers) - 1) run[key] = cur + __popc(peers);
    __syncwarp();
    if (j < n_ent) {
      int32_t p = -1, keep = -1;
      if (key >= 0) {
        const int64_t row = int64_t(base[key]) + cur + __popc(peers & ((1u << lane) - 1u));
        p = int32_t(row);
        if (row < cap) {
          row_src[row] = int32_t(split + j);
          if (recv_w) recv_w[row] = swt[j];
          keep = p;
        } else {
          report(status, EP_DEV_CAPACITY);
        }
      }
      pos[split + j] = p;
      spos[j] = keep;
    }
  }
  if (__any_sync(0xffffffffu, bad) && lane == 0) report(status, EP_DEV_BAD_EXPERT);
  __syncwarp();
}

template <Copy kMode>
__global__ void __launch_bounds__(kSmallThreads, 1)
    k_layout_small(const int32_t* __restrict__ topk, int64_t N, int K, int E,
                   int pad, int H, int num_sms,
                   int32_t* __restrict__ tokens_per_expert,
                   int32_t* __restrict__ expert_offsets,
                   int32_t* __restrict__ pos, int32_t* __restrict__ row_src,
                   int64_t cap, const uint16_t* __restrict__ hidden,
                   const float* __restrict__ w, uint8_t* __restrict__ recv,
                   float* __restrict__ scales, float* __restrict__ recv_w,
                   int32_t* __restrict__ status) {
  extern __shared__ __align__(128) uint8_t smem[];
  const SmallPlan pl = small_plan(N, K, E, H, kMode, num_sms);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t t0 = int64_t(blockIdx.x) * pl.chunk;
  const int64_t left = N - t0;
  const int n_mine = left <= 0 ? 0 : int(left < pl.chunk ? left : int64_t(pl.chunk));
  const int64_t split = t0 * K;  // first entry of this CTA's chunk
  const int n_ent = n_mine * K;
  const uint32_t row_bytes = uint32_t(H) * 2u;
  const int G = H >> 7;
  const uint32_t scale_bytes = uint32_t(G) * 4u;
  const int nb = pl.batch;

  // stage s: row in_base + s*in_bytes, FP8 output out_base + s*out_bytes.
  // Token j of the chunk (0-based) uses stage j % nb, for the (j / nb)-th
  // time: full[s] completes when its row has landed, qdone[s] when it is
  // quantised (FP8), ofree[s] when the stores of its output have read it.
  uint8_t* in_base = smem;
  uint8_t* out_base = smem + size_t(nb) * pl.in_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + pl.bar_off);
  uint64_t* qdone = full + nb;
  uint64_t* ofree = qdone + nb;
  int32_t* before = reinterpret_cast<int32_t*>(smem + pl.int_off);
  int32_t* after = before + E;   // from the chunk on; later the expert total
  int32_t* offs = after + E;     // [E+1] padded exclusive prefix
  int32_t* run = offs + E + 1;   // [E] own entries ranked so far (warp_rank)
  int32_t* spos = run + E;       // [n_ent] rows of the own entries (-1: none)
  int32_t* skey = spos + size_t(pl.chunk) * K;  // [n_ent] own expert ids
  float* swt = reinterpret_cast<float*>(skey + size_t(pl.chunk) * K);  // weights
  __shared__ int s_abort;
  __shared__ int s_next;  // next FP8 (token, unit) pair to quantise
  __shared__ int32_t s_warp[kSmallWarps];
  const int units = (H + kQuantUnit - 1) / kQuantUnit;
  const bool forced = wait_forced(EP_WAIT_SITE_SMALL);

  int issued = 0;  // rows requested (thread 0 requests them all)
  auto load_row = [&](int j) {
    ++issued;
    const int s = j % nb;
    mbar_arrive_expect_tx(&full[s], row_bytes);
    bulk_g2s(in_base + size_t(s) * pl.in_bytes, hidden + (t0 + j) * H, row_bytes,
             &full[s]);
  };

  // the count's first loads go out before the shared-memory setup
  int4 v0[kCountUnroll];
  count_loads<kSmallThreads>(topk, (N * K) & ~int64_t(3), int64_t(tid) * 4, v0);
  if (tid == 0) {
    s_abort = 0;
    s_next = 0;
    if constexpr (kMode != Copy::kNone) {
      for (int s = 0; s < nb; ++s) {
        mbar_init(&full[s], 1);
        mbar_init(&qdone[s], uint32_t(units));
        mbar_init(&ofree[s], 1);
      }
      fence_mbar_init();
      for (int j = 0; j < nb && j < n_mine; ++j) load_row(j);  // overlap the count
    }
  }
  for (int e = tid; e < E; e += kSmallThreads) {
    before[e] = 0;
    after[e] = 0;
    run[e] = 0;
  }
  __syncthreads();

  // ---- counts, by the whole CTA ------------------------------------------
  constexpr int kPerThread = int(kSmallMaxChunkEntries / kSmallThreads);
  const bool want_w = kMode != Copy::kNone && recv_w != nullptr;
  {
    // the chunk's route weights are requested first; their latency hides
    // behind the count
    float wv[kPerThread];
#pragma unroll
    for (int q = 0; q < kPerThread; ++q) {
      const int j = tid + q * kSmallThreads;
      wv[q] = (want_w && j < n_ent) ? __ldg(w + split + j) : 0.0f;
    }
    count_entries<kSmallThreads>(topk, N * K, E, split, n_ent, before, after, skey, v0);
#pragma unroll
    for (int q = 0; q < kPerThread; ++q) {
      const int j = tid + q * kSmallThreads;
      if (want_w && j < n_ent) swt[j] = wv[q];
    }
    __syncthreads();
  }
  // ---- offsets and ranks: under FP8 by warps 0-3 while the others start
  // quantising; otherwise by the whole CTA ---------------------------------
  if constexpr (kMode == Copy::kFp8) {
    // (ranks: a count over the earlier ids for short chunks, warp ballots in
    // rounds of 32 for long ones, whose quadratic count would be slow)
    if (warp < kRankWarps) {
      group_offsets<kRankWarps * 32, 1>(before, after, offs, E, pad, s_warp,
                                        tokens_per_expert, expert_offsets);
      if (n_ent <= kRankWarps * 64)
        group_rank<kRankWarps * 32>(skey, swt, before, E, split, n_ent, cap, spos,
                                    pos, row_src, want_w ? recv_w : nullptr, status);
      else if (warp == 0)
        warp_rank(skey, swt, before, run, E, split, n_ent, cap, spos, pos, row_src,
                  want_w ? recv_w : nullptr, status);
      group_sync<kRankWarps * 32, 1>();
    }
  } else {
    group_offsets<kSmallThreads, 0>(before, after, offs, E, pad, s_warp,
                                    tokens_per_expert, expert_offsets);
    group_rank<kSmallThreads>(skey, swt, before, E, split, n_ent, cap, spos, pos,
                              row_src, want_w ? recv_w : nullptr, status);
    __syncthreads();
  }

  if constexpr (kMode == Copy::kFp8) {
    const bool bulk_scales = (scale_bytes % 16u) == 0u;
    if (warp > 0) {
      // ---- quantiser warps: (token, 512-channel unit) pairs in order,
      // claimed one at a time
      for (;;) {
        int idx = 0;
        if (lane == 0) idx = atomicAdd(&s_next, 1);
        idx = __shfl_sync(0xffffffffu, idx, 0);
        if (idx >= n_mine * units || s_abort) break;
        const int j = idx / units, u = idx - j * units;
        const int s = j % nb, m = j / nb;
        bool ok = warp_wait(&full[s], uint32_t(m) & 1u, status, forced);
        if (ok && m >= 1) ok = warp_wait(&ofree[s], uint32_t(m - 1) & 1u, status, forced);
        if (!ok) {
          s_abort = 1;
          break;
        }
        uint8_t* out = out_base + size_t(s) * pl.out_bytes;
        const int c0 = u * kQuantUnit + lane * 16;
        const bool act = c0 < H;
        const float scale =
            quantize_lane16(in_base + size_t(s) * pl.in_bytes, out, c0, act);
        if (act && (lane & 7) == 0) reinterpret_cast<float*>(out + H)[c0 >> 7] = scale;
        fence_proxy_async_smem();  // the stores read this through the TMA engine
        __syncwarp();
        if (lane == 0) mbar_arrive(&qdone[s]);
      }
    } else {
      // ---- warp 0 stores each quantised token to its K rows --------------
      const bool issuer = lane < K;
      const int lag = nb >= 2 ? 1 : 0;  // tokens whose stores may still read
      for (int j = 0; j < n_mine; ++j) {
        const int s = j % nb, m = j / nb;
        if (!warp_wait(&qdone[s], uint32_t(m) & 1u, status, forced)) {
          s_abort = 1;
          break;
        }
        const uint8_t* out = out_base + size_t(s) * pl.out_bytes;
        if (issuer) {
          const int p = spos[j * K + lane];
          if (p >= 0) {
            bulk_s2g(recv + int64_t(p) * H, out, uint32_t(H));
            if (bulk_scales) bulk_s2g(scales + int64_t(p) * G, out + H, scale_bytes);
          }
          bulk_commit();
        }
        if (!bulk_scales) {  // G*4 not a multiple of 16: plain stores
          const float* sc = reinterpret_cast<const float*>(out + H);
          for (int k = 0; k < K; ++k) {
            const int p = spos[j * K + k];
            if (p >= 0)
              for (int g = lane; g < G; g += 32) scales[int64_t(p) * G + g] = sc[g];
          }
        }
        // the row of token j is quantised: its stage takes token j + nb
        if (lane == 0 && j + nb < n_mine) load_row(j + nb);
        // the output of token j - lag has been read by its stores: free it
        const int jf = j - lag;
        if (jf >= 0 && jf + nb < n_mine) {
          if (issuer) {
            if (lag == 1)
              bulk_wait_read<1>();
            else
              bulk_wait_read<0>();
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&ofree[jf % nb]);
        }
      }
      if (issuer) bulk_wait_all<0>();
    }
  } else if constexpr (kMode == Copy::kBf16) {
    const bool issuer = lane < K;  // lane k of a warp stores row k
    bool gave_up = false;
    for (int b0 = 0; b0 < n_mine; b0 += nb) {
      const int n = min(nb, n_mine - b0);
      for (int jj = warp; jj < n; jj += kSmallWarps) {
        const int j = b0 + jj;
        if (!warp_wait(&full[jj], uint32_t(j / nb) & 1u, status, forced)) {
          s_abort = 1;  // its load may still be in flight: drained at the end
          gave_up = true;
          continue;
        }
        if (issuer) {
          const int p = spos[j * K + lane];
          if (p >= 0)
            bulk_s2g(recv + int64_t(p) * row_bytes, in_base + size_t(jj) * pl.in_bytes,
                     row_bytes);
        }
      }
      if (issuer) bulk_commit();
      if (b0 + n < n_mine) {
        // the next batch reuses the stages once these stores have read them;
        // after a give-up in any warp, no further batch is loaded (the
        // decision is the barrier's, hence the same in every warp)
        if (issuer) bulk_wait_read<0>();
        if (__syncthreads_or(gave_up)) break;
        if (tid == 0)
          for (int j = b0 + n; j < b0 + n + nb && j < n_mine; ++j) load_row(j);
      }
    }
    if (issuer) bulk_wait_all<0>();
  }
  __syncthreads();

  if constexpr (kMode != Copy::kNone) {
    // after a give-up no load may still be writing shared memory: wait for
    // the last load requested into every stage
    if (tid == 0 && s_abort)
      for (int s = 0; s < nb && s < issued; ++s) {
        const int last = s + ((issued - 1 - s) / nb) * nb;
        mbar_wait_bounded(&full[s], uint32_t(last / nb) & 1u);
      }
  }

  // ---- padding rows of experts blockIdx.x, +gridDim.x, ... ---------------
  for (int e = blockIdx.x; e < E; e += gridDim.x) {
    const int64_t lo = int64_t(offs[e]) + after[e];
    const int64_t hi = min(int64_t(offs[e + 1]), cap);
    if constexpr (kMode == Copy::kNone) {
      for (int64_t r = lo + tid; r < hi; r += kSmallThreads) row_src[r] = -1;
    } else {
      const uint4 z = make_uint4(0u, 0u, 0u, 0u);
      for (int64_t r = lo + warp; r < hi; r += kSmallWarps) {
        if constexpr (kMode == Copy::kFp8) {
          for (int c = lane * 16; c < H; c += 32 * 16) st_v4(recv + r * H + c, z);
          for (int g = lane; g < G; g += 32) scales[r * G + g] = 0.0f;
        } else {
          for (int v = lane; v < (H >> 3); v += 32) st_v4(recv + r * row_bytes + v * 16, z);
        }
        if (lane == 0) {
          row_src[r] = -1;
          if (recv_w) recv_w[r] = 0.0f;
        }
      }
    }
  }
}

template <Copy kMode>
cudaError_t run_small(const int32_t* topk, int64_t N, int K, int E, int pad,
                      int H, int32_t* tokens_per_expert,
                      int32_t* expert_offsets, int32_t* pos, int32_t* row_src,
                      int64_t cap, const void* hidden, const float* w,
                      void* recv, float* scales, float* recv_w, int num_sms,
                      int32_t* status, cudaStream_t stream) {
  const SmallPlan pl = small_plan(N, K, E, H, kMode, num_sms);
  const void* kern = reinterpret_cast<const void*>(k_layout_small<kMode>);
  if (pl.smem > 48 * 1024) {
    cudaError_t err = cudaFuncSetAttribute(
        kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(pl.smem));
    if (err != cudaSuccess) return err;
  }
  k_layout_small<kMode><<<pl.grid, kSmallThreads, pl.smem, stream>>>(
      topk, N, K, E, pad, H, num_sms, tokens_per_expert, expert_offsets, pos,
      row_src, cap, static_cast<const uint16_t*>(hidden), w,
      static_cast<uint8_t*>(recv), scales, recv_w, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t set_wait_debug_layout_small(uint32_t sites, uint64_t budget_ns) {
  return set_wait_debug_here(sites, budget_ns);
}

bool small_layout_fits(int64_t N, int K, int E, int H, int copy, int num_sms) {
  if (N * K > kSmallMaxEntries) return false;
  const Copy mode = copy == 0 ? Copy::kNone : (copy == 1 ? Copy::kBf16 : Copy::kFp8);
  const SmallPlan pl = small_plan(N, K, E, H, mode, num_sms);
  return int64_t(pl.chunk) * K <= kSmallMaxChunkEntries &&
         pl.smem <= size_t(kSmallMaxSmem);
}

cudaError_t launch_layout_small(const int32_t* topk, int64_t N, int K, int E,
                                int pad, int32_t* tokens_per_expert,
                                int32_t* expert_offsets, int32_t* pos,
                                int32_t* row_src, int64_t cap, int num_sms,
                                int32_t* status, cudaStream_t stream) {
  return run_small<Copy::kNone>(topk, N, K, E, pad, 8, tokens_per_expert,
                                expert_offsets, pos, row_src, cap, nullptr,
                                nullptr, nullptr, nullptr, nullptr, num_sms,
                                status, stream);
}

cudaError_t launch_layout_dispatch_small(
    const int32_t* topk, int64_t N, int K, int E, int pad, int H, bool fp8,
    int32_t* tokens_per_expert, int32_t* expert_offsets, int32_t* pos,
    int32_t* row_src, int64_t cap, const void* hidden, const float* w,
    void* recv, float* scales, float* recv_w, int num_sms, int32_t* status,
    cudaStream_t stream) {
  if (fp8)
    return run_small<Copy::kFp8>(topk, N, K, E, pad, H, tokens_per_expert,
                                 expert_offsets, pos, row_src, cap, hidden, w,
                                 recv, scales, recv_w, num_sms, status, stream);
  return run_small<Copy::kBf16>(topk, N, K, E, pad, H, tokens_per_expert,
                                expert_offsets, pos, row_src, cap, hidden, w,
                                recv, scales, recv_w, num_sms, status, stream);
}

}  // namespace ep
