// combine.cu -- gather each token's K expert outputs and reduce them with the
// route weights, back in token order.
//
// "Экспертный параллелизм (EP)", section "Что подтверждено": expert results
// come back through the second AllToAll and are combined. "DeepSeek开源周第二天
// ：DeepEP深度分析", section "性能": BF16 combine. The sum is taken in fp32 with
// one fused multiply-add per k, k ascending from +0, then rounded to bf16
// (nearest even), so the result is a fixed function of its inputs.
//
// The kernel reads K rows per written row: it is bound by HBM read bandwidth.
// Two forms:
//   k_combine_tma  (large batches) persistent, one CTA per SM: a producer
//                  warp bulk-loads the K gathered part-rows of a (token, part)
//                  unit into a shared-memory stage (three stages, ~170 KB of
//                  reads in flight per SM); consumer threads reduce from
//                  shared memory and store the output part from registers.
//   k_combine<K>   (small batches) CTAs walk tokens, threads split the row
//                  into 16-byte vectors and issue their K gathered loads
//                  before any arithmetic.
// Both run the same fma chain in the same k order.
//
// Weights come either per entry (w[t,k], token side) or per receive row
// (w_rows[pos[t,k]]: the receive-side route_weights_nvs of
// "MoonEP核心功能深度剖析", "快速上手", combine(plan, expert_output_nvsh,
// route_weights_nvs) -> output_sh, gathered_route_weights_sk). With row
// weights the kernels also write each entry's weight back in token order
// (`gathered`), so the caller needs no separate gather launch.
#include <algorithm>

#include "ep_device.cuh"
#include "ep_launch.h"

namespace ep {
namespace {

constexpr int kCombineMaxThreads = 512;
constexpr int kChunk = 8;  // k-terms loaded together on the generic path

__device__ __forceinline__ void fma8(float (&acc)[8], float wk, const uint4& d) {
  acc[0] = fmaf(wk, bf16_lo(d.x), acc[0]);
  acc[1] = fmaf(wk, bf16_hi(d.x), acc[1]);
  acc[2] = fmaf(wk, bf16_lo(d.y), acc[2]);
  acc[3] = fmaf(wk, bf16_hi(d.y), acc[3]);
  acc[4] = fmaf(wk, bf16_lo(d.z), acc[4]);
  acc[5] = fmaf(wk, bf16_hi(d.z), acc[5]);
  acc[6] = fmaf(wk, bf16_lo(d.w), acc[6]);
  acc[7] = fmaf(wk, bf16_hi(d.w), acc[7]);
}

__device__ __forceinline__ uint4 pack8(const float (&acc)[8]) {
  return make_uint4(pack_bf16x2(acc[0], acc[1]), pack_bf16x2(acc[2], acc[3]),
                    pack_bf16x2(acc[4], acc[5]), pack_bf16x2(acc[6], acc[7]));
}

// Where the weight of entry (t,k) comes from (see the file comment).
struct Weights {
  const float* tok;   // [N,K] per entry; NULL with rows NULL: unit weights
  const float* rows;  // [cap] per receive row, or NULL
  float* gathered;    // [N,K] out: rows[pos[t,k]] (0 where pos is outside
                      // [0, cap)); written only with rows
};

// Weight of entry (t,k) whose row is p.
__device__ __forceinline__ float entry_weight(const Weights& wt, int64_t t,
                                              int K, int k, int32_t p,
                                              int64_t cap) {
  if (wt.rows) return (p >= 0 && p < cap) ? __ldg(wt.rows + p) : 0.0f;
  return wt.tok ? __ldg(wt.tok + t * K + k) : 1.0f;
}

// KT > 0: K known at compile time; KT == 0: runtime K, in chunks of kChunk
// terms (the chunks run in k order, so the fma order is unchanged). kRows:
// weights per receive row (wts.rows), else per entry or unit (wts.tok).
// Two CTAs per SM: at most 64 registers a thread.
template <int KT, bool kRows>
__global__ void __launch_bounds__(kCombineMaxThreads, 2)
    k_combine(const uint16_t* __restrict__ y, const int32_t* __restrict__ pos,
              Weights wts, int64_t N, int Kr, int H, int64_t cap,
              uint16_t* __restrict__ out, int32_t* __restrict__ status) {
  const int K = KT > 0 ? KT : Kr;
  const int V = H >> 3;
  if constexpr (kRows) wts.tok = nullptr;
  else wts.rows = nullptr;
  for (int64_t t = blockIdx.x; t < N; t += gridDim.x) {
    const int32_t* pt = pos + t * K;
    if (kRows && wts.gathered && threadIdx.x < K) {
      const int32_t p = __ldg(pt + threadIdx.x);
      wts.gathered[t * K + threadIdx.x] = entry_weight(wts, t, K, threadIdx.x, p, cap);
    }
    if constexpr (KT > 0) {
      int64_t rowoff[KT];
      float wk[KT];
#pragma unroll
      for (int k = 0; k < KT; ++k) {
        const int32_t p = __ldg(pt + k);
        wk[k] = entry_weight(wts, t, K, k, p, cap);
        const bool ok = p >= 0 && p < cap;
        if (p >= cap && threadIdx.x == 0) report(status, EP_DEV_CAPACITY);
        rowoff[k] = ok ? int64_t(p) * H : int64_t(-1);
      }
      for (int v = threadIdx.x; v < V; v += blockDim.x) {
        uint4 d[KT];
#pragma unroll
        for (int k = 0; k < KT; ++k)
          d[k] = rowoff[k] >= 0 ? ld_stream_v4(y + rowoff[k] + v * 8)
                                : make_uint4(0u, 0u, 0u, 0u);
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int k = 0; k < KT; ++k)
          if (rowoff[k] >= 0) fma8(acc, wk[k], d[k]);
        st_v4(out + t * H + v * 8, pack8(acc));
      }
    } else {
      for (int v = threadIdx.x; v < V; v += blockDim.x) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int k0 = 0; k0 < K; k0 += kChunk) {
          uint4 d[kChunk];
          int64_t off[kChunk];
          float wk[kChunk];
#pragma unroll
          for (int j = 0; j < kChunk; ++j) {
            off[j] = -1;
            wk[j] = 0.f;
            if (k0 + j < K) {
              const int32_t p = __ldg(pt + k0 + j);
              wk[j] = entry_weight(wts, t, K, k0 + j, p, cap);
              if (p >= 0 && p < cap) off[j] = int64_t(p) * H;
              if (p >= cap && v == threadIdx.x && threadIdx.x == 0)
                report(status, EP_DEV_CAPACITY);
            }
            d[j] = off[j] >= 0 ? ld_stream_v4(y + off[j] + v * 8)
                               : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
          for (int j = 0; j < kChunk; ++j)
            if (off[j] >= 0) fma8(acc, wk[j], d[j]);
        }
        st_v4(out + t * H + v * 8, pack8(acc));
      }
    }
  }
}

// ---------------------------------------------------------------------------
// TMA-fed combine: a producer warp bulk-loads, for each (token, row part),
// the K gathered part-rows into a shared-memory stage; consumer threads run
// the fma chain from shared memory and store their 16-byte output vectors
// from registers. Three stages keep ~170 KB of reads in flight per SM.
// ---------------------------------------------------------------------------

constexpr int kTmaMaxConsumerWarps = 16;
constexpr int kTmaStages = 3;
constexpr uint32_t kTmaStageTarget = 64 * 1024;  // K part-rows per stage

__host__ __device__ constexpr uint32_t al128(uint32_t x) { return (x + 127u) & ~127u; }

struct TmaShape {
  int part_ch;   // channels per part (multiple of 8)
  int parts;     // parts per row
  int cw;        // consumer warps
  uint32_t in_bytes;
  size_t smem;
};

__host__ __device__ inline TmaShape tma_shape(int H, int K) {
  TmaShape sh;
  int max_ch = int(kTmaStageTarget / (uint32_t(K) * 2u)) & ~7;
  if (max_ch < 8) max_ch = 8;
  sh.parts = (H + max_ch - 1) / max_ch;
  sh.part_ch = ((H + sh.parts - 1) / sh.parts + 7) & ~7;
  const int part_v = sh.part_ch / 8;
  int cw = (part_v + 31) / 32;
  sh.cw = cw < kTmaMaxConsumerWarps ? cw : kTmaMaxConsumerWarps;
  sh.in_bytes = al128(uint32_t(K) * uint32_t(sh.part_ch) * 2u);
  // stages, then per stage: full / empty barriers, mask, weights
  sh.smem = size_t(kTmaStages) * sh.in_bytes + size_t(kTmaStages) * (16 + 4 + 4 * 32) + 64;
  return sh;
}

__global__ void __launch_bounds__((kTmaMaxConsumerWarps + 1) * 32, 1)
    k_combine_tma(const uint16_t* __restrict__ y, const int32_t* __restrict__ pos,
                  Weights wts, int64_t N, int K, int H, int64_t cap,
                  uint16_t* __restrict__ out, int32_t* __restrict__ status) {
  extern __shared__ __align__(128) uint8_t smem[];
  const TmaShape sh = tma_shape(H, K);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cw = sh.cw;
  uint8_t* in_base = smem;
  uint8_t* meta = smem + size_t(kTmaStages) * sh.in_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(meta);
  uint64_t* empty = full + kTmaStages;
  uint32_t* vmask = reinterpret_cast<uint32_t*>(empty + kTmaStages);
  float* wk = reinterpret_cast<float*>(vmask + kTmaStages);  // [stages][32]
  const int64_t units = N * sh.parts;
  const bool forced = wait_forced(EP_WAIT_SITE_COMBINE);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTmaStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], uint32_t(cw));
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == cw) {
    // ---- producer warp: lane k handles the k-th gathered part-row --------
    // Positions run two units ahead and weights one: a receive-side weight
    // is read at its entry's row, so its load waits for the position, which
    // was loaded an iteration earlier. Both loads go out before the wait
    // for a free stage, which hides their latency.
    int it = 0;
    int64_t u = blockIdx.x;
    int p_n = -1, p_nn = -1;
    float w_n = 0.0f;
    if (u < units && lane < K) {
      const int64_t t0 = u / sh.parts;
      p_n = __ldg(pos + t0 * K + lane);
      w_n = entry_weight(wts, t0, K, lane, p_n, cap);
    }
    if (u + gridDim.x < units && lane < K)
      p_nn = __ldg(pos + ((u + gridDim.x) / sh.parts) * K + lane);
    for (; u < units; u += gridDim.x, ++it) {
      const int64_t t = u / sh.parts;
      const int part = int(u - t * sh.parts);
      const int c0 = part * sh.part_ch;
      const int len = min(sh.part_ch, H - c0);
      const uint32_t bytes = uint32_t(len) * 2u;
      const int p = p_n;
      const float wv = w_n;
      {  // the next unit's weight, and the position of the one after
        const int64_t un = u + gridDim.x, unn = un + gridDim.x;
        if (un < units && lane < K) {
          p_n = p_nn;
          w_n = entry_weight(wts, un / sh.parts, K, lane, p_n, cap);
        }
        if (unn < units && lane < K) p_nn = __ldg(pos + (unn / sh.parts) * K + lane);
      }
      if (wts.rows && wts.gathered && part == 0 && lane < K)
        wts.gathered[t * K + lane] = wv;
      const bool valid = lane < K && p >= 0 && p < cap;
      if (lane < K && p >= cap) report(status, EP_DEV_CAPACITY);
      const unsigned m = __ballot_sync(0xffffffffu, valid);
      const int s = it % kTmaStages;
      const uint32_t ph = uint32_t(it / kTmaStages) & 1u;
      bool ok = true;
      if (lane == 0 && it >= kTmaStages) ok = mbar_wait_bounded(&empty[s], ph ^ 1u, forced);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        if (lane == 0) report(status, EP_DEV_TIMEOUT);
        break;
      }
      // Every lane's weight is in shared memory before lane 0 arrives: the
      // arrive (a release) then covers the whole warp's writes, and the
      // consumers' wait on the phase (an acquire) sees them. The loads may
      // be issued before lane 0's arrive lands: the phase needs that arrive
      // as well as the bytes, whatever their order.
      wk[s * 32 + lane] = wv;
      if (lane == 0) vmask[s] = m;
      __syncwarp();
      if (lane == 0) mbar_arrive_expect_tx(&full[s], uint32_t(__popc(m)) * bytes);
      if (valid)
        bulk_g2s(in_base + size_t(s) * sh.in_bytes + size_t(lane) * sh.part_ch * 2,
                 y + int64_t(p) * H + c0, bytes, &full[s]);
    }
    // never leave with a load still writing shared memory
    if (lane == 0)
      for (int s = 0; s < kTmaStages && s < it; ++s) {
        const int last = it - 1 - ((it - 1 - s) % kTmaStages);
        if (!mbar_wait_bounded(&full[s], uint32_t(last / kTmaStages) & 1u))
          report(status, EP_DEV_TIMEOUT);
      }
    __syncwarp();
  } else {
    // ---- consumers: each warp follows the stages on its own and stores its
    // threads' 16-byte output vectors from registers ------------------------
    const int nthreads = cw * 32;
    int it = 0;
    for (int64_t u = blockIdx.x; u < units; u += gridDim.x, ++it) {
      const int64_t t = u / sh.parts;
      const int part = int(u - t * sh.parts);
      const int c0 = part * sh.part_ch;
      const int len = min(sh.part_ch, H - c0);
      const int s = it % kTmaStages;
      const uint32_t ph = uint32_t(it / kTmaStages) & 1u;
      bool ok = true;
      if (lane == 0) ok = mbar_wait_bounded(&full[s], ph, forced);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) {
        // the producer has stopped or the wait was forced: leave without
        // touching the stage (its producer waits on `empty` time out too)
        if (lane == 0) report(status, EP_DEV_TIMEOUT);
        break;
      }
      const uint32_t m = vmask[s];
      const uint8_t* st = in_base + size_t(s) * sh.in_bytes;
      for (int v = threadIdx.x; v < (len >> 3); v += nthreads) {
        float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
        for (int k = 0; k < K; ++k) {
          if (!((m >> k) & 1u)) continue;
          const uint4 d = *reinterpret_cast<const uint4*>(st + size_t(k) * sh.part_ch * 2 +
                                                          size_t(v) * 16);
          fma8(acc, wk[s * 32 + k], d);
        }
        st_v4(out + t * H + c0 + v * 8, pack8(acc));
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }
}

cudaError_t run_tma(const uint16_t* y, const int32_t* pos, const Weights& w,
                    int64_t N, int K, int H, int64_t cap, uint16_t* out,
                    int num_sms, int32_t* status, cudaStream_t stream) {
  const TmaShape sh = tma_shape(H, K);
  cudaError_t err = cudaFuncSetAttribute(
      k_combine_tma, cudaFuncAttributeMaxDynamicSharedMemorySize, int(sh.smem));
  if (err != cudaSuccess) return err;
  const int64_t units = N * sh.parts;
  const int64_t grid = std::max<int64_t>(1, std::min<int64_t>(units, num_sms));
  k_combine_tma<<<int(grid), (sh.cw + 1) * 32, sh.smem, stream>>>(
      y, pos, w, N, K, H, cap, out, status);
  return cudaGetLastError();
}

template <int KT, bool kRows>
cudaError_t run_k(const uint16_t* y, const int32_t* pos, const Weights& w,
                  int64_t N, int K, int H, int64_t cap, uint16_t* out,
                  int num_sms, int32_t* status, cudaStream_t stream) {
  const int V = H >> 3;
  // Threads per CTA: the fewest passes over the row with <= 512 threads.
  const int passes = (V + kCombineMaxThreads - 1) / kCombineMaxThreads;
  int threads = (V + passes - 1) / passes;
  threads = std::max(32, (threads + 31) / 32 * 32);
  int per_sm = 0;
  cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
      &per_sm, k_combine<KT, kRows>, threads, 0);
  if (err != cudaSuccess) return err;
  per_sm = std::max(1, per_sm);
  const int64_t grid =
      std::max<int64_t>(1, std::min<int64_t>(N, int64_t(num_sms) * per_sm));
  k_combine<KT, kRows><<<int(grid), threads, 0, stream>>>(y, pos, w, N, K, H,
                                                          cap, out, status);
  return cudaGetLastError();
}

template <int KT>
cudaError_t run(const uint16_t* y, const int32_t* pos, const Weights& w,
                int64_t N, int K, int H, int64_t cap, uint16_t* out,
                int num_sms, int32_t* status, cudaStream_t stream) {
  if (w.rows)
    return run_k<KT, true>(y, pos, w, N, K, H, cap, out, num_sms, status, stream);
  return run_k<KT, false>(y, pos, w, N, K, H, cap, out, num_sms, status, stream);
}

}  // namespace

cudaError_t set_wait_debug_combine(uint32_t sites, uint64_t budget_ns) {
  return set_wait_debug_here(sites, budget_ns);
}

cudaError_t launch_combine(const void* y_, const int32_t* pos, const float* w_tok,
                           const float* w_rows, float* gathered, int64_t N,
                           int K, int H, int64_t cap, void* out_, int num_sms,
                           int32_t* status, cudaStream_t stream) {
  const Weights w{w_rows ? nullptr : w_tok, w_rows, w_rows ? gathered : nullptr};
  const uint16_t* y = static_cast<const uint16_t*>(y_);
  uint16_t* out = static_cast<uint16_t*>(out_);
  // The TMA pipeline needs enough (token, part) units per SM to fill its
  // stages; small batches (decode) are faster with the register gather.
  const TmaShape sh = tma_shape(H, K);
  if (sh.smem <= 200 * 1024 && N * sh.parts >= 16 * int64_t(num_sms))
    return run_tma(y, pos, w, N, K, H, cap, out, num_sms, status, stream);
  switch (K) {
    case 1: return run<1>(y, pos, w, N, K, H, cap, out, num_sms, status, stream);
    case 2: return run<2>(y, pos, w, N, K, H, cap, out, num_sms, status, stream);
    case 4: return run<4>(y, pos, w, N, K, H, cap, out, num_sms, status, stream);
    case 6: return run<6>(y, pos, w, N, K, H, cap, out, num_sms, status, stream);
    case 8: return run<8>(y, pos, w, N, K, H, cap, out, num_sms, status, stream);
    default: return run<0>(y, pos, w, N, K, H, cap, out, num_sms, status, stream);
  }
}

}  // namespace ep
