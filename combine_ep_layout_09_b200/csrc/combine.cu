// combine.cu -- gather each token's K expert outputs and reduce them with the
// route weights, back in token order.
//
// "Экспертный параллелизм (EP)", section "Что подтверждено": expert results
// come back through the second AllToAll and are combined. "DeepSeek开源周第二天
// ：DeepEP深度分析", section "性能": BF16 combine. The sum is taken in fp32 with
// one fused multiply-add per k, k ascending from +0, then rounded to bf16
// (nearest even), so the result is a fixed function of its inputs.
//
// Persistent CTAs walk tokens; the threads of a CTA split the row into
// 16-byte vectors (8 channels). Each thread issues its K gathered loads
// before any arithmetic, so K * 16 bytes per thread are in flight. The kernel
// reads K rows per written row: it is bound by HBM read bandwidth.
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

// KT > 0: K known at compile time; KT == 0: runtime K, in chunks of kChunk
// terms (the chunks run in k order, so the fma order is unchanged).
template <int KT>
__global__ void __launch_bounds__(kCombineMaxThreads)
    k_combine(const uint16_t* __restrict__ y, const int32_t* __restrict__ pos,
              const float* __restrict__ w, int64_t N, int Kr, int H,
              int64_t cap, uint16_t* __restrict__ out,
              int32_t* __restrict__ status) {
  const int K = KT > 0 ? KT : Kr;
  const int V = H >> 3;
  for (int64_t t = blockIdx.x; t < N; t += gridDim.x) {
    const int32_t* pt = pos + t * K;
    const float* wt = w + t * K;
    if constexpr (KT > 0) {
      int64_t rowoff[KT];
      float wk[KT];
#pragma unroll
      for (int k = 0; k < KT; ++k) {
        const int32_t p = __ldg(pt + k);
        wk[k] = __ldg(wt + k);
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
              wk[j] = __ldg(wt + k0 + j);
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

template <int KT>
cudaError_t run(const uint16_t* y, const int32_t* pos, const float* w,
                int64_t N, int K, int H, int64_t cap, uint16_t* out,
                int num_sms, int32_t* status, cudaStream_t stream) {
  const int V = H >> 3;
  // Threads per CTA: the fewest passes over the row with <= 512 threads.
  const int passes = (V + kCombineMaxThreads - 1) / kCombineMaxThreads;
  int threads = (V + passes - 1) / passes;
  threads = std::max(32, (threads + 31) / 32 * 32);
  int per_sm = 0;
  cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
      &per_sm, k_combine<KT>, threads, 0);
  if (err != cudaSuccess) return err;
  per_sm = std::max(1, per_sm);
  const int64_t grid =
      std::max<int64_t>(1, std::min<int64_t>(N, int64_t(num_sms) * per_sm));
  k_combine<KT><<<int(grid), threads, 0, stream>>>(y, pos, w, N, K, H, cap,
                                                   out, status);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_combine(const void* y_, const int32_t* pos, const float* w,
                           int64_t N, int K, int H, int64_t cap, void* out_,
                           int num_sms, int32_t* status, cudaStream_t stream) {
  const uint16_t* y = static_cast<const uint16_t*>(y_);
  uint16_t* out = static_cast<uint16_t*>(out_);
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
