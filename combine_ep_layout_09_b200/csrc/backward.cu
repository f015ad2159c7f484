// backward.cu -- the backward pair of dispatch / combine, and the gather of
// per-row values back into token order.
//
// "DeepSeek开源周第二天：DeepEP深度分析", section "DeepEP介绍": the kernels
// serve training as well as inference. "MoonEP核心功能深度剖析", section
// "快速上手": combine returns gathered_route_weights_sk next to the output,
// for the backward pass.
//
// combine:            out[t] = bf16( sum_k w[t,k] * y[pos[t,k]] )
// backward, rows:     grad_y[pos[t,k]] = bf16( w[t,k] * grad_out[t] )
// backward, weights:  grad_w[t,k] = sum_h y[pos[t,k], h] * grad_out[t, h]
// dispatch backward:  grad_hidden[t] = bf16( sum_k grad_recv[pos[t,k]] )
//                     (combine with unit weights: launch_combine, w = NULL)
//
// k_combine_bwd: CTAs walk tokens (one CTA per token when every SM is in
// use, persistent CTAs under a num_sms limit); threads split the row into
// 16-byte vectors. Each thread loads the grad_out vector and its K gathered
// expert-output vectors, accumulates the K dot products in fp32 (its
// vectors in order, channels in order), and stores the K scaled gradient
// vectors. The K partial sums are then reduced over the CTA in a fixed tree,
// so grad_w does not depend on timing.
#include <algorithm>

#include "ep_device.cuh"
#include "ep_launch.h"

namespace ep {
namespace {

constexpr int kBwdMaxThreads = 512;
constexpr int kBwdChunk = 8;  // k-terms loaded together

__device__ __forceinline__ float dot8(const uint4& d, const float (&g)[8],
                                      float acc) {
  acc = fmaf(bf16_lo(d.x), g[0], acc);
  acc = fmaf(bf16_hi(d.x), g[1], acc);
  acc = fmaf(bf16_lo(d.y), g[2], acc);
  acc = fmaf(bf16_hi(d.y), g[3], acc);
  acc = fmaf(bf16_lo(d.z), g[4], acc);
  acc = fmaf(bf16_hi(d.z), g[5], acc);
  acc = fmaf(bf16_lo(d.w), g[6], acc);
  acc = fmaf(bf16_hi(d.w), g[7], acc);
  return acc;
}

__device__ __forceinline__ uint4 scale8(const float (&g)[8], float wk) {
  return make_uint4(pack_bf16x2(wk * g[0], wk * g[1]), pack_bf16x2(wk * g[2], wk * g[3]),
                    pack_bf16x2(wk * g[4], wk * g[5]), pack_bf16x2(wk * g[6], wk * g[7]));
}

__global__ void __launch_bounds__(kBwdMaxThreads)
    k_combine_bwd(const uint16_t* __restrict__ grad_out,
                  const uint16_t* __restrict__ y, const int32_t* __restrict__ pos,
                  const int32_t* __restrict__ row_src,
                  const int32_t* __restrict__ offsets,
                  const float* __restrict__ w, int64_t N, int K, int E, int H,
                  int64_t cap, uint16_t* __restrict__ grad_rows,
                  float* __restrict__ grad_w, int32_t* __restrict__ status) {
  __shared__ float s_part[kBwdMaxThreads / 32][32];  // [warp][k]
  const int V = H >> 3;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nwarps = blockDim.x >> 5;
  for (int64_t t = blockIdx.x; t < N; t += gridDim.x) {
    const int32_t* pt = pos + t * K;
    const float* wt = w + t * K;
    for (int k0 = 0; k0 < K; k0 += kBwdChunk) {
      int64_t off[kBwdChunk];
      float wk[kBwdChunk], part[kBwdChunk];
#pragma unroll
      for (int j = 0; j < kBwdChunk; ++j) {
        off[j] = -1;
        wk[j] = 0.0f;
        part[j] = 0.0f;
        if (k0 + j < K) {
          const int32_t p = __ldg(pt + k0 + j);
          wk[j] = __ldg(wt + k0 + j);
          if (p >= 0 && p < cap) off[j] = int64_t(p) * H;
          if (p >= cap && threadIdx.x == 0) report(status, EP_DEV_CAPACITY);
        }
      }
      for (int v = threadIdx.x; v < V; v += blockDim.x) {
        const uint4 gv = ld_stream_v4(grad_out + t * H + v * 8);
        const float g[8] = {bf16_lo(gv.x), bf16_hi(gv.x), bf16_lo(gv.y), bf16_hi(gv.y),
                            bf16_lo(gv.z), bf16_hi(gv.z), bf16_lo(gv.w), bf16_hi(gv.w)};
        uint4 d[kBwdChunk];
#pragma unroll
        for (int j = 0; j < kBwdChunk; ++j)
          d[j] = off[j] >= 0 ? ld_stream_v4(y + off[j] + v * 8)
                             : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int j = 0; j < kBwdChunk; ++j) {
          if (off[j] < 0) continue;
          part[j] = dot8(d[j], g, part[j]);
          st_v4(grad_rows + off[j] + v * 8, scale8(g, wk[j]));
        }
      }
      // fixed-order reduction of the chunk's partial dot products
#pragma unroll
      for (int j = 0; j < kBwdChunk; ++j) {
        float x = part[j];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
        if (lane == 0) s_part[warp][j] = x;
      }
      __syncthreads();
      if (threadIdx.x < kBwdChunk && k0 + threadIdx.x < K) {
        float x = 0.0f;
        for (int ww = 0; ww < nwarps; ++ww) x += s_part[ww][threadIdx.x];
        grad_w[t * K + k0 + threadIdx.x] = x;
      }
      __syncthreads();
    }
  }

  // padding rows (row_src == -1 below off[E]): zero gradient
  const int64_t used = min(int64_t(__ldg(offsets + E)), cap);
  const int64_t gw = int64_t(blockIdx.x) * nwarps + warp;
  const int64_t gstride = int64_t(gridDim.x) * nwarps;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  // lane l of warp gw looks at row gw + (32*i + l) * gstride, so that the
  // padding rows of one expert (a contiguous run) fall to different warps
  for (int64_t i0 = 0; gw + i0 * gstride < used; i0 += 32) {
    const int64_t r = gw + (i0 + lane) * gstride;
    const bool is_pad = r < used && __ldg(row_src + r) < 0;
    unsigned m = __ballot_sync(0xffffffffu, is_pad);
    while (m) {
      const int bit = __ffs(m) - 1;
      m &= m - 1;
      const int64_t row = gw + (i0 + bit) * gstride;
      for (int v = lane; v < V; v += 32) st_v4(grad_rows + row * H + v * 8, z);
    }
  }
}

__global__ void k_gather_row_values(const float* __restrict__ vals,
                                    const int32_t* __restrict__ pos, int64_t n,
                                    int64_t cap, float* __restrict__ out) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += int64_t(gridDim.x) * blockDim.x) {
    const int32_t p = __ldg(pos + i);
    out[i] = (p >= 0 && p < cap) ? __ldg(vals + p) : 0.0f;
  }
}

}  // namespace

cudaError_t launch_combine_backward(const void* grad_out, const void* y,
                                    const int32_t* pos, const int32_t* row_src,
                                    const int32_t* expert_offsets,
                                    const float* w, int64_t N, int K, int E,
                                    int H, int64_t cap, void* grad_rows,
                                    float* grad_w, int num_sms,
                                    int32_t* status, cudaStream_t stream) {
  const int V = H >> 3;
  const int passes = (V + kBwdMaxThreads - 1) / kBwdMaxThreads;
  int threads = (V + passes - 1) / passes;
  threads = std::max(32, (threads + 31) / 32 * 32);
  int per_sm = 0;
  cudaError_t err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(
      &per_sm, k_combine_bwd, threads, 0);
  if (err != cudaSuccess) return err;
  // Every SM in use: one CTA per token, so that the CTAs start in token
  // order and the rows written at any moment belong to a narrow window of
  // tokens. A num_sms limit keeps persistent CTAs (a grid of short CTAs
  // cannot be held to fewer SMs).
  const int64_t resident = num_sms >= device_sm_count()
                               ? int64_t(INT32_MAX)
                               : int64_t(num_sms) * std::max(1, per_sm);
  const int64_t grid = std::max<int64_t>(
      1, std::min<int64_t>(resident, std::max<int64_t>(N, (cap + 31) / 32)));
  k_combine_bwd<<<int(grid), threads, 0, stream>>>(
      static_cast<const uint16_t*>(grad_out), static_cast<const uint16_t*>(y),
      pos, row_src, expert_offsets, w, N, K, E, H, cap,
      static_cast<uint16_t*>(grad_rows), grad_w, status);
  return cudaGetLastError();
}

cudaError_t launch_gather_row_values(const float* vals, const int32_t* pos,
                                     int64_t n, int64_t cap, float* out,
                                     cudaStream_t stream) {
  if (n == 0) return cudaSuccess;
  const int grid = int(std::min<int64_t>((n + 255) / 256, 148 * 8));
  k_gather_row_values<<<grid, 256, 0, stream>>>(vals, pos, n, cap, out);
  return cudaGetLastError();
}

}  // namespace ep
