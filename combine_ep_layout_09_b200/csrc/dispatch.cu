// dispatch.cu -- dispatch step 4: copy every token row to its K receive rows,
// optionally quantised to FP8 E4M3 with one fp32 scale per 128 channels.
//
// "Экспертный параллелизм (EP)", section "Что подтверждено": activations,
// not expert weights, travel to the experts. "DeepSeek开源周第二天：DeepEP深度
// 分析", section "性能": FP8 dispatch. "MoonEP核心功能深度剖析", section
// "2. 高效通信机制": rows land directly in their final expert-grouped
// position (computed by the layout kernels), no later permutation.
//
// One persistent CTA per (SM, slot). Its producer lane streams whole token
// rows global -> shared with 1-D bulk copies (TMA engine) into a ring of
// mbarrier-tracked stages; the consumer warps read a row from shared memory
// once, quantise it in registers when FP8 is asked for, and write each of its
// K destination rows with 16-byte stores. Reads are 1/(K+1) of the bytes, so
// the kernel is bound by HBM write bandwidth. Padding rows are zero-filled at
// the end by all warps.
#include <algorithm>

#include "ep_device.cuh"
#include "ep_launch.h"

namespace ep {
namespace {

constexpr int kUnitCh = 512;            // channels one warp covers per pass
constexpr int kMaxConsumerWarps = 16;   // H/512 rounded up, capped
constexpr int kMaxStages = 8;
constexpr size_t kStageBudget = 100 * 1024;  // shared bytes for the ring

__host__ __device__ constexpr uint32_t align128(uint32_t x) {
  return (x + 127u) & ~127u;
}

// Quantise 16 channels held by this lane; lanes 8g..8g+7 of the warp hold the
// 128 channels of one group. Returns the 16 codes, writes the group scale.
__device__ __forceinline__ uint4 quantize16(const uint4& a, const uint4& b,
                                            float& scale_out) {
  float x[16];
  const uint32_t wd[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[2 * i] = bf16_lo(wd[i]);
    x[2 * i + 1] = bf16_hi(wd[i]);
  }
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(x[i]));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
  const float scale = __fdiv_rn(amax, 448.0f);
  scale_out = scale;
  uint4 q = make_uint4(0u, 0u, 0u, 0u);
  if (scale != 0.0f) {
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t lo = e4m3x2(__fdiv_rn(x[4 * i], scale),
                                 __fdiv_rn(x[4 * i + 1], scale));
      const uint32_t hi = e4m3x2(__fdiv_rn(x[4 * i + 2], scale),
                                 __fdiv_rn(x[4 * i + 3], scale));
      w[i] = lo | (hi << 16);
    }
    q = make_uint4(w[0], w[1], w[2], w[3]);
  }
  return q;
}

template <bool kFp8>
__global__ void __launch_bounds__((kMaxConsumerWarps + 1) * 32)
    k_dispatch(const uint16_t* __restrict__ hidden, const float* __restrict__ w,
               const int32_t* __restrict__ pos, const int32_t* __restrict__ row_src,
               const int32_t* __restrict__ offsets, int64_t N, int K, int E,
               int H, int64_t cap, uint8_t* __restrict__ recv,
               float* __restrict__ scales, float* __restrict__ recv_w,
               int stages, int32_t* __restrict__ status) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int nwarps = blockDim.x >> 5;
  const int cw = nwarps - 1;  // consumer warps; the last warp produces
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t row_bytes = uint32_t(H) * 2u;
  const uint32_t stage_bytes = align128(row_bytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + size_t(stages) * stage_bytes);
  uint64_t* empty = full + kMaxStages;
  const int G = H >> 7;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], uint32_t(cw));
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == cw) {
    // ---- producer: one lane keeps `stages` token rows in flight ----------
    if (lane == 0) {
      int it = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < N; t += gridDim.x, ++it) {
        const int s = it % stages;
        const uint32_t ph = uint32_t(it / stages) & 1u;
        if (it >= stages && !mbar_wait_bounded(&empty[s], ph ^ 1u)) {
          report(status, EP_DEV_TIMEOUT);
          ok = false;
          break;
        }
        mbar_arrive_expect_tx(&full[s], row_bytes);
        bulk_g2s(smem + size_t(s) * stage_bytes, hidden + t * H, row_bytes, &full[s]);
      }
      // Drain: never leave the CTA with a bulk copy still writing its smem.
      if (!ok || true) {
        const int issued = it;
        for (int s = 0; s < stages && s < issued; ++s) {
          const int last = issued - 1 - ((issued - 1 - s) % stages);
          if (!mbar_wait_bounded(&full[s], uint32_t(last / stages) & 1u))
            report(status, EP_DEV_TIMEOUT);
        }
      }
    }
    __syncwarp();
  } else {
    // ---- consumers -----------------------------------------------------
    int it = 0;
    for (int64_t t = blockIdx.x; t < N; t += gridDim.x, ++it) {
      const int s = it % stages;
      const uint32_t ph = uint32_t(it / stages) & 1u;
      int p_l = -1;
      float w_l = 0.0f;
      if (lane < K) {
        p_l = __ldg(pos + t * K + lane);
        w_l = __ldg(w + t * K + lane);
        if (p_l >= cap) {
          report(status, EP_DEV_CAPACITY);
          p_l = -1;
        }
      }
      if (!mbar_wait_bounded(&full[s], ph)) {
        report(status, EP_DEV_TIMEOUT);
        break;
      }
      const uint8_t* row = smem + size_t(s) * stage_bytes;
      for (int u = warp; u * kUnitCh < H; u += cw) {
        const int c0 = u * kUnitCh + lane * 16;  // first channel of this lane
        const bool act0 = c0 < H;
        const bool act1 = c0 + 8 < H;
        uint4 a = make_uint4(0u, 0u, 0u, 0u), b = a;
        if (act0) a = *reinterpret_cast<const uint4*>(row + size_t(c0) * 2);
        if (act1) b = *reinterpret_cast<const uint4*>(row + size_t(c0) * 2 + 16);
        if constexpr (kFp8) {
          float scale;
          const uint4 q = quantize16(a, b, scale);  // whole warp (shuffles)
          const int g = c0 >> 7;
          for (int k = 0; k < K; ++k) {
            const int p = __shfl_sync(0xffffffffu, p_l, k);
            if (p < 0) continue;
            if (act0) {
              st_v4(recv + int64_t(p) * H + c0, q);
              if ((lane & 7) == 0) scales[int64_t(p) * G + g] = scale;
            }
          }
        } else {
          uint16_t* recv16 = reinterpret_cast<uint16_t*>(recv);
          for (int k = 0; k < K; ++k) {
            const int p = __shfl_sync(0xffffffffu, p_l, k);
            if (p < 0) continue;
            uint16_t* dst = recv16 + int64_t(p) * H + c0;
            if (act0) st_v4(dst, a);
            if (act1) st_v4(dst + 8, b);
          }
        }
      }
      if (warp == 0 && lane < K && p_l >= 0 && recv_w) recv_w[p_l] = w_l;
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }

  // ---- padding rows (row_src == -1 below off[E]): zeros ------------------
  const int64_t used = min(int64_t(__ldg(offsets + E)), cap);
  const int64_t gw = int64_t(blockIdx.x) * nwarps + warp;
  const int64_t gstride = int64_t(gridDim.x) * nwarps;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  for (int64_t r0 = gw * 32; r0 < used; r0 += gstride * 32) {
    const int64_t r = r0 + lane;
    const bool is_pad = r < used && __ldg(row_src + r) < 0;
    unsigned m = __ballot_sync(0xffffffffu, is_pad);
    while (m) {
      const int bit = __ffs(m) - 1;
      m &= m - 1;
      const int64_t row = r0 + bit;
      if constexpr (kFp8) {
        for (int c = lane * 16; c < H; c += 32 * 16) st_v4(recv + row * H + c, z);
        for (int g = lane; g < G; g += 32) scales[row * G + g] = 0.0f;
      } else {
        uint16_t* recv16 = reinterpret_cast<uint16_t*>(recv);
        for (int v = lane; v < (H >> 3); v += 32) st_v4(recv16 + row * H + v * 8, z);
      }
      if (lane == 0 && recv_w) recv_w[row] = 0.0f;
    }
  }
}

struct DispatchCfg {
  int threads = 0;
  int stages = 0;
  size_t smem = 0;
};

DispatchCfg dispatch_cfg(int H) {
  DispatchCfg c;
  const int units = (H + kUnitCh - 1) / kUnitCh;
  const int cw = std::min(units, kMaxConsumerWarps);
  c.threads = (cw + 1) * 32;
  const uint32_t stage_bytes = align128(uint32_t(H) * 2u);
  c.stages = int(std::max<size_t>(2, std::min<size_t>(kMaxStages, kStageBudget / stage_bytes)));
  c.smem = size_t(c.stages) * stage_bytes + 2 * kMaxStages * sizeof(uint64_t);
  return c;
}

}  // namespace

cudaError_t launch_dispatch(const void* hidden, const float* w,
                            const int32_t* pos, const int32_t* row_src,
                            const int32_t* expert_offsets, int64_t N, int K,
                            int E, int H, int64_t cap, bool fp8, void* recv,
                            float* recv_scales, float* recv_w, int num_sms,
                            int32_t* status, cudaStream_t stream) {
  const DispatchCfg c = dispatch_cfg(H);
  auto kern = fp8 ? k_dispatch<true> : k_dispatch<false>;
  cudaError_t err = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(c.smem));
  if (err != cudaSuccess) return err;
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, c.threads,
                                                      c.smem);
  if (err != cudaSuccess) return err;
  per_sm = std::max(1, per_sm);
  // Enough CTAs for the token rows and for the padding sweep.
  const int64_t grid = std::max<int64_t>(
      1, std::min<int64_t>(int64_t(num_sms) * per_sm,
                           std::max<int64_t>(N, (cap + 31) / 32)));
  kern<<<int(grid), c.threads, c.smem, stream>>>(
      static_cast<const uint16_t*>(hidden), w, pos, row_src, expert_offsets, N,
      K, E, H, cap, static_cast<uint8_t*>(recv), recv_scales, recv_w, c.stages,
      status);
  return cudaGetLastError();
}

}  // namespace ep
