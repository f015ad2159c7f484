// dispatch.cu -- dispatch step 4: copy every token row to its K receive rows,
// optionally quantised to FP8 E4M3 with one fp32 scale per 128 channels.
//
// "Экспертный параллелизм (EP)", section "Что подтверждено": activations,
// not expert weights, travel to the experts. "DeepSeek开源周第二天：DeepEP深度
// 分析", section "性能": FP8 dispatch; section "代码解读": data movement through
// the TMA engine. "MoonEP核心功能深度剖析", section "2. 高效通信机制": rows land
// directly in their final expert-grouped position (computed by the layout
// kernels), with no later permutation.
//
// A token row is read once and written K times, so the kernels read
// 1/(K+1) of the bytes they move (bf16) and HBM write bandwidth bounds them.
// With every SM in use, one CTA per token:
//
//   k_dispatch_bf16_tok  each thread loads 32-byte vectors of the row (16
//                        bytes when the buffers are only 16-byte aligned)
//                        and stores each to the K rows.
//   k_dispatch_fp8_tok   each warp loads two 512-channel units, quantises
//                        them in registers and stores codes and scales to
//                        the K rows.
//
// Short CTAs start in token order, so the rows being written at any moment
// belong to a narrow window of tokens. A grid of short CTAs cannot be held
// to fewer SMs, so a num_sms limit takes the persistent kernels, which move
// rows with the TMA engine's 1-D bulk copies (no tensor map; each CTA loads
// only its own rows):
//
//   k_dispatch_bf16  one-warp CTAs; lane 0 keeps a ring of token rows in
//                    flight and, per row, issues K bulk stores from shared
//                    memory to the destination rows. No data passes through
//                    registers.
//   k_dispatch_fp8   a producer warp streams rows in; consumer warps
//                    quantise their 512-channel slice into an output stage
//                    in shared memory (codes, then the row's scales); one
//                    thread bulk-stores that stage K times.
//
// The E4M3 quantiser and its exactness argument are in ep_quant.cuh.
#include <algorithm>

#include "ep_device.cuh"
#include "ep_launch.h"
#include "ep_quant.cuh"

namespace ep {
namespace {

constexpr int kUnitCh = 512;           // channels one warp covers per pass
constexpr int kMaxConsumerWarps = 16;  // H/512 rounded up, capped
constexpr int kMaxStages = 8;

__host__ __device__ constexpr uint32_t align128(uint32_t x) {
  return (x + 127u) & ~127u;
}

// ---------------------------------------------------------------------------
// padding rows: zero payload, zero scales, zero weight (all warps of the grid)
// ---------------------------------------------------------------------------

template <bool kFp8>
__device__ void zero_padding_rows(const int32_t* __restrict__ row_src,
                                  const int32_t* __restrict__ offsets, int E,
                                  int H, int64_t cap, uint8_t* __restrict__ recv,
                                  float* __restrict__ scales,
                                  float* __restrict__ recv_w) {
  const int lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int64_t used = min(int64_t(__ldg(offsets + E)), cap);
  const int64_t gw = int64_t(blockIdx.x) * nwarps + (threadIdx.x >> 5);
  const int64_t gstride = int64_t(gridDim.x) * nwarps;
  const int G = H >> 7;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  // Lane l of warp gw looks at row gw + (32*i + l) * gstride: the padding
  // rows of one expert (a contiguous run) fall to different warps.
  for (int64_t i0 = 0; gw + i0 * gstride < used; i0 += 32) {
    const int64_t r = gw + (i0 + lane) * gstride;
    const bool is_pad = r < used && __ldg(row_src + r) < 0;
    unsigned m = __ballot_sync(0xffffffffu, is_pad);
    while (m) {
      const int bit = __ffs(m) - 1;
      m &= m - 1;
      const int64_t row = gw + (i0 + bit) * gstride;
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

// ---------------------------------------------------------------------------
// bf16: a pure TMA copy, one warp per CTA
// ---------------------------------------------------------------------------

__global__ void __launch_bounds__(32)
    k_dispatch_bf16(const uint16_t* __restrict__ hidden,
                    const float* __restrict__ w, const int32_t* __restrict__ pos,
                    const int32_t* __restrict__ row_src,
                    const int32_t* __restrict__ offsets, int64_t N, int K,
                    int E, int H, int64_t cap, uint8_t* __restrict__ recv,
                    float* __restrict__ recv_w, int stages,
                    int32_t* __restrict__ status) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x;
  const uint32_t row_bytes = uint32_t(H) * 2u;
  const uint32_t stage_bytes = align128(row_bytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + size_t(stages) * stage_bytes);
  const int64_t first = blockIdx.x, stride = gridDim.x;
  const int64_t n_mine = first < N ? (N - 1 - first) / stride + 1 : 0;
  const bool forced = wait_forced(EP_WAIT_SITE_DISPATCH);
  int64_t issued = 0;  // rows requested so far (lane 0)

  if (lane == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(&full[s], 1);
    fence_mbar_init();
    for (int64_t i = 0; i < stages && i < n_mine; ++i, ++issued) {
      mbar_arrive_expect_tx(&full[i], row_bytes);
      bulk_g2s(smem + size_t(i) * stage_bytes, hidden + (first + i * stride) * H,
               row_bytes, &full[i]);
    }
  }
  __syncwarp();
  grid_dependency_wait();  // pos / row_src / offsets may come from the layout

  bool ok = true;
  for (int64_t i = 0; i < n_mine && ok; ++i) {
    const int64_t t = first + i * stride;
    const int s = int(i % stages);
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
    if (lane == 0) ok = mbar_wait_bounded(&full[s], uint32_t(i / stages) & 1u, forced);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok) {
      if (lane == 0) report(status, EP_DEV_TIMEOUT);
      break;
    }
    for (int k = 0; k < K; ++k) {
      const int p = __shfl_sync(0xffffffffu, p_l, k);
      if (lane == 0 && p >= 0)
        bulk_s2g(recv + int64_t(p) * row_bytes, smem + size_t(s) * stage_bytes,
                 row_bytes);
    }
    if (lane == 0) {
      bulk_commit();
      // Refill the stage of the previous row once its stores have read it.
      const int64_t nxt = i - 1 + stages;
      if (i >= 1 && nxt < n_mine) {
        const int sp = int((i - 1) % stages);
        bulk_wait_read<1>();
        mbar_arrive_expect_tx(&full[sp], row_bytes);
        bulk_g2s(smem + size_t(sp) * stage_bytes, hidden + (first + nxt * stride) * H,
                 row_bytes, &full[sp]);
        ++issued;
      }
    }
    if (lane < K && p_l >= 0 && recv_w) recv_w[p_l] = w_l;
  }
  if (lane == 0) {
    // Loads still in flight after a give-up (the last row requested into
    // each stage), then all stores complete.
    if (!ok) {
      for (int64_t i = 0; i < stages && i < issued; ++i) {
        const int64_t last = issued - 1 - ((issued - 1 - i) % stages);
        mbar_wait_bounded(&full[i], uint32_t(last / stages) & 1u);
      }
    }
    bulk_wait_all<0>();
  }
  __syncwarp();
  zero_padding_rows<false>(row_src, offsets, E, H, cap, recv, nullptr, recv_w);
}

// ---------------------------------------------------------------------------
// fp8: producer warp + consumer warps, output stage bulk-stored K times
// ---------------------------------------------------------------------------

// Two CTAs share an SM (their stages take ~100 KB each), so a thread may
// use at most 60 registers: with 15 warps per CTA anything above 64 rounds
// to 72 per thread and leaves room for one CTA only.
__global__ void __launch_bounds__((kMaxConsumerWarps + 1) * 32, 2)
    k_dispatch_fp8(const uint16_t* __restrict__ hidden,
                   const float* __restrict__ w, const int32_t* __restrict__ pos,
                   const int32_t* __restrict__ row_src,
                   const int32_t* __restrict__ offsets, int64_t N, int K, int E,
                   int H, int64_t cap, uint8_t* __restrict__ recv,
                   float* __restrict__ scales, float* __restrict__ recv_w,
                   int s_in, int s_out, int32_t* __restrict__ status) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int nwarps = blockDim.x >> 5;
  const int cw = nwarps - 1;  // consumer warps; the last warp produces
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int G = H >> 7;
  const uint32_t row_bytes = uint32_t(H) * 2u;
  const uint32_t in_bytes = align128(row_bytes);
  const uint32_t scale_bytes = uint32_t(G) * 4u;
  const uint32_t out_bytes = align128(uint32_t(H) + scale_bytes);
  uint8_t* in_base = smem;
  uint8_t* out_base = smem + size_t(s_in) * in_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(out_base + size_t(s_out) * out_bytes);
  uint64_t* empty = full + kMaxStages;
  // Bulk stores need 16-byte multiples; the scales of a row qualify when
  // H is a multiple of 512, otherwise they are stored by the lanes.
  const bool bulk_scales = (scale_bytes % 16u) == 0u;
  const bool forced = wait_forced(EP_WAIT_SITE_DISPATCH);

  if (threadIdx.x == 0) {
    for (int s = 0; s < s_in; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], uint32_t(cw));
    }
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == cw) {
    // ---- producer -------------------------------------------------------
    if (lane == 0) {
      int it = 0;
      for (int64_t t = blockIdx.x; t < N; t += gridDim.x, ++it) {
        const int s = it % s_in;
        const uint32_t ph = uint32_t(it / s_in) & 1u;
        if (it >= s_in && !mbar_wait_bounded(&empty[s], ph ^ 1u, forced)) {
          report(status, EP_DEV_TIMEOUT);
          break;
        }
        mbar_arrive_expect_tx(&full[s], row_bytes);
        bulk_g2s(in_base + size_t(s) * in_bytes, hidden + t * H, row_bytes, &full[s]);
      }
      // never leave the CTA with a load still writing its shared memory
      for (int s = 0; s < s_in && s < it; ++s) {
        const int last = it - 1 - ((it - 1 - s) % s_in);
        if (!mbar_wait_bounded(&full[s], uint32_t(last / s_in) & 1u))
          report(status, EP_DEV_TIMEOUT);
      }
    }
    __syncwarp();
  } else {
    // ---- consumers --------------------------------------------------------
    const bool issuer = (warp == 0 && lane == 0);
    grid_dependency_wait();  // pos may come from the layout kernel ahead
    int it = 0;
    for (int64_t t = blockIdx.x; t < N; t += gridDim.x, ++it) {
      const int s = it % s_in;
      const uint32_t ph = uint32_t(it / s_in) & 1u;
      uint8_t* out = out_base + size_t(it % s_out) * out_bytes;
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
      bool ok = true;
      if (lane == 0) ok = mbar_wait_bounded(&full[s], ph, forced);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok && lane == 0) report(status, EP_DEV_TIMEOUT);
      const uint8_t* row = in_base + size_t(s) * in_bytes;
      for (int u = warp; u * kUnitCh < H; u += cw) {
        const int c0 = u * kUnitCh + lane * 16;  // first channel of this lane
        const bool act = c0 < H;                 // H % 128 == 0: whole groups
        const float scale = quantize_lane16(row, out, c0, act && ok);
        if (act && bulk_scales && (lane & 7) == 0)
          reinterpret_cast<float*>(out + H)[c0 >> 7] = scale;
        if (!bulk_scales) {
          // lanes store their group's scale to every destination row
          for (int k = 0; k < K; ++k) {
            const int p = __shfl_sync(0xffffffffu, p_l, k);
            if (act && (lane & 7) == 0 && p >= 0)
              scales[int64_t(p) * G + (c0 >> 7)] = scale;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
      if (warp == 0 && lane < K && p_l >= 0 && recv_w) recv_w[p_l] = w_l;
      // make this token's output stage visible to the bulk-copy engine
      fence_proxy_async_smem();
      // before the barrier: the stage the next token writes must have been
      // read by its earlier stores (at most s_out - 2 groups left pending)
      if (issuer) {
        if (s_out >= 3)
          bulk_wait_read<1>();
        else
          bulk_wait_read<0>();
      }
      // every consumer warp leaves together once any of them gave up
      if (named_barrier_or(1, cw * 32, !ok)) break;
      // lane 0 of warp 0 issues the stores; the positions reach it through a
      // shuffle that the whole warp executes
      if (warp == 0) {
        for (int k = 0; k < K; ++k) {
          const int p = __shfl_sync(0xffffffffu, p_l, k);
          if (lane == 0 && p >= 0) {
            bulk_s2g(recv + int64_t(p) * H, out, uint32_t(H));
            if (bulk_scales)
              bulk_s2g(scales + int64_t(p) * G, out + H, scale_bytes);
          }
        }
        if (lane == 0) bulk_commit();
      }
    }
    if (issuer) bulk_wait_all<0>();
  }
  grid_dependency_wait();  // row_src / offsets may come from the layout
  __syncthreads();
  zero_padding_rows<true>(row_src, offsets, E, H, cap, recv, scales, recv_w);
}

// ---------------------------------------------------------------------------
// bf16, one token per CTA (every SM in use): the threads load the token row
// in 32-byte vectors (kWide: hidden and recv 32-byte aligned, H % 16 == 0;
// else 16-byte vectors) and store each to the K rows. CTAs are short and
// the hardware starts them in token order, so the rows being written at any
// moment belong to a narrow, advancing window of tokens; persistent CTAs
// drift apart and spread the writes over many more DRAM pages (measured on
// this part: the FP8 dispatch's store pattern alone ran at 7.1 TB/s with one
// CTA per token against 5.9-6.1 TB/s from persistent CTAs).
// ---------------------------------------------------------------------------

template <bool kWide>
__global__ void __launch_bounds__(kMaxConsumerWarps * 32)
    k_dispatch_bf16_tok(const uint16_t* __restrict__ hidden,
                        const float* __restrict__ w,
                        const int32_t* __restrict__ pos,
                        const int32_t* __restrict__ row_src,
                        const int32_t* __restrict__ offsets, int64_t N, int K,
                        int E, int H, int64_t cap, uint8_t* __restrict__ recv,
                        float* __restrict__ recv_w,
                        int32_t* __restrict__ status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int kVec = kWide ? 16 : 8;  // channels a thread moves at once
  const int V = H / kVec;               // vectors of a row
  uint16_t* recv16 = reinterpret_cast<uint16_t*>(recv);
  grid_dependency_wait();  // pos / row_src / offsets may come from the layout
  for (int64_t t = blockIdx.x; t < N; t += gridDim.x) {
    int p_l = -1;
    float w_l = 0.0f;
    if (lane < K) {
      p_l = __ldg(pos + t * K + lane);
      if (warp == 0) w_l = __ldg(w + t * K + lane);
      if (p_l >= cap) {
        if (warp == 0) report(status, EP_DEV_CAPACITY);
        p_l = -1;
      }
    }
    const uint16_t* row = hidden + t * H;
    // warp-uniform loop: every lane takes part in the shuffles
    for (int v0 = warp * 32; v0 < V; v0 += blockDim.x) {
      const int v = v0 + lane;
      uint4 d = make_uint4(0u, 0u, 0u, 0u), d1 = d;
      if (v < V) {
        if constexpr (kWide)
          ld_stream_v8(row + v * kVec, d, d1);
        else
          d = ld_stream_v4(row + v * kVec);
      }
      for (int k = 0; k < K; ++k) {
        const int p = __shfl_sync(0xffffffffu, p_l, k);
        if (p >= 0 && v < V) {
          if constexpr (kWide)
            st_v8(recv16 + int64_t(p) * H + v * kVec, d, d1);
          else
            st_v4(recv16 + int64_t(p) * H + v * kVec, d);
        }
      }
    }
    if (warp == 0 && lane < K && p_l >= 0 && recv_w) recv_w[p_l] = w_l;
  }
  zero_padding_rows<false>(row_src, offsets, E, H, cap, recv, nullptr, recv_w);
}

// ---------------------------------------------------------------------------
// FP8, one token per CTA (every SM in use): each warp loads two 512-channel
// units of the row (a lane's 32 bytes of a unit in one load when kWide:
// hidden 32-byte aligned) before it quantises either, then
// quantises each unit in registers (a lane's 16 channels, 8 lanes per
// 128-channel group, as in the persistent kernel) and stores its 16 codes to
// the K rows; lanes 8g store the group's scale. 224 threads cover H=7168, so
// four CTAs share an SM: four token rows in flight per SM, written in token
// order as in the bf16 form.
// ---------------------------------------------------------------------------

constexpr int kFp8TokUnits = 2;     // 512-channel units a warp holds at once
constexpr int kFp8TokMaxWarps = 7;  // H/1024 rounded up, capped (H=7168)

template <bool kWide>
__global__ void __launch_bounds__(kFp8TokMaxWarps * 32, 4)
    k_dispatch_fp8_tok(const uint16_t* __restrict__ hidden,
                       const float* __restrict__ w,
                       const int32_t* __restrict__ pos,
                       const int32_t* __restrict__ row_src,
                       const int32_t* __restrict__ offsets, int64_t N, int K,
                       int E, int H, int64_t cap, uint8_t* __restrict__ recv,
                       float* __restrict__ scales, float* __restrict__ recv_w,
                       int32_t* __restrict__ status) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = blockDim.x >> 5;
  const int G = H >> 7;
  bool waited = false;
  for (int64_t t = blockIdx.x; t < N; t += gridDim.x) {
    const uint16_t* row = hidden + t * H;
    // warp-uniform loop over passes of nwarps * kFp8TokUnits units
    for (int u0 = warp; u0 * kUnitCh < H; u0 += nwarps * kFp8TokUnits) {
      uint4 a[kFp8TokUnits], b[kFp8TokUnits];
#pragma unroll
      for (int j = 0; j < kFp8TokUnits; ++j) {
        const int c0 = (u0 + j * nwarps) * kUnitCh + lane * 16;
        a[j] = b[j] = make_uint4(0u, 0u, 0u, 0u);
        if (c0 < H) {
          if constexpr (kWide) {
            ld_stream_v8(row + c0, a[j], b[j]);
          } else {
            a[j] = ld_stream_v4(row + c0);
            b[j] = ld_stream_v4(row + c0 + 8);
          }
        }
      }
      // the rows do not depend on the layout ahead; the positions do
      if (!waited) {
        grid_dependency_wait();
        waited = true;
      }
      int p_l = -1;
      if (lane < K) {
        p_l = __ldg(pos + t * K + lane);
        if (p_l >= cap) {
          if (warp == 0 && u0 == warp) report(status, EP_DEV_CAPACITY);
          p_l = -1;
        }
      }
#pragma unroll
      for (int j = 0; j < kFp8TokUnits; ++j) {
        const int c0 = (u0 + j * nwarps) * kUnitCh + lane * 16;
        const bool act = c0 < H;  // H % 128 == 0: whole groups
        float x[16];
        float amax = unpack16(a[j], b[j], x);
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
        const float scale = scale_of_amax(amax);
        uint4 q = make_uint4(0u, 0u, 0u, 0u);
        if (scale != 0.0f) q = quantize16(x, make_group_scale(scale));
        for (int k = 0; k < K; ++k) {
          const int p = __shfl_sync(0xffffffffu, p_l, k);
          if (act && p >= 0) {
            st_v4(recv + int64_t(p) * H + c0, q);
            if ((lane & 7) == 0) scales[int64_t(p) * G + (c0 >> 7)] = scale;
          }
        }
      }
    }
    if (warp == 0 && lane < K && recv_w) {
      const int p = __ldg(pos + t * K + lane);
      if (p >= 0 && p < cap) recv_w[p] = __ldg(w + t * K + lane);
    }
  }
  if (!waited) grid_dependency_wait();  // row_src / offsets from the layout
  zero_padding_rows<true>(row_src, offsets, E, H, cap, recv, scales, recv_w);
}

__global__ void k_debug_quantize(const float* __restrict__ x,
                                 const float* __restrict__ scale,
                                 uint8_t* __restrict__ out, int64_t n) {
  // x is [n/16][16], scale one value per 16 values; exercises quantize16
  const int64_t groups = n / 16;
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < groups;
       i += int64_t(gridDim.x) * blockDim.x) {
    float v[16];
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = x[i * 16 + j];
    const float s = scale[i];
    uint4 q = make_uint4(0u, 0u, 0u, 0u);
    if (s != 0.0f) q = quantize16(v, make_group_scale(s));
    *reinterpret_cast<uint4*>(out + i * 16) = q;
  }
}

struct Cfg {
  int threads = 0;
  int s_in = 0;
  int s_out = 0;
  size_t smem = 0;
};

Cfg fp8_cfg(int H) {
  Cfg c;
  const int units = (H + kUnitCh - 1) / kUnitCh;
  const int cw = std::min(units, kMaxConsumerWarps);
  c.threads = (cw + 1) * 32;
  const uint32_t in_bytes = align128(uint32_t(H) * 2u);
  const uint32_t out_bytes = align128(uint32_t(H) + uint32_t(H / 128) * 4u);
  // ~100 KB per CTA so that two CTAs share an SM
  c.s_in = int(std::max<size_t>(2, std::min<size_t>(4, (64 * 1024) / in_bytes)));
  c.s_out = int(std::max<size_t>(2, std::min<size_t>(3, (36 * 1024) / out_bytes)));
  c.smem = size_t(c.s_in) * in_bytes + size_t(c.s_out) * out_bytes +
           2 * kMaxStages * sizeof(uint64_t);
  return c;
}

Cfg bf16_cfg(int H) {
  Cfg c;
  c.threads = 32;
  const uint32_t in_bytes = align128(uint32_t(H) * 2u);
  c.s_in = int(std::max<size_t>(2, std::min<size_t>(kMaxStages, (72 * 1024) / in_bytes)));
  c.smem = size_t(c.s_in) * in_bytes + kMaxStages * sizeof(uint64_t);
  return c;
}

}  // namespace

cudaError_t set_wait_debug_dispatch(uint32_t sites, uint64_t budget_ns) {
  return set_wait_debug_here(sites, budget_ns);
}

cudaError_t launch_dispatch(const void* hidden, const float* w,
                            const int32_t* pos, const int32_t* row_src,
                            const int32_t* expert_offsets, int64_t N, int K,
                            int E, int H, int64_t cap, bool fp8, void* recv,
                            float* recv_scales, float* recv_w, int num_sms,
                            int32_t* status, cudaStream_t stream, bool pdl) {
  const uint16_t* h = static_cast<const uint16_t*>(hidden);
  uint8_t* r = static_cast<uint8_t*>(recv);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  const bool all_sms = num_sms >= device_sm_count();
  // 32-byte accesses where every row start is 32-byte aligned
  const bool in32 = (reinterpret_cast<uintptr_t>(hidden) & 31u) == 0;
  const bool out32 = (reinterpret_cast<uintptr_t>(recv) & 31u) == 0;
  if (all_sms && fp8) {
    // FP8 on every SM: one CTA per token, as for bf16 below
    const int units = (H + kUnitCh - 1) / kUnitCh;
    const int warps = std::min(
        kFp8TokMaxWarps, (units + kFp8TokUnits - 1) / kFp8TokUnits);
    const int64_t pad_ctas = ((cap + 31) / 32 + warps - 1) / warps;
    const int64_t grid = std::max<int64_t>(
        1, std::min<int64_t>(INT32_MAX, std::max<int64_t>(N, pad_ctas)));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(grid));
    cfg.blockDim = dim3(unsigned(warps * 32));
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    // H % 128 == 0: every row start is as aligned as the buffer
    auto kern = in32 ? k_dispatch_fp8_tok<true> : k_dispatch_fp8_tok<false>;
    return cudaLaunchKernelEx(&cfg, kern, h, w, pos, row_src, expert_offsets,
                              N, K, E, H, cap, r, recv_scales, recv_w, status);
  }
  if (all_sms && !fp8) {
    // bf16 on every SM: one CTA per token (a grid of N short CTAs cannot be
    // held to fewer SMs, so a num_sms limit takes the persistent kernel)
    const bool wide = in32 && out32 && H % 16 == 0;
    const int V = wide ? H >> 4 : H >> 3;
    const int passes = (V + kMaxConsumerWarps * 32 - 1) / (kMaxConsumerWarps * 32);
    const int threads = std::max(32, ((V + passes - 1) / passes + 31) / 32 * 32);
    const int64_t pad_ctas = ((cap + 31) / 32 + threads / 32 - 1) / (threads / 32);
    const int64_t grid = std::max<int64_t>(
        1, std::min<int64_t>(INT32_MAX, std::max<int64_t>(N, pad_ctas)));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(unsigned(grid));
    cfg.blockDim = dim3(unsigned(threads));
    cfg.stream = stream;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    auto kern = wide ? k_dispatch_bf16_tok<true> : k_dispatch_bf16_tok<false>;
    return cudaLaunchKernelEx(&cfg, kern, h, w, pos, row_src, expert_offsets,
                              N, K, E, H, cap, r, recv_w, status);
  }
  const Cfg c = fp8 ? fp8_cfg(H) : bf16_cfg(H);
  const void* kern = fp8 ? reinterpret_cast<const void*>(k_dispatch_fp8)
                         : reinterpret_cast<const void*>(k_dispatch_bf16);
  cudaError_t err = cudaFuncSetAttribute(
      kern, cudaFuncAttributeMaxDynamicSharedMemorySize, int(c.smem));
  if (err != cudaSuccess) return err;
  int per_sm = 0;
  err = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, c.threads,
                                                      c.smem);
  if (err != cudaSuccess) return err;
  per_sm = std::max(1, per_sm);
  // Persistent CTAs on the SMs allowed, each taking every grid-th token:
  // enough CTAs for the token rows and for the padding sweep.
  const int64_t grid = std::max<int64_t>(
      1, std::min<int64_t>(int64_t(num_sms) * per_sm,
                           std::max<int64_t>(N, (cap + 31) / 32)));
  // With pdl the launch may begin while the kernel ahead of it (the layout
  // that wrote pos / row_src / offsets) is still running; the kernels wait
  // for it before reading those.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned(grid));
  cfg.blockDim = dim3(unsigned(c.threads));
  cfg.dynamicSmemBytes = c.smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  if (fp8)
    return cudaLaunchKernelEx(&cfg, k_dispatch_fp8, h, w, pos, row_src,
                              expert_offsets, N, K, E, H, cap, r, recv_scales,
                              recv_w, c.s_in, c.s_out, status);
  return cudaLaunchKernelEx(&cfg, k_dispatch_bf16, h, w, pos, row_src,
                            expert_offsets, N, K, E, H, cap, r, recv_w, c.s_in,
                            status);
}

cudaError_t launch_debug_quantize(const float* x, const float* scale,
                                  uint8_t* out, int64_t n, cudaStream_t stream) {
  const int64_t groups = n / 16;
  if (groups == 0) return cudaSuccess;
  const int grid = int(std::min<int64_t>((groups + 255) / 256, 148 * 16));
  k_debug_quantize<<<grid, 256, 0, stream>>>(x, scale, out, n);
  return cudaGetLastError();
}

}  // namespace ep
