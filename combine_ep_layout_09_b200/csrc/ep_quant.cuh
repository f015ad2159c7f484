// ep_quant.cuh -- FP8 E4M3 quantisation with one fp32 scale per 128
// channels, shared by every kernel that writes FP8 rows and by the
// diagnostic entry point, so that the tests exercise this exact code.
//
// Quantisation ("bracketed reciprocal"): the code must be e4m3(RN(x/s)) with
// the fp32 quotient correctly rounded. Take inv, the hardware's approximate
// reciprocal of s (rcp.approx, at most 1 ulp from 1/s: relative error below
// 2^-22). The products lo = RN(x * RN(inv*(1-2^-20))) and
// hi = RN(x * RN(inv*(1+2^-20))) then enclose RN(x/s): the reciprocal's
// error and each rounding move a value by far less than the 2^-20 margin.
// Rounding to E4M3 is monotone, so when lo and hi encode to the same code
// that code is e4m3(RN(x/s)). Otherwise the pair is recomputed with the
// correctly rounded division __fdiv_rn. That happens for about 3e-5 of the
// values, the ones within about 2^-20 of a rounding boundary. Values in the
// fp32 subnormal range all encode to +-0 on the correct side, so the
// bracket needs no normal-range assumption there. A scale outside
// [2^-125, 2^125], whose reciprocal could overflow or be flushed to zero,
// takes the division path for the whole group.
//
// The scale itself is RN(amax/448) with amax the group's largest |x|, a
// bf16 magnitude. scale_of_amax computes it as q = RN(amax * RN(1/448))
// corrected once by the remainder r = amax - 448q, which a fused
// multiply-add gives exactly: RN(q + r * RN(1/448)) (P. Markstein, IBM J.
// Res. Dev. 34(1), 1990). Over all 32640 finite non-negative bf16 values the
// result equals the correctly rounded quotient (checked with exact rational
// arithmetic; the uncorrected product is wrong for 17468 of them).
#pragma once

#include "ep_device.cuh"

namespace ep {
namespace {

// ---------------------------------------------------------------------------
// E4M3 quantisation of 16 values by one group scale
// ---------------------------------------------------------------------------

struct GroupScale {
  float scale;   // the group's fp32 scale
  float inv_lo;  // RN(RN(1/scale) * (1 - 2^-20))
  float inv_hi;  // RN(RN(1/scale) * (1 + 2^-20))
  bool bracket;  // reciprocal path valid (scale >= 2^-125)
};

__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// RN(amax / 448) for amax a finite non-negative bf16 value, or +inf.
__device__ __forceinline__ float scale_of_amax(float amax) {
  constexpr float kInv448 = 0x1.24924ap-9f;  // RN(1/448)
  const float q = __fmul_rn(amax, kInv448);
  const float r = __fmaf_rn(-q, 448.0f, amax);
  const float q1 = __fmaf_rn(r, kInv448, q);
  return amax <= 0x1.fffffep127f ? q1 : q;  // +inf: r would be NaN
}

__device__ __forceinline__ GroupScale make_group_scale(float scale) {
  GroupScale g;
  g.scale = scale;
  g.bracket = scale >= 0x1p-125f && scale <= 0x1p125f;
  const float inv = g.bracket ? rcp_approx(scale) : 0.0f;
  g.inv_lo = inv * (1.0f - 0x1p-20f);
  g.inv_hi = inv * (1.0f + 0x1p-20f);
  return g;
}

// Two codes (low byte = a) for e4m3(RN(a/scale)), e4m3(RN(b/scale)).
__device__ __forceinline__ uint32_t codes2_exact(float a, float b,
                                                 const GroupScale& g) {
  return e4m3x2(__fdiv_rn(a, g.scale), __fdiv_rn(b, g.scale));
}

// 16 codes of x[0..15] (scale != 0); bytes in channel order.
__device__ __forceinline__ uint4 quantize16(const float (&x)[16],
                                            const GroupScale& g) {
  uint32_t c[8];
  bool agree = g.bracket;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t lo = e4m3x2(x[2 * i] * g.inv_lo, x[2 * i + 1] * g.inv_lo);
    const uint32_t hi = e4m3x2(x[2 * i] * g.inv_hi, x[2 * i + 1] * g.inv_hi);
    agree = agree && (lo == hi);
    c[i] = lo;
  }
  if (!agree) {  // rare: some value sits on a rounding boundary
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t lo = e4m3x2(x[2 * i] * g.inv_lo, x[2 * i + 1] * g.inv_lo);
      const uint32_t hi = e4m3x2(x[2 * i] * g.inv_hi, x[2 * i + 1] * g.inv_hi);
      if (!g.bracket || lo != hi) c[i] = codes2_exact(x[2 * i], x[2 * i + 1], g);
    }
  }
  return make_uint4(c[0] | (c[1] << 16), c[2] | (c[3] << 16),
                    c[4] | (c[5] << 16), c[6] | (c[7] << 16));
}

// Unpack 16 bf16 (two 16-byte words) to fp32; returns max |x|.
__device__ __forceinline__ float unpack16(const uint4& a, const uint4& b,
                                          float (&x)[16]) {
  const uint32_t wd[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x[2 * i] = bf16_lo(wd[i]);
    x[2 * i + 1] = bf16_hi(wd[i]);
    amax = fmaxf(amax, fmaxf(fabsf(x[2 * i]), fabsf(x[2 * i + 1])));
  }
  return amax;
}

// Lane's share of a 512-channel unit of a bf16 row in shared memory: the 16
// channels [c0, c0+16), c0 = unit*512 + lane*16. Lanes 8g..8g+7 hold one
// 128-channel group, so the group amax takes three shuffles (all 32 lanes
// must call). Writes the 16 codes to codes + c0 when act, and returns the
// group's scale = amax / 448 (0 when not act and the group is idle).
__device__ __forceinline__ float quantize_lane16(const uint8_t* row,
                                                 uint8_t* codes, int c0,
                                                 bool act) {
  uint4 a = make_uint4(0u, 0u, 0u, 0u), b = a;
  if (act) {
    a = *reinterpret_cast<const uint4*>(row + size_t(c0) * 2);
    b = *reinterpret_cast<const uint4*>(row + size_t(c0) * 2 + 16);
  }
  float x[16];
  float amax = unpack16(a, b, x);
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
  amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
  const float scale = scale_of_amax(amax);
  uint4 q = make_uint4(0u, 0u, 0u, 0u);
  if (scale != 0.0f) q = quantize16(x, make_group_scale(scale));
  if (act) *reinterpret_cast<uint4*>(codes + c0) = q;
  return scale;
}

}  // namespace
}  // namespace ep
