// quant_impl.cuh -- device code of the FP8 (e4m3) quantisation of 1x128
// groups and 128x128 blocks, shared by the quantiser kernels (quant.cu) and
// the expert dispatch (moe.cu).
//
//   scale = amax / 448 (FP32; 1 for an all-zero group),
//   code  = e4m3_rne_satfinite(x / scale)   (one IEEE FP32 division)
//
// The division.  A full IEEE division per element would make the kernels
// ALU-bound.  Only the e4m3 code of the quotient matters, and that code
// changes only where the quotient crosses a rounding midpoint between two
// e4m3 values.  So each element first takes q0 = x * r with r the correctly
// rounded reciprocal of the group's scale: q0 is within 2.5 FP32 ulps of the
// correctly rounded quotient fl(x / s).  When q0 lies more than 8 ulps from
// every e4m3 midpoint, both round to the same code and q0 is used; otherwise
// an exact test decides on which side of the midpoint fl(x / s) lies
// (midpoint_side, no division).  bf16 inputs put about 0.5 % of quotients on
// or next to a midpoint.  The codes are therefore those of e4m3(fl(x / s)),
// bit for bit.
#pragma once

#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace fp8g {
namespace quant {

constexpr float kE4M3Max = 448.0f;
constexpr int kUnits = 8;  // 16-byte loads per lane in flight per warp

__device__ __forceinline__ float scale_of(float amax) { return amax > 0.f ? __fdiv_rn(amax, kE4M3Max) : 1.f; }

// True when q0 is more than 8 ulps away from every rounding midpoint of e4m3
// (normal range |q0| >= 2^-6: the midpoint sits where the 20 mantissa bits
// below e4m3's 3 are 0x80000; subnormal range: quantum 2^-9, midpoints at odd
// multiples of 2^-10, checked on |q0| * 512 with a margin of 2^-17).
__device__ __forceinline__ bool far_from_midpoint(float q0) {
  const uint32_t a = __float_as_uint(q0) & 0x7FFFFFFFu;
  if (a >= 0x3C800000u) {  // 2^-6
    const int low = static_cast<int>(a & 0xFFFFFu) - 0x80000;
    return low > 8 || low < -8;
  }
  const float t = __uint_as_float(a) * 512.f;
  const float d = t - floorf(t) - 0.5f;
  return fabsf(d) > 7.62939453e-06f;  // 2^-17
}

// Two floats -> two e4m3 codes (round to nearest even, saturating at +-448),
// lo in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// For a quotient near an e4m3 rounding midpoint: a value that converts to the
// same e4m3 code as fl(x / s).  q0 = x * r lies within 2.5 ulps of fl(x / s)
// and within 8 ulps of the midpoint m nearest to it.  m has at most 5
// significant bits, so d = x - m * s is a multiple of 2^(e_m + e_s - 27) of
// at most 9 bits and the FMA computes it exactly; with s > 0,
//   |d| <= ulp(m)/2 * s  <=>  fl(x / s) == m  (m's last bit is even, so a tie
//                              of the FP32 rounding also lands on m),
//   d > ulp(m)/2 * s     <=>  fl(x / s) lies above m,  d < -... below it.
// On m itself the conversion breaks the e4m3 tie to even; off it, the next
// float on the correct side of m converts to the correct neighbour.
__device__ __forceinline__ float midpoint_side(float x, float s, float q0) {
  const uint32_t sign = __float_as_uint(q0) & 0x80000000u;
  const uint32_t a = __float_as_uint(q0) & 0x7FFFFFFFu;
  uint32_t mb;  // |m|
  if (a >= 0x3C800000u) {
    mb = (a & 0xFFF00000u) | 0x00080000u;  // keep exponent and 3 mantissa bits, set the half bit
  } else {
    const float t = __uint_as_float(a) * 512.f;
    mb = __float_as_uint((floorf(t) + 0.5f) * 0.001953125f);  // (k + 1/2) * 2^-9
  }
  const float m = __uint_as_float(mb | sign);
  const float d = fmaf(-m, s, x);
  const float half_ulp = __uint_as_float(((mb >> 23) - 24u) << 23);  // 2^(e_m - 24)
  const float lim = half_ulp * s;
  if (fabsf(d) <= lim) return m;
  return __uint_as_float((d > 0.f) == (sign == 0u) ? (mb + 1u) | sign : (mb - 1u) | sign);
}

// Codes of n values of one group with scale s, packed 4 per 32-bit word
// (lowest element in the lowest byte).  Each value takes the fast quotient
// q0 = x * r (r = 1/s correctly rounded); the few that lie near an e4m3
// midpoint are settled by midpoint_side, one per lane and loop trip, so the
// code for them exists once.  A group with a scale below 2^-90 is first
// scaled by 2^100 together with its values (exact), so that the reciprocal
// and the midpoint test stay in the normal range; no scale can exceed
// FLT_MAX / 448, so no group needs the opposite.  Every lane of the warp must
// call it (the loop runs while any lane has work).
template <int n>
__device__ __forceinline__ void encode_group(const float (&v)[n], float s, uint32_t (&c)[n / 4]) {
  const float k = s < 8.07793567e-28f ? 1.26765060e30f : 1.f;  // 2^-90, 2^100
  const float ss = s * k;
  const float r = __frcp_rn(ss);
  float qv[n];
  uint32_t near = 0u;
#pragma unroll
  for (int i = 0; i < n; ++i) {
    qv[i] = (v[i] * k) * r;
    if (!far_from_midpoint(qv[i])) near |= 1u << i;
  }
  while (__any_sync(0xffffffffu, near != 0u)) {
    const int idx = near != 0u ? __ffs(near) - 1 : 0;
    float xi = v[0], qi = qv[0];
#pragma unroll
    for (int j = 1; j < n; ++j)
      if (idx == j) xi = v[j], qi = qv[j];
    const float fixed = midpoint_side(xi * k, ss, qi);
    if (near != 0u) {
#pragma unroll
      for (int j = 0; j < n; ++j)
        if (idx == j) qv[j] = fixed;
    }
    near &= near - 1u;
  }
#pragma unroll
  for (int i = 0; i < n / 4; ++i)
    c[i] = e4m3x2(qv[4 * i], qv[4 * i + 1]) | (e4m3x2(qv[4 * i + 2], qv[4 * i + 3]) << 16);
}


// One row of K elements (K % 128 == 0) quantised per 1x128 group by one warp.
// store_codes(offset, c) stores a lane's codes c (kPerLane / 4 words) for the
// row's elements offset .. offset + kPerLane - 1; store_scale(kb, scale) is
// called by one lane per group.
// Every lane loads 16 bytes per step: for bf16 input a half-warp covers one
// group (8 elements per lane), so a warp step covers two groups of the row;
// for FP32 input a warp covers one group (4 elements per lane).  kUnits steps
// (kUnits * 16 bytes per lane) are in flight.  All 32 lanes must call it.
template <bool kF32, typename StoreCodes, typename StoreScale>
__device__ __forceinline__ void quantize_row_1x128(const void* __restrict__ x_row, int K, StoreCodes store_codes,
                                                   StoreScale store_scale) {
  constexpr int kPerLane = kF32 ? 4 : 8;          // elements per lane per step
  constexpr int kLanesPerGroup = 128 / kPerLane;  // 32 (f32) or 16 (bf16)
  constexpr int kGroupsPerStep = 32 / kLanesPerGroup;
  const int lane = threadIdx.x & 31;
  const int KB = K / 128;
  const int steps = (KB + kGroupsPerStep - 1) / kGroupsPerStep;
  const int sub = lane / kLanesPerGroup;  // which group of the step
  const int l = lane % kLanesPerGroup;    // lane within the group
  for (int s0 = 0; s0 < steps; s0 += kUnits) {
    uint4 raw[kUnits];
#pragma unroll
    for (int j = 0; j < kUnits; ++j) {
      const int kb = (s0 + j) * kGroupsPerStep + sub;
      if (s0 + j < steps && kb < KB) {
        const long e = static_cast<long>(kb) * 128 + l * kPerLane;
        raw[j] = kF32 ? __ldcs(reinterpret_cast<const uint4*>(static_cast<const float*>(x_row) + e))
                      : __ldcs(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x_row) + e));
      } else {
        raw[j] = make_uint4(0u, 0u, 0u, 0u);
      }
    }
#pragma unroll
    for (int j = 0; j < kUnits; ++j) {
      if (s0 + j >= steps) continue;  // warp-uniform
      const int kb = (s0 + j) * kGroupsPerStep + sub;
      float v[kPerLane];
      if constexpr (kF32) {
        v[0] = __uint_as_float(raw[j].x), v[1] = __uint_as_float(raw[j].y);
        v[2] = __uint_as_float(raw[j].z), v[3] = __uint_as_float(raw[j].w);
      } else {
        const uint32_t wd[4] = {raw[j].x, raw[j].y, raw[j].z, raw[j].w};
#pragma unroll
        for (int i = 0; i < 4; ++i)
          v[2 * i] = __uint_as_float(wd[i] << 16), v[2 * i + 1] = __uint_as_float(wd[i] & 0xFFFF0000u);
      }
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < kPerLane; ++i) amax = fmaxf(amax, fabsf(v[i]));
#pragma unroll
      for (int o = kLanesPerGroup / 2; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const float sc = scale_of(amax);
      uint32_t c[kPerLane / 4];
      encode_group(v, sc, c);
      if (kb < KB) {
        store_codes(static_cast<long>(kb) * 128 + l * kPerLane, c);
        if (l == 0) store_scale(kb, sc);
      }
    }
  }
}

// Stores one lane's codes (4 bytes for FP32 input, 8 for bf16) at q.
template <int n>
__device__ __forceinline__ void store_code_words(uint8_t* q, const uint32_t (&c)[n]) {
  if constexpr (n == 1) {
    __stcs(reinterpret_cast<uint32_t*>(q), c[0]);
  } else {
    __stcs(reinterpret_cast<uint2*>(q), make_uint2(c[0], c[1]));
  }
}

}  // namespace quant
}  // namespace fp8g
