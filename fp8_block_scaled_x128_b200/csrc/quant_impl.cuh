// quant_impl.cuh -- device code of the FP8 (e4m3) quantisation of 1x128
// groups and 128x128 blocks, shared by the quantiser kernels (quant.cu) and
// the expert dispatch (moe.cu).
//
//   scale = amax / 448 (FP32; 1 for an all-zero group),
//   code  = e4m3_rne_satfinite(x / scale)   (one IEEE FP32 division)
//
// The division.  A full IEEE division per element would make the kernels
// ALU-bound.  Each element instead takes the product with the correctly
// rounded reciprocal of the group's scale and two Markstein correction steps
// (quotient_rn: one multiply and four FMAs, no branch), which give the
// correctly rounded quotient fl(x / s); its e4m3 conversion is then exactly
// the code of the definition, bit for bit.
#pragma once

#include <cuda_fp8.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace fp8g {
namespace quant {

constexpr float kE4M3Max = 448.0f;
constexpr int kUnits = 8;  // 16-byte loads per lane in flight per warp

__device__ __forceinline__ float scale_of(float amax) { return amax > 0.f ? __fdiv_rn(amax, kE4M3Max) : 1.f; }

// Two floats -> two e4m3 codes (round to nearest even, saturating at +-448),
// lo in the low byte.
__device__ __forceinline__ uint32_t e4m3x2(float lo, float hi) {
  return static_cast<uint32_t>(__nv_cvt_float2_to_fp8x2(make_float2(lo, hi), __NV_SATFINITE, __NV_E4M3));
}

// fl(x / s), the correctly rounded binary32 quotient, without a division:
// Markstein's correction step (P. Markstein, "Computation of elementary
// functions on the IBM RISC System/6000 processor", IBM J. Res. Dev. 34,
// 1990; the division theorem as stated in Muller et al., Handbook of
// Floating-Point Arithmetic): with y = RN(1/s) and an approximation q within
// one ulp of x / s, the residual x - s q is exact in one FMA and
// RN(q + (x - s q) y) = RN(x / s).  q0 = RN(x y) can be up to 1.5 ulps off,
// so one correction brings it within one ulp (0.5 ulp plus 2^-23 ulp) and a
// second gives the correctly rounded quotient.  Valid while x / s and the
// residuals stay normal or zero: |x| <= 448.1 s and s is at least 2^-90 here
// (encode_group scales smaller groups up), so the quotient never overflows,
// and a quotient below 2^-126 is far under e4m3's smallest rounding boundary
// (2^-10), where only its sign matters (restored from x, so -0 stays -0).
__device__ __forceinline__ float quotient_rn(float x, float s, float y) {
  float q = x * y;
  q = fmaf(fmaf(-q, s, x), y, q);
  q = fmaf(fmaf(-q, s, x), y, q);
  return copysignf(q, x);
}

// Codes of n values of one group with scale s, packed 4 per 32-bit word
// (lowest element in the lowest byte): e4m3(fl(x / s)) for every value, from
// the correctly rounded quotient above.  A group with a scale below 2^-90 is
// first scaled by 2^100 together with its values (exact), so that the
// reciprocal and the residuals stay in the normal range; no scale can exceed
// FLT_MAX / 448, so no group needs the opposite.
template <int n>
__device__ __forceinline__ void encode_group(const float (&v)[n], float s, uint32_t (&c)[n / 4]) {
  const float k = s < 8.07793567e-28f ? 1.26765060e30f : 1.f;  // 2^-90, 2^100
  const float ss = s * k;
  const float y = __frcp_rn(ss);
  float qv[n];
#pragma unroll
  for (int i = 0; i < n; ++i) qv[i] = quotient_rn(v[i] * k, ss, y);
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
