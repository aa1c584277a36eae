// fp8_codec.cuh -- device-side FP8 encode/decode for sm_100a.
//
// Formats (blog.daoxuan.cc explainer of "Scaling FP8 training to
// trillion-token LLMs", sub-section "两种 FP8 格式差在指数位和尾数位"; bit table
// of "FP8训练的稳定性挑战…", section "FP8格式简介"):
//   E4M3 (OCP "fn"): sign, 4 exponent bits (bias 7), 3 mantissa bits; the
//     pattern S.1111.111 is NaN, there is no infinity, max 0x7E = 448.
//   E5M2: sign, 5 exponent bits (bias 15), 2 mantissa bits; exponent 31 is
//     inf (mantissa 0) or NaN, max 0x7B = 57344.
// Encoding: round to nearest, ties to the even code; |x| above max (and inf)
// saturates to +-max; the sign of zero and of underflow is kept; NaN gives a
// NaN code.
//
// Two implementations:
//   hw: PTX cvt.rn.satfinite.{e4m3x2,e5m2x2}.f32 (pack two fp32) and
//       cvt.rn.f16x2.{e4m3x2,e5m2x2} + cvt.f32.f16 (unpack two codes);
//   sw: integer manipulation of the fp32 fields.
// Packing convention of the x2 forms: the element stored at the lower byte
// of the 16-bit pair is the lower half of the f16x2 / the second cvt source.
#pragma once

#include <cuda_fp16.h>
#include <stdint.h>

namespace fp8adam {

enum Fmt : int { kE4M3 = 0, kE5M2 = 1, kFP32 = 2 };

template <int FMT> struct FmtTraits;
template <> struct FmtTraits<kE4M3> {
  static constexpr int kMant = 3;
  static constexpr int kBias = 7;
  static constexpr int kEmax = 8;              // max = 1.75 * 2^kEmax
  static constexpr uint32_t kMaxCode = 0x7Eu;
  static constexpr uint32_t kMaxBits = 0x43E00000u;  // 448.0f
  static constexpr float kMax = 448.0f;
};
template <> struct FmtTraits<kE5M2> {
  static constexpr int kMant = 2;
  static constexpr int kBias = 15;
  static constexpr int kEmax = 15;
  static constexpr uint32_t kMaxCode = 0x7Bu;
  static constexpr uint32_t kMaxBits = 0x47600000u;  // 57344.0f
  static constexpr float kMax = 57344.0f;
};

// ---------------------------------------------------------------- hardware
// Two fp32 -> two codes; `lo` lands in bits 0..7, `hi` in bits 8..15.
template <int FMT>
__device__ __forceinline__ uint32_t enc2_hw(float lo, float hi) {
  uint16_t d;
  if constexpr (FMT == kE4M3) {
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  } else {
    asm("cvt.rn.satfinite.e5m2x2.f32 %0, %1, %2;" : "=h"(d) : "f"(hi), "f"(lo));
  }
  return d;
}

// Two codes (bits 0..7 and 8..15 of `pair`) -> two fp32.
template <int FMT>
__device__ __forceinline__ float2 dec2_hw(uint32_t pair) {
  uint32_t h2;
  const uint16_t in = (uint16_t)(pair & 0xFFFFu);
  if constexpr (FMT == kE4M3) {
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(in));
  } else {
    asm("cvt.rn.f16x2.e5m2x2 %0, %1;" : "=r"(h2) : "h"(in));
  }
  __half2 h = *reinterpret_cast<__half2*>(&h2);
  return __half22float2(h);
}

// ---------------------------------------------------------------- software
template <int FMT>
__device__ __forceinline__ uint32_t enc1_sw(float x) {
  using T = FmtTraits<FMT>;
  const uint32_t u = __float_as_uint(x);
  const uint32_t sign = (u >> 24) & 0x80u;
  const uint32_t a = u & 0x7FFFFFFFu;
  if (a > 0x7F800000u) return 0x7Fu;                    // NaN
  if (a >= T::kMaxBits) return sign | T::kMaxCode;      // >= max, inf: satfinite
  const uint32_t min_normal = (uint32_t)(127 + 1 - T::kBias) << 23;  // 2^(1-bias)
  uint32_t code;
  if (a < min_normal) {
    // subnormal target: count quanta of 2^(1-bias-M); the power-of-two
    // product is exact and the conversion rounds to nearest even
    const float q = __uint_as_float(a) * __uint_as_float((uint32_t)(127 + T::kBias - 1 + T::kMant) << 23);
    code = (uint32_t)__float2int_rn(q);
  } else {
    // keep M mantissa bits, rounding the dropped 23-M bits to nearest even
    // (a carry moves into the exponent field), then rebias the exponent
    constexpr int sh = 23 - T::kMant;
    const uint32_t r = (a + ((1u << (sh - 1)) - 1u) + ((a >> sh) & 1u)) >> sh;
    code = r - ((uint32_t)(127 - T::kBias) << T::kMant);
  }
  return sign | code;
}

template <int FMT>
__device__ __forceinline__ float dec1_sw(uint32_t c) {
  const uint32_t sign = (c & 0x80u) << 24;
  const uint32_t mag = c & 0x7Fu;
  float f;
  if constexpr (FMT == kE4M3) {
    if (mag == 0x7Fu) return __uint_as_float(0x7FFFFFFFu);
    // exponent and mantissa fields placed in an fp32 (a subnormal code
    // becomes an fp32 subnormal), then rebiased by an exact 2^(127-7)
    f = __uint_as_float(mag << 20) * 0x1p120f;
  } else {
    if (mag >= 0x7Cu) return mag == 0x7Cu ? __uint_as_float(sign | 0x7F800000u) : __uint_as_float(0x7FFFFFFFu);
    f = __uint_as_float(mag << 21) * 0x1p112f;
  }
  return __uint_as_float(__float_as_uint(f) | sign);
}

// ---------------------------------------------------------------- helpers
// One element through the hardware pair form (upper half unused).
template <int FMT>
__device__ __forceinline__ uint32_t enc1_hw(float x) {
  return enc2_hw<FMT>(x, 0.0f) & 0xFFu;
}
template <int FMT>
__device__ __forceinline__ float dec1_hw(uint32_t c) {
  return dec2_hw<FMT>(c & 0xFFu).x;
}

// Largest 2^k (|k| <= 126) with amax * 2^k <= max of FMT; amax <= 0, inf or
// NaN keeps s_prev.  amax = f * 2^e with f in [1,2): k = Emax - e, one less
// when f > 1.75 (mantissa field above 0x600000).
template <int FMT>
__device__ __forceinline__ float pow2scale(float amax, float s_prev) {
  const uint32_t b = __float_as_uint(amax);
  if (!(amax > 0.0f) || b >= 0x7F800000u) return s_prev;
  int k;
  if (b < 0x00800000u) {
    k = 126;  // subnormal amax: the unclamped exponent exceeds 126
  } else {
    const int e = (int)(b >> 23) - 127;
    k = FmtTraits<FMT>::kEmax - e - ((b & 0x7FFFFFu) > 0x600000u ? 1 : 0);
    k = k > 126 ? 126 : (k < -126 ? -126 : k);
  }
  return __uint_as_float((uint32_t)(k + 127) << 23);
}

}  // namespace fp8adam
