// MXFP4 (OCP MX v1.0 FP4) helpers shared by the activation quantisers: the
// 1x32 block rule with an e8m0 shared exponent floor(log2(amax)) - 2 and
// round-to-nearest-even e2m1 elements saturating at 6 (the format named by
// aiter PR #3859, "Details": float4_e2m1fn_x2, QuantType.per_1x32).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// e2m1 codes of two floats already divided by their block scale:
// round to nearest even on the e2m1 grid, saturating to +-6.
__device__ __forceinline__ uint32_t cvt_e2m1x2(float even, float odd) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(r)
      : "f"(even), "f"(odd));
  return r & 0xffu;
}

// Shared exponent of a block with absolute maximum amax (finite, fp32):
// s = clamp(floor(log2(amax)) - 2, -127, 127); e8m0 code s + 127; 0 for amax == 0.
__device__ __forceinline__ int mx_scale_exp(float amax) {
  if (!(amax > 0.0f)) return -127;
  const uint32_t bits = __float_as_uint(amax);
  int ex = static_cast<int>((bits >> 23) & 0xffu);
  int fl;
  if (ex == 0) {
    // subnormal amax: floor(log2) = -149 + index of the highest set mantissa bit
    fl = -149 + (31 - __clz(bits & 0x7fffffu));
  } else {
    fl = ex - 127;
  }
  int s = fl - 2;
  return max(-127, min(127, s));
}

// 2^-s as an exact float for s in [-127, 127]; every value but 2^-127 is a
// normal number whose exponent field can be written directly.
__device__ __forceinline__ float exp2i_neg(int s) {
  const int e = 127 - s;  // biased exponent of 2^-s
  if (e >= 1 && e <= 254) return __uint_as_float(static_cast<uint32_t>(e) << 23);
  return ldexpf(1.0f, -s);
}

// Quantise 32 floats: returns scale code, writes 16 code bytes as 4 words.
__device__ __forceinline__ uint32_t mx_quant32(const float (&v)[32], uint32_t (&w)[4]) {
  float amax = 0.0f;
#pragma unroll
  for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
  const int s = mx_scale_exp(amax);
  const float inv = exp2i_neg(s);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t word = 0;
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int i = q * 8 + b * 2;
      word |= cvt_e2m1x2(v[i] * inv, v[i + 1] * inv) << (8 * b);
    }
    w[q] = word;
  }
  return static_cast<uint32_t>(s + 127);
}

}  // namespace moe
