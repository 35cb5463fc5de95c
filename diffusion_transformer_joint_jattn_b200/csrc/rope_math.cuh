// Per-element arithmetic of the prologue that more than one kernel performs:
// the bf16 -> fp32 widening, the (t, row, col) axis of a channel pair, the
// rotary angle's cos / sin, the query/key RMSNorm scaling and the rotation
// of one channel pair.
//
// Every rounding here is spelled out with an intrinsic (no contraction left
// to the compiler), so that a kernel that recomputes a rotated value from
// the inputs -- the token repair's gather, the correction operands of the
// high-precision 16-bit path -- gets exactly the fp32 value the prologue
// rounded to its output type.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>
#include <cuda_fp16.h>

namespace jattn {

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&x)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    x[2 * i] = __uint_as_float(w[i] << 16);
    x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ float bf16_to_f32(uint16_t u) { return __uint_as_float(static_cast<uint32_t>(u) << 16); }

// cos/sin of the angle pos_axis * omega of one channel pair: the angle is
// formed and reduced to [-pi, pi] in fp64 (multiplying by 1/(2 pi)), then
// rotated with the fp32 sincos.  omega comes from the RopeTable the host
// builds once per call (see jattn_internal.h), so every kernel that rotates
// the same pair of the same token gets the same cos/sin bits.
__device__ __forceinline__ void angle_cos_sin(int32_t pos_axis, double omega, float& c, float& s) {
  const double ang = static_cast<double>(pos_axis) * omega;
  const double two_pi = 6.283185307179586476925286766559;
  const double inv_two_pi = 0.15915494309189533576888376337251;
  const double r = ang - rint(ang * inv_two_pi) * two_pi;
  sincosf(static_cast<float>(r), &s, &c);
}

// RMSNorm of one value: x * r * w, with r = 1 / sqrt(mean(x^2) + eps) of its row.
__device__ __forceinline__ float norm_scale(float x, float r, float w) { return __fmul_rn(__fmul_rn(x, r), w); }

// 1 / sqrt(mean of squares + eps) from a row's fp32 sum of squares, by the
// hardware reciprocal square root (rsqrtf, at most 2 ulp from the exact
// value; the correctly rounded __frsqrt_rn cost the norm prologue 11%).
// Every kernel that needs a row's factor reads the one the prologue stored.
__device__ __forceinline__ float norm_factor(float sum_sq, int d, float eps) {
  return rsqrtf(__fmaf_rn(sum_sq, 1.0f / static_cast<float>(d), eps));
}

// (a, b) rotated by the angle with cosine c and sine s.
__device__ __forceinline__ void rotate_pair(float a, float b, float c, float s, float& x0, float& x1) {
  x0 = __fmaf_rn(a, c, -__fmul_rn(b, s));
  x1 = __fmaf_rn(a, s, __fmul_rn(b, c));
}

// Smallest e >= 0 with amax * 2^-e <= 65504 (the largest finite fp16): the
// 16-bit outputs of a tile whose magnitudes reach amax are stored scaled by
// 2^-e, which is exact.
// Non-finite amax (an input holding Inf / NaN, which the path does not
// support) gives 0: the values stay as they are and overflow in fp16.
__device__ __forceinline__ int f16_range_exponent(float amax) {
  if (!(amax > 65504.0f) || !isfinite(amax)) return 0;
  int e = max(ilogbf(amax) - 15, 1);              // amax < 2^128, so e <= 113
  for (int k = 0; k < 2 && ldexpf(amax, -e) > 65504.0f; ++k) ++e;
  return e;
}

}  // namespace jattn
