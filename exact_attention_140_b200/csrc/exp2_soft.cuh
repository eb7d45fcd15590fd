// exp2_soft.cuh -- 2^x on the FMA pipe, two values per call (page
// "FlashAttention-4震撼发布": the exponential is emulated in software so that
// the softmax is not limited by the hardware exponential unit, which on this
// GPU has the same per-element throughput at d = 128 as the tensor core).
//
// Method (Cody-Waite style split, our own fit):
//   x is clamped to >= -125, then x = j + f with j = round-to-nearest(x),
//   f in [-0.5, 0.5].  j is found by adding 1.5 * 2^23 (the integer lands in
//   the low mantissa bits), f = x - j exactly.  2^f = p(f) =
//   1 + f (c1 + f (c2 + f c3)), coefficients fitted by fit_exp2_poly.py for
//   minimax relative error 1.01e-4 on [-0.5, 0.5] with p(0) = 1, so 2^0 is
//   exact.  2^j is applied by adding j << 23 to the bits of p(f); with
//   j >= -125 the result stays a normal float.  Results below 2^-125 (the
//   clamp) are returned as about 2^-125 instead of 0; callers that need exact
//   zeros (masked keys) select them after the call.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace attn {

constexpr uint32_t kExpMagicBits = 0x4B400000u;  // 1.5 * 2^23
constexpr float kExpC1 = 0.693282723f, kExpC2 = 0.242211044f, kExpC3 = 0.0550097041f;

__device__ __forceinline__ void exp2_soft2(float x0, float x1, float& y0, float& y1) {
  using namespace ptx;
  const uint64_t x = f2(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t t = fadd2(x, f2_const(kExpMagicBits));
  const uint64_t jf = fsub2(t, f2_const(kExpMagicBits));
  const uint64_t f = fsub2(x, jf);
  uint64_t p = ffma2(f2_const(__float_as_uint(kExpC3)), f, f2_const(__float_as_uint(kExpC2)));
  p = ffma2(p, f, f2_const(__float_as_uint(kExpC1)));
  p = ffma2(p, f, f2_const(0x3F800000u));
  float t0, t1, p0, p1;
  unf2(t, t0, t1);
  unf2(p, p0, p1);
  y0 = __uint_as_float(__float_as_uint(t0) * (1u << 23) + __float_as_uint(p0));
  y1 = __uint_as_float(__float_as_uint(t1) * (1u << 23) + __float_as_uint(p1));
}

}  // namespace attn
