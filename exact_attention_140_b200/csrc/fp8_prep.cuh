// fp8_prep.cuh -- FP8 input preparation with incoherent processing (page
// "FlashAttention-3 — 闪电注意力-3", section 3, items 1-3): rotate each row
// by M = diag(signs) H_d / sqrt(d) (H_d the Sylvester Hadamard matrix), take
// the per-tensor absolute maximum, and quantise to E4M3 with
// descale = amax / 448.
//
// One warp owns one row of d = 128 elements, 4 consecutive elements per
// lane.  The rotation is a fast Walsh-Hadamard transform: butterflies of
// span 1 and 2 inside a lane, spans 4..64 across lanes with shuffles.  Two
// passes over the input (HBM-bound): pass 1 finds amax, pass 2 rotates again
// and writes the codes (recomputing the transform costs less than a round
// trip of the rotated tensor through HBM).
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

#include "ptx.cuh"

namespace attn {

constexpr int kPrepD = 128;
constexpr int kPrepWarps = 8;

// Loads row r (4 values per lane), applies signs and the transform when
// `signs` is not null.  Returns the lane's 4 rotated values.
__device__ __forceinline__ void prep_row(const __nv_bfloat16* __restrict__ x, long long r,
                                         const float* __restrict__ signs, float (&v)[4]) {
  const int lane = threadIdx.x & 31;
  const uint2 raw = __ldg(reinterpret_cast<const uint2*>(x + r * kPrepD) + lane);
  v[0] = __uint_as_float(raw.x << 16);
  v[1] = __uint_as_float(raw.x & 0xFFFF0000u);
  v[2] = __uint_as_float(raw.y << 16);
  v[3] = __uint_as_float(raw.y & 0xFFFF0000u);
  if (signs == nullptr) return;
  const float4 s = __ldg(reinterpret_cast<const float4*>(signs) + lane);
  v[0] *= s.x;
  v[1] *= s.y;
  v[2] *= s.z;
  v[3] *= s.w;
  // span 1 and span 2 inside the lane (element index 4*lane + e)
  float a0 = v[0] + v[1], a1 = v[0] - v[1], a2 = v[2] + v[3], a3 = v[2] - v[3];
  v[0] = a0 + a2;
  v[1] = a1 + a3;
  v[2] = a0 - a2;
  v[3] = a1 - a3;
  // spans 4, 8, 16, 32, 64 = lane distances 1, 2, 4, 8, 16
#pragma unroll
  for (int ld = 1; ld < 32; ld <<= 1) {
    const bool upper = (lane & ld) != 0;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float w = __shfl_xor_sync(0xffffffffu, v[e], ld);
      v[e] = upper ? (w - v[e]) : (v[e] + w);
    }
  }
  const float inv_sqrt_d = 0.08838834764831845f;  // 1/sqrt(128)
#pragma unroll
  for (int e = 0; e < 4; ++e) v[e] *= inv_sqrt_d;
}

__global__ void __launch_bounds__(32 * kPrepWarps) fp8_amax_kernel(const __nv_bfloat16* __restrict__ x, long long rows,
                                                                     const float* __restrict__ signs,
                                                                     unsigned int* __restrict__ amax_bits) {
  __shared__ float red[kPrepWarps];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float m = 0.f;
  for (long long r = (long long)blockIdx.x * kPrepWarps + warp; r < rows; r += (long long)gridDim.x * kPrepWarps) {
    float v[4];
    prep_row(x, r, signs, v);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v[0]), fabsf(v[1])), fmaxf(fabsf(v[2]), fabsf(v[3]))));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if (lane == 0) red[warp] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float bm = red[0];
    for (int w = 1; w < kPrepWarps; ++w) bm = fmaxf(bm, red[w]);
    atomicMax(amax_bits, __float_as_uint(bm));  // non-negative floats order like their bits
  }
}

__global__ void __launch_bounds__(32 * kPrepWarps) fp8_quant_kernel(const __nv_bfloat16* __restrict__ x, long long rows,
                                                                      const float* __restrict__ signs,
                                                                      const unsigned int* __restrict__ amax_bits,
                                                                      uint8_t* __restrict__ x8,
                                                                      float* __restrict__ descale) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float amax = __uint_as_float(*amax_bits);
  const float inv = amax > 0.f ? 448.0f / amax : 0.f;
  if (blockIdx.x == 0 && threadIdx.x == 0) *descale = amax > 0.f ? amax / 448.0f : 1.0f;
  for (long long r = (long long)blockIdx.x * kPrepWarps + warp; r < rows; r += (long long)gridDim.x * kPrepWarps) {
    float v[4];
    prep_row(x, r, signs, v);
    const uint32_t codes = ptx::pack_e4m3x4(v[0] * inv, v[1] * inv, v[2] * inv, v[3] * inv);
    reinterpret_cast<uint32_t*>(x8 + r * kPrepD)[lane] = codes;
  }
}

}  // namespace attn
