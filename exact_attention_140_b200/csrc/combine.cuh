// combine.cuh -- the output side of split-KV attention: S partial results of
// one query row over disjoint key windows, each normalised by its own row sum
// (O_s, with LSE_s = ln of that sum of exp(scores)), merge into the result
// over the union of the windows:
//   LSE = ln sum_s exp(LSE_s),   O = sum_s exp(LSE_s - LSE) O_s.
// This is the online-softmax rescaling of page "FlashAttention (SV)",
// section "Online-beräkning av Softmax", applied once per window instead of
// once per key tile.  Windows with no visible key have LSE_s = -inf and weigh
// nothing; a row with no visible key at all gets O = 0, LSE = -inf.
//
// One warp per output row (b, row, h); lane c handles the columns c, c + 32,
// ... (coalesced 128-byte accesses per split).  HBM-bound: S * (4d + 4) bytes
// read and 2d + 4 written per row.
#pragma once
#include <cuda_bf16.h>
#include <cstdint>

namespace attn {

template <int D>
__global__ void __launch_bounds__(256) attn_combine_kernel(const float* __restrict__ o_part,
                                                           const float* __restrict__ lse_part, int S, int B, int Hq,
                                                           int Nq, __nv_bfloat16* __restrict__ o,
                                                           float* __restrict__ lse) {
  constexpr int PER = D / 32;
  const long long rows = (long long)B * Nq * Hq;
  const long long warp = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  // warp -> (b, row, h) in the [B, Nq, Hq] order of O
  const int h = (int)(warp % Hq);
  const long long bi = warp / Hq;
  const int row = (int)(bi % Nq);
  const int b = (int)(bi / Nq);
  const long long split_stride_lse = (long long)B * Hq * Nq;
  const long long lse_off = ((long long)b * Hq + h) * Nq + row;
  // lane s holds LSE_s for the windows s, s + 32, ...; the row max first
  float m = -INFINITY;
  for (int s = lane; s < S; s += 32) m = fmaxf(m, __ldg(lse_part + s * split_stride_lse + lse_off));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float wsum = 0.f;
  if (m != -INFINITY) {
    const long long split_stride_o = rows * D;
    const float* src = o_part + warp * D + lane;
    // windows in groups of 32: each lane computes the weight of one window
    // (0 for an empty window), then the group's weights are broadcast and its
    // partial rows loaded 8 windows at a time, so the loads overlap
    for (int s0 = 0; s0 < S; s0 += 32) {
      const int sl = s0 + lane;
      const float ls = sl < S ? __ldg(lse_part + sl * split_stride_lse + lse_off) : -INFINITY;
      const float wl = ls == -INFINITY ? 0.f : expf(ls - m);
      const int n = S - s0 < 32 ? S - s0 : 32;
      for (int j0 = 0; j0 < n; j0 += 8) {
        float w[8], x[8][PER];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          w[u] = __shfl_sync(0xffffffffu, wl, (j0 + u) & 31);
          const bool live = j0 + u < n && w[u] != 0.f;  // uniform across the warp
#pragma unroll
          for (int e = 0; e < PER; ++e)
            x[u][e] = live ? __ldg(src + (long long)(s0 + j0 + u) * split_stride_o + 32 * e) : 0.f;
          if (!live) w[u] = 0.f;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          wsum += w[u];
#pragma unroll
          for (int e = 0; e < PER; ++e) acc[e] = fmaf(w[u], x[u][e], acc[e]);
        }
      }
    }
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* dst = o + warp * D + lane;
#pragma unroll
  for (int e = 0; e < PER; ++e) dst[32 * e] = __float2bfloat16_rn(acc[e] * inv);
  if (lse != nullptr && lane == 0) lse[lse_off] = wsum > 0.f ? m + logf(wsum) : -INFINITY;
}

}  // namespace attn
