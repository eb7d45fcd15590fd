// fp8_prep.cuh -- FP8 input preparation with incoherent processing (page
// "FlashAttention-3 — 闪电注意力-3", section 3, items 1-3): rotate each row
// by M = diag(signs) H_d / sqrt(d) (H_d the Sylvester Hadamard matrix), take
// the per-tensor absolute maximum, and quantise to E4M3 with
// descale = amax / 448.
//
// HBM-bound (2 bytes read and 1 byte written per element), so the design is
// about bytes in flight and few instructions per element:
//   * tiles of 128 rows x 128 columns (32 KB of bf16) are brought into shared
//     memory by TMA (two 128-byte-wide boxes, 128-byte swizzle) through a
//     ring of stages, several tiles ahead of the compute;
//   * thread t of a 128-thread block owns row t of the tile: it reads the row
//     from shared memory (the swizzle spreads the 16-byte chunks of eight
//     consecutive rows over all banks, so the reads are conflict-free), and
//     runs the whole fast Walsh-Hadamard transform in registers -- no
//     shuffles: a packed fp32x2 register holds elements k and k + 64, so six
//     of the seven butterfly levels are packed operations and only the last
//     one is scalar (the amax pass needs only |a| + |b| of it);
//   * the random signs are applied as XOR masks on the bf16 sign bits before
//     the values are widened (an exact multiplication by +-1), and 1/sqrt(d)
//     is folded into the final scale: fl(max|y| * c) = max fl(|y| * c) for
//     c > 0, so amax is what scaling every value first would give;
//   * the quantising pass writes each row's 128 codes into a swizzled
//     shared-memory tile that one TMA store writes back; rows past the end of
//     the tensor are zero-filled on load and clipped on store.
// Two passes (amax, then quantise) because every code depends on the global
// amax; the second pass walks the tiles in reverse order, so it starts on the
// ones the first pass read last, which are the likeliest to be in L2.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "attn_common.cuh"
#include "ptx.cuh"

namespace attn {

constexpr int kPrepD = 128;
constexpr int kPrepRows = 128;                               // rows per tile = threads per block
constexpr uint32_t kPrepHalfBytes = kPrepRows * 128;         // one 64-column box of bf16
constexpr uint32_t kPrepTileBytes = 2 * kPrepHalfBytes;      // 32 KB
constexpr uint32_t kPrepOutBytes = kPrepRows * kPrepD;       // 16 KB of codes
constexpr float kPrepInvSqrtD = 0.08838834764831845f;        // 1/sqrt(128)

template <bool QUANT>
struct PrepCfg {
  // the amax pass keeps 128 values and little else per thread (under 170
  // registers): three blocks per SM; the quantising pass needs more registers
  // and an output buffer: two blocks per SM
  static constexpr int BLOCKS_PER_SM = QUANT ? 2 : 3;
  static constexpr int STAGES = 2;
  static constexpr uint32_t OFF_IN = 0;
  static constexpr uint32_t OFF_OUT = STAGES * kPrepTileBytes;
  static constexpr uint32_t OFF_BAR = OFF_OUT + (QUANT ? kPrepOutBytes : 0);
  // the sign masks are read as 16-byte vectors: 16-byte aligned
  static constexpr uint32_t OFF_MASK = (OFF_BAR + 8 * STAGES + 15u) & ~15u;
  static constexpr uint32_t OFF_ABORT = OFF_MASK + 64 * 4;
  static constexpr uint32_t OFF_RED = OFF_ABORT + 16;
  static constexpr uint32_t SMEM_BYTES = OFF_RED + 4 * 4 + 1024;  // + alignment slack
  static_assert(OFF_MASK % 16 == 0 && OFF_IN % 1024 == 0 && OFF_OUT % 1024 == 0, "vector and TMA alignment");
  static_assert(BLOCKS_PER_SM * (SMEM_BYTES + 1024) <= 228 * 1024, "blocks per SM");
};

struct PrepParams {
  long long rows;
  int n_tiles;
  const float* signs;        // d values, +1 or -1; nullptr: no rotation
  unsigned int* amax_bits;   // running max of |rotated value| as float bits
  float* descale;            // amax / 448 (quantising pass)
  unsigned int* err;
  unsigned long long timeout_ns;
};

// Row r of the tile in stage memory `tile` (two swizzled 64-column boxes) ->
// 128 fp32 values, signs applied (XOR masks on the bf16 sign bits), then, when
// ROT, levels 0..5 of the unnormalised Walsh-Hadamard transform.  The packed
// register pair P[k] holds elements k and k + 64 (column k of each box), so
// the butterflies of spans 1..32 are packed fp32x2 operations on both halves
// at once; the last level (span 64) pairs the two halves of each P[k]:
// y[k] = a + b, y[k + 64] = a - b for P[k] = (a, b), and is left to the
// caller (the amax pass needs only max(|a + b|, |a - b|) = |a| + |b|).
template <bool ROT>
__device__ __forceinline__ void prep_load_transform(const uint8_t* tile, const uint4* mask4, int r,
                                                    uint64_t (&P)[64]) {
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    const int off = r * 128 + ((c ^ (r & 7)) << 4);
    uint4 w0 = *reinterpret_cast<const uint4*>(tile + off);                   // elements 8c .. 8c+7
    uint4 w1 = *reinterpret_cast<const uint4*>(tile + kPrepHalfBytes + off);  // elements 64+8c ..
    if constexpr (ROT) {
      const uint4 m0 = mask4[c], m1 = mask4[8 + c];
      w0.x ^= m0.x;
      w0.y ^= m0.y;
      w0.z ^= m0.z;
      w0.w ^= m0.w;
      w1.x ^= m1.x;
      w1.y ^= m1.y;
      w1.z ^= m1.z;
      w1.w ^= m1.w;
    }
    const uint32_t a[4] = {w0.x, w0.y, w0.z, w0.w}, b[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      P[8 * c + 2 * e] = ptx::f2(__uint_as_float(a[e] << 16), __uint_as_float(b[e] << 16));
      P[8 * c + 2 * e + 1] = ptx::f2(__uint_as_float(a[e] & 0xFFFF0000u), __uint_as_float(b[e] & 0xFFFF0000u));
    }
  }
  if constexpr (ROT) {
#pragma unroll
    for (int sp = 1; sp < 64; sp <<= 1)
#pragma unroll
      for (int k = 0; k < 64; ++k)
        if ((k & sp) == 0) {
          const uint64_t x = P[k], y = P[k + sp];
          P[k] = ptx::fadd2(x, y);
          P[k + sp] = ptx::fsub2(x, y);
        }
  }
}

// Element j (0..127) of the transformed row: the last butterfly level when ROT.
template <bool ROT>
__device__ __forceinline__ float prep_elem(const uint64_t (&P)[64], int j) {
  float a, b;
  ptx::unf2(P[j & 63], a, b);
  if constexpr (ROT) return j < 64 ? a + b : a - b;
  return j < 64 ? a : b;
}

// One pass over the tensor: QUANT = false accumulates amax (one atomicMax per
// block), QUANT = true writes the codes and, from block 0, the descale.
template <bool ROT, bool QUANT>
__global__ void __launch_bounds__(kPrepRows, PrepCfg<QUANT>::BLOCKS_PER_SM)
    fp8_prep_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmX8,
                    const PrepParams p) {
  using C = PrepCfg<QUANT>;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = ptx::smem_u32(smem_raw);
  const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw_u32);
  auto bar = [&](int s) -> uint32_t { return sbase + C::OFF_BAR + 8u * (uint32_t)s; };
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sgen + C::OFF_ABORT);
  const WaitCtx wc{abort_flag, p.err, p.timeout_ns};
  const int tid = threadIdx.x;
  const int G = (int)gridDim.x;
  // tile of this block's k-th step (the quantising pass walks them backwards)
  auto tile_at = [&](int k) -> int {
    const long long i = (long long)blockIdx.x + (long long)k * G;
    if (i >= p.n_tiles) return -1;
    return QUANT ? p.n_tiles - 1 - (int)i : (int)i;
  };

  uint32_t* mask = reinterpret_cast<uint32_t*>(sgen + C::OFF_MASK);
  if (tid < 64) {
    uint32_t m = 0u;
    if (ROT) {
      if (__ldg(p.signs + 2 * tid) < 0.f) m |= 0x00008000u;
      if (__ldg(p.signs + 2 * tid + 1) < 0.f) m |= 0x80000000u;
    }
    mask[tid] = m;
  }
  if (tid == 0) {
    for (int s = 0; s < C::STAGES; ++s) ptx::mbar_init(bar(s), 1);
    *abort_flag = 0u;
    ptx::fence_mbar_init();
    ptx::prefetch_tmap(&tmX);
    if (QUANT) ptx::prefetch_tmap(&tmX8);
  }
  __syncthreads();

  int issued[C::STAGES];
#pragma unroll
  for (int s = 0; s < C::STAGES; ++s) issued[s] = 0;
  auto issue = [&](int k) {  // thread 0: load the tile of step k into stage k % STAGES
    const int tile = tile_at(k);
    if (tile < 0) return;
    const int s = k % C::STAGES;
    const uint32_t dst = sbase + C::OFF_IN + (uint32_t)s * kPrepTileBytes;
    ptx::mbar_arrive_expect_tx(bar(s), kPrepTileBytes);
    ptx::tma_load_2d(dst, &tmX, bar(s), 0, tile * kPrepRows);
    ptx::tma_load_2d(dst + kPrepHalfBytes, &tmX, bar(s), 64, tile * kPrepRows);
    ++issued[s];
  };
  if (tid == 0)
    for (int k = 0; k < C::STAGES; ++k) issue(k);

  float mult = 0.f;
  if constexpr (QUANT) {
    const float amax = __uint_as_float(*p.amax_bits);
    const float inv = amax > 0.f ? 448.0f / amax : 0.f;
    mult = ROT ? kPrepInvSqrtD * inv : inv;
    if (blockIdx.x == 0 && tid == 0) *p.descale = amax > 0.f ? amax / 448.0f : 1.0f;
  }
  const uint4* mask4 = reinterpret_cast<const uint4*>(mask);
  float m0 = 0.f, m1 = 0.f;
  for (int k = 0;; ++k) {
    const int tile = tile_at(k);
    if (tile < 0) break;
    const int s = k % C::STAGES;
    bool ok = wait_bar<kRoleSoftmax>(bar(s), (uint32_t)((k / C::STAGES) & 1), wc, kSiteKFull);
    uint64_t P[64];
    if (ok) prep_load_transform<ROT>(sgen + C::OFF_IN + (uint32_t)s * kPrepTileBytes, mask4, tid, P);
    if constexpr (QUANT) {
      if (tid == 0) ptx::bulk_wait_read0();  // the previous tile's store has read the output buffer
    }
    if (!__syncthreads_and(ok)) break;  // stage s is consumed by every thread
    if (tid == 0) issue(k + C::STAGES);
    if constexpr (!QUANT) {
#pragma unroll
      for (int i = 0; i < 64; ++i) {
        float a, b;
        ptx::unf2(P[i], a, b);
        if constexpr (ROT) {
          m0 = fmaxf(m0, fabsf(a) + fabsf(b));  // = max(|a + b|, |a - b|), also in fp32
        } else {
          m0 = fmaxf(m0, fabsf(a));
          m1 = fmaxf(m1, fabsf(b));
        }
      }
    } else {
      uint8_t* out = sgen + C::OFF_OUT;
#pragma unroll
      for (int c = 0; c < 8; ++c) {  // 16 codes (one 16-byte chunk) at a time
        uint32_t w[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 16 * c + 4 * e;
          w[e] = ptx::pack_e4m3x4(prep_elem<ROT>(P, j) * mult, prep_elem<ROT>(P, j + 1) * mult,
                                  prep_elem<ROT>(P, j + 2) * mult, prep_elem<ROT>(P, j + 3) * mult);
        }
        *reinterpret_cast<uint4*>(out + tid * 128 + ((c ^ (tid & 7)) << 4)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      ptx::fence_proxy_async_smem();
      __syncthreads();
      if (tid == 0) {
        ptx::tma_store_2d(&tmX8, sbase + C::OFF_OUT, 0, tile * kPrepRows);
        ptx::bulk_commit();
      }
    }
  }
  if (tid == 0) {
    // every issued load must land and every store must finish before exit
#pragma unroll
    for (int s = 0; s < C::STAGES; ++s)
      if (issued[s] > 0) wait_bar_drain<kRoleProducer>(bar(s), (uint32_t)((issued[s] - 1) & 1), wc, kSiteDrain);
    if (QUANT) ptx::bulk_wait0();
  }
  if constexpr (!QUANT) {
    float m = fmaxf(m0, m1);
    if (ROT) m *= kPrepInvSqrtD;  // monotone: the max of the scaled values
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float* red = reinterpret_cast<float*>(sgen + C::OFF_RED);
    if ((tid & 31) == 0) red[tid >> 5] = m;
    __syncthreads();
    if (tid == 0) {
      const float bm = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
      atomicMax(p.amax_bits, __float_as_uint(bm));  // non-negative floats order like their bits
    }
  }
}

}  // namespace attn
