// gemm_add.cuh -- D = A B + C on tcgen05 for small reduction sizes K.
//
// Page "FlashAttention-4震撼发布" reports an A@B+C kernel for Blackwell that is
// faster than the vendor library when K is small, by overlapping the epilogue
// through two accumulation buffers; it gives no further detail, so this design
// is ours.  With small K the work is the epilogue: reading C and writing D
// (2 x 2 bytes per element) against 2K FLOPs per element, so the kernel is
// HBM-bound and the tensor-core products must hide under the epilogue.
//
// Persistent grid (one block per SM, tiles of 128 x 256 in round-robin
// order).  Warp roles:
//   warps 0..7   epilogue, two warpgroups: warpgroup g takes columns
//                [128 g, 128 g + 128) of the tile, warp w its TMEM lanes
//                32 (w % 4) .. +31 (one tile row per thread); it reads the
//                accumulator from TMEM, adds C from shared memory, writes D
//                back over C in shared memory, and one thread stores the
//                tile with TMA;
//   warp 8       TMA producer: A (K-major) and B (MN-major) blocks of BK = 64
//                through a STAGES-deep ring, and each tile's C into one of two
//                tile buffers;
//   warp 9       MMA issuer (converged warp, elected lane), also allocates
//                tensor memory: tile i accumulates into TMEM columns
//                [256 (i % 2), +256), so the products of tile i + 1 run while
//                the epilogue drains tile i.
// C and D move as whole 128-byte-swizzled boxes (64 columns x 128 rows) by
// TMA, so HBM sees full lines in both directions; a thread reads and writes
// the 16-byte chunks of its own row, which the swizzle spreads over all banks.
// Tile buffer b is reused by tile i + 2 once the TMA store of tile i has read
// it (barrier cd_free).
// Layouts: A [M, K], B [K, N], C and D [M, N], row-major bf16; fp32
// accumulation; D = bf16(A B + C) with round-to-nearest-even.  C may be D
// itself: a tile's C is loaded before its D is stored, and tiles are disjoint.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "attn_common.cuh"
#include "ptx.cuh"

namespace attn {

struct GemmCfg {
  static constexpr int BM = 128, BN = 256, BK = 64;
  static constexpr int STAGES = 2;
  static constexpr uint32_t A_BYTES = BM * 128;            // 128 rows of 64 bf16
  static constexpr uint32_t B_CHUNK = BK * 128;            // 64 K-rows of 64 N-columns
  static constexpr uint32_t B_BYTES = B_CHUNK * (BN / 64);
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr uint32_t BOX_BYTES = BM * 128;          // 128 rows of 64 bf16 (one C/D box)
  static constexpr uint32_t CD_BYTES = BOX_BYTES * (BN / 64);
  static constexpr int B_FULL = 0, B_EMPTY = STAGES, B_ACCF = 2 * STAGES, B_ACCE = 2 * STAGES + 2;
  static constexpr int B_CFULL = 2 * STAGES + 4, B_CDFREE = 2 * STAGES + 6;
  static constexpr int B_DRAIN = 2 * STAGES + 8, NBAR = 2 * STAGES + 9;
  static constexpr uint32_t OFF_CD = STAGES * STAGE_BYTES;
  static constexpr uint32_t OFF_BAR = OFF_CD + 2 * CD_BYTES;
  static constexpr uint32_t OFF_SLOT = OFF_BAR + NBAR * 8;
  static constexpr uint32_t OFF_ABORT = OFF_SLOT + 4;
  static constexpr uint32_t SMEM_BYTES = OFF_ABORT + 4 + 1024;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per block");
  static_assert(OFF_CD % 1024 == 0 && CD_BYTES % 1024 == 0, "swizzled boxes need 1024-byte alignment");
  static constexpr int EPI_WARPS = 8, TMA_WARP = 8, MMA_WARP = 9, NTHREADS = 384;
  static constexpr int EPI_THREADS = 32 * EPI_WARPS;
  static constexpr uint32_t IDESC = ptx::idesc<false>(BM, BN, true);  // B is MN-major
};

struct GemmParams {
  int has_c;  // 0: D = A B
  int M, N, K;
  int tiles_m, n_tiles, k_steps;
  unsigned int* err;
  unsigned long long timeout_ns;
};

__global__ void __launch_bounds__(GemmCfg::NTHREADS, 1)
    gemm_add_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmD,
                    const GemmParams p) {
  using G = GemmCfg;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = ptx::smem_u32(smem_raw);
  const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw_u32);
  auto bar = [&](int i) -> uint32_t { return sbase + G::OFF_BAR + 8u * (uint32_t)i; };
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sgen + G::OFF_ABORT);
  const WaitCtx wc{abort_flag, p.err, p.timeout_ns};
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto tile_at = [&](int k) -> int {
    const long long t = (long long)blockIdx.x + (long long)k * gridDim.x;
    return t < p.n_tiles ? (int)t : -1;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < G::STAGES; ++s) {
      ptx::mbar_init(bar(G::B_FULL + s), 1);
      ptx::mbar_init(bar(G::B_EMPTY + s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(bar(G::B_ACCF + a), 1);
      ptx::mbar_init(bar(G::B_ACCE + a), G::EPI_THREADS);
      ptx::mbar_init(bar(G::B_CFULL + a), 1);
      ptx::mbar_init(bar(G::B_CDFREE + a), 1);
    }
    ptx::mbar_init(bar(G::B_DRAIN), 1);
    *abort_flag = 0u;
    ptx::fence_mbar_init();
  }
  if (warp == G::TMA_WARP && lane == 0) {
    ptx::prefetch_tmap(&tmA);
    ptx::prefetch_tmap(&tmB);
    if (p.has_c) ptx::prefetch_tmap(&tmC);
    ptx::prefetch_tmap(&tmD);
  }
  if (warp == G::MMA_WARP) {
    ptx::tmem_alloc(sbase + G::OFF_SLOT, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sgen + G::OFF_SLOT);

  if (warp < G::EPI_WARPS) {
    // ------------------------------------------------------------ epilogue
    const int wg = warp >> 2, wq = warp & 3;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const int r = wq * 32 + lane;  // this thread's row of the tile
    bool ok = true;
    int stored = 0;  // TMA store groups committed by thread 0
    for (int k = 0; ok; ++k) {
      const int tile = tile_at(k);
      if (tile < 0) break;
      const int acc = k & 1, buf = k & 1;
      const int m0 = (tile % p.tiles_m) * G::BM, n0 = (tile / p.tiles_m) * G::BN;
      ok = wait_bar<kRoleSoftmax>(bar(G::B_ACCF + acc), (uint32_t)((k >> 1) & 1), wc, kSiteODone);
      if (ok && p.has_c)  // this tile's C is in the buffer
        ok = wait_bar<kRoleSoftmax>(bar(G::B_CFULL + buf), (uint32_t)((k >> 1) & 1), wc, kSiteVFull);
      else if (ok && k >= 2)  // no C: the store of tile k - 2 must have read the buffer
        ok = wait_bar<kRoleSoftmax>(bar(G::B_CDFREE + buf), (uint32_t)(((k >> 1) - 1) & 1), wc, kSiteVEmpty);
      // all epilogue warps take the same branch (they meet at a named barrier below)
      ok = ptx::bar_red_and(1, G::EPI_THREADS, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      uint8_t* cd = sgen + G::OFF_CD + (uint32_t)buf * G::CD_BYTES;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t rr[32];
        if (p.k_steps > 0) {
          ptx::tmem_ld32(tmem + lane_off + (uint32_t)(acc * 256 + wg * 128 + 32 * c), rr);
          ptx::tmem_wait_ld_dep(rr);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) rr[e] = 0u;
        }
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          // columns wg*128 + 32c + 8g .. +7: box 2wg + c/2, chunk 4(c%2) + g of row r
          const int box = 2 * wg + c / 2, q = 4 * (c % 2) + g;
          uint4* chunk = reinterpret_cast<uint4*>(cd + box * G::BOX_BYTES + r * 128 + ((q ^ (r & 7)) << 4));
          const uint4 cv = p.has_c ? *chunk : make_uint4(0u, 0u, 0u, 0u);
          const uint32_t w4[4] = {cv.x, cv.y, cv.z, cv.w};
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e)
            w[e] = ptx::pack_bf16x2(__uint_as_float(rr[8 * g + 2 * e]) + __uint_as_float(w4[e] << 16),
                                    __uint_as_float(rr[8 * g + 2 * e + 1]) + __uint_as_float(w4[e] & 0xFFFF0000u));
          *chunk = make_uint4(w[0], w[1], w[2], w[3]);
        }
      }
      // the accumulator has been read out: tile k + 2 may overwrite it
      ptx::tc_fence_before();
      ptx::mbar_arrive(bar(G::B_ACCE + acc));
      // D is in the buffer: every epilogue thread's writes reach the async
      // proxy, then one thread stores the four boxes
      ptx::fence_proxy_async_smem();
      asm volatile("bar.sync 1, %0;" ::"n"(G::EPI_THREADS) : "memory");
      if (threadIdx.x == 0) {
        const uint32_t cds = sbase + G::OFF_CD + (uint32_t)buf * G::CD_BYTES;
#pragma unroll
        for (int j = 0; j < G::BN / 64; ++j) ptx::tma_store_2d(&tmD, cds + (uint32_t)j * G::BOX_BYTES, n0 + 64 * j, m0);
        ptx::bulk_commit();
        ++stored;
        ptx::bulk_wait_read0();  // the stores have read the buffer
        ptx::mbar_arrive(bar(G::B_CDFREE + buf));
      }
    }
    if (threadIdx.x == 0 && stored > 0) ptx::bulk_wait0();  // D is written before the block exits
  } else if (warp == G::TMA_WARP) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int issued[G::STAGES], c_issued[2] = {0, 0};
#pragma unroll
      for (int s = 0; s < G::STAGES; ++s) issued[s] = 0;
      int it = 0;  // k-blocks issued into the ring, across tiles
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int tile = tile_at(k);
        if (tile < 0) break;
        const int m0 = (tile % p.tiles_m) * G::BM, n0 = (tile / p.tiles_m) * G::BN;
        for (int kb = 0; kb < p.k_steps; ++kb, ++it) {
          const int s = it % G::STAGES;
          if (it >= G::STAGES &&
              !wait_bar<kRoleProducer>(bar(G::B_EMPTY + s), (uint32_t)(((it / G::STAGES) - 1) & 1), wc,
                                       kSiteKEmpty)) {
            ok = false;
            break;
          }
          const uint32_t fb = bar(G::B_FULL + s);
          const uint32_t st = sbase + (uint32_t)s * G::STAGE_BYTES;
          ptx::mbar_arrive_expect_tx(fb, G::STAGE_BYTES);
          ptx::tma_load_4d(st, &tmA, fb, kb * G::BK, m0, 0, 0);
#pragma unroll
          for (int c = 0; c < G::BN / 64; ++c)
            ptx::tma_load_4d(st + G::A_BYTES + (uint32_t)c * G::B_CHUNK, &tmB, fb, n0 + 64 * c, kb * G::BK, 0, 0);
          ++issued[s];
        }
        if (!ok) break;
        if (p.has_c) {
          // C of tile k into buffer k % 2, once the store of tile k - 2 has read it
          const int buf = k & 1;
          if (k >= 2 && !wait_bar<kRoleProducer>(bar(G::B_CDFREE + buf), (uint32_t)(((k >> 1) - 1) & 1), wc,
                                                  kSiteVEmpty))
            break;
          const uint32_t fb = bar(G::B_CFULL + buf);
          const uint32_t cds = sbase + G::OFF_CD + (uint32_t)buf * G::CD_BYTES;
          ptx::mbar_arrive_expect_tx(fb, G::CD_BYTES);
#pragma unroll
          for (int j = 0; j < G::BN / 64; ++j)
            ptx::tma_load_2d(cds + (uint32_t)j * G::BOX_BYTES, &tmC, fb, n0 + 64 * j, m0);
          ++c_issued[buf];
        }
      }
      // every issued copy must land before the block may exit
#pragma unroll
      for (int s = 0; s < G::STAGES; ++s)
        if (issued[s] > 0)
          wait_bar_drain<kRoleProducer>(bar(G::B_FULL + s), (uint32_t)((issued[s] - 1) & 1), wc, kSiteKFull);
#pragma unroll
      for (int b = 0; b < 2; ++b)
        if (c_issued[b] > 0)
          wait_bar_drain<kRoleProducer>(bar(G::B_CFULL + b), (uint32_t)((c_issued[b] - 1) & 1), wc, kSiteVFull);
    }
  } else if (warp == G::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    bool ok = true;
    int it = 0;
    for (int k = 0; ok; ++k) {
      const int tile = tile_at(k);
      if (tile < 0) break;
      const int acc = k & 1;
      if (k >= 2) {  // the epilogue of tile k - 2 must have read this accumulator
        ok = wait_bar_warp<kRoleMma>(bar(G::B_ACCE + acc), (uint32_t)(((k >> 1) - 1) & 1), wc, kSiteODone);
        if (!ok) break;
        ptx::tc_fence_after();
      }
      const uint32_t d_t = tmem + (uint32_t)(acc * 256);
      for (int kb = 0; kb < p.k_steps; ++kb, ++it) {
        const int s = it % G::STAGES;
        ok = wait_bar_warp<kRoleMma>(bar(G::B_FULL + s), (uint32_t)((it / G::STAGES) & 1), wc, kSiteKFull);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t st = sbase + (uint32_t)s * G::STAGE_BYTES;
        const uint64_t ad0 = ptx::sdesc_sw128(st, 16u, 1024u);
        const uint64_t bd0 = ptx::sdesc_sw128(st + G::A_BYTES, G::B_CHUNK, 1024u);
#pragma unroll
        for (int kk = 0; kk < G::BK / 16; ++kk) {
          const uint64_t ad = ad0 + (uint64_t)(((uint32_t)kk * 32u) >> 4);       // 32 bytes along a row
          const uint64_t bd = bd0 + (uint64_t)(((uint32_t)kk * 16u * 128u) >> 4);  // 16 rows of 128 bytes
          ptx::warp_mma_ss<false>(d_t, ad, bd, G::IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
        }
        ptx::warp_commit(bar(G::B_EMPTY + s));
      }
      if (!ok) break;
      ptx::warp_commit(bar(G::B_ACCF + acc));
    }
    // all issued MMAs must finish before tensor memory is freed
    ptx::warp_commit(bar(G::B_DRAIN));
    wait_bar_warp<kRoleMma>(bar(G::B_DRAIN), 0u, wc, kSiteDrain);
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == G::MMA_WARP) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

}  // namespace attn
