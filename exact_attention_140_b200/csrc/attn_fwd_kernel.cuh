// attn_fwd_kernel.cuh -- fused exact-attention forward for sm_100a.
//
// One CTA computes NQT query tiles of 128 rows for one (batch, query head).
// It walks the key/value tiles of that head once, keeping the output
// accumulator on chip, so neither the score matrix nor partial outputs ever
// reach HBM (page "FlashAttention (SV)": tiling, online softmax and operator
// fusion; the query-tile-outer loop order is the one page "FlashAttention-4
// 震撼发布" credits to FlashAttention-2's re-partitioned work).
//
// Warp roles (warp specialisation, page "FlashAttention-3 — 闪电注意力-3",
// section 1, recast for tcgen05):
//   warps 0 .. 4*NQT-1  softmax: warp w serves query tile w/4 and TMEM lanes
//                       32*(w%4) .. +31, so thread = one query row;
//   warp 4*NQT          TMA producer: Q tiles once, then K_j and V_j through
//                       KST / VST-stage shared-memory rings (section 2: the
//                       next block is fetched while the current one computes);
//   warp 4*NQT+1        MMA issuer: the warp runs the issue loop and one
//                       elected lane issues every tcgen05.mma; it also
//                       allocates and frees tensor memory;
//   warps 4*NQT+2, +3   idle (they complete the control warpgroup, whose
//                       registers are handed to the softmax warpgroups).
//
// Tensor memory (128 lanes x 512 fp32 columns): per query tile t, SB score
// buffers S of BN columns (P overwrites S in place: BN/2 columns of packed
// bf16, or BN/4 of e4m3) and the output accumulator O of D columns.  With two
// query tiles (NQT = 2) the tensor core alternates between them, so one
// tile's softmax runs under the other's matrix products (the ping-pong idea
// of section 1); with one tile the score buffer is doubled instead (SB = 2)
// so S_{j+1} = Q K_{j+1}^T runs under the softmax of S_j.
//
// Per key tile j and query tile t:
//   S   = Q_t K_j^T                          (tcgen05, SS operands, fp32 in TMEM)
//   m_b = rowmax(scale*log2e * S)            (masked on partial tiles)
//   if m_b > m_ref + TAU: rescale O_t and l by 2^(m_ref - m_b), m_ref = m_b
//   P   = 2^(scale*log2e * S - m_ref);  l += rowsum(P)
//   O_t += P V_j                             (tcgen05, A = P from TMEM)
// The reference max only moves when the block max exceeds it by more than
// TAU (lazy rescaling; page "FlashAttention-4震撼发布", the new online
// softmax that skips most output rescalings).  The result is the same for any
// TAU because the reference cancels in O = acc / l; TAU = 8 bounds P by 2^8.
// Epilogue: O = O_t / l (bf16), LSE = ln2 * (m_ref + log2 l).
//
// Split-KV (launch parameters n_splits, kv_chunk, o_part, lse_part): a block
// then covers one window of the keys (grid z = batch x window; the tile plan
// is shifted so that the causal rule keeps absolute key indices) and writes
// fp32 partials O_s = O_t / l and LSE_s for attn_combine.  With head packing
// (PACK configurations, launch parameter pack = g) the g query heads of one
// key/value head share the query tiles: query row i of head h sits at tile
// row i * g + h % g, and grid y runs over key/value heads.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>
#include <type_traits>

#include "attn_common.cuh"
#include "exp2_soft.cuh"
#include "ptx.cuh"
#include "tiles.h"

namespace attn {



template <class Cfg>
__global__ void __launch_bounds__(Cfg::NTHREADS, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const FwdParams p) {
  constexpr int BM = Cfg::BM, BN = Cfg::BN, D = Cfg::D, NQT = Cfg::NQT, SB = Cfg::SB;
  static_assert(!Cfg::PSEP, "P overwrites S in this kernel");
  constexpr int KST = Cfg::KST, VST = Cfg::VST;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = ptx::smem_u32(smem_raw);
  const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw_u32);
  auto bar = [&](int i) -> uint32_t { return sbase + Cfg::OFF_BAR + 8u * (uint32_t)i; };
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sgen + Cfg::OFF_ABORT);
  const WaitCtx wc{abort_flag, p.err, p.timeout_ns};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = Cfg::PACK ? p.pack : 1;  // query heads stacked per tile row group
  int qb, hy, b, split;
  if (p.band > 0) {
    // longest-first within bands of (batch, head) pairs: a band's K/V stay in
    // L2 while its blocks run, and the hardware hands out blocks in this
    // order as SMs free up, so the long causal blocks do not end up last
    const int L = (int)blockIdx.x, nbh = p.nb * p.nh;
    const int bi = L / (p.band * p.n_qblocks);
    const int within = L - bi * p.band * p.n_qblocks;
    const int bsz = nbh - bi * p.band < p.band ? nbh - bi * p.band : p.band;
    const int r = bi * p.band + within % bsz;
    qb = p.n_qblocks - 1 - within / bsz;
    hy = p.h0 + r % p.nh;
    b = p.b0 + r / p.nh;
    split = 0;
  } else {
    qb = p.n_qblocks - 1 - (int)blockIdx.x;  // longest causal blocks first
    // query head, or key/value head when packed (grid y covers the launch's heads)
    hy = (g > 1 ? p.h0 / g : p.h0) + (int)blockIdx.y;
    b = p.b0 + (int)blockIdx.z / p.n_splits;
    split = (int)blockIdx.z % p.n_splits;
  }
  // key window of this block: [kv0, kv0 + nk), `shift` keys after it
  const int kv0 = split * p.kv_chunk;
  const int nk = p.Nk - kv0 < p.kv_chunk ? p.Nk - kv0 : p.kv_chunk;
  const int shift = p.Nk - kv0 - nk;
  const int kh = g > 1 ? hy : hy / p.group;
  const int q0 = qb * BM * NQT;
  int n_kv[NQT];
  int nmax = 0;
  // query rows [ia, ib) of tile t (packed rows r hold query row r / g)
  auto tile_rows = [&](int t, int& ia, int& ib) {
    ia = (q0 + t * BM) / g;
    ib = (q0 + (t + 1) * BM + g - 1) / g;
  };
#pragma unroll
  for (int t = 0; t < NQT; ++t) {
    int ia, ib;
    tile_rows(t, ia, ib);
    n_kv[t] = kv_tile_count(ia, ib, p.Nq, nk, BN, Cfg::CAUSAL, shift);
    nmax = n_kv[t] > nmax ? n_kv[t] : nmax;
  }

  if (threadIdx.x == 0) {
    for (int t = 0; t < NQT; ++t) ptx::mbar_init(bar(Cfg::B_QFULL + t), 1);
    for (int s = 0; s < KST; ++s) {
      ptx::mbar_init(bar(Cfg::B_KFULL + s), 1);
      ptx::mbar_init(bar(Cfg::B_KEMPTY + s), 1);
    }
    for (int s = 0; s < VST; ++s) {
      ptx::mbar_init(bar(Cfg::B_VFULL + s), 1);
      ptx::mbar_init(bar(Cfg::B_VEMPTY + s), 1);
    }
    for (int i = 0; i < NQT * SB; ++i) {
      ptx::mbar_init(bar(Cfg::B_SFULL + i), 1);
      ptx::mbar_init(bar(Cfg::B_PFULL + i), 128);
      ptx::mbar_init(bar(Cfg::B_PHALF + i), 128);
    }
    for (int t = 0; t < NQT; ++t) {
      ptx::mbar_init(bar(Cfg::B_ODONE + t), 1);
      ptx::mbar_init(bar(Cfg::B_OFINAL + t), 1);
    }
    ptx::mbar_init(bar(Cfg::B_DRAIN), 1);
    *abort_flag = 0u;
    ptx::fence_mbar_init();
  }
  if (warp == Cfg::TMA_WARP && lane == 0) {
    ptx::prefetch_tmap(&tmQ);
    ptx::prefetch_tmap(&tmK);
    ptx::prefetch_tmap(&tmV);
  }
  if (warp == Cfg::MMA_WARP) {
    ptx::tmem_alloc(sbase + Cfg::OFF_SLOT, Cfg::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sgen + Cfg::OFF_SLOT);

  if (warp < Cfg::SM_WARPS) {
    // ------------------------------------------------------------ softmax
    if constexpr (Cfg::SPLIT_REGS) ptx::setmaxnreg_inc<Cfg::REG_SOFTMAX>();
    const int t = warp >> 2, wq = warp & 3;
    int ia, ib;
    tile_rows(t, ia, ib);
    const int prow = q0 + t * BM + wq * 32 + lane;  // this thread's (packed) tile row
    const int row = prow / g;                         // its query row
    const int h = g > 1 ? kh * g + (prow - row * g) : hy;
    const int nt = n_kv[t];
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t o_taddr = tmem + lane_off + (uint32_t)(Cfg::O_COL0 + t * D);
    float sl2 = p.sl2;
    if constexpr (Cfg::FP8) sl2 *= __ldg(p.dq) * __ldg(p.dk);
    const long long vend = vis_end(row, p.Nq, nk, Cfg::CAUSAL, shift);
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < nt; ++j) {
      const int si = t * SB + (j % SB);
      ok = wait_bar<kRoleSoftmax>(bar(Cfg::B_SFULL + si), (uint32_t)((j / SB) & 1), wc, kSiteSFull);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      ptx::tc_fence_after();
      const uint32_t s_taddr = tmem + lane_off + (uint32_t)(si * BN);
      const bool partial = tile_kind(ia, ib, j, p.Nq, nk, BN, Cfg::CAUSAL, shift) == kTilePartial;
      const int nvis = (int)(vend - (long long)j * BN);  // visible keys of this tile (masks partial tiles)
      // ---- one read of the whole score row per tile, in two halves: the
      // second half's loads are in flight while the first half's maximum is
      // taken (full tiles, scale >= 0)
      uint32_t sr[BN];
      constexpr int NCH = BN / 32, NCH0 = NCH / 2 > 0 ? NCH / 2 : 1;
      const bool fast_max = !partial && sl2 >= 0.f;
      float a0 = -INFINITY, a1 = -INFINITY, a2 = -INFINITY, a3 = -INFINITY;
#pragma unroll
      for (int c = 0; c < NCH0; ++c)
        ptx::tmem_ld32(s_taddr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
#pragma unroll
      for (int c = 0; c < NCH0; ++c) ptx::tmem_wait_ld_dep(*reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
#pragma unroll
      for (int c = NCH0; c < NCH; ++c)
        ptx::tmem_ld32(s_taddr + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
      auto fold = [&](int c0, int c1) {  // a0..a3 <- their max with scores [c0, c1)
#pragma unroll
        for (int c = c0; c < c1; c += 8) {
          a0 = ptx::fmax3(a0, __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
          a1 = ptx::fmax3(a1, __uint_as_float(sr[c + 2]), __uint_as_float(sr[c + 3]));
          a2 = ptx::fmax3(a2, __uint_as_float(sr[c + 4]), __uint_as_float(sr[c + 5]));
          a3 = ptx::fmax3(a3, __uint_as_float(sr[c + 6]), __uint_as_float(sr[c + 7]));
        }
      };
      if (fast_max) fold(0, 32 * NCH0);
#pragma unroll
      for (int c = NCH0; c < NCH; ++c) ptx::tmem_wait_ld_dep(*reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
      float m_blk;
      if (partial) {
        m_blk = masked_max_scaled<BN>(sr, nvis, sl2);
      } else if (sl2 >= 0.f) {
        fold(32 * NCH0, BN);
        m_blk = ptx::fmax3(a0, a1, fmaxf(a2, a3)) * sl2;
      } else {  // a negative scale turns the row max into the row min
        float mn = __uint_as_float(sr[0]);
#pragma unroll
        for (int c = 1; c < BN; ++c) mn = fminf(mn, __uint_as_float(sr[c]));
        m_blk = mn * sl2;
      }
      float alpha = 1.f;
      bool resc = false;
      if (m_blk > m_ref + kTau) {
        alpha = ptx::ex2(m_ref - m_blk);  // 0 when m_ref = -inf
        resc = (m_ref != -INFINITY);
        m_ref = m_blk;
        l *= alpha;
      }
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      const bool resc_any = __any_sync(0xffffffffu, resc);
      // P released in two halves (non-causal: measured faster; with causal
      // masks the extra live state costs more than the overlap gains)
      constexpr bool kHalfP = !Cfg::CAUSAL;
      // ---- exponentiate 32 columns at a time; each chunk's packed P is
      // stored at once (over score columns already read), so the registers of
      // a chunk die before the next chunk is processed
      uint64_t lsum[4] = {ptx::f2(0.f, 0.f), ptx::f2(0.f, 0.f), ptx::f2(0.f, 0.f), ptx::f2(0.f, 0.f)};
      const uint64_t sl2x2 = ptx::f2(sl2, sl2), negm2 = ptx::f2(-m_use, -m_use);
      constexpr int PW = Cfg::FP8 ? 8 : 16;  // packed P words per 32 scores
      // The tile kind is resolved once, outside the unrolled loop: one loop
      // body per kind, no per-element branches.
      auto exp_row = [&](auto partial_tag) {
        constexpr bool PARTIAL = decltype(partial_tag)::value;
#pragma unroll
        for (int ch = 0; ch < BN / 32; ++ch) {
          uint32_t pk[PW];
          [[maybe_unused]] float hold0 = 0.f, hold1 = 0.f;
#pragma unroll
          for (int c = 0; c < 16; ++c) {
            const int col = 32 * ch + 2 * c;
            const float s0 = __uint_as_float(sr[col]), s1 = __uint_as_float(sr[col + 1]);
            float e0, e1;
            const uint64_t x = ptx::ffma2(ptx::f2(s0, s1), sl2x2, negm2);
            float x0, x1;
            ptx::unf2(x, x0, x1);
            if (((16 * ch + c) % 8) < Cfg::EMU) {
              exp2_soft2(x0, x1, e0, e1);
            } else {
              e0 = ptx::ex2(x0);
              e1 = ptx::ex2(x1);
            }
            if constexpr (PARTIAL) {  // masked keys (a prefix is visible) get exact zeros
              e0 = col < nvis ? e0 : 0.f;
              e1 = col + 1 < nvis ? e1 : 0.f;
            }
            lsum[c % 4] = ptx::fadd2(lsum[c % 4], ptx::f2(e0, e1));
            if constexpr (Cfg::FP8) {
              if (c % 2 == 0) {
                hold0 = e0;
                hold1 = e1;
              } else {
                pk[c / 2] = ptx::pack_e4m3x4(hold0, hold1, e0, e1);
              }
            } else {
              pk[c] = ptx::pack_bf16x2(e0, e1);
            }
          }
          if constexpr (Cfg::FP8)
            ptx::tmem_st8(s_taddr + (uint32_t)(PW * ch), pk);
          else
            ptx::tmem_st16(s_taddr + (uint32_t)(PW * ch), pk);
          if (kHalfP && ch == BN / 64 - 1 && !resc_any) {
            // the first half of P is in tensor memory: the P V over the first
            // half of the keys can start while the second half is
            // exponentiated (a warp that must rescale O first releases it
            // after the rescale instead)
            ptx::tmem_wait_st();
            ptx::tc_fence_before();
            ptx::mbar_arrive(bar(Cfg::B_PHALF + si));
          }
        }
      };
      if (partial)
        exp_row(std::true_type{});
      else
        exp_row(std::false_type{});
      {
        float la, lb;
        ptx::unf2(ptx::fadd2(ptx::fadd2(lsum[0], lsum[1]), ptx::fadd2(lsum[2], lsum[3])), la, lb);
        l += la + lb;
      }
      ptx::tmem_wait_st();
      if (resc_any) {
        // O_t must hold exactly the products of key tiles < j: wait for
        // PV(t, j-1).  Whenever S(t, j) is ready, PV(t, j-2) has completed (it
        // was issued before QK(t, j)) and PV(t, j) is not issued yet, so the
        // o_done barrier has completed j-1 or j phases and the parity test
        // for phase j-1 is unambiguous.
        ok = wait_bar<kRoleSoftmax>(bar(Cfg::B_ODONE + t), (uint32_t)((j - 1) & 1), wc, kSiteODone);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ptx::tc_fence_after();
        const float a = resc ? alpha : 1.f;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          ptx::tmem_ld32(o_taddr + 32 * c, r);
          ptx::tmem_wait_ld_dep(r);
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * a);
          ptx::tmem_st32(o_taddr + 32 * c, r);
        }
        ptx::tmem_wait_st();
      }
      ptx::tc_fence_before();
      if (!Cfg::CAUSAL && resc_any) ptx::mbar_arrive(bar(Cfg::B_PHALF + si));
      ptx::mbar_arrive(bar(Cfg::B_PFULL + si));
    }
    // ------------------------------------------------------------ epilogue
    if (ok && nt > 0) {  // o_final completes once, after the tile's last PV
      ok = wait_bar<kRoleSoftmax>(bar(Cfg::B_OFINAL + t), 0u, wc, kSiteODone);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      ptx::tc_fence_after();
      const bool store = row < p.Nq;
      float inv = l > 0.f ? 1.f / l : 0.f;
      if constexpr (Cfg::FP8) inv *= __ldg(p.dv);
      const float lse = l > 0.f ? (m_ref + log2f(l)) * 0.6931471805599453f : -INFINITY;
      if (p.o_part == nullptr) {
        __nv_bfloat16* orow =
            reinterpret_cast<__nv_bfloat16*>(p.o) + (((long long)b * p.Nq + row) * p.Hq + h) * (long long)D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          if (nt > 0) {
            ptx::tmem_ld32(o_taddr + 32 * c, r);
            ptx::tmem_wait_ld_dep(r);
          }
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[e] = nt > 0 ? ptx::pack_bf16x2(__uint_as_float(r[2 * e]) * inv, __uint_as_float(r[2 * e + 1]) * inv)
                          : 0u;
          if (store) {
            uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
          }
        }
        if (store && p.lse != nullptr) p.lse[((long long)b * p.Hq + h) * p.Nq + row] = lse;
      } else {
        // split-KV partial of window `split`: fp32 O_s and LSE_s
        const long long zs = (long long)split * p.B + b;
        float* orow = p.o_part + ((zs * p.Nq + row) * p.Hq + h) * (long long)D;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          if (nt > 0) {
            ptx::tmem_ld32(o_taddr + 32 * c, r);
            ptx::tmem_wait_ld_dep(r);
          }
          if (store) {
            float4* dst = reinterpret_cast<float4*>(orow + 32 * c);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = nt > 0 ? make_float4(__uint_as_float(r[4 * e]) * inv, __uint_as_float(r[4 * e + 1]) * inv,
                                            __uint_as_float(r[4 * e + 2]) * inv, __uint_as_float(r[4 * e + 3]) * inv)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
        if (store) p.lse_part[(zs * p.Hq + h) * p.Nq + row] = lse;
      }
    }
  } else if (warp == Cfg::TMA_WARP) {
    // ------------------------------------------------------------ producer
    if constexpr (Cfg::SPLIT_REGS) ptx::setmaxnreg_dec<Cfg::REG_CONTROL>();
    if (lane == 0) {
      int k_issued[KST], v_issued[VST];
#pragma unroll
      for (int s = 0; s < KST; ++s) k_issued[s] = 0;
#pragma unroll
      for (int s = 0; s < VST; ++s) v_issued[s] = 0;
      bool q_issued[NQT];
#pragma unroll
      for (int t = 0; t < NQT; ++t) {
        q_issued[t] = n_kv[t] > 0;
        if (!q_issued[t]) continue;
        const uint32_t fb = bar(Cfg::B_QFULL + t);
        ptx::mbar_arrive_expect_tx(fb, Cfg::QT_BYTES);
#pragma unroll
        for (int c = 0; c < Cfg::NCH; ++c) {
          const uint32_t dst = sbase + Cfg::OFF_Q + t * Cfg::QT_BYTES + c * Cfg::CH_Q;
          if (Cfg::PACK && g > 1)  // box: g heads x BM / g rows of kv head kh
            ptx::tma_load_5d(dst, &tmQ, fb, c * Cfg::BOXE, 0, kh, (q0 + t * BM) / g, b);
          else
            ptx::tma_load_4d(dst, &tmQ, fb, c * Cfg::BOXE, hy, q0 + t * BM, b);
        }
      }
      for (int j = 0; j < nmax; ++j) {
        const int ks = j % KST;
        if (j >= KST && !wait_bar<kRoleProducer>(bar(Cfg::B_KEMPTY + ks), (uint32_t)(((j / KST) - 1) & 1), wc, kSiteKEmpty))
          break;
        {
          const uint32_t fb = bar(Cfg::B_KFULL + ks);
          ptx::mbar_arrive_expect_tx(fb, Cfg::KV_BYTES);
#pragma unroll
          for (int c = 0; c < Cfg::NCH; ++c)
            ptx::tma_load_4d(sbase + Cfg::OFF_K + ks * Cfg::KV_BYTES + c * Cfg::CH_KV, &tmK, fb, c * Cfg::BOXE,
                             kh, kv0 + j * BN, b);
          ++k_issued[ks];
        }
        const int vs = j % VST;
        if (j >= VST && !wait_bar<kRoleProducer>(bar(Cfg::B_VEMPTY + vs), (uint32_t)(((j / VST) - 1) & 1), wc, kSiteVEmpty))
          break;
        {
          const uint32_t fb = bar(Cfg::B_VFULL + vs);
          ptx::mbar_arrive_expect_tx(fb, Cfg::KV_BYTES);
#pragma unroll
          for (int c = 0; c < Cfg::NCH; ++c)
            ptx::tma_load_4d(sbase + Cfg::OFF_V + vs * Cfg::KV_BYTES + c * Cfg::CH_KV, &tmV, fb, c * Cfg::BOXE,
                             kh, kv0 + j * BN, b);
          ++v_issued[vs];
        }
      }
      // Every issued copy must land before the block may exit (no-op in the
      // normal path, where the consumers have already seen them all).
#pragma unroll
      for (int t = 0; t < NQT; ++t)
        if (q_issued[t]) wait_bar_drain<kRoleProducer>(bar(Cfg::B_QFULL + t), 0u, wc, kSiteQ);
#pragma unroll
      for (int s = 0; s < KST; ++s)
        if (k_issued[s] > 0) wait_bar_drain<kRoleProducer>(bar(Cfg::B_KFULL + s), (uint32_t)((k_issued[s] - 1) & 1), wc, kSiteKFull);
#pragma unroll
      for (int s = 0; s < VST; ++s)
        if (v_issued[s] > 0) wait_bar_drain<kRoleProducer>(bar(Cfg::B_VFULL + s), (uint32_t)((v_issued[s] - 1) & 1), wc, kSiteVFull);
    }
  } else {
    if constexpr (Cfg::SPLIT_REGS) ptx::setmaxnreg_dec<Cfg::REG_CONTROL>();
  }
  if (warp == Cfg::MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop (waits, counters, descriptors); one
    // elected lane issues the tcgen05 instructions.
    {
      bool ok = true;
#pragma unroll
      for (int t = 0; t < NQT && ok; ++t)
        if (n_kv[t] > 0) ok = wait_bar_warp<kRoleMma>(bar(Cfg::B_QFULL + t), 0u, wc, kSiteQ);
      ptx::tc_fence_after();
      const uint32_t q_s = sbase + Cfg::OFF_Q, k_s = sbase + Cfg::OFF_K, v_s = sbase + Cfg::OFF_V;
      auto issue_qk = [&](int t, int j) {
        const uint32_t d_t = tmem + (uint32_t)((t * SB + j % SB) * BN);
        // descriptors advance by 32 bytes (>> 4 = 2) per K step inside a
        // 128-byte chunk and by one chunk (CH_Q / CH_KV bytes) after four
        const uint64_t ad0 = ptx::sdesc_sw128(q_s + t * Cfg::QT_BYTES, 16u, 1024u);
        const uint64_t bd0 = ptx::sdesc_sw128(k_s + (j % KST) * Cfg::KV_BYTES, 16u, 1024u);
#pragma unroll
        for (int kk = 0; kk < Cfg::QK_STEPS; ++kk) {
          const uint32_t ch = (uint32_t)kk / 4u, in = (uint32_t)kk % 4u;
          const uint64_t ad = ad0 + (uint64_t)((ch * Cfg::CH_Q + in * 32u) >> 4);
          const uint64_t bd = bd0 + (uint64_t)((ch * Cfg::CH_KV + in * 32u) >> 4);
          ptx::warp_mma_ss<Cfg::FP8>(d_t, ad, bd, Cfg::IDESC_QK, kk > 0 ? 1u : 0u);
        }
        ptx::warp_commit(bar(Cfg::B_SFULL + t * SB + j % SB));
      };
      auto issue_pv = [&](int t, int jj) -> bool {
        const int si = t * SB + jj % SB;
        const uint32_t ph = (uint32_t)((jj / SB) & 1);
        const uint32_t d_t = tmem + (uint32_t)(Cfg::O_COL0 + t * D);
        const uint32_t a_t = tmem + (uint32_t)(si * BN);
        const uint64_t bd0 = ptx::sdesc_sw128(v_s + (jj % VST) * Cfg::KV_BYTES, Cfg::CH_KV, 1024u);
        // non-causal: the first half of the keys as soon as their P is
        // written, the rest when the whole P is; causal: all at once
#pragma unroll
        for (int half = Cfg::CAUSAL ? 1 : 0; half < 2; ++half) {
          if (!wait_bar_warp<kRoleMma>(bar((half == 0 ? Cfg::B_PHALF : Cfg::B_PFULL) + si), ph, wc, kSitePFull))
            return false;
          ptx::tc_fence_after();
#pragma unroll
          for (int kk = (Cfg::CAUSAL ? 0 : half * Cfg::PV_STEPS / 2); kk < (half + 1) * Cfg::PV_STEPS / 2; ++kk) {
            const uint64_t bd = bd0 + (uint64_t)(((uint32_t)kk * Cfg::KSTEP * 128u) >> 4);
            ptx::warp_mma_ts<Cfg::FP8>(d_t, a_t + (uint32_t)kk * 8u, bd, Cfg::IDESC_PV,
                                       (jj > 0 || kk > 0) ? 1u : 0u);
          }
        }
        ptx::warp_commit(bar(Cfg::B_ODONE + t));
        if (jj == n_kv[t] - 1) ptx::warp_commit(bar(Cfg::B_OFINAL + t));
        return true;
      };
      for (int j = 0; ok && j <= nmax; ++j) {
        const bool has_k = j < nmax, has_v = j >= 1;
        if constexpr (SB == 2) {
          // S is double-buffered: the products for key tile j go first, so
          // they run under the softmax of key tile j-1; then the P V of
          // key tile j-1 as each tile's P is released
          if (has_k) {
            ok = wait_bar_warp<kRoleMma>(bar(Cfg::B_KFULL + j % KST), (uint32_t)((j / KST) & 1), wc, kSiteKFull);
            if (!ok) break;
            ptx::tc_fence_after();
#pragma unroll
            for (int t = 0; t < NQT; ++t)
              if (j < n_kv[t]) issue_qk(t, j);
            ptx::warp_commit(bar(Cfg::B_KEMPTY + j % KST));
          }
          if (has_v) {
            ok = wait_bar_warp<kRoleMma>(bar(Cfg::B_VFULL + (j - 1) % VST), (uint32_t)(((j - 1) / VST) & 1),
                                         wc, kSiteVFull);
            if (!ok) break;
            ptx::tc_fence_after();
#pragma unroll
            for (int t = 0; t < NQT && ok; ++t)
              if (j - 1 < n_kv[t]) ok = issue_pv(t, j - 1);
            if (!ok) break;
            ptx::warp_commit(bar(Cfg::B_VEMPTY + (j - 1) % VST));
          }
        } else {
          // P overwrites S in place: PV(t, j-1) must be issued before
          // QK(t, j) reuses the buffer
          if (has_k) {
            ok = wait_bar_warp<kRoleMma>(bar(Cfg::B_KFULL + j % KST), (uint32_t)((j / KST) & 1), wc, kSiteKFull);
            if (!ok) break;
          }
          if (has_v) {
            ok = wait_bar_warp<kRoleMma>(bar(Cfg::B_VFULL + (j - 1) % VST), (uint32_t)(((j - 1) / VST) & 1),
                                         wc, kSiteVFull);
            if (!ok) break;
          }
          ptx::tc_fence_after();
#pragma unroll
          for (int t = 0; t < NQT && ok; ++t) {
            if (has_v && j - 1 < n_kv[t]) ok = issue_pv(t, j - 1);
            if (ok && has_k && j < n_kv[t]) issue_qk(t, j);
          }
          if (!ok) break;
          if (has_k) ptx::warp_commit(bar(Cfg::B_KEMPTY + j % KST));
          if (has_v) ptx::warp_commit(bar(Cfg::B_VEMPTY + (j - 1) % VST));
        }
      }
      // All issued MMAs must finish before tensor memory is freed.
      ptx::warp_commit(bar(Cfg::B_DRAIN));
      wait_bar_warp<kRoleMma>(bar(Cfg::B_DRAIN), 0u, wc, kSiteDrain);
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == Cfg::MMA_WARP) {
    __syncwarp();
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, Cfg::TMEM_COLS);
  }
}

}  // namespace attn
