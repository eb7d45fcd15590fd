// attn_fwd_persistent_kernel.cuh -- persistent variant of the fused
// attention forward, for short key ranges.
//
// It computes the same thing as attn_fwd_kernel (same tiles, warp roles,
// online softmax with lazy rescaling and epilogue; see that file), but a grid
// of one block per SM loops over the work items (batch, query head, query
// block) instead of launching one block per item.  With short key ranges an
// item is only a few key tiles long and the fixed costs around it -- block
// start, tensor-memory allocation, the first Q and K/V loads, the epilogue's
// read-out of O -- are a large share of its time; here they overlap with the
// neighbouring items:
//   * the producer issues the next item's first K/V tile while the current
//     item is still computing, and its Q tile as soon as the last Q K^T of
//     the current item has completed (barrier q_empty);
//   * the MMA warp starts the next item's products while the softmax
//     warpgroups write out the previous output; only its first P V waits
//     for that output's read-out (barrier o_free);
//   * each P is released in two halves (barrier p_half): the P V over the
//     first half of the keys starts while the second half is exponentiated.
// Ring slots and barrier phases are counted across items, so the pipeline
// never drains between them.
//
// Two layouts of the block:
//   * NS = 1: NQT query tiles of one item share the K/V stream (as in
//     attn_fwd_kernel);
//   * NS = 2 (d = 64): two independent streams, each with one softmax
//     warpgroup, its own TMA and MMA warps (the four warps of the control
//     warpgroup), K/V rings, barriers and 256 tensor-memory columns, taking
//     128-row work items of their own.  The streams do not wait for each
//     other at item boundaries, which with causal masks (query tiles of one
//     item differ in length) left a tile idle for about a step per item.
// PSEP (d = 64) gives P columns of its own (S 128 + P 64 + O 64 per tile), so
// Q K_{j+1}^T runs during the softmax of tile j; the softmax signals s_free
// once S is in registers and waits for the previous P V before storing the
// first chunk of P (after that chunk's exponentials, which hide the product).
// OST (d = 64) stages each output tile in shared memory and writes it with one
// TMA store: the rows of O are H * d elements apart, so one row per thread
// would make every store instruction touch 32 rows; o_free is signalled as
// soon as O has left tensor memory.
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

// Work items are (batch, query head, query block).  The grid is persistent
// (one block per SM, NS streams per block); stream c of G takes items c,
// 2G-1-c, 2G+c, 4G-1-c, ... of an order sorted longest-first (for causal
// masks), so long and short items pair up.  Head-major order keeps the query
// blocks of one head on the GPU at the same time (their K/V tiles are shared
// through L2).
__device__ __forceinline__ int item_at(int k, int G, int T, int c) {
  const long long pos = (long long)k * G + ((k & 1) ? (G - 1 - c) : c);
  return pos < T ? (int)pos : -1;
}
struct Item {
  int qb, h, b;
};
__device__ __forceinline__ Item decode_item(int i, const FwdParams& p) {
  const int bh = p.nb * p.nh;
  int qr, r;
  if (p.qb_major) {
    qr = i / bh;
    r = i - qr * bh;
  } else {
    r = i / p.n_qblocks;
    qr = i - r * p.n_qblocks;
  }
  return Item{p.n_qblocks - 1 - qr, p.h0 + r % p.nh, p.b0 + r / p.nh};
}

template <class Cfg>
__global__ void __launch_bounds__(Cfg::NTHREADS, 1)
    attn_fwd_persistent_kernel(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                               const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                               const FwdParams p) {
  constexpr int BM = Cfg::BM, BN = Cfg::BN, D = Cfg::D, NQT = Cfg::NQT, SB = Cfg::SB;
  constexpr int KST = Cfg::KST, VST = Cfg::VST;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = ptx::smem_u32(smem_raw);
  const uint32_t sbase = (raw_u32 + 1023u) & ~1023u;
  uint8_t* sgen = smem_raw + (sbase - raw_u32);
  volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(sgen + Cfg::OFF_ABORT);
  const WaitCtx wc{abort_flag, p.err, p.timeout_ns};

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // role and stream of this warp
  const int cw = warp - Cfg::SM_WARPS;  // index within the control warpgroup
  const bool is_tma = cw >= 0 && cw < 2 * Cfg::NS && (cw & 1) == 0;
  const bool is_mma = cw >= 0 && cw < 2 * Cfg::NS && (cw & 1) == 1;
  const int s = warp < Cfg::SM_WARPS ? warp / (4 * NQT) : ((is_tma || is_mma) ? (cw >> 1) : 0);
  auto bar_s = [&](int ss, int i) -> uint32_t {
    return sbase + Cfg::OFF_BAR + 8u * (uint32_t)(ss * Cfg::NBAR + i);
  };
  auto bar = [&](int i) -> uint32_t { return bar_s(s, i); };
  const uint32_t sstream = sbase + (uint32_t)s * Cfg::STREAM_BYTES;  // Q/K/V tiles of this stream
  const int G = (int)gridDim.x * Cfg::NS, T = p.n_items;
  const int c = (int)blockIdx.x * Cfg::NS + s;  // this stream's index in the grid
  // key tiles the query tiles of an item visit (0 = none)
  auto plan = [&](const Item& it, int (&n_kv)[NQT]) -> int {
    const int q0 = it.qb * BM * NQT;
    int nmax = 0;
#pragma unroll
    for (int t = 0; t < NQT; ++t) {
      n_kv[t] = kv_tile_count(q0 + t * BM, q0 + (t + 1) * BM, p.Nq, p.Nk, BN, Cfg::CAUSAL);
      nmax = n_kv[t] > nmax ? n_kv[t] : nmax;
    }
    return nmax;
  };

  if (threadIdx.x == 0) {
    for (int ss = 0; ss < Cfg::NS; ++ss) {
    for (int t = 0; t < NQT; ++t) ptx::mbar_init(bar_s(ss, Cfg::B_QFULL + t), 1);
    for (int s = 0; s < KST; ++s) {
      ptx::mbar_init(bar_s(ss, Cfg::B_KFULL + s), 1);
      ptx::mbar_init(bar_s(ss, Cfg::B_KEMPTY + s), 1);
    }
    for (int s = 0; s < VST; ++s) {
      ptx::mbar_init(bar_s(ss, Cfg::B_VFULL + s), 1);
      ptx::mbar_init(bar_s(ss, Cfg::B_VEMPTY + s), 1);
    }
    for (int i = 0; i < NQT * SB; ++i) {
      ptx::mbar_init(bar_s(ss, Cfg::B_SFULL + i), 1);
      ptx::mbar_init(bar_s(ss, Cfg::B_PFULL + i), 128);
      ptx::mbar_init(bar_s(ss, Cfg::B_PHALF + i), 128);
    }
    for (int t = 0; t < NQT; ++t) {
      ptx::mbar_init(bar_s(ss, Cfg::B_ODONE + t), 1);
      ptx::mbar_init(bar_s(ss, Cfg::B_OFINAL + t), 1);
      ptx::mbar_init(bar_s(ss, Cfg::B_OFREE + t), 128);
    }
    ptx::mbar_init(bar_s(ss, Cfg::B_QEMPTY), 1);
    for (int i = 0; i < NQT * SB; ++i) ptx::mbar_init(bar_s(ss, Cfg::B_SFREE + i), 128);
    ptx::mbar_init(bar_s(ss, Cfg::B_DRAIN), 1);
    }
    *abort_flag = 0u;
    ptx::fence_mbar_init();
  }
  if (is_tma && lane == 0) {
    ptx::prefetch_tmap(&tmQ);
    ptx::prefetch_tmap(&tmK);
    ptx::prefetch_tmap(&tmV);
    if constexpr (Cfg::OST) ptx::prefetch_tmap(&tmO);
  }
  if (warp == Cfg::MMA_WARP) {
    ptx::tmem_alloc(sbase + Cfg::OFF_SLOT, Cfg::TMEM_COLS);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *reinterpret_cast<volatile uint32_t*>(sgen + Cfg::OFF_SLOT);
  const uint32_t tmem_s = tmem + (uint32_t)(s * Cfg::TMEM_USED);  // this stream's columns

  if (warp < Cfg::SM_WARPS) {
    // ------------------------------------------------------------ softmax
    if constexpr (Cfg::SPLIT_REGS) ptx::setmaxnreg_inc<Cfg::REG_SOFTMAX>();
    const int t = (warp >> 2) % NQT, wq = warp & 3;
    const uint32_t lane_off = (uint32_t)(wq * 32) << 16;
    const uint32_t o_taddr = tmem_s + lane_off + (uint32_t)(Cfg::O_COL0 + t * D);
    float sl2 = p.sl2;
    if constexpr (Cfg::FP8) sl2 *= __ldg(p.dq) * __ldg(p.dk);
    int scount = 0;       // score buffers of this query tile consumed so far (= P V products issued before)
    int finals = 0;       // items whose output this tile has written
    bool ok = true;
    for (int k = 0; ok; ++k) {
      const int item = item_at(k, G, T, c);
      if (item < 0) break;
      const Item it = decode_item(item, p);
      int n_kv[NQT];
      plan(it, n_kv);
      const int row0 = it.qb * BM * NQT + t * BM;
      const int row = row0 + wq * 32 + lane;
      const int nt = n_kv[t];
      const int vend = (int)vis_end(row, p.Nq, p.Nk, Cfg::CAUSAL);
      float m_ref = -INFINITY, l = 0.f;
      for (int j = 0; j < nt; ++j, ++scount) {
        const int si = t * SB + (scount % SB);
        ok = wait_bar<kRoleSoftmax>(bar(Cfg::B_SFULL + si), (uint32_t)((scount / SB) & 1), wc, kSiteSFull);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        ptx::tc_fence_after();
        const uint32_t s_taddr = tmem_s + lane_off + (uint32_t)(si * BN);
        const bool partial = tile_kind(row0, row0 + BM, j, p.Nq, p.Nk, BN, Cfg::CAUSAL) == kTilePartial;
        const int nvis = vend - j * BN;  // visible keys of this tile (masks partial tiles)
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
        if constexpr (Cfg::PSEP) {
          // S is in registers: the next Q K^T of this tile may overwrite it
          ptx::tc_fence_before();
          ptx::mbar_arrive(bar(Cfg::B_SFREE + si));
        }
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
        const uint32_t p_taddr =
            Cfg::PSEP ? tmem_s + lane_off + (uint32_t)(Cfg::P_COL0 + t * Cfg::P_COLS) : s_taddr;
        // ---- exponentiate 32 columns at a time; each chunk's packed P is
        // stored at once (over score columns already read), so the registers
        // of a chunk die before the next chunk is processed
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
            if constexpr (Cfg::PSEP) {
              // P has one buffer per tile: the previous P V (product scount -
              // 1) must have read it before the first chunk of this P is
              // stored; the wait comes after the first chunk's exponentials,
              // which hide most of that product.  Product scount cannot have
              // completed (its P is not written yet) and product scount - 2
              // was waited for one tile earlier, so the parity test is
              // unambiguous.  A failed wait stores the rest anyway (the block
              // is aborting; the addresses are its own) and leaves the loop
              // after this tile.  (A separate barrier for the first half of
              // the product, releasing the first chunks earlier, measured
              // slower: one more commit per tile on the MMA warp.)
              if (ch == 0 && scount > 0) {
                ok = wait_bar<kRoleSoftmax>(bar(Cfg::B_ODONE + t), (uint32_t)((scount - 1) & 1), wc, kSiteODone);
                ok = __all_sync(0xffffffffu, ok);
                ptx::tc_fence_after();
              }
            }
            if constexpr (Cfg::FP8)
              ptx::tmem_st8(p_taddr + (uint32_t)(PW * ch), pk);
            else
              ptx::tmem_st16(p_taddr + (uint32_t)(PW * ch), pk);
            if (ch == BN / 64 - 1 && !resc_any) {
              // the first half of P is in TMEM: its P V can start while the
              // second half is exponentiated (a warp that must rescale O
              // first releases it after the rescale instead)
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
        if (!ok) break;
        {
          float la, lb;
          ptx::unf2(ptx::fadd2(ptx::fadd2(lsum[0], lsum[1]), ptx::fadd2(lsum[2], lsum[3])), la, lb);
          l += la + lb;
        }
        ptx::tmem_wait_st();
        if (resc_any) {
          // O_t must hold exactly the products of key tiles < j: wait for
          // PV(t, j-1), the (scount - 1)-th product of this tile (one product
          // per score tile).  Whenever S(t, j) is ready the product before
          // that one has completed (it was issued before QK(t, j)) and PV(t, j)
          // is not issued yet, so the o_done barrier is within one phase of
          // the target and the parity test is unambiguous.
          ok = wait_bar<kRoleSoftmax>(bar(Cfg::B_ODONE + t), (uint32_t)((scount - 1) & 1), wc, kSiteODone);
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
        if (resc_any) ptx::mbar_arrive(bar(Cfg::B_PHALF + si));
        ptx::mbar_arrive(bar(Cfg::B_PFULL + si));
      }
      if (!Cfg::OST && !ok) break;
      // ---------------------------------------------------------- epilogue
      if (ok && nt > 0) {  // o_final completes once per item, after the tile's last PV
        ok = wait_bar<kRoleSoftmax>(bar(Cfg::B_OFINAL + t), (uint32_t)(finals & 1), wc, kSiteODone);
        ok = __all_sync(0xffffffffu, ok);
        if (ok) ++finals;
      }
      if constexpr (Cfg::OST) {
        // The staging tile is free once the previous item's store has read
        // it.  The four warps of the stream meet at this named barrier on
        // every item, failed waits included, and leave together.
        if (wq == 0 && lane == 0) ptx::bulk_wait_read0();
        ok = ptx::bar_red_and(1u + (uint32_t)s, 128u, ok);
      }
      if (!ok) break;
      ptx::tc_fence_after();
      const bool store = row < p.Nq;
      float inv = l > 0.f ? 1.f / l : 0.f;
      if constexpr (Cfg::FP8) inv *= __ldg(p.dv);
      const Item ie = decode_item(item, p);  // recomputed: keeps fewer values live through the key loop
      if constexpr (Cfg::OST) {
        // row r of the tile -> 128-byte row r of the staging tile, 16-byte
        // unit u at position u ^ (r % 8) (the 128-byte swizzle of the map)
        const uint32_t ost = sstream + Cfg::OFF_OST;
        const uint32_t r = (uint32_t)(wq * 32 + lane);
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t rr[32];
          if (nt > 0) {
            ptx::tmem_ld32(o_taddr + 32 * c, rr);
            ptx::tmem_wait_ld_dep(rr);
          }
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 16; ++e)
            w[e] = nt > 0 ? ptx::pack_bf16x2(__uint_as_float(rr[2 * e]) * inv, __uint_as_float(rr[2 * e + 1]) * inv)
                          : 0u;
          const uint32_t rbase = ost + (uint32_t)(c / 2) * (uint32_t)(BM * 128) + r * 128u;
#pragma unroll
          for (int e = 0; e < 4; ++e)
            ptx::st_shared_v4(rbase + ((((uint32_t)(c & 1) * 4u + (uint32_t)e) ^ (r & 7u)) << 4), w[4 * e],
                              w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
        if (nt > 0) {  // O of this tile is read out: the next item may overwrite it
          ptx::tc_fence_before();
          ptx::mbar_arrive(bar(Cfg::B_OFREE + t));
        }
        ptx::fence_proxy_async_smem();
        ptx::bar_sync(1u + (uint32_t)s, 128u);
        if (wq == 0 && lane == 0) {
          // rows at or past Nq fall outside the map and are not written
#pragma unroll
          for (int cb = 0; cb < Cfg::NCH; ++cb)
            ptx::tma_store_4d(&tmO, ost + (uint32_t)cb * (uint32_t)(BM * 128), cb * 64, ie.h, row0, ie.b);
          ptx::bulk_commit();
        }
      } else {
        __nv_bfloat16* orow = reinterpret_cast<__nv_bfloat16*>(p.o) +
                              (((long long)ie.b * p.Nq + row) * p.Hq + ie.h) * (long long)D;
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
        if (nt > 0) {  // O of this tile is read out: the next item may overwrite it
          ptx::tc_fence_before();
          ptx::mbar_arrive(bar(Cfg::B_OFREE + t));
        }
      }
      if (store && p.lse != nullptr) {
        const float lse = l > 0.f ? (m_ref + log2f(l)) * 0.6931471805599453f : -INFINITY;
        p.lse[((long long)ie.b * p.Hq + ie.h) * p.Nq + row] = lse;
      }
    }
    // the staging tile's last store must be complete before the block exits
    if constexpr (Cfg::OST)
      if (wq == 0 && lane == 0) ptx::bulk_wait0();
  } else if (is_tma) {
    // ------------------------------------------------------------ producer
    constexpr int kProducerRole = Cfg::NS > 1 ? kRoleProducerBackoff : kRoleProducer;
    if constexpr (Cfg::SPLIT_REGS) ptx::setmaxnreg_dec<Cfg::REG_CONTROL>();
    if (lane == 0) {
      int k_issued[KST], v_issued[VST], q_issued[NQT];
#pragma unroll
      for (int s = 0; s < KST; ++s) k_issued[s] = 0;
#pragma unroll
      for (int s = 0; s < VST; ++s) v_issued[s] = 0;
#pragma unroll
      for (int t = 0; t < NQT; ++t) q_issued[t] = 0;
      int kc = 0, vc = 0;  // loads issued into the K and V rings
      bool ok = true;
      for (int k = 0; ok; ++k) {
        const int item = item_at(k, G, T, c);
        if (item < 0) break;
        const Item it = decode_item(item, p);
        int n_kv[NQT];
        const int nmax = plan(it, n_kv);
        const int kh = it.h / p.group;
        const int q0 = it.qb * BM * NQT;
        auto load_kv = [&](int j, bool do_k = true, bool do_v = true) -> bool {
          const int ks = kc % KST;
          if (do_k) {
            if (kc >= KST &&
                !wait_bar<kProducerRole>(bar(Cfg::B_KEMPTY + ks), (uint32_t)(((kc / KST) - 1) & 1), wc, kSiteKEmpty))
              return false;
            const uint32_t fb = bar(Cfg::B_KFULL + ks);
            ptx::mbar_arrive_expect_tx(fb, Cfg::KV_BYTES);
#pragma unroll
            for (int c = 0; c < Cfg::NCH; ++c)
              ptx::tma_load_4d(sstream + Cfg::OFF_K + ks * Cfg::KV_BYTES + c * Cfg::CH_KV, &tmK, fb, c * Cfg::BOXE, kh,
                               j * BN, it.b);
            ++k_issued[ks];
            ++kc;
          }
          if (!do_v) return true;
          const int vs = vc % VST;
          if (vc >= VST &&
              !wait_bar<kProducerRole>(bar(Cfg::B_VEMPTY + vs), (uint32_t)(((vc / VST) - 1) & 1), wc, kSiteVEmpty))
            return false;
          {
            const uint32_t fb = bar(Cfg::B_VFULL + vs);
            ptx::mbar_arrive_expect_tx(fb, Cfg::KV_BYTES);
#pragma unroll
            for (int c = 0; c < Cfg::NCH; ++c)
              ptx::tma_load_4d(sstream + Cfg::OFF_V + vs * Cfg::KV_BYTES + c * Cfg::CH_KV, &tmV, fb, c * Cfg::BOXE, kh,
                               j * BN, it.b);
            ++v_issued[vs];
            ++vc;
          }
          return true;
        };
        auto load_q = [&]() {
#pragma unroll
          for (int t = 0; t < NQT; ++t) {
            if (n_kv[t] == 0) continue;
            const uint32_t fb = bar(Cfg::B_QFULL + t);
            ptx::mbar_arrive_expect_tx(fb, Cfg::QT_BYTES);
#pragma unroll
            for (int c = 0; c < Cfg::NCH; ++c)
              ptx::tma_load_4d(sstream + Cfg::OFF_Q + t * Cfg::QT_BYTES + c * Cfg::CH_Q, &tmQ, fb, c * Cfg::BOXE,
                               it.h, q0 + t * BM, it.b);
            ++q_issued[t];
          }
        };
        if (k == 0) {
          // At launch every block loads at once and the copies share the
          // memory bandwidth: the first Q K^T needs only Q and K_0, so the
          // other tiles go out once those two have landed.
          load_q();
          if (nmax > 0 && !load_kv(0, true, false)) break;
#pragma unroll
          for (int t = 0; t < NQT && ok; ++t)
            if (n_kv[t] > 0) ok = wait_bar<kProducerRole>(bar(Cfg::B_QFULL + t), 0u, wc, kSiteQ);
          if (ok && nmax > 0) ok = wait_bar<kProducerRole>(bar(Cfg::B_KFULL), 0u, wc, kSiteKFull);
          if (!ok) break;
          if (nmax > 0 && !load_kv(0, false, true)) break;
        } else {
          // the first key/value tile goes out before waiting for Q smem, so
          // it is in flight while the previous item finishes
          if (nmax > 0 && !load_kv(0)) break;
          // Q smem is free once the previous item's last Q K^T has completed
          if (!wait_bar<kProducerRole>(bar(Cfg::B_QEMPTY), (uint32_t)((k - 1) & 1), wc, kSiteQ)) break;
          load_q();
        }
        for (int j = 1; j < nmax; ++j)
          if (!load_kv(j)) {
            ok = false;
            break;
          }
      }
      // Every issued copy must land before the block may exit (no-op in the
      // normal path, where the consumers have already seen them all).
#pragma unroll
      for (int t = 0; t < NQT; ++t)
        if (q_issued[t] > 0)
          wait_bar_drain<kProducerRole>(bar(Cfg::B_QFULL + t), (uint32_t)((q_issued[t] - 1) & 1), wc, kSiteQ);
#pragma unroll
      for (int s = 0; s < KST; ++s)
        if (k_issued[s] > 0)
          wait_bar_drain<kProducerRole>(bar(Cfg::B_KFULL + s), (uint32_t)((k_issued[s] - 1) & 1), wc, kSiteKFull);
#pragma unroll
      for (int s = 0; s < VST; ++s)
        if (v_issued[s] > 0)
          wait_bar_drain<kProducerRole>(bar(Cfg::B_VFULL + s), (uint32_t)((v_issued[s] - 1) & 1), wc, kSiteVFull);
    }
  } else {
    if constexpr (Cfg::SPLIT_REGS) ptx::setmaxnreg_dec<Cfg::REG_CONTROL>();
  }
  if (is_mma) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs this loop (waits, counters, descriptors); one
    // elected lane issues the tcgen05 instructions.
    {
      bool ok = true;
      const uint32_t q_s = sstream + Cfg::OFF_Q, k_s = sstream + Cfg::OFF_K, v_s = sstream + Cfg::OFF_V;
      int kc = 0, vc = 0;                  // K / V ring slots consumed
      int scount[NQT], pcount[NQT], qcount[NQT], ouse[NQT];
#pragma unroll
      for (int t = 0; t < NQT; ++t) scount[t] = pcount[t] = qcount[t] = ouse[t] = 0;
      auto issue_qk = [&](int t, int kslot) -> bool {
        const int buf = scount[t] % SB;
        if constexpr (Cfg::PSEP) {
          // the softmax must have read the previous S of this buffer
          if (scount[t] > 0 && !wait_bar_warp<kRoleMma>(bar(Cfg::B_SFREE + t * SB + buf),
                                                        (uint32_t)((scount[t] - 1) & 1), wc, kSiteSFull))
            return false;
          ptx::tc_fence_after();
        }
        const uint32_t d_t = tmem_s + (uint32_t)((t * SB + buf) * BN);
        // descriptors advance by 32 bytes (>> 4 = 2) per K step inside a
        // 128-byte chunk and by one chunk (CH_Q / CH_KV bytes) after four
        const uint64_t ad0 = ptx::sdesc_sw128(q_s + t * Cfg::QT_BYTES, 16u, 1024u);
        const uint64_t bd0 = ptx::sdesc_sw128(k_s + kslot * Cfg::KV_BYTES, 16u, 1024u);
#pragma unroll
        for (int kk = 0; kk < Cfg::QK_STEPS; ++kk) {
          const uint32_t ch = (uint32_t)kk / 4u, in = (uint32_t)kk % 4u;
          const uint64_t ad = ad0 + (uint64_t)((ch * Cfg::CH_Q + in * 32u) >> 4);
          const uint64_t bd = bd0 + (uint64_t)((ch * Cfg::CH_KV + in * 32u) >> 4);
          ptx::warp_mma_ss<Cfg::FP8>(d_t, ad, bd, Cfg::IDESC_QK, kk > 0 ? 1u : 0u);
        }
        ptx::warp_commit(bar(Cfg::B_SFULL + t * SB + buf));
        ++scount[t];
        return true;
      };
      // P V of key tile jj of the current item; jj == 0 starts a new output
      auto issue_pv = [&](int t, int jj, int vslot, bool last) -> bool {
        if (jj == 0) {
          // the previous item's output of this tile must have been read out
          if (ouse[t] > 0 &&
              !wait_bar_warp<kRoleMma>(bar(Cfg::B_OFREE + t), (uint32_t)((ouse[t] - 1) & 1), wc, kSiteODone))
            return false;
          ++ouse[t];
        }
        const int buf = pcount[t] % SB;
        const int si = t * SB + buf;
        const uint32_t ph = (uint32_t)((pcount[t] / SB) & 1);
        const uint32_t d_t = tmem_s + (uint32_t)(Cfg::O_COL0 + t * D);
        const uint32_t a_t = tmem_s + (uint32_t)(Cfg::PSEP ? Cfg::P_COL0 + t * Cfg::P_COLS : si * BN);
        const uint64_t bd0 = ptx::sdesc_sw128(v_s + vslot * Cfg::KV_BYTES, Cfg::CH_KV, 1024u);
        // the first half of the keys as soon as their P is written, the rest
        // when the whole P is
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          if (!wait_bar_warp<kRoleMma>(bar((half == 0 ? Cfg::B_PHALF : Cfg::B_PFULL) + si), ph, wc, kSitePFull))
            return false;
          ptx::tc_fence_after();
#pragma unroll
          for (int kk = half * Cfg::PV_STEPS / 2; kk < (half + 1) * Cfg::PV_STEPS / 2; ++kk) {
            const uint64_t bd = bd0 + (uint64_t)(((uint32_t)kk * Cfg::KSTEP * 128u) >> 4);
            ptx::warp_mma_ts<Cfg::FP8>(d_t, a_t + (uint32_t)kk * 8u, bd, Cfg::IDESC_PV, (jj > 0 || kk > 0) ? 1u : 0u);
          }
        }
        ptx::warp_commit(bar(Cfg::B_ODONE + t));
        if (last) ptx::warp_commit(bar(Cfg::B_OFINAL + t));
        ++pcount[t];
        return true;
      };
      for (int k = 0; ok; ++k) {
        const int item = item_at(k, G, T, c);
        if (item < 0) break;
        const Item it = decode_item(item, p);
        int n_kv[NQT];
        const int nmax = plan(it, n_kv);
#pragma unroll
        for (int t = 0; t < NQT && ok; ++t)
          if (n_kv[t] > 0) {
            ok = wait_bar_warp<kRoleMma>(bar(Cfg::B_QFULL + t), (uint32_t)(qcount[t] & 1), wc, kSiteQ);
            ++qcount[t];
          }
        if (!ok) break;
        ptx::tc_fence_after();
        for (int j = 0; ok && j <= nmax; ++j) {
          const bool has_k = j < nmax, has_v = j >= 1;
          const int ks = kc % KST, vs = vc % VST;
          if constexpr (SB == 2) {
            // S is double-buffered: the products for key tile j go first, so
            // they run under the softmax of key tile j-1; then the P V of
            // key tile j-1 as each tile's P is released
            if (has_k) {
              ok = wait_bar_warp<kRoleMma>(bar(Cfg::B_KFULL + ks), (uint32_t)((kc / KST) & 1), wc, kSiteKFull);
              if (!ok) break;
              ptx::tc_fence_after();
#pragma unroll
              for (int t = 0; t < NQT; ++t)
                if (j < n_kv[t]) issue_qk(t, ks);  // no wait inside: SB == 2 excludes PSEP
              ptx::warp_commit(bar(Cfg::B_KEMPTY + ks));
              ++kc;
            }
            if (has_v) {
              ok = wait_bar_warp<kRoleMma>(bar(Cfg::B_VFULL + vs), (uint32_t)((vc / VST) & 1), wc, kSiteVFull);
              if (!ok) break;
              ptx::tc_fence_after();
#pragma unroll
              for (int t = 0; t < NQT && ok; ++t)
                if (j - 1 < n_kv[t]) ok = issue_pv(t, j - 1, vs, j == n_kv[t]);
              if (!ok) break;
              ptx::warp_commit(bar(Cfg::B_VEMPTY + vs));
              ++vc;
            }
          } else {
            // P overwrites S in place: PV(t, j-1) must be issued before
            // QK(t, j) reuses the buffer.  With a separate P buffer the order
            // turns round: QK(t, j) needs only S(t, j-1) read out, which the
            // softmax signals early, and PV(t, j-1) waits for the whole P.
            if (has_k) {
              ok = wait_bar_warp<kRoleMma>(bar(Cfg::B_KFULL + ks), (uint32_t)((kc / KST) & 1), wc, kSiteKFull);
              if (!ok) break;
            }
            if (has_v) {
              ok = wait_bar_warp<kRoleMma>(bar(Cfg::B_VFULL + vs), (uint32_t)((vc / VST) & 1), wc, kSiteVFull);
              if (!ok) break;
            }
            ptx::tc_fence_after();
#pragma unroll
            for (int t = 0; t < NQT && ok; ++t) {
              if constexpr (Cfg::PSEP) {
                if (has_k && j < n_kv[t]) ok = issue_qk(t, ks);
                if (ok && has_v && j - 1 < n_kv[t]) ok = issue_pv(t, j - 1, vs, j == n_kv[t]);
              } else {
                if (has_v && j - 1 < n_kv[t]) ok = issue_pv(t, j - 1, vs, j == n_kv[t]);
                if (ok && has_k && j < n_kv[t]) ok = issue_qk(t, ks);
              }
            }
            if (!ok) break;
            if (has_k) {
              ptx::warp_commit(bar(Cfg::B_KEMPTY + ks));
              ++kc;
            }
            if (has_v) {
              ptx::warp_commit(bar(Cfg::B_VEMPTY + vs));
              ++vc;
            }
          }
          // after the item's last Q K^T: Q smem is free once it completes,
          // so the next item's Q can load under this item's last P V
          if (j == nmax - 1) ptx::warp_commit(bar(Cfg::B_QEMPTY));
        }
        if (nmax == 0) ptx::warp_commit(bar(Cfg::B_QEMPTY));
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
