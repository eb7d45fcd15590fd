// attn_common.cuh -- pieces shared by the two forward kernels: launch
// parameters, the tile/warp/memory configuration, and the bounded mbarrier
// wait that turns a stalled pipeline into an error status instead of a hang.
#pragma once
#include <cuda.h>
#include <cstdint>

#include "ptx.cuh"

namespace attn {

struct FwdParams {
  void* o;          // [B, Nq, Hq, D] bf16
  float* lse;       // [B, Hq, Nq] fp32 or nullptr
  int B, Hq, Hkv, Nq, Nk;
  int group;        // Hq / Hkv
  // the part of the problem this launch computes: batches [b0, b0 + nb) and
  // query heads [h0, h0 + nh) (whole key/value groups); the tensors above are
  // the full [B, N, H, d] ones
  int b0, nb, h0, nh;
  int n_qblocks;    // ceil(Nq / (128 * NQT))
  int n_items;      // nb * nh * n_qblocks work items
  int qb_major;     // 1: order items by query block (longest first) across heads; 0: head-major
  // one-block-per-item kernel: band > 0 runs a 1-D grid in which the
  // (batch, head) pairs are cut into bands of `band` pairs, bands one after
  // another, and within a band the items go longest query block first across
  // its pairs; 0: grid (query block, head, batch x window)
  int band;
  float sl2;        // scale * log2(e)
  // split-KV (one-block-per-item kernel): the keys are cut into n_splits
  // windows of kv_chunk keys (a multiple of the key tile); window s of batch b
  // runs as grid z = b * n_splits + s and writes fp32 partials, O_s =
  // o_part[s][b][row][h][:] (normalised by its own row sum) and LSE_s =
  // lse_part[s][b][h][row].  n_splits = 1, kv_chunk = Nk, o_part = nullptr:
  // no split, bf16 O written to o.
  int n_splits, kv_chunk;
  float* o_part;
  float* lse_part;
  // head packing (one-block-per-item kernel): pack = g > 1 stacks the g query
  // heads of a key/value head in one query tile, packed row r = i * g + (h %
  // g) (query row i); grid y is then the key/value head, n_qblocks counts
  // tiles of packed rows, and Q is read through a 5-D map (d, g, Hkv, Nq, B).
  // pack = 1: grid y is the query head.
  int pack;
  const float* dq;  // FP8 descales (device scalars), nullptr for bf16
  const float* dk;
  const float* dv;
  unsigned int* err;            // device error word
  unsigned long long timeout_ns;
};

constexpr float kTau = 8.0f;  // lazy-rescale threshold, log2 units

// Maximum of sl2 * s[c] over the visible columns c < nvis of N scores (the
// keys of a partially masked tile form a prefix); -inf when none is visible.
// Four independent chains of three-input max on the raw scores, one multiply
// at the end (sl2 >= 0 keeps the order; a negative scale takes the minimum).
template <int N>
__device__ __forceinline__ float masked_max_scaled(const uint32_t* sr, int nvis, float sl2) {
  if (sl2 >= 0.f) {
    float a[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int c = 0; c < N; c += 2) {
      const float x0 = c < nvis ? __uint_as_float(sr[c]) : -INFINITY;
      const float x1 = c + 1 < nvis ? __uint_as_float(sr[c + 1]) : -INFINITY;
      a[(c / 2) % 4] = ptx::fmax3(a[(c / 2) % 4], x0, x1);
    }
    const float m = fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3]));
    return m == -INFINITY ? -INFINITY : m * sl2;
  }
  float a[4] = {INFINITY, INFINITY, INFINITY, INFINITY};
#pragma unroll
  for (int c = 0; c < N; c += 2) {
    const float x0 = c < nvis ? __uint_as_float(sr[c]) : INFINITY;
    const float x1 = c + 1 < nvis ? __uint_as_float(sr[c + 1]) : INFINITY;
    a[(c / 2) % 4] = fminf(a[(c / 2) % 4], fminf(x0, x1));
  }
  const float m = fminf(fminf(a[0], a[1]), fminf(a[2], a[3]));
  return m == INFINITY ? -INFINITY : m * sl2;
}

template <int D_, int BN_, int NQT_, int KST_, int VST_, bool CAUSAL_, bool FP8_, int EMU_ = 0,
          int SB_ = (NQT_ == 1 ? 2 : 1), bool PSEP_ = false, int NS_ = 1, bool PACK_ = false, bool OST_ = false>
struct FwdCfg {
  // PACK: the one-block-per-item kernel reads the head-packing factor from the
  // launch parameters (split-KV); otherwise it is compiled out
  static constexpr bool PACK = PACK_;
  static constexpr int D = D_, BN = BN_, NQT = NQT_, KST = KST_, VST = VST_;
  // NS: independent streams per block (persistent kernel): each has its own
  // softmax warpgroup(s), TMA and MMA warps, K/V rings, barriers and tensor
  // memory columns, and takes its own work items
  static constexpr int NS = NS_;
  static_assert(NS == 1 || (NS == 2 && NQT == 1), "two streams of one query tile each");
  // PSEP: P gets tensor-memory columns of its own instead of overwriting S,
  // so Q K_{j+1}^T can be computed while the softmax of tile j still runs
  // (persistent kernel only; needs a single score buffer per query tile)
  static constexpr bool PSEP = PSEP_;
  // software exp2 share on full tiles: element pairs with (pair % 8) < EMU
  static constexpr int EMU = EMU_;
  static constexpr bool CAUSAL = CAUSAL_, FP8 = FP8_;
  static constexpr int BM = 128;
  // OST (persistent kernel, bf16): each stream stages its output tile in
  // shared memory (the 128-byte-swizzled layout of a Q tile) and writes it
  // with one TMA store, instead of one row per thread
  static constexpr bool OST = OST_;
  static_assert(!OST || (!FP8 && NQT == 1), "staged output: bf16, one query tile per stream");
  static constexpr int SB = SB_;  // score buffers per query tile
  static_assert(SB == 1 || SB == 2, "one or two score buffers");
  static constexpr int ELEM = FP8 ? 1 : 2;
  static constexpr int NCH = D * ELEM / 128;  // 128-byte column chunks per row
  static constexpr int BOXE = 128 / ELEM;     // elements per chunk row
  static constexpr uint32_t CH_Q = BM * 128;  // bytes of one chunk of a Q tile
  static constexpr uint32_t CH_KV = BN * 128;
  static constexpr uint32_t QT_BYTES = CH_Q * NCH;
  static constexpr uint32_t KV_BYTES = CH_KV * NCH;
  static constexpr int KSTEP = FP8 ? 32 : 16;  // reduction depth of one MMA
  static constexpr int QK_STEPS = D / KSTEP;
  static constexpr int PV_STEPS = BN / KSTEP;
  static constexpr int P_COLS = BN * ELEM / 4;
  static constexpr int P_COL0 = NQT * SB * BN;  // P of tile t at P_COL0 + t * P_COLS (PSEP only)
  static constexpr int O_COL0 = NQT * SB * BN + (PSEP ? NQT * P_COLS : 0);
  static_assert(!PSEP || SB == 1, "separate P with one score buffer");
  static constexpr int TMEM_USED = O_COL0 + NQT * D;  // columns of one stream
  static constexpr int TMEM_ALL = NS * TMEM_USED;
  static constexpr int TMEM_COLS = TMEM_ALL <= 128 ? 128 : (TMEM_ALL <= 256 ? 256 : 512);
  static_assert(TMEM_ALL <= 512, "tensor memory has 512 columns");
  static_assert(D % 64 == 0 && NCH >= 1, "head size");
  static_assert(BN % 32 == 0 && BN <= 256, "key tile");
  // barriers
  static constexpr int B_QFULL = 0;
  static constexpr int B_KFULL = B_QFULL + NQT;
  static constexpr int B_KEMPTY = B_KFULL + KST;
  static constexpr int B_VFULL = B_KEMPTY + KST;
  static constexpr int B_VEMPTY = B_VFULL + VST;
  static constexpr int B_SFULL = B_VEMPTY + VST;
  static constexpr int B_PFULL = B_SFULL + NQT * SB;
  static constexpr int B_PHALF = B_PFULL + NQT * SB;  // first half of P written
  static constexpr int B_ODONE = B_PHALF + NQT * SB;
  static constexpr int B_OFINAL = B_ODONE + NQT;
  static constexpr int B_OFREE = B_OFINAL + NQT;
  static constexpr int B_QEMPTY = B_OFREE + NQT;
  static constexpr int B_SFREE = B_QEMPTY + 1;  // S read out of tensor memory (PSEP)
  static constexpr int B_DRAIN = B_SFREE + NQT * SB;
  static constexpr int NBAR = B_DRAIN + 1;
  // shared memory (offsets from a 1024-byte aligned base; stream s adds
  // s * STREAM_BYTES to the tile offsets and s * NBAR to barrier indices)
  static constexpr uint32_t OFF_Q = 0;
  static constexpr uint32_t OFF_K = OFF_Q + NQT * QT_BYTES;
  static constexpr uint32_t OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr uint32_t OFF_OST = OFF_V + VST * KV_BYTES;  // output staging tile (OST)
  static constexpr uint32_t STREAM_BYTES = OFF_OST + (OST ? (uint32_t)BM * D * 2 : 0u);
  static constexpr uint32_t OFF_BAR = NS * STREAM_BYTES;
  static constexpr uint32_t OFF_SLOT = OFF_BAR + NS * NBAR * 8;
  static constexpr uint32_t OFF_ABORT = OFF_SLOT + 4;
  static constexpr uint32_t SMEM_BYTES = OFF_ABORT + 4 + 1024;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory per block");
  // warps: softmax warpgroups (stream s owns warps 4*NQT*s ..), then one
  // warpgroup holding the TMA and MMA warps of each stream (TMA warp of stream
  // s = SM_WARPS + 2s, its MMA warp the next one) and, with one stream, two
  // idle warps (a whole warpgroup, so that registers can be moved to the
  // softmax warpgroups with setmaxnreg)
  static constexpr int SM_WARPS = 4 * NQT * NS;
  static constexpr int TMA_WARP = SM_WARPS;
  static constexpr int MMA_WARP = SM_WARPS + 1;
  static constexpr int NTHREADS = 32 * (SM_WARPS + 4);
  // register split (two softmax warpgroups: 384 threads launch with 168
  // registers each = 64512; the softmax warpgroups get 200, the control
  // warpgroup 104: 2*128*200 + 128*104 = 64512)
  static constexpr int REG_LAUNCH = 65536 / NTHREADS >= 255 ? 255 : (65536 / NTHREADS) / 8 * 8;
  static constexpr bool SPLIT_REGS = NQT * NS == 2;
  static constexpr int REG_SOFTMAX = 200, REG_CONTROL = 104;
  static_assert(!SPLIT_REGS || 2 * 128 * REG_SOFTMAX + 128 * REG_CONTROL <= NTHREADS * REG_LAUNCH,
                "register split exceeds the launch allocation");
  static constexpr uint32_t IDESC_QK = ptx::idesc<FP8>(128, BN, false);
  static constexpr uint32_t IDESC_PV = ptx::idesc<FP8>(128, D, true);
};

// Wait sites recorded in the device error word.
enum : uint32_t {
  kSiteQ = 1, kSiteKFull, kSiteVFull, kSiteKEmpty, kSiteVEmpty, kSiteSFull, kSitePFull,
  kSiteODone, kSiteDrain, kSiteProbe
};

struct WaitCtx {
  volatile uint32_t* abort;
  unsigned int* err;
  unsigned long long timeout_ns;
};

// Warp roles, for the per-role instantiation of the polling loop.  A producer
// that shares its scheduler with busy softmax warps (two streams per block)
// polls with a short sleep between rounds (kRoleProducerBackoff): it runs
// stages ahead, so the added wake-up latency costs nothing, and the issue
// slots go to the softmax warps.
enum : int { kRoleSoftmax = 0, kRoleProducer = 1, kRoleMma = 2, kRoleProducerBackoff = 3 };

// Bounded mbarrier wait: true when the phase with `parity` has completed;
// false after the time limit (recording the site in the error word and
// raising the block's abort flag) or when another role already aborted.
// The first probe is inline; only a wait that does not succeed at once pays
// for the call into the polling loop.  The polling loop is instantiated once
// per warp role (ROLE), because roles run under different register budgets
// (setmaxnreg) and a called function is compiled for one budget.
template <int ROLE>
__device__ __noinline__ bool wait_bar_slow(uint32_t bar, uint32_t parity, const WaitCtx& c, uint32_t site) {
  const uint64_t t0 = ptx::globaltimer();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 16; ++i)
      if (ptx::mbar_try_wait(bar, parity)) return true;
    if (*c.abort) return false;
    if constexpr (ROLE == kRoleProducerBackoff) __nanosleep(64);
    if (ptx::globaltimer() - t0 > c.timeout_ns) {
      *c.abort = 1u;
      const uint32_t blk = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
      atomicOr(c.err, 1u | (site << 8) | ((blk & 0xFFFFu) << 16));
      return false;
    }
  }
}
template <int ROLE = 0>
__device__ __forceinline__ bool wait_bar(uint32_t bar, uint32_t parity, const WaitCtx& c, uint32_t site) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  return wait_bar_slow<ROLE>(bar, parity, c, site);
}

// Drain wait of a producer before its block exits: a TMA copy that was issued
// lands whether or not anything consumes it, so this wait ignores the block's
// abort flag (the block must not free its shared memory under a copy in
// flight) and ends only when the phase completes or the time limit passes.
template <int ROLE>
__device__ __noinline__ bool wait_bar_drain(uint32_t bar, uint32_t parity, const WaitCtx& c, uint32_t site) {
  if (ptx::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = ptx::globaltimer();
  for (;;) {
#pragma unroll 1
    for (int i = 0; i < 16; ++i)
      if (ptx::mbar_try_wait(bar, parity)) return true;
    if constexpr (ROLE == kRoleProducerBackoff) __nanosleep(64);
    if (ptx::globaltimer() - t0 > c.timeout_ns) {
      *c.abort = 1u;
      const uint32_t blk = blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z);
      atomicOr(c.err, 1u | (site << 8) | ((blk & 0xFFFFu) << 16));
      return false;
    }
  }
}

// Wait by a whole warp (every lane polls the same barrier); the result is made
// warp-uniform so that the warp stays converged on the error path too.
template <int ROLE>
__device__ __forceinline__ bool wait_bar_warp(uint32_t bar, uint32_t parity, const WaitCtx& c, uint32_t site) {
  return __all_sync(0xffffffffu, wait_bar<ROLE>(bar, parity, c, site));
}

}  // namespace attn
