// tiles.h -- which key tiles a query tile must visit, and which need a mask.
//
// Bottom-right causal alignment: query row i sees key j iff
// j < Nk and (!causal || j <= i + (Nk - Nq)).  The visible keys of every row
// form a prefix [0, vis_end(i)), with vis_end non-decreasing in i, so for the
// rows [row0, row1) of a query tile:
//   * the visited key tiles are a prefix, ending at the tile that holds
//     vis_end(row1 - 1) - 1;
//   * a key tile is "full" (no element masked for any row of the tile) iff its
//     last key is visible to the tile's first row row0;
//   * a key tile is skipped iff even the tile's last row sees none of its keys.
// Page "FlashAttention (SV)", section "Sammanslagning av operationer till en
// enda CUDA-kärna", puts the masking inside the fused kernel; skipping fully
// masked tiles is what makes the causal pass cost half the FLOPs.
#pragma once

#ifdef __CUDACC__
#define ATTN_HD __host__ __device__ __forceinline__
#else
#define ATTN_HD inline
#endif

namespace attn {

enum TileKind : int { kTileSkip = 0, kTileFull = 1, kTilePartial = 2 };

// Key windows (split-KV): a launch may see only the keys [kv0, kv0 + Nk) of a
// longer range of Nk + kv0 + shift keys, with `shift` keys after the window.
// In window-local indices the causal rule becomes j <= i + (Nk - Nq) + shift;
// shift = 0 is the whole range.

// Exclusive end of the visible key range of query row i (clamped to [0, Nk]).
ATTN_HD long long vis_end(long long i, long long Nq, long long Nk, bool causal, long long shift = 0) {
  if (!causal) return Nk;
  long long e = i + (Nk - Nq) + shift + 1;
  return e < 0 ? 0 : (e > Nk ? Nk : e);
}

// Number of leading key tiles (of bn keys) that the query rows [row0, row1)
// must visit; row1 is clipped to Nq.  0 when the rows see no key.
ATTN_HD int kv_tile_count(int row0, int row1, int Nq, int Nk, int bn, bool causal, int shift = 0) {
  if (row1 > Nq) row1 = Nq;
  if (row0 >= row1 || Nk <= 0) return 0;
  const long long e = vis_end(row1 - 1, Nq, Nk, causal, shift);
  return (int)((e + bn - 1) / bn);
}

ATTN_HD int tile_kind(int row0, int row1, int kt, int Nq, int Nk, int bn, bool causal, int shift = 0) {
  if (row1 > Nq) row1 = Nq;
  if (row0 >= row1 || kt < 0) return kTileSkip;
  const long long k0 = (long long)kt * bn, k1 = k0 + bn;  // keys [k0, k1)
  if (k0 >= vis_end(row1 - 1, Nq, Nk, causal, shift)) return kTileSkip;
  if (k1 <= vis_end(row0, Nq, Nk, causal, shift)) return kTileFull;
  return kTilePartial;
}

}  // namespace attn
