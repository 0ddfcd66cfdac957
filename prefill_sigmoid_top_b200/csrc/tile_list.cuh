// Tile lists of the persistent grouped kernels (single-SM, 2-SM pair, NVFP4).
//
// A tile = (expert e, weight tile w, token tile t).  Tiles are numbered expert
// by expert; expert e owns W x ceil(count[e] / kNmax) of them, ordered w, then
// t (fastest), so tiles that stream the same weight panel are neighbours and
// run at about the same time (the panel comes from HBM once).  Each CTA (or
// pair) takes the tiles of a static round-robin list over that numbering.
#pragma once

namespace moe {

struct TileCoord {
  int e, w, t;
};

// Warp 0 writes prefix[e] = first tile of expert e and prefix[E] = the tile
// count, from the per-expert counts in shared memory.  Called by one warp.
template <int kNmax>
__device__ __forceinline__ void build_tile_prefix(const int* cnt, int* prefix, int E, int W, int lane) {
  const int per = (E + 31) / 32;
  const int lo = min(E, lane * per), hi = min(E, lo + per);
  int sum = 0;
  for (int e = lo; e < hi; ++e) sum += W * ((cnt[e] + kNmax - 1) / kNmax);
  int incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int v = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += v;
  }
  int run = incl - sum;
  for (int e = lo; e < hi; ++e) {
    prefix[e] = run;
    run += W * ((cnt[e] + kNmax - 1) / kNmax);
  }
  if (lane == 31) prefix[E] = incl;
}

// Tile index -> (expert, weight tile, token tile): the largest e with prefix[e] <= idx.
template <int kNmax>
__device__ __forceinline__ TileCoord decode_tile(const int* prefix, const int* cnt, int E, int idx) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (prefix[mid] <= idx) lo = mid; else hi = mid - 1;
  }
  const int ntiles = (cnt[lo] + kNmax - 1) / kNmax;
  const int rel = idx - prefix[lo];
  return TileCoord{lo, rel / ntiles, rel % ntiles};
}

// ids[i] for a run-time i without indexing a register array.
template <int kN>
__device__ __forceinline__ int pick(const int (&ids)[kN], int i) {
  int v = ids[0];
#pragma unroll
  for (int j = 1; j < kN; ++j) v = (i == j) ? ids[j] : v;
  return v;
}

}  // namespace moe
