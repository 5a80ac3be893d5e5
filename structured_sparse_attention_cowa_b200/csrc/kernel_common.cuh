// kernel_common.cuh -- small device helpers shared by the attention kernels: the list of
// KV tiles a query tile visits (from the planner in cowa_pattern.h) and a cursor over it.
#pragma once

#include "cowa_pattern.h"

namespace cowa {

constexpr int kTile = 128;  // query and key tile edge (BM = BN = 128)

struct Tiles {
  Range r[3];
  int n;      // number of disjoint tile-index ranges
  int count;  // number of tiles
};

__device__ __forceinline__ Tiles plan_tiles(const Pat& p, Range iv, int t0, int t1) {
  Tiles T;
  T.n = fwd_tile_ranges(p, iv, t0, t1, kTile, T.r);
  T.count = 0;
  for (int x = 0; x < T.n; ++x) T.count += T.r[x].hi - T.r[x].lo;
  return T;
}

// Walks the tile list in order.
struct TileCursor {
  int x, j;
  __device__ __forceinline__ void init(const Tiles& T) { x = 0; j = T.n > 0 ? T.r[0].lo : 0; }
  __device__ __forceinline__ void next(const Tiles& T) {
    if (++j >= T.r[x].hi && x + 1 < T.n) { ++x; j = T.r[x].lo; }
  }
};

// Packed variable-length batches.  A sequence table in device memory, written by the
// seq_table kernel (launch_seq_table) from the caller's cu_seqlens, n = number of sequences:
//   tab[0 .. n]          tiles of 128 rows before sequence s (tab[n]: all tiles)
//   tab[n+1 .. 2n]       first row of sequence s on the packed token axis
//   tab[2n+1 .. 3n]      length of sequence s
// The offsets are clamped so that the sequences lie in order, disjoint, inside [0, total):
// start = clamp(cu[s], end of s-1, total), end = clamp(cu[s+1], start, total).
__device__ __forceinline__ int seq_of_tile(const int32_t* tab, int n, int tg) {
  int lo = 0, hi = n - 1;  // largest s with tab[s] <= tg (empty sequences share their offset)
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tab[mid] <= tg) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ uint8_t* align1024(uint8_t* p) {
  return reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(p) + 1023) & ~uintptr_t(1023));
}

}  // namespace cowa
