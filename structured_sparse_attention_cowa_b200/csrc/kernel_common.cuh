// kernel_common.cuh -- small device helpers shared by the attention kernels: the list of
// KV tiles a query tile visits (from the planner in cowa_pattern.h) and a cursor over it.
#pragma once

#include "cowa_pattern.h"

namespace cowa {

constexpr int kTile = 128;  // query and key tile edge (BM = BN = 128)

struct Tiles {
  Range r[3];  // disjoint tile-index ranges r[0..n); the rest are empty sentinels
  int n;       // number of ranges
  int count;   // number of tiles
};

__device__ __forceinline__ Tiles plan_tiles(const Pat& p, Range iv, int t0, int t1) {
  Tiles T;
  T.n = fwd_tile_ranges(p, iv, t0, t1, kTile, T.r);
  // fixed indices only (the sentinels [INT_MAX, INT_MAX) count 0), so T stays in registers
  T.count = (T.r[0].hi - T.r[0].lo) + (T.r[1].hi - T.r[1].lo) + (T.r[2].hi - T.r[2].lo);
  return T;
}

// Walks the tile list in order, in registers: the current tile, the end of its range and the
// ranges still to come (no array indexed at run time, which would live in local memory).
struct TileCursor {
  int j, hi, lo1, hi1, lo2, hi2;
  __device__ __forceinline__ void init(const Tiles& T) {
    j = T.n > 0 ? T.r[0].lo : 0;
    hi = T.n > 0 ? T.r[0].hi : 0;
    lo1 = T.r[1].lo; hi1 = T.r[1].hi;
    lo2 = T.r[2].lo; hi2 = T.r[2].hi;
  }
  __device__ __forceinline__ void next(const Tiles&) {
    if (++j >= hi && lo1 != 0x7fffffff) {
      j = lo1; hi = hi1;
      lo1 = lo2; hi1 = hi2;
      lo2 = 0x7fffffff; hi2 = 0x7fffffff;
    }
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
