// cowa_pattern.h -- CoWA visibility pattern and tile planner as plain integer arithmetic.
//
// Used unchanged by the host (validation, introspection) and by every kernel
// (on the fly, per CTA).  The pattern is a function of positions and of the
// global KV-head index only ("CoWindow Attention: Full Causal Coverage Is a
// Collective Property", Abstract: no learned router or indexer; skillfed.io
// news summary, paragraphs 2 and 4).
//
//   visible(t, s, G) = s <= t  and  ( s < S  or  s > t - L  or  s in I_G )
//   I_G = [b_p, b_{p+1}),  b_i = S + floor(i*(T-S)/H),  p = (G mod D) * (H/D)
//
// Everything here returns half-open ranges [lo, hi) and never touches memory.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define COWA_HD __host__ __device__ __forceinline__
#else
#define COWA_HD inline
#endif

namespace cowa {

struct Pat {
  int S, L, T, D;
  int G0;  // global index of local KV head 0
  int H;   // KV heads in the layer
};

struct Range {
  int lo, hi;  // [lo, hi); empty if lo >= hi
};

COWA_HD int imin(int a, int b) { return a < b ? a : b; }
COWA_HD int imax(int a, int b) { return a > b ? a : b; }

// b_i = S + floor(i * (T - S) / H), in 64-bit to avoid overflow of i*(T-S).
COWA_HD int bound(const Pat& p, int i) {
  return p.S + (int)(((int64_t)i * (int64_t)(p.T - p.S)) / (int64_t)p.H);
}

// Long-range interval of local KV head g.
COWA_HD Range interval_of(const Pat& p, int g) {
  const int G = p.G0 + g;
  const int slot = (G % p.D) * (p.H / p.D);
  return Range{bound(p, slot), bound(p, slot + 1)};
}

COWA_HD bool visible(const Pat& p, Range iv, int t, int s) {
  return s <= t && (s < p.S || s > t - p.L || (s >= iv.lo && s < iv.hi));
}

// Sort up to three ranges by lo, drop empty ones and merge overlapping or
// touching ones.  Returns the number n of disjoint ranges written to r[0..n);
// r[n..3) are set to the empty sentinel [INT_MAX, INT_MAX).  Written with fixed
// indices only, so that a kernel keeps everything in registers.
COWA_HD int merge3(Range a, Range b, Range c, Range* r) {
  constexpr int kNone = 0x7fffffff;
  Range v0 = a, v1 = b, v2 = c;
  // 3-element sorting network on lo (empty ranges pushed last by lo = INT_MAX)
  if (v0.lo >= v0.hi) { v0.lo = kNone; v0.hi = kNone; }
  if (v1.lo >= v1.hi) { v1.lo = kNone; v1.hi = kNone; }
  if (v2.lo >= v2.hi) { v2.lo = kNone; v2.hi = kNone; }
  if (v1.lo < v0.lo) { Range x = v0; v0 = v1; v1 = x; }
  if (v2.lo < v1.lo) { Range x = v1; v1 = v2; v2 = x; }
  if (v1.lo < v0.lo) { Range x = v0; v0 = v1; v1 = x; }
  Range o0 = v0, o1{kNone, kNone}, o2{kNone, kNone};
  int n = v0.lo != kNone ? 1 : 0;
  if (v1.lo != kNone) {
    if (v1.lo <= o0.hi) o0.hi = imax(o0.hi, v1.hi);
    else { o1 = v1; n = 2; }
  }
  if (v2.lo != kNone) {
    if (n == 1) {
      if (v2.lo <= o0.hi) o0.hi = imax(o0.hi, v2.hi);
      else { o1 = v2; n = 2; }
    } else {
      if (v2.lo <= o1.hi) o1.hi = imax(o1.hi, v2.hi);
      else { o2 = v2; n = 3; }
    }
  }
  r[0] = o0; r[1] = o1; r[2] = o2;
  return n;
}

// Keys visible to position t (local KV head g, interval iv), as <= 3 disjoint
// sorted ranges: sink [0, min(S, t+1)), band [max(0, t-L+1), t+1), and
// interval [lo, min(hi, t+1)).
COWA_HD int row_ranges(const Pat& p, Range iv, int t, Range* r) {
  Range sink{0, imin(p.S, t + 1)};
  Range band{imax(0, t - p.L + 1), t + 1};
  Range lr{iv.lo, imin(iv.hi, t + 1)};
  return merge3(sink, band, lr, r);
}

// Forward plan: KV tiles (of BN keys) that rows [t0, t1) visit, as <= 3
// disjoint sorted tile-index ranges.  Exactly the tiles whose block holds at
// least one visible element: the union over t in [t0, t1) of the row ranges
// is sink [0, min(S, t1)), band [max(0, t0-L+1), t1), interval [lo, min(hi, t1)).
COWA_HD int fwd_tile_ranges(const Pat& p, Range iv, int t0, int t1, int BN, Range* r) {
  Range sink{0, imin(p.S, t1)};
  Range band{imax(0, t0 - p.L + 1), t1};
  Range lr{iv.lo, imin(iv.hi, t1)};
  Range tk[3];
  const Range src[3] = {sink, band, lr};
  for (int i = 0; i < 3; ++i) {
    if (src[i].lo < src[i].hi) {
      tk[i].lo = src[i].lo / BN;
      tk[i].hi = (src[i].hi + BN - 1) / BN;
    } else {
      tk[i].lo = 0; tk[i].hi = 0;
    }
  }
  return merge3(tk[0], tk[1], tk[2], r);
}

// True iff every (t, s) with t in [t0, t1), s in [s0, s1) is visible.
// Requires s1 - 1 <= t0 (all keys at or before every query); the hardest row
// is t1 - 1, whose band starts latest, so [s0, s1) must lie inside
// [0, S) U I_g U [t1 - L, inf).
COWA_HD bool tile_full(const Pat& p, Range iv, int t0, int t1, int s0, int s1) {
  if (s1 - 1 > t0) return false;
  int x = s0;
  // walk right through the covering segments; at most three steps
  for (int it = 0; it < 4 && x < s1; ++it) {
    if (x < p.S) { x = p.S; continue; }
    if (x >= iv.lo && x < iv.hi) { x = iv.hi; continue; }
    if (x >= t1 - p.L) { x = s1; continue; }
    return false;
  }
  return x >= s1;
}

// Backward plan: the rows that see any key of [s0, s1) form one contiguous
// range starting at s0: a sink or interval key s is seen by every t >= s, a
// band-only key s by t in [s, s+L).  Returns rows [s0, end) clipped to N.
COWA_HD Range bwd_row_range(const Pat& p, Range iv, int s0, int s1, int N) {
  // smallest key of the tile that is in the sink or the interval
  bool special = (s0 < p.S) || (iv.lo < iv.hi && iv.lo < s1 && iv.hi > s0);
  // band-only: rows up to s1 - 1 + L, written so that a window of up to INT_MAX cannot overflow
  int end = special ? N : (p.L >= N - s1 + 1 ? N : s1 - 1 + p.L);
  return Range{s0, imax(s0, end)};
}

}  // namespace cowa
