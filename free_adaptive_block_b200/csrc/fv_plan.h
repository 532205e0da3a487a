// Work plan of the fused pool-and-route kernel: the order of its items in one queue.
// Host and device code; no CUDA types, so host tests compile it with a C++ compiler.
#pragma once

#ifdef __CUDACC__
#define FV_HD __host__ __device__
#else
#define FV_HD
#endif

namespace fv {

constexpr int kLogitTile = 64;         // query x key blocks per logits tile

// Items per (b, h) slice: 2 nB pool items (Q blocks, then K blocks), tiles^2 logits tiles
// and ceil(nB / 8) select items (8 query blocks each).  Step i of the queue holds the
// pool items of slice i, then the logits tiles of slice i - 1, then the select items of
// slice i - 2 (those that exist), so that every item comes after the items it needs.
struct PrPlan {
  int S, nP, nL, nS, tiles;
  long long total;
};

FV_HD inline PrPlan pr_plan(int slices, int nB) {
  PrPlan pl;
  pl.S = slices;
  pl.tiles = (nB + kLogitTile - 1) / kLogitTile;
  pl.nP = 2 * nB;
  pl.nL = pl.tiles * pl.tiles;
  pl.nS = (nB + 7) / 8;
  pl.total = static_cast<long long>(pl.S) * (pl.nP + pl.nL + pl.nS);
  return pl;
}

// Items before step i.
FV_HD inline long long pr_prefix(const PrPlan& pl, long long i) {
  const long long S = pl.S;
  const long long a = i < S ? i : S;
  const long long b = i - 1 < 0 ? 0 : (i - 1 < S ? i - 1 : S);
  const long long c = i - 2 < 0 ? 0 : (i - 2 < S ? i - 2 : S);
  return a * pl.nP + b * pl.nL + c * pl.nS;
}

// Item t (0 <= t < total) -> kind (0 pool, 1 logits, 2 select), slice, and index among
// the slice's items of that kind.
FV_HD inline void pr_decode(const PrPlan& pl, long long t, int& kind, int& slice, int& idx) {
  long long lo = 0, hi = static_cast<long long>(pl.S) + 2;   // the step, in [lo, hi)
  while (hi - lo > 1) {
    const long long mid = (lo + hi) / 2;
    if (pr_prefix(pl, mid) <= t) lo = mid; else hi = mid;
  }
  const long long i = lo;
  long long r = t - pr_prefix(pl, i);
  if (i < pl.S) {
    if (r < pl.nP) { kind = 0; slice = static_cast<int>(i); idx = static_cast<int>(r); return; }
    r -= pl.nP;
  }
  if (i >= 1 && i - 1 < pl.S) {
    if (r < pl.nL) { kind = 1; slice = static_cast<int>(i - 1); idx = static_cast<int>(r); return; }
    r -= pl.nL;
  }
  kind = 2;
  slice = static_cast<int>(i - 2);
  idx = static_cast<int>(r);
}

}  // namespace fv
