// mlra_plan.cuh -- the split plan shared by the host replica and the device kernels.
//
// The decode work of a batch is the concatenation of every sequence's KV tiles: sequence s owns
// global tiles [prefix[s], prefix[s+1]) of the T = prefix[N] tiles.  The batch is cut into R
// contiguous work ranges, one persistent CTA (per branch group) each.  A range may cover the
// tail of one sequence, whole sequences and the head of another: each (range, sequence) overlap
// is a segment with its own partial softmax state, stored in partial slot r + s (slots are
// unique because both r and s never decrease along the tile order).  A sequence split over
// several ranges is merged by the combine kernel.  The plan depends only on the logical
// lengths, never on physical page ids.
//
// Balance.  A CTA pays a fixed price each time a new sequence starts inside its range (the
// segment epilogue, the new queries' load), about `cost` tiles of streaming.  So the ranges
// split a virtual length in which every non-empty sequence counts cost + tiles:
//   vprefix[s] = prefix[s] + cost * (non-empty sequences before s),   V = vprefix[N],
//   range r starts at virtual position v_r = floor(r V / R)
// and v maps back to a real tile as g(v) = prefix[s] + max(0, v - vprefix[s] - cost) for the
// sequence s whose virtual interval [vprefix[s], vprefix[s+1]) holds v.  The ranges are
// [g(v_r), g(v_{r+1})); one may be empty (two boundaries inside one sequence's cost zone), and
// then it lies at a sequence start, never between two parts of one sequence.  With cost = 0 this
// is the equal split [floor(rT/R), floor((r+1)T/R)).  R is first cut to the tile count T
// (effective_ranges).
#pragma once
#include <cstdint>

namespace mlra {

constexpr int kTile = 64;  // KV positions per tile-row block of the page arithmetic

// Ranges actually used for `total` tiles when R are available (never more than the tiles).
__host__ __device__ inline int64_t effective_ranges(int64_t R, int64_t total) {
  return total < R ? (total > 0 ? total : 1) : R;
}

// First sequence s with prefix[s] <= g < prefix[s+1]  (prefix has n+1 entries, g < prefix[n]).
// Equal entries (empty sequences) resolve to the last of them, i.e. the non-empty sequence.
__host__ __device__ inline int seq_of_tile(const int32_t* prefix, int n, int64_t g) {
  int lo = 0, hi = n;  // answer in [lo, hi)
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (prefix[mid] <= g) lo = mid; else hi = mid;
  }
  return lo;
}

// The real and the virtual tile prefix of a batch (see the top of the file).
struct PlanView {
  const int32_t* prefix;   // [n + 1]
  const int32_t* vprefix;  // [n + 1]
  int n;
  int64_t total, vtotal;   // prefix[n], vprefix[n]
  int64_t R;               // effective ranges
  int cost;
};

// First real tile of range r (r in [0, R]); range_start(R) = total.
__host__ __device__ inline int64_t range_start(const PlanView& pv, int64_t r) {
  if (r >= pv.R || pv.total == 0) return r <= 0 ? 0 : pv.total;
  const int64_t v = (r * pv.vtotal) / pv.R;
  const int s = seq_of_tile(pv.vprefix, pv.n, v);
  const int64_t o = v - pv.vprefix[s] - pv.cost;
  return pv.prefix[s] + (o > 0 ? o : 0);
}

struct Segment {
  int seq;        // sequence index
  int tile0;      // first tile of the segment, counted inside the sequence
  int ntiles;     // tiles in the segment (>= 1)
  bool whole;     // the segment covers the whole sequence (no merge needed)
};

// Walks the segments of the real tiles [g_begin, g_end) in tile order.
struct SegmentWalker {
  const int32_t* prefix;
  int n;
  int64_t g, end;
  int s;
  __host__ __device__ SegmentWalker(const int32_t* prefix_, int n_, int64_t g_begin, int64_t g_end)
      : prefix(prefix_), n(n_), g(g_begin), end(g_end), s(0) {
    if (g < end) s = seq_of_tile(prefix, n, g);
  }
  __host__ __device__ bool next(Segment& seg) {
    if (g >= end) return false;
    while (prefix[s + 1] <= g) ++s;
    const int64_t p0 = prefix[s], p1 = prefix[s + 1];
    const int64_t stop = end < p1 ? end : p1;
    seg.seq = s;
    seg.tile0 = static_cast<int>(g - p0);
    seg.ntiles = static_cast<int>(stop - g);
    seg.whole = (g == p0) && (stop == p1);
    g = stop;
    return true;
  }
};

}  // namespace mlra
