// mlra_plan.cuh -- the split plan shared by the host replica and the device kernels.
//
// The decode work of a batch is the concatenation of every sequence's KV tiles (64 positions
// each): sequence s owns global tiles [prefix[s], prefix[s+1]).  The batch is cut into R equal
// contiguous ranges, range r = [floor(r*T/R), floor((r+1)*T/R)) with T = prefix[N]; one
// persistent CTA (per branch group) handles one range.  A range may cover the tail of one
// sequence, whole sequences and the head of another: each (range, sequence) overlap is a
// segment with its own partial softmax state, stored in partial slot r + s (slots are unique
// because both r and s never decrease along the tile order).  A sequence split over several
// ranges is merged inside the decode kernel, by the CTA that finishes the last of its parts.
// The plan depends only on the logical lengths, never on physical page ids.  When the batch has fewer tiles than ranges, the number of ranges is
// cut to the tile count (effective_ranges) so that every range holds at least one tile and the
// ranges covering one sequence are consecutive.
#pragma once
#include <cstdint>

namespace mlra {

constexpr int kTile = 64;  // KV positions per tile

// Ranges actually used for `total` tiles when R are available (never more than the tiles).
__host__ __device__ inline int64_t effective_ranges(int64_t R, int64_t total) {
  return total < R ? (total > 0 ? total : 1) : R;
}

__host__ __device__ inline int64_t range_begin(int64_t r, int64_t total, int64_t R) {
  return (r * total) / R;
}

// The range holding global tile g: the largest r with range_begin(r) <= g.
__host__ __device__ inline int64_t range_of_tile(int64_t g, int64_t total, int64_t R) {
  return ((g + 1) * R + total - 1) / total - 1;
}

// First sequence s with prefix[s] <= g < prefix[s+1]  (prefix has n+1 entries, g < prefix[n]).
__host__ __device__ inline int seq_of_tile(const int32_t* prefix, int n, int64_t g) {
  int lo = 0, hi = n;  // answer in [lo, hi)
  while (hi - lo > 1) {
    int mid = (lo + hi) >> 1;
    if (prefix[mid] <= g) lo = mid; else hi = mid;
  }
  return lo;
}

struct Segment {
  int seq;        // sequence index
  int tile0;      // first tile of the segment, counted inside the sequence
  int ntiles;     // tiles in the segment (>= 1)
  bool whole;     // the segment covers the whole sequence (no merge needed)
};

// Walks the segments of one range in tile order (R: the effective number of ranges).
struct SegmentWalker {
  const int32_t* prefix;
  int n;
  int64_t g, end;
  int s;
  // A range index r >= R (a CTA beyond the effective ranges) walks nothing.  first_seq >= 0 is
  // the sequence holding the range's first tile when the caller knows it (saves the search).
  __host__ __device__ SegmentWalker(const int32_t* prefix_, int n_, int64_t total, int64_t R,
                                    int64_t r, int first_seq = -1)
      : prefix(prefix_), n(n_), g(r < R ? range_begin(r, total, R) : total),
        end(r < R ? range_begin(r + 1, total, R) : total), s(0) {
    if (g < end) s = first_seq >= 0 ? first_seq : seq_of_tile(prefix, n, g);
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

// For sequence s: the first range touching it and the number of ranges (partials) it spans.
// R must be the effective number of ranges.
__host__ __device__ inline void seq_parts(const int32_t* prefix, int s, int64_t total, int64_t R,
                                          int* first_range, int* nparts) {
  const int64_t p0 = prefix[s], p1 = prefix[s + 1];
  if (p1 <= p0) {
    *first_range = 0;
    *nparts = 0;
    return;
  }
  const int64_t r0 = range_of_tile(p0, total, R), r1 = range_of_tile(p1 - 1, total, R);
  *first_range = static_cast<int>(r0);
  *nparts = static_cast<int>(r1 - r0 + 1);
}

}  // namespace mlra
