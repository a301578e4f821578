// index_common.cuh -- pieces shared by the indexer's tensor-core scorers
// (bf16 keys in index_tc.cu, MXFP4 keys in index_fp4.cu): the tile size,
// the score histogram of the top-k, and the walk of a CTA over its share of
// the flat (query group, entry tile) work list.
#pragma once

#include "common.cuh"

namespace csa {

constexpr int kHistBins = 4096;    // top 12 bits of the order-preserving score key
constexpr int kTileM = 128;        // entries per tile (the MMA's M)
constexpr int kInlineGroups = 64;  // groups whose tile prefix a CTA computes itself

// Walk of a CTA over its slice of the flat (group, tile) list.
struct TileCursor {
  int g, t, left;
  __device__ void init(const int* prefix, int ngroups, int start, int count) {
    int lo = 0, hi = ngroups;
    while (lo < hi) {  // last g with prefix[g] <= start
      int mid = (lo + hi + 1) >> 1;
      if (prefix[mid] <= start) lo = mid; else hi = mid - 1;
    }
    g = lo;
    t = start - prefix[g];
    left = count;
  }
  __device__ int tiles(const int* prefix) const { return prefix[g + 1] - prefix[g]; }
  __device__ bool first(int pos_in_cta) const { return t == 0 || pos_in_cta == 0; }
  __device__ bool last(const int* prefix) const { return left == 1 || t + 1 == tiles(prefix); }
  __device__ void next(const int* prefix, int ngroups) {
    --left;
    if (++t >= tiles(prefix)) {
      t = 0;
      do { ++g; } while (g < ngroups && prefix[g + 1] == prefix[g]);
    }
  }
};


}  // namespace csa
