// common.cuh -- small device helpers shared by the indexer, top-k and attention kernels.
#pragma once
#include <cstdint>

namespace csa {

// Compressed entries visible to a query at position `pos`: entry j covers tokens up to
// m(j+1)-1 and is visible once that token is (position <= pos); capped by the number of
// entries the cache holds.
__device__ __forceinline__ int visible_entries(int pos, int m, int n_entries) {
  int v = (pos + 1) / m;
  v = v < 0 ? 0 : v;
  return v < n_entries ? v : n_entries;
}

}  // namespace csa
