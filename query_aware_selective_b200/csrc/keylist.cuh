// keylist.cuh - the ordered key list one ESA chunk attends (ESA write-up,
// implementation paragraph: initial tokens + selected middle tokens + local tokens).
//   t in [0, ni)            -> position t                (initial)
//   t in [ni, ni + cnt)     -> idx[b, t - ni]            (selected, ascending)
//   t in [ni + cnt, ...)    -> lo + (t - ni - cnt)       (local, then the chunk)
// Positions are clamped into [0, n_cap) so a corrupt index list cannot read outside
// the cache.
#pragma once
#include <stdint.h>

namespace esa {

struct KeyList {
  const int32_t* idx;    // [B, idx_stride]
  int64_t idx_stride;
  int64_t ni;            // initial tokens
  int64_t lo;            // first local position
  int64_t n_cap;
  const int32_t* count;  // [B]
  __device__ __forceinline__ int64_t pos(int b, int cnt, int64_t t) const {
    int64_t p;
    if (t < ni) p = t;
    else if (t < ni + cnt) p = idx[b * idx_stride + (t - ni)];
    else p = lo + (t - ni - cnt);
    return p < 0 ? 0 : (p >= n_cap ? n_cap - 1 : p);
  }
};

}  // namespace esa
