// keylist.cuh - the ordered key list one ESA chunk attends (ESA write-up,
// implementation paragraph: initial tokens + selected middle tokens + local tokens).
//   t in [0, ni)            -> position t                (initial)
//   t in [ni, ni + cnt)     -> idx[b, t - ni]            (selected, ascending)
//   t in [ni + cnt, ...)    -> lo + (t - ni - cnt)       (local, then the chunk)
// Positions are clamped into [0, n_cap) so a corrupt index list cannot read outside
// the cache. In a variable-length decode batch ni and lo differ per sequence (resolve).
#pragma once
#include <stdint.h>

#include "common.cuh"

namespace esa {

struct KeyList {
  const int32_t* idx;    // [B, idx_stride]
  int64_t idx_stride;
  int64_t ni;            // initial tokens
  int64_t lo;            // first local position
  int64_t n_cap;
  const int32_t* count;  // [B]
  VarLen vl;             // vl.len null: ni and lo as given (every sequence's query at the call's c0)
  // Sequence b of a variable-length batch: sets ni and lo from its own query position
  // and returns that position.
  __device__ __forceinline__ int64_t resolve(int b, unsigned site) {
    const int64_t c0 = vl.c0(b, site);
    lo = vl.lo(c0);
    ni = lo < (int64_t)vl.n_init ? lo : (int64_t)vl.n_init;
    return c0;
  }
  __device__ __forceinline__ int64_t pos(int b, int cnt, int64_t t) const {
    int64_t p;
    if (t < ni) p = t;
    else if (t < ni + cnt) p = idx[b * idx_stride + (t - ni)];
    else p = lo + (t - ni - cnt);
    return p < 0 ? 0 : (p >= n_cap ? n_cap - 1 : p);
  }
};

}  // namespace esa
