// topk.cuh - neighbour influence and fixed-count top-k over the middle tokens
// (ESA write-up: neighbour-influence paragraph - a token's score is lifted by the
// tokens around it, read as s'_j = max_{|m - j| <= eps, m in middle} s_m; core-steps
// paragraph - a fixed number k of tokens is kept).
//
// Order: s' descending, then position ascending. Exact selection in three radix
// levels over order-preserving 32-bit keys (11 + 11 + 10 bits): each level builds a
// histogram of the candidates that still share the threshold's prefix and picks the
// bin that holds the k-th key. The threshold key T and the number of keys equal to T
// that are kept (the lowest positions first) then drive an ordered compaction, so
// the output is ascending by position without a sort. Integer atomics only: the
// result does not depend on scheduling.
#pragma once
#include <cub/block/block_reduce.cuh>
#include <cub/block/block_scan.cuh>

#include "common.cuh"

namespace esa {

constexpr int kTkTile = 1024;      // elements per CTA in the streaming kernels
constexpr int kTkThreads = 256;    // 4 elements per thread
constexpr int kTkBins = 2048;

struct SelState {      // per sequence
  uint32_t prefix;     // high bits of T fixed so far
  uint32_t want;       // keys still to take at or below the current prefix
  uint32_t thresh;     // final T
  uint32_t pad;
};

__host__ __device__ constexpr int level_shift(int level) { return level == 0 ? 21 : (level == 1 ? 10 : 0); }
__host__ __device__ constexpr int level_bits(int level) { return level == 2 ? 10 : 11; }

// s' (neighbour max), order keys u, optional s' copy out, and the level-0 histogram.
__global__ void __launch_bounds__(kTkThreads) pool_hist_kernel(const float* __restrict__ s, int64_t n, int eps,
                                                              uint32_t* __restrict__ u, float* __restrict__ s_prime_out,
                                                              uint32_t* __restrict__ hist) {
  __shared__ float sv[kTkTile + 2 * 64];
  __shared__ uint32_t h[kTkBins];
  const int b = blockIdx.y;
  const int64_t j0 = (int64_t)blockIdx.x * kTkTile;
  const float* sb = s + (int64_t)b * n;
  for (int t = threadIdx.x; t < kTkBins; t += kTkThreads) h[t] = 0;
  for (int t = threadIdx.x; t < kTkTile + 2 * eps; t += kTkThreads) {
    const int64_t j = j0 - eps + t;
    sv[t] = (j >= 0 && j < n) ? sb[j] : -INFINITY;
  }
  __syncthreads();
  for (int t = threadIdx.x; t < kTkTile; t += kTkThreads) {
    const int64_t j = j0 + t;
    if (j >= n) break;
    float m = sv[t + eps];
    for (int o = 1; o <= eps; ++o) m = fmaxf(m, fmaxf(sv[t + eps - o], sv[t + eps + o]));
    const uint32_t key = order_key(m);
    u[(int64_t)b * n + j] = key;
    if (s_prime_out) s_prime_out[(int64_t)b * n + j] = m;
    atomicAdd(&h[key >> 21], 1u);
  }
  __syncthreads();
  uint32_t* hb = hist + (int64_t)b * 3 * kTkBins;
  for (int t = threadIdx.x; t < kTkBins; t += kTkThreads)
    if (h[t]) atomicAdd(&hb[t], h[t]);
}

// Histogram of level `level` over keys whose bits above level_shift(level-1)... match.
__global__ void __launch_bounds__(kTkThreads) radix_hist_kernel(const uint32_t* __restrict__ u, int64_t n, int level,
                                                               const SelState* __restrict__ st,
                                                               uint32_t* __restrict__ hist) {
  __shared__ uint32_t h[kTkBins];
  const int b = blockIdx.y;
  const int64_t j0 = (int64_t)blockIdx.x * kTkTile;
  for (int t = threadIdx.x; t < kTkBins; t += kTkThreads) h[t] = 0;
  __syncthreads();
  const uint32_t prefix = st[b].prefix;
  const int hi_shift = level_shift(level - 1);
  const int shift = level_shift(level);
  const uint32_t mask = (1u << level_bits(level)) - 1u;
  const uint32_t* ub = u + (int64_t)b * n;
  for (int t = threadIdx.x; t < kTkTile; t += kTkThreads) {
    const int64_t j = j0 + t;
    if (j >= n) break;
    const uint32_t key = ub[j];
    if ((key >> hi_shift) == prefix) atomicAdd(&h[(key >> shift) & mask], 1u);
  }
  __syncthreads();
  uint32_t* hb = hist + ((int64_t)b * 3 + level) * kTkBins;
  for (int t = threadIdx.x; t < kTkBins; t += kTkThreads)
    if (h[t]) atomicAdd(&hb[t], h[t]);
}

// One CTA per sequence: find the bin holding the want-th largest key of this level.
// level 0 starts from want = kk (keys to keep).
__global__ void __launch_bounds__(1024) radix_select_kernel(const uint32_t* __restrict__ hist, int level, uint32_t kk,
                                                           SelState* __restrict__ st) {
  using Scan = cub::BlockScan<uint32_t, 1024>;
  __shared__ typename Scan::TempStorage tmp;
  __shared__ uint32_t found_bin, found_above;
  const int b = blockIdx.x;
  const int nb = 1 << level_bits(level);
  const uint32_t want = level == 0 ? kk : st[b].want;
  const uint32_t* hb = hist + ((int64_t)b * 3 + level) * kTkBins;
  // thread t owns bins in descending order: rank r = 2t, 2t+1 -> bin nb-1-r
  const int per = nb / 1024;
  uint32_t c[2] = {0, 0};
  uint32_t sum = 0;
  for (int q = 0; q < per; ++q) {
    c[q] = hb[nb - 1 - (threadIdx.x * per + q)];
    sum += c[q];
  }
  uint32_t before;
  Scan(tmp).ExclusiveSum(sum, before);
  uint32_t acc = before;
  for (int q = 0; q < per; ++q) {
    if (acc < want && acc + c[q] >= want) {
      found_bin = nb - 1 - (threadIdx.x * per + q);
      found_above = acc;
    }
    acc += c[q];
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t prefix = level == 0 ? 0u : st[b].prefix;
    const uint32_t np = (prefix << level_bits(level)) | found_bin;
    st[b].prefix = np;
    st[b].want = want - found_above;
    if (level == 2) st[b].thresh = np;
  }
}

// Per tile: number of keys above T and equal to T.
__global__ void __launch_bounds__(kTkThreads) compact_count_kernel(const uint32_t* __restrict__ u, int64_t n,
                                                                  const SelState* __restrict__ st,
                                                                  uint2* __restrict__ tile_counts, int n_tiles) {
  using Red = cub::BlockReduce<uint32_t, kTkThreads>;
  __shared__ typename Red::TempStorage t1, t2;
  const int b = blockIdx.y;
  const int64_t j0 = (int64_t)blockIdx.x * kTkTile;
  const uint32_t T = st[b].thresh;
  const uint32_t* ub = u + (int64_t)b * n;
  uint32_t gt = 0, eq = 0;
  for (int t = threadIdx.x; t < kTkTile; t += kTkThreads) {
    const int64_t j = j0 + t;
    if (j >= n) break;
    const uint32_t key = ub[j];
    gt += key > T;
    eq += key == T;
  }
  gt = Red(t1).Sum(gt);
  eq = Red(t2).Sum(eq);
  if (threadIdx.x == 0) tile_counts[(int64_t)b * n_tiles + blockIdx.x] = make_uint2(gt, eq);
}

// Ordered compaction: keep key > T, and key == T while fewer than `want` equal keys
// at lower positions were kept. Writes positions mid0 + j ascending.
__global__ void __launch_bounds__(kTkThreads) compact_write_kernel(const uint32_t* __restrict__ u, int64_t n,
                                                                  const SelState* __restrict__ st,
                                                                  const uint2* __restrict__ tile_counts, int n_tiles,
                                                                  int64_t mid0, int topk, int32_t* __restrict__ idx) {
  using Scan = cub::BlockScan<uint32_t, kTkThreads>;
  __shared__ typename Scan::TempStorage t1, t2;
  __shared__ uint32_t base_gt, base_eq;
  const int b = blockIdx.y;
  const int64_t j0 = (int64_t)blockIdx.x * kTkTile;
  const uint32_t T = st[b].thresh;
  const uint32_t want = st[b].want;
  if (threadIdx.x < 32) {
    uint32_t g = 0, e = 0;
    for (int t = threadIdx.x; t < blockIdx.x; t += 32) {
      const uint2 c = tile_counts[(int64_t)b * n_tiles + t];
      g += c.x;
      e += c.y;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      g += __shfl_xor_sync(0xffffffffu, g, o);
      e += __shfl_xor_sync(0xffffffffu, e, o);
    }
    if (threadIdx.x == 0) { base_gt = g; base_eq = e; }
  }
  __syncthreads();
  // 4 consecutive elements per thread keep index order within the tile
  uint32_t key[4];
  uint32_t eq_cnt = 0;
  const uint32_t* ub = u + (int64_t)b * n;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int64_t j = j0 + threadIdx.x * 4 + q;
    key[q] = j < n ? ub[j] : 0u;
    if (j < n && key[q] == T) ++eq_cnt;
  }
  uint32_t eq_before;
  Scan(t1).ExclusiveSum(eq_cnt, eq_before);
  eq_before += base_eq;
  bool keep[4];
  uint32_t keep_cnt = 0;
  uint32_t eq_run = eq_before;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int64_t j = j0 + threadIdx.x * 4 + q;
    keep[q] = false;
    if (j < n) {
      if (key[q] > T) keep[q] = true;
      else if (key[q] == T) { keep[q] = eq_run < want; ++eq_run; }
    }
    keep_cnt += keep[q];
  }
  uint32_t pos;
  Scan(t2).ExclusiveSum(keep_cnt, pos);
  pos += base_gt + min(base_eq, want);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    if (keep[q]) {
      if (pos < (uint32_t)topk) idx[(int64_t)b * topk + pos] = (int32_t)(mid0 + j0 + threadIdx.x * 4 + q);
      ++pos;
    }
  }
}

// idx[b, kk..topk) = -1, count[b] = kk; with all_mid, also idx[b, j] = mid0 + j for j < kk.
__global__ void fill_selection_kernel(int32_t* __restrict__ idx, int32_t* __restrict__ count, int topk, int kk,
                                      int64_t mid0, int all_mid) {
  const int b = blockIdx.y;
  for (int t = blockIdx.x * blockDim.x + threadIdx.x; t < topk; t += gridDim.x * blockDim.x) {
    if (t >= kk) idx[(int64_t)b * topk + t] = -1;
    else if (all_mid) idx[(int64_t)b * topk + t] = (int32_t)(mid0 + t);
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) count[b] = kk;
}

}  // namespace esa
