// topk.cuh - neighbour influence and fixed-count top-k over the middle tokens of each
// sequence, in one launch (ESA write-up: neighbour-influence paragraph - a token's
// score is lifted by the tokens around it, read as s'_j = max_{|m - j| <= eps, m in
// middle} s_m; core-steps paragraph - a fixed number k of tokens is kept;
// score-correction paragraph - when raw scores come in, s_j = sum_i max(S_ij - m_i, -C)
// is formed on the fly in query order).
//
// One thread-block cluster per sequence (16 CTAs when every sequence's cluster can be
// resident at once, else 8);
// CTA r owns a contiguous range of middle positions. Order: s' descending, then
// position ascending. Exact selection in three radix levels over order-preserving
// 32-bit keys (11 + 11 + 10 bits). At each level every CTA histograms its keys that
// still share the threshold's prefix (shared-memory atomics) and adds each non-zero bin
// into the CTA that owns the bin's slice (distributed shared-memory reductions: CTA r
// owns slice r); after one cluster barrier every CTA reads the merged bins it scans with
// 16-byte loads from their owners and finds the same bin holding the want-th largest
// key. The threshold key T and the number of keys equal to T to keep (lowest positions
// first) then drive an ordered compaction: every CTA pushes its (above T, equal to T)
// counts to the higher ranks, and a block scan in position order writes the kept
// positions ascending, so no sort is needed. Integer atomics
// only: the result does not depend on scheduling. The keys stay in shared memory when
// a CTA's range fits (kSelUCap), else in a global scratch array.
#pragma once
#include <cub/block/block_scan.cuh>

#include "common.cuh"

namespace esa {

constexpr int kSelThreads = 512;
constexpr int kSelBins = 2048;
constexpr int kSelTile = 4096;       // positions per pooling tile
constexpr int kSelMaxEps = 64;
constexpr int kSelUCap = 16384;      // order keys a CTA keeps in shared memory

struct SelectArgs {
  const float* S;          // [B, lq, n_mid] raw scores, with m_key; or null
  const uint32_t* m_key;   // [B, lq] order keys of the per-query maxima
  const float* s;          // [B, n_mid] chunk-summed corrected scores (when S is null)
  int lq;
  float clamp_c;
  int64_t n_mid, mid0;
  int eps;                 // <= kSelMaxEps
  int kk;                  // keys to keep: min(topk, n_mid) >= 1
  int topk;
  VarLen vl;               // vl.len: a variable-length decode batch; n_mid is then the longest
                           // possible middle (the row stride of S, s, s_prime_out) and kk == topk
  uint32_t* u;             // [B, n_mid] key scratch (used when a CTA's range exceeds kSelUCap)
  float* s_prime_out;      // [B, n_mid] or null
  int32_t* idx;            // [B, topk]
  int32_t* count;          // [B]
};

struct SelSmem {
  uint32_t hist[kSelBins];                 // this CTA's histogram of the current level
  uint32_t merged[2 * kSelBins + 1024];    // per level: the cluster's counts of the bin slice this CTA owns
  float sv[kSelTile + 2 * kSelMaxEps + 16];   // + slack: the vector pooling reads 16 values per group
  uint32_t cnt_lo[16][2];                  // (above T, equal to T) of each lower-ranked CTA, pushed by it
  uint32_t sel_bin, sel_above;
  typename cub::BlockScan<uint32_t, kSelThreads>::TempStorage scan;
  uint32_t ucache[kSelUCap];
};
constexpr int kSelSmemBytes = (int)sizeof(SelSmem);

// Raw scores of the tile [g0 - eps, g0 - eps + kSelHaloTile) for this thread's slots
// (slot e = position tid + e * kSelThreads), or -inf outside the middle.
constexpr int kSelHaloTile = kSelTile + 2 * kSelMaxEps;
constexpr int kSelSlots = (kSelHaloTile + kSelThreads - 1) / kSelThreads;

__device__ __forceinline__ void sel_load_tile(const SelectArgs& a, int b, int64_t n, int64_t g0, int nt, float* v) {
  const int tid = threadIdx.x;
  const int width = nt + 2 * a.eps;
  if (!a.S) {
    const float* sb = a.s + (int64_t)b * a.n_mid;
#pragma unroll
    for (int e = 0; e < kSelSlots; ++e) {
      const int t = tid + e * kSelThreads;
      const int64_t j = g0 - a.eps + t;
      v[e] = (t < width && j >= 0 && j < n) ? __ldcg(sb + j) : -INFINITY;
    }
    return;
  }
  const float lo = -a.clamp_c;
#pragma unroll
  for (int e = 0; e < kSelSlots; ++e) v[e] = 0.f;
  for (int i = 0; i < a.lq; ++i) {
    const float m = key_to_float(__ldg(&a.m_key[b * a.lq + i]));
    const float* Sb = a.S + ((int64_t)b * a.lq + i) * a.n_mid;
    float x[kSelSlots];
#pragma unroll
    for (int e = 0; e < kSelSlots; ++e) {
      const int t = tid + e * kSelThreads;
      const int64_t j = g0 - a.eps + t;
      x[e] = (t < width && j >= 0 && j < n) ? __ldcg(Sb + j) : 0.f;
    }
#pragma unroll
    for (int e = 0; e < kSelSlots; ++e) v[e] += fmaxf(x[e] - m, lo);
  }
#pragma unroll
  for (int e = 0; e < kSelSlots; ++e) {
    const int t = tid + e * kSelThreads;
    const int64_t j = g0 - a.eps + t;
    if (!(t < width && j >= 0 && j < n)) v[e] = -INFINITY;
  }
}

// grid (CL, B), cluster (CL, 1, 1), kSelThreads threads, kSelSmemBytes dynamic shared memory.
template <int CL>
__global__ void __launch_bounds__(kSelThreads, 2) select_cluster_kernel(const SelectArgs a) {
  extern __shared__ __align__(16) uint8_t sel_dsm[];
  SelSmem& sm = *reinterpret_cast<SelSmem*>(sel_dsm);
  using Scan = cub::BlockScan<uint32_t, kSelThreads>;
  const uint32_t rank = cluster_rank();
  const int b = blockIdx.y;
  const int tid = threadIdx.x;
  // this selection's middle length and keep count (a variable-length batch: its own)
  const int64_t n = a.vl.len ? a.vl.n_mid(b, 901) : a.n_mid;
  const int kk = (int)min((int64_t)a.kk, n);
  if (kk == 0) {                           // empty middle: nothing kept (before any cluster step)
    if (rank == 0) {
      for (int t = tid; t < a.topk; t += kSelThreads) a.idx[(int64_t)b * a.topk + t] = -1;
      if (tid == 0) a.count[b] = 0;
    }
    return;
  }
  const int64_t per = ((n + CL - 1) / CL + 3) & ~(int64_t)3;   // a multiple of 4: 16-byte key groups
  const int64_t per_stride = ((a.n_mid + CL - 1) / CL + 3) & ~(int64_t)3;
  const int64_t j0 = min(n, (int64_t)rank * per);
  const int nloc = (int)(min(n, j0 + per) - j0);
  // key of position j0 + t at ub[t]; the global scratch gives every CTA per_stride slots
  uint32_t* ub = per <= kSelUCap ? sm.ucache : a.u + ((int64_t)b * CL + rank) * per_stride;
  const int eps = a.eps;

  // every CTA clears its merged slices; the barrier phase this arrival opens is waited
  // for only after the pooling pass below
  for (int t = tid; t < 2 * kSelBins + 1024; t += kSelThreads) sm.merged[t] = 0;
  cluster_arrive();

  // ---- s', order keys and the level-0 histogram; the next tile's scores load while
  //      this tile is pooled
  for (int t = tid; t < kSelBins; t += kSelThreads) sm.hist[t] = 0;
  __syncthreads();
  const int n_tiles = (nloc + kSelTile - 1) / kSelTile;
  float v[kSelSlots];
  if (n_tiles > 0) sel_load_tile(a, b, n, j0, min(nloc, kSelTile), v);
  for (int tile = 0; tile < n_tiles; ++tile) {
    const int t0 = tile * kSelTile;
    const int nt = min(kSelTile, nloc - t0);
#pragma unroll
    for (int e = 0; e < kSelSlots; ++e) {
      const int t = tid + e * kSelThreads;
      if (t < kSelHaloTile) sm.sv[t] = v[e];
    }
    __syncthreads();
    if (tile + 1 < n_tiles) sel_load_tile(a, b, n, j0 + t0 + kSelTile, min(kSelTile, nloc - t0 - kSelTile), v);
    // four consecutive positions per thread; with eps <= 6 the window of all four is one
    // run of 16 values read as four 16-byte loads
    for (int t = 4 * tid; t < nt; t += 4 * kSelThreads) {
      float mq[4];
      if (eps == 2) {
        const float4 x0 = *reinterpret_cast<const float4*>(&sm.sv[t]);
        const float4 x1 = *reinterpret_cast<const float4*>(&sm.sv[t + 4]);
        const float m12 = fmaxf(x0.y, x0.z), m23 = fmaxf(x0.z, x0.w), m45 = fmaxf(x1.x, x1.y);
        const float m34 = fmaxf(x0.w, x1.x), m56 = fmaxf(x1.y, x1.z);
        mq[0] = fmaxf(fmaxf(x0.x, m12), fmaxf(x0.w, x1.x));
        mq[1] = fmaxf(fmaxf(m12, m34), x1.y);
        mq[2] = fmaxf(fmaxf(m23, m45), x1.z);
        mq[3] = fmaxf(fmaxf(m34, m56), x1.w);
      } else if (eps <= 6) {
        float w[16];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const float4 x = *reinterpret_cast<const float4*>(&sm.sv[t + 4 * c]);
          w[4 * c] = x.x; w[4 * c + 1] = x.y; w[4 * c + 2] = x.z; w[4 * c + 3] = x.w;
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          mq[q] = w[q];
#pragma unroll
          for (int o = 1; o <= 12; ++o)
            if (o <= 2 * eps) mq[q] = fmaxf(mq[q], w[q + o]);
        }
      } else {
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float m = sm.sv[t + q];
          for (int o = 1; o <= 2 * eps; ++o) m = fmaxf(m, sm.sv[t + q + o]);
          mq[q] = m;
        }
      }
      uint4 k4;
      k4.x = order_key(mq[0]); k4.y = order_key(mq[1]); k4.z = order_key(mq[2]); k4.w = order_key(mq[3]);
      *reinterpret_cast<uint4*>(&ub[t0 + t]) = k4;   // slots past nt hold junk that is never read as a key
      const uint32_t kq[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (t + q < nt) {
          if (a.s_prime_out) a.s_prime_out[(int64_t)b * a.n_mid + j0 + t0 + t + q] = mq[q];
          atomicAdd(&sm.hist[kq[q] >> 21], 1u);
        }
      }
    }
    __syncthreads();
  }

  // ---- three radix levels, histograms merged slice by slice across the cluster
  cluster_wait();                          // every CTA's merged slices are cleared
  uint32_t prefix = 0, want = (uint32_t)kk;
  for (int level = 0; level < 3; ++level) {
    const int bits = level == 2 ? 10 : 11;
    const int nb = 1 << bits;
    if (level > 0) {
      const int shift = level == 1 ? 10 : 0;
      const int hi_shift = level == 1 ? 21 : 10;
      for (int t = tid; t < nb; t += kSelThreads) sm.hist[t] = 0;
      __syncthreads();
      for (int t = 4 * tid; t < nloc; t += 4 * kSelThreads) {
        const uint4 k4 = *reinterpret_cast<const uint4*>(&ub[t]);
        const uint32_t kq[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (t + q < nloc && (kq[q] >> hi_shift) == prefix)
            atomicAdd(&sm.hist[(kq[q] >> shift) & (uint32_t)(nb - 1)], 1u);
      }
      __syncthreads();
    }
    // levels of 2048, 2048 and 1024 bins, one after the other; bin t lives in CTA t / slice
    const int slice = nb / CL;
    const uint32_t merged = smem_u32(&sm.merged[level * kSelBins]);
    for (int t = tid; t < nb; t += kSelThreads) {
      const uint32_t c = sm.hist[t];
      if (c) red_dsmem_add_u32(dsmem_map(merged + 4u * t, (uint32_t)(t / slice)), c);
    }
    cluster_sync_all();                    // every slice holds its merged counts
    // thread tid owns the bins of descending rank tid * per_t + q, i.e. the per_t
    // consecutive bins ending at nb - 1 - tid * per_t: one vector load from their owner
    const int per_t = nb / kSelThreads;
    uint32_t c[kSelBins / kSelThreads];
    {
      const int lo_bin = nb - per_t * (tid + 1);
      const uint32_t src = dsmem_map(merged + 4u * lo_bin, (uint32_t)(lo_bin / slice));
      if (per_t == 4) {
        const uint4 v4 = ld_dsmem_u4(src);
        c[0] = v4.w; c[1] = v4.z; c[2] = v4.y; c[3] = v4.x;
      } else {
        const uint2 v2 = ld_dsmem_u2(src);
        c[0] = v2.y; c[1] = v2.x; c[2] = 0u; c[3] = 0u;
      }
    }
    uint32_t sum = 0;
#pragma unroll
    for (int q = 0; q < kSelBins / kSelThreads; ++q) sum += c[q];
    uint32_t before;
    Scan(sm.scan).ExclusiveSum(sum, before);
    uint32_t acc = before;
#pragma unroll
    for (int q = 0; q < kSelBins / kSelThreads; ++q) {
      if (q < per_t && acc < want && acc + c[q] >= want) {
        sm.sel_bin = (uint32_t)(nb - 1 - (tid * per_t + q));
        sm.sel_above = acc;
      }
      acc += c[q];
    }
    __syncthreads();
    prefix = (prefix << bits) | sm.sel_bin;
    want -= sm.sel_above;
    __syncthreads();
  }
  const uint32_t T = prefix;

  // ---- ordered compaction: keep key > T, and key == T while fewer than `want` equal
  //      keys at lower positions were kept. Thread tid owns the contiguous run
  //      [tid * R, tid * R + R) of this CTA's positions; R is 4 x an odd number, so the
  //      16-byte loads of a quarter-warp fall in distinct bank groups.
  const int R = 4 * ((((nloc + kSelThreads - 1) / kSelThreads + 3) / 4) | 1);
  const int r0 = min(nloc, tid * R), r1 = min(nloc, r0 + R);
  uint32_t gt = 0, eq = 0;
  for (int t = r0; t < r1; t += 4) {
    const uint4 k4 = *reinterpret_cast<const uint4*>(&ub[t]);
    const uint32_t kq[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (t + q < r1) {
        gt += kq[q] > T;
        eq += kq[q] == T;
      }
    }
  }
  uint32_t eq_before, eq_total, gt_before, gt_total;
  Scan(sm.scan).ExclusiveSum(eq, eq_before, eq_total);
  __syncthreads();
  Scan(sm.scan).ExclusiveSum(gt, gt_before, gt_total);
  // push this CTA's totals to every higher rank; after the barrier nothing in the
  // cluster touches another CTA's shared memory, so each CTA may then finish alone
  if ((uint32_t)tid > rank && tid < CL) {
    st_dsmem_u32(dsmem_map(smem_u32(&sm.cnt_lo[rank][0]), (uint32_t)tid), gt_total);
    st_dsmem_u32(dsmem_map(smem_u32(&sm.cnt_lo[rank][1]), (uint32_t)tid), eq_total);
  }
  cluster_sync_all();
  uint32_t bg = 0, be = 0;
  for (uint32_t r = 0; r < rank; ++r) {
    bg += sm.cnt_lo[r][0];
    be += sm.cnt_lo[r][1];
  }
  const uint32_t base_gt = bg, base_eq = be;
  uint32_t eq_run = base_eq + eq_before;
  uint32_t keep_n = 0;
  for (int t = r0; t < r1; t += 4) {
    const uint4 k4 = *reinterpret_cast<const uint4*>(&ub[t]);
    const uint32_t kq[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (t + q >= r1) break;
      if (kq[q] > T) ++keep_n;
      else if (kq[q] == T) { keep_n += eq_run < want; ++eq_run; }
    }
  }
  uint32_t pos;
  Scan(sm.scan).ExclusiveSum(keep_n, pos);
  pos += base_gt + min(base_eq, want);
  eq_run = base_eq + eq_before;
  int32_t* out = a.idx + (int64_t)b * a.topk;
  for (int t = r0; t < r1; t += 4) {
    const uint4 k4 = *reinterpret_cast<const uint4*>(&ub[t]);
    const uint32_t kq[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (t + q >= r1) break;
      bool keep = kq[q] > T;
      if (kq[q] == T) { keep = eq_run < want; ++eq_run; }
      if (keep) {
        if (pos < (uint32_t)a.topk) out[pos] = (int32_t)(a.mid0 + j0 + t + q);
        ++pos;
      }
    }
  }
  if (rank == 0) {
    for (int t = kk + tid; t < a.topk; t += kSelThreads) out[t] = -1;
    if (tid == 0) a.count[b] = kk;
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
