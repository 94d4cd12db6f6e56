// score.cuh - importance score of every middle token against the chunk's compressed
// queries, per-query max correction with clamp, and the sum over the chunk
// (ESA write-up: implementation paragraph - importance is the merged-head q.k dot
// product summed over the current chunk's queries; score-correction paragraph -
// each query's scores are shifted by its maximum and bounded below by -C).
//
//   S_ij = q_c[i] . k_c[mid0 + j]           (fp32)
//   m_i  = max_j S_ij                       (atomicMax on order keys: order-independent)
// The kernels here store S and m; the selection kernel (topk.cuh) forms
//   s_j  = sum_i max(S_ij - m_i, -C)        (fixed order i = 0, 1, ...)
// as it reads them.
#pragma once
#include "common.cuh"

namespace esa {

// ------------------------------------------------------------ few queries (decode) --
// One group of LPK lanes holds one key (VPL floats per lane); a warp covers KPW keys
// per step and UNR steps per iteration. Lq <= kScoreSmallLq queries live in registers.
constexpr int kScoreSmallLq = 8;

template <int DC>
struct SmallScoreShape {
  static constexpr int VPL = DC >= 128 ? DC / 32 : 4;
  static constexpr int LPK = DC / VPL;
  static constexpr int KPW = 32 / LPK;
};

template <int DC, int LQ>
__global__ void __launch_bounds__(256) score_small_kernel(const float* __restrict__ q_c, const float* __restrict__ k_c,
                                                          int lq, int64_t n_cap, int64_t mid0, int64_t n_mid,
                                                          int64_t keys_per_cta, float* __restrict__ s_out,
                                                          uint32_t* __restrict__ m_key) {
  using Sh = SmallScoreShape<DC>;
  constexpr int VPL = Sh::VPL, LPK = Sh::LPK, KPW = Sh::KPW;
  constexpr int UNR = 4;
  const int b = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarp = blockDim.x >> 5;
  const int grp = lane / LPK, sub = lane % LPK;
  const float* kb = k_c + ((int64_t)b * n_cap + mid0) * DC;
  float q[LQ][VPL];
#pragma unroll
  for (int i = 0; i < LQ; ++i)
#pragma unroll
    for (int v = 0; v < VPL; v += 4) {
      if (i < lq) load_vec(q_c + ((int64_t)b * lq + i) * DC + sub * VPL + v, &q[i][v]);
      else q[i][v] = q[i][v + 1] = q[i][v + 2] = q[i][v + 3] = 0.f;
    }
  float mx[LQ];
#pragma unroll
  for (int i = 0; i < LQ; ++i) mx[i] = -INFINITY;

  const int64_t j_begin = (int64_t)blockIdx.x * keys_per_cta;
  const int64_t j_end = min(n_mid, j_begin + keys_per_cta);
  for (int64_t jb = j_begin + (int64_t)warp * KPW * UNR; jb < j_end; jb += (int64_t)nwarp * KPW * UNR) {
    float kv[UNR][VPL];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int64_t j = jb + u * KPW + grp;
      if (j < j_end) {
#pragma unroll
        for (int v = 0; v < VPL; v += 4) {
          uint4 raw = ld_stream16(kb + j * DC + sub * VPL + v);
          widen(raw, (const float*)nullptr, &kv[u][v]);
        }
      } else {
#pragma unroll
        for (int v = 0; v < VPL; ++v) kv[u][v] = 0.f;
      }
    }
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int64_t j = jb + u * KPW + grp;
#pragma unroll
      for (int i = 0; i < LQ; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int v = 0; v < VPL; ++v) acc = fmaf(q[i][v], kv[u][v], acc);
#pragma unroll
        for (int o = LPK / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (j < j_end && i < lq) {
          mx[i] = fmaxf(mx[i], acc);
          if (sub == 0) s_out[((int64_t)b * lq + i) * n_mid + j] = acc;
        }
      }
    }
  }
  __shared__ float red[LQ][32];
#pragma unroll
  for (int i = 0; i < LQ; ++i) {
    float v = warp_max(mx[i]);
    if (lane == 0) red[i][warp] = v;
  }
  __syncthreads();
  if (threadIdx.x < lq) {
    float v = -INFINITY;
    for (int w = 0; w < nwarp; ++w) v = fmaxf(v, red[threadIdx.x][w]);
    if (v > -INFINITY) atomicMax(&m_key[b * lq + threadIdx.x], order_key(v));
  }
}

// ------------------------------------------------------------ many queries (prefill) --
// Plain SIMT tile: 64 queries x 64 keys per CTA, reduction over d_c in slices of 16.
// Writes S and folds the tile's row maxima into m_key.
constexpr int kScT = 64;
constexpr int kScK = 16;

__global__ void __launch_bounds__(256) score_tiled_kernel(const float* __restrict__ q_c, const float* __restrict__ k_c,
                                                          int lq, int64_t n_cap, int64_t mid0, int64_t n_mid, int dc,
                                                          float* __restrict__ s_out, uint32_t* __restrict__ m_key) {
  __shared__ float qs[kScK][kScT + 4];
  __shared__ float ks[kScK][kScT + 4];
  __shared__ float rmax[kScT][17];
  const int b = blockIdx.z;
  const int i0 = blockIdx.y * kScT;
  const int64_t j0 = (int64_t)blockIdx.x * kScT;
  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;   // 16 x 16 threads, 4 x 4 outputs each
  float acc[4][4] = {};
  const float* qb = q_c + (int64_t)b * lq * dc;
  const float* kb = k_c + ((int64_t)b * n_cap + mid0) * dc;
  for (int d0 = 0; d0 < dc; d0 += kScK) {
    for (int t = tid; t < kScT * kScK; t += 256) {
      const int r = t / kScK, c = t % kScK;
      qs[c][r] = (i0 + r < lq) ? qb[(int64_t)(i0 + r) * dc + d0 + c] : 0.f;
      ks[c][r] = (j0 + r < n_mid) ? kb[(j0 + r) * dc + d0 + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int c = 0; c < kScK; ++c) {
      float a[4], bb[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) { a[u] = qs[c][ty * 4 + u]; bb[u] = ks[c][tx * 4 + u]; }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], bb[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = i0 + ty * 4 + u;
    float m = -INFINITY;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int64_t j = j0 + tx * 4 + v;
      if (i < lq && j < n_mid) {
        s_out[((int64_t)b * lq + i) * n_mid + j] = acc[u][v];
        m = fmaxf(m, acc[u][v]);
      }
    }
    rmax[ty * 4 + u][tx] = m;
  }
  __syncthreads();
  if (tid < kScT && i0 + tid < lq) {
    float m = -INFINITY;
    for (int x = 0; x < 16; ++x) m = fmaxf(m, rmax[tid][x]);
    if (m > -INFINITY) atomicMax(&m_key[b * lq + i0 + tid], order_key(m));
  }
}

}  // namespace esa
