// attn_simt.cuh - exact attention over initial + selected + local tokens for few
// queries (decode), memory-bound: 16-byte coalesced loads of the gathered K/V rows,
// fp32 math on CUDA cores, split over the key list and merged by log-sum-exp
// (ESA write-up: implementation and final-attention paragraphs - global part =
// initial + selected tokens, window part = local tokens, fused into one output).
//
// A CTA owns (sequence b, query i, KV head g, key split). All G = Hq / Hkv query heads
// of the group share each loaded K/V row. LPK lanes hold one key row (16 bytes each);
// a warp covers KPW rows per step. Online softmax in base 2 per key group; groups and
// warps are merged through shared memory at the end.
#pragma once
#include "common.cuh"
#include "keylist.cuh"

namespace esa {

struct SimtAttnArgs {
  const void* q;       // [B, Lq, Hq, D]
  const void* k;       // [B, n_cap, Hkv, D]
  const void* v;
  void* o;             // [B, Lq, Hq, D]
  float* lse;          // [B, Lq, Hq] or null
  float* part;         // [B, Lq, Hq, nsplit, D + 2] partials (nsplit > 1)
  KeyList keys;
  int64_t n_cap, c0;
  int lq, hq, hkv, nsplit;
  int lists;           // key lists per sequence: 1, or Hkv (one per KV head)
  int64_t keys_per_split;
  float scale_log2;    // scale * log2(e)
};

template <typename T, int D, int G>
struct SimtShape {
  static constexpr int VEC = 16 / sizeof(T);       // elements per 16-byte load
  static constexpr int LPK = D / VEC;              // lanes per key row
  static constexpr int KPW = 32 / LPK;             // key rows per warp step
};

constexpr int kSimtWarps = 4;

template <typename T, int D, int G>
__global__ void __launch_bounds__(kSimtWarps * 32) attn_simt_kernel(SimtAttnArgs a) {
  using Sh = SimtShape<T, D, G>;
  constexpr int VEC = Sh::VEC, LPK = Sh::LPK, KPW = Sh::KPW;
  constexpr int UNR = 2;
  const int split = blockIdx.x;
  const int g = blockIdx.y;
  const int b = blockIdx.z / a.lq;
  const int i = blockIdx.z % a.lq;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = lane / LPK, sub = lane % LPK;

  const int list = a.lists > 1 ? b * a.lists + g : b;
  KeyList kl = a.keys;
  const int64_t c0 = kl.vl.len ? kl.resolve(b, 703) : a.c0;
  const int cnt = min(max(kl.count[list], 0), (int)kl.idx_stride);
  const int64_t n_prior = kl.ni + cnt + (c0 - kl.lo);
  const int64_t n_keys = n_prior + i + 1;                     // causal: keys up to position c0 + i
  const int64_t t_begin = (int64_t)split * a.keys_per_split;
  const int64_t t_end = min(n_keys, t_begin + a.keys_per_split);

  const T* qp = reinterpret_cast<const T*>(a.q) + (((int64_t)b * a.lq + i) * a.hq + g * G) * D;
  float q[G][VEC];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    load_vec(qp + h * D + sub * VEC, q[h]);
#pragma unroll
    for (int e = 0; e < VEC; ++e) q[h][e] *= a.scale_log2;
  }
  float m[G], l[G], o[G][VEC];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < VEC; ++e) o[h][e] = 0.f;
  }
  const T* kbase = reinterpret_cast<const T*>(a.k) + ((int64_t)b * a.n_cap * a.hkv + g) * D + sub * VEC;
  const T* vbase = reinterpret_cast<const T*>(a.v) + ((int64_t)b * a.n_cap * a.hkv + g) * D + sub * VEC;
  const int64_t row_stride = (int64_t)a.hkv * D;

  for (int64_t tb = t_begin + (int64_t)warp * KPW * UNR; tb < t_end; tb += (int64_t)kSimtWarps * KPW * UNR) {
    uint4 kr[UNR], vr[UNR];
    bool ok[UNR];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      const int64_t t = tb + u * KPW + grp;
      ok[u] = t < t_end;
      if (ok[u]) {
        const int64_t p = kl.pos(list, cnt, t);
        kr[u] = ld_stream16(kbase + p * row_stride);
        vr[u] = ld_stream16(vbase + p * row_stride);
      }
    }
    float x[UNR][G];
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      float kf[VEC];
      widen(kr[u], (const T*)nullptr, kf);
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float acc = 0.f;
#pragma unroll
        for (int e = 0; e < VEC; ++e) acc = fmaf(q[h][e], kf[e], acc);
#pragma unroll
        for (int s = LPK / 2; s > 0; s >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, s);
        x[u][h] = ok[u] ? acc : -INFINITY;
      }
    }
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float mx = m[h];
#pragma unroll
      for (int u = 0; u < UNR; ++u) mx = fmaxf(mx, x[u][h]);
      if (mx == -INFINITY) continue;
      const float alpha = fast_exp2(m[h] - mx);
      m[h] = mx;
      l[h] *= alpha;
#pragma unroll
      for (int e = 0; e < VEC; ++e) o[h][e] *= alpha;
#pragma unroll
      for (int u = 0; u < UNR; ++u) {
        if (!ok[u]) continue;
        const float p = fast_exp2(x[u][h] - mx);
        l[h] += p;
        float vf[VEC];
        widen(vr[u], (const T*)nullptr, vf);
#pragma unroll
        for (int e = 0; e < VEC; ++e) o[h][e] = fmaf(p, vf[e], o[h][e]);
      }
    }
  }

  // merge the kSimtWarps * KPW key groups of this CTA
  constexpr int NGRP = kSimtWarps * KPW;
  __shared__ float sm_m[NGRP][G], sm_l[NGRP][G];
  __shared__ float sm_o[NGRP][G][D];
  const int gid = warp * KPW + grp;
#pragma unroll
  for (int h = 0; h < G; ++h) {
    if (sub == 0) { sm_m[gid][h] = m[h]; sm_l[gid][h] = l[h]; }
#pragma unroll
    for (int e = 0; e < VEC; ++e) sm_o[gid][h][sub * VEC + e] = o[h][e];
  }
  __syncthreads();
  for (int t = threadIdx.x; t < G * D; t += blockDim.x) {
    const int h = t / D, e = t % D;
    float M = -INFINITY;
    for (int r = 0; r < NGRP; ++r) M = fmaxf(M, sm_m[r][h]);
    float L = 0.f, O = 0.f;
    if (M > -INFINITY) {
      for (int r = 0; r < NGRP; ++r) {
        const float w = fast_exp2(sm_m[r][h] - M);
        L += sm_l[r][h] * w;
        O += sm_o[r][h][e] * w;
      }
    }
    const int hh = g * G + h;
    const int64_t row = ((int64_t)b * a.lq + i) * a.hq + hh;
    if (a.nsplit == 1) {
      reinterpret_cast<T*>(a.o)[row * D + e] = from_float<T>(O / L);
      if (e == 0 && a.lse) a.lse[row] = (M + __log2f(L)) * 0.69314718055994531f;
    } else {
      float* pp = a.part + (row * a.nsplit + split) * (D + 2);
      pp[e] = O;
      if (e == 0) { pp[D] = M; pp[D + 1] = L; }
    }
  }
}

// Merge the split partials of each (b, i, head) row by log-sum-exp. One warp per row.
template <typename T, int D>
__global__ void __launch_bounds__(256) attn_combine_kernel(const float* __restrict__ part, int64_t n_rows, int nsplit,
                                                           T* __restrict__ o, float* __restrict__ lse) {
  const int64_t row = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  const float* pr = part + row * nsplit * (D + 2);
  float M = -INFINITY;
  for (int s = 0; s < nsplit; ++s) M = fmaxf(M, pr[s * (D + 2) + D]);
  float L = 0.f;
  float acc[D / 32];
#pragma unroll
  for (int e = 0; e < D / 32; ++e) acc[e] = 0.f;
  for (int s = 0; s < nsplit; ++s) {
    const float ms = pr[s * (D + 2) + D];
    if (ms == -INFINITY) continue;
    const float w = fast_exp2(ms - M);
    L += pr[s * (D + 2) + D + 1] * w;
#pragma unroll
    for (int e = 0; e < D / 32; ++e) acc[e] += pr[s * (D + 2) + lane + 32 * e] * w;
  }
#pragma unroll
  for (int e = 0; e < D / 32; ++e) o[row * D + lane + 32 * e] = from_float<T>(acc[e] / L);
  if (lane == 0 && lse) lse[row] = (M + __log2f(L)) * 0.69314718055994531f;
}

}  // namespace esa
