// cca.cuh - CCA-style attention (CCA-Attention article: global-aware pooling,
// locality-preserving module, fusion of the two).
//
//   pooling  group j of g tokens -> core key and value: the group's keys and values
//            weighted by the softmax (scale 1/sqrt(D)) of the group's last query
//            against the group's keys, per query head (head h pools KV head h / G)
//   window   query i sees the tokens [lo_i, i], lo_i = max(0, g floor(i / g) - w)
//   fusion   one softmax over the core tokens of the groups that end before lo_i and
//            the window's tokens
//
// Three launches. cca_pool_kernel writes the core keys and values [B, S / g, Hq, D]
// (bf16), one warp per (sequence, group, KV head): the warp streams the group's key
// and value rows once for the G query heads it serves, keeping an online softmax per
// head. The attention runs on the tensor cores (attn_tc_kernel) in two passes over
// tiles of 128 consecutive queries of one head. With g a multiple of 128 a tile lies in
// one group, so all its rows share the window start and the number of core tokens:
// the first pass (CcaCoreProblem) attends the core tokens, a contiguous run of the core
// buffer, and writes a normalised bf16 partial with its base-2 log-sum-exp; the second
// (CcaWindowProblem) attends the window, consecutive rows of the cache cut causally,
// and its epilogue merges the partial and writes the output.
#pragma once
#include "attn_tc.cuh"
#include "common.cuh"

namespace esa {

constexpr int kCcaPoolWarps = 4;

// grid (cdiv(B * m * Hkv, kCcaPoolWarps)), kCcaPoolWarps * 32 threads; D = 128.
template <int G>
__global__ void __launch_bounds__(kCcaPoolWarps * 32)
    cca_pool_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                    const __nv_bfloat16* __restrict__ v, int batch, int64_t seq, int hkv, int group, int64_t m,
                    float scale_log2, __nv_bfloat16* __restrict__ kc, __nv_bfloat16* __restrict__ vc) {
  constexpr int D = 128;
  const int lane = threadIdx.x & 31;
  const int64_t item = (int64_t)blockIdx.x * kCcaPoolWarps + (threadIdx.x >> 5);   // (b, j, kvh)
  if (item >= (int64_t)batch * m * hkv) return;
  const int kvh = (int)(item % hkv);
  const int64_t j = (item / hkv) % m;
  const int b = (int)(item / ((int64_t)hkv * m));
  const int hq = hkv * G;
  const int64_t t0 = j * group;
  const int64_t last = t0 + group - 1;

  float qv[G][4];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const __nv_bfloat16* qp = q + (((int64_t)b * seq + last) * hq + kvh * G + hh) * D + lane * 4;
    const uint2 u = *reinterpret_cast<const uint2*>(qp);
    const float2 a = bf16x2_to_float2(u.x), c = bf16x2_to_float2(u.y);
    qv[hh][0] = a.x * scale_log2; qv[hh][1] = a.y * scale_log2;
    qv[hh][2] = c.x * scale_log2; qv[hh][3] = c.y * scale_log2;
  }
  float mx[G], den[G], ak[G][4], av[G][4];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    mx[hh] = -INFINITY;
    den[hh] = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) ak[hh][e] = av[hh][e] = 0.f;
  }
  const int64_t row_stride = (int64_t)hkv * D;
  const __nv_bfloat16* kp = k + (((int64_t)b * seq + t0) * hkv + kvh) * D + lane * 4;
  const __nv_bfloat16* vp = v + (((int64_t)b * seq + t0) * hkv + kvh) * D + lane * 4;
  for (int t = 0; t < group; ++t) {
    const uint2 ku = __ldg(reinterpret_cast<const uint2*>(kp + t * row_stride));
    const uint2 vu = __ldg(reinterpret_cast<const uint2*>(vp + t * row_stride));
    const float2 k01 = bf16x2_to_float2(ku.x), k23 = bf16x2_to_float2(ku.y);
    const float2 v01 = bf16x2_to_float2(vu.x), v23 = bf16x2_to_float2(vu.y);
    const float kf[4] = {k01.x, k01.y, k23.x, k23.y};
    const float vf[4] = {v01.x, v01.y, v23.x, v23.y};
#pragma unroll
    for (int hh = 0; hh < G; ++hh) {
      float x = qv[hh][0] * kf[0];
      x = fmaf(qv[hh][1], kf[1], x);
      x = fmaf(qv[hh][2], kf[2], x);
      x = fmaf(qv[hh][3], kf[3], x);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
      const float mn = fmaxf(mx[hh], x);
      const float corr = exp2f(mx[hh] - mn);       // 0 on the first key (mx = -inf)
      const float p = exp2f(x - mn);
      den[hh] = den[hh] * corr + p;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ak[hh][e] = fmaf(p, kf[e], ak[hh][e] * corr);
        av[hh][e] = fmaf(p, vf[e], av[hh][e] * corr);
      }
      mx[hh] = mn;
    }
  }
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const float inv = 1.f / den[hh];
    const int64_t o = (((int64_t)b * m + j) * hq + kvh * G + hh) * D + lane * 4;
    uint2 ku, vu;
    ku.x = bf16x2_rn(ak[hh][0] * inv, ak[hh][1] * inv);
    ku.y = bf16x2_rn(ak[hh][2] * inv, ak[hh][3] * inv);
    vu.x = bf16x2_rn(av[hh][0] * inv, av[hh][1] * inv);
    vu.y = bf16x2_rn(av[hh][2] * inv, av[hh][3] * inv);
    *reinterpret_cast<uint2*>(kc + o) = ku;
    *reinterpret_cast<uint2*>(vc + o) = vu;
  }
}

// Tiles: grid (cdiv(seq, 128), Hq, B); rows = 128 consecutive queries of head h.
struct CcaTile {
  int64_t seq, m;
  int hq, hkv, G, group, window;
  float sl2;
  int b, h;
  int64_t p0, nrows, lo, n_core;

  __device__ bool setup_tile() {
    b = blockIdx.z;
    h = blockIdx.y;
    p0 = (int64_t)blockIdx.x * kTcRows;
    if (p0 >= seq) return false;
    nrows = min((int64_t)kTcRows, seq - p0);
    const int64_t start = (p0 / group) * group - window;     // the tile lies in one group
    lo = start > 0 ? start : 0;
    n_core = lo / group;
    return true;
  }
  __device__ int32_t q_row(int r) const {
    if (r >= nrows) return -1;
    return (int32_t)(((int64_t)b * seq + p0 + r) * hq + h);
  }
  __device__ bool q_box(int* y, int* z) const {
    *y = h;
    *z = (int)((int64_t)b * seq + p0);
    return true;
  }
  __device__ float scale_log2() const { return sl2; }
};

// Pass 1: the core tokens [0, n_core) of the tile's rows (staged maps = core buffers).
// Partials: part_o [B, seq, Hq, D] bf16 (normalised), part_lse [B, seq, Hq] fp32, base 2.
struct CcaCoreProblem : CcaTile {
  __nv_bfloat16* part_o;
  float* part_lse;

  __device__ bool setup() { return setup_tile() && n_core > 0; }
  __device__ int64_t n_keys() const { return n_core; }
  __device__ int32_t kv_row(int64_t) const { return (int32_t)((int64_t)b * seq * hkv); }   // never gathered
  __device__ int kv_box(int j, int* y, int* z) const {
    *y = h;
    *z = (int)((int64_t)b * m + (int64_t)j * kTcKeys);
    return 2;
  }
  __device__ int64_t limit(int) const { return n_core - 1; }
  __device__ void store(int r, int col0, const float* acc, float m2, float l) {
    constexpr int HC = kTcD / kTcSplit;
    if (r >= nrows) return;
    const int64_t row = ((int64_t)b * seq + p0 + r) * hq + h;
    const float inv = 1.f / l;
    uint4* dst = reinterpret_cast<uint4*>(part_o + row * kTcD + col0);
#pragma unroll
    for (int c = 0; c < HC / 8; ++c) {
      uint4 u;
      u.x = bf16x2_rn(acc[8 * c] * inv, acc[8 * c + 1] * inv);
      u.y = bf16x2_rn(acc[8 * c + 2] * inv, acc[8 * c + 3] * inv);
      u.z = bf16x2_rn(acc[8 * c + 4] * inv, acc[8 * c + 5] * inv);
      u.w = bf16x2_rn(acc[8 * c + 6] * inv, acc[8 * c + 7] * inv);
      dst[c] = u;
    }
    if (col0 == 0) part_lse[row] = m2 + __log2f(l);
  }
};

// Pass 2: the window [lo, p0 + r] of row r, merged with pass 1's partial.
struct CcaWindowProblem : CcaTile {
  const __nv_bfloat16* part_o;
  const float* part_lse;
  __nv_bfloat16* o;      // [B, seq, Hq, D]
  float* lse;            // [B, seq, Hq] or null

  __device__ bool setup() { return setup_tile(); }
  __device__ int64_t n_keys() const { return p0 + nrows - lo; }
  __device__ int32_t kv_row(int64_t t) const { return (int32_t)(((int64_t)b * seq + lo + t) * hkv + h / G); }
  __device__ int kv_box(int j, int* y, int* z) const {
    *y = h / G;
    *z = (int)((int64_t)b * seq + lo + (int64_t)j * kTcKeys);
    return 1;
  }
  __device__ int64_t limit(int r) const { return p0 + min((int64_t)r, nrows - 1) - lo; }
  __device__ void store(int r, int col0, const float* acc, float m2, float l) {
    constexpr int HC = kTcD / kTcSplit;
    if (r >= nrows) return;
    const int64_t row = ((int64_t)b * seq + p0 + r) * hq + h;
    const float lw = m2 + __log2f(l);
    float M = lw, lp = -INFINITY;
    if (n_core > 0) {
      lp = __ldg(part_lse + row);
      M = fmaxf(M, lp);
    }
    const float ww = exp2f(lw - M);
    const float wp = n_core > 0 ? exp2f(lp - M) : 0.f;
    const float L = ww + wp;
    float out[HC];
    const float cw = ww / l;
#pragma unroll
    for (int c = 0; c < HC; ++c) out[c] = acc[c] * cw;
    if (n_core > 0) {
      const uint4* src = reinterpret_cast<const uint4*>(part_o + row * kTcD + col0);
#pragma unroll
      for (int c = 0; c < HC / 8; ++c) {
        const uint4 u = __ldg(src + c);
        const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = bf16x2_to_float2(wd[e]);
          out[8 * c + 2 * e] = fmaf(wp, f.x, out[8 * c + 2 * e]);
          out[8 * c + 2 * e + 1] = fmaf(wp, f.y, out[8 * c + 2 * e + 1]);
        }
      }
    }
    const float inv = 1.f / L;
    uint4* dst = reinterpret_cast<uint4*>(o + row * kTcD + col0);
#pragma unroll
    for (int c = 0; c < HC / 8; ++c) {
      uint4 u;
      u.x = bf16x2_rn(out[8 * c] * inv, out[8 * c + 1] * inv);
      u.y = bf16x2_rn(out[8 * c + 2] * inv, out[8 * c + 3] * inv);
      u.z = bf16x2_rn(out[8 * c + 4] * inv, out[8 * c + 5] * inv);
      u.w = bf16x2_rn(out[8 * c + 6] * inv, out[8 * c + 7] * inv);
      dst[c] = u;
    }
    if (col0 == 0 && lse) lse[row] = (M + __log2f(L)) * 0.69314718055994531f;
  }
};

}  // namespace esa
