// compress.cuh - one-layer linear map of the merged heads (ESA write-up, core steps:
// q and k pass through a one-layer MLP that shrinks 4096 to 128).
//
//   y[r, c] = sum_{h < Hout} sum_{e < D} x[r, h / G, e] * W[h * D + e, c]
//   (row r of x starts at r * xstride elements)
//
// fp32 FMA, fp32 accumulate. A CTA owns RT rows x CT output columns and walks the
// Hout * D reduction in slices of KC, staging the x slice and the W slice in shared
// memory. Each thread accumulates one output column for RPT rows.
#pragma once
#include "common.cuh"

namespace esa {

constexpr int kCmpRT = 16;   // rows per CTA
constexpr int kCmpKC = 64;   // reduction slice (elements of one head's row)
constexpr int kCmpThreads = 128;

// CT output columns per CTA (16 or 32). Thread map: column c = tid % CT, row group
// rg = tid / CT, each group RPT consecutive rows.
template <typename T, int CT>
__global__ void __launch_bounds__(kCmpThreads) compress_kernel(const T* __restrict__ x, int64_t rows,
                                                               int64_t xstride, int hin,
                                                               int hout, int d, const float* __restrict__ w,
                                                               int dout, float* __restrict__ y, int64_t ystride) {
  constexpr int RPT = kCmpRT * CT / kCmpThreads;
  __shared__ float xs[kCmpRT][kCmpKC + 1];
  __shared__ float ws[kCmpKC][CT];
  const int tid = threadIdx.x;
  const int64_t r0 = (int64_t)blockIdx.x * kCmpRT;
  const int c0 = blockIdx.y * CT;
  const int g = hout / hin;
  const int col = tid % CT;
  const int rg = tid / CT;
  float acc[RPT];
#pragma unroll
  for (int i = 0; i < RPT; ++i) acc[i] = 0.f;

  for (int h = 0; h < hout; ++h) {
    const int hi = h / g;
    for (int e0 = 0; e0 < d; e0 += kCmpKC) {
      // x slice: RT rows x KC elements of input head hi
      for (int t = tid; t < kCmpRT * kCmpKC; t += kCmpThreads) {
        const int rr = t / kCmpKC, ee = t % kCmpKC;
        const int64_t r = r0 + rr;
        float v = 0.f;
        if (r < rows) v = static_cast<float>(x[r * xstride + (int64_t)hi * d + e0 + ee]);
        xs[rr][ee] = v;
      }
      // W slice: KC reduction rows x CT columns
      for (int t = tid; t < kCmpKC * CT; t += kCmpThreads) {
        const int kk = t / CT, cc = t % CT;
        ws[kk][cc] = __ldg(&w[(int64_t)(h * d + e0 + kk) * dout + c0 + cc]);
      }
      __syncthreads();
#pragma unroll 8
      for (int kk = 0; kk < kCmpKC; ++kk) {
        const float wv = ws[kk][col];
#pragma unroll
        for (int i = 0; i < RPT; ++i) acc[i] = fmaf(xs[rg * RPT + i][kk], wv, acc[i]);
      }
      __syncthreads();
    }
  }
#pragma unroll
  for (int i = 0; i < RPT; ++i) {
    const int64_t r = r0 + rg * RPT + i;
    if (r < rows) y[r * ystride + c0 + col] = acc[i];
  }
}

}  // namespace esa
