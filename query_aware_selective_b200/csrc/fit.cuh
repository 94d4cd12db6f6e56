// fit.cuh - offline fit of ESA's two compression maps (ESA write-up, compression
// paragraph: the maps are learned offline from queries and keys kept from a calibration
// run, the model untouched; what matters is the relative size of the scores).
//
// The fit is least squares of the compressed scores against the merged-head scores over
// every (calibration query, calibration key) pair. With X [n, dq] the queries, Y [n, dk]
// the keys, E [dq, dk] the GQA expansion and Cholesky factors X^T X = Rq^T Rq,
// Y^T Y = Rk^T Rk, the best rank-d' score map is Rq^-1 (P_Q C) Rk^-T with
// C = Rq E Rk^T and P_Q the projector on C's leading d'-dimensional left singular
// subspace (Eckart-Young). With V the leading d' right singular vectors of C (P_Q C =
// C V V^T), W_q = Rq^-1 C V and the folded key map B = Rk^-1 V give exactly these
// scores (the expanded key map is E B / G); V is found as the leading eigenvectors of
// A = C^T C by subspace iteration with l = d' + oversampling columns and a
// Rayleigh-Ritz step (the l x l projected problem solved by the cyclic Jacobi method).
//
// Kernels:
//   gram_kernel     X^T X on the tensor cores (tcgen05 kind::f16, bf16 inputs, fp32 in
//                   TMEM): one CTA per 128 x 128 tile of the upper triangle (and a slice
//                   of the rows n), both operands MN-major straight from the TMA boxes
//   gram_finish     sum of the row slices (fp64) in a fixed order
//   gemm64          C = alpha op(A) op(B) + beta C in fp64 (any strides)
//   chol_block      Cholesky of one <= 160 x 160 diagonal block in shared memory (fp64)
//   trsm_block      triangular solve with one <= 160 x 160 upper block, many right sides
//                   (eight threads per right side)
//   jacobi_eig      eigenvectors of a symmetric <= 160 x 160 matrix (one CTA), the
//                   leading d' of them gathered in descending order of eigenvalue
//   small helpers   trace, diagonal shift, GQA fold of Rq's columns, key-map expansion
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace esa {

// ------------------------------------------------------------------ Gram (tensor) --
// The tensor cores sum kGmFlush * 128 rows at a time into one of two fp32 TMEM
// accumulators; sixteen epilogue warps drain each finished interval into fp64
// registers while the MMAs fill the other. A fit whitens the calibration tokens by the
// Cholesky factor of this matrix, so rounding errors in it are divided by its smallest
// eigenvalues: fp32 sums over all n rows (n / 16 roundings per entry) are not accurate
// enough, fp64 sums of 256-row fp32 intervals are.
constexpr int kGmRows = 128;                          // rows of X per stage (the K of the MMAs)
constexpr int kGmStages = 3;
constexpr int kGmFlush = 2;                           // stages per fp32 interval
constexpr uint32_t kGmTile = 128 * 256;               // 128 rows x 128 bf16 columns
constexpr uint32_t kGmBlk = 128 * 128;                // one 64-column block of a tile
constexpr int kGmEpiWarps = 16;                       // warp w: TMEM lanes 32 (w % 4), columns 32 (w / 4)
constexpr int kGmMmaWarp = kGmEpiWarps, kGmTmaWarp = kGmEpiWarps + 1;
constexpr int kGmThreads = (kGmEpiWarps + 2) * 32;
constexpr uint32_t kGmCtrl = 1024;
constexpr uint32_t kGmSmem = kGmStages * 2 * kGmTile + kGmCtrl;
static_assert(kGmSmem <= 232448, "exceeds the shared memory of a CTA");

struct GramArgs {
  int dim;                 // columns of X (a multiple of 128)
  int tiles;               // dim / 128
  int64_t n;               // rows of X
  int64_t rows_per_split;  // a multiple of 128
  double* part;            // [splits, dim, dim] fp64
};

struct GmSmem {
  uint64_t full[kGmStages], empty[kGmStages], acc_full[2], acc_empty[2], done;
  uint32_t tmem_base;
  int abort_flag;
};

// grid (tiles * (tiles + 1) / 2, splits): tile (I, J), I <= J, of slice blockIdx.y.
// D[i, j] = sum over the slice's rows r of X[r, 128 I + i] X[r, 128 J + j]: A = X^T and
// B = X, both with the 128 columns contiguous (MN-major); K steps of 16 rows.
__global__ void __launch_bounds__(kGmThreads, 1) gram_kernel(const __grid_constant__ CUtensorMap tm_x, GramArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_u32(smem_raw) & 1023u) {
    if (threadIdx.x == 0) record_status(5u, 600);
    return;
  }
  const uint32_t s0 = smem_u32(smem_raw);
  GmSmem& sm = *reinterpret_cast<GmSmem*>(smem_raw + kGmStages * 2 * kGmTile);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int t = blockIdx.x, I = 0;
  while (t >= a.tiles - I) {
    t -= a.tiles - I;
    ++I;
  }
  const int J = I + t;
  const bool diag = I == J;
  const int64_t r0 = (int64_t)blockIdx.y * a.rows_per_split;
  const int64_t r1 = min(a.n, r0 + a.rows_per_split);
  const int nk = r1 > r0 ? (int)((r1 - r0 + kGmRows - 1) / kGmRows) : 0;
  const int nu = (nk + kGmFlush - 1) / kGmFlush;    // fp32 intervals

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGmStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.acc_full[b], 1);
      mbar_init(&sm.acc_empty[b], kGmEpiWarps);
    }
    mbar_init(&sm.done, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kGmMmaWarp) {
    tmem_alloc(&sm.tmem_base, 256);                   // two 128-column accumulators
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == kGmTmaWarp) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint32_t bytes = diag ? kGmTile : 2 * kGmTile;
      for (int k = 0; k < nk; ++k) {
        const int s = k % kGmStages;
        if (!mbar_wait(&sm.empty[s], ((k / kGmStages) & 1) ^ 1, abort_flag, 601)) break;
        const int32_t y = (int32_t)(r0 + (int64_t)k * kGmRows);
        const uint32_t sa = s0 + s * 2 * kGmTile, sb = sa + kGmTile;
        mbar_arrive_expect_tx(&sm.full[s], bytes);
        tma_load_2d(sa, &tm_x, I * 128, y, &sm.full[s]);
        tma_load_2d(sa + kGmBlk, &tm_x, I * 128 + 64, y, &sm.full[s]);
        if (!diag) {
          tma_load_2d(sb, &tm_x, J * 128, y, &sm.full[s]);
          tma_load_2d(sb + kGmBlk, &tm_x, J * 128 + 64, y, &sm.full[s]);
        }
      }
    }
    __syncwarp();
  } else if (warp == kGmMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = umma_idesc(kFmtBF16, 128, 128, 1, 1);
      bool ok = true;
      for (int k = 0; k < nk && ok; ++k) {
        const int s = k % kGmStages, u = k / kGmFlush, b = u & 1;
        const bool first = k % kGmFlush == 0, last = k % kGmFlush == kGmFlush - 1 || k == nk - 1;
        // an interval's accumulator was drained by the epilogue two intervals ago
        if (first && u >= 2 && !(ok = mbar_wait(&sm.acc_empty[b], ((u >> 1) - 1) & 1, abort_flag, 605))) break;
        if (!(ok = mbar_wait(&sm.full[s], (k / kGmStages) & 1, abort_flag, 602))) break;
        tc_fence_after();
        const uint32_t sa = s0 + s * 2 * kGmTile, sb = diag ? sa : sa + kGmTile;
        // MN-major: 64-column blocks 16 KB apart (LBO), 8-row groups of 1024 bytes (SBO);
        // K step kk (16 rows) is +2048 bytes
        const uint64_t da = sdesc_sw128(sa, kGmBlk, 1024), db = sdesc_sw128(sb, kGmBlk, 1024);
        const uint32_t a_lo = (uint32_t)da, a_hi = (uint32_t)(da >> 32);
        const uint32_t b_lo = (uint32_t)db, b_hi = (uint32_t)(db >> 32);
        const uint32_t d = tmem + b * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          umma_f16_ss2(d, a_lo + kk * 128, a_hi, b_lo + kk * 128, b_hi, idesc, (!first || kk > 0) ? 1u : 0u);
        umma_commit(&sm.empty[s]);
        if (last) umma_commit(&sm.acc_full[b]);
      }
      umma_commit(&sm.done);           // arrives once every MMA issued above has completed
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (fp64 sums)
    const int quad = warp & 3, part = warp >> 2;
    const int row = quad * 32 + lane;                 // row i of the tile (TMEM lane)
    double acc[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) acc[e] = 0.0;
    bool ok = true;
    for (int u = 0; u < nu && ok; ++u) {
      const int b = u & 1;
      if (!(ok = mbar_wait_warp(&sm.acc_full[b], (u >> 1) & 1, abort_flag, 603))) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t v[8];
        tmem_ld8(tmem + ((uint32_t)(quad * 32) << 16) + b * 128 + part * 32 + c * 8, v);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[c * 8 + e] += (double)__uint_as_float(v[e]);
      }
      tc_fence_before();
      mbar_arrive_warp(&sm.acc_empty[b]);
    }
    if (ok) {
      double* base = a.part + (size_t)blockIdx.y * a.dim * a.dim;
      const int col0 = J * 128 + part * 32;
      double2* dst = reinterpret_cast<double2*>(base + (size_t)(I * 128 + row) * a.dim + col0);
#pragma unroll
      for (int e = 0; e < 16; ++e) dst[e] = make_double2(acc[2 * e], acc[2 * e + 1]);
      if (!diag) {
        // the mirrored tile (J, I): the warp's 32 lanes (consecutive rows here) write 32
        // consecutive entries of each mirrored row
#pragma unroll
        for (int e = 0; e < 32; ++e) base[(size_t)(col0 + e) * a.dim + I * 128 + row] = acc[e];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kGmMmaWarp) {
    // every MMA has completed before TMEM is released
    if (lane == 0) mbar_wait(&sm.done, 0, abort_flag, 604, /*respect_abort=*/false);
    __syncwarp();
    tmem_dealloc(tmem, 256);
  }
}

// G[i] = sum over s of part[s][i] (fixed order). grid-stride over dim * dim.
__global__ void gram_finish_kernel(const double* __restrict__ part, int splits, int64_t count,
                                   double* __restrict__ g) {
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x) {
    double acc = 0.0;
    for (int s = 0; s < splits; ++s) acc += part[(size_t)s * count + i];
    g[i] = acc;
  }
}

// Ridge: G += r * trace(G) / dim * I. One CTA.
__global__ void ridge_kernel(double* g, int dim, double r) {
  __shared__ double red[256];
  double t = 0.0;
  for (int i = threadIdx.x; i < dim; i += blockDim.x) t += g[(size_t)i * dim + i];
  red[threadIdx.x] = t;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  const double add = r * red[0] / dim;
  for (int i = threadIdx.x; i < dim; i += blockDim.x) g[(size_t)i * dim + i] += add;
}

// ------------------------------------------------------------------ fp64 GEMM --
// C[i, j] = alpha * sum_k A(i, k) B(k, j) + beta * C[i, j], A(i, k) = A[i * ar + k * ac],
// B(k, j) = B[k * br + j * bc], C[i, j] = C[i * ldc + j]. 64 x 64 tiles, 256 threads, a
// 4 x 4 block of C per thread, K in steps of 16 through shared memory.
constexpr int kG64Tile = 64, kG64K = 16;
__global__ void __launch_bounds__(256) gemm64_kernel(int m, int n, int k, double alpha, const double* __restrict__ A,
                                                     int64_t ar, int64_t ac, const double* __restrict__ B, int64_t br,
                                                     int64_t bc, double beta, double* __restrict__ C, int64_t ldc) {
  __shared__ double As[kG64K][kG64Tile + 1];
  __shared__ double Bs[kG64K][kG64Tile + 1];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  const int i0 = blockIdx.y * kG64Tile, j0 = blockIdx.x * kG64Tile;
  double acc[4][4] = {};
  for (int k0 = 0; k0 < k; k0 += kG64K) {
    // consecutive threads walk the operand's contiguous index (coalesced loads)
    const bool a_kc = ac <= ar, b_jc = bc <= br;
    for (int e = threadIdx.x; e < kG64K * kG64Tile; e += 256) {
      const int kk = a_kc ? e % kG64K : e / kG64Tile, ii = a_kc ? e / kG64K : e % kG64Tile;
      const int i = i0 + ii, kq = k0 + kk;
      As[kk][ii] = (i < m && kq < k) ? A[i * ar + kq * ac] : 0.0;
      const int kb = b_jc ? e / kG64Tile : e % kG64K, jj = b_jc ? e % kG64Tile : e / kG64K;
      const int j = j0 + jj, kr = k0 + kb;
      Bs[kb][jj] = (j < n && kr < k) ? B[kr * br + j * bc] : 0.0;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kG64K; ++kk) {
      double av[4], bv[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        av[q] = As[kk][ty + 16 * q];
        bv[q] = Bs[kk][tx + 16 * q];
      }
#pragma unroll
      for (int p = 0; p < 4; ++p)
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[p][q] = fma(av[p], bv[q], acc[p][q]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int p = 0; p < 4; ++p)
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int i = i0 + ty + 16 * p, j = j0 + tx + 16 * q;
      if (i < m && j < n) {
        double* c = C + (int64_t)i * ldc + j;
        *c = beta == 0.0 ? alpha * acc[p][q] : fma(alpha, acc[p][q], beta * *c);
      }
    }
}

// ------------------------------------------------------------------ Cholesky block --
// In place: the nb x nb block at A (row stride lda), symmetric positive definite,
// becomes its upper Cholesky factor R (A = R^T R; the strict lower part is zeroed). One
// CTA of 256 threads, the block in shared memory (nb <= 128). A pivot that is not
// positive (or not finite) records status 6 at `site` and stops the factorisation.
constexpr int kCholMax = 160;
constexpr uint32_t kCholSmem = kCholMax * (kCholMax + 1) * sizeof(double);
__global__ void __launch_bounds__(256) chol_block_kernel(double* A, int64_t lda, int nb, unsigned site) {
  extern __shared__ double cs[];                     // [nb][nb + 1]
  const int ld = nb + 1;
  for (int e = threadIdx.x; e < nb * nb; e += blockDim.x) cs[(e / nb) * ld + e % nb] = A[(e / nb) * lda + e % nb];
  __shared__ int bad;
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  for (int k = 0; k < nb; ++k) {
    const double d = cs[k * ld + k];
    if (!(d > 0.0) || !isfinite(d)) {
      if (threadIdx.x == 0) {
        bad = 1;
        record_status(6u, site);
      }
      break;                                          // every thread reads the same d
    }
    const double r = sqrt(d), inv = 1.0 / r;
    __syncthreads();                                  // all have read cs[k][k]
    for (int j = k + threadIdx.x; j < nb; j += blockDim.x) cs[k * ld + j] = j == k ? r : cs[k * ld + j] * inv;
    __syncthreads();
    // trailing update of the upper triangle: A[i][j] -= R[k][i] R[k][j], k < i <= j
    // (16 x 16 threads over (i, j), no division in the index arithmetic)
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    for (int i = k + 1 + ty; i < nb; i += 16) {
      const double rki = cs[k * ld + i];
      for (int j = i + tx; j < nb; j += 16) cs[i * ld + j] -= rki * cs[k * ld + j];
    }
    __syncthreads();
  }
  __syncthreads();
  if (bad) return;
  for (int e = threadIdx.x; e < nb * nb; e += blockDim.x) {
    const int i = e / nb, j = e % nb;
    A[i * lda + j] = j >= i ? cs[i * ld + j] : 0.0;
  }
}

// ------------------------------------------------------------------ triangular solve --
// Solves, for the ncols right sides x_c (element i of side c at X[i * xr + c * xc]), in
// place: trans = 1: R^T x = b (forward substitution), trans = 0: R x = b (back
// substitution), with R the nb x nb upper block at T (row stride ldt, nb <= 160).
// Eight threads of a warp share a right side: thread r holds rows r, r + 8, ... in
// registers; at step i the owner of row i forms x_i, a shuffle hands it to the other
// seven, and each updates its own rows. A CTA takes 32 right sides (256 threads); R is
// staged in shared memory when nb <= 128 (else read as broadcasts through L1).
constexpr int kTrsmCols = 32;
constexpr int kTrsmThreads = 8 * kTrsmCols;
constexpr int kTrsmRowsPer = kCholMax / 8;            // rows a thread holds (nb <= 160)
constexpr int kTrsmStageMax = 128;
constexpr uint32_t kTrsmSmem = kTrsmStageMax * kTrsmStageMax * sizeof(double);
__global__ void __launch_bounds__(kTrsmThreads, 1) trsm_block_kernel(const double* __restrict__ T, int64_t ldt, int nb,
                                                                    double* X, int64_t xr, int64_t xc, int64_t ncols,
                                                                    int trans) {
  extern __shared__ double tsm[];
  const bool staged = nb <= kTrsmStageMax;
  const double* tr = staged ? tsm : T;               // R, row stride tl
  const int64_t tl = staged ? nb : ldt;
  if (staged)
    for (int e = threadIdx.x; e < nb * nb; e += blockDim.x) tsm[e] = T[(e / nb) * ldt + e % nb];
  const int r = threadIdx.x & 7, lane = threadIdx.x & 31;
  const int src0 = lane & ~7;                        // lane of this side's thread 0
  const int64_t c = (int64_t)blockIdx.x * kTrsmCols + (threadIdx.x >> 3);
  const bool live = c < ncols;
  double b[kTrsmRowsPer];
#pragma unroll
  for (int t = 0; t < kTrsmRowsPer; ++t) {
    const int j = r + 8 * t;
    b[t] = (live && j < nb) ? X[j * xr + c * xc] : 0.0;
  }
  __syncthreads();
  if (trans) {
    for (int i = 0; i < nb; ++i) {
      double x = 0.0;
#pragma unroll
      for (int t = 0; t < kTrsmRowsPer; ++t)
        if (r + 8 * t == i) {
          b[t] = b[t] / tr[i * tl + i];
          x = b[t];
        }
      x = __shfl_sync(0xffffffffu, x, src0 + (i & 7));
#pragma unroll
      for (int t = 0; t < kTrsmRowsPer; ++t) {
        const int j = r + 8 * t;
        if (j > i && j < nb) b[t] -= tr[i * tl + j] * x;
      }
    }
  } else {
    for (int i = nb - 1; i >= 0; --i) {
      double x = 0.0;
#pragma unroll
      for (int t = 0; t < kTrsmRowsPer; ++t)
        if (r + 8 * t == i) {
          b[t] = b[t] / tr[i * tl + i];
          x = b[t];
        }
      x = __shfl_sync(0xffffffffu, x, src0 + (i & 7));
#pragma unroll
      for (int t = 0; t < kTrsmRowsPer; ++t) {
        const int j = r + 8 * t;
        if (j < i) b[t] -= tr[j * tl + i] * x;
      }
    }
  }
  if (live) {
#pragma unroll
    for (int t = 0; t < kTrsmRowsPer; ++t) {
      const int j = r + 8 * t;
      if (j < nb) X[j * xr + c * xc] = b[t];
    }
  }
}

// ------------------------------------------------------------------ Jacobi eigensolver --
// Eigenvectors of the symmetric l x l matrix H (row stride l, l <= 160) by the cyclic
// Jacobi method: each rotation in the (p, q) plane, J_pp = J_qq = c, J_pq = s,
// J_qp = -s with t = s / c the smaller root of t^2 + 2 t theta - 1 = 0,
// theta = (h_qq - h_pp) / (2 h_pq), zeroes h_pq (H <- J^T H J, Z <- Z J). A round
// rotates the L / 2 disjoint pairs of the round-robin (circle) schedule at once (the
// angles from the matrix before the round; disjoint rotations commute); L - 1 rounds
// are a sweep, and sweeps stop when the off-diagonal part is below 1e-14 of the whole.
// Output: zsel [l, d] = the eigenvectors of the d largest eigenvalues, as columns in
// descending order of eigenvalue (ties to the lower index). One CTA of 512 threads; H
// lives in shared memory, Z [L, L] (global scratch, stored transposed so that a
// rotation's two columns are contiguous) accumulates the rotations.
constexpr int kJacobiThreads = 512;
constexpr uint32_t kJacobiSmem = (kCholMax * (kCholMax + 1) + 4 * (kCholMax / 2) + kCholMax) * sizeof(double);
__global__ void __launch_bounds__(kJacobiThreads) jacobi_eig_kernel(const double* __restrict__ H, int l, double* Z,
                                                                       int d, double* __restrict__ zsel,
                                                                       int max_sweeps) {
  extern __shared__ double js[];
  const int L = l + (l & 1);                         // an odd size gets a decoupled zero row / column
  const int ld = L + 1;
  double* h = js;                                    // [L][L + 1]
  double* rc = h + L * ld;                           // c per pair
  double* rs = rc + L / 2;                           // s per pair
  int* rp = reinterpret_cast<int*>(rs + L / 2);      // p per pair
  int* rq = rp + L / 2;                              // q per pair
  double* red = rs + 3 * (L / 2);                    // [L] reductions
  for (int e = threadIdx.x; e < L * L; e += blockDim.x) {
    const int i = e / L, j = e % L;
    h[i * ld + j] = (i < l && j < l) ? H[i * l + j] : 0.0;
    Z[e] = i == j ? 1.0 : 0.0;                       // stored transposed: Z[p * L + i] = z_ip
  }
  __syncthreads();
  const int P = L / 2;
  for (int sweep = 0; sweep < max_sweeps; ++sweep) {
    // convergence: sum of squares off the diagonal against the whole
    double off = 0.0, all = 0.0;
    for (int e = threadIdx.x; e < L * L; e += blockDim.x) {
      const double v = h[(e / L) * ld + e % L];
      all += v * v;
      if (e / L != e % L) off += v * v;
    }
    __shared__ double s_off[kJacobiThreads], s_all[kJacobiThreads];
    s_off[threadIdx.x] = off;
    s_all[threadIdx.x] = all;
    __syncthreads();
    for (int w = kJacobiThreads / 2; w > 0; w >>= 1) {
      if (threadIdx.x < w) {
        s_off[threadIdx.x] += s_off[threadIdx.x + w];
        s_all[threadIdx.x] += s_all[threadIdx.x + w];
      }
      __syncthreads();
    }
    const bool done = !(s_off[0] > 1e-28 * s_all[0]);
    __syncthreads();
    if (done) break;
    for (int round = 0; round < L - 1; ++round) {
      if (threadIdx.x < P) {
        // circle method: L - 1 fixed, the others rotate
        const int k = threadIdx.x;
        int p, q;
        if (k == 0) {
          p = round;
          q = L - 1;
        } else {
          p = (round + k) % (L - 1);
          q = (round - k + (L - 1)) % (L - 1);
        }
        if (p > q) {
          const int tmp = p;
          p = q;
          q = tmp;
        }
        const double app = h[p * ld + p], aqq = h[q * ld + q], apq = h[p * ld + q];
        double c = 1.0, sn = 0.0;
        if (fabs(apq) > 1e-300) {
          const double theta = (aqq - app) / (2.0 * apq);
          const double t = fabs(theta) > 1e150 ? 0.5 / theta
                                               : (theta >= 0.0 ? 1.0 : -1.0) / (fabs(theta) + sqrt(theta * theta + 1.0));
          c = 1.0 / sqrt(t * t + 1.0);
          sn = t * c;
        }
        rc[k] = c;
        rs[k] = sn;
        rp[k] = p;
        rq[k] = q;
      }
      __syncthreads();
      for (int e = threadIdx.x; e < P * L; e += blockDim.x) {   // rows: H <- J^T H
        const int k = e / L, j = e % L;
        const int p = rp[k], q = rq[k];
        const double c = rc[k], sn = rs[k];
        const double hp = h[p * ld + j], hq = h[q * ld + j];
        h[p * ld + j] = c * hp - sn * hq;
        h[q * ld + j] = sn * hp + c * hq;
      }
      __syncthreads();
      for (int e = threadIdx.x; e < P * L; e += blockDim.x) {   // columns: H <- H J, Z <- Z J
        const int k = e / L, i = e % L;
        const int p = rp[k], q = rq[k];
        const double c = rc[k], sn = rs[k];
        const double hp = h[i * ld + p], hq = h[i * ld + q];
        h[i * ld + p] = c * hp - sn * hq;
        h[i * ld + q] = sn * hp + c * hq;
        const double zp = Z[(int64_t)p * L + i], zq = Z[(int64_t)q * L + i];
        Z[(int64_t)p * L + i] = c * zp - sn * zq;
        Z[(int64_t)q * L + i] = sn * zp + c * zq;
      }
      __syncthreads();
    }
  }
  // the d largest eigenvalues (ties to the lower index), their vectors in that order;
  // the padding index (l odd) is not a candidate
  for (int i = threadIdx.x; i < l; i += blockDim.x) red[i] = h[i * ld + i];
  __syncthreads();
  for (int i = threadIdx.x; i < l; i += blockDim.x) {
    int rank = 0;
    for (int j = 0; j < l; ++j) rank += (red[j] > red[i]) || (red[j] == red[i] && j < i);
    if (rank < d)
      for (int r = 0; r < l; ++r) zsel[r * d + rank] = Z[(int64_t)i * L + r];
  }
}

// ------------------------------------------------------------------ small helpers --
// Strict lower triangle of a dim x dim matrix set to zero.
__global__ void zero_lower_kernel(double* A, int dim) {
  const int64_t count = (int64_t)dim * dim;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < count; e += (int64_t)gridDim.x * blockDim.x)
    if (e % dim < e / dim) A[e] = 0.0;
}

// RqE[i, g d + e] = sum over the G query heads h of group g of Rq[i, h d + e]: the GQA
// expansion E applied from the right (query head h reads KV head h / G).
__global__ void fold_heads_kernel(const double* __restrict__ rq, int dq, int hkv, int group, int d,
                                  double* __restrict__ out) {
  const int dk = hkv * d;
  const int64_t count = (int64_t)dq * dk;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < count; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = e / dk;
    const int col = (int)(e % dk), g = col / d, c = col % d;
    double acc = 0.0;
    for (int h = g * group; h < (g + 1) * group; ++h) acc += rq[i * dq + h * d + c];
    out[e] = acc;
  }
}

// The maps in fp32: w_q[i][c] = Wq[i][c]; w_k[h d + e][c] = B[(h / G) d + e][c] / G (each
// query head's rows of the expanded key map are its KV head's rows of the folded map,
// divided by the group size, so that summing a group's rows gives B back).
__global__ void emit_maps_kernel(const double* __restrict__ wq, const double* __restrict__ bk, int hq, int group,
                                 int d, int dc, float* __restrict__ w_q, float* __restrict__ w_k) {
  const int64_t count = (int64_t)hq * d * dc;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < count; e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = e / dc;
    const int c = (int)(e % dc), h = (int)(row / d), x = (int)(row % d);
    w_q[e] = (float)wq[e];
    w_k[e] = (float)(bk[((int64_t)(h / group) * d + x) * dc + c] / group);
  }
}

}  // namespace esa
