// compress_pk.cuh - the one-layer linear map with a pre-packed weight (ESA write-up,
// core steps: q and k pass through a one-layer MLP, 4096 -> 128).
//
//   y[r, :] = sum_k x[r, k] * Weff[k, :]        k = input head * head_dim + e
//   Weff[hi * D + e, :] = sum_{j < G} W[(hi * G + j) * D + e, :]      (GQA fold)
//
// The weight is static across calls, so its preparation is done once by
// compress_pack_kernel: fold the G rows, split each fp32 element into bf16 hi + lo
// (hi = rn(w), lo = rn(w - hi), |w - hi - lo| <= 2^-17 |w|) and store it transposed,
// K-major, as Wt[h][n][k] for the two 64-column halves h of the output:
//   n <  64: hi part of output column 64 h + n,   n >= 64: lo part of column 64 h + n - 64.
// compress_pk_kernel is then pure TMA + tcgen05: per 64-element reduction chunk one
// 128-row x tile and one 128 x 64 Wt tile (both 16 KB, K-major, 128-byte swizzle) go
// through a 4-stage ring, four M128 N128 K16 MMAs accumulate [hi | lo] in TMEM, and
// the epilogue adds the two halves. The reduction is split over the CTAs of a cluster
// (8 or 16) and summed through distributed shared memory in rank order: no workspace,
// no float atomics, the same result on every run.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "compress_tc.cuh"   // dsmem_map, ld_dsmem_f4, cluster_sync_all, cluster_rank

namespace esa {

constexpr int kCpThreads = 128;
constexpr int kCpRows = 128;
constexpr int kCpK = 64;                                   // reduction elements per chunk
constexpr int kCpStages = 4;
constexpr uint32_t kCpTile = 128 * kCpK * 2;               // 16 KB: x tile or Wt tile
constexpr uint32_t kCpStageBytes = 2 * kCpTile;
constexpr uint32_t kCpCtrl = 256;
constexpr uint32_t kCpSmemBytes = kCpStages * kCpStageBytes + kCpCtrl;
constexpr int kCpPStride = 64 + 4;                         // padded fp32 partial row
static_assert(kCpRows * kCpPStride * 4 <= kCpStages * kCpStageBytes, "partial must fit in the ring");

// Wt[(h * 128 + n) * K + k] from W [n_out_heads * D, 128] fp32. One block per 64 k x
// 64 output columns: the G folded rows are read coalesced along the columns, split,
// transposed through shared memory and written coalesced along k.
__global__ void __launch_bounds__(256) compress_pack_kernel(const float* __restrict__ w, int hin, int G, int d,
                                                            int K, __nv_bfloat16* __restrict__ wt) {
  __shared__ float hi_s[64][65], lo_s[64][65];
  const int k0 = blockIdx.x * 64, h = blockIdx.y;
  const int t = threadIdx.x;
  for (int i = t; i < 64 * 64; i += 256) {
    const int kk = i / 64, c = i % 64;
    const int k = k0 + kk, hi_ = k / d, e = k % d;
    float v = 0.f;
    for (int j = 0; j < G; ++j) v += w[((int64_t)(hi_ * G + j) * d + e) * 128 + h * 64 + c];
    const float vh = __bfloat162float(__float2bfloat16_rn(v));
    hi_s[kk][c] = vh;
    lo_s[kk][c] = v - vh;
  }
  __syncthreads();
  for (int i = t; i < 128 * 64; i += 256) {
    const int n = i / 64, kk = i % 64;
    const float v = n < 64 ? hi_s[kk][n] : lo_s[kk][n - 64];
    wt[((int64_t)h * 128 + n) * K + k0 + kk] = __float2bfloat16_rn(v);
  }
}

// grid (cl, row tiles, 2 halves), cluster (cl, 1, 1); cl in {8, 16}; K % (64 cl) == 0.
// Row r of x goes to row r of y; with yl.len (one new key per sequence of a
// variable-length batch) to row r * yl.n_cap + yl.len[r] - 1, its sequence's last token.
__global__ void __launch_bounds__(kCpThreads, 1)
    compress_pk_kernel(const __grid_constant__ CUtensorMap tx, const __grid_constant__ CUtensorMap tw, int64_t rows,
                       int K, float* __restrict__ y, int64_t ystride, const VarLen yl) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  const uint32_t s0 = smem_u32(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kCpStages * kCpStageBytes);   // [kCpStages]
  uint64_t* empty = full + kCpStages;                                                // [kCpStages]
  uint64_t* done = empty + kCpStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* part = reinterpret_cast<float*>(smem);                                      // [128][68] after the MMAs

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t cl = gridDim.x;                      // cluster = the whole x extent of the grid
  const uint32_t rank = cluster_rank();
  const int64_t r0 = (int64_t)blockIdx.y * kCpRows;
  const int h = blockIdx.z;
  const int kc = K / (int)cl;                         // reduction elements of this CTA
  const int nch = kc / kCpK;
  const int kb = (int)rank * kc;
  // the ring needs 1024-byte aligned stages; a misaligned window is reported, and the
  // CTA still takes part in both cluster barriers below
  const bool aligned = (s0 & 1023u) == 0;

  if (tid == 0) {
    for (int s = 0; s < kCpStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    *abort_flag = 0;
    fence_barrier_init();
    if (!aligned) record_status(5u, 310);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  bool ok = aligned;
  if (ok && warp == 0 && lane == 0) {
    // producer: chunk c into stage c % 4 once the MMAs of chunk c - 4 have drained it
    int issued = 0;
    for (int c = 0; c < nch; ++c) {
      const int s = c % kCpStages;
      if (!mbar_wait(&empty[s], ((c / kCpStages) & 1) ^ 1, abort_flag, 311)) break;
      const uint32_t sx = s0 + s * kCpStageBytes, sw = sx + kCpTile;
      mbar_arrive_expect_tx(&full[s], kCpStageBytes);
      tma_load_2d(sx, &tx, kb + c * kCpK, (int32_t)r0, &full[s]);
      tma_load_2d(sw, &tw, kb + c * kCpK, h * 128, &full[s]);
      issued = c + 1;
    }
    // after a wait ran out, let the loads still in flight land before shared memory is
    // reused (only the last kCpStages chunks can be outstanding)
    if (*abort_flag)
      for (int c = max(0, issued - kCpStages); c < issued; ++c)
        mbar_wait(&full[c % kCpStages], (c / kCpStages) & 1, abort_flag, 314, /*respect_abort=*/false);
  } else if (ok && warp == 1 && lane == 0) {
    // MMA issuer: D[128 x 128] (+)= x_c (128 x 64, K-major) . Wt_c^T (64 x 128, K-major)
    constexpr uint32_t idesc = umma_idesc(kFmtBF16, 128, 128, 0, 0);
    for (int c = 0; c < nch; ++c) {
      const int s = c % kCpStages;
      if (!mbar_wait(&full[s], (c / kCpStages) & 1, abort_flag, 312)) break;
      tc_fence_after();
      const uint32_t sx = s0 + s * kCpStageBytes, sw = sx + kCpTile;
#pragma unroll
      for (int ks = 0; ks < kCpK / 16; ++ks)
        umma_f16_ss(tmem, sdesc_sw128(sx + ks * 32, 16, 1024), sdesc_sw128(sw + ks * 32, 16, 1024), idesc,
                    (c > 0 || ks > 0) ? 1u : 0u);
      umma_commit(&empty[s]);
    }
    // every MMA issued has completed (this commit follows them) before TMEM is read
    // or released, also after a wait ran out
    umma_commit(done);
    mbar_wait(done, 0, abort_flag, 313, /*respect_abort=*/false);
  }
  __syncwarp();
  // D row tid -> hi + lo -> shared partial (zeros if anything failed)
  const bool fin = __syncthreads_and(ok && *abort_flag == 0) != 0;
  tc_fence_after();
  {
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    float* prow = part + tid * kCpPStride;
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float vh[32], vl[32];
      if (fin) {
        tmem_ld32(lane_base + c * 32, vh);
        tmem_ld32(lane_base + 64 + c * 32, vl);
        tmem_wait_ld();
      }
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(prow + c * 32 + e) =
            fin ? make_float4(vh[e] + vl[e], vh[e + 1] + vl[e + 1], vh[e + 2] + vl[e + 2], vh[e + 3] + vl[e + 3])
                : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  tc_fence_before();
  cluster_sync_all();
  // rows [rank * 128 / cl, ...) summed over the cl partials in rank order
  {
    const int rpc = kCpRows / (int)cl;                // rows reduced by this CTA (8 or 16)
    const int nq = rpc * 16;                          // float4 slots: rows x 64 columns / 4
    for (int q = tid; q < nq; q += kCpThreads) {
      const int rl = (int)rank * rpc + q / 16, c4 = (q % 16) * 4;
      const uint32_t local = smem_u32(part + rl * kCpPStride + c4);
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
      for (uint32_t src = 0; src < cl; ++src) {
        const float4 v = ld_dsmem_f4(dsmem_map(local, src));
        acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
      }
      const int64_t row = r0 + rl;
      if (fin && row < rows) {
        const int64_t yrow = yl.len ? row * yl.n_cap + yl.c0((int)row, 321) : row;
        *reinterpret_cast<float4*>(y + yrow * ystride + h * 64 + c4) = acc;
      }
    }
  }
  cluster_sync_all();
  if (warp == 0) tmem_dealloc(tmem, 128);
}

}  // namespace esa
