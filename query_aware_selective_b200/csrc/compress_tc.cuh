// compress_tc.cuh - the one-layer linear map on the tensor cores (ESA write-up, core
// steps: q and k pass through a one-layer MLP, 4096 -> 128).
//
//   y[r, :] = sum_{hi, e} x[r, hi, e] * Weff[hi * D + e, :],
//   Weff[hi * D + e, :] = sum_{j < G} W[(hi * G + j) * D + e, :]      (GQA fold)
//
// x is bf16 (exact in the MMA). W is fp32: each element is split into bf16 hi + lo
// (hi = rn(w), lo = rn(w - hi), |w - hi - lo| <= 2^-17 |w|) and both halves are
// multiplied, so the product keeps fp32-level accuracy on the bf16 tensor-core path
// (tcgen05.mma kind::f16, fp32 accumulate in TMEM).
//
// A CTA owns 128 rows, 64 of the 128 output columns and a slice of the reduction; the
// 8 CTAs of a cluster split the reduction, park their fp32 partials in shared memory,
// and each reduces 16 of the rows over the 8 partials in rank order through
// distributed shared memory: deterministic, no workspace, no float atomics.
// W is read straight into registers, a whole reduction chunk per batch, and the next
// chunk's W is in flight while the current chunk is converted and multiplied.
#pragma once
#include "common.cuh"

namespace esa {

constexpr int kCtCluster = 8;
constexpr int kCtThreads = 128;
constexpr int kCtRows = 128;
constexpr int kCtN = 128;              // d_out handled by this kernel
constexpr int kCtNS = 64;              // output columns per CTA
constexpr int kCtK = 64;               // reduction elements per chunk
constexpr uint32_t kCtABytes = kCtRows * kCtK * 2;      // 16 KB: A tile (x), one 128-byte column block
constexpr uint32_t kCtBBytes = kCtK * kCtNS * 2;        // 8 KB: B tile (W hi or lo), one 64-column block
constexpr uint32_t kCtStage = kCtABytes + 2 * kCtBBytes;
constexpr uint32_t kCtSmemBytes = 1024 + 2 * kCtStage + 256;
constexpr int kCtPStride = kCtNS + 4;   // padded row of the fp32 partial (spreads shared-memory banks)
static_assert(kCtRows * kCtPStride * 4 <= 2 * kCtStage, "partial must fit in the stage buffers");
constexpr int kCtWq = kCtK * kCtNS / 4 / kCtThreads;    // float4 of one W slice per thread per chunk (8)

// G = query heads per input head (1 for queries, Hq / Hkv for GQA keys)
template <int G>
__global__ void __cluster_dims__(kCtCluster, 1, 1) __launch_bounds__(kCtThreads, 1)
    compress_tc_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows, int64_t xstride, int hin, int d,
                       const float* __restrict__ w, float* __restrict__ y, int64_t ystride) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t s0 = smem_u32(smem);
  uint64_t* mma_bar = reinterpret_cast<uint64_t*>(smem + 2 * kCtStage);          // [2]
  uint64_t* done_bar = mma_bar + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  float* part = reinterpret_cast<float*>(smem);                                   // [128][68] after the MMAs

  const int tid = threadIdx.x;
  const uint32_t rank = cluster_rank();
  const int64_t r0 = (int64_t)blockIdx.y * kCtRows;
  const int n0 = blockIdx.z * kCtNS;                                              // output columns of this CTA
  const int kf = hin * d;                                                         // folded reduction length
  const int nchunks = kf / kCtK;
  const int per = (nchunks + kCtCluster - 1) / kCtCluster;
  const int c_begin = (int)rank * per;
  const int c_end = min(nchunks, c_begin + per);
  const int my_chunks = max(0, c_end - c_begin);

  if (tid == 0) {
    mbar_init(&mma_bar[0], 1);
    mbar_init(&mma_bar[1], 1);
    mbar_init(done_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (tid < 32) {
    tmem_alloc(tmem_slot, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // W slice of chunk c: rows k0 .. k0 + 63 of Weff, columns n0 .. n0 + 63; thread owns
  // float4 (kk, nq) with idx = tid + q * 128, kk = idx / 16, nq = idx % 16
  float4 wr[G][kCtWq];
  auto load_w = [&](int c) {
    const int k0 = c * kCtK;
    const int hi_ = k0 / d, e0 = k0 % d;
#pragma unroll
    for (int j = 0; j < G; ++j)
#pragma unroll
      for (int q = 0; q < kCtWq; ++q) {
        const int idx = tid + q * kCtThreads;
        const int kk = idx >> 4, nq = idx & 15;
        wr[j][q] = __ldg(reinterpret_cast<const float4*>(w + ((int64_t)(hi_ * G + j) * d + e0 + kk) * kCtN + n0) + nq);
      }
  };
  auto stage_a = [&](int c, int buf) {       // x tile by cp.async: 128 rows x 8 pieces of 16 bytes
    const uint32_t sa = s0 + buf * kCtStage;
    const int k0 = c * kCtK;
    const int hi_ = k0 / d, e0 = k0 % d;
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const int idx = tid + q * kCtThreads;
      const int r = idx >> 3, piece = idx & 7;
      const int64_t row = r0 + r;
      const bool ok = row < rows;
      const void* src = ok ? (const void*)(x + row * xstride + (int64_t)hi_ * d + e0 + piece * 8) : (const void*)x;
      cp_async16(sa + sw128_off(r, piece), src, ok ? 16u : 0u);
    }
    cp_async_commit();
  };
  auto stage_b = [&](int buf) {              // fold, split into hi / lo, MN-major swizzled stores
    const uint32_t sbh = s0 + buf * kCtStage + kCtABytes;
    const uint32_t sbl = sbh + kCtBBytes;
#pragma unroll
    for (int q = 0; q < kCtWq; ++q) {
      const int idx = tid + q * kCtThreads;
      const int kk = idx >> 4, nq = idx & 15;
      float4 acc = wr[0][q];
#pragma unroll
      for (int j = 1; j < G; ++j) {
        acc.x += wr[j][q].x; acc.y += wr[j][q].y; acc.z += wr[j][q].z; acc.w += wr[j][q].w;
      }
      const __nv_bfloat162 h01 = __floats2bfloat162_rn(acc.x, acc.y);
      const __nv_bfloat162 h23 = __floats2bfloat162_rn(acc.z, acc.w);
      const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
      const __nv_bfloat162 l01 = __floats2bfloat162_rn(acc.x - f01.x, acc.y - f01.y);
      const __nv_bfloat162 l23 = __floats2bfloat162_rn(acc.z - f23.x, acc.w - f23.y);
      // MN-major 128-byte swizzle: k-row kk, 16-byte chunk n / 8 of the 64-column block
      const int n = nq * 4;
      const uint32_t off = sw128_off(kk, n >> 3) + (n & 7) * 2;
      const uint32_t hw0 = *reinterpret_cast<const uint32_t*>(&h01), hw1 = *reinterpret_cast<const uint32_t*>(&h23);
      const uint32_t lw0 = *reinterpret_cast<const uint32_t*>(&l01), lw1 = *reinterpret_cast<const uint32_t*>(&l23);
      asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(sbh + off), "r"(hw0), "r"(hw1) : "memory");
      asm volatile("st.shared.v2.b32 [%0], {%1, %2};" ::"r"(sbl + off), "r"(lw0), "r"(lw1) : "memory");
    }
  };

  constexpr uint32_t idesc = umma_idesc(kFmtBF16, 128, kCtNS, 0, 1);   // A K-major (x), B MN-major (W)
  bool ok = true;
  if (my_chunks > 0) load_w(c_begin);
  for (int i = 0; i < my_chunks && ok; ++i) {
    const int buf = i & 1;
    if (i >= 2) ok = __syncthreads_and(mbar_wait(&mma_bar[buf], ((i - 2) >> 1) & 1, abort_flag, 301));
    if (!ok) break;
    stage_a(c_begin + i, buf);
    stage_b(buf);
    if (i + 1 < my_chunks) load_w(c_begin + i + 1);   // in flight during this chunk's MMA
    cp_async_wait_all();
    fence_proxy_async();
    __syncthreads();
    if (tid == 0) {
      tc_fence_after();
      const uint32_t sa = s0 + buf * kCtStage;
      const uint32_t sbh = sa + kCtABytes, sbl = sbh + kCtBBytes;
#pragma unroll
      for (int ks = 0; ks < kCtK / 16; ++ks) {
        const uint64_t da = sdesc_sw128(sa + ks * 32, 16, 1024);
        umma_f16_ss(tmem, da, sdesc_sw128(sbh + ks * 2048, kCtBBytes, 1024), idesc, (i > 0 || ks > 0) ? 1u : 0u);
        umma_f16_ss(tmem, da, sdesc_sw128(sbl + ks * 2048, kCtBBytes, 1024), idesc, 1u);
      }
      umma_commit(&mma_bar[buf]);
    }
  }
  if (tid == 0) {
    umma_commit(done_bar);
    mbar_wait(done_bar, 0, abort_flag, 302, /*respect_abort=*/false);
  }
  __syncthreads();
  tc_fence_after();
  // TMEM -> shared partial (row = lane = tid); a CTA without chunks contributes zeros
  {
    const uint32_t lane_base = tmem + ((uint32_t)((tid >> 5) * 32) << 16);
    float* prow = part + tid * kCtPStride;
    const bool have = my_chunks > 0 && ok;
#pragma unroll
    for (int c = 0; c < kCtNS / 32; ++c) {
      float v[32];
      tmem_ld32(lane_base + c * 32, v);
      tmem_wait_ld();
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(prow + c * 32 + e) =
            have ? make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  tc_fence_before();
  cluster_sync_all();
  // reduce rows [rank * 16, rank * 16 + 16) over the 8 partials in rank order
  {
    const int rl = (int)rank * (kCtRows / kCtCluster) + (tid >> 3);
    const int c0 = (tid & 7) * 8;
    float4 acc[2];
#pragma unroll
    for (int q = 0; q < 2; ++q) acc[q] = make_float4(0.f, 0.f, 0.f, 0.f);
    const uint32_t local = smem_u32(part + rl * kCtPStride + c0);
    for (uint32_t src = 0; src < kCtCluster; ++src) {
      const uint32_t ra = dsmem_map(local, src);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const float4 v = ld_dsmem_f4(ra + q * 16);
        acc[q].x += v.x; acc[q].y += v.y; acc[q].z += v.z; acc[q].w += v.w;
      }
    }
    const int64_t row = r0 + rl;
    if (row < rows) {
#pragma unroll
      for (int q = 0; q < 2; ++q) *reinterpret_cast<float4*>(y + row * ystride + n0 + c0 + 4 * q) = acc[q];
    }
  }
  cluster_sync_all();
  if (tid < 32) tmem_dealloc(tmem, 64);
}

}  // namespace esa
