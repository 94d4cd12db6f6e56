// score_tc.cuh - compressed importance scores of a prefill chunk on the tensor cores
// (ESA write-up: implementation paragraph - a middle token's importance is its q.k
// product with every query of the current chunk; score-correction paragraph - each
// query's scores are shifted by its maximum and bounded below by -C; the selection
// runs in the low-dimensional space, which is what makes it cheap).
//
// Two passes over the compressed middle keys, tcgen05.mma kind::tf32 (fp32 operands
// read as tf32, fp32 accumulate), operands brought in by TMA with 128-byte swizzle:
//   pass 1: D[query, key] = Q~ K~^T; every query's maximum over the CTA's 128 keys is
//           folded into m_i with atomicMax on order-preserving keys (exact, and the
//           same in any order);
//   pass 2: D[key, query] = K~ Q~^T; thread = key: s_j = sum_i max(D - m_i, -C) over
//           the queries in increasing order (deterministic).
// A CTA owns 128 middle keys and walks the chunk's queries 128 at a time; the key
// tile stays in shared memory, query tiles stream through two buffers, and TMEM holds
// two 128-column accumulators so the epilogue of one query tile overlaps the MMA of
// the next. Warps 0-3: epilogue (thread = TMEM lane); warp 4: TMA + MMA issue.
#pragma once
#include <cuda.h>

#include "common.cuh"

namespace esa {

constexpr int kStThreads = 160;
constexpr int kStRows = 128;          // keys per CTA, queries per tile

struct ScoreTcArgs {
  int lq;                 // queries of the chunk
  int dc;                 // compressed dim (32, 64 or 128)
  int64_t n_cap, mid0, n_mid;
  uint32_t* m_key;        // [B, lq] order keys of the row maxima (pass 1 output, pass 2 input)
  float* s;               // [B, n_mid] clamped chunk sums (pass 2 output)
  float clamp_c;
};

struct StSmem {
  uint64_t k_full, q_full[2], q_empty[2], d_full[2], d_empty[2], done;
  uint32_t tmem_base;
  int abort_flag;
};

template <int PASS>
__global__ void __launch_bounds__(kStThreads, 1)
    score_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_q,
                    ScoreTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const uint32_t tile_bytes = kStRows * a.dc * 4;             // 128 rows x dc fp32
  const uint32_t sK = smem_u32(smem);
  const uint32_t sQ = sK + tile_bytes;                        // 2 buffers
  StSmem& sm = *reinterpret_cast<StSmem*>(smem + 3 * tile_bytes);
  float* m_s = reinterpret_cast<float*>(smem + 3 * tile_bytes + 256);   // lq maxima (pass 2)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.y;
  const int64_t j0 = (int64_t)blockIdx.x * kStRows;           // first middle key of the CTA
  const int nqt = (a.lq + kStRows - 1) / kStRows;
  const int kblocks = a.dc / 32;                              // 128-byte column blocks

  if (threadIdx.x == 0) {
    mbar_init(&sm.k_full, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sm.q_full[i], 1);
      mbar_init(&sm.q_empty[i], 1);
      mbar_init(&sm.d_full[i], 1);
      mbar_init(&sm.d_empty[i], 4);                 // one arrival per epilogue warp
    }
    mbar_init(&sm.done, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (PASS == 2) {
    for (int i = threadIdx.x; i < a.lq; i += kStThreads) {
      const uint32_t k = a.m_key[(int64_t)b * a.lq + i];
      m_s[i] = __uint_as_float((k & 0x80000000u) ? (k & 0x7fffffffu) : ~k);
    }
  }
  if (warp == 4) {
    tmem_alloc(&sm.tmem_base, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == 4) {
    if (lane == 0) {
      // K~ tile: rows b*n_cap + mid0 + j0 .. +127 (rows past the middle are masked later)
      const int32_t krow = (int32_t)((int64_t)b * a.n_cap + a.mid0 + j0);
      mbar_arrive_expect_tx(&sm.k_full, tile_bytes);
      for (int kb = 0; kb < kblocks; ++kb) tma_load_2d(sK + kb * kStRows * 128, &tm_k, kb * 32, krow, &sm.k_full);
      auto load_q = [&](int t) -> bool {
        const int buf = t & 1;
        if (!mbar_wait(&sm.q_empty[buf], ((t >> 1) & 1) ^ 1, abort_flag, 201)) return false;
        const int32_t qrow = b * a.lq + t * kStRows;
        mbar_arrive_expect_tx(&sm.q_full[buf], tile_bytes);
        for (int kb = 0; kb < kblocks; ++kb)
          tma_load_2d(sQ + buf * tile_bytes + kb * kStRows * 128, &tm_q, kb * 32, qrow, &sm.q_full[buf]);
        return true;
      };
      bool ok = load_q(0);
      if (ok && nqt > 1) ok = load_q(1);
      if (ok) ok = mbar_wait(&sm.k_full, 0, abort_flag, 202);
      constexpr uint32_t idesc = umma_idesc(kFmtTF32, 128, 128, 0, 0);
      for (int t = 0; t < nqt && ok; ++t) {
        const int buf = t & 1;
        if (!(ok = mbar_wait(&sm.q_full[buf], (t >> 1) & 1, abort_flag, 203))) break;
        if (!(ok = mbar_wait(&sm.d_empty[buf], ((t >> 1) & 1) ^ 1, abort_flag, 204))) break;
        tc_fence_after();
        const uint32_t qt = sQ + buf * tile_bytes;
        for (int kk = 0; kk < a.dc / 8; ++kk) {
          const uint32_t off = (kk >> 2) * kStRows * 128 + (kk & 3) * 32;
          const uint64_t dq = sdesc_sw128(qt + off, 16, 1024);
          const uint64_t dk = sdesc_sw128(sK + off, 16, 1024);
          // pass 1: rows = queries (A = Q~); pass 2: rows = keys (A = K~)
          if (PASS == 1) umma_tf32_ss(tmem + buf * 128, dq, dk, idesc, kk > 0);
          else umma_tf32_ss(tmem + buf * 128, dk, dq, idesc, kk > 0);
        }
        umma_commit(&sm.d_full[buf]);
        umma_commit(&sm.q_empty[buf]);
        if (t + 2 < nqt && !(ok = load_q(t + 2))) break;
      }
      umma_commit(&sm.done);
      mbar_wait(&sm.done, 0, abort_flag, 205, /*respect_abort=*/false);
    }
    __syncwarp();
  } else {
    // epilogue: thread = TMEM lane r (query row in pass 1, key row in pass 2)
    const int r = threadIdx.x;
    const uint32_t lane_base = tmem + ((uint32_t)(warp * 32) << 16);
    const int64_t j_r = j0 + r;                               // pass 2: this thread's key
    const float lo = -a.clamp_c;
    float acc = 0.f;
    for (int t = 0; t < nqt; ++t) {
      const int buf = t & 1;
      if (!mbar_wait_warp(&sm.d_full[buf], (t >> 1) & 1, abort_flag, 206)) break;
      tc_fence_after();
      if (PASS == 1) {
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float x[32];
          tmem_ld32(lane_base + buf * 128 + c * 32, x);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (j0 + c * 32 + e < a.n_mid) mx = fmaxf(mx, x[e]);
        }
        tc_fence_before();
        mbar_arrive_warp(&sm.d_empty[buf]);
        const int q = t * kStRows + r;
        if (q < a.lq && mx > -INFINITY) atomicMax(&a.m_key[(int64_t)b * a.lq + q], order_key(mx));
      } else {
        const int qn = min(kStRows, a.lq - t * kStRows);
        const float* mt = m_s + t * kStRows;
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          float x[32];
          tmem_ld32(lane_base + buf * 128 + c * 32, x);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (c * 32 + e < qn) acc += fmaxf(x[e] - mt[c * 32 + e], lo);
        }
        tc_fence_before();
        mbar_arrive_warp(&sm.d_empty[buf]);
      }
    }
    if (PASS == 2 && j_r < a.n_mid) a.s[(int64_t)b * a.n_mid + j_r] = acc;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 4) tmem_dealloc(tmem, 256);
}

}  // namespace esa
