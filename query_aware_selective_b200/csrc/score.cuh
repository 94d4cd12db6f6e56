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
// HBM-bound stream over the compressed keys of the middle. A CTA owns a contiguous run
// of keys and moves it into shared memory with one bulk copy (cp.async.bulk, mbarrier
// completion) per stage of kSsStageBytes, through a ring of kSsStages stages; the last
// of the eight warps to finish a stage issues its refill. In a stage, a group of LPK
// lanes holds one key (VPL floats per lane, 16-byte shared loads) and a warp covers KPW
// keys per step. Lq <= kScoreSmallLq queries live in registers.
//
// With NG > 1 groups (the per-head variant: group g owns compressed columns
// [g d_g, (g + 1) d_g)) the LPK lanes of a key split into NG runs of LPK / NG lanes,
// each reduced on its own: S is written as [B, NG, Lq, n_mid] and the maxima as
// [B, NG, Lq], i.e. B * NG independent selections.
constexpr int kScoreSmallLq = 8;
constexpr int kSsWarps = 8;
constexpr int kSsThreads = kSsWarps * 32;
constexpr int kSsStageBytes = 32768;
constexpr int kSsStages = 3;
constexpr int kSsSmemBytes = kSsStages * kSsStageBytes + 128 + 64;

template <int DC>
struct SmallScoreShape {
  static constexpr int VPL = DC >= 128 ? DC / 32 : 4;
  static constexpr int LPK = DC / VPL;
  static constexpr int KPW = 32 / LPK;
  static constexpr int KS = kSsStageBytes / (DC * 4);     // keys per stage
};

struct SsSmem {
  uint64_t full[kSsStages];
  int done[kSsStages];
  int abort_flag;
  int issued;
};

// grid (ctas per sequence, B); kSsThreads threads; kSsSmemBytes dynamic shared memory.
// CTA c scores keys [c * keys_per_cta, ...) of the middle (keys_per_cta a multiple of KS);
// in a variable-length batch (vl.len) CTAs past their sequence's middle have nothing to do.
template <int DC, int LQ, int NG>
__global__ void __launch_bounds__(kSsThreads, 2) score_small_kernel(const float* __restrict__ q_c,
                                                                   const float* __restrict__ k_c, int lq,
                                                                   int64_t n_cap, int64_t mid0, int64_t n_mid,
                                                                   int64_t keys_per_cta, float* __restrict__ s_out,
                                                                   uint32_t* __restrict__ m_key, const VarLen vl) {
  using Sh = SmallScoreShape<DC>;
  constexpr int VPL = Sh::VPL, LPK = Sh::LPK, KPW = Sh::KPW, KS = Sh::KS;
  constexpr int KEYS_PER_WARP = KS / kSsWarps;             // of a stage
  constexpr int LPG = LPK / NG;                            // lanes per group of a key
  static_assert(LPK % NG == 0, "groups split a key's lanes evenly");
  extern __shared__ __align__(128) uint8_t ss_dsm[];
  const uint32_t stage0 = (smem_u32(ss_dsm) + 127u) & ~127u;
  uint8_t* const stage0_ptr = ss_dsm + (stage0 - smem_u32(ss_dsm));
  SsSmem& sm = *reinterpret_cast<SsSmem*>(stage0_ptr + kSsStages * kSsStageBytes);
  const int b = blockIdx.y;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int grp = lane / LPK, sub = lane % LPK;
  const int hg = sub / LPG;                                // this lane's group
  const int64_t j_begin = (int64_t)blockIdx.x * keys_per_cta;
  // n_mid is the row stride of S; a variable-length batch scores each sequence's own middle
  const int64_t j_end = min(vl.len ? vl.n_mid(b, 801) : n_mid, j_begin + keys_per_cta);
  const int nst = j_end > j_begin ? (int)((j_end - j_begin + KS - 1) / KS) : 0;
  const float* kb = k_c + ((int64_t)b * n_cap + mid0) * DC;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSsStages; ++s) {
      mbar_init(&sm.full[s], 1);
      sm.done[s] = 0;
    }
    sm.abort_flag = 0;
    sm.issued = 0;
    fence_barrier_init();
  }
  __syncthreads();
  volatile int* abort_flag = &sm.abort_flag;
  // stage j: keys [j_begin + j KS, ...) as one contiguous copy
  auto issue = [&](int j) {
    const int s = j % kSsStages;
    const int64_t k0 = j_begin + (int64_t)j * KS;
    const int n_in = (int)(j_end - k0 < KS ? j_end - k0 : KS);
    const uint32_t bytes = (uint32_t)(n_in * DC * 4);
    mbar_arrive_expect_tx(&sm.full[s], bytes);
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     stage0 + s * kSsStageBytes),
                 "l"(kb + k0 * DC), "r"(bytes), "r"(smem_u32(&sm.full[s]))
                 : "memory");
    atomicMax(&sm.issued, j + 1);
  };
  if (threadIdx.x == 0)
    for (int j = 0; j < min(nst, kSsStages); ++j) issue(j);

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

  for (int j = 0; j < nst; ++j) {
    const int s = j % kSsStages;
    if (!mbar_wait_warp(&sm.full[s], (j / kSsStages) & 1, abort_flag, 401)) break;
    const int64_t k0 = j_begin + (int64_t)j * KS;
    const float* st = reinterpret_cast<const float*>(stage0_ptr + s * kSsStageBytes);
#pragma unroll
    for (int r = 0; r < KEYS_PER_WARP; r += KPW) {
      const int kk = warp * KEYS_PER_WARP + r + grp;      // key within the stage
      const int64_t jj = k0 + kk;
      float kv[VPL];
#pragma unroll
      for (int v = 0; v < VPL; v += 4) {
        const float4 x = *reinterpret_cast<const float4*>(st + kk * DC + sub * VPL + v);
        kv[v] = x.x; kv[v + 1] = x.y; kv[v + 2] = x.z; kv[v + 3] = x.w;
      }
#pragma unroll
      for (int i = 0; i < LQ; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int v = 0; v < VPL; ++v) acc = fmaf(q[i][v], kv[v], acc);
#pragma unroll
        for (int o = LPG / 2; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
        if (jj < j_end && i < lq) {
          mx[i] = fmaxf(mx[i], acc);
          if (sub % LPG == 0) s_out[(((int64_t)b * NG + hg) * lq + i) * n_mid + jj] = acc;
        }
      }
    }
    // release the stage; the last warp out refills it
    __syncwarp();
    int prev = 0;
    if (lane == 0) {
      __threadfence_block();
      prev = atomicAdd(&sm.done[s], 1);
      if (prev == kSsWarps - 1) {
        sm.done[s] = 0;
        if (j + kSsStages < nst) {
          fence_proxy_async();
          issue(j + kSsStages);
        }
      }
    }
  }
  __syncthreads();
  if (*abort_flag) {
    // drain the copies that may still be in flight before the CTA's shared memory goes away
    if (threadIdx.x == 0) {
      const int issued = sm.issued;
      for (int j = max(0, issued - kSsStages); j < issued; ++j)
        mbar_wait(&sm.full[j % kSsStages], (j / kSsStages) & 1, abort_flag, 402, /*respect_abort=*/false);
    }
    return;
  }
  if (NG == 1) {
    __shared__ float red[LQ][kSsWarps];
#pragma unroll
    for (int i = 0; i < LQ; ++i) {
      float v = warp_max(mx[i]);
      if (lane == 0) red[i][warp] = v;
    }
    __syncthreads();
    if (threadIdx.x < lq) {
      float v = -INFINITY;
      for (int w = 0; w < kSsWarps; ++w) v = fmaxf(v, red[threadIdx.x][w]);
      if (v > -INFINITY) atomicMax(&m_key[b * lq + threadIdx.x], order_key(v));
    }
  } else {
    // per (query, group): shared-memory order-key maxima, then one global atomic each
    __shared__ uint32_t redk[LQ][NG];
    for (int t = threadIdx.x; t < LQ * NG; t += kSsThreads) (&redk[0][0])[t] = 0u;
    __syncthreads();
#pragma unroll
    for (int i = 0; i < LQ; ++i)
      if (i < lq && sub % LPG == 0 && mx[i] > -INFINITY) atomicMax(&redk[i][hg], order_key(mx[i]));
    __syncthreads();
    for (int t = threadIdx.x; t < lq * NG; t += kSsThreads) {
      const int i = t / NG, g = t % NG;
      if (redk[i][g]) atomicMax(&m_key[((int64_t)b * NG + g) * lq + i], redk[i][g]);
    }
  }
}

// ------------------------------------------------------------ many queries (prefill) --
// Plain SIMT tile: 64 queries x 64 keys per CTA, reduction over d_c in slices of 16.
// Writes S and folds the tile's row maxima into m_key.
constexpr int kScT = 64;
constexpr int kScK = 16;

// grid (key tiles, query tiles, B * ng); sequence b, group g = blockIdx.z / ng, % ng
// reduces over the compressed columns [g dg, (g + 1) dg) of rows of dc floats.
__global__ void __launch_bounds__(256) score_tiled_kernel(const float* __restrict__ q_c, const float* __restrict__ k_c,
                                                          int lq, int64_t n_cap, int64_t mid0, int64_t n_mid, int dc,
                                                          int ng, float* __restrict__ s_out,
                                                          uint32_t* __restrict__ m_key) {
  __shared__ float qs[kScK][kScT + 4];
  __shared__ float ks[kScK][kScT + 4];
  __shared__ float rmax[kScT][17];
  const int bg = blockIdx.z;                     // sequence * ng + group
  const int b = bg / ng, col0 = (bg % ng) * (dc / ng), dg = dc / ng;
  const int i0 = blockIdx.y * kScT;
  const int64_t j0 = (int64_t)blockIdx.x * kScT;
  const int tid = threadIdx.x;
  const int ty = tid / 16, tx = tid % 16;   // 16 x 16 threads, 4 x 4 outputs each
  float acc[4][4] = {};
  const float* qb = q_c + (int64_t)b * lq * dc;
  const float* kb = k_c + ((int64_t)b * n_cap + mid0) * dc;
  for (int d0 = col0; d0 < col0 + dg; d0 += kScK) {
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
        s_out[((int64_t)bg * lq + i) * n_mid + j] = acc[u][v];
        m = fmaxf(m, acc[u][v]);
      }
    }
    rmax[ty * 4 + u][tx] = m;
  }
  __syncthreads();
  if (tid < kScT && i0 + tid < lq) {
    float m = -INFINITY;
    for (int x = 0; x < 16; ++x) m = fmaxf(m, rmax[tid][x]);
    if (m > -INFINITY) atomicMax(&m_key[(int64_t)bg * lq + i0 + tid], order_key(m));
  }
}

}  // namespace esa
