// attn_pp.cuh - tensor-core attention over an indexed key list, two query tiles per CTA
// in ping-pong (sm_100a tcgen05).
//
// One CTA computes two tiles of 128 query rows (Q0, Q1: consecutive row tiles that
// share their key list) against that list, 128 keys a step.
// Each key tile is loaded once and used by both query tiles:
//   S_t = Q_t K_j^T          tcgen05.mma kind::f16 (bf16 in, fp32 accumulate), TMEM
//   P_t = exp2(S_t c - m)    softmax warpgroup t reads S_t from TMEM, writes bf16 P_t
//                            back over the first half of S_t's columns
//   O_t += P_t V_j           tcgen05.mma, A = P_t from TMEM
// The MMA warp issues, for every key tile j, PV_0(j), S_0(j+1), PV_1(j), S_1(j+1): while
// warpgroup 0 turns S_0(j+1) into probabilities, the tensor pipe works for tile 1
// (PV_1(j), S_1(j+1)), and the other way round, so the exponentials of one query tile
// overlap the matrix products of the other. Each warpgroup has one thread per query
// row (128 key columns a thread): no exchange between threads for the row maximum or
// the sum.
// Roles (384 threads, four warpgroups): warpgroup 0 softmax of Q0, 1 softmax of Q1
// (warp w reads TMEM lanes 32 (w % 4) .. + 31), warpgroup 2: warp 8 issues the MMAs,
// warp 9 loads Q0, Q1 and the K tiles, warp 10 the V tiles, warp 11 has no role.
// Warpgroup 2 gives registers back (setmaxnreg) so that a softmax thread has 200.
//
// TMEM (512 columns): S_0/P_0 at 0, S_1/P_1 at 128, O_0 at 256, O_1 at 384.
// Shared memory: Q0, Q1 32 KB each, K 3 x 32 KB, V 2 x 32 KB, 1 KB of control.
// S_t(j+1) overwrites P_t(j): it is issued after PV_t(j) by the same thread, and the
// tensor pipe executes one thread's MMAs in issue order. The commit of S_t(j) also
// covers PV_t(j-1) (a commit tracks every earlier MMA of the thread), so once a
// softmax thread has seen S_t(j) complete, O_t holds PV_t(0 .. j-1) and may be rescaled
// in place; the MMA warp issues PV_t(j) only after that thread's p_full arrival.
//
// m is the running row maximum used for the exponentials (log2 units); it is raised
// (and O, l rescaled) only when a tile's maximum exceeds it by more than 2^8, so most
// tiles skip the rescale and P stays <= 2^8 (exact softmax either way: o = O / l).
//
// The problem policy is the one of attn_tc_kernel (attn_tc.cuh), with
// `bool setup_at(int tile)` in place of setup(): per-CTA fields for row tile `tile`
// (2 blockIdx.x or 2 blockIdx.x + 1; blockIdx.y, blockIdx.z as the policy defines
// them), false = no such tile. store() takes 64 columns at a time.
#pragma once
#include <cuda.h>

#include "attn_tc.cuh"
#include "common.cuh"

namespace esa {

constexpr int kPpThreads = 12 * 32;
constexpr int kPpMmaWarp = 8, kPpKWarp = 9, kPpVWarp = 10;
constexpr int kPpKStages = 3, kPpVStages = 2;
// registers a thread after the reallocation: the launch grants 384 x 168
constexpr uint32_t kPpRegsSoftmax = 200, kPpRegsOther = 88;
static_assert(256 * kPpRegsSoftmax + 128 * kPpRegsOther <= 384 * 168, "register split exceeds the launch's");
constexpr uint32_t kPpCtrlBytes = 1024;
constexpr uint32_t kPpSmemBytes = (2 + kPpKStages + kPpVStages) * kTileBytes + kPpCtrlBytes;
static_assert(kPpSmemBytes <= 232448, "exceeds the 227 KB of shared memory per CTA");
static_assert(kTcD / kTcSplit == 64, "store() takes 64 columns");
struct PpSmem {
  uint64_t q_full;
  uint64_t k_full[kPpKStages], k_empty[kPpKStages], v_full[kPpVStages], v_empty[kPpVStages];
  uint64_t s_full[2], p_full[2], pv_full[2];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
};
static_assert(sizeof(PpSmem) <= kPpCtrlBytes, "control block overflows its reservation");

template <class Problem>
__global__ void __launch_bounds__(kPpThreads, 1)
    attn_pp_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tb_q,
                   const __grid_constant__ CUtensorMap tb_k, const __grid_constant__ CUtensorMap tb_v,
                   const __grid_constant__ CUtensorMap ts_k, const __grid_constant__ CUtensorMap ts_v,
                   Problem prob0) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) record_status(5u, 120);
    return;
  }
  const uint32_t sQ = smem_u32(smem);                 // Q0, then Q1
  const uint32_t sK = sQ + 2 * kTileBytes;
  const uint32_t sV = sK + kPpKStages * kTileBytes;
  PpSmem& sm = *reinterpret_cast<PpSmem*>(smem + (2 + kPpKStages + kPpVStages) * kTileBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x;
  // pk: the policy of the pair's later tile (it sees the most keys), which the loaders
  // use for the key list; each role sets up its own copy for its tile below
  Problem pk = prob0;
  if (!pk.setup_at(2 * pair)) return;                  // the whole CTA (and its pair) has nothing
  bool has1;
  {
    Problem p1 = prob0;
    has1 = p1.setup_at(2 * pair + 1);
    if (has1) pk = p1;
  }
  const int64_t n_keys = pk.n_keys();
  const int nt = (int)((n_keys + kTcKeys - 1) / kTcKeys);
  const int n = nt;
  // Q tiles as TMA boxes (consecutive queries), or gathered rows: then each softmax
  // thread copies its own row with 16-byte cp.async (a TMA gather4 moves 4 rows an
  // instruction, and the 128 instructions of two tiles took about 11 us to land)
  int qy = 0, qz = 0;
  const bool q_tma = pk.q_box(&qy, &qz);

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, q_tma ? 1 : 256);          // the TMA's arrival, or every softmax thread's
    for (int s = 0; s < kPpKStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int s = 0; s < kPpVStages; ++s) {
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&sm.s_full[t], 1);
      mbar_init(&sm.p_full[t], 4);                     // one arrival per softmax warp of the group
      mbar_init(&sm.pv_full[t], 1);
    }
    mbar_init(&sm.mma_done, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kPpMmaWarp) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  if (warp >= 8) {
    setmaxnreg_dec<kPpRegsOther>();
    if (warp == kPpKWarp) {
      // -------------------------------------------------------------- Q + K loader
      if (n > 0 && q_tma && lane == 0) {
        mbar_arrive_expect_tx(&sm.q_full, (has1 ? 2u : 1u) * kTileBytes);
        for (int tq = 0; tq < (has1 ? 2 : 1); ++tq) {
          Problem pq = prob0;
          pq.setup_at(2 * pair + tq);
          int y = 0, z = 0;
          pq.q_box(&y, &z);
          const uint32_t dst = sQ + tq * kTileBytes;
          tma_load_3d(dst, &tb_q, 0, y, z, &sm.q_full);
          tma_load_3d(dst + kBlkBytes, &tb_q, 64, y, z, &sm.q_full);
        }
      }
      stream_kv<kPpKStages>(pk, &tm_k, &tb_k, &ts_k, sK, sm.k_full, sm.k_empty, n, n_keys, lane, abort_flag, 121);
    } else if (warp == kPpVWarp) {
      // -------------------------------------------------------------- V loader
      stream_kv<kPpVStages>(pk, &tm_v, &tb_v, &ts_v, sV, sm.v_full, sm.v_empty, n, n_keys, lane, abort_flag, 122);
    } else if (warp == kPpMmaWarp && n > 0) {
      // -------------------------------------------------------------- MMA issuer
      // The whole warp runs the loop (converged: the warp-uniform descriptors stay in
      // uniform registers); one elected lane issues each MMA and commit. Between a
      // softmax group's p_full and the S it then waits for, the loop does no other wait:
      // the V tile of PV_t(j) and the K tile of S_t(j+1) are waited for beforehand.
      constexpr uint32_t idesc_qk = umma_idesc(kFmtBF16, 128, 128, 0, 0);
      constexpr uint32_t idesc_pv = umma_idesc(kFmtBF16, 128, 128, 0, 1);
      // descriptors built once; only the low word (address in 16-byte units) moves:
      // K step kk of a K-major operand is +2 kk within a 64-column block and +1024 per
      // block; of the MN-major V tile, +128 kk
      const uint64_t dq = sdesc_sw128(sQ, 16, 1024), dk = sdesc_sw128(sK, 16, 1024);
      const uint64_t dv = sdesc_sw128(sV, kBlkBytes, 1024);
      const uint32_t q_lo = (uint32_t)dq, q_hi = (uint32_t)(dq >> 32);
      const uint32_t k_lo = (uint32_t)dk, k_hi = (uint32_t)(dk >> 32);
      const uint32_t v_lo = (uint32_t)dv, v_hi = (uint32_t)(dv >> 32);
      auto mma_s = [&](int t, int u) {
        const uint32_t qb = q_lo + t * (kTileBytes >> 4);
        const uint32_t kb = k_lo + (u % kPpKStages) * (kTileBytes >> 4), d = tmem + t * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * (kBlkBytes >> 4) + (kk & 3) * 2;
          umma_f16_ss2_elect(d, qb + off, q_hi, kb + off, k_hi, idesc_qk, kk > 0);
        }
        umma_commit_elect(&sm.s_full[t]);
      };
      auto mma_pv = [&](int t, int u) {
        const uint32_t vb = v_lo + (u % kPpVStages) * (kTileBytes >> 4), pa = tmem + t * 128;
        const uint32_t acc0 = u > 0;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // A = P from TMEM (keys 16 kk .. + 15 in columns 8 kk .. + 7 of the S/P buffer);
          // B = V (MN-major: 8-key row groups of 1024 bytes, d blocks 16 KB apart)
          umma_f16_ts2_elect(tmem + 256 + t * 128, pa + kk * 8, vb + kk * 128, v_hi, idesc_pv, kk > 0 ? 1u : acc0);
        }
        umma_commit_elect(&sm.pv_full[t]);
      };
      auto wait = [&](uint64_t* bar, uint32_t parity, unsigned site) -> bool {
        const bool got = __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, site));
        if (got) tc_fence_after();
        return got;
      };
      auto wait_p = [&](int t, int u, unsigned site) -> bool {
        const bool got = __all_sync(0xffffffffu, mbar_wait_spin(&sm.p_full[t], u & 1, abort_flag, site));
        if (got) tc_fence_after();
        return got;
      };
      bool ok = wait(&sm.q_full, 0, 124) && wait(&sm.k_full[0], 0, 123);
      if (ok) {
        mma_s(0, 0);
        if (has1) mma_s(1, 0);
        umma_commit_elect(&sm.k_empty[0]);
      }
      for (int u = 0; u < n && ok; ++u) {
        const bool next = u + 1 < n;
        if (!(ok = wait(&sm.v_full[u % kPpVStages], (u / kPpVStages) & 1, 126))) break;
        if (next && !(ok = wait(&sm.k_full[(u + 1) % kPpKStages], ((u + 1) / kPpKStages) & 1, 123))) break;
        if (!(ok = wait_p(0, u, 125))) break;
        mma_pv(0, u);
        if (next) mma_s(0, u + 1);
        if (has1) {
          if (!(ok = wait_p(1, u, 127))) break;
          mma_pv(1, u);
        }
        umma_commit_elect(&sm.v_empty[u % kPpVStages]);
        if (next) {
          if (has1) mma_s(1, u + 1);
          umma_commit_elect(&sm.k_empty[(u + 1) % kPpKStages]);
        }
      }
      // every MMA issued so far has completed before TMEM is released
      umma_commit_elect(&sm.mma_done);
      mbar_wait(&sm.mma_done, 0, abort_flag, 128, /*respect_abort=*/false);
    }
    __syncwarp();
  } else {
    setmaxnreg_inc<kPpRegsSoftmax>();
    // ---------------------------------------------------------------- softmax (rows)
    const int t = warp >> 2, quad = warp & 3;
    const int r = quad * 32 + lane;                  // row of query tile t = TMEM lane
    const bool active = t == 0 || has1;
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t s_addr = lane_base + t * 128, o_addr = lane_base + 256 + t * 128;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    if (!q_tma) {
      // this thread's query row into the 128-byte-swizzled Q tile (row r: 16-byte chunk c
      // of 64-column block c / 8 at sw128_off(r, c % 8)); padding rows copy the tile's
      // first row (a real query; its scores are never stored)
      if (n > 0 && active) {
        Problem pq = prob0;
        pq.setup_at(2 * pair + t);
        int32_t row = pq.q_row(r);
        if (row < 0) row = pq.q_row(0);
        const __nv_bfloat16* src = pq.q + (int64_t)row * kTcD;
        const uint32_t dst = sQ + t * kTileBytes;
#pragma unroll
        for (int c = 0; c < kTcD / 8; ++c) cp_async16(dst + (c >> 3) * kBlkBytes + sw128_off(r, c & 7), src + c * 8, 16);
        cp_async_wait_all();
        fence_proxy_async();                         // written through the generic proxy, read by the MMA
      }
      mbar_arrive(&sm.q_full);
    }
    // The tile maximum is needed only to decide a rescale (tile max > m + 2^8 in log2
    // units), so it is computed only when that can be the case: while m is not set yet,
    // in tiles with masked keys, or when the tile's sum of exp2(s c - m) exceeds 2^8
    // (every term is at most the sum, so a sum <= 2^8 shows every s c <= m + 8). Then
    // the exponentials are taken again with the raised m. The decisions are those of
    // always taking the maximum first.
    constexpr float kRescale = 8.0f;                 // log2 units
    if (active) {
      int64_t lim;
      float sl2;
      {
        Problem pr = prob0;                          // (set up again for the epilogue: fewer live registers)
        pr.setup_at(2 * pair + t);
        lim = pr.limit(r);
        sl2 = pr.scale_log2();
      }
      // key tiles u < u_mask have no masked key for any row of this warp (keys
      // u * 128 + e with e <= limit - u * 128 are visible; limits are below 2^31)
      const int lim_min = __reduce_min_sync(0xffffffffu, (int)lim);
      const int u_mask = lim_min >= kTcKeys - 1 ? (lim_min - (kTcKeys - 1)) / kTcKeys + 1 : 0;
      if constexpr (HasPrefetch<Problem>::value) {
        Problem pf = prob0;
        pf.setup_at(2 * pair + t);
        pf.prefetch(r, 0);
        pf.prefetch(r, 64);
      }
      const float2 scale2 = make_float2(sl2, sl2);
      float v[kTcKeys];
      // P = exp2(v c - m') to the TMEM buffer over S (keys 32 c .. + 31 to columns
      // 16 c .. + 15), bf16 rounded to nearest (unbiased, so l may add the unrounded
      // values); returns this tile's sum
      auto exps = [&](float m_use) -> float {
        const float2 shift2 = make_float2(-m_use, -m_use);
        float2 ls2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
        for (int c = 0; c < kTcKeys / 32; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int f = 32 * c + e;
            const float2 x = __ffma2_rn(make_float2(v[f], v[f + 1]), scale2, shift2);
            const float2 pe = make_float2(fast_exp2(x.x), fast_exp2(x.y));
            ls2[(e >> 1) & 1] = __fadd2_rn(ls2[(e >> 1) & 1], pe);
            pk[e / 2] = pack_bf16x2(pe.x, pe.y);
          }
          tmem_st16(s_addr + c * 16, pk);
        }
        const float2 l2 = __fadd2_rn(ls2[0], ls2[1]);
        return l2.x + l2.y;
      };
      auto tile_max = [&]() -> float {
        float m8[8];                                 // 8 independent chains of 3-input max
#pragma unroll
        for (int q = 0; q < 8; ++q) m8[q] = fmaxf(v[q], v[8 + q]);
#pragma unroll
        for (int e = 16; e < kTcKeys; e += 16) {
#pragma unroll
          for (int q = 0; q < 8; ++q) m8[q] = fmax3f(m8[q], v[e + q], v[e + 8 + q]);
        }
        return fmaxf(fmax3f(m8[0], m8[1], m8[2]), fmax3f(fmax3f(m8[3], m8[4], m8[5]), m8[6], m8[7])) * sl2;
      };
      // raise m to the tile maximum where it exceeds m + 2^8 (warp-uniform call: the
      // TMEM accesses of the O rescale are collective); returns whether any row did
      auto raise = [&](int u, float mx) -> bool {
        const bool need = mx > m + kRescale;         // -inf + 8 = -inf
        if (!__any_sync(0xffffffffu, need)) return false;
        const float m_new = need ? mx : m;
        const float alpha = need ? fast_exp2(m - m_new) : 1.f;    // m = -inf: 0
        if (u > 0) {
          // O_t holds PV_t(0 .. u-1), complete (the commit of S_t(u) covers them);
          // 8 columns at a time beside the 128 live scores
#pragma unroll 1
          for (int c = 0; c < kTcD / 8; ++c) {
            uint32_t ov[8];
            tmem_ld8(o_addr + c * 8, ov);
            tmem_wait_ld();
#pragma unroll
            for (int e = 0; e < 8; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
            tmem_st8(o_addr + c * 8, ov);
          }
          tmem_wait_st();
        }
        l *= alpha;
        m = m_new;
        return true;
      };
      for (int u = 0; u < n; ++u) {
        if (!(ok = mbar_wait_warp(&sm.s_full[t], u & 1, abort_flag, 129))) break;
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < kTcKeys / 32; ++c) tmem_ld32(s_addr + c * 32, v + c * 32);
        tmem_wait_ld();
        float lt;
        if (u >= u_mask) {
          // the causal cut: keys j * 128 + e with e <= rem are visible (rem >= 127: all)
          const int64_t rem64 = lim - (int64_t)u * kTcKeys;
          const int rem = rem64 < 0 ? -1 : (rem64 >= kTcKeys ? kTcKeys : (int)rem64);
#pragma unroll
          for (int e = 0; e < kTcKeys; ++e) v[e] = e <= rem ? v[e] : -INFINITY;
          raise(u, tile_max());
          lt = exps(m == -INFINITY ? 0.f : m);          // a row with no visible key yet: all 0
        } else if (__any_sync(0xffffffffu, m == -INFINITY)) {
          raise(u, tile_max());
          lt = exps(m);
        } else {
          lt = exps(m);
          if (__any_sync(0xffffffffu, lt > 256.f) && raise(u, tile_max())) lt = exps(m);
        }
        l += lt;
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive_warp(&sm.p_full[t]);
      }
    }
    __syncwarp();

    // -------------------------------------------------------------- epilogue
    // O_t complete, then the rows are stored, 64 columns at a time from TMEM
    if (active && ok && n > 0 && mbar_wait_warp(&sm.pv_full[t], (n - 1) & 1, abort_flag, 130)) {
      tc_fence_after();
      Problem pr = prob0;
      pr.setup_at(2 * pair + t);
#pragma unroll 1
      for (int h = 0; h < 2; ++h) {
        float o[64];
        tmem_ld32(o_addr + h * 64, o);
        tmem_ld32(o_addr + h * 64 + 32, o + 32);
        tmem_wait_ld();
        pr.store(r, h * 64, o, m, l);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kPpMmaWarp) tmem_dealloc(tmem, 512);
}

}  // namespace esa
