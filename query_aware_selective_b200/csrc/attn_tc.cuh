// attn_tc.cuh - tensor-core attention over an indexed key list (sm_100a tcgen05).
//
// One CTA computes 128 query rows against a list of key rows, 128 keys per step:
//   S_j  = Q K_j^T          tcgen05.mma kind::f16 (bf16 in, fp32 accumulate), TMEM
//   P_j  = exp2(S_j * c - m) softmax warps read S_j from TMEM, write bf16 P_j back
//                            over the first half of S_j's columns
//   O   += P_j V_j          tcgen05.mma accumulating in TMEM
// P is the A operand of the second MMA and is read from TMEM (the .kind::f16 form
// with [a_tmem]).
// m is the running row maximum used for the exponentials; it is raised (and O, l
// rescaled in place) only when a tile's maximum exceeds it by more than 2^8, so most
// tiles skip the rescale and P stays <= 2^8 (exact softmax either way: o = O / l).
// Roles (352 threads): warps 0-7 softmax (warp w owns TMEM lanes 32 (w % 4) .. + 31,
// i.e. rows, and key columns 64 (w / 4) .. + 63: two threads per row, exchanging the
// row max and sum through shared memory), warp 8 issues the MMAs (one lane), warp 9
// loads Q and the K tiles, warp 10 loads the V tiles.
// Tiles come in by TMA straight into the 128-byte swizzled layout the MMA descriptors
// name, and the "full" barriers complete on the transaction count. A tile whose 128
// keys are consecutive tokens (initial tokens, local window, chunk, MoBA blocks) is
// one 3D box per 64-column half ([tokens, heads, 128] map, one head); a tile of
// scattered keys (the selected middle tokens) is 32 tile::gather4 loads per half
// (4 arbitrary rows each; each lane of the loader warp issues its 4 rows).
//
// Shared memory: Q 32 KB, K 3 x 32 KB, V 3 x 32 KB (each operand tile is two 16 KB
// column blocks of 128 rows x 128 bytes). TMEM (512 columns): three S/P buffers at 0,
// 128 and 256, the O accumulator at 384.
// A group of MMAs that starts on an idle tensor pipe pays a fill latency of several
// hundred cycles, so the MMA warp keeps S two tiles ahead: right after PV_j it issues
// S_{j+3}, and the softmax warps find S_{j+1} ready when they finish P_j.
// P_j overwrites S_j, and S_{j+3} overwrites P_j. The MMA warp issues S_{j+3} only after
// PV_j, which it issues only after the softmax warps have signalled (p_full) that they
// have read S_j and stored P_j; the tensor pipe executes one thread's MMAs in issue
// order, so PV_j has read P_j before S_{j+3} is written.
//
// The problem policy P says which rows and keys a CTA owns:
//   bool setup(): per-CTA fields; false = nothing to do
//   int32_t q_row(int r): row of the Q row map for tile row r (-1: padding)
//   bool q_box(int* y, int* z): true if the Q tile is one box of the Q box map at (y, z)
//   int32_t kv_row(int64_t t): row of the K / V row maps for key t (t < n_keys())
//   int kv_box(int j, int* y, int* z): 1 if key tile j is one box of the K / V box maps
//        at (head y, token z), 2 if it is one box of the staged copies, 0 if gathered
//   int64_t n_keys(); int64_t limit(int r): last key index row r may attend
//   void store(int r, const float* o, float m2, float l): o is unnormalised,
//        m2 the running max in log2 units, l the denominator
#pragma once
#include <cuda.h>

#include <type_traits>
#include <utility>

#include "common.cuh"
#include "keylist.cuh"

namespace esa {

// Two softmax threads per row, 64 key columns each: the two warps of a row group on a
// sub-partition run in lockstep (they agree on the row maximum every tile), and with
// 64 independent exponentials per thread the pair keeps the MUFU busy where four
// warps of 32 columns stalled together (kTcSplit = 4: ESA chunk attention 72.3 ->
// 69.4 us at 2, MoBA 64K 9.27 -> 8.78 ms; one thread per row, with no exchange at
// all, measured slower: 74.5 us). 11 warps leave 168 registers a thread.
#ifndef KTC_SPLIT
#define KTC_SPLIT 2
#endif
constexpr int kTcSplit = KTC_SPLIT;                          // softmax threads per row (2 or 4)
static_assert(kTcSplit == 4 || kTcSplit == 2, "64 or 32 key columns per softmax thread");
constexpr int kTcThreads = (4 * kTcSplit + 3) * 32;
constexpr int kTcMmaWarp = 4 * kTcSplit, kTcKWarp = kTcMmaWarp + 1, kTcVWarp = kTcMmaWarp + 2;
constexpr int kTcRows = 128;
constexpr int kTcKeys = 128;
constexpr int kTcD = 128;
constexpr uint32_t kTileBytes = 128 * 256;            // 128 rows x 128 bf16
constexpr uint32_t kBlkBytes = 128 * 128;             // one 64-column block of a tile
constexpr uint32_t kTcCtrlBytes = 3072;                       // barriers, TMEM address, row exchange
// No alignment slack: the kernel checks that the dynamic shared memory starts on a
// 1024-byte boundary (the 128-byte swizzle atoms need it) and stops with an error if not.
constexpr int kTcKStages = 3, kTcVStages = 3;
constexpr uint32_t kTcSmemBytes = (1 + kTcKStages + kTcVStages) * kTileBytes + kTcCtrlBytes;
constexpr int kTcSBufs = 3;                                   // S/P buffers in TMEM
constexpr uint32_t kTmemO = 384;                              // O accumulator column
static_assert(kTcSmemBytes <= 232448, "exceeds the 227 KB of shared memory per CTA");

struct TcSmem {
  uint64_t q_full;
  uint64_t k_full[kTcKStages], k_empty[kTcKStages], v_full[kTcVStages], v_empty[kTcVStages];
  uint64_t s_full[kTcSBufs], p_full[kTcSBufs];
  // PV_j completes pv_full[j % 3]. The softmax waits on it only now and then (a
  // rescale, the epilogue), and a parity wait is sound only if the slot's previous
  // phase has completed. Once S_j is seen complete, PV_{j-3} is (S_j was issued after
  // it, and a commit covers every earlier MMA), so three slots make every such wait
  // safe; with two, the epilogue's wait could pass on PV_{j-2}'s phase still open.
  uint64_t pv_full[3];
  uint64_t mma_done;
  uint32_t tmem_base;
  int abort_flag;
  float red[kTcSplit][128];  // per-row partial max / sum of the column parts
};
static_assert(sizeof(TcSmem) <= kTcCtrlBytes, "control block overflows its reservation");

// Gather 128 rows of a [rows, 128] bf16 tensor into one swizzled tile (two 64-column
// blocks). Lane l issues rows 4l..4l+3; row ids < 0 are replaced by `fallback` (a
// valid row whose data the caller masks out). Caller has set the expected bytes.
__device__ __forceinline__ void gather_tile(uint32_t dst, const CUtensorMap* tm, const int32_t* rows4,
                                            int32_t fallback, uint64_t* bar, int lane) {
  int32_t r[4];
#pragma unroll
  for (int q = 0; q < 4; ++q) r[q] = rows4[q] >= 0 ? rows4[q] : fallback;
  const uint32_t d = dst + lane * 4 * 128;
  tma_gather4(d, tm, 0, r[0], r[1], r[2], r[3], bar);
  tma_gather4(d + kBlkBytes, tm, 64, r[0], r[1], r[2], r[3], bar);
}

// One loader warp streams nt key tiles of one operand (K or V), tiles j0, j0 + js,
// j0 + 2 js, ..., through its NST stages (the u-th of them, tile j0 + u js, in stage
// u % NST, the barrier's u / NST-th phase). The rows of the next tile are looked up (4 per lane,
// consecutive keys, so a gathered index list is read coalesced) while the current one
// waits for its stage.
template <int NST, class Problem>
__device__ __forceinline__ void stream_kv(const Problem& prob, const CUtensorMap* tm_rows, const CUtensorMap* tm_box,
                                          const CUtensorMap* tm_staged, uint32_t stage0, uint64_t* full,
                                          uint64_t* empty, int nt, int64_t n_keys, int lane,
                                          volatile int* abort_flag, unsigned site, int j0 = 0, int js = 1) {
  int32_t cur[4], nxt[4];
  auto fetch = [&](int j, int32_t* out) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int64_t t = (int64_t)j * kTcKeys + lane * 4 + q;
      out[q] = t < n_keys ? prob.kv_row(t) : -1;
    }
  };
  if (nt == 0) return;
  const int32_t fallback = prob.kv_row(0);
  int by = 0, bz = 0;
  int box_next = prob.kv_box(j0, &by, &bz);       // 0: gather, 1: cache box, 2: staged box
  if (!box_next) fetch(j0, nxt);
  for (int u = 0; u < nt; ++u) {
    const int s = u % NST;
    const int ph = (u / NST) & 1;
    const int box = box_next;
    const int y = by, z = bz;
#pragma unroll
    for (int q = 0; q < 4; ++q) cur[q] = nxt[q];
    if (u + 1 < nt) {
      box_next = prob.kv_box(j0 + (u + 1) * js, &by, &bz);
      if (!box_next) fetch(j0 + (u + 1) * js, nxt);
    }
    bool ok = mbar_wait(&empty[s], ph ^ 1, abort_flag, site);
    if (!__all_sync(0xffffffffu, ok)) return;
    const uint32_t dst = stage0 + s * kTileBytes;
    if (box) {
      if (lane == 0) {
        const CUtensorMap* tm = box == 2 ? tm_staged : tm_box;
        mbar_arrive_expect_tx(&full[s], kTileBytes);
        tma_load_3d(dst, tm, 0, y, z, &full[s]);
        tma_load_3d(dst + kBlkBytes, tm, 64, y, z, &full[s]);
      }
    } else {
      if (lane == 0) mbar_arrive_expect_tx(&full[s], kTileBytes);
      __syncwarp();
      gather_tile(dst, tm_rows, cur, fallback, &full[s], lane);
    }
  }
}

// Optional hook: a policy with `void prefetch(int r, int col0)` has it called by each
// softmax thread before the key loop, to start loads its store() will need.
template <class P, class = void>
struct HasPrefetch : std::false_type {};
template <class P>
struct HasPrefetch<P, std::void_t<decltype(std::declval<P&>().prefetch(0, 0))>> : std::true_type {};

template <class Problem>
__global__ void __launch_bounds__(kTcThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tb_q,
                   const __grid_constant__ CUtensorMap tb_k, const __grid_constant__ CUtensorMap tb_v,
                   const __grid_constant__ CUtensorMap ts_k, const __grid_constant__ CUtensorMap ts_v,
                   Problem prob) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = smem_raw;
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) record_status(5u, 100);
    return;
  }
  const uint32_t sQ = smem_u32(smem);
  const uint32_t sK = sQ + kTileBytes;
  const uint32_t sV = sK + kTcKStages * kTileBytes;
  TcSmem& sm = *reinterpret_cast<TcSmem*>(smem + (1 + kTcKStages + kTcVStages) * kTileBytes);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (!prob.setup()) return;
  const int64_t n_keys = prob.n_keys();
  const int nt = (int)((n_keys + kTcKeys - 1) / kTcKeys);

  if (threadIdx.x == 0) {
    mbar_init(&sm.q_full, 1);
    for (int s = 0; s < kTcKStages; ++s) {
      mbar_init(&sm.k_full[s], 1);
      mbar_init(&sm.k_empty[s], 1);
    }
    for (int s = 0; s < kTcVStages; ++s) {
      mbar_init(&sm.v_full[s], 1);
      mbar_init(&sm.v_empty[s], 1);
    }
    for (int s = 0; s < kTcSBufs; ++s) {
      mbar_init(&sm.s_full[s], 1);
      mbar_init(&sm.p_full[s], 4 * kTcSplit);        // one arrival per softmax warp
    }
    for (int s = 0; s < 3; ++s) mbar_init(&sm.pv_full[s], 1);
    mbar_init(&sm.mma_done, 1);
    sm.abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == kTcMmaWarp) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == kTcKWarp) {
    // ---------------------------------------------------------------- Q + K loader
    int qy = 0, qz = 0;
    if (prob.q_box(&qy, &qz)) {
      if (lane == 0) {
        mbar_arrive_expect_tx(&sm.q_full, kTileBytes);
        tma_load_3d(sQ, &tb_q, 0, qy, qz, &sm.q_full);
        tma_load_3d(sQ + kBlkBytes, &tb_q, 64, qy, qz, &sm.q_full);
      }
    } else {
      int32_t qr[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) qr[q] = prob.q_row(lane * 4 + q);
      const int32_t q_fallback = __shfl_sync(0xffffffffu, qr[0], 0);    // row 0 is always a real query
      if (lane == 0) mbar_arrive_expect_tx(&sm.q_full, kTileBytes);
      __syncwarp();
      gather_tile(sQ, &tm_q, qr, q_fallback, &sm.q_full, lane);
    }
    stream_kv<kTcKStages>(prob, &tm_k, &tb_k, &ts_k, sK, sm.k_full, sm.k_empty, nt, n_keys, lane, abort_flag, 101);
  } else if (warp == kTcVWarp) {
    // ---------------------------------------------------------------- V loader
    stream_kv<kTcVStages>(prob, &tm_v, &tb_v, &ts_v, sV, sm.v_full, sm.v_empty, nt, n_keys, lane, abort_flag, 102);
  } else if (warp == kTcMmaWarp) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_qk = umma_idesc(kFmtBF16, 128, 128, 0, 0);
      constexpr uint32_t idesc_pv = umma_idesc(kFmtBF16, 128, 128, 0, 1);
      // This thread shares its issue slots with four busy softmax warps, so the loops
      // below do as little as possible per MMA: descriptors are built once and only the
      // low word moves (16-byte units: K step kk of a K-major operand is +2 kk within a
      // 64-column block and +1024 per block; of the MN-major V tile, +128 kk).
      const uint64_t dq = sdesc_sw128(sQ, 16, 1024), dk = sdesc_sw128(sK, 16, 1024);
      const uint64_t dv = sdesc_sw128(sV, kBlkBytes, 1024);
      const uint32_t q_lo = (uint32_t)dq, q_hi = (uint32_t)(dq >> 32);
      const uint32_t k_lo = (uint32_t)dk, k_hi = (uint32_t)(dk >> 32);
      const uint32_t v_lo = (uint32_t)dv, v_hi = (uint32_t)(dv >> 32);
      auto issue_s = [&](int j) -> bool {
        const int s = j % kTcSBufs, ks = j % kTcKStages;
        // buffer s last held P_{j-3}: PV_{j-3} is already issued (p_full[s] was waited for)
        if (!mbar_wait(&sm.k_full[ks], (j / kTcKStages) & 1, abort_flag, 103)) return false;
        tc_fence_after();
        const uint32_t kb = k_lo + ks * (kTileBytes >> 4), d = tmem + s * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * (kBlkBytes >> 4) + (kk & 3) * 2;
          umma_f16_ss2(d, q_lo + off, q_hi, kb + off, k_hi, idesc_qk, kk > 0);
        }
        umma_commit(&sm.s_full[s]);
        umma_commit(&sm.k_empty[ks]);
        return true;
      };
      bool ok = nt == 0 || mbar_wait(&sm.q_full, 0, abort_flag, 105);
      for (int j = 0; j < kTcSBufs - 1 && j < nt && ok; ++j) ok = issue_s(j);
      for (int j = 0; j < nt && ok; ++j) {
        const int s = j % kTcSBufs, vs = j % kTcVStages;
        if (j + kTcSBufs - 1 < nt && !(ok = issue_s(j + kTcSBufs - 1))) break;
        if (!(ok = mbar_wait(&sm.p_full[s], (j / kTcSBufs) & 1, abort_flag, 106))) break;
        if (!(ok = mbar_wait(&sm.v_full[vs], (j / kTcVStages) & 1, abort_flag, 107))) break;
        tc_fence_after();
        const uint32_t vb = v_lo + vs * (kTileBytes >> 4), pa = tmem + s * 128;
        const uint32_t acc0 = j > 0;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // A = P from TMEM (keys 16 kk .. + 15 in columns 8 kk .. + 7 of buffer s);
          // B = V (MN-major: 8-key row groups of 1024 bytes, d blocks 16 KB apart)
          umma_f16_ts2(tmem + kTmemO, pa + kk * 8, vb + kk * 128, v_hi, idesc_pv, kk > 0 ? 1u : acc0);
        }
        umma_commit(&sm.pv_full[j % 3]);
        umma_commit(&sm.v_empty[vs]);
      }
      // every MMA issued so far has completed before TMEM is released
      umma_commit(&sm.mma_done);
      mbar_wait(&sm.mma_done, 0, abort_flag, 109, /*respect_abort=*/false);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- softmax (rows)
    constexpr int HC = kTcKeys / kTcSplit;     // key columns per thread (32 or 64)
    // HC columns of 32-bit TMEM data at addr (HC / 32 loads of 32 columns)
    auto ld_cols = [&](uint32_t addr, float* dst) {
#pragma unroll
      for (int c = 0; c < HC / 32; ++c) tmem_ld32(addr + c * 32, dst + c * 32);
    };
    // half a tile's P of this thread: HC / 4 packed bf16 pairs
    auto st_p = [&](uint32_t addr, const uint32_t* pk) {
      if constexpr (HC == 32) tmem_st8(addr, pk);
      else tmem_st16(addr, pk);
    };
    constexpr uint32_t kGroup = 32 * kTcSplit; // threads sharing a row set (named barrier size)
    const int quad = warp & 3, part = warp >> 2;
    const int r = quad * 32 + lane;            // row = TMEM lane
    const uint32_t lane_base = tmem + ((uint32_t)(quad * 32) << 16);
    const uint32_t o_addr = lane_base + kTmemO + part * HC;
    const uint32_t row_bar = 1 + quad;         // named barrier of the kTcSplit warps of this quadrant
    // O *= alpha for this thread's columns, 32 at a time (few live registers)
    auto rescale_o = [&](float alpha) {
#pragma unroll 1
      for (int c = 0; c < HC / 32; ++c) {
        float ov[32];
        tmem_ld32(o_addr + c * 32, ov);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) ov[e] *= alpha;
        tmem_st32(o_addr + c * 32, ov);
      }
      tmem_wait_st();
    };
    if constexpr (HasPrefetch<Problem>::value) prob.prefetch(r, part * (kTcD / kTcSplit));
    const int64_t lim = prob.limit(r);
    const float sl2 = prob.scale_log2();
    constexpr float kRescale = 8.0f;           // log2 units: rescale when the max grows by > 2^8
    float m = -INFINITY, l = 0.f;
    bool ok = true;

    // Keys t0 + e of tile j with e <= rem are visible (causal cut); rem >= HC - 1: all.
    auto rem_of = [&](int j) -> int {
      const int64_t rem64 = lim - ((int64_t)j * kTcKeys + part * HC);
      return rem64 < 0 ? -1 : (rem64 >= HC ? HC : (int)rem64);
    };
    // Wait for S_j; then load_s starts loading this thread's scores (complete at
    // tmem_wait_ld).
    auto wait_s = [&](int j) -> bool {
      const bool got = mbar_wait_warp(&sm.s_full[j % kTcSBufs], (j / kTcSBufs) & 1, abort_flag, 111);
      if (got) tc_fence_after();
      return got;
    };
    auto load_s = [&](int j, float* dst) { ld_cols(lane_base + (j % kTcSBufs) * 128 + part * HC, dst); };
    // Masked scores become -inf; returns this part's maximum in log2 units (scale > 0).
    auto mask_max = [&](int rem, float* v) -> float {
      float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
      if (rem >= HC - 1) {
#pragma unroll
        for (int e = 0; e < HC; ++e) m4[e & 3] = fmaxf(m4[e & 3], v[e]);
      } else {
#pragma unroll
        for (int e = 0; e < HC; ++e) {
          v[e] = e <= rem ? v[e] : -INFINITY;
          m4[e & 3] = fmaxf(m4[e & 3], v[e]);
        }
      }
      return fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
    };
    // The kTcSplit warps of a row group meet once per tile at a bar.red.or: unless some
    // part's maximum exceeds m by more than 2^8 (or a wait of some warp ran out), m stays
    // and no exchange is needed. Otherwise they agree on success (bar_all: a named
    // barrier has no timeout, so all warps of a group leave together), exchange the part
    // maxima through shared memory, and rescale O (which then holds PV_0 .. PV_{j-1})
    // and l. Returns false when the group has to stop.
    auto decide = [&](int j, float mx) -> bool {
      if (!bar_any(row_bar, kGroup, !ok || mx > m + kRescale)) return true;   // -inf + 8 = -inf
      if (!(ok = bar_all(row_bar, kGroup, ok))) return false;
      sm.red[part][r] = mx;
      asm volatile("bar.sync %0, %1;" ::"r"(row_bar), "r"(kGroup) : "memory");
#pragma unroll
      for (int q = 0; q < kTcSplit; ++q) mx = fmaxf(mx, sm.red[q][r]);
      asm volatile("bar.sync %0, %1;" ::"r"(row_bar), "r"(kGroup) : "memory");   // red[] is reused
      const float m_new = fmaxf(m, mx);        // > m + 2^8 for the whole row group
      if (m != -INFINITY) {
        const float alpha = fast_exp2(m - m_new);
        const bool done = mbar_wait_warp(&sm.pv_full[(j - 1) % 3], ((j - 1) / 3) & 1, abort_flag, 110);
        if (!(ok = bar_all(row_bar, kGroup, done))) return false;
        tc_fence_after();
        rescale_o(alpha);
        l *= alpha;
      }
      m = m_new;
      return true;
    };
    // One tile, software-pipelined: cur holds S_j (masked, m decided). P_j is formed in
    // two halves (MUFU exp2); S_{j+1} is loaded into nxt after the first half (when half
    // of cur is no longer needed, which keeps the live registers within what a thread
    // has here), and its maximum is taken between the exponentials of the second half,
    // so the ALU reduction hides behind the exp2 unit. P_j goes to
    // the TMEM buffer over S_j (every warp of the row group has read its part of S_j,
    // the barrier in decide), keys HC part .. + HC - 1 to columns HC / 2 part .. +
    // HC / 2 - 1. Then the group decides m for tile j + 1. Returns false when there is
    // no next tile or the group has to stop.
    auto step = [&](int j, float* cur, float* nxt) -> bool {
      const int s = j % kTcSBufs;
      const bool has_next = j + 1 < nt;
      const bool got_n = has_next && wait_s(j + 1);
      const int rem_n = has_next ? rem_of(j + 1) : HC;
      const float m_use = m == -INFINITY ? 0.f : m;
      const float2 scale2 = make_float2(sl2, sl2), shift2 = make_float2(-m_use, -m_use);
      float2 ls2[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
      uint32_t pk[HC / 4];
      // P goes to the MMA as bf16, rounded to nearest (unbiased, so l may add the
      // unrounded values)
      auto pair = [&](int e) -> uint32_t {
        const float2 t = __ffma2_rn(make_float2(cur[e], cur[e + 1]), scale2, shift2);
        const float2 pe = make_float2(fast_exp2(t.x), fast_exp2(t.y));
        ls2[(e >> 1) & 1] = __fadd2_rn(ls2[(e >> 1) & 1], pe);
        const __nv_bfloat162 h = __floats2bfloat162_rn(pe.x, pe.y);
        return *reinterpret_cast<const uint32_t*>(&h);
      };
#pragma unroll
      for (int e = 0; e < HC / 2; e += 2) pk[e / 2] = pair(e);
      st_p(lane_base + s * 128 + part * (HC / 2), pk);
      float mx_n = -INFINITY;
      if (got_n) {
        load_s(j + 1, nxt);
        tmem_wait_ld();
      }
      if (__all_sync(0xffffffffu, got_n && rem_n >= HC - 1)) {
        float m4[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int e = HC / 2; e < HC; e += 2) {
          pk[(e - HC / 2) / 2] = pair(e);
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int f = (e - HC / 2) * 2 + q;             // 4 of S_{j+1} per pair of P_j
            m4[q] = fmaxf(m4[q], nxt[f]);
          }
        }
        mx_n = fmaxf(fmaxf(m4[0], m4[1]), fmaxf(m4[2], m4[3])) * sl2;
      } else {
#pragma unroll
        for (int e = HC / 2; e < HC; e += 2) pk[(e - HC / 2) / 2] = pair(e);
        if (got_n) mx_n = mask_max(rem_n, nxt);
      }
      st_p(lane_base + s * 128 + part * (HC / 2) + HC / 4, pk);
      const float2 l2 = __fadd2_rn(ls2[0], ls2[1]);
      l += l2.x + l2.y;
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive_warp(&sm.p_full[s]);
      if (!has_next) return false;
      ok = ok && got_n;
      return decide(j + 1, mx_n);
    };

    float xa[HC], xb[HC];
    if (nt > 0) {
      const bool got = wait_s(0);
      float mx = -INFINITY;
      if (got) {
        load_s(0, xa);
        tmem_wait_ld();
        mx = mask_max(rem_of(0), xa);
      }
      ok = ok && got;
      if (decide(0, mx)) {
        for (int j = 0; j < nt; ++j) {
          if (!step(j, xa, xb)) break;
#pragma unroll
          for (int e = 0; e < HC; ++e) xa[e] = xb[e];
        }
      }
    }
    bool fin = ok;
    if (ok && nt > 0) fin = mbar_wait_warp(&sm.pv_full[(nt - 1) % 3], ((nt - 1) / 3) & 1, abort_flag, 113);
    ok = bar_all(row_bar, kGroup, fin);        // every warp of the row group gets here
    sm.red[part][r] = l;
    asm volatile("bar.sync %0, %1;" ::"r"(row_bar), "r"(kGroup) : "memory");
    float l_row = 0.f;
#pragma unroll
    for (int q = 0; q < kTcSplit; ++q) l_row += sm.red[q][r];
    if (ok) {
      tc_fence_after();
      float o[HC];
      ld_cols(o_addr, o);
      tmem_wait_ld();
      prob.store(r, part * HC, o, m, l_row);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kTcMmaWarp) tmem_dealloc(tmem, 512);
}

// ------------------------------------------------------------------ ESA problem --
// CTA (row tile, KV head g, sequence b). Row R = tile * 128 + r packs (query i, head
// in group hl) as i = R / G, hl = R % G, so each loaded K/V row serves G query heads.
struct EsaTcProblem {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  __nv_bfloat16* o;
  float* lse;
  KeyList keys;
  int64_t n_cap, c0;
  int lq, hq, hkv, G;
  float sl2;
  int staged;            // selected K/V rows were copied to contiguous buffers
  int lists;             // key lists per sequence: 1, or Hkv (one per KV head)
  // per CTA
  int b, g, tile, cnt, list;
  int64_t n_prior, nk;

  __device__ bool setup() { return setup_at(blockIdx.x); }
  __device__ bool setup_at(int t) {
    tile = t;
    g = blockIdx.y;
    b = blockIdx.z;
    list = lists > 1 ? b * lists + g : b;
    cnt = min(max(keys.count[list], 0), (int)keys.idx_stride);
    n_prior = keys.ni + cnt + (c0 - keys.lo);
    const int rows = lq * G;
    if (tile * kTcRows >= rows) return false;
    const int imax = min(lq - 1, (tile * kTcRows + kTcRows - 1) / G);
    nk = n_prior + imax + 1;
    return true;
  }
  __device__ int32_t q_row(int r) const {
    const int R = tile * kTcRows + r;
    if (R >= lq * G) return -1;
    const int i = R / G, hl = R % G;
    return (int32_t)(((int64_t)b * lq + i) * hq + g * G + hl);
  }
  __device__ int32_t kv_row(int64_t t) const {
    return (int32_t)(((int64_t)b * n_cap + keys.pos(list, cnt, t)) * hkv + g);
  }
  // Q tile = 128 / G consecutive queries x the G heads of group g: one box of the
  // [B * lq, hq, 128] map (rows past the chunk belong to no stored output)
  __device__ bool q_box(int* y, int* z) const {
    *y = g * G;
    *z = (int)((int64_t)b * lq + (tile * kTcRows) / G);
    return true;
  }
  // a key tile inside the initial tokens or inside the local part (window + chunk) is
  // 128 consecutive tokens of the cache; one inside the selected tokens is 128
  // consecutive rows of the staged copy [B, topk, Hkv, D]; keys past n_keys are loaded
  // but masked by limit()
  __device__ int kv_box(int j, int* y, int* z) const {
    const int64_t t0 = (int64_t)j * kTcRows, t1 = t0 + kTcRows - 1;
    *y = g;
    if (t1 < keys.ni) {
      *z = (int)((int64_t)b * n_cap + t0);
      return 1;
    }
    if (t0 >= keys.ni + cnt) {
      *z = (int)((int64_t)b * n_cap + keys.lo + (t0 - keys.ni - cnt));
      return 1;
    }
    if (staged && t0 >= keys.ni && t1 < keys.ni + cnt) {
      *z = (int)((int64_t)b * keys.idx_stride + (t0 - keys.ni));
      return 2;
    }
    return 0;
  }
  __device__ int64_t n_keys() const { return nk; }
  __device__ int64_t limit(int r) const {
    const int R = tile * kTcRows + r;
    return n_prior + min(R / G, lq - 1);
  }
  __device__ float scale_log2() const { return sl2; }
  // columns [col0, col0 + kTcD / kTcSplit) of row r; the LSE comes with the first part
  __device__ void store(int r, int col0, const float* acc, float m2, float l) {
    const int R = tile * kTcRows + r;
    if (R >= lq * G) return;
    const int i = R / G, hl = R % G;
    const int64_t row = ((int64_t)b * lq + i) * hq + g * G + hl;
    const float inv = 1.f / l;
    uint4* dst = reinterpret_cast<uint4*>(o + row * kTcD + col0);
#pragma unroll
    for (int c = 0; c < kTcD / kTcSplit / 8; ++c) {
      uint4 w;
      w.x = pack_bf16x2(acc[8 * c + 0] * inv, acc[8 * c + 1] * inv);
      w.y = pack_bf16x2(acc[8 * c + 2] * inv, acc[8 * c + 3] * inv);
      w.z = pack_bf16x2(acc[8 * c + 4] * inv, acc[8 * c + 5] * inv);
      w.w = pack_bf16x2(acc[8 * c + 6] * inv, acc[8 * c + 7] * inv);
      dst[c] = w;
    }
    if (lse && col0 == 0) lse[row] = (m2 + __log2f(l)) * 0.69314718055994531f;
  }
};

}  // namespace esa

namespace esa {

// Copy the selected K and V rows of every sequence into contiguous buffers
// [B, topk, Hkv, D] (all heads of a token are one contiguous row of Hkv * D elements),
// so that the attention kernel loads selected keys as boxes instead of row gathers.
// With one list per KV head (lists = Hkv), slot t of head g holds the row of head g
// of that head's t-th selected token. One CTA per (selected entry, list); 16-byte
// pieces. row_vec: 16-byte pieces of one token's row (all heads); head_vec: of one head.
__global__ void __launch_bounds__(256) gather_selected_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                                                              const int32_t* __restrict__ idx,
                                                              const int32_t* __restrict__ count, int64_t n_cap,
                                                              int topk, int row_vec, int lists, int head_vec,
                                                              uint4* __restrict__ ks, uint4* __restrict__ vs) {
  const int list = blockIdx.y;
  const int b = list / lists, g = list % lists;
  const int cnt = min(max(count[list], 0), topk);
  const int width = lists > 1 ? head_vec : row_vec;        // pieces copied per entry
  const int off = lists > 1 ? g * head_vec : 0;
  for (int t = blockIdx.x; t < cnt; t += gridDim.x) {
    int64_t p = idx[(int64_t)list * topk + t];
    p = p < 0 ? 0 : (p >= n_cap ? n_cap - 1 : p);
    const uint4* ksrc = k + ((int64_t)b * n_cap + p) * row_vec + off;
    const uint4* vsrc = v + ((int64_t)b * n_cap + p) * row_vec + off;
    uint4* kd = ks + ((int64_t)b * topk + t) * row_vec + off;
    uint4* vd = vs + ((int64_t)b * topk + t) * row_vec + off;
    for (int e = threadIdx.x; e < width; e += blockDim.x) {
      kd[e] = ld_stream16(ksrc + e);
      vd[e] = ld_stream16(vsrc + e);
    }
  }
}

}  // namespace esa
