// moba.cuh - Mixture of Block Attention (MoBA article, sections 2-3).
//
//   block means   Kbar[b, h, blk] = mean of K over block blk (fp32)
//   gate          s_blk = <q, Kbar[blk]> for past blocks blk < cur; keep the top
//                 min(topk, cur) by (score desc, block asc); add the current block
//   attention     softmax over the kept blocks, the current block cut causally
//
// The attention is grouped by key block instead of by query: for every (sequence,
// head, past block) the queries that chose that block form a list, and one tensor-core
// CTA attends 128 listed queries to the block's contiguous keys. Each (query, head)
// thereby gets one partial per attended past block, written to its slot (the block's
// rank in the query's list) as a normalised bf16 row and a base-2 log-sum-exp. The
// CTA that attends a query tile to its own (current) block, causally, runs after them
// and merges the tile's past partials into its result by log-sum-exp in its epilogue,
// writing the output. The work is exactly the selected (query, block) pairs, so no
// key is attended that the gate did not keep.
#pragma once
#include <cub/block/block_scan.cuh>

#include "attn_tc.cuh"
#include "common.cuh"

namespace esa {

constexpr int kMobaMaxTopk = 15;

// ------------------------------------------------------------------ block means --
// grid (n_blocks, H, B), 256 threads: thread = (d pair, row phase); fixed order sums.
template <typename T>
// Blocks [blk0, blk0 + gridDim.x) of kbar [B, H, nb_total, D].
__global__ void __launch_bounds__(256) moba_mean_kernel(const T* __restrict__ k, int64_t seq, int heads, int d,
                                                        int block, int blk0, int nb_total, float* __restrict__ kbar) {
  __shared__ float part[256][2];
  const int blk = blk0 + (int)blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int pairs = d / 2;
  const int dp = threadIdx.x % pairs;
  const int ph = threadIdx.x / pairs;
  const int nph = 256 / pairs;
  const int64_t r0 = (int64_t)blk * block;
  const int64_t r1 = min(seq, r0 + block);
  float a0 = 0.f, a1 = 0.f;
  for (int64_t r = r0 + ph; r < r1; r += nph) {
    const T* p = k + ((b * seq + r) * heads + h) * d + 2 * dp;
    a0 += static_cast<float>(p[0]);
    a1 += static_cast<float>(p[1]);
  }
  part[threadIdx.x][0] = a0;
  part[threadIdx.x][1] = a1;
  __syncthreads();
  if (threadIdx.x < pairs) {
    float s0 = 0.f, s1 = 0.f;
    for (int q = 0; q < nph; ++q) {
      s0 += part[q * pairs + threadIdx.x][0];
      s1 += part[q * pairs + threadIdx.x][1];
    }
    const float inv = 1.f / (float)(r1 - r0);
    float* o = kbar + (((int64_t)b * heads + h) * nb_total + blk) * d + 2 * threadIdx.x;
    o[0] = s0 * inv;
    o[1] = s1 * inv;
  }
}

// ------------------------------------------------------------------ gate --
// grid (ceil(seq / 128), H, B), 128 threads; thread = query position. The query row
// lives in registers; block means are staged 32 blocks at a time in shared memory and
// read as broadcasts. Kept list: insertion that never moves an element past an equal
// one, visiting blocks in ascending order -> ties go to the lower block. TK >= topk is
// the kept list's compile-time length: the insertion runs over TK entries for every
// block, so the host picks the smallest instantiation that holds topk.
template <typename T, int D, int TK>
__global__ void __launch_bounds__(128) moba_gate_kernel(const T* __restrict__ q, const float* __restrict__ kbar,
                                                        int64_t seq, int heads, int block, int n_blocks, int topk,
                                                        int16_t* __restrict__ blocks_out) {
  constexpr int CB = 32;
  __shared__ float4 kb[CB][D / 4];
  const int h = blockIdx.y, b = blockIdx.z;
  const int64_t p = (int64_t)blockIdx.x * 128 + threadIdx.x;
  const bool valid = p < seq;
  const int cur = valid ? (int)(p / block) : 0;
  const int64_t p_last = min(seq - 1, (int64_t)blockIdx.x * 128 + 127);
  const int cur_max = (int)(p_last / block);
  float qv[D];
  if (valid) {
    const T* qp = q + ((b * seq + p) * heads + h) * D;
#pragma unroll
    for (int e = 0; e < D; e += 16 / sizeof(T)) load_vec(qp + e, &qv[e]);
  }
  float vals[TK];
  int ids[TK];
#pragma unroll
  for (int i = 0; i < TK; ++i) { vals[i] = -INFINITY; ids[i] = -1; }
  const float* kbh = kbar + ((int64_t)b * heads + h) * n_blocks * D;
  for (int c0 = 0; c0 < cur_max; c0 += CB) {
    __syncthreads();
    for (int t = threadIdx.x; t < CB * D / 4; t += 128) {
      const int c = t / (D / 4), e = t % (D / 4);
      kb[c][e] = (c0 + c < n_blocks) ? reinterpret_cast<const float4*>(kbh + (int64_t)(c0 + c) * D)[e]
                                     : make_float4(0.f, 0.f, 0.f, 0.f);
    }
    __syncthreads();
    if (!valid) continue;
    const int cend = min(CB, cur - c0);
    // two blocks at a time, four partial sums each: eight independent FMA chains (one
    // chain of D dependent FMAs per block left the FMA pipe waiting on its latency)
    for (int c = 0; c < cend; c += 2) {
      float a0[4] = {0.f, 0.f, 0.f, 0.f}, a1[4] = {0.f, 0.f, 0.f, 0.f};
      const int c1 = c + 1 < CB ? c + 1 : c;       // (a block past cend is computed, not kept)
#pragma unroll
      for (int e = 0; e < D / 4; ++e) {
        const float4 w = kb[c][e], x = kb[c1][e];
        a0[0] = fmaf(qv[4 * e], w.x, a0[0]);
        a0[1] = fmaf(qv[4 * e + 1], w.y, a0[1]);
        a0[2] = fmaf(qv[4 * e + 2], w.z, a0[2]);
        a0[3] = fmaf(qv[4 * e + 3], w.w, a0[3]);
        a1[0] = fmaf(qv[4 * e], x.x, a1[0]);
        a1[1] = fmaf(qv[4 * e + 1], x.y, a1[1]);
        a1[2] = fmaf(qv[4 * e + 2], x.z, a1[2]);
        a1[3] = fmaf(qv[4 * e + 3], x.w, a1[3]);
      }
      const float s2[2] = {(a0[0] + a0[1]) + (a0[2] + a0[3]), (a1[0] + a1[1]) + (a1[2] + a1[3])};
#pragma unroll
      for (int q2 = 0; q2 < 2; ++q2) {
        if (c + q2 >= cend) break;
        float v = s2[q2];
        int id = c0 + c + q2;
#pragma unroll
        for (int i = 0; i < TK; ++i) {
          if (i < topk && v > vals[i]) {
            const float tv = vals[i]; vals[i] = v; v = tv;
            const int ti = ids[i]; ids[i] = id; id = ti;
          }
        }
      }
    }
  }
  if (!valid) return;
  // ascending block order: small unrolled exchange sort on the kept ids (-1 last)
#pragma unroll
  for (int i = 0; i < TK; ++i)
#pragma unroll
    for (int j = 0; j + 1 < TK - i; ++j) {
      const int a = ids[j], c = ids[j + 1];
      const bool swap = (a < 0 && c >= 0) || (a >= 0 && c >= 0 && c < a);
      ids[j] = swap ? c : a;
      ids[j + 1] = swap ? a : c;
    }
  int16_t* out = blocks_out + ((b * seq + p) * heads + h) * (topk + 1);
  int n = 0;
#pragma unroll
  for (int i = 0; i < TK; ++i)
    if (i < topk && ids[i] >= 0) out[n++] = (int16_t)ids[i];
  out[n++] = (int16_t)cur;
  for (; n < topk + 1; ++n) out[n] = -1;
}

// ------------------------------------------------------------------ query lists --
// For each (b, p, h) and each past block in its list (the first min(topk, p / block)
// entries), count (pass 0) or append (pass 1) the pair (p, slot) to the list of
// (b, h, block). The order inside a list is not fixed, but every pair owns its own
// output slot, so the results do not depend on it.
//
// grid (query blocks, H, B): a CTA takes the queries of one query block c for one head.
// They all choose among the same past blocks (< c), so their entries are counted in
// shared memory first and each past block costs one global atomic per CTA (pass 0: add
// the count; pass 1: reserve the CTA's range of the list) instead of one per entry.
constexpr int kMobaListThreads = 256;

__global__ void __launch_bounds__(kMobaListThreads) moba_list_kernel(const int16_t* __restrict__ blocks, int64_t seq,
                                                                     int heads, int block, int n_blocks, int topk,
                                                                     int pass, uint32_t* __restrict__ cnt,
                                                                     const uint32_t* __restrict__ off,
                                                                     uint32_t* __restrict__ fill,
                                                                     uint32_t* __restrict__ list) {
  extern __shared__ uint32_t lsm[];        // [n_blocks] counts, then [n_blocks] bases / cursors
  uint32_t* c_s = lsm;
  uint32_t* base_s = lsm + n_blocks;
  const int c = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int64_t p0 = (int64_t)c * block, p1 = min(seq, p0 + block);
  for (int i = threadIdx.x; i < c; i += kMobaListThreads) c_s[i] = 0;
  __syncthreads();
  const int n_past = min(topk, c);         // the same for every query of the block
  for (int64_t p = p0 + threadIdx.x; p < p1; p += kMobaListThreads) {
    const int16_t* lst = blocks + (((int64_t)b * seq + p) * heads + h) * (topk + 1);
    for (int s2 = 0; s2 < n_past; ++s2) {
      const int blk = lst[s2];
      if (blk < 0 || blk >= c) break;
      atomicAdd(&c_s[blk], 1u);
    }
  }
  __syncthreads();
  const int64_t lbase = ((int64_t)b * heads + h) * n_blocks;
  if (pass == 0) {
    for (int i = threadIdx.x; i < c; i += kMobaListThreads)
      if (c_s[i]) atomicAdd(&cnt[lbase + i], c_s[i]);
    return;
  }
  for (int i = threadIdx.x; i < c; i += kMobaListThreads)
    base_s[i] = c_s[i] ? off[lbase + i] + atomicAdd(&fill[lbase + i], c_s[i]) : 0u;
  __syncthreads();
  for (int64_t p = p0 + threadIdx.x; p < p1; p += kMobaListThreads) {
    const int16_t* lst = blocks + (((int64_t)b * seq + p) * heads + h) * (topk + 1);
    for (int s2 = 0; s2 < n_past; ++s2) {
      const int blk = lst[s2];
      if (blk < 0 || blk >= c) break;
      const uint32_t at = atomicAdd(&base_s[blk], 1u);
      list[at] = ((uint32_t)p << 4) | (uint32_t)s2;
    }
  }
}

// Exclusive scans over all lists: entry offsets and offsets of units of unit_rows rows
// (a pair of 128-row tiles: 256); then unit_list[u] = the list of unit u (n_lists for
// u past the last unit, up to n_units), so that a CTA finds its list with one load. One CTA.
__global__ void __launch_bounds__(1024) moba_scan_kernel(const uint32_t* __restrict__ cnt, int64_t n_lists,
                                                         uint32_t* __restrict__ off, uint32_t* __restrict__ tile_off,
                                                         uint32_t* __restrict__ totals, uint32_t unit_rows,
                                                         uint32_t* __restrict__ unit_list, int64_t n_units) {
  using Scan = cub::BlockScan<uint32_t, 1024>;
  __shared__ typename Scan::TempStorage t1, t2;
  __shared__ uint32_t carry_e, carry_t;
  if (threadIdx.x == 0) { carry_e = 0; carry_t = 0; }
  __syncthreads();
  for (int64_t base = 0; base < n_lists; base += 1024) {
    const int64_t i = base + threadIdx.x;
    const uint32_t c = i < n_lists ? cnt[i] : 0u;
    const uint32_t t = (c + unit_rows - 1) / unit_rows;
    uint32_t ec, tc, es, ts;
    Scan(t1).ExclusiveSum(c, ec, es);
    Scan(t2).ExclusiveSum(t, tc, ts);
    if (i < n_lists) {
      off[i] = carry_e + ec;
      tile_off[i] = carry_t + tc;
    }
    __syncthreads();
    if (threadIdx.x == 0) { carry_e += es; carry_t += ts; }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    tile_off[n_lists] = carry_t;
    totals[0] = carry_e;
    totals[1] = carry_t;
  }
  __syncthreads();                                   // tile_off complete (this CTA wrote it)
  for (int64_t i = threadIdx.x; i < n_lists; i += 1024)
    for (uint32_t u = tile_off[i]; u < tile_off[i + 1] && u < n_units; ++u) unit_list[u] = (uint32_t)i;
  for (int64_t u = (int64_t)carry_t + threadIdx.x; u < n_units; u += 1024) unit_list[u] = (uint32_t)n_lists;
}

// ------------------------------------------------------------------ TC problems --
// Past partials: part_o [B, seq, H, topk, D] bf16 (normalised), part_lse [B, seq, H,
// topk] fp32, base 2; slot s of (b, p, h) is the s-th kept past block of that query.
struct MobaPastProblem {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  __nv_bfloat16* part_o;
  float* part_lse;
  const uint32_t* tile_off;   // [n_lists + 1], in pairs of 128-row tiles
  const uint32_t* unit_list;  // [grid]: list of each pair (n_lists past the last)
  const uint32_t* off;        // [n_lists]
  const uint32_t* cnt;        // [n_lists]
  const uint32_t* list;       // packed (p << 4 | slot)
  int64_t seq;
  int heads, n_blocks, block, topk;
  int64_t n_lists;
  float sl2;
  // per CTA
  int b, h, blk;
  uint32_t e0, n_rows;

  // tile = 2 pair + t: half t of the pair-th 256-row unit (units numbered over the lists)
  __device__ bool setup_at(int tile) {
    const uint32_t pair = (uint32_t)tile >> 1, t = (uint32_t)tile & 1u;
    const int64_t li = unit_list[pair];
    if (li >= n_lists) return false;
    const uint32_t start = (pair - tile_off[li]) * 2 * kTcRows + t * kTcRows;
    if (start >= cnt[li]) return false;
    blk = (int)(li % n_blocks);
    h = (int)((li / n_blocks) % heads);
    b = (int)(li / ((int64_t)n_blocks * heads));
    e0 = off[li] + start;
    n_rows = min((uint32_t)kTcRows, cnt[li] - start);
    return true;
  }
  __device__ int32_t q_row(int r) const {
    if ((uint32_t)r >= n_rows) return -1;
    const int64_t p = list[e0 + r] >> 4;
    return (int32_t)(((int64_t)b * seq + p) * heads + h);
  }
  __device__ int64_t n_keys() const { return min((int64_t)block, seq - (int64_t)blk * block); }
  __device__ int32_t kv_row(int64_t t) const {
    return (int32_t)(((int64_t)b * seq + (int64_t)blk * block + t) * heads + h);
  }
  __device__ bool q_box(int*, int*) const { return false; }        // listed queries: gathered
  __device__ int kv_box(int j, int* y, int* z) const {              // a block is consecutive tokens
    *y = h;
    *z = (int)((int64_t)b * seq + (int64_t)blk * block + (int64_t)j * kTcKeys);
    return 1;
  }
  __device__ int64_t limit(int) const { return n_keys() - 1; }
  __device__ float scale_log2() const { return sl2; }
  __device__ void store(int r, int col0, const float* acc, float m2, float l) {
    if ((uint32_t)r >= n_rows) return;
    const uint32_t e = list[e0 + r];
    const int64_t p = e >> 4;
    const int slot = e & 15;
    const int64_t row = (((int64_t)b * seq + p) * heads + h) * topk + slot;
    const float inv = 1.f / l;
    uint4* dst = reinterpret_cast<uint4*>(part_o + row * kTcD + col0);
#pragma unroll
    for (int c = 0; c < kTcD / kTcSplit / 8; ++c) {
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

// Current block: grid (pairs_per_block * n_blocks, H, B), a pair = two consecutive
// 128-row tiles of one block; rows = 128 consecutive queries of one head inside one
// block; keys = the block up to each query (causal).
struct MobaCurrentProblem {
  const __nv_bfloat16* q;
  const __nv_bfloat16* k;
  const __nv_bfloat16* v;
  const __nv_bfloat16* part_o;   // the past partials (MobaPastProblem), complete before this kernel
  const float* part_lse;
  __nv_bfloat16* o;              // [B, seq, H, D]
  float* lse;                    // [B, seq, H] or null
  int64_t seq;
  int heads, n_blocks, block, topk, tiles_per_block;
  float sl2;
  int b, h, blk;
  int64_t p0, kb0, nrows;

  // tile = 2 pair + t: tile 2 (pair % pairs_per_block) + t of block pair / pairs_per_block
  __device__ bool setup_at(int tile) {
    const int ppb = (tiles_per_block + 1) / 2;
    const int pair = tile >> 1;
    blk = pair / ppb;
    const int t = (pair % ppb) * 2 + (tile & 1);
    if (t >= tiles_per_block) return false;
    h = blockIdx.y;
    b = blockIdx.z;
    kb0 = (int64_t)blk * block;
    p0 = kb0 + (int64_t)t * kTcRows;
    const int64_t bend = min(seq, kb0 + block);
    if (p0 >= bend) return false;
    nrows = min((int64_t)kTcRows, bend - p0);
    return true;
  }
  __device__ int32_t q_row(int r) const {
    if (r >= nrows) return -1;
    return (int32_t)(((int64_t)b * seq + p0 + r) * heads + h);
  }
  __device__ int64_t n_keys() const { return p0 + nrows - kb0; }
  __device__ int32_t kv_row(int64_t t) const { return (int32_t)(((int64_t)b * seq + kb0 + t) * heads + h); }
  __device__ bool q_box(int* y, int* z) const {                     // 128 consecutive queries of head h
    *y = h;
    *z = (int)((int64_t)b * seq + p0);
    return true;
  }
  __device__ int kv_box(int j, int* y, int* z) const {
    *y = h;
    *z = (int)((int64_t)b * seq + kb0 + (int64_t)j * kTcKeys);
    return 1;
  }
  __device__ int64_t limit(int r) const { return p0 + min((int64_t)r, nrows - 1) - kb0; }
  __device__ float scale_log2() const { return sl2; }
  // The epilogue reads the query's past partials (a scattered 64-byte piece of each
  // partial row per thread, and its LSE): prefetched into L2 when the CTA starts, so
  // the loads in store() do not wait on DRAM after the last tile.
  __device__ void prefetch(int r, int col0) const {
    if (r >= nrows) return;
    const int64_t row = ((int64_t)b * seq + p0 + r) * heads + h;
    const int ns = min(topk, blk);
    for (int s = 0; s < ns; ++s) prefetch_l2(part_o + (row * topk + s) * kTcD + col0);
    if (col0 == 0 && ns > 0) prefetch_l2(part_lse + row * topk);
  }
  // this part of the row merged with the query's min(topk, blk) past partials by
  // log-sum-exp (base 2), then written as the output
  __device__ void store(int r, int col0, const float* acc, float m2, float l) {
    constexpr int HC = kTcD / kTcSplit;
    if (r >= nrows) return;
    const int64_t row = ((int64_t)b * seq + p0 + r) * heads + h;
    const int ns = min(topk, blk);
    const float* pl = part_lse + row * topk;
    const float lc = m2 + __log2f(l);
    float M = lc;
    for (int s = 0; s < ns; ++s) M = fmaxf(M, __ldg(pl + s));
    const float wc = exp2f(lc - M);
    float L = wc;
    float out[HC];
    const float cw = wc / l;
#pragma unroll
    for (int c = 0; c < HC; ++c) out[c] = acc[c] * cw;
    for (int s = 0; s < ns; ++s) {
      const float w = exp2f(__ldg(pl + s) - M);
      L += w;
      const uint4* src = reinterpret_cast<const uint4*>(part_o + (row * topk + s) * kTcD + col0);
#pragma unroll
      for (int c = 0; c < HC / 8; ++c) {
        const uint4 u = __ldg(src + c);
        const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = bf16x2_to_float2(wd[e]);
          out[8 * c + 2 * e] = fmaf(w, f.x, out[8 * c + 2 * e]);
          out[8 * c + 2 * e + 1] = fmaf(w, f.y, out[8 * c + 2 * e + 1]);
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

// ------------------------------------------------------------------ decode gate --
// One query per (sequence, head) at position pos (decode; MoBA article, section 2: the
// gate of one query over the means of the past blocks). One warp per (sequence, head):
// the query row is spread over the lanes (D / 32 values each), every past block's mean
// is one warp dot product, and the kept list is the prefill gate's (ties to the lower
// block). The kept blocks, ascending, are expanded into positions: idx[list, j * block
// + t] = blk_j * block + t, count[list] = kept * block, so that the attention can take
// them as a per-head list of selected middle positions (the current block is the local
// part [cur * block, pos]). blocks_out (optional): kept blocks then the current block.
template <typename T, int D>
__global__ void __launch_bounds__(128) moba_decode_gate_kernel(const T* __restrict__ q, const float* __restrict__ kbar,
                                                               int batch, int heads, int nb, int block, int64_t pos,
                                                               int topk, int32_t* __restrict__ idx,
                                                               int32_t* __restrict__ count,
                                                               int16_t* __restrict__ blocks_out) {
  constexpr int VPL = D / 32;
  const int list = blockIdx.x * 4 + (threadIdx.x >> 5);     // sequence * heads + head
  const int lane = threadIdx.x & 31;
  if (list >= batch * heads) return;
  const int cur = (int)(pos / block);
  float qv[VPL];
  load_vec(q + (int64_t)list * D + lane * VPL, qv);
  if (VPL == 8) load_vec(q + (int64_t)list * D + lane * VPL + 4, qv + 4);
  float vals[kMobaMaxTopk];
  int ids[kMobaMaxTopk];
#pragma unroll
  for (int i = 0; i < kMobaMaxTopk; ++i) { vals[i] = -INFINITY; ids[i] = -1; }
  const float* kb = kbar + (int64_t)list * nb * D;
  constexpr int UNR = 8;                   // block means in flight per round
  for (int blk0 = 0; blk0 < cur; blk0 += UNR) {
    float kv[UNR][VPL];
#pragma unroll
    for (int u = 0; u < UNR; ++u)
#pragma unroll
      for (int e = 0; e < VPL; ++e)
        kv[u][e] = blk0 + u < cur ? __ldg(kb + (int64_t)(blk0 + u) * D + lane * VPL + e) : 0.f;
#pragma unroll
    for (int u = 0; u < UNR; ++u) {
      if (blk0 + u >= cur) break;
      float acc = 0.f;
#pragma unroll
      for (int e = 0; e < VPL; ++e) acc = fmaf(qv[e], kv[u][e], acc);
      acc = warp_sum(acc);
      // insert (acc, blk) into the descending list; equal values stay ahead (lower block)
      float v = acc;
      int id = blk0 + u;
#pragma unroll
      for (int i = 0; i < kMobaMaxTopk; ++i) {
        if (i < topk && v > vals[i]) {
          const float tv = vals[i];
          const int ti = ids[i];
          vals[i] = v; ids[i] = id;
          v = tv; id = ti;
        }
      }
    }
  }
  // kept blocks in ascending order (selection sort over at most kMobaMaxTopk entries)
  const int kept = min(topk, cur);
  int asc[kMobaMaxTopk];
#pragma unroll
  for (int i = 0; i < kMobaMaxTopk; ++i) asc[i] = i < kept ? ids[i] : 0x7fffffff;
#pragma unroll
  for (int i = 0; i < kMobaMaxTopk; ++i)
#pragma unroll
    for (int j = i + 1; j < kMobaMaxTopk; ++j)
      if (asc[j] < asc[i]) { const int t = asc[i]; asc[i] = asc[j]; asc[j] = t; }
  const int64_t stride = (int64_t)topk * block;
  int32_t* out = idx + (int64_t)list * stride;
  for (int i = 0; i < kept; ++i)
    for (int t = lane; t < block; t += 32) out[(int64_t)i * block + t] = asc[i] * block + t;
  for (int64_t t = (int64_t)kept * block + lane; t < stride; t += 32) out[t] = -1;
  if (lane == 0) {
    count[list] = kept * block;
    if (blocks_out) {
      int16_t* bo = blocks_out + (int64_t)list * (topk + 1);
      for (int i = 0; i <= topk; ++i) bo[i] = (int16_t)(i < kept ? asc[i] : (i == kept ? cur : -1));
    }
  }
}

}  // namespace esa
