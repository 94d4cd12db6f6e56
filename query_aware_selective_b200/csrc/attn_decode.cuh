// attn_decode.cuh - exact attention of one query per sequence (decode) over the
// initial + selected + local tokens, bf16 K/V with head_dim 128 (ESA write-up:
// implementation and final-attention paragraphs - global part = initial + selected
// tokens, window part = local tokens, fused into one output by one softmax).
//
// HBM-bound: every attended key row is read once. In the [B, n_cap, Hkv, 128] cache
// one token's rows for all KV heads are Hkv * 256 contiguous bytes, so a CTA takes a
// slice of one sequence's key list for ALL KV heads and moves each token with one bulk
// copy (cp.async.bulk, completion on an mbarrier) per operand, through a ring of
// kDecStages stages. In shared memory a token's row is padded by 16 bytes, so that the
// eight rows an ldmatrix phase reads start in eight different bank groups. There is no
// loader warp: the last of the eight warps to finish a stage (a shared-memory counter)
// issues its refill, which keeps the CTA at two warps per SM sub-partition.
//
// Warp w serves KV head w % Hkv and 16 keys of every stage. Its two contractions run on
// the tensor cores as m16n8k16 bf16 MMAs with fp32 accumulation, rows = the G query
// heads of the KV head (zero-padded to 16; only one query exists per sequence):
//   S [16 x 16 keys]  = Q [16 x 128] . K^T      (B fragments: ldmatrix of K rows)
//   O [16 x 128]     += P [16 x 16 keys] . V    (B fragments: ldmatrix.trans of V rows)
// P is rounded to bf16 for the second product and the row sums add the rounded values.
// The online softmax runs in base 2 on the S fragments (4 lanes per row); O is rescaled
// only when a row maximum moves. Warps are merged by log-sum-exp at the end; with
// several CTAs per sequence (key splits) each CTA writes its partial (o, m, l) rows to a
// workspace and counts itself in, and the last CTA of the sequence merges the splits.
#pragma once
#include "common.cuh"
#include "keylist.cuh"

namespace esa {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecD = 128;
constexpr int kDecKeysPerWarp = 16;                   // keys of a stage each warp takes
constexpr int kDecStageRowsBytes = 32768;             // unpadded K (or V) bytes per stage
constexpr int kDecStages = 3;
constexpr int kDecMaxSplitKeys = 4096;                // key positions staged in shared memory
// padded operand area: ks rows of (row_bytes + 16); ks * row_bytes == 32768 for every Hkv
__host__ __device__ constexpr int dec_operand_bytes(int hkv) {
  return (kDecStageRowsBytes / (hkv * kDecD * 2)) * (hkv * kDecD * 2 + 16);
}
constexpr int kDecOperandMax = dec_operand_bytes(1);  // 128 rows of 272 bytes = 34816
constexpr int kDecPartStride = kDecD + 4;             // partial row: o, m, l, 2 pad (16-byte rows)
constexpr int kDecSmemBytes = 2 * kDecStages * kDecOperandMax + kDecMaxSplitKeys * 4 + 256;

struct DecodeAttnArgs {
  const __nv_bfloat16* q;   // [B, 1, Hq, 128]
  const __nv_bfloat16* k;   // [B, n_cap, Hkv, 128]
  const __nv_bfloat16* v;
  __nv_bfloat16* o;         // [B, 1, Hq, 128]
  float* lse;               // [B, 1, Hq] or null
  float* part;              // [B, Hq, nsplit, kDecPartStride] when nsplit > 1: o[128], m, l
  int* arrive;              // [B] zeroed split counters when nsplit > 1
  KeyList keys;
  int64_t n_cap, c0;
  int hq, hkv, nsplit;       // per (virtual) sequence
  int keys_per_split;       // a multiple of the keys per stage, <= kDecMaxSplitKeys
  float scale_log2;         // softmax scale * log2(e)
  // Sequence b of the grid is cache sequence b / vheads, KV heads from (b % vheads) * hkv:
  // 1 normally; with per-head key lists every (sequence, KV head) is a sequence of its
  // own with hkv = 1. tok_stride: elements from one token's K row to the next (Hkv * 128
  // of the cache).
  int vheads;
  int64_t tok_stride;
};

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
// D = A . B + D, m16n8k16, bf16 in, fp32 accumulate. Rows 8-15 of A are zero here, so
// the a1/a3 registers are passed as zero.
__device__ __forceinline__ void mma_bf16_rows8(float* d, uint32_t a0, uint32_t a2, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1));
}

struct DecSmem {
  uint64_t full[kDecStages];
  int done[kDecStages];   // warps finished with the stage's current fill
  int abort_flag;
  int issued;             // stages issued so far
};

// Issue stage j (keys [t_begin + j ks, ...)) into ring slot j % kDecStages: one bulk
// copy per token and operand, spread over the warp's lanes. Called by one whole warp.
__device__ __forceinline__ void dec_issue(const DecodeAttnArgs& a, DecSmem& sm, const int32_t* pos, uint32_t stage0,
                                          int b, int64_t t_begin, int64_t t_end, int ks, int row_bytes, int op_bytes,
                                          int j, int lane) {
  const int s = j % kDecStages;
  const int64_t t0 = t_begin + (int64_t)j * ks;
  const int n_in = (int)(t_end - t0 < ks ? t_end - t0 : ks);
  if (lane == 0) mbar_arrive_expect_tx(&sm.full[s], (uint32_t)(2 * n_in * row_bytes));
  __syncwarp();
  const int64_t seq = (int64_t)(b / a.vheads) * a.n_cap * a.tok_stride + (int64_t)(b % a.vheads) * a.hkv * kDecD;
  const uint32_t kdst = stage0 + s * 2 * op_bytes;
  const int rs = row_bytes + 16;
  for (int c = lane; c < 2 * n_in; c += 32) {
    const int kk = c >> 1;
    const int64_t p = pos[j * ks + kk];
    const __nv_bfloat16* src = ((c & 1) ? a.v : a.k) + seq + p * a.tok_stride;
    bulk_g2s(kdst + (c & 1) * op_bytes + kk * rs, src, row_bytes, &sm.full[s]);
  }
  if (lane == 0) atomicMax(&sm.issued, j + 1);
}

// After the key loop: merge the warps' states of each query head and write the output
// (one split) or the split's partial rows; with several splits the last CTA of the
// sequence to finish merges them. red: at least 64 KB of free shared memory; last: a
// shared int. acc/m/l: the lane's O fragments, row max (base 2) and row sum.
template <int G>
__device__ __forceinline__ void dec_finish(const DecodeAttnArgs& a, const float (&acc)[16][4], float m, float l,
                                           uint8_t* red_area, int* last, int b, int split, int g) {
  const int hkv = a.hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gid = lane >> 2, tig = lane & 3;
  float* red0 = reinterpret_cast<float*>(red_area);
  float* red = red0;
  if (hkv == kDecWarps && a.nsplit > 1) {
    // one warp per KV head: its rows are this CTA's partial rows as they stand
    if (gid < G) {
      float* pp = a.part + (((int64_t)b * a.hq + g * G + gid) * a.nsplit + split) * kDecPartStride;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt)
        *reinterpret_cast<float2*>(pp + nt * 8 + 2 * tig) = make_float2(acc[nt][0], acc[nt][1]);
      if (tig == 0) *reinterpret_cast<float2*>(pp + kDecD) = make_float2(m, l);
    }
  } else {
  // per-warp state to shared memory: red[warp][row][0..127 o, 128 m, 129 l]
  if (gid < G) {
    float* r = red + (warp * G + gid) * (kDecD + 2);
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      r[nt * 8 + 2 * tig] = acc[nt][0];
      r[nt * 8 + 2 * tig + 1] = acc[nt][1];
    }
    if (tig == 0) { r[kDecD] = m; r[kDecD + 1] = l; }
  }
  __syncthreads();
  // merge the warps of each KV head and write (o, lse) or the split's partial row
  const int nph = kDecWarps / hkv;
  for (int t = threadIdx.x; t < a.hq * kDecD; t += kDecThreads) {
    const int head = t / kDecD, e = t % kDecD;
    const int gg = head / G, h = head % G;
    float M = -INFINITY;
    for (int ph = 0; ph < nph; ++ph) M = fmaxf(M, red[((ph * hkv + gg) * G + h) * (kDecD + 2) + kDecD]);
    const float Mr = M == -INFINITY ? 0.f : M;
    float L = 0.f, O = 0.f;
    for (int ph = 0; ph < nph; ++ph) {
      const float* r = red + ((ph * hkv + gg) * G + h) * (kDecD + 2);
      const float w = fast_exp2(r[kDecD] - Mr);
      L += r[kDecD + 1] * w;
      O += r[e] * w;
    }
    const int64_t row = (int64_t)b * a.hq + head;
    if (a.nsplit == 1) {
      a.o[row * kDecD + e] = __float2bfloat16_rn(O / L);
      if (e == 0 && a.lse) a.lse[row] = (M + __log2f(L)) * 0.69314718055994531f;
    } else {
      float* pp = a.part + (row * a.nsplit + split) * kDecPartStride;
      pp[e] = O;
      if (e == 0) { pp[kDecD] = M; pp[kDecD + 1] = L; }
    }
  }
  }
  if (a.nsplit == 1) return;

  // ---- the last CTA of the sequence to finish merges the splits by log-sum-exp
  __threadfence();                 // this CTA's partial rows are visible before it counts itself in
  __syncthreads();
  if (threadIdx.x == 0) *last = atomicAdd(&a.arrive[b], 1) == a.nsplit - 1;
  __syncthreads();
  if (!*last) return;
  __threadfence();
  const int ns = a.nsplit;
  float* coef = red;               // [Hq][nsplit] merge weights 2^(m - M) / L
  float* lse2 = red + a.hq * ns;   // [Hq] log-sum-exp, base 2
  float* ml = lse2 + a.hq;         // [Hq][nsplit] (m, l) pairs
  const float* pb = a.part + (int64_t)b * a.hq * ns * kDecPartStride;
  for (int i = threadIdx.x; i < a.hq * ns; i += kDecThreads) {
    const float2 x = __ldcg(reinterpret_cast<const float2*>(pb + (int64_t)i * kDecPartStride + kDecD));
    ml[2 * i] = x.x;
    ml[2 * i + 1] = x.y;
  }
  __syncthreads();
  for (int head = threadIdx.x; head < a.hq; head += kDecThreads) {
    float M = -INFINITY;
    for (int sp = 0; sp < ns; ++sp) M = fmaxf(M, ml[2 * (head * ns + sp)]);
    const float Mr = M == -INFINITY ? 0.f : M;
    float L = 0.f;
    for (int sp = 0; sp < ns; ++sp) {
      const float w = fast_exp2(ml[2 * (head * ns + sp)] - Mr);
      coef[head * ns + sp] = w;
      L += ml[2 * (head * ns + sp) + 1] * w;
    }
    const float inv = 1.f / L;
    for (int sp = 0; sp < ns; ++sp) coef[head * ns + sp] *= inv;
    lse2[head] = M + __log2f(L);
  }
  __syncthreads();
  // thread t takes the (head, 4 dims) items t, t + 256, ...: with Hq <= 32 at most four,
  // whose loads for eight splits are all in flight in each round
  constexpr int kItems = 32 * (kDecD / 4) / kDecThreads;   // 4
  const int n_items = a.hq * (kDecD / 4);
  float4 res[kItems];
#pragma unroll
  for (int u = 0; u < kItems; ++u) res[u] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int sp0 = 0; sp0 < ns; sp0 += 8) {
    float4 x[kItems][8];
#pragma unroll
    for (int u = 0; u < kItems; ++u) {
      const int it = threadIdx.x + u * kDecThreads;
      const int head = it / (kDecD / 4), d4 = (it % (kDecD / 4)) * 4;
      const float* base = pb + (int64_t)head * ns * kDecPartStride + d4;
#pragma unroll
      for (int w = 0; w < 8; ++w)
        x[u][w] = (it < n_items && sp0 + w < ns)
                      ? __ldcg(reinterpret_cast<const float4*>(base + (int64_t)(sp0 + w) * kDecPartStride))
                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kItems; ++u) {
      const int it = threadIdx.x + u * kDecThreads;
      const int head = it < n_items ? it / (kDecD / 4) : 0;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const float c = (it < n_items && sp0 + w < ns) ? coef[head * ns + sp0 + w] : 0.f;
        res[u].x = fmaf(c, x[u][w].x, res[u].x);
        res[u].y = fmaf(c, x[u][w].y, res[u].y);
        res[u].z = fmaf(c, x[u][w].z, res[u].z);
        res[u].w = fmaf(c, x[u][w].w, res[u].w);
      }
    }
  }
#pragma unroll
  for (int u = 0; u < kItems; ++u) {
    const int it = threadIdx.x + u * kDecThreads;
    if (it >= n_items) break;
    const int head = it / (kDecD / 4), d4 = (it % (kDecD / 4)) * 4;
    const int64_t row = (int64_t)b * a.hq + head;
    __nv_bfloat162 lo2 = __floats2bfloat162_rn(res[u].x, res[u].y), hi2 = __floats2bfloat162_rn(res[u].z, res[u].w);
    uint2 packed;
    packed.x = *reinterpret_cast<uint32_t*>(&lo2);
    packed.y = *reinterpret_cast<uint32_t*>(&hi2);
    *reinterpret_cast<uint2*>(a.o + row * kDecD + d4) = packed;
    if (d4 == 0 && a.lse) a.lse[row] = lse2[head] * 0.69314718055994531f;
  }
  if (threadIdx.x == 0) a.arrive[b] = 0;

}

// grid (nsplit, B); kDecThreads threads; kDecSmemBytes dynamic shared memory.
template <int G>
__global__ void __launch_bounds__(kDecThreads, 1) attn_decode_kernel(const DecodeAttnArgs a) {
  extern __shared__ __align__(128) uint8_t dsm[];
  const uint32_t stage0 = (smem_u32(dsm) + 127u) & ~127u;     // bulk copies need 16 bytes
  uint8_t* const stage0_ptr = dsm + (stage0 - smem_u32(dsm));

  const int split = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hkv = a.hkv;
  const int row_bytes = hkv * kDecD * 2;
  const int rs = row_bytes + 16;                         // padded row stride in shared memory
  const int ks = kDecStageRowsBytes / row_bytes;         // keys per stage: 16 (Hkv 8) .. 128 (Hkv 1)
  const int op_bytes = ks * rs;
  int32_t* pos = reinterpret_cast<int32_t*>(stage0_ptr + 2 * kDecStages * op_bytes);   // this split's keys
  DecSmem& sm = *reinterpret_cast<DecSmem*>(pos + kDecMaxSplitKeys);

  KeyList kl = a.keys;
  const int64_t c0 = kl.vl.len ? kl.resolve(b, 701) : a.c0;
  const int cnt = min(max(kl.count[b], 0), (int)kl.idx_stride);
  const int64_t n_keys = kl.ni + cnt + (c0 - kl.lo) + 1;
  const int64_t t_begin = (int64_t)split * a.keys_per_split;
  const int64_t t_end = min(n_keys, t_begin + a.keys_per_split);
  const int nst = t_end > t_begin ? (int)((t_end - t_begin + ks - 1) / ks) : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kDecStages; ++s) {
      mbar_init(&sm.full[s], 1);
      sm.done[s] = 0;
    }
    sm.abort_flag = 0;
    sm.issued = 0;
    fence_barrier_init();
  }
  for (int64_t t = t_begin + threadIdx.x; t < t_end; t += kDecThreads) pos[t - t_begin] = (int32_t)kl.pos(b, cnt, t);
  if (nst > 0) {
    // V rows past the end of the last stage are multiplied by P = 0: make sure they hold
    // finite values (zeros) if that ring slot is never filled by an earlier stage
    const int n_last = (int)(t_end - t_begin - (int64_t)(nst - 1) * ks);
    uint8_t* vlast = stage0_ptr + ((nst - 1) % kDecStages) * 2 * op_bytes + op_bytes;
    for (int i = n_last * rs / 16 + threadIdx.x; i < op_bytes / 16; i += kDecThreads)
      reinterpret_cast<uint4*>(vlast)[i] = make_uint4(0u, 0u, 0u, 0u);
    fence_proxy_async();
  }
  __syncthreads();
  volatile int* abort_flag = &sm.abort_flag;

  if (warp == 0)
    for (int j = 0; j < min(nst, kDecStages); ++j)
      dec_issue(a, sm, pos, stage0, b, t_begin, t_end, ks, row_bytes, op_bytes, j, lane);

  const int g = warp % hkv;                        // KV head
  const int kw0 = (warp / hkv) * kDecKeysPerWarp;  // this warp's first key slot in a stage
  const int gid = lane >> 2, tig = lane & 3;       // fragment row (query head) and column pair

  // Q as the A operand: row gid = query head g * G + gid (rows >= G are zero)
  uint32_t qa[8][2];
  {
    const __nv_bfloat16* qp = a.q + ((int64_t)b * a.hq + g * G + (gid < G ? gid : 0)) * kDecD;
#pragma unroll
    for (int kt = 0; kt < 8; ++kt) {
      qa[kt][0] = gid < G ? __ldg(reinterpret_cast<const uint32_t*>(qp + kt * 16 + 2 * tig)) : 0u;
      qa[kt][1] = gid < G ? __ldg(reinterpret_cast<const uint32_t*>(qp + kt * 16 + 8 + 2 * tig)) : 0u;
    }
  }
  float acc[16][4];   // O fragments: dims nt * 8 + 2 tig (+1) of row gid; [2], [3] are padding rows
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  float m = -INFINITY, l = 0.f;                    // row gid, base 2, scaled logits

  // per-lane ldmatrix row addresses (relative to a stage's K or V area)
  //   K (non-trans): lanes 8i..8i+7 -> key kw0 + nt * 8 + (lane & 7), 16-byte chunk 4c + i
  //   V (trans):     matrix i = lane >> 3 -> key kw0 + (i & 1) * 8 + (lane & 7), chunk 2c + (i >> 1)
  const uint32_t k_lane = (uint32_t)((kw0 + (lane & 7)) * rs + g * kDecD * 2 + (lane >> 3) * 16);
  const uint32_t v_lane =
      (uint32_t)((kw0 + ((lane >> 3) & 1) * 8 + (lane & 7)) * rs + g * kDecD * 2 + (lane >> 4) * 16);
  const float sl2 = a.scale_log2;

  for (int j = 0; j < nst; ++j) {
    const int s = j % kDecStages;
    if (!mbar_wait_warp(&sm.full[s], (j / kDecStages) & 1, abort_flag, 302)) break;
    const uint32_t kst = stage0 + s * 2 * op_bytes;
    const uint32_t vst = kst + op_bytes;
    const int64_t t0 = t_begin + (int64_t)j * ks + kw0;   // this warp's first key

    // S = Q K^T for the warp's 16 keys (two n-tiles of 8)
    float sc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kst + k_lane + nt * 8 * rs + c * 64, b0, b1, b2, b3);
        mma_bf16_rows8(sc[nt], qa[2 * c][0], qa[2 * c][1], b0, b1);
        mma_bf16_rows8(sc[nt], qa[2 * c + 1][0], qa[2 * c + 1][1], b2, b3);
      }
    }
    // online softmax on row gid: keys nt * 8 + 2 tig + {0, 1}
    float x[4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool ok = t0 + nt * 8 + 2 * tig + e < t_end;
        x[nt * 2 + e] = ok ? sc[nt][e] * sl2 : -INFINITY;
      }
    float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m, mx);
    const float mref = m_new == -INFINITY ? 0.f : m_new;   // no key yet: keep everything at zero
    if (!__all_sync(0xffffffffu, m_new == m)) {
      const float alpha = fast_exp2(m - mref);
      l *= alpha;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        acc[nt][0] *= alpha;
        acc[nt][1] *= alpha;
      }
    }
    m = m_new;
    uint32_t pa[2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      pa[nt] = bf16x2_rn(fast_exp2(x[nt * 2] - mref), fast_exp2(x[nt * 2 + 1] - mref));
      const float2 pr = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pa[nt]));
      l += pr.x + pr.y;
    }
    if (gid >= G) pa[0] = pa[1] = 0u;
    // O += P V over the 16 keys: 16 n-tiles of 8 dims, two per ldmatrix.x4.trans
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(vst + v_lane + c * 32, b0, b1, b2, b3);
      mma_bf16_rows8(acc[2 * c], pa[0], pa[1], b0, b1);
      mma_bf16_rows8(acc[2 * c + 1], pa[0], pa[1], b2, b3);
    }

    // release the stage; the last warp out refills it with stage j + kDecStages
    __syncwarp();
    int prev = 0;
    if (lane == 0) {
      __threadfence_block();
      prev = atomicAdd(&sm.done[s], 1);
      if (prev == kDecWarps - 1) sm.done[s] = 0;
      __threadfence_block();
    }
    prev = __shfl_sync(0xffffffffu, prev, 0);
    if (prev == kDecWarps - 1 && j + kDecStages < nst) {
      fence_proxy_async();
      dec_issue(a, sm, pos, stage0, b, t_begin, t_end, ks, row_bytes, op_bytes, j + kDecStages, lane);
    }
  }
  // row sum over the 4 lanes of the row
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);

  __syncthreads();   // every stage consumed (or the CTA aborted): the stage area is free
  if (*abort_flag) {
    // drain the copies that may still be in flight before the CTA's shared memory goes away
    if (threadIdx.x == 0) {
      const int issued = sm.issued;
      for (int j = max(0, issued - kDecStages); j < issued; ++j)
        mbar_wait(&sm.full[j % kDecStages], (j / kDecStages) & 1, abort_flag, 303, /*respect_abort=*/false);
    }
    return;
  }
  dec_finish<G>(a, acc, m, l, stage0_ptr, &sm.done[0], b, split, g);
}

// ------------------------------------------------------------------ one KV head --
// The same attention when a sequence has one KV head (hkv == 1: the per-head key
// lists, every (sequence, KV head) its own sequence). A token's row is then 256 bytes,
// and every row of a selection may be somewhere else, so bulk copies would be one small
// TMA operation per row. Instead each warp owns 16 key slots of every 128-key stage and
// streams its own rows with 16-byte cp.async copies into a private ring of
// kRowStages slots (rows padded to 272 bytes, as above), refilling a slot as soon as it
// has used it: no cross-warp hand-off, no barriers in the key loop. Slots past the end
// of the list are zero-filled (no read). Contractions, softmax and epilogue as above.
constexpr int kRowStages = 3;
constexpr int kRowStride = kDecD * 2 + 16;                         // padded 256-byte row
constexpr int kRowWarpSlot = 2 * kDecKeysPerWarp * kRowStride;     // K then V rows of 16 keys
constexpr int kRowSmemBytes = kDecWarps * kRowStages * kRowWarpSlot + 256;

template <int G>
__global__ void __launch_bounds__(kDecThreads, 1) attn_decode_rows_kernel(const DecodeAttnArgs a) {
  extern __shared__ __align__(128) uint8_t rsm[];
  uint8_t* const ring = rsm + ((128u - (smem_u32(rsm) & 127u)) & 127u);
  int* last = reinterpret_cast<int*>(ring + kDecWarps * kRowStages * kRowWarpSlot);
  const int split = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr int ks = kDecWarps * kDecKeysPerWarp;                  // 128 keys per stage
  KeyList kl = a.keys;
  const int64_t c0 = kl.vl.len ? kl.resolve(b, 702) : a.c0;
  const int cnt = min(max(kl.count[b], 0), (int)kl.idx_stride);
  const int64_t n_keys = kl.ni + cnt + (c0 - kl.lo) + 1;
  const int64_t t_begin = (int64_t)split * a.keys_per_split;
  const int64_t t_end = min(n_keys, t_begin + a.keys_per_split);
  const int nst = t_end > t_begin ? (int)((t_end - t_begin + ks - 1) / ks) : 0;
  const int64_t seq = (int64_t)(b / a.vheads) * a.n_cap * a.tok_stride + (int64_t)(b % a.vheads) * kDecD;
  const uint32_t wring = smem_u32(ring) + warp * kRowStages * kRowWarpSlot;

  // copies of this warp's 16 rows of stage j into slot j % kRowStages: lane (op, piece)
  // moves 16-byte piece `piece` of operand op (K, V) of every one of the 16 rows
  auto issue = [&](int j) {
    if (j < nst) {
      const int64_t t0 = t_begin + (int64_t)j * ks + warp * kDecKeysPerWarp;
      const int my_pos = (lane < kDecKeysPerWarp && t0 + lane < t_end) ? (int)kl.pos(b, cnt, t0 + lane) : -1;
      const int op = lane >> 4, pc = lane & 15;
      const __nv_bfloat16* src = (op ? a.v : a.k) + seq + pc * 8;
      const uint32_t dst = wring + (j % kRowStages) * kRowWarpSlot + op * kDecKeysPerWarp * kRowStride + pc * 16;
#pragma unroll
      for (int kk = 0; kk < kDecKeysPerWarp; ++kk) {
        const int p = __shfl_sync(0xffffffffu, my_pos, kk);
        cp_async16(dst + kk * kRowStride, src + (int64_t)(p < 0 ? 0 : p) * a.tok_stride, p < 0 ? 0u : 16u);
      }
    }
    cp_async_commit();                    // one group per stage, empty past the end
  };
#pragma unroll
  for (int j = 0; j < kRowStages; ++j) issue(j);

  const int gid = lane >> 2, tig = lane & 3;
  uint32_t qa[8][2];
  {
    const __nv_bfloat16* qp = a.q + ((int64_t)b * a.hq + (gid < G ? gid : 0)) * kDecD;
#pragma unroll
    for (int kt = 0; kt < 8; ++kt) {
      qa[kt][0] = gid < G ? __ldg(reinterpret_cast<const uint32_t*>(qp + kt * 16 + 2 * tig)) : 0u;
      qa[kt][1] = gid < G ? __ldg(reinterpret_cast<const uint32_t*>(qp + kt * 16 + 8 + 2 * tig)) : 0u;
    }
  }
  float acc[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
  float m = -INFINITY, l = 0.f;
  const uint32_t k_lane = (uint32_t)((lane & 7) * kRowStride + (lane >> 3) * 16);
  const uint32_t v_lane = (uint32_t)((((lane >> 3) & 1) * 8 + (lane & 7)) * kRowStride + (lane >> 4) * 16);
  const float sl2 = a.scale_log2;

  for (int j = 0; j < nst; ++j) {
    cp_async_wait<kRowStages - 1>();      // this lane's pieces of stage j have landed
    __syncwarp();                         // ... and every other lane's
    const uint32_t kst = wring + (j % kRowStages) * kRowWarpSlot;
    const uint32_t vst = kst + kDecKeysPerWarp * kRowStride;
    const int64_t t0 = t_begin + (int64_t)j * ks + warp * kDecKeysPerWarp;
    float sc[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(kst + k_lane + nt * 8 * kRowStride + c * 64, b0, b1, b2, b3);
        mma_bf16_rows8(sc[nt], qa[2 * c][0], qa[2 * c][1], b0, b1);
        mma_bf16_rows8(sc[nt], qa[2 * c + 1][0], qa[2 * c + 1][1], b2, b3);
      }
    }
    float x[4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool ok = t0 + nt * 8 + 2 * tig + e < t_end;
        x[nt * 2 + e] = ok ? sc[nt][e] * sl2 : -INFINITY;
      }
    float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    const float m_new = fmaxf(m, mx);
    const float mref = m_new == -INFINITY ? 0.f : m_new;
    if (!__all_sync(0xffffffffu, m_new == m)) {
      const float alpha = fast_exp2(m - mref);
      l *= alpha;
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        acc[nt][0] *= alpha;
        acc[nt][1] *= alpha;
      }
    }
    m = m_new;
    uint32_t pa[2];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      pa[nt] = bf16x2_rn(fast_exp2(x[nt * 2] - mref), fast_exp2(x[nt * 2 + 1] - mref));
      const float2 pr = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pa[nt]));
      l += pr.x + pr.y;
    }
    if (gid >= G) pa[0] = pa[1] = 0u;
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(vst + v_lane + c * 32, b0, b1, b2, b3);
      mma_bf16_rows8(acc[2 * c], pa[0], pa[1], b0, b1);
      mma_bf16_rows8(acc[2 * c + 1], pa[0], pa[1], b2, b3);
    }
    __syncwarp();                         // every lane is done with the slot
    issue(j + kRowStages);
  }
  l += __shfl_xor_sync(0xffffffffu, l, 1);
  l += __shfl_xor_sync(0xffffffffu, l, 2);
  cp_async_wait_all();
  __syncthreads();                        // the rings are free: the epilogue reuses them
  dec_finish<G>(a, acc, m, l, ring, last, b, split, 0);
}

}  // namespace esa
