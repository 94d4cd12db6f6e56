// attn_decode.cuh - exact attention of one query per sequence (decode) over the
// initial + selected + local tokens, bf16 K/V with head_dim 128 (ESA write-up:
// implementation and final-attention paragraphs - global part = initial + selected
// tokens, window part = local tokens, fused into one output by one softmax).
//
// HBM-bound: every attended key row is read once. In the [B, n_cap, Hkv, 128] cache
// one token's rows for all KV heads are Hkv * 256 contiguous bytes, so a CTA takes a
// slice of one sequence's key list for ALL KV heads and moves each token with one bulk
// copy (cp.async.bulk, completion on an mbarrier) per operand, through a ring of
// kDecStages stages (K rows then V rows of kDecStageBytes each). There is no loader
// warp: the last of the eight warps to finish a stage (a shared-memory counter) issues
// its refill, so the CTA stays at two warps per SM sub-partition and every thread may
// hold up to 255 registers (a ninth warp would cap them at 168).
//
// Compute warp w serves KV head w % Hkv (and every (8 / Hkv)-th key slot of a stage).
// Its lanes form 4 groups of 8; a group holds one key at a time, each lane 16 of the
// 128 dims ([8 sub, 8 sub + 8) and [64 + 8 sub, 72 + 8 sub)), so a quarter-warp reads
// one 128-byte span of shared memory. All G query heads of the KV head reuse each
// loaded row. Dot products and the P.V update use packed fp32x2 FMAs. Every group keeps
// its own online softmax (base 2); groups, then warps, are merged by log-sum-exp at the
// end. With several CTAs per sequence (key splits) the partial (o, m, l) rows go to a
// workspace and attn_combine_kernel merges them.
#pragma once
#include "common.cuh"
#include "keylist.cuh"

namespace esa {

constexpr int kDecWarps = 8;
constexpr int kDecThreads = kDecWarps * 32;
constexpr int kDecStageBytes = 32768;                 // K (and again V) bytes per stage
constexpr int kDecStages = 3;
constexpr int kDecMaxSplitKeys = 4096;                // key positions staged in shared memory
constexpr int kDecSmemBytes = 2 * kDecStages * kDecStageBytes + kDecMaxSplitKeys * 4 + 256;
constexpr int kDecD = 128;

struct DecodeAttnArgs {
  const __nv_bfloat16* q;   // [B, 1, Hq, 128]
  const __nv_bfloat16* k;   // [B, n_cap, Hkv, 128]
  const __nv_bfloat16* v;
  __nv_bfloat16* o;         // [B, 1, Hq, 128]
  float* lse;               // [B, 1, Hq] or null
  float* part;              // [B, Hq, nsplit, 130] when nsplit > 1
  KeyList keys;
  int64_t n_cap, c0;
  int hq, hkv, nsplit;
  int keys_per_split;       // a multiple of the keys per stage, <= kDecMaxSplitKeys
  float scale_log2;         // softmax scale * log2(e)
};

__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
      "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
  return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  float2 d;
  asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
      "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
      "mul.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
      : "=f"(d.x), "=f"(d.y)
      : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
  return d;
}
// Two bf16 packed in a 32-bit word (element 0 in the low half) -> two fp32.
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
               "l"(src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
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
                                          int b, int64_t t_begin, int64_t t_end, int ks, int row_bytes, int j,
                                          int lane) {
  const int s = j % kDecStages;
  const int64_t t0 = t_begin + (int64_t)j * ks;
  const int n_in = (int)(t_end - t0 < ks ? t_end - t0 : ks);
  if (lane == 0) mbar_arrive_expect_tx(&sm.full[s], (uint32_t)(2 * n_in * row_bytes));
  __syncwarp();
  const int64_t seq = (int64_t)b * a.n_cap * a.hkv * kDecD;
  const uint32_t kdst = stage0 + s * 2 * kDecStageBytes;
  for (int c = lane; c < 2 * n_in; c += 32) {
    const int kk = c >> 1;
    const int64_t p = pos[j * ks + kk];
    const __nv_bfloat16* src = ((c & 1) ? a.v : a.k) + seq + p * a.hkv * kDecD;
    bulk_g2s(kdst + (c & 1) * kDecStageBytes + kk * row_bytes, src, row_bytes, &sm.full[s]);
  }
  if (lane == 0) atomicMax(&sm.issued, j + 1);
}

// grid (nsplit, B); kDecThreads threads; kDecSmemBytes dynamic shared memory.
template <int G>
__global__ void __launch_bounds__(kDecThreads, 1) attn_decode_kernel(const DecodeAttnArgs a) {
  extern __shared__ __align__(128) uint8_t dsm[];
  const uint32_t stage0 = (smem_u32(dsm) + 127u) & ~127u;     // bulk copies need 16 bytes
  uint8_t* const stage0_ptr = dsm + (stage0 - smem_u32(dsm));
  int32_t* pos = reinterpret_cast<int32_t*>(stage0_ptr + 2 * kDecStages * kDecStageBytes);   // this split's keys
  DecSmem& sm = *reinterpret_cast<DecSmem*>(pos + kDecMaxSplitKeys);

  const int split = blockIdx.x, b = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int hkv = a.hkv;
  const int row_bytes = hkv * kDecD * 2;
  const int ks = kDecStageBytes / row_bytes;            // keys per stage: 16 (Hkv 8) .. 128 (Hkv 1)
  const int cnt = min(max(a.keys.count[b], 0), (int)a.keys.idx_stride);
  const int64_t n_keys = a.keys.ni + cnt + (a.c0 - a.keys.lo) + 1;
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
  for (int64_t t = t_begin + threadIdx.x; t < t_end; t += kDecThreads) pos[t - t_begin] = (int32_t)a.keys.pos(b, cnt, t);
  __syncthreads();
  volatile int* abort_flag = &sm.abort_flag;

  // merged per-warp state, written after the loop (reuses stage 0's K area)
  float* red = reinterpret_cast<float*>(stage0_ptr);    // [kDecWarps][G][130]

  // per-lane softmax state of the compute warps: running max (base 2), sum, output
  float m[G], l[G];
  float2 o[G][8];
#pragma unroll
  for (int h = 0; h < G; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) o[h][e] = make_float2(0.f, 0.f);
  }

  if (warp == 0)
    for (int j = 0; j < min(nst, kDecStages); ++j)
      dec_issue(a, sm, pos, stage0, b, t_begin, t_end, ks, row_bytes, j, lane);
  {
    // ------------------------------------------------------------------ compute
    const int hh = warp % hkv;                 // KV head
    const int nph = kDecWarps / hkv;           // warps per KV head
    const int grp = lane >> 3, sub = lane & 7;
    const int slot = (warp / hkv) * 4 + grp;   // key slot within a stage
    const int slot_step = nph * 4;             // ks / slot_step == 4 keys per group and stage
    const uint32_t lane_off = hh * kDecD * 2 + sub * 16;

    float2 q[G][8];
    {
      const __nv_bfloat16* qp = a.q + ((int64_t)b * a.hq + hh * G) * kDecD;
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const uint4 x0 = __ldg(reinterpret_cast<const uint4*>(qp + h * kDecD + sub * 8));
        const uint4 x1 = __ldg(reinterpret_cast<const uint4*>(qp + h * kDecD + 64 + sub * 8));
        const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float2 f = bf16x2_to_f2(w[e]);
          q[h][e] = make_float2(f.x * a.scale_log2, f.y * a.scale_log2);
        }
      }
    }

    for (int j = 0; j < nst; ++j) {
      const int s = j % kDecStages;
      if (!mbar_wait_warp(&sm.full[s], (j / kDecStages) & 1, abort_flag, 302)) break;
      const int64_t t0 = t_begin + (int64_t)j * ks;
      const uint32_t kst = stage0 + s * 2 * kDecStageBytes + lane_off;
      const uint32_t vst = kst + kDecStageBytes;
      float x[4][G];
      bool valid[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int kk = slot + r * slot_step;
        valid[r] = t0 + kk < t_end;
        const uint4 k0 = lds128(kst + kk * row_bytes);
        const uint4 k1 = lds128(kst + kk * row_bytes + 128);
        const uint32_t w[8] = {k0.x, k0.y, k0.z, k0.w, k1.x, k1.y, k1.z, k1.w};
        float2 acc[G];
#pragma unroll
        for (int h = 0; h < G; ++h) acc[h] = make_float2(0.f, 0.f);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float2 kf = bf16x2_to_f2(w[e]);
#pragma unroll
          for (int h = 0; h < G; ++h) acc[h] = ffma2(q[h][e], kf, acc[h]);
        }
#pragma unroll
        for (int h = 0; h < G; ++h) x[r][h] = acc[h].x + acc[h].y;
      }
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int h = 0; h < G; ++h) {
          float v = x[r][h];
          v += __shfl_xor_sync(0xffffffffu, v, 1);
          v += __shfl_xor_sync(0xffffffffu, v, 2);
          v += __shfl_xor_sync(0xffffffffu, v, 4);
          x[r][h] = valid[r] ? v : -INFINITY;
        }
      float p[4][G];
#pragma unroll
      for (int h = 0; h < G; ++h) {
        float mx = m[h];
#pragma unroll
        for (int r = 0; r < 4; ++r) mx = fmaxf(mx, x[r][h]);
        const float mref = mx == -INFINITY ? 0.f : mx;   // no key yet: keep everything at zero
        const float alpha = fast_exp2(m[h] - mref);
        m[h] = mx;
        float ps = 0.f;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          p[r][h] = fast_exp2(x[r][h] - mref);
          ps += p[r][h];
        }
        l[h] = fmaf(l[h], alpha, ps);
        const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
        for (int e = 0; e < 8; ++e) o[h][e] = fmul2(o[h][e], a2);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if (!valid[r]) continue;               // stale shared memory: never multiplied in
        const int kk = slot + r * slot_step;
        const uint4 v0 = lds128(vst + kk * row_bytes);
        const uint4 v1 = lds128(vst + kk * row_bytes + 128);
        const uint32_t w[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float2 vf = bf16x2_to_f2(w[e]);
#pragma unroll
          for (int h = 0; h < G; ++h) o[h][e] = ffma2(make_float2(p[r][h], p[r][h]), vf, o[h][e]);
        }
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
        dec_issue(a, sm, pos, stage0, b, t_begin, t_end, ks, row_bytes, j + kDecStages, lane);
      }
    }

    // merge the 4 groups of the warp (lanes sub, sub + 8, sub + 16, sub + 24)
#pragma unroll
    for (int off = 8; off <= 16; off <<= 1) {
#pragma unroll
      for (int h = 0; h < G; ++h) {
        const float mo = __shfl_xor_sync(0xffffffffu, m[h], off);
        const float lo = __shfl_xor_sync(0xffffffffu, l[h], off);
        const float M = fmaxf(m[h], mo);
        const float Mr = M == -INFINITY ? 0.f : M;
        const float wa = fast_exp2(m[h] - Mr), wb = fast_exp2(mo - Mr);
        l[h] = l[h] * wa + lo * wb;
        m[h] = M;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float ox = __shfl_xor_sync(0xffffffffu, o[h][e].x, off);
          const float oy = __shfl_xor_sync(0xffffffffu, o[h][e].y, off);
          o[h][e] = make_float2(o[h][e].x * wa + ox * wb, o[h][e].y * wa + oy * wb);
        }
      }
    }
  }
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
  if (warp < kDecWarps && lane < 8) {
    const int sub = lane;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      float* r = red + (warp * G + h) * (kDecD + 2);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        r[sub * 8 + 2 * e] = o[h][e].x;
        r[sub * 8 + 2 * e + 1] = o[h][e].y;
        r[64 + sub * 8 + 2 * e] = o[h][4 + e].x;
        r[64 + sub * 8 + 2 * e + 1] = o[h][4 + e].y;
      }
      if (sub == 0) { r[kDecD] = m[h]; r[kDecD + 1] = l[h]; }
    }
  }
  __syncthreads();
  // merge the warps of each KV head and write (o, lse) or the split's partial row
  const int nph = kDecWarps / hkv;
  for (int t = threadIdx.x; t < a.hq * kDecD; t += kDecThreads) {
    const int head = t / kDecD, e = t % kDecD;
    const int g = head / G, h = head % G;
    float M = -INFINITY;
    for (int ph = 0; ph < nph; ++ph) M = fmaxf(M, red[((ph * hkv + g) * G + h) * (kDecD + 2) + kDecD]);
    const float Mr = M == -INFINITY ? 0.f : M;
    float L = 0.f, O = 0.f;
    for (int ph = 0; ph < nph; ++ph) {
      const float* r = red + ((ph * hkv + g) * G + h) * (kDecD + 2);
      const float w = fast_exp2(r[kDecD] - Mr);
      L += r[kDecD + 1] * w;
      O += r[e] * w;
    }
    const int64_t row = (int64_t)b * a.hq + head;
    if (a.nsplit == 1) {
      a.o[row * kDecD + e] = __float2bfloat16_rn(O / L);
      if (e == 0 && a.lse) a.lse[row] = (M + __log2f(L)) * 0.69314718055994531f;
    } else {
      float* pp = a.part + (row * a.nsplit + split) * (kDecD + 2);
      pp[e] = O;
      if (e == 0) { pp[kDecD] = M; pp[kDecD + 1] = L; }
    }
  }
}

}  // namespace esa
