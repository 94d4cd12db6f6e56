// esa_lib.cu - the C ABI of libesa (include/esa.h): argument checks, workspace
// layout and kernel launches. Every kernel lives in the .cuh files included here, so
// the library is one translation unit with one copy of the device status word.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <map>
#include <mutex>
#include <string>
#include <type_traits>

#include "../../include/esa.h"
#include "attn_decode.cuh"
#include "attn_pp.cuh"
#include "attn_simt.cuh"
#include "attn_tc.cuh"
#include "cca.cuh"
#include "common.cuh"
#include "compress.cuh"
#include "compress_tc.cuh"
#include "compress_pk.cuh"
#include "fit.cuh"
#include "moba.cuh"
#include "score.cuh"
#include "score_tc.cuh"
#include "topk.cuh"

namespace {

thread_local std::string g_err;
std::atomic<unsigned long long> g_launches{0};

esa_status_t fail(esa_status_t st, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return st;
}

esa_status_t ok() {
  g_err.clear();
  return ESA_OK;
}

esa_status_t check_launch(const char* what) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(ESA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return ESA_OK;
}

#define ESA_LAUNCH_CHECK(what)                         \
  do {                                                 \
    const esa_status_t st_ = check_launch(what);       \
    if (st_ != ESA_OK) return st_;                     \
  } while (0)

#define ESA_CUDA(call)                                                               \
  do {                                                                               \
    const cudaError_t e_ = (call);                                                   \
    if (e_ != cudaSuccess) return fail(ESA_ERR_CUDA, "%s: %s", #call, cudaGetErrorString(e_)); \
  } while (0)

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t up256(size_t x) { return (x + 255) & ~size_t(255); }
inline int64_t cdiv(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Region rule of a chunk [c0, c1): lo = min(c0, max(n_init, c0 - window)).
struct Regions {
  int64_t lo, ni, mid0, n_mid;
};
Regions regions(int64_t c0, const esa_params_t& p) {
  Regions r;
  r.lo = std::min<int64_t>(c0, std::max<int64_t>(p.n_init, c0 - p.window));
  r.ni = std::min<int64_t>(p.n_init, r.lo);
  r.mid0 = p.n_init;
  r.n_mid = std::max<int64_t>(0, r.lo - p.n_init);
  return r;
}

// Carves a workspace into 256-byte aligned regions in a fixed order.
struct Carver {
  uint8_t* base;
  size_t off = 0;
  template <typename T>
  T* take(size_t count) {
    T* p = base ? reinterpret_cast<T*>(base + off) : nullptr;
    off += up256(count * sizeof(T));
    return p;
  }
};

template <typename K>
esa_status_t set_max_smem(K kernel, int bytes) {
  ESA_CUDA(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes));
  return ESA_OK;
}

// ------------------------------------------------------ set-up once per CUDA context --
// Kernel attributes (dynamic shared memory, cluster sizes), occupancy answers and the
// no-alloc scratch address belong to the CUDA context they were made in, which is not
// always the device's primary context (a plugin inside another runtime may make its own
// current). Each is made once per context and remembered under the context's id
// (cuCtxGetId: unique for the life of the process, never reused), so a context created
// after another was destroyed never inherits its set-up. One mutex guards the table:
// calls from several host threads neither race on it nor repeat the set-up.
struct CtxFns {
  PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  PFN_cuCtxGetId_v12000 get_id = nullptr;
};

const CtxFns& ctx_fns() {
  static const CtxFns fns = [] {
    CtxFns f;
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(fn);
    fn = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      f.get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(fn);
    cudaGetLastError();
    return f;
  }();
  return fns;
}

// The id of the context the runtime uses for this thread's calls (the device's primary
// context, initialised here, when none is current).
esa_status_t current_context_id(unsigned long long* id) {
  const CtxFns& f = ctx_fns();
  if (!f.get_current || !f.get_id) return fail(ESA_ERR_CUDA, "cuCtxGetCurrent / cuCtxGetId not available");
  CUcontext ctx = nullptr;
  if (f.get_current(&ctx) != CUDA_SUCCESS) return fail(ESA_ERR_CUDA, "cuCtxGetCurrent failed");
  if (!ctx) {
    ESA_CUDA(cudaFree(nullptr));     // no allocation: makes the runtime's context current
    if (f.get_current(&ctx) != CUDA_SUCCESS || !ctx) return fail(ESA_ERR_CUDA, "no current CUDA context");
  }
  if (f.get_id(ctx, id) != CUDA_SUCCESS) return fail(ESA_ERR_CUDA, "cuCtxGetId failed");
  return ESA_OK;
}

std::mutex g_setup_mu;
std::map<std::pair<const void*, unsigned long long>, intptr_t> g_setup;   // (what, context id) -> value

// The value `make` produced for `what` in the current context, making it on the first
// call there (make returns ESA_OK and writes *value; a failure is not remembered).
template <class F>
esa_status_t per_context(const void* what, intptr_t* value, F&& make) {
  unsigned long long id = 0;
  const esa_status_t st = current_context_id(&id);
  if (st != ESA_OK) return st;
  std::lock_guard<std::mutex> lock(g_setup_mu);
  const auto key = std::make_pair(what, id);
  const auto it = g_setup.find(key);
  if (it != g_setup.end()) {
    *value = it->second;
    return ESA_OK;
  }
  intptr_t v = 0;
  const esa_status_t made = make(&v);
  if (made != ESA_OK) return made;
  g_setup.emplace(key, v);
  *value = v;
  return ESA_OK;
}

// Runs `set` (kernel attributes) once per context; `what` names the group of kernels.
template <class F>
esa_status_t once_per_context(const void* what, F&& set) {
  intptr_t unused = 0;
  return per_context(what, &unused, [&](intptr_t* v) {
    *v = 1;
    return set();
  });
}

esa_status_t check_params(const esa_params_t& p) {
  if (p.n_init < 0 || p.window < 0) return fail(ESA_ERR_INVALID_ARG, "n_init and window must be >= 0");
  if (p.topk < 1) return fail(ESA_ERR_INVALID_ARG, "topk must be >= 1 (got %d)", p.topk);
  if (p.eps < 0 || p.eps > 64) return fail(ESA_ERR_INVALID_ARG, "eps must be in [0, 64] (got %d)", p.eps);
  if (std::isnan(p.clamp_c) || p.clamp_c < 0.f) return fail(ESA_ERR_INVALID_ARG, "clamp_c must be >= 0 or +inf");
  return ESA_OK;
}

// ------------------------------------------------------------------ score_select --
// Scoring path: few queries -> registers (S stored); a prefill chunk -> tensor cores
// (two passes, S never stored); anything else -> SIMT tiles (S stored).
enum class ScorePath { Small, TensorCore, Tiled };

// With ng > 1 groups (per-head selection) there is no tensor-core path, and the small
// path needs the groups to split a key's lanes (LPK = min(d_c, 128) / 4, 32 from 128 on).
ScorePath score_path(int32_t batch, int32_t lq, int64_t n_cap, int32_t d_c, int ng = 1) {
  const int lpk = d_c >= 128 ? 32 : d_c / 4;
  if (lq <= esa::kScoreSmallLq && (d_c == 16 || d_c == 32 || d_c == 64 || d_c == 128 || d_c == 256) &&
      lpk % ng == 0)
    return ScorePath::Small;
  if (ng > 1) return ScorePath::Tiled;
  // TMA row coordinates are 32-bit
  const bool rows_fit = (int64_t)batch * n_cap < ((int64_t)1 << 31) && (int64_t)batch * lq < ((int64_t)1 << 31);
  if (lq >= 16 && rows_fit && (d_c == 32 || d_c == 64 || d_c == 128)) return ScorePath::TensorCore;
  return ScorePath::Tiled;
}

struct SelWs {
  uint32_t* m_key;   // [B, lq] order keys of the per-query maxima (cleared before scoring)
  float* S;          // [B, lq, n_mid] raw scores (SIMT paths)
  float* s;          // [B, n_mid] chunk-summed corrected scores (tensor-core path)
  uint32_t* u;       // [B, n_mid] order keys, when a cluster CTA's range exceeds its shared memory
  size_t bytes;
};

SelWs carve_select(void* ws, int32_t batch, int32_t lq, int64_t n_mid, ScorePath path) {
  Carver c{reinterpret_cast<uint8_t*>(ws)};
  SelWs w;
  w.m_key = c.take<uint32_t>((size_t)batch * lq);
  w.S = path == ScorePath::TensorCore ? nullptr : c.take<float>((size_t)batch * lq * n_mid);
  w.s = path == ScorePath::TensorCore ? c.take<float>((size_t)batch * n_mid) : nullptr;
  w.u = c.take<uint32_t>((size_t)batch * (n_mid + 64));   // up to 16 cluster CTAs, each range padded to 4
  w.bytes = c.off;
  return w;
}

// Cluster size of the selection kernel: 16 CTAs only when the middle overflows the
// shared memory of 8 (8 x kSelUCap keys) and `batch` such clusters (one per sequence)
// can be resident at once; else the portable 8. A 16-CTA cluster needs 16 free SMs in
// one GPC, which a chunked prefill's attention (128 CTAs, one per SM) does not leave:
// its next chunk's selection then waited for the attention to end (8-CTA clusters:
// 32K prefill 6.05 -> 5.65 ms). Occupancy is queried once per context.
int select_cluster_size(int32_t batch, int64_t n_mid) {
  if (n_mid <= (int64_t)8 * esa::kSelUCap) return 8;
  static const char what = 0;
  intptr_t max16 = -1;          // -1: 16-CTA clusters unavailable
  const esa_status_t st = per_context(&what, &max16, [](intptr_t* v) {
    *v = -1;
    if (cudaFuncSetAttribute(esa::select_cluster_kernel<16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
        cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(16, 1, 1);
      cfg.blockDim = dim3(esa::kSelThreads);
      cfg.dynamicSmemBytes = esa::kSelSmemBytes;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 16;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, esa::select_cluster_kernel<16>, &cfg) == cudaSuccess && n >= 1) *v = n;
    }
    cudaGetLastError();   // a refused query is not an error of this call
    return ESA_OK;
  });
  // (smaller clusters for many selections were measured slower: a CTA then sweeps tens
  // of thousands of keys through the global scratch)
  return (st == ESA_OK && max16 > 0 && batch <= max16) ? 16 : 8;
}

// 2D tensor map over a row-major fp32 matrix [rows, cols], 32 x 128 boxes, 128-byte
// swizzle (the shared-memory layout the tf32 MMA descriptors expect).
esa_status_t get_encoder(PFN_cuTensorMapEncodeTiled_v12000* out) {
  // looked up once (a thread-safe static initialisation); the driver's entry point is
  // the same for every context
  static const PFN_cuTensorMapEncodeTiled_v12000 encode = [] {
    cudaDriverEntryPointQueryResult q;
    void* fn = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      fn = nullptr;
    cudaGetLastError();
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  }();
  if (!encode) return fail(ESA_ERR_CUDA, "cuTensorMapEncodeTiled not available");
  *out = encode;
  return ESA_OK;
}

// 2D tensor map over bf16 rows of 128 elements [rows, 128], boxes of one row x 64
// columns with 128-byte swizzle: the form tile::gather4 loads (4 rows per instruction).
esa_status_t make_tmap_rows_bf16(CUtensorMap* m, const void* base, uint64_t rows) {
  PFN_cuTensorMapEncodeTiled_v12000 encode;
  esa_status_t st = get_encoder(&encode);
  if (st != ESA_OK) return st;
  cuuint64_t dims[2] = {128, rows};
  cuuint64_t strides[1] = {128 * 2};
  cuuint32_t box[2] = {64, 1};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ESA_ERR_CUDA, "cuTensorMapEncodeTiled (rows) failed (%d)", (int)r);
  return ESA_OK;
}

// 3D tensor map over bf16 [tokens, heads, 128]; a box is box_tokens consecutive tokens x
// box_heads consecutive heads x 64 columns, 128-byte swizzle (rows ordered token-major).
esa_status_t make_tmap_box_bf16(CUtensorMap* m, const void* base, uint64_t heads, uint64_t tokens,
                                uint32_t box_heads, uint32_t box_tokens) {
  PFN_cuTensorMapEncodeTiled_v12000 encode;
  esa_status_t st = get_encoder(&encode);
  if (st != ESA_OK) return st;
  cuuint64_t dims[3] = {128, heads, tokens};
  cuuint64_t strides[2] = {128 * 2, heads * 128 * 2};
  cuuint32_t box[3] = {64, box_heads, box_tokens};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ESA_ERR_CUDA, "cuTensorMapEncodeTiled (box) failed (%d)", (int)r);
  return ESA_OK;
}

esa_status_t make_tmap_f32(CUtensorMap* m, const float* base, uint64_t rows, uint64_t cols) {
  PFN_cuTensorMapEncodeTiled_v12000 encode;
  esa_status_t st0 = get_encoder(&encode);
  if (st0 != ESA_OK) return st0;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * sizeof(float)};
  cuuint32_t box[2] = {32, 128};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ESA_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return ESA_OK;
}

template <int DC, int NG>
void launch_score_small_ng(const float* q_c, const float* k_c, int lq, int64_t n_cap, int64_t mid0, int64_t n_mid,
                           int batch, float* S, uint32_t* m_key, const esa::VarLen& vl, cudaStream_t s) {
  // one wave of two CTAs per SM over all sequences, each CTA a multiple of a stage; with
  // variable lengths four such waves for the longest possible middles, so that the CTAs
  // of short sequences end at once and the block scheduler spreads the rest
  constexpr int64_t ks = esa::SmallScoreShape<DC>::KS;
  const int64_t waves = vl.len ? 4 : 1;
  const int64_t per_seq = std::max<int64_t>(1, std::min<int64_t>(cdiv(n_mid, ks), waves * (2 * 148) / batch));
  const int64_t keys_per_cta = cdiv(cdiv(n_mid, per_seq), ks) * ks;
  const dim3 grid((unsigned)cdiv(n_mid, keys_per_cta), batch);
  static const char what = 0;   // one per instantiation
  // a failure here shows as the launch's error, which the caller checks
  once_per_context(&what, [] {
    esa_status_t st = set_max_smem(esa::score_small_kernel<DC, 1, NG>, esa::kSsSmemBytes);
    if (st == ESA_OK) st = set_max_smem(esa::score_small_kernel<DC, esa::kScoreSmallLq, NG>, esa::kSsSmemBytes);
    return st;
  });
  if (lq == 1)
    esa::score_small_kernel<DC, 1, NG><<<grid, esa::kSsThreads, esa::kSsSmemBytes, s>>>(
        q_c, k_c, lq, n_cap, mid0, n_mid, keys_per_cta, S, m_key, vl);
  else
    esa::score_small_kernel<DC, esa::kScoreSmallLq, NG><<<grid, esa::kSsThreads, esa::kSsSmemBytes, s>>>(
        q_c, k_c, lq, n_cap, mid0, n_mid, keys_per_cta, S, m_key, vl);
}

// groups must split a key's LPK lanes evenly (checked by score_path)
template <int DC>
void launch_score_small(const float* q_c, const float* k_c, int lq, int64_t n_cap, int64_t mid0, int64_t n_mid,
                        int batch, int ng, float* S, uint32_t* m_key, const esa::VarLen& vl, cudaStream_t s) {
  constexpr int LPK = esa::SmallScoreShape<DC>::LPK;
  if (ng == 1) launch_score_small_ng<DC, 1>(q_c, k_c, lq, n_cap, mid0, n_mid, batch, S, m_key, vl, s);
  else if (ng == 2) launch_score_small_ng<DC, 2>(q_c, k_c, lq, n_cap, mid0, n_mid, batch, S, m_key, vl, s);
  else if (ng == 4) launch_score_small_ng<DC, 4>(q_c, k_c, lq, n_cap, mid0, n_mid, batch, S, m_key, vl, s);
  else if constexpr (LPK % 8 == 0)
    launch_score_small_ng<DC, 8>(q_c, k_c, lq, n_cap, mid0, n_mid, batch, S, m_key, vl, s);
}

}  // namespace

// Every exported function below is declared extern "C" in esa.h, which gives these
// definitions C linkage.

const char* esa_version(void) { return "libesa 0.1 (sm_100a)"; }

const char* esa_last_error(void) { return g_err.c_str(); }

uint64_t esa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

esa_status_t esa_wait_selftest(uint64_t limit_ns, void* stream) {
  if (limit_ns < 1000 || limit_ns > ESA_WAIT_LIMIT_NS)
    return fail(ESA_ERR_INVALID_ARG, "limit_ns must be in [1 us, %llu ns]", (unsigned long long)ESA_WAIT_LIMIT_NS);
  esa::wait_selftest_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(limit_ns);
  ESA_LAUNCH_CHECK("wait_selftest_kernel");
  return ok();
}

esa_status_t esa_device_status(void* stream) {
  ESA_CUDA(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
  unsigned long long v = 0;
  ESA_CUDA(cudaMemcpyFromSymbol(&v, esa::g_status, sizeof(v)));
  if (v == 0) return ok();
  const unsigned long long zero = 0;
  ESA_CUDA(cudaMemcpyToSymbol(esa::g_status, &zero, sizeof(zero)));
  const unsigned code = (unsigned)(v >> 32), site = (unsigned)(v & 0xffffffffu);
  if (code == 5u) return fail(ESA_ERR_CUDA, "kernel site %u found its shared memory misaligned and stopped", site);
  if (code == 1u)
    return fail(ESA_ERR_INVALID_ARG, "kernel site %u read a sequence length outside [1, n_cap] (clamped)", site);
  if (code == 6u)
    return fail(ESA_ERR_INVALID_ARG,
                "site %u: a Cholesky pivot was not positive (the matrix is not positive definite; a ridge helps)",
                site);
  return fail(ESA_ERR_TIMEOUT, "device wait ran out at site %u (status %u)", site, code);
}

// ------------------------------------------------------- packed-weight compression --
size_t esa_compress_pack_size(int32_t n_heads_in, int32_t head_dim, int32_t d_out) {
  if (n_heads_in <= 0 || head_dim <= 0 || d_out != 128) return 0;
  const int64_t K = (int64_t)n_heads_in * head_dim;
  if (K % 512 || K > (int64_t)1 << 20) return 0;
  return (size_t)(2 * 128 * K * 2);
}

esa_status_t esa_compress_pack(const float* w, int32_t n_heads_in, int32_t n_heads_out, int32_t head_dim,
                               int32_t d_out, void* packed, size_t packed_bytes, void* stream) {
  if (!w || !packed) return fail(ESA_ERR_INVALID_ARG, "null pointer");
  if (n_heads_in <= 0 || n_heads_out <= 0 || n_heads_out % n_heads_in)
    return fail(ESA_ERR_INVALID_ARG, "n_heads_out (%d) must be a positive multiple of n_heads_in (%d)", n_heads_out,
                n_heads_in);
  const size_t need = esa_compress_pack_size(n_heads_in, head_dim, d_out);
  if (need == 0)
    return fail(ESA_ERR_UNSUPPORTED, "packed compression needs d_out 128 and n_heads_in * head_dim a multiple of 512");
  if (packed_bytes < need) return fail(ESA_ERR_INVALID_ARG, "packed buffer %zu bytes, need %zu", packed_bytes, need);
  if (!aligned(packed, 16)) return fail(ESA_ERR_INVALID_ARG, "packed buffer must be 16-byte aligned");
  const int K = n_heads_in * head_dim;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  esa::compress_pack_kernel<<<dim3(K / 64, 2), 256, 0, s>>>(w, n_heads_in, n_heads_out / n_heads_in, head_dim, K,
                                                            static_cast<__nv_bfloat16*>(packed));
  ESA_LAUNCH_CHECK("compress_pack_kernel");
  return ok();
}

namespace {
// 2D bf16 tensor map [outer, inner] (inner contiguous, row pitch in elements), boxes
// of 128 rows x 64 columns with 128-byte swizzle: K-major MMA operand tiles.
esa_status_t make_tmap_kmajor_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                                   uint64_t pitch_elems) {
  PFN_cuTensorMapEncodeTiled_v12000 encode;
  esa_status_t st = get_encoder(&encode);
  if (st != ESA_OK) return st;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {pitch_elems * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ESA_ERR_CUDA, "cuTensorMapEncodeTiled (k-major) failed (%d)", (int)r);
  return ESA_OK;
}

// Cluster size for the packed compression: 16 CTAs when the device can co-schedule
// them (one CTA per SM, so a whole 16-SM group), else the portable 8.
esa_status_t pk_cluster_size(int* cl) {
  static const char what = 0;
  intptr_t best = 8;
  const esa_status_t st = per_context(&what, &best, [](intptr_t* v) {
    *v = 8;
    ESA_CUDA(cudaFuncSetAttribute(esa::compress_pk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  esa::kCpSmemBytes));
    if (cudaFuncSetAttribute(esa::compress_pk_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
        cudaSuccess) {
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3(16, 1, 2);
      cfg.blockDim = dim3(esa::kCpThreads);
      cfg.dynamicSmemBytes = esa::kCpSmemBytes;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = 16;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      int n = 0;
      if (cudaOccupancyMaxActiveClusters(&n, esa::compress_pk_kernel, &cfg) == cudaSuccess && n >= 1) *v = 16;
      cudaGetLastError();   // a refused query is not an error of this call
    }
    return ESA_OK;
  });
  if (st != ESA_OK) return st;
  *cl = (int)best;
  return ESA_OK;
}
}  // namespace

namespace {
esa_status_t compress_packed_impl(const void* x, int64_t rows, int64_t x_row_stride, int32_t n_heads_in,
                                  int32_t head_dim, const void* packed, int32_t d_out, float* y, int64_t y_row_stride,
                                  const esa::VarLen& yl, void* stream);
}  // namespace

esa_status_t esa_compress_packed(const void* x, int64_t rows, int64_t x_row_stride, int32_t n_heads_in,
                                 int32_t head_dim, const void* packed, int32_t d_out, float* y,
                                 int64_t y_row_stride, void* stream) {
  return compress_packed_impl(x, rows, x_row_stride, n_heads_in, head_dim, packed, d_out, y, y_row_stride,
                              esa::VarLen{}, stream);
}

esa_status_t esa_compress_packed_varlen(const void* x, int32_t batch, int64_t x_row_stride, int32_t n_heads_in,
                                        int32_t head_dim, const void* packed, int32_t d_out, float* k_c,
                                        int64_t n_cap, const int64_t* seq_len, void* stream) {
  if (!seq_len) return fail(ESA_ERR_INVALID_ARG, "null pointer");
  if (n_cap < 1) return fail(ESA_ERR_INVALID_ARG, "n_cap must be >= 1");
  return compress_packed_impl(x, batch, x_row_stride, n_heads_in, head_dim, packed, d_out, k_c, d_out,
                              esa::VarLen{seq_len, n_cap, 0, 0, 1}, stream);
}

namespace {
esa_status_t compress_packed_impl(const void* x, int64_t rows, int64_t x_row_stride, int32_t n_heads_in,
                                  int32_t head_dim, const void* packed, int32_t d_out, float* y, int64_t y_row_stride,
                                  const esa::VarLen& yl, void* stream) {
  if (rows < 0) return fail(ESA_ERR_INVALID_ARG, "rows must be >= 0");
  if (rows == 0) return ok();
  if (!x || !packed || !y) return fail(ESA_ERR_INVALID_ARG, "null pointer");
  if (esa_compress_pack_size(n_heads_in, head_dim, d_out) == 0)
    return fail(ESA_ERR_UNSUPPORTED, "packed compression needs d_out 128 and n_heads_in * head_dim a multiple of 512");
  const int K = n_heads_in * head_dim;
  if (x_row_stride < K || x_row_stride % 8) return fail(ESA_ERR_INVALID_ARG, "x_row_stride must be >= n_heads_in * head_dim and a multiple of 8");
  if (y_row_stride < 128 || y_row_stride % 4) return fail(ESA_ERR_INVALID_ARG, "y_row_stride must be >= 128 and a multiple of 4");
  if (!aligned(x, 16) || !aligned(packed, 16) || !aligned(y, 16))
    return fail(ESA_ERR_INVALID_ARG, "x, packed and y must be 16-byte aligned");
  int cl = 8;
  esa_status_t st = pk_cluster_size(&cl);
  if (st != ESA_OK) return st;
  // small calls (a chunk's keys or queries, a decode step) take 8-CTA clusters, which
  // fit beside a running attention kernel (a 16-CTA cluster needs 16 free SMs in a GPC)
  if (K % (64 * cl) || rows <= 4096) cl = 8;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  CUtensorMap tw;
  st = make_tmap_kmajor_bf16(&tw, packed, (uint64_t)K, 256, (uint64_t)K);
  if (st != ESA_OK) return st;
  const int64_t max_rows = (int64_t)65535 * esa::kCpRows;
  for (int64_t r0 = 0; r0 < rows; r0 += max_rows) {
    const int64_t nr = std::min(rows - r0, max_rows);
    CUtensorMap tx;
    st = make_tmap_kmajor_bf16(&tx, static_cast<const __nv_bfloat16*>(x) + r0 * x_row_stride, (uint64_t)K,
                               (uint64_t)nr, (uint64_t)x_row_stride);
    if (st != ESA_OK) return st;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)cl, (unsigned)cdiv(nr, esa::kCpRows), 2);
    cfg.blockDim = dim3(esa::kCpThreads);
    cfg.dynamicSmemBytes = esa::kCpSmemBytes;
    cfg.stream = s;
    cudaLaunchAttribute at[1];
    at[0].id = cudaLaunchAttributeClusterDimension;
    at[0].val.clusterDim.x = (unsigned)cl;
    at[0].val.clusterDim.y = 1;
    at[0].val.clusterDim.z = 1;
    cfg.attrs = at;
    cfg.numAttrs = 1;
    if (yl.len && r0 > 0) return fail(ESA_ERR_UNSUPPORTED, "too many sequences");
    cudaLaunchKernelEx(&cfg, esa::compress_pk_kernel, tx, tw, nr, K, y + r0 * y_row_stride, y_row_stride, yl);
    ESA_LAUNCH_CHECK("compress_pk_kernel");
  }
  return ok();
}
}  // namespace

// ------------------------------------------------------------------ esa_compress --
esa_status_t esa_compress(const void* x, esa_dtype_t x_dtype, int64_t rows, int64_t x_row_stride,
                          int32_t n_heads_in, int32_t n_heads_out, int32_t head_dim, const float* w, int32_t d_out,
                          float* y, int64_t y_row_stride, void* stream) {
  if (rows < 0) return fail(ESA_ERR_INVALID_ARG, "rows must be >= 0");
  if (rows == 0) return ok();
  if (!x || !w || !y) return fail(ESA_ERR_INVALID_ARG, "null pointer");
  if (x_dtype != ESA_F32 && x_dtype != ESA_BF16) return fail(ESA_ERR_INVALID_ARG, "bad dtype %d", (int)x_dtype);
  if (n_heads_in <= 0 || n_heads_out <= 0 || n_heads_out % n_heads_in)
    return fail(ESA_ERR_INVALID_ARG, "n_heads_out (%d) must be a positive multiple of n_heads_in (%d)", n_heads_out,
                n_heads_in);
  if (head_dim != 64 && head_dim != 128) return fail(ESA_ERR_UNSUPPORTED, "head_dim %d (64 or 128)", head_dim);
  if (d_out <= 0 || d_out % 16 || d_out > 256) return fail(ESA_ERR_UNSUPPORTED, "d_out %d (multiple of 16, <= 256)", d_out);
  if (y_row_stride < d_out) return fail(ESA_ERR_INVALID_ARG, "y_row_stride < d_out");
  if (x_row_stride < (int64_t)n_heads_in * head_dim || x_row_stride % 8)
    return fail(ESA_ERR_INVALID_ARG, "x_row_stride must be >= n_heads_in * head_dim and a multiple of 8");
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int g = n_heads_out / n_heads_in;
  if (x_dtype == ESA_BF16 && d_out == esa::kCtN && (g == 1 || g == 2 || g == 4)) {
    // tensor-core path: 8-CTA clusters split the reduction, 128 rows x 64 columns per CTA
    static const char what = 0;
    const esa_status_t sa = once_per_context(&what, [] {
      esa_status_t st = set_max_smem(esa::compress_tc_kernel<1>, esa::kCtSmemBytes);
      if (st == ESA_OK) st = set_max_smem(esa::compress_tc_kernel<2>, esa::kCtSmemBytes);
      if (st == ESA_OK) st = set_max_smem(esa::compress_tc_kernel<4>, esa::kCtSmemBytes);
      return st;
    });
    if (sa != ESA_OK) return sa;
    const int64_t max_rows = (int64_t)65535 * esa::kCtRows;
    for (int64_t r0 = 0; r0 < rows; r0 += max_rows) {
      const int64_t nr = std::min(rows - r0, max_rows);
      const dim3 grid(esa::kCtCluster, (unsigned)cdiv(nr, esa::kCtRows), esa::kCtN / esa::kCtNS);
      const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x) + r0 * x_row_stride;
      float* yb = y + r0 * y_row_stride;
      if (g == 1)
        esa::compress_tc_kernel<1><<<grid, esa::kCtThreads, esa::kCtSmemBytes, s>>>(xb, nr, x_row_stride, n_heads_in,
                                                                                    head_dim, w, yb, y_row_stride);
      else if (g == 2)
        esa::compress_tc_kernel<2><<<grid, esa::kCtThreads, esa::kCtSmemBytes, s>>>(xb, nr, x_row_stride, n_heads_in,
                                                                                    head_dim, w, yb, y_row_stride);
      else
        esa::compress_tc_kernel<4><<<grid, esa::kCtThreads, esa::kCtSmemBytes, s>>>(xb, nr, x_row_stride, n_heads_in,
                                                                                    head_dim, w, yb, y_row_stride);
      ESA_LAUNCH_CHECK("compress_tc_kernel");
    }
    return ok();
  }
  const int ct = d_out % 32 == 0 ? 32 : 16;
  dim3 grid((unsigned)cdiv(rows, esa::kCmpRT), d_out / ct);
  if (x_dtype == ESA_F32) {
    if (ct == 32)
      esa::compress_kernel<float, 32><<<grid, esa::kCmpThreads, 0, s>>>(static_cast<const float*>(x), rows, x_row_stride, n_heads_in,
                                                                       n_heads_out, head_dim, w, d_out, y, y_row_stride);
    else
      esa::compress_kernel<float, 16><<<grid, esa::kCmpThreads, 0, s>>>(static_cast<const float*>(x), rows, x_row_stride, n_heads_in,
                                                                       n_heads_out, head_dim, w, d_out, y, y_row_stride);
  } else {
    const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
    if (ct == 32)
      esa::compress_kernel<__nv_bfloat16, 32><<<grid, esa::kCmpThreads, 0, s>>>(xb, rows, x_row_stride, n_heads_in, n_heads_out,
                                                                               head_dim, w, d_out, y, y_row_stride);
    else
      esa::compress_kernel<__nv_bfloat16, 16><<<grid, esa::kCmpThreads, 0, s>>>(xb, rows, x_row_stride, n_heads_in, n_heads_out,
                                                                               head_dim, w, d_out, y, y_row_stride);
  }
  ESA_LAUNCH_CHECK("compress_kernel");
  return ok();
}

// ------------------------------------------------------------------ score_select --
namespace {

size_t score_select_ws(int32_t batch, int32_t lq, int64_t n_cap, int64_t c0, int32_t d_c, int ng,
                       const esa_params_t& p) {
  if (batch <= 0 || lq <= 0 || ng <= 0) return 0;
  const Regions r = regions(c0, p);
  return carve_select(nullptr, batch * ng, lq, r.n_mid, score_path(batch, lq, n_cap, d_c, ng)).bytes;
}

esa_status_t score_select_impl(const float* q_c, const float* k_c, int32_t batch, int32_t lq, int64_t n_cap,
                               int64_t c0, int32_t d_c, int ng, esa_params_t p, int32_t* idx_out,
                               int32_t* count_out, float* score_out, void* workspace, size_t ws_bytes,
                               void* stream, const int64_t* seq_len = nullptr);

}  // namespace

size_t esa_score_select_workspace_size(int32_t batch, int32_t lq, int64_t n_cap, int64_t c0, int32_t d_c,
                                       esa_params_t p) {
  return score_select_ws(batch, lq, n_cap, c0, d_c, 1, p);
}

size_t esa_score_select_heads_workspace_size(int32_t batch, int32_t lq, int64_t n_cap, int64_t c0, int32_t d_c,
                                             int32_t n_groups, esa_params_t p) {
  return score_select_ws(batch, lq, n_cap, c0, d_c, n_groups, p);
}

esa_status_t esa_score_select(const float* q_c, const float* k_c, int32_t batch, int32_t lq, int64_t n_cap,
                              int64_t c0, int32_t d_c, esa_params_t p, int32_t* idx_out, int32_t* count_out,
                              float* score_out, void* workspace, size_t ws_bytes, void* stream) {
  return score_select_impl(q_c, k_c, batch, lq, n_cap, c0, d_c, 1, p, idx_out, count_out, score_out, workspace,
                           ws_bytes, stream);
}

esa_status_t esa_score_select_heads(const float* q_c, const float* k_c, int32_t batch, int32_t lq, int64_t n_cap,
                                    int64_t c0, int32_t d_c, int32_t n_groups, esa_params_t p, int32_t* idx_out,
                                    int32_t* count_out, float* score_out, void* workspace, size_t ws_bytes,
                                    void* stream) {
  if (n_groups != 1 && n_groups != 2 && n_groups != 4 && n_groups != 8)
    return fail(ESA_ERR_UNSUPPORTED, "n_groups %d (1, 2, 4 or 8)", n_groups);
  return score_select_impl(q_c, k_c, batch, lq, n_cap, c0, d_c, n_groups, p, idx_out, count_out, score_out,
                           workspace, ws_bytes, stream);
}

size_t esa_score_select_varlen_workspace_size(int32_t batch, int64_t n_cap, int32_t d_c, int32_t n_groups,
                                              esa_params_t p) {
  if (n_cap < 1) return 0;
  return score_select_ws(batch, 1, n_cap, n_cap - 1, d_c, n_groups, p);
}

esa_status_t esa_score_select_varlen(const float* q_c, const float* k_c, int32_t batch, int64_t n_cap,
                                     const int64_t* seq_len, int32_t d_c, int32_t n_groups, esa_params_t p,
                                     int32_t* idx_out, int32_t* count_out, float* score_out, void* workspace,
                                     size_t ws_bytes, void* stream) {
  if (n_groups != 1 && n_groups != 2 && n_groups != 4 && n_groups != 8)
    return fail(ESA_ERR_UNSUPPORTED, "n_groups %d (1, 2, 4 or 8)", n_groups);
  if (!seq_len) return fail(ESA_ERR_INVALID_ARG, "null pointer");
  if (n_cap < 1) return fail(ESA_ERR_INVALID_ARG, "n_cap must be >= 1");
  return score_select_impl(q_c, k_c, batch, 1, n_cap, n_cap - 1, d_c, n_groups, p, idx_out, count_out, score_out,
                           workspace, ws_bytes, stream, seq_len);
}

namespace {

esa_status_t score_select_impl(const float* q_c, const float* k_c, int32_t batch, int32_t lq, int64_t n_cap,
                               int64_t c0, int32_t d_c, int ng, esa_params_t p, int32_t* idx_out,
                               int32_t* count_out, float* score_out, void* workspace, size_t ws_bytes,
                               void* stream, const int64_t* seq_len) {
  esa_status_t st = check_params(p);
  if (st != ESA_OK) return st;
  if (batch <= 0) return fail(ESA_ERR_INVALID_ARG, "batch must be >= 1");
  if (lq < 1 || lq > 4096) return fail(ESA_ERR_INVALID_ARG, "lq must be in [1, 4096] (got %d)", lq);
  if (c0 < 0 || c0 + lq > n_cap) return fail(ESA_ERR_INVALID_ARG, "need 0 <= c0 and c0 + lq <= n_cap");
  if (d_c <= 0 || d_c % 16 || d_c > 256) return fail(ESA_ERR_UNSUPPORTED, "d_c %d (multiple of 16, <= 256)", d_c);
  if (!q_c || !k_c || !idx_out || !count_out) return fail(ESA_ERR_INVALID_ARG, "null pointer");
  if (!aligned(q_c, 16) || !aligned(k_c, 16)) return fail(ESA_ERR_INVALID_ARG, "q_c and k_c need 16-byte alignment");
  const Regions r = regions(c0, p);
  if (r.n_mid > (int64_t)1 << 30) return fail(ESA_ERR_UNSUPPORTED, "middle longer than 2^30 tokens");
  if (d_c % ng || (ng > 1 && (d_c / ng) % 16 && score_path(batch, lq, n_cap, d_c, ng) != ScorePath::Small))
    return fail(ESA_ERR_UNSUPPORTED, "d_c %d in %d groups: each group needs a multiple of 16 columns here", d_c, ng);
  const int64_t vb = (int64_t)batch * ng;   // independent selections: sequence x group
  if (vb > 65535) return fail(ESA_ERR_UNSUPPORTED, "batch x groups must be <= 65535 (got %lld)", (long long)vb);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // a variable-length batch (c0 = n_cap - 1 here: the longest middle) selects per sequence
  // in the selection kernel, so it always scores
  const esa::VarLen vl_score{seq_len, n_cap, p.n_init, p.window, 1};
  const esa::VarLen vl_sel{seq_len, n_cap, p.n_init, p.window, ng};
  const int64_t kk = std::min<int64_t>(p.topk, r.n_mid);
  const bool need_scores = r.n_mid > p.topk || ((score_out || seq_len) && r.n_mid > 0);
  if (need_scores) {
    const ScorePath path = score_path(batch, lq, n_cap, d_c, ng);
    if (seq_len && path != ScorePath::Small)
      return fail(ESA_ERR_UNSUPPORTED, "variable lengths need one query and d_c in {16, 32, 64, 128, 256}");
    const SelWs need = carve_select(nullptr, (int32_t)vb, lq, r.n_mid, path);
    if (!workspace || ws_bytes < need.bytes || !aligned(workspace, 256))
      return fail(ESA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned (got %zu)", need.bytes, ws_bytes);
    const SelWs w = carve_select(workspace, (int32_t)vb, lq, r.n_mid, path);
    ESA_CUDA(cudaMemsetAsync(w.m_key, 0, (size_t)vb * lq * sizeof(uint32_t), s));
    if (path == ScorePath::Small) {
      auto launch = [&](auto dc) {
        launch_score_small<decltype(dc)::value>(q_c, k_c, lq, n_cap, r.mid0, r.n_mid, batch, ng, w.S, w.m_key,
                                                vl_score, s);
      };
      switch (d_c) {
        case 16: launch(std::integral_constant<int, 16>{}); break;
        case 32: launch(std::integral_constant<int, 32>{}); break;
        case 64: launch(std::integral_constant<int, 64>{}); break;
        case 128: launch(std::integral_constant<int, 128>{}); break;
        default: launch(std::integral_constant<int, 256>{}); break;
      }
      ESA_LAUNCH_CHECK("score_small_kernel");
    } else if (path == ScorePath::Tiled) {
      dim3 grid((unsigned)cdiv(r.n_mid, esa::kScT), (unsigned)cdiv(lq, esa::kScT), (unsigned)vb);
      esa::score_tiled_kernel<<<grid, 256, 0, s>>>(q_c, k_c, lq, n_cap, r.mid0, r.n_mid, d_c, ng, w.S, w.m_key);
      ESA_LAUNCH_CHECK("score_tiled_kernel");
    }
    if (path == ScorePath::TensorCore) {
      CUtensorMap tm_k, tm_q;
      st = make_tmap_f32(&tm_k, k_c, (uint64_t)batch * n_cap, d_c);
      if (st != ESA_OK) return st;
      st = make_tmap_f32(&tm_q, q_c, (uint64_t)batch * lq, d_c);
      if (st != ESA_OK) return st;
      esa::ScoreTcArgs a{lq, d_c, n_cap, r.mid0, r.n_mid, w.m_key, w.s, p.clamp_c};
      const int smem = 1024 + 3 * esa::kStRows * d_c * 4 + 256 + lq * 4;
      static const char what = 0;
      st = once_per_context(&what, [] {
        const int max_smem = 1024 + 3 * esa::kStRows * 128 * 4 + 256 + 4096 * 4;
        esa_status_t sa = set_max_smem(esa::score_tc_kernel<1>, max_smem);
        if (sa == ESA_OK) sa = set_max_smem(esa::score_tc_kernel<2>, max_smem);
        return sa;
      });
      if (st != ESA_OK) return st;
      const dim3 grid((unsigned)cdiv(r.n_mid, esa::kStRows), batch);
      esa::score_tc_kernel<1><<<grid, esa::kStThreads, smem, s>>>(tm_k, tm_q, a);
      ESA_LAUNCH_CHECK("score_tc_kernel<1>");
      esa::score_tc_kernel<2><<<grid, esa::kStThreads, smem, s>>>(tm_k, tm_q, a);
      ESA_LAUNCH_CHECK("score_tc_kernel<2>");
    }
    if (kk > 0) {
      esa::SelectArgs sa{};
      sa.S = path == ScorePath::TensorCore ? nullptr : w.S;
      sa.m_key = w.m_key;
      sa.s = w.s;
      sa.lq = lq;
      sa.clamp_c = p.clamp_c;
      sa.n_mid = r.n_mid;
      sa.mid0 = r.mid0;
      sa.eps = p.eps;
      sa.kk = (int)kk;
      sa.topk = p.topk;
      sa.vl = vl_sel;
      sa.u = w.u;
      sa.s_prime_out = score_out;
      sa.idx = idx_out;
      sa.count = count_out;
      static const char what = 0;
      st = once_per_context(&what, [] {
        esa_status_t sa = set_max_smem(esa::select_cluster_kernel<8>, esa::kSelSmemBytes);
        if (sa == ESA_OK) sa = set_max_smem(esa::select_cluster_kernel<16>, esa::kSelSmemBytes);
        return sa;
      });
      if (st != ESA_OK) return st;
      const int cl = select_cluster_size((int32_t)vb, r.n_mid);
      cudaLaunchConfig_t cfg = {};
      cfg.gridDim = dim3((unsigned)cl, (unsigned)vb, 1);
      cfg.blockDim = dim3(esa::kSelThreads);
      cfg.dynamicSmemBytes = esa::kSelSmemBytes;
      cfg.stream = s;
      cudaLaunchAttribute at[1];
      at[0].id = cudaLaunchAttributeClusterDimension;
      at[0].val.clusterDim.x = (unsigned)cl;
      at[0].val.clusterDim.y = 1;
      at[0].val.clusterDim.z = 1;
      cfg.attrs = at;
      cfg.numAttrs = 1;
      if (cl == 16) cudaLaunchKernelEx(&cfg, esa::select_cluster_kernel<16>, sa);
      else cudaLaunchKernelEx(&cfg, esa::select_cluster_kernel<8>, sa);
      ESA_LAUNCH_CHECK("select_cluster_kernel");
      return ok();
    }
  }
  const bool all_mid = r.n_mid <= p.topk;
  esa::fill_selection_kernel<<<dim3((unsigned)std::max<int64_t>(1, cdiv(p.topk, 256)), (unsigned)vb), 256, 0, s>>>(
      idx_out, count_out, p.topk, (int)kk, r.mid0, all_mid ? 1 : 0);
  ESA_LAUNCH_CHECK("fill_selection_kernel");
  return ok();
}

}  // namespace

// ------------------------------------------------------------------ sparse_attn --
namespace {

struct AttnPlan {
  bool tc;
  bool dec;          // bulk-copy decode kernel (bf16, head_dim 128, one query)
  int nsplit;
  int64_t keys_per_split;
  size_t ws_bytes;
};

AttnPlan plan_attn(int32_t batch, int32_t lq, int64_t c0, int32_t hq, int32_t hkv, int32_t head_dim, esa_dtype_t dt,
                   const esa_params_t& p) {
  AttnPlan pl{};
  const Regions r = regions(c0, p);
  const int g = hq / hkv;
  pl.tc = dt == ESA_BF16 && head_dim == 128 && (int64_t)lq * g >= 64;
  if (pl.tc) {
    // staged copies of the selected K and V rows: [B, topk, Hkv, D] bf16 each
    pl.ws_bytes = 2 * up256((size_t)batch * p.topk * hkv * head_dim * 2);
    return pl;
  }
  const int64_t n_keys_max = r.ni + std::min<int64_t>(p.topk, r.n_mid) + (c0 - r.lo) + lq;
  pl.dec = dt == ESA_BF16 && head_dim == 128 && lq == 1 && (hkv == 1 || hkv == 2 || hkv == 4 || hkv == 8) &&
           (g == 1 || g == 2 || g == 4);
  if (pl.dec) {
    // one CTA per SM: split each sequence's key list so that batch x nsplit fills the
    // 148 SMs once, with at least 4 stages per split
    const int64_t ks = esa::kDecStageRowsBytes / (hkv * head_dim * 2);
    const int64_t by_sm = std::max<int64_t>(1, 148 / batch);
    int64_t nsp = std::max<int64_t>(1, std::min(by_sm, cdiv(n_keys_max, 4 * ks)));
    nsp = std::max(nsp, cdiv(n_keys_max, esa::kDecMaxSplitKeys));   // positions fit in shared memory
    pl.keys_per_split = cdiv(cdiv(n_keys_max, nsp), ks) * ks;
    pl.nsplit = (int)cdiv(n_keys_max, pl.keys_per_split);
    // the last CTA of a sequence merges its splits in the freed stage ring: 3 floats per
    // (head, split) must fit in it
    if ((int64_t)hq * pl.nsplit * 3 * 4 > 2 * esa::kDecStages * esa::dec_operand_bytes(8)) pl.dec = false;
  }
  if (pl.dec) {
    // [B] arrival counters, then the split partials
    pl.ws_bytes = pl.nsplit > 1 ? up256((size_t)batch * sizeof(int)) +
                                      up256((size_t)batch * hq * pl.nsplit * esa::kDecPartStride * sizeof(float))
                                : 0;
    return pl;
  }
  const int64_t base = (int64_t)batch * lq * hkv;
  const int64_t want_ctas = 4 * 148;
  int64_t per = std::max<int64_t>(256, cdiv(n_keys_max, std::max<int64_t>(1, want_ctas / base)));
  per = cdiv(per, 64) * 64;
  pl.keys_per_split = per;
  pl.nsplit = (int)cdiv(n_keys_max, per);
  pl.ws_bytes = pl.nsplit > 1 ? up256((size_t)batch * lq * hq * pl.nsplit * (head_dim + 2) * sizeof(float)) : 0;
  return pl;
}

template <typename T, int D, int G>
void launch_simt(const esa::SimtAttnArgs& a, int batch, cudaStream_t s) {
  dim3 grid(a.nsplit, a.hkv, batch * a.lq);
  esa::attn_simt_kernel<T, D, G><<<grid, esa::kSimtWarps * 32, 0, s>>>(a);
}

template <typename T, int D>
bool dispatch_simt_g(const esa::SimtAttnArgs& a, int g, int batch, cudaStream_t s) {
  switch (g) {
    case 1: launch_simt<T, D, 1>(a, batch, s); return true;
    case 2: launch_simt<T, D, 2>(a, batch, s); return true;
    case 4: launch_simt<T, D, 4>(a, batch, s); return true;
    case 8: launch_simt<T, D, 8>(a, batch, s); return true;
    default: return false;
  }
}

}  // namespace

namespace {

// With one key list per KV head (lists > 1), a one-query bf16 call runs the bulk-copy
// decode kernel over batch x Hkv virtual sequences of one KV head each.
bool heads_as_sequences(int lists, esa_dtype_t dt, int32_t lq, int32_t hq, int32_t hkv, int32_t head_dim) {
  const int g = hq / hkv;
  return lists > 1 && dt == ESA_BF16 && head_dim == 128 && lq == 1 && (g == 1 || g == 2 || g == 4);
}

size_t sparse_attn_ws(int32_t batch, int32_t lq, int64_t c0, int32_t hq, int32_t hkv, int32_t head_dim,
                      esa_dtype_t dt, const esa_params_t& p, int lists) {
  if (batch <= 0 || lq <= 0 || hkv <= 0 || hq <= 0 || hq % hkv) return 0;
  if (heads_as_sequences(lists, dt, lq, hq, hkv, head_dim))
    return plan_attn(batch * hkv, lq, c0, hq / hkv, 1, head_dim, dt, p).ws_bytes;
  return plan_attn(batch, lq, c0, hq, hkv, head_dim, dt, p).ws_bytes;
}

esa_status_t sparse_attn_impl(const void* q, const void* k, const void* v, esa_dtype_t dt, int32_t batch,
                              int32_t lq, int64_t n_cap, int64_t c0, int32_t hq, int32_t hkv, int32_t head_dim,
                              const int32_t* idx, const int32_t* count, esa_params_t p, float scale, void* o,
                              float* lse, void* workspace, size_t ws_bytes, void* stream, int lists,
                              const int64_t* seq_len = nullptr);

}  // namespace

size_t esa_sparse_attn_workspace_size(int32_t batch, int32_t lq, int64_t c0, int32_t hq, int32_t hkv,
                                      int32_t head_dim, esa_dtype_t dt, esa_params_t p) {
  return sparse_attn_ws(batch, lq, c0, hq, hkv, head_dim, dt, p, 1);
}

size_t esa_sparse_attn_heads_workspace_size(int32_t batch, int32_t lq, int64_t c0, int32_t hq, int32_t hkv,
                                            int32_t head_dim, esa_dtype_t dt, esa_params_t p) {
  return sparse_attn_ws(batch, lq, c0, hq, hkv, head_dim, dt, p, hkv);
}

esa_status_t esa_sparse_attn(const void* q, const void* k, const void* v, esa_dtype_t dt, int32_t batch, int32_t lq,
                             int64_t n_cap, int64_t c0, int32_t hq, int32_t hkv, int32_t head_dim,
                             const int32_t* idx, const int32_t* count, esa_params_t p, float scale, void* o,
                             float* lse, void* workspace, size_t ws_bytes, void* stream) {
  return sparse_attn_impl(q, k, v, dt, batch, lq, n_cap, c0, hq, hkv, head_dim, idx, count, p, scale, o, lse,
                          workspace, ws_bytes, stream, 1);
}

esa_status_t esa_sparse_attn_heads(const void* q, const void* k, const void* v, esa_dtype_t dt, int32_t batch,
                                   int32_t lq, int64_t n_cap, int64_t c0, int32_t hq, int32_t hkv, int32_t head_dim,
                                   const int32_t* idx, const int32_t* count, esa_params_t p, float scale, void* o,
                                   float* lse, void* workspace, size_t ws_bytes, void* stream) {
  if (hkv <= 0) return fail(ESA_ERR_INVALID_ARG, "hkv must be >= 1");
  return sparse_attn_impl(q, k, v, dt, batch, lq, n_cap, c0, hq, hkv, head_dim, idx, count, p, scale, o, lse,
                          workspace, ws_bytes, stream, hkv);
}

size_t esa_sparse_attn_varlen_workspace_size(int32_t batch, int64_t n_cap, int32_t hq, int32_t hkv, int32_t head_dim,
                                             esa_dtype_t dt, int32_t lists, esa_params_t p) {
  if (n_cap < 1) return 0;
  return sparse_attn_ws(batch, 1, n_cap - 1, hq, hkv, head_dim, dt, p, lists);
}

esa_status_t esa_sparse_attn_varlen(const void* q, const void* k, const void* v, esa_dtype_t dt, int32_t batch,
                                    int64_t n_cap, const int64_t* seq_len, int32_t hq, int32_t hkv,
                                    int32_t head_dim, const int32_t* idx, const int32_t* count, int32_t lists,
                                    esa_params_t p, float scale, void* o, float* lse, void* workspace,
                                    size_t ws_bytes, void* stream) {
  if (hkv <= 0) return fail(ESA_ERR_INVALID_ARG, "hkv must be >= 1");
  if (lists != 1 && lists != hkv) return fail(ESA_ERR_INVALID_ARG, "lists must be 1 or hkv (got %d)", lists);
  if (!seq_len) return fail(ESA_ERR_INVALID_ARG, "null pointer");
  if (n_cap < 1) return fail(ESA_ERR_INVALID_ARG, "n_cap must be >= 1");
  return sparse_attn_impl(q, k, v, dt, batch, 1, n_cap, n_cap - 1, hq, hkv, head_dim, idx, count, p, scale, o, lse,
                          workspace, ws_bytes, stream, lists, seq_len);
}

namespace {


esa_status_t sparse_attn_impl(const void* q, const void* k, const void* v, esa_dtype_t dt, int32_t batch,
                              int32_t lq, int64_t n_cap, int64_t c0, int32_t hq, int32_t hkv, int32_t head_dim,
                              const int32_t* idx, const int32_t* count, esa_params_t p, float scale, void* o,
                              float* lse, void* workspace, size_t ws_bytes, void* stream, int lists,
                              const int64_t* seq_len) {
  esa_status_t st = check_params(p);
  if (st != ESA_OK) return st;
  if (dt != ESA_F32 && dt != ESA_BF16) return fail(ESA_ERR_INVALID_ARG, "bad dtype %d", (int)dt);
  if (batch <= 0 || lq <= 0) return fail(ESA_ERR_INVALID_ARG, "batch and lq must be >= 1");
  if (hq <= 0 || hkv <= 0 || hq % hkv) return fail(ESA_ERR_INVALID_ARG, "hq must be a positive multiple of hkv");
  if (head_dim != 64 && head_dim != 128) return fail(ESA_ERR_UNSUPPORTED, "head_dim %d (64 or 128)", head_dim);
  const int g = hq / hkv;
  if (g != 1 && g != 2 && g != 4 && g != 8) return fail(ESA_ERR_UNSUPPORTED, "GQA group %d (1, 2, 4 or 8)", g);
  if (c0 < 0 || c0 + lq > n_cap) return fail(ESA_ERR_INVALID_ARG, "need 0 <= c0 and c0 + lq <= n_cap");
  if (n_cap >= ((int64_t)1 << 31)) return fail(ESA_ERR_UNSUPPORTED, "n_cap must be < 2^31");
  if (!q || !k || !v || !o || !idx || !count) return fail(ESA_ERR_INVALID_ARG, "null pointer");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16))
    return fail(ESA_ERR_INVALID_ARG, "q, k, v, o need 16-byte alignment");
  const Regions r = regions(c0, p);
  const bool vseq = heads_as_sequences(lists, dt, lq, hq, hkv, head_dim);
  const AttnPlan pl = vseq ? plan_attn(batch * hkv, lq, c0, hq / hkv, 1, head_dim, dt, p)
                           : plan_attn(batch, lq, c0, hq, hkv, head_dim, dt, p);
  if (pl.ws_bytes && (!workspace || ws_bytes < pl.ws_bytes || !aligned(workspace, 256)))
    return fail(ESA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned (got %zu)", pl.ws_bytes, ws_bytes);
  if (scale <= 0.f) scale = 1.f / std::sqrt((float)head_dim);
  const float sl2 = scale * 1.4426950408889634f;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  esa::KeyList keys{idx, p.topk, r.ni, r.lo, n_cap, count};
  if (seq_len) {
    // a variable-length decode batch (c0 = n_cap - 1 here: the plan covers the longest key list)
    if (lq != 1 || pl.tc) return fail(ESA_ERR_UNSUPPORTED, "variable lengths need one query per sequence");
    keys.vl = esa::VarLen{seq_len, n_cap, p.n_init, p.window, vseq ? hkv : 1};
  }
  if (pl.tc) {
    static const char what = 0;
    st = once_per_context(&what, [] { return set_max_smem(esa::attn_tc_kernel<esa::EsaTcProblem>, esa::kTcSmemBytes); });
    if (st != ESA_OK) return st;
    esa::EsaTcProblem pr{};
    pr.q = static_cast<const __nv_bfloat16*>(q);
    pr.k = static_cast<const __nv_bfloat16*>(k);
    pr.v = static_cast<const __nv_bfloat16*>(v);
    pr.o = static_cast<__nv_bfloat16*>(o);
    pr.lse = lse;
    pr.keys = keys;
    pr.n_cap = n_cap;
    pr.c0 = c0;
    pr.lq = lq;
    pr.hq = hq;
    pr.hkv = hkv;
    pr.G = g;
    pr.sl2 = sl2;
    pr.lists = lists;
    if ((int64_t)batch * n_cap * hkv >= ((int64_t)1 << 31) || (int64_t)batch * lq * hq >= ((int64_t)1 << 31))
      return fail(ESA_ERR_UNSUPPORTED, "more than 2^31 K/V or Q rows");
    const size_t staged_bytes = up256((size_t)batch * p.topk * hkv * head_dim * 2);
    uint8_t* ks = static_cast<uint8_t*>(workspace);
    uint8_t* vs = ks + staged_bytes;
    const int row_vec = hkv * head_dim * 2 / 16;
    const int64_t max_sel = std::min<int64_t>(p.topk, r.n_mid);
    pr.staged = max_sel > 0 ? 1 : 0;
    if (max_sel > 0) {
      const dim3 ggrid((unsigned)std::min<int64_t>(max_sel, 4096), (unsigned)(batch * lists));
      esa::gather_selected_kernel<<<ggrid, 128, 0, s>>>(
          static_cast<const uint4*>(k), static_cast<const uint4*>(v), idx, count, n_cap, p.topk, row_vec, lists,
          head_dim * 2 / 16, reinterpret_cast<uint4*>(ks), reinterpret_cast<uint4*>(vs));
      ESA_LAUNCH_CHECK("gather_selected_kernel");
    }
    CUtensorMap tq, tk, tv, bq, bk, bv, sk, sv;
    if ((st = make_tmap_box_bf16(&sk, ks, hkv, (uint64_t)batch * p.topk, 1, esa::kTcKeys)) != ESA_OK) return st;
    if ((st = make_tmap_box_bf16(&sv, vs, hkv, (uint64_t)batch * p.topk, 1, esa::kTcKeys)) != ESA_OK) return st;
    if ((st = make_tmap_rows_bf16(&tq, q, (uint64_t)batch * lq * hq)) != ESA_OK) return st;
    if ((st = make_tmap_rows_bf16(&tk, k, (uint64_t)batch * n_cap * hkv)) != ESA_OK) return st;
    if ((st = make_tmap_rows_bf16(&tv, v, (uint64_t)batch * n_cap * hkv)) != ESA_OK) return st;
    if ((st = make_tmap_box_bf16(&bq, q, hq, (uint64_t)batch * lq, g, esa::kTcRows / g)) != ESA_OK) return st;
    if ((st = make_tmap_box_bf16(&bk, k, hkv, (uint64_t)batch * n_cap, 1, esa::kTcKeys)) != ESA_OK) return st;
    if ((st = make_tmap_box_bf16(&bv, v, hkv, (uint64_t)batch * n_cap, 1, esa::kTcKeys)) != ESA_OK) return st;
    dim3 grid((unsigned)cdiv((int64_t)lq * g, esa::kTcRows), hkv, batch);
    esa::attn_tc_kernel<esa::EsaTcProblem><<<grid, esa::kTcThreads, esa::kTcSmemBytes, s>>>(tq, tk, tv, bq, bk, bv,
                                                                                           sk, sv, pr);
    ESA_LAUNCH_CHECK("attn_tc_kernel<esa>");
    return ok();
  }
  if (pl.dec) {
    static const char what_dec = 0;
    st = once_per_context(&what_dec, [] {
      esa_status_t sa = set_max_smem(esa::attn_decode_kernel<1>, esa::kDecSmemBytes);
      if (sa == ESA_OK) sa = set_max_smem(esa::attn_decode_kernel<2>, esa::kDecSmemBytes);
      if (sa == ESA_OK) sa = set_max_smem(esa::attn_decode_kernel<4>, esa::kDecSmemBytes);
      return sa;
    });
    if (st != ESA_OK) return st;
    esa::DecodeAttnArgs d{};
    d.q = static_cast<const __nv_bfloat16*>(q);
    d.k = static_cast<const __nv_bfloat16*>(k);
    d.v = static_cast<const __nv_bfloat16*>(v);
    d.o = static_cast<__nv_bfloat16*>(o);
    d.lse = lse;
    if (pl.nsplit > 1) {
      const size_t nseq = (size_t)(vseq ? batch * hkv : batch);
      d.arrive = static_cast<int*>(workspace);
      d.part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + up256(nseq * sizeof(int)));
      ESA_CUDA(cudaMemsetAsync(d.arrive, 0, nseq * sizeof(int), s));
    }
    d.keys = keys;
    d.n_cap = n_cap;
    d.c0 = c0;
    d.hq = vseq ? hq / hkv : hq;
    d.hkv = vseq ? 1 : hkv;
    d.vheads = vseq ? hkv : 1;
    d.tok_stride = (int64_t)hkv * head_dim;
    d.nsplit = pl.nsplit;
    d.keys_per_split = (int)pl.keys_per_split;
    d.scale_log2 = sl2;
    const dim3 grid((unsigned)pl.nsplit, (unsigned)(vseq ? batch * hkv : batch));
    if (d.hkv == 1) {
      // one KV head per sequence: per-warp row streams instead of per-row bulk copies
      static const char what_rows = 0;
      st = once_per_context(&what_rows, [] {
        esa_status_t sa = set_max_smem(esa::attn_decode_rows_kernel<1>, esa::kRowSmemBytes);
        if (sa == ESA_OK) sa = set_max_smem(esa::attn_decode_rows_kernel<2>, esa::kRowSmemBytes);
        if (sa == ESA_OK) sa = set_max_smem(esa::attn_decode_rows_kernel<4>, esa::kRowSmemBytes);
        return sa;
      });
      if (st != ESA_OK) return st;
      if (g == 1) esa::attn_decode_rows_kernel<1><<<grid, esa::kDecThreads, esa::kRowSmemBytes, s>>>(d);
      else if (g == 2) esa::attn_decode_rows_kernel<2><<<grid, esa::kDecThreads, esa::kRowSmemBytes, s>>>(d);
      else esa::attn_decode_rows_kernel<4><<<grid, esa::kDecThreads, esa::kRowSmemBytes, s>>>(d);
      ESA_LAUNCH_CHECK("attn_decode_rows_kernel");
      return ok();
    }
    if (g == 1) esa::attn_decode_kernel<1><<<grid, esa::kDecThreads, esa::kDecSmemBytes, s>>>(d);
    else if (g == 2) esa::attn_decode_kernel<2><<<grid, esa::kDecThreads, esa::kDecSmemBytes, s>>>(d);
    else esa::attn_decode_kernel<4><<<grid, esa::kDecThreads, esa::kDecSmemBytes, s>>>(d);
    ESA_LAUNCH_CHECK("attn_decode_kernel");
    return ok();
  }
  esa::SimtAttnArgs a{};
  a.q = q;
  a.k = k;
  a.v = v;
  a.o = o;
  a.lse = lse;
  a.part = static_cast<float*>(workspace);
  a.keys = keys;
  a.n_cap = n_cap;
  a.c0 = c0;
  a.lq = lq;
  a.hq = hq;
  a.hkv = hkv;
  a.nsplit = pl.nsplit;
  a.lists = lists;
  a.keys_per_split = pl.keys_per_split;
  a.scale_log2 = sl2;
  bool launched;
  if (dt == ESA_BF16)
    launched = head_dim == 128 ? dispatch_simt_g<__nv_bfloat16, 128>(a, g, batch, s)
                               : dispatch_simt_g<__nv_bfloat16, 64>(a, g, batch, s);
  else
    launched = head_dim == 128 ? dispatch_simt_g<float, 128>(a, g, batch, s) : dispatch_simt_g<float, 64>(a, g, batch, s);
  if (!launched) return fail(ESA_ERR_UNSUPPORTED, "GQA group %d", g);
  ESA_LAUNCH_CHECK("attn_simt_kernel");
  if (pl.nsplit > 1) {
    const int64_t rows = (int64_t)batch * lq * hq;
    const dim3 cgrid((unsigned)cdiv(rows, 8));
    if (dt == ESA_BF16) {
      if (head_dim == 128)
        esa::attn_combine_kernel<__nv_bfloat16, 128><<<cgrid, 256, 0, s>>>(a.part, rows, pl.nsplit,
                                                                          static_cast<__nv_bfloat16*>(o), lse);
      else
        esa::attn_combine_kernel<__nv_bfloat16, 64><<<cgrid, 256, 0, s>>>(a.part, rows, pl.nsplit,
                                                                         static_cast<__nv_bfloat16*>(o), lse);
    } else {
      if (head_dim == 128)
        esa::attn_combine_kernel<float, 128><<<cgrid, 256, 0, s>>>(a.part, rows, pl.nsplit, static_cast<float*>(o),
                                                                  lse);
      else
        esa::attn_combine_kernel<float, 64><<<cgrid, 256, 0, s>>>(a.part, rows, pl.nsplit, static_cast<float*>(o),
                                                                 lse);
    }
    ESA_LAUNCH_CHECK("attn_combine_kernel");
  }
  return ok();
}

}  // namespace

// ------------------------------------------------------------------ MoBA --
namespace {

struct MobaWs {
  float* kbar;
  int16_t* blocks;
  uint32_t* cnt;    // cnt, fill contiguous (cleared together)
  uint32_t* fill;
  uint32_t* off;
  uint32_t* tile_off;
  uint32_t* totals;
  uint32_t* unit_list;     // [max_tiles]: the list of each 256-row unit (n_lists past the last)
  uint32_t* list;
  __nv_bfloat16* part_o;   // past partials: [B, seq, H, topk, D] bf16, lse [B, seq, H, topk]
  float* part_lse;
  size_t zero_bytes;
  size_t bytes;
  int64_t n_lists, pairs, max_tiles;
};

int64_t moba_pairs(int64_t seq, int block, int topk) {
  const int64_t nb = cdiv(seq, block);
  int64_t pairs = 0;
  for (int64_t c = 0; c < nb; ++c) pairs += std::min<int64_t>(block, seq - c * block) * std::min<int64_t>(topk, c);
  return pairs;
}

// which: 0 gate only, 1 attention only, 2 both (blocks live in the workspace)
MobaWs carve_moba(void* ws, int which, int32_t batch, int64_t seq, int32_t heads, int32_t d, int32_t block,
                  int32_t topk) {
  Carver c{reinterpret_cast<uint8_t*>(ws)};
  MobaWs w{};
  const int64_t nb = cdiv(seq, block);
  w.n_lists = (int64_t)batch * heads * nb;
  w.pairs = moba_pairs(seq, block, topk) * batch * heads;
  w.max_tiles = cdiv(w.pairs, 2 * esa::kTcRows) + w.n_lists;   // units of a pair of 128-row tiles
  if (which == 0 || which == 2) w.kbar = c.take<float>((size_t)batch * heads * nb * d);
  if (which == 2) w.blocks = c.take<int16_t>((size_t)batch * seq * heads * (topk + 1));
  if (which >= 1) {
    const size_t z0 = c.off;
    w.cnt = c.take<uint32_t>(w.n_lists);
    w.fill = c.take<uint32_t>(w.n_lists);
    w.zero_bytes = c.off - z0;
    w.off = c.take<uint32_t>(w.n_lists);
    w.tile_off = c.take<uint32_t>(w.n_lists + 1);
    w.totals = c.take<uint32_t>(2);
    w.unit_list = c.take<uint32_t>(w.max_tiles);
    w.list = c.take<uint32_t>(std::max<int64_t>(1, w.pairs));
    w.part_o = c.take<__nv_bfloat16>((size_t)batch * seq * heads * topk * d);
    w.part_lse = c.take<float>((size_t)batch * seq * heads * topk);
  }
  w.bytes = c.off;
  return w;
}

esa_status_t moba_check(const void* q, const void* k, esa_dtype_t dt, int32_t batch, int64_t seq, int32_t heads,
                        int32_t head_dim, int32_t block, int32_t topk) {
  if (dt != ESA_BF16) return fail(ESA_ERR_UNSUPPORTED, "MoBA kernels take bf16 tensors");
  if (batch <= 0 || seq <= 0 || heads <= 0) return fail(ESA_ERR_INVALID_ARG, "batch, seq, heads must be >= 1");
  if (head_dim != 128) return fail(ESA_ERR_UNSUPPORTED, "MoBA head_dim %d (128)", head_dim);
  if (block < 16 || block % 16) return fail(ESA_ERR_INVALID_ARG, "block must be a multiple of 16, >= 16");
  if (topk < 0 || topk > esa::kMobaMaxTopk) return fail(ESA_ERR_INVALID_ARG, "topk must be in [0, 15]");
  if (cdiv(seq, block) > 1024) return fail(ESA_ERR_UNSUPPORTED, "more than 1024 blocks");
  if (seq >= ((int64_t)1 << 27)) return fail(ESA_ERR_UNSUPPORTED, "seq must be < 2^27");
  if (!q || !k) return fail(ESA_ERR_INVALID_ARG, "null pointer");
  if (!aligned(q, 16) || !aligned(k, 16)) return fail(ESA_ERR_INVALID_ARG, "16-byte alignment required");
  return ESA_OK;
}

esa_status_t moba_gate_launch(const MobaWs& w, const void* q, const void* k, int32_t batch, int64_t seq, int32_t heads,
                              int32_t block, int32_t topk, int16_t* blocks_out, cudaStream_t s) {
  const int nb = (int)cdiv(seq, block);
  esa::moba_mean_kernel<__nv_bfloat16><<<dim3(nb, heads, batch), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(k), seq, heads, 128, block, 0, nb, w.kbar);
  ESA_LAUNCH_CHECK("moba_mean_kernel");
  const dim3 ggrid((unsigned)cdiv(seq, 128), heads, batch);
  const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);
  if (topk <= 1)
    esa::moba_gate_kernel<__nv_bfloat16, 128, 1><<<ggrid, 128, 0, s>>>(qb, w.kbar, seq, heads, block, nb, topk, blocks_out);
  else if (topk <= 2)
    esa::moba_gate_kernel<__nv_bfloat16, 128, 2><<<ggrid, 128, 0, s>>>(qb, w.kbar, seq, heads, block, nb, topk, blocks_out);
  else if (topk <= 3)
    esa::moba_gate_kernel<__nv_bfloat16, 128, 3><<<ggrid, 128, 0, s>>>(qb, w.kbar, seq, heads, block, nb, topk, blocks_out);
  else if (topk <= 4)
    esa::moba_gate_kernel<__nv_bfloat16, 128, 4><<<ggrid, 128, 0, s>>>(qb, w.kbar, seq, heads, block, nb, topk, blocks_out);
  else if (topk <= 8)
    esa::moba_gate_kernel<__nv_bfloat16, 128, 8><<<ggrid, 128, 0, s>>>(qb, w.kbar, seq, heads, block, nb, topk, blocks_out);
  else
    esa::moba_gate_kernel<__nv_bfloat16, 128, esa::kMobaMaxTopk><<<ggrid, 128, 0, s>>>(qb, w.kbar, seq, heads, block,
                                                                                         nb, topk, blocks_out);
  ESA_LAUNCH_CHECK("moba_gate_kernel");
  return ESA_OK;
}

esa_status_t moba_attn_launch(const MobaWs& w, const void* q, const void* k, const void* v, int32_t batch,
                              int64_t seq, int32_t heads, int32_t block, int32_t topk, const int16_t* blocks,
                              float scale, void* o, float* lse, cudaStream_t s) {
  const int nb = (int)cdiv(seq, block);
  if (scale <= 0.f) scale = 1.f / std::sqrt(128.f);
  const float sl2 = scale * 1.4426950408889634f;
  static const char what = 0;
  const esa_status_t sa = once_per_context(&what, [] {
    esa_status_t st = set_max_smem(esa::attn_pp_kernel<esa::MobaPastProblem>, esa::kPpSmemBytes);
    if (st == ESA_OK) st = set_max_smem(esa::attn_pp_kernel<esa::MobaCurrentProblem>, esa::kPpSmemBytes);
    return st;
  });
  if (sa != ESA_OK) return sa;
  CUtensorMap tq, tk, tv, bq, bk, bv;
  esa_status_t st;
  if ((st = make_tmap_rows_bf16(&tq, q, (uint64_t)batch * seq * heads)) != ESA_OK) return st;
  if ((st = make_tmap_rows_bf16(&tk, k, (uint64_t)batch * seq * heads)) != ESA_OK) return st;
  if ((st = make_tmap_rows_bf16(&tv, v, (uint64_t)batch * seq * heads)) != ESA_OK) return st;
  if ((st = make_tmap_box_bf16(&bq, q, heads, (uint64_t)batch * seq, 1, esa::kTcRows)) != ESA_OK) return st;
  if ((st = make_tmap_box_bf16(&bk, k, heads, (uint64_t)batch * seq, 1, esa::kTcKeys)) != ESA_OK) return st;
  if ((st = make_tmap_box_bf16(&bv, v, heads, (uint64_t)batch * seq, 1, esa::kTcKeys)) != ESA_OK) return st;
  ESA_CUDA(cudaMemsetAsync(w.cnt, 0, w.zero_bytes, s));
  const dim3 lgrid((unsigned)nb, heads, batch);
  const size_t lsmem = 2 * (size_t)nb * sizeof(uint32_t);
  if (topk > 0 && w.pairs > 0) {
    esa::moba_list_kernel<<<lgrid, esa::kMobaListThreads, lsmem, s>>>(blocks, seq, heads, block, nb, topk, 0, w.cnt,
                                                                      w.off, w.fill, w.list);
    ESA_LAUNCH_CHECK("moba_list_kernel(count)");
    esa::moba_scan_kernel<<<1, 1024, 0, s>>>(w.cnt, w.n_lists, w.off, w.tile_off, w.totals, 2 * esa::kTcRows,
                                             w.unit_list, w.max_tiles);
    ESA_LAUNCH_CHECK("moba_scan_kernel");
    esa::moba_list_kernel<<<lgrid, esa::kMobaListThreads, lsmem, s>>>(blocks, seq, heads, block, nb, topk, 1, w.cnt,
                                                                      w.off, w.fill, w.list);
    ESA_LAUNCH_CHECK("moba_list_kernel(fill)");
    esa::MobaPastProblem pp{};
    pp.q = static_cast<const __nv_bfloat16*>(q);
    pp.k = static_cast<const __nv_bfloat16*>(k);
    pp.v = static_cast<const __nv_bfloat16*>(v);
    pp.part_o = w.part_o;
    pp.part_lse = w.part_lse;
    pp.tile_off = w.tile_off;
    pp.unit_list = w.unit_list;
    pp.off = w.off;
    pp.cnt = w.cnt;
    pp.list = w.list;
    pp.seq = seq;
    pp.heads = heads;
    pp.n_blocks = nb;
    pp.block = block;
    pp.topk = topk;
    pp.n_lists = w.n_lists;
    pp.sl2 = sl2;
    esa::attn_pp_kernel<esa::MobaPastProblem><<<(unsigned)w.max_tiles, esa::kPpThreads, esa::kPpSmemBytes, s>>>(
        tq, tk, tv, bq, bk, bv, bk, bv, pp);
    ESA_LAUNCH_CHECK("attn_pp_kernel<moba past>");
  }
  esa::MobaCurrentProblem cp{};
  cp.q = static_cast<const __nv_bfloat16*>(q);
  cp.k = static_cast<const __nv_bfloat16*>(k);
  cp.v = static_cast<const __nv_bfloat16*>(v);
  cp.part_o = w.part_o;
  cp.part_lse = w.part_lse;
  cp.o = static_cast<__nv_bfloat16*>(o);
  cp.lse = lse;
  cp.seq = seq;
  cp.heads = heads;
  cp.n_blocks = nb;
  cp.block = block;
  cp.topk = topk;
  cp.tiles_per_block = (int)cdiv(block, esa::kTcRows);
  cp.sl2 = sl2;
  esa::attn_pp_kernel<esa::MobaCurrentProblem>
      <<<dim3((unsigned)(cdiv(cp.tiles_per_block, 2) * nb), heads, batch), esa::kPpThreads, esa::kPpSmemBytes, s>>>(
          tq, tk, tv, bq, bk, bv, bk, bv, cp);
  ESA_LAUNCH_CHECK("attn_pp_kernel<moba current>");
  return ESA_OK;
}

}  // namespace

size_t moba_workspace_size(int32_t which, int32_t batch, int64_t seq, int32_t heads, int32_t head_dim, int32_t block,
                           int32_t topk) {
  if (which < 0 || which > 2 || batch <= 0 || seq <= 0 || heads <= 0 || block <= 0 || topk < 0) return 0;
  return carve_moba(nullptr, which, batch, seq, heads, head_dim, block, topk).bytes;
}

esa_status_t moba_block_gate(const void* q, const void* k, esa_dtype_t dt, int32_t batch, int64_t seq, int32_t heads,
                             int32_t head_dim, int32_t block, int32_t topk, int16_t* blocks_out, void* workspace,
                             size_t ws_bytes, void* stream) {
  esa_status_t st = moba_check(q, k, dt, batch, seq, heads, head_dim, block, topk);
  if (st != ESA_OK) return st;
  if (!blocks_out) return fail(ESA_ERR_INVALID_ARG, "null blocks_out");
  const MobaWs need = carve_moba(nullptr, 0, batch, seq, heads, head_dim, block, topk);
  if (!workspace || ws_bytes < need.bytes || !aligned(workspace, 256))
    return fail(ESA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned (got %zu)", need.bytes, ws_bytes);
  const MobaWs w = carve_moba(workspace, 0, batch, seq, heads, head_dim, block, topk);
  st = moba_gate_launch(w, q, k, batch, seq, heads, block, topk, blocks_out, reinterpret_cast<cudaStream_t>(stream));
  return st == ESA_OK ? ok() : st;
}

esa_status_t moba_block_attn(const void* q, const void* k, const void* v, esa_dtype_t dt, int32_t batch, int64_t seq,
                             int32_t heads, int32_t head_dim, int32_t block, int32_t topk, const int16_t* blocks,
                             float scale, void* o, float* lse, void* workspace, size_t ws_bytes, void* stream) {
  esa_status_t st = moba_check(q, k, dt, batch, seq, heads, head_dim, block, topk);
  if (st != ESA_OK) return st;
  if (!v || !o || !blocks) return fail(ESA_ERR_INVALID_ARG, "null pointer");
  if (!aligned(v, 16) || !aligned(o, 16)) return fail(ESA_ERR_INVALID_ARG, "16-byte alignment required");
  const MobaWs need = carve_moba(nullptr, 1, batch, seq, heads, head_dim, block, topk);
  if (!workspace || ws_bytes < need.bytes || !aligned(workspace, 256))
    return fail(ESA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned (got %zu)", need.bytes, ws_bytes);
  const MobaWs w = carve_moba(workspace, 1, batch, seq, heads, head_dim, block, topk);
  st = moba_attn_launch(w, q, k, v, batch, seq, heads, block, topk, blocks, scale, o, lse,
                        reinterpret_cast<cudaStream_t>(stream));
  return st == ESA_OK ? ok() : st;
}

esa_status_t moba_block_gate_attn(const void* q, const void* k, const void* v, esa_dtype_t dt, int32_t batch,
                                  int64_t seq, int32_t heads, int32_t head_dim, int32_t block, int32_t topk,
                                  float scale, void* o, float* lse, int16_t* blocks_out, void* workspace,
                                  size_t ws_bytes, void* stream) {
  esa_status_t st = moba_check(q, k, dt, batch, seq, heads, head_dim, block, topk);
  if (st != ESA_OK) return st;
  if (!v || !o) return fail(ESA_ERR_INVALID_ARG, "null pointer");
  if (!aligned(v, 16) || !aligned(o, 16)) return fail(ESA_ERR_INVALID_ARG, "16-byte alignment required");
  const MobaWs need = carve_moba(nullptr, 2, batch, seq, heads, head_dim, block, topk);
  if (!workspace || ws_bytes < need.bytes || !aligned(workspace, 256))
    return fail(ESA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned (got %zu)", need.bytes, ws_bytes);
  const MobaWs w = carve_moba(workspace, 2, batch, seq, heads, head_dim, block, topk);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  int16_t* blocks = blocks_out ? blocks_out : w.blocks;
  st = moba_gate_launch(w, q, k, batch, seq, heads, block, topk, blocks, s);
  if (st != ESA_OK) return st;
  st = moba_attn_launch(w, q, k, v, batch, seq, heads, block, topk, blocks, scale, o, lse, s);
  return st == ESA_OK ? ok() : st;
}

// ------------------------------------------------------------------ CCA-style attention --
namespace {

struct CcaWs {
  __nv_bfloat16* kc;        // [B, m, Hq, D] core keys
  __nv_bfloat16* vc;        // [B, m, Hq, D] core values
  __nv_bfloat16* part_o;    // [B, S, Hq, D] core-pass partials
  float* part_lse;          // [B, S, Hq]
  size_t bytes;
};

CcaWs carve_cca(void* ws, int32_t batch, int64_t seq, int32_t hq, int32_t head_dim, int32_t group) {
  Carver c{reinterpret_cast<uint8_t*>(ws)};
  CcaWs w{};
  const int64_t m = seq / group;
  w.kc = c.take<__nv_bfloat16>((size_t)std::max<int64_t>(1, batch * m * hq) * head_dim);
  w.vc = c.take<__nv_bfloat16>((size_t)std::max<int64_t>(1, batch * m * hq) * head_dim);
  w.part_o = c.take<__nv_bfloat16>((size_t)batch * seq * hq * head_dim);
  w.part_lse = c.take<float>((size_t)batch * seq * hq);
  w.bytes = c.off;
  return w;
}

esa_status_t cca_check(const void* q, const void* k, const void* v, const void* o, esa_dtype_t dt, int32_t batch,
                       int64_t seq, int32_t hq, int32_t hkv, int32_t head_dim, int32_t group, int32_t window) {
  if (dt != ESA_BF16) return fail(ESA_ERR_UNSUPPORTED, "CCA attention takes bf16 tensors");
  if (batch <= 0 || seq <= 0) return fail(ESA_ERR_INVALID_ARG, "batch and seq must be >= 1");
  if (hq <= 0 || hkv <= 0 || hq % hkv) return fail(ESA_ERR_INVALID_ARG, "hq must be a positive multiple of hkv");
  const int g = hq / hkv;
  if (g != 1 && g != 2 && g != 4 && g != 8) return fail(ESA_ERR_UNSUPPORTED, "GQA group %d (1, 2, 4 or 8)", g);
  if (head_dim != 128) return fail(ESA_ERR_UNSUPPORTED, "head_dim %d (128)", head_dim);
  if (group < 128 || group % 128) return fail(ESA_ERR_UNSUPPORTED, "group %d (a multiple of 128)", group);
  if (window < 0 || window % group) return fail(ESA_ERR_INVALID_ARG, "window must be a multiple of the group (>= 0)");
  if ((int64_t)batch * seq * hq >= ((int64_t)1 << 31)) return fail(ESA_ERR_UNSUPPORTED, "more than 2^31 query rows");
  if (!q || !k || !v || !o) return fail(ESA_ERR_INVALID_ARG, "null pointer");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16))
    return fail(ESA_ERR_INVALID_ARG, "q, k, v, o need 16-byte alignment");
  return ESA_OK;
}

template <int G>
void launch_cca_pool(const void* q, const void* k, const void* v, int32_t batch, int64_t seq, int32_t hkv,
                     int32_t group, float sl2, const CcaWs& w, cudaStream_t s) {
  const int64_t m = seq / group;
  const int64_t items = (int64_t)batch * m * hkv;
  esa::cca_pool_kernel<G><<<(unsigned)cdiv(items, esa::kCcaPoolWarps), esa::kCcaPoolWarps * 32, 0, s>>>(
      static_cast<const __nv_bfloat16*>(q), static_cast<const __nv_bfloat16*>(k),
      static_cast<const __nv_bfloat16*>(v), batch, seq, hkv, group, m, sl2, w.kc, w.vc);
}

}  // namespace

size_t cca_workspace_size(int32_t batch, int64_t seq, int32_t hq, int32_t head_dim, int32_t group) {
  if (batch <= 0 || seq <= 0 || hq <= 0 || head_dim <= 0 || group <= 0) return 0;
  return carve_cca(nullptr, batch, seq, hq, head_dim, group).bytes;
}

esa_status_t cca_attn(const void* q, const void* k, const void* v, esa_dtype_t dt, int32_t batch, int64_t seq,
                      int32_t hq, int32_t hkv, int32_t head_dim, int32_t group, int32_t window, float scale, void* o,
                      float* lse, void* workspace, size_t ws_bytes, void* stream) {
  esa_status_t st = cca_check(q, k, v, o, dt, batch, seq, hq, hkv, head_dim, group, window);
  if (st != ESA_OK) return st;
  const size_t need = carve_cca(nullptr, batch, seq, hq, head_dim, group).bytes;
  if (!workspace || ws_bytes < need || !aligned(workspace, 256))
    return fail(ESA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned (got %zu)", need, ws_bytes);
  const CcaWs w = carve_cca(workspace, batch, seq, hq, head_dim, group);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (scale <= 0.f) scale = 1.f / std::sqrt((float)head_dim);
  const float sl2 = scale * 1.4426950408889634f;
  const int g = hq / hkv;
  const int64_t m = seq / group;
  if (m > 0) {
    if (g == 1) launch_cca_pool<1>(q, k, v, batch, seq, hkv, group, sl2, w, s);
    else if (g == 2) launch_cca_pool<2>(q, k, v, batch, seq, hkv, group, sl2, w, s);
    else if (g == 4) launch_cca_pool<4>(q, k, v, batch, seq, hkv, group, sl2, w, s);
    else launch_cca_pool<8>(q, k, v, batch, seq, hkv, group, sl2, w, s);
    ESA_LAUNCH_CHECK("cca_pool_kernel");
  }
  static const char what = 0;
  st = once_per_context(&what, [] {
    esa_status_t sa = set_max_smem(esa::attn_tc_kernel<esa::CcaCoreProblem>, esa::kTcSmemBytes);
    if (sa == ESA_OK) sa = set_max_smem(esa::attn_tc_kernel<esa::CcaWindowProblem>, esa::kTcSmemBytes);
    return sa;
  });
  if (st != ESA_OK) return st;
  CUtensorMap tq, tk, tv, bq, bk, bv, sk, sv;
  const uint64_t rows_q = (uint64_t)batch * seq * hq, rows_kv = (uint64_t)batch * seq * hkv;
  if ((st = make_tmap_rows_bf16(&tq, q, rows_q)) != ESA_OK) return st;
  if ((st = make_tmap_rows_bf16(&tk, k, rows_kv)) != ESA_OK) return st;
  if ((st = make_tmap_rows_bf16(&tv, v, rows_kv)) != ESA_OK) return st;
  if ((st = make_tmap_box_bf16(&bq, q, hq, (uint64_t)batch * seq, 1, esa::kTcRows)) != ESA_OK) return st;
  if ((st = make_tmap_box_bf16(&bk, k, hkv, (uint64_t)batch * seq, 1, esa::kTcKeys)) != ESA_OK) return st;
  if ((st = make_tmap_box_bf16(&bv, v, hkv, (uint64_t)batch * seq, 1, esa::kTcKeys)) != ESA_OK) return st;
  const uint64_t core_tokens = (uint64_t)std::max<int64_t>(1, (int64_t)batch * m);
  if ((st = make_tmap_box_bf16(&sk, w.kc, hq, core_tokens, 1, esa::kTcKeys)) != ESA_OK) return st;
  if ((st = make_tmap_box_bf16(&sv, w.vc, hq, core_tokens, 1, esa::kTcKeys)) != ESA_OK) return st;
  const dim3 grid((unsigned)cdiv(seq, esa::kTcRows), (unsigned)hq, (unsigned)batch);
  auto tile = [&](esa::CcaTile& t) {
    t.seq = seq;
    t.m = m;
    t.hq = hq;
    t.hkv = hkv;
    t.G = g;
    t.group = group;
    t.window = window;
    t.sl2 = sl2;
  };
  if (m > 0) {
    esa::CcaCoreProblem cp{};
    tile(cp);
    cp.part_o = w.part_o;
    cp.part_lse = w.part_lse;
    esa::attn_tc_kernel<esa::CcaCoreProblem><<<grid, esa::kTcThreads, esa::kTcSmemBytes, s>>>(tq, tk, tv, bq, bk, bv,
                                                                                           sk, sv, cp);
    ESA_LAUNCH_CHECK("attn_tc_kernel<cca core>");
  }
  esa::CcaWindowProblem wp{};
  tile(wp);
  wp.part_o = w.part_o;
  wp.part_lse = w.part_lse;
  wp.o = static_cast<__nv_bfloat16*>(o);
  wp.lse = lse;
  esa::attn_tc_kernel<esa::CcaWindowProblem><<<grid, esa::kTcThreads, esa::kTcSmemBytes, s>>>(tq, tk, tv, bq, bk, bv,
                                                                                           sk, sv, wp);
  ESA_LAUNCH_CHECK("attn_tc_kernel<cca window>");
  return ok();
}

// ------------------------------------------------------------------ MoBA decode --
esa_status_t moba_block_means(const void* k, esa_dtype_t dt, int32_t batch, int64_t n_cap, int32_t heads,
                              int32_t head_dim, int32_t block, int32_t blk_begin, int32_t blk_end, float* kbar,
                              void* stream) {
  esa_status_t st = moba_check(k, k, dt, batch, n_cap, heads, head_dim, block, 0);
  if (st != ESA_OK) return st;
  if (!kbar) return fail(ESA_ERR_INVALID_ARG, "null pointer");
  const int nb = (int)cdiv(n_cap, block);
  blk_begin = std::max(0, blk_begin);
  blk_end = std::min(nb, blk_end);
  if (blk_end <= blk_begin) return ok();
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  esa::moba_mean_kernel<__nv_bfloat16><<<dim3(blk_end - blk_begin, heads, batch), 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(k), n_cap, heads, 128, block, blk_begin, nb, kbar);
  ESA_LAUNCH_CHECK("moba_mean_kernel");
  return ok();
}

namespace {

// the attention half of a MoBA decode step, as esa_sparse_attn_heads sees it: no
// initial tokens, the kept blocks' positions as the selected middle, and the current
// block up to the query as the local part
esa_params_t moba_decode_params(int64_t pos, int32_t block, int32_t topk) {
  esa_params_t p{};
  p.n_init = 0;
  p.window = (int32_t)(pos - (pos / block) * block);
  p.topk = topk * block;
  p.eps = 0;
  p.clamp_c = INFINITY;
  return p;
}

}  // namespace

size_t moba_decode_workspace_size(int32_t batch, int64_t n_cap, int64_t pos, int32_t heads, int32_t head_dim,
                                  int32_t block, int32_t topk) {
  if (batch <= 0 || heads <= 0 || block <= 0 || topk <= 0) return 0;
  const int64_t lists = (int64_t)batch * heads;
  const esa_params_t p = moba_decode_params(pos, block, topk);
  (void)n_cap;
  return up256((size_t)lists * topk * block * sizeof(int32_t)) + up256((size_t)lists * sizeof(int32_t)) +
         sparse_attn_ws(batch, 1, pos, heads, heads, head_dim, ESA_BF16, p, heads);
}

esa_status_t moba_decode_attn(const void* q, const void* k, const void* v, esa_dtype_t dt, int32_t batch,
                              int64_t n_cap, int64_t pos, int32_t heads, int32_t head_dim, int32_t block,
                              int32_t topk, const float* kbar, float scale, void* o, float* lse,
                              int16_t* blocks_out, void* workspace, size_t ws_bytes, void* stream) {
  esa_status_t st = moba_check(q, k, dt, batch, n_cap, heads, head_dim, block, topk);
  if (st != ESA_OK) return st;
  if (topk < 1) return fail(ESA_ERR_INVALID_ARG, "topk must be >= 1");
  if (pos < 0 || pos >= n_cap) return fail(ESA_ERR_INVALID_ARG, "need 0 <= pos < n_cap");
  if (!v || !o || !kbar) return fail(ESA_ERR_INVALID_ARG, "null pointer");
  if (!aligned(v, 16) || !aligned(o, 16) || !aligned(kbar, 16))
    return fail(ESA_ERR_INVALID_ARG, "16-byte alignment required");
  const size_t need = moba_decode_workspace_size(batch, n_cap, pos, heads, head_dim, block, topk);
  if (!workspace || ws_bytes < need || !aligned(workspace, 256))
    return fail(ESA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned (got %zu)", need, ws_bytes);
  const int64_t lists = (int64_t)batch * heads;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int32_t* idx = reinterpret_cast<int32_t*>(ws);
  ws += up256((size_t)lists * topk * block * sizeof(int32_t));
  int32_t* cnt = reinterpret_cast<int32_t*>(ws);
  ws += up256((size_t)lists * sizeof(int32_t));
  const size_t ws_att = ws_bytes - (size_t)(ws - static_cast<uint8_t*>(workspace));
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int nb = (int)cdiv(n_cap, block);
  esa::moba_decode_gate_kernel<__nv_bfloat16, 128><<<(unsigned)cdiv(lists, 4), 128, 0, s>>>(
      static_cast<const __nv_bfloat16*>(q), kbar, batch, heads, nb, block, pos, topk, idx, cnt, blocks_out);
  ESA_LAUNCH_CHECK("moba_decode_gate_kernel");
  return sparse_attn_impl(q, k, v, dt, batch, 1, n_cap, pos, heads, heads, head_dim, idx, cnt,
                          moba_decode_params(pos, block, topk), scale, o, lse, ws, ws_att, stream, heads);
}


// ------------------------------------------------------------------ no-alloc selection --
// Scratch for esa_score_select_noalloc: a fixed array in device memory that every GPU
// loading this library holds until the process exits. Host code may not use the name
// as a device address; the address comes from cudaGetSymbolAddress, once per context.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;     // 8 MiB
__device__ __align__(256) unsigned char g_select_scratch[kNoAllocScratchBytes];

// The array's device address in the current context, looked up with
// cudaGetSymbolAddress on the first call in each context and remembered under the
// context's unique id (a context made after another was destroyed gets its own lookup).
esa_status_t scratch_for_current_context(void** out) {
  static const char what = 0;
  intptr_t addr = 0;
  const esa_status_t st = per_context(&what, &addr, [](intptr_t* v) {
    void* p = nullptr;
    ESA_CUDA(cudaGetSymbolAddress(&p, g_select_scratch));
    *v = reinterpret_cast<intptr_t>(p);
    return ESA_OK;
  });
  if (st != ESA_OK) return st;
  *out = reinterpret_cast<void*>(addr);
  return ESA_OK;
}

}  // namespace

esa_status_t esa_score_select_noalloc(const float* q_c, const float* k_c, int32_t batch, int32_t lq, int64_t n_cap,
                                      int64_t c0, int32_t d_c, esa_params_t p, int32_t* idx_out, int32_t* count_out,
                                      float* score_out, void* stream) {
  if (batch <= 0 || lq <= 0) return fail(ESA_ERR_INVALID_ARG, "batch and lq must be >= 1");
  const size_t need = esa_score_select_workspace_size(batch, lq, n_cap, c0, d_c, p);
  if (need > kNoAllocScratchBytes)
    return fail(ESA_ERR_WORKSPACE,
                "this selection needs %zu bytes of scratch; the no-alloc entry point has %zu (use esa_score_select "
                "with a workspace)",
                need, kNoAllocScratchBytes);
  void* scratch = nullptr;
  const esa_status_t st = scratch_for_current_context(&scratch);
  if (st != ESA_OK) return st;
  return esa_score_select(q_c, k_c, batch, lq, n_cap, c0, d_c, p, idx_out, count_out, score_out, scratch,
                          kNoAllocScratchBytes, stream);
}

size_t esa_score_select_noalloc_capacity(void) { return kNoAllocScratchBytes; }

// ------------------------------------------------------------------ offline fit --
namespace {

int gram_splits(int dim, int64_t n) {
  const int tiles = dim / 128;
  const int64_t pairs = (int64_t)tiles * (tiles + 1) / 2;
  const int64_t chunks = std::max<int64_t>(1, cdiv(n, esa::kGmRows));
  return (int)std::max<int64_t>(1, std::min<int64_t>(chunks, 148 / pairs));
}

size_t gram_part_bytes(int dim, int64_t n) { return up256((size_t)gram_splits(dim, n) * dim * dim * sizeof(double)); }

esa_status_t gram_check(const void* x, esa_dtype_t dt, int64_t n, int32_t dim) {
  if (dt != ESA_BF16) return fail(ESA_ERR_UNSUPPORTED, "the Gram product takes bf16 rows");
  if (n <= 0) return fail(ESA_ERR_INVALID_ARG, "n must be >= 1");
  if (n >= ((int64_t)1 << 31)) return fail(ESA_ERR_UNSUPPORTED, "n must be < 2^31");
  if (dim <= 0 || dim % 128 || dim > 16384) return fail(ESA_ERR_UNSUPPORTED, "dim %d (a multiple of 128, <= 16384)", dim);
  if (!x) return fail(ESA_ERR_INVALID_ARG, "null pointer");
  if (!aligned(x, 16)) return fail(ESA_ERR_INVALID_ARG, "x needs 16-byte alignment");
  return ESA_OK;
}

// G [dim, dim] fp64 = X^T X for X [n, dim] bf16 (rows contiguous); part: scratch.
esa_status_t gram_launch(const void* x, int64_t n, int32_t dim, double* part, double* g, cudaStream_t s) {
  static const char what = 0;
  esa_status_t st = once_per_context(&what, [] {
    ESA_CUDA(cudaFuncSetAttribute(esa::gram_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, esa::kGmSmem));
    return ESA_OK;
  });
  if (st != ESA_OK) return st;
  PFN_cuTensorMapEncodeTiled_v12000 encode;
  if ((st = get_encoder(&encode)) != ESA_OK) return st;
  CUtensorMap tm;
  cuuint64_t dims[2] = {(cuuint64_t)dim, (cuuint64_t)n};
  cuuint64_t strides[1] = {(cuuint64_t)dim * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)esa::kGmRows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = encode(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), dims, strides, box, estr,
                            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(ESA_ERR_CUDA, "cuTensorMapEncodeTiled (Gram rows) failed (%d)", (int)r);
  const int splits = gram_splits(dim, n);
  esa::GramArgs a{};
  a.dim = dim;
  a.tiles = dim / 128;
  a.n = n;
  a.rows_per_split = cdiv(cdiv(n, splits), esa::kGmRows) * esa::kGmRows;
  a.part = part;
  const unsigned pairs = (unsigned)(a.tiles * (a.tiles + 1) / 2);
  esa::gram_kernel<<<dim3(pairs, splits), esa::kGmThreads, esa::kGmSmem, s>>>(tm, a);
  ESA_LAUNCH_CHECK("gram_kernel");
  const int64_t count = (int64_t)dim * dim;
  esa::gram_finish_kernel<<<(unsigned)std::min<int64_t>(4096, cdiv(count, 256)), 256, 0, s>>>(part, splits, count, g);
  ESA_LAUNCH_CHECK("gram_finish_kernel");
  return ESA_OK;
}

esa_status_t gemm64(int m, int n, int k, double alpha, const double* A, int64_t ar, int64_t ac, const double* B,
                    int64_t br, int64_t bc, double beta, double* C, int64_t ldc, cudaStream_t s) {
  if (m <= 0 || n <= 0) return ESA_OK;
  const dim3 grid((unsigned)cdiv(n, esa::kG64Tile), (unsigned)cdiv(m, esa::kG64Tile));
  esa::gemm64_kernel<<<grid, 256, 0, s>>>(m, n, k, alpha, A, ar, ac, B, br, bc, beta, C, ldc);
  ESA_LAUNCH_CHECK("gemm64_kernel");
  return ESA_OK;
}

esa_status_t fit_kernels_setup() {
  static const char what = 0;
  return once_per_context(&what, [] {
    ESA_CUDA(cudaFuncSetAttribute(esa::chol_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  esa::kCholSmem));
    ESA_CUDA(cudaFuncSetAttribute(esa::trsm_block_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  esa::kTrsmSmem));
    ESA_CUDA(cudaFuncSetAttribute(esa::jacobi_eig_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  esa::kJacobiSmem));
    return ESA_OK;
  });
}

esa_status_t chol_block(double* A, int64_t lda, int nb, unsigned site, cudaStream_t s) {
  esa::chol_block_kernel<<<1, 256, (size_t)nb * (nb + 1) * sizeof(double), s>>>(A, lda, nb, site);
  ESA_LAUNCH_CHECK("chol_block_kernel");
  return ESA_OK;
}

esa_status_t trsm_block(const double* T, int64_t ldt, int nb, double* X, int64_t xr, int64_t xc, int64_t ncols,
                        int trans, cudaStream_t s) {
  if (ncols <= 0) return ESA_OK;
  const size_t smem = nb <= esa::kTrsmStageMax ? (size_t)nb * nb * sizeof(double) : 0;
  esa::trsm_block_kernel<<<(unsigned)cdiv(ncols, esa::kTrsmCols), esa::kTrsmThreads, smem, s>>>(T, ldt, nb, X, xr,
                                                                                                 xc, ncols, trans);
  ESA_LAUNCH_CHECK("trsm_block_kernel");
  return ESA_OK;
}

// In place: A [dim, dim] symmetric positive definite -> its upper Cholesky factor R
// (A = R^T R, strict lower part zeroed). Right-looking, 128-wide blocks: factor the
// diagonal block, solve its row panel (R_kk^T P = A_k,rest), update the trailing matrix
// (A_rest -= P^T P) with the fp64 GEMM.
esa_status_t cholesky(double* A, int dim, unsigned site, cudaStream_t s) {
  esa_status_t st;
  const int T = dim / 128;
  for (int kb = 0; kb < T; ++kb) {
    double* akk = A + (int64_t)kb * 128 * (dim + 1);
    if ((st = chol_block(akk, dim, 128, site, s)) != ESA_OK) return st;
    const int m = dim - (kb + 1) * 128;
    if (m == 0) break;
    double* panel = A + (int64_t)kb * 128 * dim + (kb + 1) * 128;
    if ((st = trsm_block(akk, dim, 128, panel, dim, 1, m, 1, s)) != ESA_OK) return st;
    if ((st = gemm64(m, m, 128, -1.0, panel, 1, dim, panel, dim, 1, 1.0, A + (int64_t)(kb + 1) * 128 * (dim + 1), dim,
                     s)) != ESA_OK)
      return st;
  }
  esa::zero_lower_kernel<<<(unsigned)std::min<int64_t>(4096, cdiv((int64_t)dim * dim, 256)), 256, 0, s>>>(A, dim);
  ESA_LAUNCH_CHECK("zero_lower_kernel");
  return ESA_OK;
}

// In place: Y [dim, l] <- R^-1 Y for R [dim, dim] upper (blocked back substitution).
esa_status_t upper_solve(const double* R, int dim, double* Y, int l, cudaStream_t s) {
  esa_status_t st;
  for (int kb = dim / 128 - 1; kb >= 0; --kb) {
    double* yk = Y + (int64_t)kb * 128 * l;
    if ((st = trsm_block(R + (int64_t)kb * 128 * (dim + 1), dim, 128, yk, l, 1, l, 0, s)) != ESA_OK) return st;
    if (kb > 0 &&
        (st = gemm64(kb * 128, l, 128, -1.0, R + (int64_t)kb * 128, dim, 1, yk, l, 1, 1.0, Y, l, s)) != ESA_OK)
      return st;
  }
  return ESA_OK;
}

// In place: Y [m, l] <- an orthonormal basis of its columns (CholeskyQR twice: G = Y^T Y,
// G = R^T R, Y <- Y R^-1, repeated once for accuracy). gs: [l, l] scratch.
esa_status_t orthonormalize(double* Y, int m, int l, double* gs, unsigned site, cudaStream_t s) {
  esa_status_t st;
  for (int pass = 0; pass < 2; ++pass) {
    if ((st = gemm64(l, l, m, 1.0, Y, 1, l, Y, l, 1, 0.0, gs, l, s)) != ESA_OK) return st;
    if ((st = chol_block(gs, l, l, site + pass, s)) != ESA_OK) return st;
    // row y of Y solves x R = y, i.e. R^T x^T = y^T: forward substitution on each row
    if ((st = trsm_block(gs, l, l, Y, 1, l, m, 1, s)) != ESA_OK) return st;
  }
  return ESA_OK;
}

struct FitWs {
  double* part;     // Gram row-slice partials
  double* gq;       // [dq, dq] -> Rq
  double* gk;       // [dk, dk] -> Rk
  double* rqe;      // [dq, dk] Rq E
  double* c;        // [dq, dk] C = Rq E Rk^T
  double* a;        // [dk, dk] A = C^T C
  double* v;        // [dk, l] subspace basis
  double* w;        // [dk, l] A V
  double* gs;       // [l, l] Gram of the basis / projected problem
  double* z;        // [L, L] Jacobi rotations (L = l rounded up to even)
  double* zsel;     // [l, d_c] leading eigenvectors of the projected problem
  double* vd;       // [dk, d_c] leading right singular vectors of C -> folded key map
  double* cv;       // [dq, d_c] C V -> query map
  size_t bytes;
};

FitWs carve_fit(void* ws, int64_t n_q, int64_t n_k, int dq, int dk, int l, int d_c) {
  Carver cv{reinterpret_cast<uint8_t*>(ws)};
  FitWs w{};
  const size_t part = std::max(gram_part_bytes(dq, n_q), gram_part_bytes(dk, n_k));
  const int L = l + (l & 1);
  w.part = cv.take<double>(part / sizeof(double));
  w.gq = cv.take<double>((size_t)dq * dq);
  w.gk = cv.take<double>((size_t)dk * dk);
  w.rqe = cv.take<double>((size_t)dq * dk);
  w.c = cv.take<double>((size_t)dq * dk);
  w.a = cv.take<double>((size_t)dk * dk);
  w.v = cv.take<double>((size_t)dk * l);
  w.w = cv.take<double>((size_t)dk * l);
  w.gs = cv.take<double>((size_t)l * l);
  w.z = cv.take<double>((size_t)L * L);
  w.zsel = cv.take<double>((size_t)l * d_c);
  w.vd = cv.take<double>((size_t)dk * d_c);
  w.cv = cv.take<double>((size_t)dq * d_c);
  w.bytes = cv.off;
  return w;
}

}  // namespace

size_t esa_gram_workspace_size(int64_t n, int32_t dim) {
  if (n <= 0 || dim <= 0 || dim % 128) return 0;
  return gram_part_bytes(dim, n);
}

esa_status_t esa_gram(const void* x, esa_dtype_t dt, int64_t n, int32_t dim, double* g, void* workspace,
                      size_t ws_bytes, void* stream) {
  esa_status_t st = gram_check(x, dt, n, dim);
  if (st != ESA_OK) return st;
  if (!g) return fail(ESA_ERR_INVALID_ARG, "null pointer");
  const size_t need = gram_part_bytes(dim, n);
  if (!workspace || ws_bytes < need || !aligned(workspace, 256))
    return fail(ESA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned (got %zu)", need, ws_bytes);
  st = gram_launch(x, n, dim, static_cast<double*>(workspace), g, reinterpret_cast<cudaStream_t>(stream));
  return st == ESA_OK ? ok() : st;
}

size_t esa_fit_workspace_size(int64_t n_q, int64_t n_k, int32_t hq, int32_t hkv, int32_t head_dim, int32_t d_c,
                              int32_t oversample) {
  if (n_q <= 0 || n_k <= 0 || hq <= 0 || hkv <= 0 || head_dim <= 0 || d_c <= 0 || oversample < 0) return 0;
  const int dq = hq * head_dim, dk = hkv * head_dim;
  if (dq % 128 || dk % 128) return 0;
  return carve_fit(nullptr, n_q, n_k, dq, dk, d_c + oversample, d_c).bytes;
}

esa_status_t esa_fit_maps(const void* xq, int64_t n_q, const void* yk, int64_t n_k, esa_dtype_t dt, int32_t hq,
                          int32_t hkv, int32_t head_dim, int32_t d_c, int32_t oversample, double ridge,
                          int32_t power_iters, const double* omega, float* w_q, float* w_k, void* workspace,
                          size_t ws_bytes, void* stream) {
  if (hq <= 0 || hkv <= 0 || hq % hkv) return fail(ESA_ERR_INVALID_ARG, "hq must be a positive multiple of hkv");
  if (head_dim <= 0) return fail(ESA_ERR_INVALID_ARG, "head_dim must be >= 1");
  const int dq = hq * head_dim, dk = hkv * head_dim, group = hq / hkv;
  esa_status_t st = gram_check(xq, dt, n_q, dq);
  if (st != ESA_OK) return st;
  if ((st = gram_check(yk, dt, n_k, dk)) != ESA_OK) return st;
  const int l = d_c + oversample;
  if (d_c < 1 || oversample < 0 || l > esa::kCholMax || l > dk)
    return fail(ESA_ERR_UNSUPPORTED, "d_c %d + oversample %d must be in [1, min(%d, hkv * head_dim)]", d_c,
                oversample, esa::kCholMax);
  if (!(ridge >= 0.0) || !std::isfinite(ridge)) return fail(ESA_ERR_INVALID_ARG, "ridge must be finite and >= 0");
  if (power_iters < 0 || power_iters > 64) return fail(ESA_ERR_INVALID_ARG, "power_iters must be in [0, 64]");
  if (!omega || !w_q || !w_k) return fail(ESA_ERR_INVALID_ARG, "null pointer");
  const size_t need = carve_fit(nullptr, n_q, n_k, dq, dk, l, d_c).bytes;
  if (!workspace || ws_bytes < need || !aligned(workspace, 256))
    return fail(ESA_ERR_WORKSPACE, "workspace needs %zu bytes, 256-byte aligned (got %zu)", need, ws_bytes);
  if ((st = fit_kernels_setup()) != ESA_OK) return st;
  const FitWs w = carve_fit(workspace, n_q, n_k, dq, dk, l, d_c);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // Gram matrices (+ ridge), then their upper Cholesky factors
  if ((st = gram_launch(xq, n_q, dq, w.part, w.gq, s)) != ESA_OK) return st;
  if (ridge > 0.0) {
    esa::ridge_kernel<<<1, 256, 0, s>>>(w.gq, dq, ridge);
    ESA_LAUNCH_CHECK("ridge_kernel");
  }
  if ((st = gram_launch(yk, n_k, dk, w.part, w.gk, s)) != ESA_OK) return st;
  if (ridge > 0.0) {
    esa::ridge_kernel<<<1, 256, 0, s>>>(w.gk, dk, ridge);
    ESA_LAUNCH_CHECK("ridge_kernel");
  }
  if ((st = cholesky(w.gq, dq, 700, s)) != ESA_OK) return st;
  if ((st = cholesky(w.gk, dk, 701, s)) != ESA_OK) return st;
  // C = (Rq E) Rk^T and A = C^T C
  esa::fold_heads_kernel<<<(unsigned)std::min<int64_t>(4096, cdiv((int64_t)dq * dk, 256)), 256, 0, s>>>(
      w.gq, dq, hkv, group, head_dim, w.rqe);
  ESA_LAUNCH_CHECK("fold_heads_kernel");
  if ((st = gemm64(dq, dk, dk, 1.0, w.rqe, dk, 1, w.gk, 1, dk, 0.0, w.c, dk, s)) != ESA_OK) return st;
  if ((st = gemm64(dk, dk, dq, 1.0, w.c, 1, dk, w.c, dk, 1, 0.0, w.a, dk, s)) != ESA_OK) return st;
  // subspace iteration: V = orth(A Omega), then power_iters rounds of V = orth(A V)
  if ((st = gemm64(dk, l, dk, 1.0, w.a, dk, 1, omega, l, 1, 0.0, w.v, l, s)) != ESA_OK) return st;
  if ((st = orthonormalize(w.v, dk, l, w.gs, 710, s)) != ESA_OK) return st;
  double* v = w.v;
  double* t = w.w;
  for (int it = 0; it < power_iters; ++it) {
    if ((st = gemm64(dk, l, dk, 1.0, w.a, dk, 1, v, l, 1, 0.0, t, l, s)) != ESA_OK) return st;
    if ((st = orthonormalize(t, dk, l, w.gs, 720, s)) != ESA_OK) return st;
    std::swap(v, t);
  }
  // Rayleigh-Ritz: H = V^T A V, its leading d_c eigenvectors, V_d = V Z_sel
  if ((st = gemm64(dk, l, dk, 1.0, w.a, dk, 1, v, l, 1, 0.0, t, l, s)) != ESA_OK) return st;
  if ((st = gemm64(l, l, dk, 1.0, v, 1, l, t, l, 1, 0.0, w.gs, l, s)) != ESA_OK) return st;
  esa::jacobi_eig_kernel<<<1, esa::kJacobiThreads, esa::kJacobiSmem, s>>>(w.gs, l, w.z, d_c, w.zsel, 30);
  ESA_LAUNCH_CHECK("jacobi_eig_kernel");
  if ((st = gemm64(dk, d_c, l, 1.0, v, l, 1, w.zsel, d_c, 1, 0.0, w.vd, d_c, s)) != ESA_OK) return st;
  // query map W_q = Rq^-1 C V_d, folded key map B = Rk^-1 V_d
  if ((st = gemm64(dq, d_c, dk, 1.0, w.c, dk, 1, w.vd, d_c, 1, 0.0, w.cv, d_c, s)) != ESA_OK) return st;
  if ((st = upper_solve(w.gq, dq, w.cv, d_c, s)) != ESA_OK) return st;
  if ((st = upper_solve(w.gk, dk, w.vd, d_c, s)) != ESA_OK) return st;
  esa::emit_maps_kernel<<<(unsigned)std::min<int64_t>(4096, cdiv((int64_t)dq * d_c, 256)), 256, 0, s>>>(
      w.cv, w.vd, hq, group, head_dim, d_c, w_q, w_k);
  ESA_LAUNCH_CHECK("emit_maps_kernel");
  return ok();
}
