/*
 * esa.h - C ABI of libesa: query-aware top-k selective attention on B200 (sm_100a).
 *
 * Two forms of the method:
 *   ESA  - Efficient Selective Attention (Huawei Noah's Ark write-up, arXiv 2502.14477):
 *          compress query and key with a one-layer linear map, score every middle
 *          cached token against the current chunk's queries in that low-dimensional
 *          space, correct each query's scores, sum over the chunk, lift each score by
 *          its neighbours, keep the top-k, and attend exactly over initial + selected +
 *          local tokens.
 *   MoBA - Mixture of Block Attention (MoBA article, arXiv 2502.13189): a gate picks
 *          the top-k past blocks by <q, mean-pooled block keys>, the current block is
 *          always added with a causal mask, and attention runs over those blocks.
 *
 * Conventions for every call:
 *   - Every tensor pointer is DEVICE memory owned by the caller. The library never
 *     allocates, frees or keeps a pointer after the call returns. Scratch memory is
 *     passed in through `workspace`; its size comes from the matching *_workspace_size
 *     call, and it needs 256-byte alignment.
 *   - Tensors are dense and row-major in the order the shapes are written. q, k, v, o
 *     need 16-byte aligned base pointers; compressed tensors (q_c, k_c) too.
 *   - `stream` is a cudaStream_t passed as an opaque pointer (NULL = legacy default
 *     stream). Every call only enqueues work on it and returns; none synchronises.
 *   - Arguments are checked on the host before anything is launched. A bad argument
 *     returns ESA_ERR_INVALID_ARG (or ESA_ERR_WORKSPACE / ESA_ERR_UNSUPPORTED) and
 *     launches nothing. A failed launch returns ESA_ERR_CUDA. esa_last_error() then
 *     gives a message (thread-local, valid until the next call on the same thread).
 *   - Kernels that wait on barriers wait a bounded time. If a wait runs out, the
 *     kernel records ESA_ERR_TIMEOUT in a device status word and returns without
 *     hanging; esa_device_status() reads and clears that word.
 *   - Calls are thread-compatible: calls on different streams may overlap only if
 *     they use different workspaces and write different outputs.
 *
 * Citations name the page and passage each operation follows.
 */
#ifndef ESA_H_
#define ESA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  ESA_OK = 0,
  ESA_ERR_INVALID_ARG = 1,  /* a shape, pointer, alignment or parameter is wrong */
  ESA_ERR_UNSUPPORTED = 2,  /* valid, but this build has no kernel for it (e.g. head_dim 96) */
  ESA_ERR_CUDA = 3,         /* a CUDA runtime call or launch failed */
  ESA_ERR_TIMEOUT = 4,      /* a device-side bounded wait ran out (see esa_device_status) */
  ESA_ERR_WORKSPACE = 5     /* workspace is NULL, misaligned or smaller than required */
} esa_status_t;

typedef enum { ESA_F32 = 0, ESA_BF16 = 1 } esa_dtype_t;

/* ESA selection parameters.
 *   n_init  - initial tokens always attended (ESA write-up, implementation paragraph:
 *             the sequence is split into initial, middle, local and current parts)
 *   window  - local tokens before the chunk that are always attended
 *   topk    - middle tokens kept (ESA write-up, core steps: a fixed number of tokens)
 *   eps     - neighbour radius of the neighbour-influence step (ESA write-up,
 *             neighbour-influence paragraph; read as a max over +-eps)
 *   clamp_c - lower bound -C of each query's max-shifted score (ESA write-up,
 *             score-correction paragraph); +INFINITY disables the clamp.
 * Regions of a chunk [c0, c1) (c1 = c0 + lq):
 *   lo = min(c0, max(n_init, c0 - window));
 *   initial = [0, min(n_init, lo)), middle = [n_init, lo), local = [lo, c1) (causal). */
typedef struct {
  int32_t n_init;
  int32_t window;
  int32_t topk;
  int32_t eps;
  float clamp_c;
} esa_params_t;

/* ---------------------------------------------------------------- ESA calls -- */

/* esa_compress - one-layer linear map of the merged heads (ESA write-up, core-steps
 * and implementation paragraphs: q and k pass through a one-layer MLP, 4096 -> 128).
 *   y[r, :] = concat_{h < n_heads_out} x[r, h / G, :] @ W,   G = n_heads_out / n_heads_in
 * i.e. under GQA each query head h reads KV head h / G (keys are expanded to the
 * query-head count before the map). No bias, no activation.
 *   x:  rows of [n_heads_in, head_dim], dtype x_dtype (ESA_F32 or ESA_BF16); row r starts
 *       at element r * x_row_stride (x_row_stride >= n_heads_in * head_dim, a multiple of 8),
 *       so one call can read the new key of every sequence of a batched cache
 *   w:  [n_heads_out * head_dim, d_out] fp32
 *   y:  rows of d_out fp32, row r at y + r * y_row_stride (y_row_stride >= d_out), so a
 *       call can write straight into a compressed key cache at any row offset.
 * Requires head_dim in {64, 128}, d_out % 16 == 0, d_out <= 256, rows >= 0 (0 = no-op).
 * Accumulates in fp32. */
esa_status_t esa_compress(const void* x, esa_dtype_t x_dtype, int64_t rows, int64_t x_row_stride,
                          int32_t n_heads_in, int32_t n_heads_out, int32_t head_dim,
                          const float* w, int32_t d_out, float* y, int64_t y_row_stride,
                          void* stream);

/* esa_compress_pack_size / esa_compress_pack / esa_compress_packed - the same map
 * with the weight prepared once for the tensor cores. The weight is static across
 * calls (it is the compression layer), so folding the GQA rows and splitting fp32
 * into bf16 high + low parts (|w - hi - lo| <= 2^-17 |w|; both halves are multiplied,
 * so the product keeps fp32-level accuracy) is done by esa_compress_pack, and every
 * later esa_compress_packed call only streams x and the packed weight.
 *   esa_compress_pack_size: bytes of the packed weight for a reduction length
 *       K = n_heads_in * head_dim and d_out; 0 if the packed path does not support the
 *       shape (it needs d_out == 128 and K a multiple of 512).
 *   esa_compress_pack: w as for esa_compress ([n_heads_out * head_dim, d_out] fp32,
 *       n_heads_out a multiple of n_heads_in) -> packed (device, caller-owned,
 *       packed_bytes >= esa_compress_pack_size, 16-byte aligned). The packed layout is
 *       the library's own; it is only valid as input to esa_compress_packed with the
 *       same n_heads_in, head_dim and d_out.
 *   esa_compress_packed: y = the map of x (bf16 rows of [n_heads_in, head_dim], row r at
 *       x + r * x_row_stride, x_row_stride a multiple of 8, base 16-byte aligned) with
 *       the packed weight; y as for esa_compress (fp32, y_row_stride >= 128, base and
 *       y_row_stride giving 16-byte aligned rows). rows >= 0 (0 = no-op).
 * Results equal esa_compress's up to fp32 summation order (both split the weight the
 * same way and accumulate in fp32). Errors: ESA_ERR_UNSUPPORTED for shapes the packed
 * path does not take, ESA_ERR_INVALID_ARG for null, misaligned or short buffers. */
size_t esa_compress_pack_size(int32_t n_heads_in, int32_t head_dim, int32_t d_out);
esa_status_t esa_compress_pack(const float* w, int32_t n_heads_in, int32_t n_heads_out, int32_t head_dim,
                               int32_t d_out, void* packed, size_t packed_bytes, void* stream);
esa_status_t esa_compress_packed(const void* x, int64_t rows, int64_t x_row_stride, int32_t n_heads_in,
                                 int32_t head_dim, const void* packed, int32_t d_out, float* y,
                                 int64_t y_row_stride, void* stream);

/* esa_score_select - importance score, correction, chunk sum, neighbour max-pool and
 * top-k for one chunk of every sequence in a batch (ESA write-up, implementation,
 * score-correction and neighbour-influence paragraphs).
 *   S_ij = q_c[b, i] . k_c[b, j]                 for i < lq, j in middle
 *   m_i  = max_j S_ij
 *   s_j  = sum_i max(S_ij - m_i, -clamp_c)
 *   s'_j = max_{m in middle, |m - j| <= eps} s_m
 *   keep min(topk, |middle|) tokens by (s' descending, position ascending)
 *   q_c:       [batch, lq, d_c] fp32, compressed queries at positions [c0, c0 + lq)
 *   k_c:       [batch, n_cap, d_c] fp32, compressed key cache; rows [0, c0 + lq) valid
 *   idx_out:   [batch, topk] int32 absolute positions, ascending, -1 after count
 *   count_out: [batch] int32 = min(topk, |middle|) (the same for every sequence)
 *   score_out: NULL, or [batch, |middle|] fp32 receiving s' (for checking)
 * Requires d_c % 16 == 0 and d_c <= 256, 1 <= lq <= 4096, c0 + lq <= n_cap,
 * topk >= 1, 0 <= eps <= 64. An empty middle gives count 0 and all -1. */
esa_status_t esa_score_select(const float* q_c, const float* k_c, int32_t batch, int32_t lq,
                              int64_t n_cap, int64_t c0, int32_t d_c, esa_params_t p,
                              int32_t* idx_out, int32_t* count_out, float* score_out,
                              void* workspace, size_t ws_bytes, void* stream);

size_t esa_score_select_workspace_size(int32_t batch, int32_t lq, int64_t n_cap, int64_t c0,
                                       int32_t d_c, esa_params_t p);

/* esa_sparse_attn - exact attention over initial + selected + local tokens (ESA
 * write-up, implementation and final-attention paragraphs: initial and selected
 * tokens form the global part, local tokens the window part, fused into one output
 * with the full queries, keys and values). One softmax over the union; causal inside
 * the local part; GQA: query head h reads KV head h / (hq / hkv).
 *   q:     [batch, lq, hq, head_dim]   queries at positions [c0, c0 + lq)
 *   k, v:  [batch, n_cap, hkv, head_dim]; rows [0, c0 + lq) valid
 *   idx:   [batch, >= p.topk] int32 selected middle positions, ascending (as
 *          esa_score_select writes them); count: [batch] int32 entries used
 *   o:     [batch, lq, hq, head_dim], dtype dt
 *   lse:   NULL or [batch, lq, hq] fp32, natural log of the softmax denominator
 *   scale: softmax scale; <= 0 means 1/sqrt(head_dim)
 * Requires head_dim in {64, 128}, hq % hkv == 0, c0 + lq <= n_cap. The selected
 * positions must lie in the middle region; entries are not re-checked on the device. */
esa_status_t esa_sparse_attn(const void* q, const void* k, const void* v, esa_dtype_t dt,
                             int32_t batch, int32_t lq, int64_t n_cap, int64_t c0,
                             int32_t hq, int32_t hkv, int32_t head_dim,
                             const int32_t* idx, const int32_t* count, esa_params_t p,
                             float scale, void* o, float* lse,
                             void* workspace, size_t ws_bytes, void* stream);

size_t esa_sparse_attn_workspace_size(int32_t batch, int32_t lq, int64_t c0, int32_t hq,
                                      int32_t hkv, int32_t head_dim, esa_dtype_t dt,
                                      esa_params_t p);

/* esa_score_select_heads - the per-head selection variant (ESA write-up, ablation
 * after the experiments: ESA merges all heads into one importance score; the
 * comparison it is tested against chooses tokens per head). Reading: one selection
 * per group of compressed columns. Group g owns columns [g * d_g, (g + 1) * d_g) of
 * q_c and k_c (d_g = d_c / n_groups; compress with a block-diagonal map, group g's
 * block taking the query heads of KV head g), and runs exactly the steps of
 * esa_score_select on them:
 *   S^g_ij = q_c[b, i, group g] . k_c[b, j, group g], then correction, clamp, chunk
 *   sum, neighbour max-pool and top-k per (sequence, group).
 *   q_c, k_c: as for esa_score_select
 *   idx_out:   [batch, n_groups, topk] int32, ascending, -1 after count
 *   count_out: [batch, n_groups] int32
 *   score_out: NULL, or [batch, n_groups, |middle|] fp32 receiving s'
 * Requires n_groups in {1, 2, 4, 8} and d_c % n_groups == 0. With lq <= 8 the groups
 * must split a key's lanes (d_c >= 128, or d_c / 4 divisible by n_groups); with more
 * queries d_g must be a multiple of 16. n_groups = 1 is esa_score_select. Errors as for
 * esa_score_select, ESA_ERR_UNSUPPORTED for group shapes outside these. */
esa_status_t esa_score_select_heads(const float* q_c, const float* k_c, int32_t batch, int32_t lq,
                                    int64_t n_cap, int64_t c0, int32_t d_c, int32_t n_groups,
                                    esa_params_t p, int32_t* idx_out, int32_t* count_out,
                                    float* score_out, void* workspace, size_t ws_bytes,
                                    void* stream);

size_t esa_score_select_heads_workspace_size(int32_t batch, int32_t lq, int64_t n_cap, int64_t c0,
                                             int32_t d_c, int32_t n_groups, esa_params_t p);

/* esa_sparse_attn_heads - esa_sparse_attn with one key list per KV head (the attention
 * of the per-head selection variant): query head h attends initial + the selected
 * tokens of KV head h / (hq / hkv) + local.
 *   idx:   [batch, hkv, >= p.topk] int32 per-head selected middle positions, ascending
 *          (esa_score_select_heads with n_groups = hkv writes them); count: [batch, hkv]
 * Everything else, requirements and errors as for esa_sparse_attn. */
esa_status_t esa_sparse_attn_heads(const void* q, const void* k, const void* v, esa_dtype_t dt,
                                   int32_t batch, int32_t lq, int64_t n_cap, int64_t c0,
                                   int32_t hq, int32_t hkv, int32_t head_dim,
                                   const int32_t* idx, const int32_t* count, esa_params_t p,
                                   float scale, void* o, float* lse,
                                   void* workspace, size_t ws_bytes, void* stream);

size_t esa_sparse_attn_heads_workspace_size(int32_t batch, int32_t lq, int64_t c0, int32_t hq,
                                            int32_t hkv, int32_t head_dim, esa_dtype_t dt,
                                            esa_params_t p);

/* esa_score_select_noalloc - esa_score_select without a workspace argument. The pages
 * have no counterpart of this call: it exists for callers that cannot allocate device
 * memory - a service that plans all its memory at start-up and allows no allocation
 * afterwards, a plugin running inside another runtime with no access to that runtime's
 * allocator, a latency-critical loop where an allocation's stall or failure is not
 * acceptable. It allocates nothing (no cudaMalloc, no cudaFree, no allocating library
 * routine): its scratch is a fixed 8 MiB array in device memory
 * (esa_score_select_noalloc_capacity() bytes) that every GPU loading this library
 * holds until the process exits.
 *   - Arguments and results are those of esa_score_select.
 *   - A selection whose scratch (esa_score_select_workspace_size) exceeds the array
 *     returns ESA_ERR_WORKSPACE without launching anything.
 *   - The first call in each CUDA context (the device's primary context, or one the
 *     caller made current) looks up the array's device address there (a one-time host
 *     call per context, remembered under the context's unique id); make that first
 *     call before any stream capture.
 *   - All calls share the one array, and it keeps the previous call's contents; the
 *     call clears what must start at zero itself. Calls whose GPU work overlaps (on
 *     different streams or threads, for the same device) race on the array and give
 *     wrong results: serialise them. */
esa_status_t esa_score_select_noalloc(const float* q_c, const float* k_c, int32_t batch, int32_t lq,
                                      int64_t n_cap, int64_t c0, int32_t d_c, esa_params_t p,
                                      int32_t* idx_out, int32_t* count_out, float* score_out,
                                      void* stream);

/* Bytes of the fixed scratch array esa_score_select_noalloc uses. */
size_t esa_score_select_noalloc_capacity(void);

/* --------------------------------------------------------------- MoBA calls -- */

/* moba_block_gate - block choice of MoBA (MoBA article, section 3: blocks of size
 * `block`, gate s_i = <q, mean_pool(K[block i])>, top-k gate, causality).
 * Block b covers [b*block, min((b+1)*block, seq)). For a query at position p in block
 * c = p / block, the candidates are the past blocks 0..c-1 (reading: "strictly before
 * the query's block"); the kept ones are the top min(topk, c) by (score descending,
 * block ascending); the current block c is always added.
 *   q, k:       [batch, seq, heads, head_dim], dtype dt
 *   blocks_out: [batch, seq, heads, topk + 1] int16: attended blocks ascending (the
 *               current block last), then -1.
 * Requires head_dim in {64, 128}, block >= 16 and a multiple of 16,
 * 0 <= topk <= 15, seq / block <= 1024 blocks. Means and scores are fp32. */
esa_status_t moba_block_gate(const void* q, const void* k, esa_dtype_t dt, int32_t batch,
                             int64_t seq, int32_t heads, int32_t head_dim, int32_t block,
                             int32_t topk, int16_t* blocks_out,
                             void* workspace, size_t ws_bytes, void* stream);

/* moba_block_attn - attention of each (query, head) over the blocks listed for it
 * (MoBA article, section 2: MoBA(q, K, V) = Softmax(q K[I]^T) V[I]); the current
 * block is cut causally at the query (section 3, causality). Scale as esa_sparse_attn.
 *   blocks: [batch, seq, heads, topk + 1] int16 as moba_block_gate writes them.
 *   o:      [batch, seq, heads, head_dim] dtype dt; lse: NULL or [batch, seq, heads] fp32. */
esa_status_t moba_block_attn(const void* q, const void* k, const void* v, esa_dtype_t dt,
                             int32_t batch, int64_t seq, int32_t heads, int32_t head_dim,
                             int32_t block, int32_t topk, const int16_t* blocks, float scale,
                             void* o, float* lse, void* workspace, size_t ws_bytes,
                             void* stream);

/* moba_block_gate_attn - the whole MoBA causal prefill: moba_block_gate then
 * moba_block_attn. blocks_out may be NULL (the lists then live in the workspace). */
esa_status_t moba_block_gate_attn(const void* q, const void* k, const void* v, esa_dtype_t dt,
                                  int32_t batch, int64_t seq, int32_t heads, int32_t head_dim,
                                  int32_t block, int32_t topk, float scale, void* o, float* lse,
                                  int16_t* blocks_out, void* workspace, size_t ws_bytes,
                                  void* stream);

/* Workspace bytes for moba_block_gate (which = 0), moba_block_attn (1) and
 * moba_block_gate_attn (2). */
size_t moba_workspace_size(int32_t which, int32_t batch, int64_t seq, int32_t heads,
                           int32_t head_dim, int32_t block, int32_t topk);

/* moba_block_means - the block means of a key cache (MoBA article, section 2: a block
 * is represented by the mean of its keys), for blocks [blk_begin, blk_end) of
 * kbar [batch, heads, ceil(n_cap / block), head_dim] fp32 (caller-owned). k: [batch,
 * n_cap, heads, head_dim] bf16. A decode loop computes the means of the complete
 * blocks once and one more each time a block fills. Requires head_dim 128, block a
 * multiple of 16 (<= 1024 blocks). */
esa_status_t moba_block_means(const void* k, esa_dtype_t dt, int32_t batch, int64_t n_cap, int32_t heads,
                              int32_t head_dim, int32_t block, int32_t blk_begin, int32_t blk_end,
                              float* kbar, void* stream);

/* moba_decode_attn - one MoBA decode step (MoBA article, sections 2-3, for a single
 * query): per (sequence, head) the gate scores the query at position pos against the
 * means of the past blocks (blocks < pos / block), keeps the top min(topk, past) by
 * (score desc, block asc), and the attention runs over the kept blocks plus the
 * current block up to pos (one softmax).
 *   q:    [batch, 1, heads, head_dim] bf16;  k, v: [batch, n_cap, heads, head_dim] bf16
 *   kbar: [batch, heads, ceil(n_cap / block), head_dim] fp32 with every past block's
 *         mean (moba_block_means)
 *   o:    [batch, 1, heads, head_dim];  lse: NULL or [batch, 1, heads] fp32
 *   blocks_out: NULL or [batch, heads, topk + 1] int16: kept blocks ascending, the
 *         current block, -1 padding
 * Requires 1 <= topk <= 15, 0 <= pos < n_cap, head_dim 128. */
esa_status_t moba_decode_attn(const void* q, const void* k, const void* v, esa_dtype_t dt, int32_t batch,
                              int64_t n_cap, int64_t pos, int32_t heads, int32_t head_dim, int32_t block,
                              int32_t topk, const float* kbar, float scale, void* o, float* lse,
                              int16_t* blocks_out, void* workspace, size_t ws_bytes, void* stream);

size_t moba_decode_workspace_size(int32_t batch, int64_t n_cap, int64_t pos, int32_t heads, int32_t head_dim,
                                  int32_t block, int32_t topk);

/* ------------------------------------------------------- CCA-style attention -- */

/* cca_attn - causal prefill of one layer with CCA-style attention (CCA-Attention
 * article: global-aware pooling, locality-preserving module, and their fusion). The
 * sequence is cut into groups of `group` tokens; a complete group's core key and value
 * are its keys and values weighted by the softmax (scale as below) of the group's last
 * query against the group's keys, per query head. Query i attends, in one softmax, the
 * core tokens of the groups that end before its window and the window's tokens
 * [max(0, group * floor(i / group) - window), i].
 *   q: [batch, seq, hq, head_dim]; k, v: [batch, seq, hkv, head_dim]; o like q;
 *   lse: NULL or [batch, seq, hq] fp32 (natural log).
 *   scale: softmax scale; <= 0 means 1/sqrt(head_dim).
 * Requires bf16, head_dim 128, hq / hkv in {1, 2, 4, 8}, group a multiple of 128,
 * window a multiple of group. Workspace: cca_workspace_size bytes, 256-byte aligned
 * (core keys and values bf16, the core pass's bf16 partials and fp32 LSE). Errors as
 * for esa_sparse_attn. */
esa_status_t cca_attn(const void* q, const void* k, const void* v, esa_dtype_t dt, int32_t batch, int64_t seq,
                      int32_t hq, int32_t hkv, int32_t head_dim, int32_t group, int32_t window, float scale,
                      void* o, float* lse, void* workspace, size_t ws_bytes, void* stream);
size_t cca_workspace_size(int32_t batch, int64_t seq, int32_t hq, int32_t head_dim, int32_t group);

/* ----------------------------------------------- variable-length decode batches -- */

/* A decode batch whose sequences hold different numbers of cached tokens (ESA write-up,
 * problem statement: decode over each sequence's own KV cache; the pages batch nothing,
 * so this is the plain reading: every sequence runs the one-query step on its own).
 *   seq_len: device int64 [batch], caller-owned. Sequence b holds seq_len[b] tokens:
 *            rows [0, seq_len[b]) of its K/V and compressed caches; its one query sits
 *            at position seq_len[b] - 1, and the region rule (initial, middle, local)
 *            applies with c0 = seq_len[b] - 1. Rows past seq_len[b] are never read.
 *            The lengths stay on the device (a captured decode graph can replay with
 *            new lengths); a length outside [1, n_cap] is clamped into it and recorded
 *            in the device status word, which esa_device_status() then reports as
 *            ESA_ERR_INVALID_ARG.
 * Caches are laid out as for the equal-length calls with n_cap rows per sequence. */

/* esa_compress_packed_varlen - esa_compress_packed of one new key row per sequence,
 * written to that sequence's last token: x row b (bf16 [n_heads_in, head_dim] at
 * x + b * x_row_stride) -> k_c[b * n_cap + seq_len[b] - 1] (fp32 [batch, n_cap, d_out],
 * rows of d_out floats). Requirements and errors as for esa_compress_packed. */
esa_status_t esa_compress_packed_varlen(const void* x, int32_t batch, int64_t x_row_stride, int32_t n_heads_in,
                                        int32_t head_dim, const void* packed, int32_t d_out, float* k_c,
                                        int64_t n_cap, const int64_t* seq_len, void* stream);

/* esa_score_select_varlen - esa_score_select (n_groups 1) or esa_score_select_heads
 * (n_groups 2, 4, 8) for one query per sequence at its own position.
 *   q_c:       [batch, 1, d_c] fp32 (16-byte aligned); k_c: [batch, n_cap, d_c] fp32
 *   idx_out:   [batch, n_groups, topk] int32, ascending, -1 past count;
 *   count_out: [batch, n_groups] int32 = min(topk, that sequence's middle length)
 *   score_out: NULL or [batch, n_groups, n_mid_max] fp32 s', n_mid_max the middle
 *              length of a query at n_cap - 1; entries past a sequence's own middle
 *              are left unwritten.
 * Requires d_c in {16, 32, 64, 128, 256} with d_c / 4 (32 from 128 on) lanes per key
 * divisible by n_groups; else ESA_ERR_UNSUPPORTED. Workspace: ..._workspace_size
 * bytes (256-byte aligned), which covers every length up to n_cap. */
esa_status_t esa_score_select_varlen(const float* q_c, const float* k_c, int32_t batch, int64_t n_cap,
                                     const int64_t* seq_len, int32_t d_c, int32_t n_groups, esa_params_t p,
                                     int32_t* idx_out, int32_t* count_out, float* score_out, void* workspace,
                                     size_t ws_bytes, void* stream);
size_t esa_score_select_varlen_workspace_size(int32_t batch, int64_t n_cap, int32_t d_c, int32_t n_groups,
                                              esa_params_t p);

/* esa_sparse_attn_varlen - esa_sparse_attn (lists 1) or esa_sparse_attn_heads (lists
 * == hkv) for one query per sequence at position seq_len[b] - 1: it attends initial +
 * idx[:count] + local [lo, seq_len[b]) of its own sequence.
 *   q: [batch, 1, hq, head_dim]; k, v: [batch, n_cap, hkv, head_dim]; o like q;
 *   lse: NULL or [batch, 1, hq]; idx/count as esa_score_select_varlen writes them.
 * Dtypes, head dims, GQA groups, scale and errors as for esa_sparse_attn. */
esa_status_t esa_sparse_attn_varlen(const void* q, const void* k, const void* v, esa_dtype_t dt, int32_t batch,
                                    int64_t n_cap, const int64_t* seq_len, int32_t hq, int32_t hkv,
                                    int32_t head_dim, const int32_t* idx, const int32_t* count, int32_t lists,
                                    esa_params_t p, float scale, void* o, float* lse, void* workspace,
                                    size_t ws_bytes, void* stream);
size_t esa_sparse_attn_varlen_workspace_size(int32_t batch, int64_t n_cap, int32_t hq, int32_t hkv,
                                             int32_t head_dim, esa_dtype_t dt, int32_t lists, esa_params_t p);

/* ------------------------------------------- offline fit of the compression maps -- */

/* esa_gram - the Gram matrix G = X^T X of calibration rows X [n, dim] (bf16, rows
 * contiguous), accumulated in fp32 on the tensor cores (bf16 products are exact in
 * fp32) and returned in fp64 [dim, dim] (both triangles). The first step of the offline
 * fit below (ESA write-up, compression paragraph).
 *   Requires dim a multiple of 128 (<= 16384), 1 <= n < 2^31, x 16-byte aligned.
 *   workspace: esa_gram_workspace_size(n, dim) bytes, 256-byte aligned (fp32 partial
 *   sums over slices of the rows, added in a fixed order: the result is deterministic). */
esa_status_t esa_gram(const void* x, esa_dtype_t dt, int64_t n, int32_t dim, double* g, void* workspace,
                      size_t ws_bytes, void* stream);
size_t esa_gram_workspace_size(int64_t n, int32_t dim);

/* esa_fit_maps - the two one-layer compression maps fitted offline from calibration
 * queries and keys (ESA write-up, compression paragraph: the maps are learned from
 * queries and keys kept from a calibration run, the model untouched; experiments
 * paragraph: 4096 -> 128). The loss is not on the pages; this call minimises the plain
 * least squares of the compressed scores against the merged-head scores over every
 * (calibration query, calibration key) pair,
 *     sum_ij ( q~_i . k~_j - sum_h q_i^h . k_j^{h / G} )^2 .
 * Method: Gram matrices X^T X, Y^T Y (tensor cores, fp32 accumulation) plus a ridge of
 * ridge * trace / dim on the diagonal, their upper Cholesky factors Rq, Rk (fp64), the
 * matrix C = Rq E Rk^T (E the GQA expansion), the leading d_c right singular vectors V
 * of C (the leading eigenvectors of C^T C: subspace iteration with l = d_c + oversample
 * columns from the caller's Gaussian start omega, power_iters rounds with CholeskyQR2
 * re-orthonormalisation, then a Rayleigh-Ritz step whose l x l problem is solved by the
 * cyclic Jacobi method), then W_q = Rq^-1 C V and the folded key map B = Rk^-1 V. The
 * compressed scores q~ . k~ = x W_q B^T y^T are the least-squares optimum
 * (Eckart-Young); the maps themselves are one of the equivalent pairs (W_q T, W_k T^-T
 * for invertible T). The error of the subspace falls like (lambda_{l+1} / lambda_{d_c})
 * ^ power_iters in the eigenvalues of C^T C.
 *   xq:    [n_q, hq, head_dim] bf16 calibration queries; yk: [n_k, hkv, head_dim] keys.
 *   omega: [hkv * head_dim, d_c + oversample] fp64 on the device, standard normal
 *          entries (the random start is an input: the call draws no random numbers).
 *   w_q:   [hq * head_dim, d_c] fp32, the query map of esa_compress (n_heads_out = hq).
 *   w_k:   [hq * head_dim, d_c] fp32, the key map of esa_compress with the keys expanded
 *          to hq heads (each query head's rows are its KV head's rows of B divided by
 *          the group size hq / hkv; esa_compress_pack folds it back to B).
 *   Requires hq * head_dim and hkv * head_dim multiples of 128, d_c >= 1, oversample
 *   >= 0, d_c + oversample <= min(160, hkv * head_dim), 0 <= power_iters <= 64,
 *   ridge >= 0 (needed when n_q < hq * head_dim or n_k < hkv * head_dim). A Gram matrix that is not positive definite is reported by
 *   esa_device_status (a Cholesky pivot was not positive) and the maps are then invalid.
 *   workspace: esa_fit_workspace_size(...) bytes, 256-byte aligned. Asynchronous on the
 *   stream; the library allocates nothing. */
esa_status_t esa_fit_maps(const void* xq, int64_t n_q, const void* yk, int64_t n_k, esa_dtype_t dt, int32_t hq,
                          int32_t hkv, int32_t head_dim, int32_t d_c, int32_t oversample, double ridge,
                          int32_t power_iters, const double* omega, float* w_q, float* w_k, void* workspace,
                          size_t ws_bytes, void* stream);
size_t esa_fit_workspace_size(int64_t n_q, int64_t n_k, int32_t hq, int32_t hkv, int32_t head_dim, int32_t d_c,
                              int32_t oversample);

/* ------------------------------------------------------------------- status -- */

/* Message for the last non-OK status returned on this thread ("" if none). */
const char* esa_last_error(void);

/* Waits for `stream`, then reads and clears the device status word of the current
 * device. Returns ESA_OK, ESA_ERR_TIMEOUT if a kernel's bounded wait ran out since the
 * last read (the message names the kernel and the wait), ESA_ERR_CUDA if a kernel
 * stopped early on a launch-environment check (e.g. misaligned shared memory), or
 * ESA_ERR_INVALID_ARG if a variable-length call read a length outside [1, n_cap]. */
esa_status_t esa_device_status(void* stream);

/* esa_wait_selftest - runs the bounded-wait path on demand: one CTA waits on a barrier
 * that nothing arrives at; after limit_ns (1 us .. 2 s) the wait gives up, records
 * ESA_ERR_TIMEOUT at site 9901 in the device status word and the kernel returns, with
 * no fault and no hang. The next esa_device_status() reports it. ESA_ERR_INVALID_ARG for
 * a limit out of range. For tests of the failure path. */
esa_status_t esa_wait_selftest(uint64_t limit_ns, void* stream);

/* Number of kernels this library has launched in this process, all devices and
 * threads together (accounting only). */
uint64_t esa_launch_count(void);

/* Library version string. */
const char* esa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ESA_H_ */
