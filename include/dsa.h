/*
 * dsa.h -- C ABI of a B200 (sm_100a) library for the hot path of DeepSeek
 * Sparse Attention (DSA).
 *
 * The method ("DeepSeek-V3.2-Exp DSA 技术深度解析", section 1; "DeepSeek V4 ...
 * 稀疏注意力" on hotdry, section on the lightning indexer and the fine-grained
 * selector): before the main attention, a light "lightning indexer" with few
 * heads, a low-dimensional FP8 query/key (index_head_dim 128) and ReLU scores
 * every history token of each query token; a top-k selector keeps the k
 * best-scoring KV entries; the main attention then runs over those k entries
 * only, so its cost falls from O(n^2) to O(n k) while the indexer stays O(n^2)
 * with a tiny constant.  Concretely, for query token t and history token s<=t:
 *
 *     I[t,s] = sum_h w[t,h] * ReLU( qI[t,h] . kI[s] )                 (indexer)
 *     S_t    = the min(k, t+1) positions s <= t with the largest I[t,s],
 *              ties broken toward the lower s                          (top-k)
 *     o[t,h] = sum_{j in S_t} softmax_j( sm * q[t,h] . K[j] ) V[j]     (attention)
 *
 * with one shared index-key head, per-head weights w, FP8 E4M3 index query
 * and key values each carrying one fp32 scale per token
 * (qI[t,h,:] = e4m3(q8[t,h,:]) * sq[t], kI[s,:] = e4m3(k8[s,:]) * sk[s]), and
 * one shared K/V head for all query heads (multi-query attention; one index
 * set S_t shared by all query heads of token t).
 *
 * Conventions for every entry point
 *  - Returns dsa_status.  No C++ exception crosses this boundary.
 *  - Tensor pointers are DEVICE memory owned by the caller, dense row-major
 *    in the layouts stated per function, 16-byte aligned.  The library never
 *    keeps a pointer after the call returns and never frees one.
 *  - The library allocates no device memory.  Entry points that need scratch
 *    take a caller workspace of at least dsa_*_workspace_size(...) bytes,
 *    256-byte aligned; its first 256 bytes hold a device status word.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream).  Argument errors are detected on the host and
 *    returned before anything is enqueued.  Errors that only the device can
 *    see (a bounded wait that timed out, a page id out of range) are written
 *    to the workspace status word; read them with dsa_stream_status().
 *  - All sizes are element counts unless stated otherwise.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define DSA_VERSION_MAJOR 0
#define DSA_VERSION_MINOR 1

typedef enum dsa_status {
    DSA_OK = 0,
    DSA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, non-positive k, ... */
    DSA_ERR_UNSUPPORTED = 2,  /* shape or dtype this build has no kernel for */
    DSA_ERR_WORKSPACE = 3,    /* workspace missing or smaller than required */
    DSA_ERR_CUDA = 4,         /* a CUDA runtime call failed (launch, sync, ...) */
    DSA_ERR_TIMEOUT = 5       /* a device-side bounded wait gave up */
} dsa_status;

typedef enum dsa_dtype {
    DSA_F32 = 0,   /* all operands fp32 (no FP8 scales) */
    DSA_BF16 = 1,  /* bf16 values */
    DSA_E4M3 = 2   /* FP8 E4M3 index query/key bytes + fp32 per-token scales; bf16 w, Q, K, V */
} dsa_dtype;

/* Human-readable name of a status code (static storage, never NULL). */
const char *dsa_status_string(dsa_status s);

/* (DSA_VERSION_MAJOR << 16) | DSA_VERSION_MINOR. */
int dsa_version(void);

/*
 * dsa_index_scores -- lightning-indexer scores of a block of query rows
 * (DSA section 1: light indexer, few heads, FP8, ReLU, every history token).
 *
 *   dtype == DSA_E4M3: q_idx uint8 E4M3 [T, H_I, d_I]; q_scale f32 [T];
 *                      k_idx uint8 E4M3 [T, d_I];    k_scale f32 [T];
 *                      w bf16 [T, H_I].  Scales finite and > 0.
 *   dtype == DSA_F32:  q_idx f32 [T, H_I, d_I]; k_idx f32 [T, d_I]; w f32
 *                      [T, H_I]; q_scale and k_scale must be NULL.
 * Writes, for r in [0, q_row_count) and s in [0, t], with t = q_row_begin + r:
 *   scores_out[r * ld_scores + s] = I[t, s] (fp32);
 * and, if fill_upper != 0, -inf for s in (t, T); with fill_upper == 0 the
 * entries above the diagonal are left untouched (saves their bandwidth).
 * Requires 0 <= q_row_begin, q_row_begin + q_row_count <= T, ld_scores >= T.
 * Supported: E4M3 with d_I == 128 and 1 <= H_I <= 128 (H_I <= 64 runs on the
 * tcgen05 tensor-core kernel); F32 with d_I <= 256, H_I <= 64.
 * q_row_count == 0 is a no-op.
 */
dsa_status dsa_index_scores(const void *q_idx, const float *q_scale, const void *k_idx,
                            const float *k_scale, const void *w, int64_t T, int H_I, int d_I,
                            int64_t q_row_begin, int64_t q_row_count, float *scores_out,
                            int64_t ld_scores, int fill_upper, dsa_dtype dtype, void *stream);

/*
 * dsa_topk -- the top-k selector (DSA section 1; the "fine-grained selector"):
 * for each row r (query position t = row_begin + r), the min(k, t+1)
 * positions s in [0, t] with the largest scores[r * ld_scores + s]; equal
 * scores go to the lower s, and +0 equals -0.  Entries past t are not read.
 *   idx_out int32 [row_count, k]: selected positions in ascending order,
 *   padded with -1.  Scores must not be NaN.
 * Bit-exact: the set is unique under the stated order.
 * Requires row_begin + row_count <= T, ld_scores >= T, 1 <= k <= 65536.
 * workspace: at least dsa_topk_workspace_size(row_count, T, k) bytes (may be
 * NULL when that size is 0).
 */
size_t dsa_topk_workspace_size(int64_t row_count, int64_t T, int k);
dsa_status dsa_topk(const float *scores, int64_t ld_scores, int64_t row_begin,
                    int64_t row_count, int64_t T, int k, int32_t *idx_out, void *workspace,
                    size_t ws_bytes, void *stream);

/*
 * dsa_topk_window -- the selector with a sliding window ("DeepSeek-V4 百万
 * token 上下文的工程实现", section on the sliding-window KV cache and the
 * hybrid strategy: the most recent 4K-16K tokens keep their full KV, older
 * tokens are kept only as far as an importance score retains them).  For row
 * r (query position t = row_begin + r, n = t + 1 causal positions) the last
 * `window` positions max(0, n - window) .. t are always selected, and
 * min(k, n - window) of the older positions 0 .. t - window are selected as
 * dsa_topk does (largest score, ties to the lower s, +0 equals -0).
 *   idx_out int32 [row_count, k + window]: the selected older positions
 *   ascending, then the window positions ascending, then -1 padding.
 * window == 0 gives dsa_topk's result.  Requires 0 <= window <= 2^24 and the
 * other constraints of dsa_topk; workspace as dsa_topk.
 */
dsa_status dsa_topk_window(const float *scores, int64_t ld_scores, int64_t row_begin,
                           int64_t row_count, int64_t T, int k, int window, int32_t *idx_out,
                           void *workspace, size_t ws_bytes, void *stream);

/*
 * dsa_sparse_attn -- main attention restricted to the selected KV rows
 * (DSA section 1: the main attention only looks at the selected subset).
 *   q   [T, H_q, d], k and v [T, d] (one shared KV head), out [T, H_q, d]:
 *       all bf16 (dtype DSA_BF16 or DSA_E4M3) or all f32 (DSA_F32).
 *   idx int32 [T, k_sel]: row t lists the KV rows query t attends to; -1
 *       entries are skipped, and so is any entry outside [0, T).
 *   lse_out f32 [T, H_q] (nullable): natural-log log-sum-exp of the scaled
 *       logits sm_scale * q.K over the attended rows (-inf if none).
 *   o[t,h] = sum_j softmax_j(sm_scale * q[t,h].K[j]) V[j]; 0 if no row.
 * Supported: bf16 with d in {64, 128}, H_q <= 128 or a multiple of 128;
 * f32 with d <= 128.
 */
dsa_status dsa_sparse_attn(const void *q, const void *k, const void *v, const int32_t *idx,
                           int64_t T, int H_q, int d, int k_sel, float sm_scale, void *out,
                           float *lse_out, dsa_dtype dtype, void *stream);

/*
 * dsa_prefill -- the whole prefill hot path of one sequence: indexer, top-k
 * and sparse attention for every query token 0..T-1 (layouts as in the
 * three stage functions above; dtype DSA_E4M3 or DSA_F32).
 *   out [T, H_q, d]; lse_out [T, H_q] (nullable); idx_out int32 [T, k_sel]
 *   (nullable: the selection is then kept in the workspace only).
 * With DSA_E4M3 index values, at most 64 index heads and k_sel <= 4096 the
 * selection is fused into the indexer (the pages' indexer -> top-k selector
 * flow, "DeepSeek-V3.2-Exp 稀疏注意力机制(DSA)技术深度解析", section 1; the
 * sider.ai page's point that selection must stay cheap and cache-aware): the
 * causal score matrix is never written.  Query rows go in passes of R rows:
 * the indexer first scores a sample of the keys (one pseudo-random position
 * per 64) to fix a per-row threshold, then scores every key and keeps only
 * the (score, position) pairs at or above it, and an exact select finishes
 * each row from those.  A row whose count of kept pairs is below k_sel or
 * above the list's capacity (4 k_sel, at least 4096) -- for example when
 * many scores tie -- is recomputed by the score epilogue and selected by the
 * stand-alone top-k, so the result is always the exact top-k of the same
 * fp32 scores that dsa_index_scores returns.  Otherwise (f32 inputs, more
 * heads, larger k) the indexer writes row blocks of scores and dsa_topk's
 * kernel selects from them.
 * workspace: at least dsa_prefill_workspace_size(...) bytes; with a smaller
 * one the call returns DSA_ERR_WORKSPACE.  The fused path's size is the
 * selection (T x k_sel indices, unless idx_out is given) plus per-pass
 * scratch of at most 4096 rows and 1 GiB of repair score rows: linear in T.
 * A larger workspace lets a pass take more query rows.
 */
size_t dsa_prefill_workspace_size(int64_t T, int H_I, int d_I, int H_q, int d, int k_sel,
                                  dsa_dtype dtype);
dsa_status dsa_prefill(const void *q_idx, const float *q_scale, const void *k_idx,
                       const float *k_scale, const void *w, const void *q, const void *k,
                       const void *v, int64_t T, int H_I, int d_I, int H_q, int d, int k_sel,
                       float sm_scale, void *out, float *lse_out, int32_t *idx_out,
                       dsa_dtype dtype, void *workspace, size_t ws_bytes, void *stream);

/*
 * dsa_prefill_window -- dsa_prefill with dsa_topk_window's selection: the last
 * `window` positions of every query are always attended, and the indexer's
 * top-k picks k_sel of the older ones.  idx_out is [T, k_sel + window]; the
 * workspace must hold dsa_prefill_workspace_size(T, H_I, d_I, H_q, d,
 * k_sel + window, dtype) bytes.  window == 0 is dsa_prefill.
 */
dsa_status dsa_prefill_window(const void *q_idx, const float *q_scale, const void *k_idx,
                              const float *k_scale, const void *w, const void *q, const void *k,
                              const void *v, int64_t T, int H_I, int d_I, int H_q, int d, int k_sel,
                              int window, float sm_scale, void *out, float *lse_out,
                              int32_t *idx_out, dsa_dtype dtype, void *workspace, size_t ws_bytes,
                              void *stream);

/*
 * dsa_prefill_rows -- the fused prefill of the query rows [row_begin,
 * row_begin + row_count) of a T-token sequence, for a split of one long
 * prefill over devices: each device takes a set of query rows (a causal row
 * costs in proportion to its position, so rows are dealt in a zigzag of 2G
 * chunks, device g taking chunks g and 2G - 1 - g) and needs the key side of
 * every earlier position.  None of the pages describes a multi-device
 * prefill; the hotdry page's million-token setting motivates it.
 *   Query side, row_count rows (row r is position row_begin + r):
 *     q_idx u8 [row_count, H_I, d_I], q_scale f32 [row_count],
 *     w bf16 [row_count, H_I], q bf16 [row_count, H_q, d].
 *   Key side, positions 0..T-1: k_idx u8 [T, d_I], k_scale f32 [T],
 *     k, v bf16 [T, d] (only positions < row_begin + row_count are read).
 *   Outputs for those rows: out [row_count, H_q, d], lse_out [row_count, H_q]
 *     (nullable), idx_out int32 [row_count, k_sel] (nullable: then kept in
 *     the workspace).
 * Row r's results equal, bit for bit, row row_begin + r of dsa_prefill on the
 * whole sequence.  Requires dtype DSA_E4M3, H_I <= 64, k_sel <= 4096 (the
 * fused selection); else DSA_ERR_UNSUPPORTED.  Workspace: at least
 * dsa_prefill_rows_workspace_size(...) bytes (0 when unsupported).
 */
size_t dsa_prefill_rows_workspace_size(int64_t T, int64_t row_count, int H_I, int d_I, int H_q, int d,
                                       int k_sel, dsa_dtype dtype);
dsa_status dsa_prefill_rows(const void *q_idx, const float *q_scale, const void *k_idx, const float *k_scale,
                            const void *w, const void *q, const void *k, const void *v, int64_t T,
                            int64_t row_begin, int64_t row_count, int H_I, int d_I, int H_q, int d, int k_sel,
                            float sm_scale, void *out, float *lse_out, int32_t *idx_out, dsa_dtype dtype,
                            void *workspace, size_t ws_bytes, void *stream);

/*
 * dsa_prefill_host -- dsa_prefill for inputs and outputs in HOST memory
 * (dtype DSA_E4M3 only; layouts as in dsa_prefill).  The pages define the
 * computation; moving it from and to the host is this library's.
 *   q_idx, q_scale, k_idx, k_scale, w, q, k, v: host inputs (page-locked memory
 *     lets the copies overlap the computation; pageable memory still works,
 *     with the copies serialised by the driver);
 *   out, lse_out (nullable), idx_out (nullable): host outputs.
 * The query rows move to the device, and their outputs back, pass by pass on
 * two copy streams of the library's own (created once per device), while the
 * indexer, top-k and attention of the previous pass run on `stream`.  The
 * index keys, their scales, the query scales and the head weights move first,
 * then the first pass's index queries, then K and V; each pass's selection
 * waits only for its index queries, its attention also for its bf16 queries.
 * Passes run from the last rows to the first, the first and the last of them
 * at most 512 rows, so that the computation starts early and little output is
 * left to copy after it.  The call is asynchronous: the outputs are complete
 * once `stream` reaches the point after the call (e.g. cudaStreamSynchronize).
 * Host buffers must stay valid until then.
 * workspace: device memory of at least dsa_prefill_host_workspace_size(...)
 * bytes (device copies of every input and output plus the prefill scratch),
 * 256-byte aligned.  Errors: DSA_ERR_INVALID_ARG (null pointer, bad size),
 * DSA_ERR_UNSUPPORTED (dtype or shape), DSA_ERR_WORKSPACE, DSA_ERR_CUDA.
 */
size_t dsa_prefill_host_workspace_size(int64_t T, int H_I, int d_I, int H_q, int d, int k_sel,
                                       dsa_dtype dtype);
dsa_status dsa_prefill_host(const void *q_idx, const float *q_scale, const void *k_idx,
                            const float *k_scale, const void *w, const void *q, const void *k,
                            const void *v, int64_t T, int H_I, int d_I, int H_q, int d, int k_sel,
                            float sm_scale, void *out, float *lse_out, int32_t *idx_out,
                            dsa_dtype dtype, void *workspace, size_t ws_bytes, void *stream);

/*
 * dsa_decode -- one decode step of B sequences against paged caches (the
 * current token is already appended; DSA on the decode path, plus the FP8
 * index-key cache).
 *   q_idx  uint8 E4M3 [B, H_I, d_I]; q_scale f32 [B]; w bf16 [B, H_I];
 *   q      bf16 [B, H_q, d];
 *   kidx_cache   uint8 E4M3 [num_pages, page_size, d_I];
 *   kscale_cache f32 [num_pages, page_size];
 *   k_cache, v_cache bf16 [num_pages, page_size, d];
 *   block_table  int32 [B, max_pages_per_seq]: physical page of each logical
 *                page (position s of sequence b is in page
 *                block_table[b, s / page_size], slot s % page_size);
 *   context_lens int32 [B]: tokens cached per sequence, current one included;
 *                each in [1, max_context] and <= max_pages_per_seq*page_size.
 * Outputs: out bf16 [B, H_q, d]; lse_out f32 [B, H_q] (nullable); idx_out
 * int32 [B, k_sel] (nullable): selected positions ascending, -1 padded.
 * A page id outside [0, num_pages) or a context length out of range is
 * reported as DSA_ERR_INVALID_ARG through dsa_stream_status (the offending
 * rows are skipped, nothing is read out of bounds).
 * Supported: d_I == 128, H_I <= 64 and a multiple of 8, d == 128,
 * page_size a multiple of 16, H_q <= 128 or a multiple of 128.
 */
size_t dsa_decode_workspace_size(int B, int64_t max_context, int H_q, int d, int k_sel);
dsa_status dsa_decode(const void *q_idx, const float *q_scale, const void *w, const void *q,
                      const void *kidx_cache, const float *kscale_cache, const void *k_cache,
                      const void *v_cache, const int32_t *block_table,
                      const int32_t *context_lens, int64_t num_pages, int max_pages_per_seq,
                      int page_size, int B, int64_t max_context, int H_I, int d_I, int H_q,
                      int d, int k_sel, float sm_scale, void *out, float *lse_out,
                      int32_t *idx_out, void *workspace, size_t ws_bytes, void *stream);

/*
 * dsa_decode_window -- dsa_decode with dsa_topk_window's selection (the last
 * `window` cached positions of each sequence are always attended; the top-k
 * picks k_sel of the older ones).  idx_out is [B, k_sel + window]; the
 * workspace must hold dsa_decode_workspace_size(B, max_context, H_q, d,
 * k_sel + window) bytes.  window == 0 is dsa_decode.
 */
dsa_status dsa_decode_window(const void *q_idx, const float *q_scale, const void *w, const void *q,
                             const void *kidx_cache, const float *kscale_cache, const void *k_cache,
                             const void *v_cache, const int32_t *block_table,
                             const int32_t *context_lens, int64_t num_pages, int max_pages_per_seq,
                             int page_size, int B, int64_t max_context, int H_I, int d_I, int H_q,
                             int d, int k_sel, int window, float sm_scale, void *out, float *lse_out,
                             int32_t *idx_out, void *workspace, size_t ws_bytes, void *stream);

/*
 * dsa_decode_kv8 -- dsa_decode_window over FP8 K/V caches (the DeepSeek-V4
 * engineering page's FP8 decoding section: the KV cache moves from 16-bit to
 * FP8, halving its memory and the bytes each decode step gathers).
 *   k_cache, v_cache uint8 E4M3 [num_pages, page_size, d] (16-byte aligned);
 *   k_cache_scale, v_cache_scale f32 [num_pages, page_size]: the attention
 *   uses Khat[s] = e4m3(k_cache[s]) * k_cache_scale[s] and likewise V
 *   (dsa_cache_append_kv8 writes this layout).
 * Every other argument, the result and the workspace are those of
 * dsa_decode_window (window 0: no window).  Supported as dsa_decode, with
 * H_q a multiple of 128 and d == 128 (else DSA_ERR_UNSUPPORTED).  The
 * attention widens the gathered codes to bf16 times their scale (one
 * rounding) before the tensor-core products.
 */
dsa_status dsa_decode_kv8(const void *q_idx, const float *q_scale, const void *w, const void *q,
                          const void *kidx_cache, const float *kscale_cache, const void *k_cache,
                          const float *k_cache_scale, const void *v_cache, const float *v_cache_scale,
                          const int32_t *block_table, const int32_t *context_lens, int64_t num_pages,
                          int max_pages_per_seq, int page_size, int B, int64_t max_context, int H_I,
                          int d_I, int H_q, int d, int k_sel, int window, float sm_scale, void *out,
                          float *lse_out, int32_t *idx_out, void *workspace, size_t ws_bytes, void *stream);

/*
 * Decode of one context split over G devices.  The pages' decode step
 * (indexer, top-k, attention over the selected rows; the 1M-context setting of
 * "DeepSeek V4 ... 稀疏注意力" on hotdry) is computed exactly when the cached
 * positions of every sequence are cut into G contiguous shards, shard g
 * holding positions [pos_base_g[b], pos_base_g[b] + context_lens_g[b]) in its
 * own paged caches at local positions 0.. context_lens_g[b]-1, shards in
 * position order:
 *   1. dsa_decode_select on every shard: its indexer scores and its own top-k
 *      (k_sel) as GLOBAL positions with their scores.  Every member of the
 *      global top-k is in its shard's top-k, so the union holds it.
 *   2. the G candidate lists are gathered (an all-gather of G*B*k_sel*8 bytes)
 *      into cand_pos [G, B, k_sel] / cand_score [G, B, k_sel], shard order.
 *   3. dsa_merge_selections on every device: the exact top-k of the union,
 *      ties toward the lower position -- the selection dsa_decode makes over
 *      the whole context, bit for bit.
 *   4. dsa_decode_attend on every shard: attention over the selected positions
 *      that shard holds, giving a partial bf16 output and its log-sum-exp
 *      (-inf and zeros when the shard holds none of them).
 *   5. the G partials are gathered into [G, B, H_q, d] / [G, B, H_q] and
 *      dsa_merge_partials combines them:
 *        lse = log sum_g exp(lse_g),  out = sum_g exp(lse_g - lse) * out_g.
 * Every shard must hold at least one position of every sequence
 * (context_lens_g[b] >= 1); a zero length is reported as DSA_ERR_INVALID_ARG
 * through dsa_stream_status, as in dsa_decode.
 * One workspace of dsa_split_workspace_size(G, B, max_context, H_q, d, k_sel)
 * bytes (max_context: the largest shard length) serves all four calls.
 */
size_t dsa_split_workspace_size(int G, int B, int64_t max_context, int H_q, int d, int k_sel);

/*
 * dsa_decode_select -- step 1 on one shard.  Inputs as dsa_decode's indexer
 * half (q_idx, q_scale, w, kidx_cache, kscale_cache, block_table,
 * context_lens, ... with the shard's local lengths, max_context the largest);
 * pos_base int32 [B]: the global position of each sequence's first position
 * on this shard.  Outputs cand_pos_out int32 [B, k_sel]: the shard's top-k as
 * global positions, ascending, -1 padded; cand_score_out f32 [B, k_sel]:
 * their indexer scores (-inf for -1).  A negative base or a global position
 * past INT32_MAX is reported through dsa_stream_status.  Supported as
 * dsa_decode.
 */
dsa_status dsa_decode_select(const void *q_idx, const float *q_scale, const void *w, const void *kidx_cache,
                             const float *kscale_cache, const int32_t *block_table, const int32_t *context_lens,
                             const int32_t *pos_base, int64_t num_pages, int max_pages_per_seq, int page_size,
                             int B, int64_t max_context, int H_I, int d_I, int k_sel, int32_t *cand_pos_out,
                             float *cand_score_out, void *workspace, size_t ws_bytes, void *stream);

/*
 * dsa_merge_selections -- step 3.  G candidate lists as dsa_decode_select
 * wrote them, list g from shard g: positions int32 [B, k_sel] at
 * cand_pos + g * list_stride and scores f32 [B, k_sel] at
 * cand_score + g * list_stride (elements; 0 means B * k_sel, i.e. dense
 * [G, B, k_sel] arrays).  A stride lets one all-gathered buffer of
 * [G][positions | scores] serve both.  idx_out int32 [B, k_sel]: the k_sel
 * best positions of the union (score descending, ties to the lower
 * position), ascending, -1 padded.  Entries with position -1 never win.
 */
dsa_status dsa_merge_selections(const int32_t *cand_pos, const float *cand_score, int64_t list_stride, int G,
                                int B, int k_sel, int32_t *idx_out, void *workspace, size_t ws_bytes, void *stream);

/*
 * dsa_decode_attend -- step 4 on one shard.  q bf16 [B, H_q, d]; the shard's
 * caches, block_table, context_lens and pos_base as in dsa_decode_select;
 * k_cache_scale / v_cache_scale NULL for bf16 K/V, or both given for FP8
 * E4M3 K/V as in dsa_decode_kv8; idx int32 [B, k_sel]: the merged global
 * selection.  Positions outside this shard are skipped.  Outputs out bf16
 * [B, H_q, d] and lse_out f32 [B, H_q] (required): the attention over this
 * shard's part of the selection.  Supported as dsa_decode (FP8: as
 * dsa_decode_kv8).
 */
dsa_status dsa_decode_attend(const void *q, const void *k_cache, const float *k_cache_scale, const void *v_cache,
                             const float *v_cache_scale, const int32_t *block_table, const int32_t *context_lens,
                             const int32_t *pos_base, int64_t num_pages, int max_pages_per_seq, int page_size, int B,
                             int H_q, int d, int k_sel, const int32_t *idx, float sm_scale, void *out,
                             float *lse_out, void *workspace, size_t ws_bytes, void *stream);

/*
 * dsa_merge_partials -- step 5.  Partial g: out bf16 [B, H_q, d] at
 * part_out + g * out_stride and lse f32 [B, H_q] at part_lse + g * lse_stride
 * (elements of each type; 0 means dense [G, B, H_q, d] / [G, B, H_q]; a stride
 * lets one all-gathered buffer of [G][out | lse] serve both; out_stride a
 * multiple of 8).  out bf16 [B, H_q, d], lse_out f32 [B, H_q] (nullable).  A
 * head whose every partial has lse -inf gets zeros and -inf.  d == 128.
 * Needs no workspace; device errors are CUDA launch errors only.
 */
dsa_status dsa_merge_partials(const void *part_out, int64_t out_stride, const float *part_lse, int64_t lse_stride,
                              int G, int B, int H_q, int d, void *out, float *lse_out, void *stream);

/*
 * dsa_quantize_e4m3 -- FP8 E4M3 quantisation with one fp32 scale per row, the
 * storage of the indexer's query and key ("DeepSeek-V3.2-Exp DSA 技术深度解析",
 * section 1: FP8 indexer; the DeepSeek-V4 engineering page's FP8 decoding
 * section).  For each row r of x [rows, cols] (bf16 or fp32, x_dtype DSA_BF16
 * or DSA_F32):
 *   scale_out[r] = amax_r / 448 (fp32 division; 1 when that is 0), where
 *                  amax_r = max_j |x[r, j]|;
 *   codes_out[r, j] = the E4M3 value nearest to x[r, j] / scale_out[r] (fp32
 *                  division), ties to the even code, magnitudes past 448
 *                  saturating to +-448 (OCP E4M3FN bytes).
 * For the indexer query pass x = q_I viewed as [T, H_I * d_I] (one scale per
 * token over all heads); for the key x = k_I [T, d_I].
 * x: device, 16-byte aligned; codes_out uint8 [rows, cols], 8-byte aligned;
 * scale_out f32 [rows].  cols a multiple of 8, at most 16384 (else
 * DSA_ERR_UNSUPPORTED).  x must be finite (a NaN or infinity makes its row's
 * scale and codes meaningless).  rows == 0 is a no-op.
 */
dsa_status dsa_quantize_e4m3(const void *x, dsa_dtype x_dtype, int64_t rows, int64_t cols,
                             uint8_t *codes_out, float *scale_out, void *stream);

/*
 * dsa_cache_append -- writes N new tokens into the paged decode caches (the
 * step before dsa_decode in every decode step: the current token is appended,
 * then attended).  Token i belongs to sequence seq_ids[i] at position
 * positions[i], i.e. physical page block_table[seq_ids[i], positions[i] /
 * page_size], slot positions[i] % page_size.  Its index key kidx_new[i, :]
 * (bf16 or fp32 [N, d_I], kidx_dtype DSA_BF16 or DSA_F32) is quantised as by
 * dsa_quantize_e4m3 into kidx_cache [num_pages, page_size, d_I] (uint8) and
 * kscale_cache [num_pages, page_size] (f32); its K and V rows k_new, v_new
 * (bf16 [N, d]) are copied into k_cache, v_cache (bf16 [num_pages,
 * page_size, d]).  Tokens must address distinct slots.
 * A token whose sequence is outside [0, B), whose position is outside
 * [0, max_pages_per_seq * page_size) or whose page id is outside
 * [0, num_pages) is skipped, and DSA_ERR_INVALID_ARG is written to *status
 * (a device uint32_t the caller zeroes beforehand; nullable) unless it
 * already holds an error.  Supported: d_I a multiple of 8 up to 256, d a
 * multiple of 8.  kidx_new, k_new, v_new, k_cache, v_cache 16-byte aligned,
 * kidx_cache 8-byte aligned.  N == 0 is a no-op.
 */
dsa_status dsa_cache_append(const void *kidx_new, dsa_dtype kidx_dtype, const void *k_new,
                            const void *v_new, const int32_t *seq_ids, const int32_t *positions,
                            int64_t N, int B, const int32_t *block_table, int max_pages_per_seq,
                            int64_t num_pages, int page_size, int d_I, int d, void *kidx_cache,
                            float *kscale_cache, void *k_cache, void *v_cache, uint32_t *status,
                            void *stream);

/*
 * dsa_cache_append_kv8 -- dsa_cache_append for FP8 K/V caches: each new
 * token's index key, K row and V row are each quantised as by
 * dsa_quantize_e4m3 (one scale per row) into kidx_cache/kscale_cache,
 * k_cache/k_cache_scale and v_cache/v_cache_scale (uint8 [num_pages,
 * page_size, d] and f32 [num_pages, page_size]).  k_new, v_new bf16 [N, d].
 * Supported: d_I and d multiples of 8 up to 256.  kidx_new, k_new, v_new
 * 16-byte aligned; the code caches 8-byte aligned.  Errors and out-of-range
 * tokens as dsa_cache_append.
 */
dsa_status dsa_cache_append_kv8(const void *kidx_new, dsa_dtype kidx_dtype, const void *k_new,
                                const void *v_new, const int32_t *seq_ids, const int32_t *positions,
                                int64_t N, int B, const int32_t *block_table, int max_pages_per_seq,
                                int64_t num_pages, int page_size, int d_I, int d, void *kidx_cache,
                                float *kscale_cache, void *k_cache, float *k_cache_scale, void *v_cache,
                                float *v_cache_scale, uint32_t *status, void *stream);

/*
 * dsa_decode_noalloc -- dsa_decode without a caller workspace.  The paper has
 * no counterpart: this entry point exists for callers that cannot allocate
 * device memory for the library -- for example a plugin whose host process
 * has reserved all device memory in its own pool, or code on a
 * latency-critical path where a device allocation (which can synchronise the
 * device) is not allowed.  It calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *
 * Arguments and results are those of dsa_decode, minus workspace/ws_bytes,
 * plus status_out: nullable DEVICE pointer to one uint32_t that receives the
 * step's device status word (a dsa_status) on `stream` after the step.
 *
 * The scratch is a fixed device array of DSA_DECODE_NOALLOC_SCRATCH_BYTES
 * (64 MiB) inside the library.  CUDA loads the library's device code lazily,
 * so that array is reserved on a device by the FIRST call on that device
 * (when the call looks up the array's device address with the device
 * current); the reservation then lasts as long as the device's context.
 * That first call can therefore fail with DSA_ERR_CUDA when the device has no
 * 64 MiB left, and may synchronise the device: make it early, as a warm-up,
 * before filling a memory pool or starting a stream capture.  Later calls on
 * the same context reserve nothing.  A device reset (or a released and
 * recreated primary context) loads the code again; the next call notices the
 * new context and looks the address up again (that call reserves again).
 * A problem whose dsa_decode_workspace_size() exceeds the array is rejected
 * with DSA_ERR_WORKSPACE before any launch (64 sequences x 64K context x
 * k 2048 x 128 heads needs about 33 MiB).
 * Every call on a device shares the one array and leaves its contents behind
 * (the status word is cleared at the start of each call): calls whose GPU
 * work overlaps -- on different streams, or from different host threads --
 * race and must be serialised by the caller.
 */
#define DSA_DECODE_NOALLOC_SCRATCH_BYTES (64u << 20)
dsa_status dsa_decode_noalloc(const void *q_idx, const float *q_scale, const void *w, const void *q,
                              const void *kidx_cache, const float *kscale_cache,
                              const void *k_cache, const void *v_cache,
                              const int32_t *block_table, const int32_t *context_lens,
                              int64_t num_pages, int max_pages_per_seq, int page_size, int B,
                              int64_t max_context, int H_I, int d_I, int H_q, int d, int k_sel,
                              float sm_scale, void *out, float *lse_out, int32_t *idx_out,
                              uint32_t *status_out, void *stream);

/*
 * Stage timing -- a tracing aid with no counterpart on the pages.  While
 * enabled (process-wide), dsa_prefill and dsa_prefill_host record a pair of
 * CUDA events on their stream around each stage's launches; the events are
 * timed on the device, so enabling this does not synchronise the stream.
 * dsa_profile_read waits for the recorded events, adds each stage's elapsed
 * milliseconds into ms_out[stage] and the number of times the stage ran into
 * launches_out[stage] (nullable), both arrays of DSA_STAGE_COUNT entries
 * (the caller zeroes them), and forgets the records.  Do not enable it
 * around a stream capture.  The events belong to
 * the device that was current when they were recorded.
 * Stages: the fused selection's sample scores, thresholds, select epilogue,
 * finish and repair; the stand-alone indexer and top-k of the unfused
 * prefill; the sparse attention.
 */
typedef enum dsa_stage {
    DSA_STAGE_SAMPLE = 0,
    DSA_STAGE_TAU = 1,
    DSA_STAGE_SELECT = 2,
    DSA_STAGE_FINISH = 3,
    DSA_STAGE_REPAIR = 4,
    DSA_STAGE_SCORES = 5,
    DSA_STAGE_TOPK = 6,
    DSA_STAGE_ATTN = 7,
    DSA_STAGE_COUNT = 8
} dsa_stage;
dsa_status dsa_profile_enable(int on);
dsa_status dsa_profile_read(double *ms_out, int64_t *launches_out);

/*
 * dsa_test_stall_next -- a test hook for the device-side bounded waits (no
 * counterpart on the pages; off by default).  It arms a one-shot fault on the
 * host side: the next launch of the named tcgen05 indexer (the prefill one,
 * inside dsa_prefill / dsa_index_scores, or the decode one, inside
 * dsa_decode) has its producer warp in CTA 0 stop early (before its second
 * query copy in the prefill indexer, before its first copy in the decode
 * one), so the CTA's consumer waits for data that never comes.  That wait gives up
 * after its limit (2 s); the CTA records DSA_ERR_TIMEOUT in the workspace
 * status word, lets the copies and MMAs it did issue land, frees its tensor
 * memory and returns; the other CTAs finish normally, and the context stays
 * usable (the call's outputs are then incomplete).  DSA_STALL_NONE disarms.
 * Process-wide; not for production use.
 */
typedef enum dsa_stall_target {
    DSA_STALL_NONE = 0,
    DSA_STALL_PREFILL_INDEXER = 1,
    DSA_STALL_DECODE_INDEXER = 2
} dsa_stall_target;
dsa_status dsa_test_stall_next(dsa_stall_target target);

/*
 * dsa_stream_status -- waits for `stream`, then returns the device status
 * word of `workspace` (DSA_OK if no device-side error was recorded by the
 * last call that used this workspace) and resets it to DSA_OK.
 * Returns DSA_ERR_CUDA if the synchronisation itself fails.
 */
dsa_status dsa_stream_status(void *workspace, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
