// Internal launchers of the DSA library.  Each returns cudaGetLastError()
// of its launches; shapes were validated by the C entry points.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "dsa_common.cuh"

namespace dsa {

// ---- test hook (api.cu): true once after dsa_test_stall_next armed `target`
// (0: the prefill indexer, 1: the decode indexer); that launch leaves one copy
// unissued so that a bounded wait runs out.
bool consume_test_stall(int target);

// ---- indexer (index.cu, index_tc.cu) ----
// Scores of rows [row_begin, row_begin+row_count) into out[(t-row_begin)*ld + s].
// write_upper: also write -inf for s in (t, T).
cudaError_t launch_index_fp8(const uint8_t *q8, const float *sq, const uint8_t *k8,
                             const float *sk, const uint16_t *w, int64_t T, int H,
                             int64_t row_begin, int64_t row_count, float *out, int64_t ld,
                             bool write_upper, cudaStream_t st);
bool index_tc_supported(int H);
// Epilogue modes of the tcgen05 indexer (index_tc.cu).
enum IndexTcMode { IT_SCORES = 0, IT_SAMPLE = 1, IT_SELECT = 2 };
constexpr int kCandCntStride = 32;      // uint32 words per candidate counter (one per 128 bytes)
struct IndexTcOpts {
    int mode = IT_SCORES;
    int64_t nkeys = 0;                  // keys of k8/sk (0: T); the sample count in IT_SAMPLE
    int window = 0;                     // IT_SAMPLE, IT_SELECT: competing positions [0, t + 1 - window)
    int sample_stride = 0;              // IT_SAMPLE: S (a power of two; see sample_pos)
    const float *tau = nullptr;         // IT_SELECT: [row_count] thresholds
    uint2 *cand = nullptr;              // IT_SELECT: [row_count][cap] (score bits, position)
    uint32_t *cand_cnt = nullptr;       // IT_SELECT: [row_count * kCandCntStride], zero before
    int cap = 0;
    const uint32_t *rb_mask = nullptr;  // IT_SCORES: visit only row blocks (128 rows) flagged here
    const uint32_t *any = nullptr;      // IT_SCORES: do nothing when *any == 0
    int64_t q_base = 0;                 // q8, sq and w hold positions [q_base, q_base + q_rows)
    int64_t q_rows = 0;                 // 0: T - q_base
};
// IT_SCORES writes out[(t-row_begin)*ld + s] for s <= t; IT_SAMPLE writes
// out[(t-row_begin)*ld + j] for the samples j before the row's window (k8/sk
// are the gathered samples); IT_SELECT appends candidates, out unused.
cudaError_t launch_index_tc(const uint8_t *q8, const float *sq, const uint8_t *k8, const float *sk,
                            const uint16_t *w, int64_t T, int H, int64_t row_begin,
                            int64_t row_count, float *out, int64_t ld, bool write_upper,
                            WsHeader *hdr, cudaStream_t st, const IndexTcOpts *opts = nullptr);
cudaError_t launch_index_f32(const float *q, const float *k, const float *w, int64_t T, int H,
                             int D, int64_t row_begin, int64_t row_count, float *out,
                             int64_t ld, bool write_upper, cudaStream_t st);

// ---- top-k (topk.cu) ----
// Row r: candidates scores[r*ld + s] for s < n_r, where n_r = lens[r] if
// lens != nullptr, else row_begin + r + 1.  Output idx[r*(k+window) ...]
// ascending, -1 padded.  With window > 0 only s < n_r - window compete and
// the window positions follow the selected ones.  Rows with lens[r] outside
// [1, max_len] are skipped (set to -1) and reported in hdr.
cudaError_t launch_topk_rows(const float *scores, int64_t ld, int64_t row_begin,
                             const int32_t *lens, int64_t max_len, int64_t row_count, int k,
                             int32_t *idx, WsHeader *hdr, cudaStream_t st, int window = 0);
// The rows list[0, *count) of a pass of `rows` rows (row r is position
// row_begin + r, its scores at scores[r * ld], its output at idx[r * (k + window)]).
cudaError_t launch_topk_rows_list(const float *scores, int64_t ld, int64_t row_begin, int64_t rows, int k,
                                  int32_t *idx, cudaStream_t st, int window, const uint32_t *list,
                                  const uint32_t *count);

// Rows of lengths lens[r] (decode): each row split over CTAs of 16384
// positions that share a sampled threshold and collect their candidates, then
// one CTA per row finishes the exact select.  Scratch of
// topk_split_ws_bytes(rows, max_len) at ws_base.
size_t topk_split_ws_bytes(int64_t rows, int64_t max_len);
cudaError_t launch_topk_split(const float *scores, int64_t ld, const int32_t *lens, int64_t max_len,
                              int64_t rows, int k, int32_t *idx, void *ws_base, WsHeader *hdr,
                              cudaStream_t st, int window = 0);

// ---- fused prefill selection (index_tc.cu, topk.cu) ----
// Gathers the M = sample_count(T, S) sampled index keys and their scales.
cudaError_t launch_gather_samples(const uint8_t *k8, const float *sk, int64_t M, int S, uint8_t *ks,
                                  float *sks, cudaStream_t st);
// Per row of the pass: tau from the sample scores ss[r * ld + j], the
// candidate counter zeroed, the repair state (rb_fail, *fail_cnt) cleared.
cudaError_t launch_prefill_tau(const float *ss, int64_t ld, int64_t row_begin, int64_t rows, int k, int window,
                               int S, int cap, float *tau, uint32_t *cnt, uint32_t *rb_fail, uint32_t *fail_cnt,
                               cudaStream_t st);
// Per row: the exact selection from its candidates into idx[r * (k + window)],
// or the row listed for repair (fail_list[*fail_cnt++], rb_fail per 128 rows).
size_t prefill_finish_smem(int cap);
cudaError_t launch_prefill_finish(const uint2 *cand, int cap, const uint32_t *cnt, int64_t row_begin, int64_t rows,
                                  int k, int window, int32_t *idx, uint32_t *rb_fail, uint32_t *fail_cnt,
                                  uint32_t *fail_list, cudaStream_t st);

// ---- FP8 quantisation and cache append (quant.cu) ----
// codes[r, :] / scale[r] of x[r, 0..cols) (bf16 or fp32), one scale per row;
// cols a multiple of 8 and at most 16384, x 16-byte and codes 8-byte aligned.
cudaError_t launch_quantize_e4m3(const void *x, bool bf16_in, int64_t rows, int cols, uint8_t *codes,
                                 float *scale, cudaStream_t st);
// Token i -> sequence seq[i], position pos[i] of the paged caches: quantised
// index key (d_I <= 256, a multiple of 8), bf16 K and V rows (d a multiple
// of 8) -- or, when k_cache_scale is given, K and V rows quantised to E4M3
// with one scale each (d <= 256).  Out-of-range tokens are skipped and
// DSA_ERR_INVALID_ARG is recorded in *status (nullable).
cudaError_t launch_cache_append(const void *kidx_new, bool bf16_in, const uint16_t *k_new,
                                const uint16_t *v_new, const int32_t *seq, const int32_t *pos, int64_t N,
                                int B, const int32_t *bt, int max_pages, int64_t num_pages, int ps,
                                int d_I, int d, uint8_t *kidx_cache, float *kscale_cache,
                                void *k_cache, void *v_cache, float *k_cache_scale, float *v_cache_scale,
                                uint32_t *status, cudaStream_t st);

// ---- sparse attention (sparse_attn.cu) ----
struct PagedKV {
    const uint16_t *k_cache;     // [num_pages, page_size, d]
    const uint16_t *v_cache;
    const int32_t *block_table;  // [B, max_pages]
    const int32_t *context_lens; // [B]
    int64_t num_pages;
    int max_pages;
    int page_size;
};
// Contiguous K/V [T, d]; one query row per idx row; bf16.
cudaError_t launch_sparse_attn_bf16(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                    const int32_t *idx, int64_t rows, int64_t T, int H, int d,
                                    int ksel, float sm_scale, uint16_t *out, float *lse,
                                    cudaStream_t st);
// Paged K/V, one query row per sequence, split over `splits` chunks of the
// index list; partials in `part` (see sparse_attn.cu for the layout).
cudaError_t launch_sparse_attn_paged_bf16(const uint16_t *q, const PagedKV &kv,
                                          const int32_t *idx, int B, int H, int d, int ksel,
                                          float sm_scale, uint16_t *out, float *lse,
                                          float *part, int splits, WsHeader *hdr,
                                          cudaStream_t st);
size_t sparse_attn_paged_part_bytes(int B, int H, int d, int splits);
cudaError_t launch_merge_splits(const float *part, int rows, int splits, int H, int d, uint16_t *out,
                               float *lse, cudaStream_t st);
int sparse_attn_paged_splits(int B, int ksel);
cudaError_t launch_sparse_attn_f32(const float *q, const float *k, const float *v,
                                   const int32_t *idx, int64_t T, int H, int d, int ksel,
                                   float sm_scale, float *out, float *lse, cudaStream_t st);

// tcgen05 attention (sparse_attn_tc.cu): H a multiple of 128, d == 128.
// Contiguous K/V when block_table is null (positions < T), else paged.
// chained: launched so that it may start while the kernel before it on the
// stream finishes (it waits for that kernel before reading idx).
bool sparse_attn_tc_supported(int H, int d);
cudaError_t launch_sparse_attn_tc(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                  int64_t kv_rows, int64_t T, const int32_t *block_table,
                                  const int32_t *context_lens, int64_t num_pages, int max_pages,
                                  int page_size, const int32_t *idx, int64_t rows, int H, int d,
                                  int ksel, float sm_scale, uint16_t *out, float *lse, float *part,
                                  int splits, WsHeader *hdr, cudaStream_t st, bool chained = false);

// The same over paged FP8 E4M3 K/V caches with one fp32 scale per cached row
// (k8/v8 [num_pages * page_size, d], ks/vs [num_pages * page_size]).
cudaError_t launch_sparse_attn_tc_kv8(const uint16_t *q, const uint8_t *k8, const float *ks, const uint8_t *v8,
                                      const float *vs, int64_t kv_rows, const int32_t *block_table,
                                      const int32_t *context_lens, int64_t num_pages, int max_pages,
                                      int page_size, const int32_t *idx, int64_t rows, int H, int d, int ksel,
                                      float sm_scale, uint16_t *out, float *lse, float *part, int splits,
                                      WsHeader *hdr, cudaStream_t st, bool chained = false);

// ---- decode indexer (decode_tc.cu: tcgen05 + TMA; decode.cu: mma.sync) ----
bool decode_index_tc_supported(int H, int page_size);
cudaError_t launch_decode_index_tc(const uint8_t *q8, const float *sq, const uint16_t *w,
                                   const uint8_t *kidx, const float *kscale,
                                   const int32_t *block_table, const int32_t *context_lens,
                                   int64_t num_pages, int max_pages, int page_size, int B,
                                   int64_t max_context, int H, float *scores, int64_t ld,
                                   WsHeader *hdr, cudaStream_t st);
cudaError_t launch_decode_index(const uint8_t *q8, const float *sq, const uint16_t *w,
                                const uint8_t *kidx, const float *kscale,
                                const int32_t *block_table, const int32_t *context_lens,
                                int64_t num_pages, int max_pages, int page_size, int B,
                                int64_t max_context, int H, float *scores, int64_t ld,
                                WsHeader *hdr, cudaStream_t st);

// ---- context split over devices (split.cu) ----
// Shard-local selections [B, k] -> global positions (+ base[b]) and their scores.
cudaError_t launch_gather_selected(const float *scores, int64_t ld, const int32_t *idx_local, const int32_t *base,
                                   int B, int k, int32_t *idx_out, float *score_out, WsHeader *hdr,
                                   cudaStream_t st);
// Exact top-k of the union of G candidate lists [B, k] (list g at g * stride
// elements; positions ascending within a list, lists in position order),
// positions out [B, k].
size_t merge_selections_ws_bytes(int B, int G, int k);
cudaError_t launch_merge_selections(const int32_t *cand_pos, const float *cand_score, int64_t stride, int B, int G,
                                    int k, int32_t *idx_out, void *ws, WsHeader *hdr, cudaStream_t st);
// Global positions -> this shard's positions [base[b], base[b] + lens[b]) - base[b], else -1.
cudaError_t launch_local_idx(const int32_t *idx, const int32_t *base, const int32_t *lens, int B, int k,
                             int32_t *idx_local, cudaStream_t st);
// Log-sum-exp merge of G partial attentions (bf16 [B, H, d] and f32 [B, H]
// each, partial g at g * out_stride / g * lse_stride elements); d == 128.
cudaError_t launch_merge_partials(const uint16_t *part_out, int64_t out_stride, const float *part_lse,
                                  int64_t lse_stride, int G, int B, int H, int d, uint16_t *out, float *lse,
                                  cudaStream_t st);

}  // namespace dsa
