// Top-k selector ("DeepSeek-V3.2-Exp DSA 技术深度解析", section 1: keep only
// the k best-scoring KV per query token; the hotdry page's "fine-grained
// selector").  Exact: the min(k, n) largest scores of a row, ties toward the
// lower position, emitted in ascending position order.
//
// One CTA per row.  The fp32 scores are mapped to order-preserving uint32
// keys (-0 folded onto +0) and the k-th largest key is found by a three-pass
// radix select (11 + 11 + 10 bits) with shared-memory histograms; the pass
// after the first only counts keys that share the digits found so far.  A
// final pass streams the row in position order and keeps every key above the
// threshold plus the first `need` keys equal to it; one packed block scan per
// 4096 positions gives each kept position its output slot, so the output is
// ascending by construction and needs no sort.
#include "kernels.h"

namespace dsa {
namespace {

constexpr int TK_THREADS = 512;
constexpr int TK_WARPS = TK_THREADS / 32;
constexpr int TK_ITEMS = 8;           // consecutive positions per thread in the output pass

// Exclusive block-wide prefix sum of `v`; returns the exclusive prefix and
// writes the block total to *total.  All threads must call it.
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *warp_buf, uint32_t *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_buf[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t s = lane < TK_WARPS ? warp_buf[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < TK_WARPS) warp_buf[lane] = s;    // inclusive warp-total prefix
    }
    __syncthreads();
    uint32_t before = (warp > 0 ? warp_buf[warp - 1] : 0u) + x - v;
    *total = warp_buf[TK_WARPS - 1];
    __syncthreads();
    return before;
}

__global__ void __launch_bounds__(TK_THREADS)
topk_rows_kernel(const float *__restrict__ scores, int64_t ld, int64_t row_begin,
                 const int32_t *__restrict__ lens, int64_t max_len, int k,
                 int32_t *__restrict__ idx, WsHeader *hdr)
{
    __shared__ uint32_t hist[2048];
    __shared__ uint32_t warp_buf[32];
    __shared__ uint32_t sh_bin, sh_above;

    const int64_t r = blockIdx.x;
    const int tid = threadIdx.x;
    const float *row = scores + r * ld;
    int32_t *out = idx + r * (int64_t)k;
    int64_t n;
    if (lens) {
        n = lens[r];
        if (n < 1 || n > max_len) {
            if (tid == 0) record_error(hdr, DSA_ERR_INVALID_ARG, (unsigned)r);
            for (int i = tid; i < k; i += TK_THREADS) out[i] = -1;
            return;
        }
    } else {
        n = row_begin + r + 1;
    }
    if (n <= k) {
        for (int i = tid; i < k; i += TK_THREADS) out[i] = i < n ? i : -1;
        return;
    }

    // ---- radix select of the k-th largest key ----
    uint32_t prefix = 0, pmask = 0, remaining = (uint32_t)k;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int width = pass == 2 ? 10 : 11;
        const int nb = 1 << width;
        const uint32_t bmask = (uint32_t)nb - 1u;
        for (int i = tid; i < nb; i += TK_THREADS) hist[i] = 0u;
        __syncthreads();
        for (int64_t s = tid; s < n; s += TK_THREADS) {
            uint32_t key = float_key(row[s]);
            if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & bmask], 1u);
        }
        __syncthreads();
        // suffix counts from the top bin down: thread i owns reverse positions [i*bpt, (i+1)*bpt)
        const int bpt = nb / TK_THREADS;
        uint32_t local = 0;
        for (int j = 0; j < bpt; ++j) local += hist[nb - 1 - (tid * bpt + j)];
        uint32_t tot;
        uint32_t cum = block_excl_scan(local, warp_buf, &tot);
        for (int j = 0; j < bpt; ++j) {
            int b = nb - 1 - (tid * bpt + j);
            uint32_t c = hist[b];
            if (cum < remaining && remaining <= cum + c) { sh_bin = (uint32_t)b; sh_above = cum; }
            cum += c;
        }
        __syncthreads();
        remaining -= sh_above;
        prefix |= sh_bin << shift;
        pmask |= bmask << shift;
        __syncthreads();
    }
    const uint32_t thr = prefix;          // the k-th largest key
    const uint32_t need = remaining;      // how many keys equal to thr are kept (lowest positions)

    // ---- ordered compaction ----
    uint32_t base_gt = 0, base_eq = 0;
    for (int64_t c0 = 0; c0 < n; c0 += (int64_t)TK_THREADS * TK_ITEMS) {
        const int64_t s_first = c0 + (int64_t)tid * TK_ITEMS;
        uint32_t flags_gt = 0, flags_eq = 0, n_gt = 0, n_eq = 0;
#pragma unroll
        for (int i = 0; i < TK_ITEMS; ++i) {
            int64_t s = s_first + i;
            if (s < n) {
                uint32_t key = float_key(row[s]);
                if (key > thr) { flags_gt |= 1u << i; ++n_gt; }
                else if (key == thr) { flags_eq |= 1u << i; ++n_eq; }
            }
        }
        uint32_t tot;
        uint32_t ex = block_excl_scan((n_gt << 16) | n_eq, warp_buf, &tot);
        uint32_t gt_before = base_gt + (ex >> 16), eq_before = base_eq + (ex & 0xffffu);
#pragma unroll
        for (int i = 0; i < TK_ITEMS; ++i) {
            bool gt = (flags_gt >> i) & 1u, eq = (flags_eq >> i) & 1u;
            if (gt || (eq && eq_before < need)) {
                uint32_t pos = gt_before + min(eq_before, need);
                if (pos < (uint32_t)k) out[pos] = (int32_t)(s_first + i);
            }
            gt_before += gt;
            eq_before += eq;
        }
        base_gt += tot >> 16;
        base_eq += tot & 0xffffu;
    }
}

}  // namespace

cudaError_t launch_topk_rows(const float *scores, int64_t ld, int64_t row_begin,
                             const int32_t *lens, int64_t max_len, int64_t row_count, int k,
                             int32_t *idx, WsHeader *hdr, cudaStream_t st)
{
    if (row_count <= 0) return cudaSuccess;
    topk_rows_kernel<<<(unsigned)row_count, TK_THREADS, 0, st>>>(scores, ld, row_begin, lens,
                                                                  max_len, k, idx, hdr);
    return cudaGetLastError();
}

}  // namespace dsa
