// Decode of contexts split over several devices: the small kernels around the
// decode indexer, top-k and attention that let each device work on its own
// shard of positions and the shards' results be merged exactly.
//
// A sequence's context is cut into G contiguous shards of positions; device g
// holds shard g's caches.  Each device scores its keys and selects its own
// top-k (positions made global, with their scores); the G candidate lists
// are gathered, and the global top-k of their union -- which contains the
// global top-k, since every member of it is in its shard's top-k -- is taken
// with ties to the lower position (shard lists are in position order, so the
// lower column is the lower position).  Each device then attends the selected
// positions it holds, and the G partial results (normalised output and
// log-sum-exp) are merged:  lse = log sum_g exp(lse_g),
// o = sum_g exp(lse_g - lse) o_g.
#include "kernels.h"

namespace dsa {
namespace {

// One thread per entry (grid: entry blocks x sequences), so that every load of
// a launch is in flight at once: the merges move a few KB per sequence and are
// bound by memory latency, not bandwidth.

// idx_out[b, j] = idx_local[b, j] + base[b] (or -1), score_out[b, j] = its
// score (-inf for -1).  A global position past INT32_MAX or a negative base is
// reported and its entry dropped.
__global__ void gather_selected_kernel(const float *__restrict__ scores, int64_t ld,
                                       const int32_t *__restrict__ idx_local, const int32_t *__restrict__ base,
                                       int k, int32_t *__restrict__ idx_out, float *__restrict__ score_out,
                                       WsHeader *hdr)
{
    const int64_t b = blockIdx.y;
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= k) return;
    const int64_t pb = __ldg(base + b);
    const int32_t p = __ldg(idx_local + b * k + j);
    bool ok = p >= 0;
    if (ok && (pb < 0 || pb + p > (int64_t)INT32_MAX)) {
        record_error(hdr, DSA_ERR_INVALID_ARG, (unsigned)b);
        ok = false;
    }
    idx_out[b * k + j] = ok ? (int32_t)(pb + p) : -1;
    score_out[b * k + j] = ok ? __ldg(scores + b * ld + p) : -INFINITY;
}

// Candidate lists (list g at g * stride, [B][k] each) -> one score row per
// sequence [B][G * k] in shard order (-inf for empty entries), and the rows'
// lengths.
__global__ void merge_prep_kernel(const int32_t *__restrict__ cand_pos, const float *__restrict__ cand_score,
                                  int64_t stride, int G, int k, float *__restrict__ scores_t,
                                  int32_t *__restrict__ lens)
{
    const int64_t b = blockIdx.y;
    const int n = G * k;
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j == 0) lens[b] = n;
    if (j >= n) return;
    const int g = j / k, i = j - g * k;
    const int64_t src = g * stride + b * k + i;
    const int32_t p = __ldg(cand_pos + src);
    const float sc = __ldg(cand_score + src);
    scores_t[b * n + j] = p >= 0 ? sc : -INFINITY;
}

// Selected columns -> global positions, in order, the empty ones dropped: one
// CTA of 1024 threads per sequence, 1024 entries per round, ordered by warp
// ballots and the warps' counts in shared memory.
constexpr int kFinishThreads = 1024;

__global__ void __launch_bounds__(kFinishThreads)
merge_finish_kernel(const int32_t *__restrict__ sel_cols, const int32_t *__restrict__ cand_pos, int64_t stride,
                    int k, int32_t *__restrict__ idx_out)
{
    __shared__ int warp_count[kFinishThreads / 32];
    const int64_t b = blockIdx.x;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int written = 0;                                 // block-uniform
    for (int j0 = 0; j0 < k; j0 += kFinishThreads) {
        const int j = j0 + threadIdx.x;
        int32_t p = -1;
        if (j < k) {
            const int32_t c = __ldg(sel_cols + b * k + j);
            if (c >= 0) {
                const int g = c / k, i = c - g * k;
                p = __ldg(cand_pos + g * stride + b * k + i);
            }
        }
        const unsigned m = __ballot_sync(0xffffffffu, p >= 0);
        if (lane == 0) warp_count[warp] = __popc(m);
        __syncthreads();
        int before = 0, total = 0;
        #pragma unroll 8
        for (int w = 0; w < kFinishThreads / 32; ++w) {
            const int c = warp_count[w];
            before += w < warp ? c : 0;
            total += c;
        }
        if (p >= 0) idx_out[b * k + written + before + __popc(m & ((1u << lane) - 1u))] = p;
        written += total;
        __syncthreads();                             // the counts are rewritten next round
    }
    for (int j = written + threadIdx.x; j < k; j += kFinishThreads) idx_out[b * k + j] = -1;
}

// Global positions -> positions of this shard (p - base when in [base, base + n), else -1).
__global__ void local_idx_kernel(const int32_t *__restrict__ idx, const int32_t *__restrict__ base,
                                 const int32_t *__restrict__ lens, int k, int32_t *__restrict__ idx_local)
{
    const int64_t b = blockIdx.y;
    const int j = blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= k) return;
    const int64_t pb = __ldg(base + b), n = __ldg(lens + b);
    const int64_t p = __ldg(idx + b * k + j);
    idx_local[b * k + j] = (p >= 0 && p >= pb && p < pb + n) ? (int32_t)(p - pb) : -1;
}

// out[b, h] = sum_g exp(lse_g - lse) o_g[b, h], lse = log sum_g exp(lse_g),
// partial g at part_out + g * out_stride, part_lse + g * lse_stride; one warp
// per (b, h), d = 128 (four values per lane).  Lane g holds partial g's lse
// and weight (32 partials a round); the partial rows are loaded eight at a
// time, all in flight together.
__global__ void merge_partials_kernel(const uint16_t *__restrict__ part_out, int64_t out_stride,
                                      const float *__restrict__ part_lse, int64_t lse_stride, int G, int H,
                                      uint16_t *__restrict__ out, float *__restrict__ lse)
{
    constexpr int D = 128, U = 8;
    const int64_t b = blockIdx.x;
    const int h = blockIdx.y * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (h >= H) return;
    const float *pl = part_lse + b * H + h;
    float mx = -INFINITY;
    for (int g0 = 0; g0 < G; g0 += 32)
        if (g0 + lane < G) mx = fmaxf(mx, __ldg(pl + (g0 + lane) * lse_stride));
    #pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    float den = 0.f;                                 // this lane's partials' weights
    if (mx != -INFINITY) {
        const uint16_t *po = part_out + (b * H + h) * (int64_t)D + lane * 4;
        for (int g0 = 0; g0 < G; g0 += 32) {
            const int g = g0 + lane;
            const float lg = g < G ? __ldg(pl + g * lse_stride) : -INFINITY;
            const float wl = lg == -INFINITY ? 0.f : __expf(lg - mx);
            den += wl;
            const int n = G - g0 < 32 ? G - g0 : 32;
            for (int i0 = 0; i0 < n; i0 += U) {
                uint2 v[U];
                #pragma unroll
                for (int u = 0; u < U; ++u)
                    v[u] = i0 + u < n ? __ldg(reinterpret_cast<const uint2 *>(po + (g0 + i0 + u) * out_stride))
                                      : make_uint2(0u, 0u);
                #pragma unroll
                for (int u = 0; u < U; ++u) {
                    const float wgt = __shfl_sync(0xffffffffu, wl, (i0 + u) & 31);
                    if (i0 + u < n && wgt != 0.f) {  // an empty partial's row is not read into the sum
                        acc[0] += wgt * bf16_to_f32((uint16_t)(v[u].x & 0xffffu));
                        acc[1] += wgt * bf16_to_f32((uint16_t)(v[u].x >> 16));
                        acc[2] += wgt * bf16_to_f32((uint16_t)(v[u].y & 0xffffu));
                        acc[3] += wgt * bf16_to_f32((uint16_t)(v[u].y >> 16));
                    }
                }
            }
        }
    }
    #pragma unroll
    for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    const float inv = den > 0.f ? 1.f / den : 0.f;
    uint2 packed;
    packed.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
    packed.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
    *reinterpret_cast<uint2 *>(out + (b * H + h) * (int64_t)D + lane * 4) = packed;
    if (lse && lane == 0) lse[b * H + h] = den > 0.f ? mx + logf(den) : -INFINITY;
}

}  // namespace

cudaError_t launch_gather_selected(const float *scores, int64_t ld, const int32_t *idx_local, const int32_t *base,
                                   int B, int k, int32_t *idx_out, float *score_out, WsHeader *hdr,
                                   cudaStream_t st)
{
    if (B <= 0) return cudaSuccess;
    gather_selected_kernel<<<dim3((unsigned)ceil_div(k, 256), (unsigned)B), 256, 0, st>>>(scores, ld, idx_local, base,
                                                                                         k, idx_out, score_out, hdr);
    return cudaGetLastError();
}

size_t merge_selections_ws_bytes(int B, int G, int k)
{
    return align_up(sizeof(float) * (size_t)B * G * k, 256) + align_up(sizeof(int32_t) * (size_t)B, 256) +
           align_up(sizeof(int32_t) * (size_t)B * k, 256);
}

cudaError_t launch_merge_selections(const int32_t *cand_pos, const float *cand_score, int64_t stride, int B, int G,
                                    int k, int32_t *idx_out, void *ws, WsHeader *hdr, cudaStream_t st)
{
    if (B <= 0) return cudaSuccess;
    uint8_t *p = static_cast<uint8_t *>(ws);
    float *scores_t = reinterpret_cast<float *>(p);
    p += align_up(sizeof(float) * (size_t)B * G * k, 256);
    int32_t *lens = reinterpret_cast<int32_t *>(p);
    p += align_up(sizeof(int32_t) * (size_t)B, 256);
    int32_t *sel = reinterpret_cast<int32_t *>(p);
    merge_prep_kernel<<<dim3((unsigned)ceil_div((int64_t)G * k, 256), (unsigned)B), 256, 0, st>>>(
        cand_pos, cand_score, stride, G, k, scores_t, lens);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // the exact top-k of each candidate row, ties to the lower column = lower position
    e = launch_topk_rows(scores_t, (int64_t)G * k, 0, lens, (int64_t)G * k, B, k, sel, hdr, st);
    if (e != cudaSuccess) return e;
    merge_finish_kernel<<<(unsigned)B, kFinishThreads, 0, st>>>(sel, cand_pos, stride, k, idx_out);
    return cudaGetLastError();
}

cudaError_t launch_local_idx(const int32_t *idx, const int32_t *base, const int32_t *lens, int B, int k,
                             int32_t *idx_local, cudaStream_t st)
{
    if (B <= 0) return cudaSuccess;
    local_idx_kernel<<<dim3((unsigned)ceil_div(k, 256), (unsigned)B), 256, 0, st>>>(idx, base, lens, k, idx_local);
    return cudaGetLastError();
}

cudaError_t launch_merge_partials(const uint16_t *part_out, int64_t out_stride, const float *part_lse,
                                  int64_t lse_stride, int G, int B, int H, int d, uint16_t *out, float *lse,
                                  cudaStream_t st)
{
    if (B <= 0) return cudaSuccess;
    if (d != 128) return cudaErrorNotSupported;
    merge_partials_kernel<<<dim3((unsigned)B, (unsigned)ceil_div(H, 8)), 256, 0, st>>>(
        part_out, out_stride, part_lse, lse_stride, G, H, out, lse);
    return cudaGetLastError();
}

}  // namespace dsa
