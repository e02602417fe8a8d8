// Decode-step lightning indexer over a paged FP8 index-key cache.
//
// One new query token per sequence scores every cached token s < n_b:
//   I[s] = ksc[s] * sum_h (w[h] * sq) * ReLU(q8[h,:] . k8[s,:])
// ("DeepSeek-V3.2-Exp DSA 技术深度解析", section 1 for the indexer; section 6:
// decode still pays the O(n) indexer per token; FP8 index keys as in the
// hotdry page's FP8 cache).  The work is a skinny GEMM, keys x heads, that is
// bound by streaming the 128-byte keys from HBM, so keys are the MMA rows and
// are read straight from global memory into registers, fully coalesced, with
// no shared-memory staging: the query's 64 heads stay resident as the MMA's B
// fragments for the whole kernel.  The dot product runs over the 128 bytes in
// a permuted order that is the same for both operands (the contraction is
// order-free), which lets every lane load two 16-byte runs of a key row.
#include "kernels.h"

namespace dsa {
namespace {

constexpr int DEC_WARPS = 8;
constexpr int DEC_CHUNK = 1024;     // keys per CTA (multiple of 16)

__device__ __forceinline__ void ld_row_frag(const uint8_t *row, int tig, uint32_t (&wds)[8])
{
    // bytes [tig*16, tig*16+16) and [64 + tig*16, 64 + tig*16 + 16)
    uint4 x = __ldg(reinterpret_cast<const uint4 *>(row + tig * 16));
    uint4 y = __ldg(reinterpret_cast<const uint4 *>(row + 64 + tig * 16));
    wds[0] = x.x; wds[1] = x.y; wds[2] = x.z; wds[3] = x.w;
    wds[4] = y.x; wds[5] = y.y; wds[6] = y.z; wds[7] = y.w;
}

__device__ __forceinline__ void ld_row_frag_stream(const uint8_t *row, int tig, uint32_t (&wds)[8])
{
    uint4 x, y;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(x.x), "=r"(x.y), "=r"(x.z), "=r"(x.w) : "l"(row + tig * 16));
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(y.x), "=r"(y.y), "=r"(y.z), "=r"(y.w) : "l"(row + 64 + tig * 16));
    wds[0] = x.x; wds[1] = x.y; wds[2] = x.z; wds[3] = x.w;
    wds[4] = y.x; wds[5] = y.y; wds[6] = y.z; wds[7] = y.w;
}

template <int NT>
__global__ void __launch_bounds__(DEC_WARPS * 32)
decode_index_kernel(const uint8_t *__restrict__ q8, const float *__restrict__ sq,
                    const uint16_t *__restrict__ w, const uint8_t *__restrict__ kidx,
                    const float *__restrict__ kscale, const int32_t *__restrict__ block_table,
                    const int32_t *__restrict__ context_lens, int64_t num_pages, int max_pages,
                    int page_size, int64_t max_context, float *__restrict__ scores, int64_t ld,
                    WsHeader *hdr)
{
    constexpr int H = NT * 8;
    const int b = blockIdx.y;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, tig = lane & 3;
    const int64_t n = context_lens[b];
    if (n < 1 || n > max_context || n > (int64_t)max_pages * page_size) {
        if (blockIdx.x == 0 && threadIdx.x == 0) record_error(hdr, DSA_ERR_INVALID_ARG, (unsigned)b);
        return;
    }
    const int64_t c0 = (int64_t)blockIdx.x * DEC_CHUNK;
    if (c0 >= n) return;

    // query head fragments (B operand) and combined head weights, resident
    uint32_t qb[NT][8];
    float cw[NT][2];
    const float s_q = sq[b];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        ld_row_frag(q8 + ((int64_t)b * H + nt * 8 + g) * 128, tig, qb[nt]);
        cw[nt][0] = bf16_to_f32(w[(int64_t)b * H + nt * 8 + tig * 2]) * s_q;
        cw[nt][1] = bf16_to_f32(w[(int64_t)b * H + nt * 8 + tig * 2 + 1]) * s_q;
    }
    const int32_t *bt = block_table + (int64_t)b * max_pages;
    float *srow = scores + (int64_t)b * ld;
    const int64_t c1 = min(n, c0 + DEC_CHUNK);

    for (int64_t p0 = c0 + warp * 16; p0 < c1; p0 += DEC_WARPS * 16) {
        const int page = bt[p0 / page_size];
        if (page < 0 || page >= num_pages) {
            if (lane == 0) record_error(hdr, DSA_ERR_INVALID_ARG, (unsigned)b);
            continue;
        }
        const int64_t slot0 = (int64_t)page * page_size + p0 % page_size;
        const uint8_t *base = kidx + slot0 * 128;
        uint32_t a_lo[8], a_hi[8];
        ld_row_frag_stream(base + g * 128, tig, a_lo);
        ld_row_frag_stream(base + (g + 8) * 128, tig, a_hi);
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) acc[nt][0] = acc[nt][1] = acc[nt][2] = acc[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            const uint32_t af[4] = {a_lo[2 * ks], a_hi[2 * ks], a_lo[2 * ks + 1], a_hi[2 * ks + 1]};
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) mma_e4m3_16832(acc[nt], af, qb[nt][2 * ks], qb[nt][2 * ks + 1]);
        }
        float s_lo = 0.f, s_hi = 0.f;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            s_lo = fmaf(cw[nt][0], fmaxf(acc[nt][0], 0.f), s_lo);
            s_lo = fmaf(cw[nt][1], fmaxf(acc[nt][1], 0.f), s_lo);
            s_hi = fmaf(cw[nt][0], fmaxf(acc[nt][2], 0.f), s_hi);
            s_hi = fmaf(cw[nt][1], fmaxf(acc[nt][3], 0.f), s_hi);
        }
        s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 1);
        s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 2);
        s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 1);
        s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 2);
        if (tig == 0) {
            if (p0 + g < c1) srow[p0 + g] = s_lo * kscale[slot0 + g];
            if (p0 + g + 8 < c1) srow[p0 + g + 8] = s_hi * kscale[slot0 + g + 8];
        }
    }
}

}  // namespace

cudaError_t launch_decode_index(const uint8_t *q8, const float *sq, const uint16_t *w,
                                const uint8_t *kidx, const float *kscale,
                                const int32_t *block_table, const int32_t *context_lens,
                                int64_t num_pages, int max_pages, int page_size, int B,
                                int64_t max_context, int H, float *scores, int64_t ld,
                                WsHeader *hdr, cudaStream_t st)
{
    if (B <= 0) return cudaSuccess;
    dim3 grid((unsigned)ceil_div(max_context, DEC_CHUNK), (unsigned)B);
    const int threads = DEC_WARPS * 32;
#define DEC_CASE(NTV)                                                                        \
    case NTV:                                                                                \
        decode_index_kernel<NTV><<<grid, threads, 0, st>>>(q8, sq, w, kidx, kscale,          \
                                                           block_table, context_lens,        \
                                                           num_pages, max_pages, page_size,  \
                                                           max_context, scores, ld, hdr);    \
        break;
    switch (H / 8) {
        DEC_CASE(1) DEC_CASE(2) DEC_CASE(3) DEC_CASE(4) DEC_CASE(5) DEC_CASE(6) DEC_CASE(7) DEC_CASE(8)
    default: return cudaErrorInvalidValue;
    }
#undef DEC_CASE
    return cudaGetLastError();
}

}  // namespace dsa
