// FP8 E4M3 quantisation of the indexer's query and key, and the append of new
// tokens to the paged caches ("DeepSeek-V3.2-Exp 稀疏注意力机制(DSA)技术深度解析",
// section 1: the lightning indexer works on FP8 query/key; "DeepSeek-V4 百万
// token 上下文的工程实现", FP8 decoding section: the caches hold FP8).
//
// Per row (token): amax = max |x|, scale = amax / 448 in fp32 (1 when that is
// 0), code = the E4M3 value nearest to x / scale (fp32 quotient, ties to even,
// magnitudes past 448 saturating).  The quotient and the scale are IEEE
// round-to-nearest fp32 operations and the conversion is the hardware's
// round-to-nearest-even saturating cvt, so every code is exactly defined.
//
// HBM-bound: each row is read once into registers (16-byte loads), reduced,
// converted and written once (8-byte code stores), so the traffic is the
// algorithmic bytes: in bytes + codes + 4 per row.  Rows of up to 256 values
// take one warp each; longer rows (the query's H_I * d_I values) one CTA.
#include <cuda_fp8.h>

#include "kernels.h"

namespace dsa {
namespace {

constexpr int QZ_THREADS = 256;
constexpr int QZ_VEC = 8;                            // values per thread per chunk

template <typename In>
struct Chunk8;
template <>
struct Chunk8<uint16_t> {                            // bf16: one 16-byte load
    static __device__ __forceinline__ void load(const uint16_t *p, float (&v)[QZ_VEC])
    {
        const uint4 a = __ldg(reinterpret_cast<const uint4 *>(p));
        const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            v[2 * i] = __uint_as_float(w[i] << 16);
            v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};
template <>
struct Chunk8<float> {                               // fp32: two 16-byte loads
    static __device__ __forceinline__ void load(const float *p, float (&v)[QZ_VEC])
    {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(p));
        const float4 b = __ldg(reinterpret_cast<const float4 *>(p + 4));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
        v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    }
};

__device__ __forceinline__ float e4m3_scale_of(float amax)
{
    const float s = __fdiv_rn(amax, 448.0f);
    return s > 0.0f ? s : 1.0f;
}

// The quotient v / s that decides a code, taken cheaply where that is exact.
// With r = RN(1 / s), the product q' = RN(v * r) equals (v / s)(1 + d1)(1 + d2)
// with |d1|, |d2| <= 2^-24, so it lies within 2 ulps of v / s, and the IEEE
// quotient q = RN(v / s) within half an ulp of it: q and q' are at most 3 ulps
// apart.  The E4M3 rounding of a value only changes at the midpoints between
// neighbouring codes; for |q'| >= 2^-6 (the normal E4M3 range) those are the
// fp32 values whose low 20 mantissa bits are 0x80000 (code spacing 2^20 fp32
// ulps, midpoint half-way), so if q' is more than 4 ulps from such a pattern,
// q and q' round to the same code.  Otherwise -- near a midpoint, below 2^-6
// (the E4M3 subnormal range), or when r is not finite (s below 2^-126) -- the
// IEEE division decides.
__device__ __forceinline__ float e4m3_quotient(float v, float s, float r, bool r_ok)
{
    const float q = v * r;
    // near a midpoint: the low 20 bits within 4 of 0x80000, i.e. (low 20 bits of
    // b - 0x7FFFC) <= 8 (a wrap-around of the low bits only happens next to a
    // binade boundary, which is no midpoint, and leaves the value large)
    const bool near = ((__float_as_uint(q) - 0x7FFFCu) & 0xFFFFFu) < 9u;
    const bool safe = r_ok && fabsf(q) >= 0.015625f && !near;
    return safe ? q : __fdiv_rn(v, s);
}

// Eight codes of v / s, packed little-endian (value i in byte i); r = RN(1 / s).
__device__ __forceinline__ uint2 e4m3_codes8(const float (&v)[QZ_VEC], float s, float r, bool r_ok)
{
    uint32_t w[2];
#pragma unroll
    for (int h = 0; h < 2; ++h) {
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            float2 pr;
            pr.x = e4m3_quotient(v[4 * h + 2 * i], s, r, r_ok);
            pr.y = e4m3_quotient(v[4 * h + 2 * i + 1], s, r, r_ok);
            const __nv_fp8x2_storage_t c = __nv_cvt_float2_to_fp8x2(pr, __NV_SATFINITE, __NV_E4M3);
            word |= (uint32_t)c << (16 * i);
        }
        w[h] = word;
    }
    return make_uint2(w[0], w[1]);
}

// RN(1 / s) and whether it is finite (it is not for s below 2^-126 or so).
__device__ __forceinline__ float e4m3_recip(float s, bool &ok)
{
    const float r = __frcp_rn(s);
    ok = isfinite(r);
    return r;
}

// Rows of `cols` values (cols a multiple of 8, at most TPR * 8 * NCH), TPR
// threads per row (32: a warp, or the whole CTA of 256), chunks of 8 values
// per thread held in registers between the reduction and the conversion.
template <typename In, int TPR, int NCH>
__global__ void __launch_bounds__(QZ_THREADS)
quantize_rows_kernel(const In *__restrict__ x, int64_t rows, int cols, uint8_t *__restrict__ codes,
                     float *__restrict__ scale)
{
    constexpr int RPB = QZ_THREADS / TPR;            // rows per CTA per step
    __shared__ float red[QZ_THREADS / 32];
    const int tid = threadIdx.x, lane = tid & 31;
    const int sub = tid % TPR;
    const int nch = cols / QZ_VEC;
    for (int64_t r0 = (int64_t)blockIdx.x * RPB; r0 < rows; r0 += (int64_t)gridDim.x * RPB) {
        const int64_t r = r0 + tid / TPR;
        const bool live = r < rows;                  // uniform per row group
        float v[NCH][QZ_VEC];
        float amax = 0.0f;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int ch = sub + c * TPR;
            if (live && ch < nch) {
                Chunk8<In>::load(x + r * cols + (int64_t)ch * QZ_VEC, v[c]);
#pragma unroll
                for (int i = 0; i < QZ_VEC; ++i) amax = fmaxf(amax, fabsf(v[c][i]));
            }
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (TPR > 32) {
            if (lane == 0) red[tid >> 5] = amax;
            __syncthreads();
#pragma unroll
            for (int w = 0; w < TPR / 32; ++w) amax = fmaxf(amax, red[w]);
            __syncthreads();                         // red is reused by the next row
        }
        const float s = e4m3_scale_of(amax);
        bool r_ok;
        const float rs = e4m3_recip(s, r_ok);
        if (!live) continue;
        if (sub == 0) scale[r] = s;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int ch = sub + c * TPR;
            if (ch < nch)
                *reinterpret_cast<uint2 *>(codes + r * cols + (int64_t)ch * QZ_VEC) = e4m3_codes8(v[c], s, rs, r_ok);
        }
    }
}

// bf16 rows: each chunk stays packed (four 32-bit words) between the two
// passes, and the amax is taken on the packed pairs (sign bits cleared, a bf16x2
// max: exact), which halves the registers a chunk holds and the instructions
// the reduction costs.  The codes are those of the fp32 path.
template <int TPR, int NCH>
__global__ void __launch_bounds__(QZ_THREADS)
quantize_rows_bf16_kernel(const uint16_t *__restrict__ x, int64_t rows, int cols, uint8_t *__restrict__ codes,
                          float *__restrict__ scale)
{
    constexpr int RPB = QZ_THREADS / TPR;
    __shared__ float red[QZ_THREADS / 32];
    const int tid = threadIdx.x, lane = tid & 31;
    const int sub = tid % TPR;
    const int nch = cols / QZ_VEC;
    for (int64_t r0 = (int64_t)blockIdx.x * RPB; r0 < rows; r0 += (int64_t)gridDim.x * RPB) {
        const int64_t r = r0 + tid / TPR;
        const bool live = r < rows;                  // uniform per row group
        uint4 raw[NCH];
        __nv_bfloat162 m2 = __float2bfloat162_rn(0.f);
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int ch = sub + c * TPR;
            raw[c] = make_uint4(0u, 0u, 0u, 0u);
            if (live && ch < nch) raw[c] = __ldg(reinterpret_cast<const uint4 *>(x + r * cols + (int64_t)ch * QZ_VEC));
            const uint32_t w[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const uint32_t a = w[i] & 0x7fff7fffu;     // |x| of both halves
                m2 = __hmax2(m2, *reinterpret_cast<const __nv_bfloat162 *>(&a));
            }
        }
        float amax = fmaxf(__low2float(m2), __high2float(m2));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        if (TPR > 32) {
            if (lane == 0) red[tid >> 5] = amax;
            __syncthreads();
#pragma unroll
            for (int w = 0; w < TPR / 32; ++w) amax = fmaxf(amax, red[w]);
            __syncthreads();                         // red is reused by the next row
        }
        const float s = e4m3_scale_of(amax);
        bool r_ok;
        const float rs = e4m3_recip(s, r_ok);
        if (!live) continue;
        if (sub == 0) scale[r] = s;
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
            const int ch = sub + c * TPR;
            if (ch < nch) {
                float v[QZ_VEC];
                const uint32_t w[4] = {raw[c].x, raw[c].y, raw[c].z, raw[c].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    v[2 * i] = __uint_as_float(w[i] << 16);
                    v[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
                }
                *reinterpret_cast<uint2 *>(codes + r * cols + (int64_t)ch * QZ_VEC) = e4m3_codes8(v, s, rs, r_ok);
            }
        }
    }
}

template <typename In, int TPR, int NCH>
cudaError_t launch_quantize_t(const In *x, int64_t rows, int cols, uint8_t *codes, float *scale,
                              cudaStream_t st)
{
    constexpr int RPB = QZ_THREADS / TPR;
    int dev = 0, sms = 148, per_sm = 4;
    if (cudaGetDevice(&dev) == cudaSuccess)
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    constexpr bool kBf16 = sizeof(In) == 2;
    if constexpr (kBf16)
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_rows_bf16_kernel<TPR, NCH>, QZ_THREADS, 0);
    else
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_rows_kernel<In, TPR, NCH>, QZ_THREADS, 0);
    if (per_sm < 1) per_sm = 1;
    const int64_t need = ceil_div(rows, RPB);
    const int64_t cap = (int64_t)sms * per_sm;        // persistent: every resident CTA loops over rows
    const unsigned grid = (unsigned)(need < cap ? need : cap);
    if constexpr (kBf16)
        quantize_rows_bf16_kernel<TPR, NCH><<<grid, QZ_THREADS, 0, st>>>(reinterpret_cast<const uint16_t *>(x), rows, cols,
                                                                         codes, scale);
    else
        quantize_rows_kernel<In, TPR, NCH><<<grid, QZ_THREADS, 0, st>>>(x, rows, cols, codes, scale);
    return cudaGetLastError();
}

template <typename In>
cudaError_t launch_quantize_in(const In *x, int64_t rows, int cols, uint8_t *codes, float *scale,
                               cudaStream_t st)
{
    const int nch = cols / QZ_VEC;
    if (nch <= 32) return launch_quantize_t<In, 32, 1>(x, rows, cols, codes, scale, st);
    if (nch <= QZ_THREADS) return launch_quantize_t<In, QZ_THREADS, 1>(x, rows, cols, codes, scale, st);
    if (nch <= 2 * QZ_THREADS) return launch_quantize_t<In, QZ_THREADS, 2>(x, rows, cols, codes, scale, st);
    if (nch <= 4 * QZ_THREADS) return launch_quantize_t<In, QZ_THREADS, 4>(x, rows, cols, codes, scale, st);
    return launch_quantize_t<In, QZ_THREADS, 8>(x, rows, cols, codes, scale, st);
}

// A warp quantises one row of `cols` values (cols a multiple of 8, at most
// 256; lane l holds chunk l) into dst[0, cols) and *dst_scale.
template <typename In>
__device__ __forceinline__ void warp_quantize_row(const In *src, int cols, uint8_t *dst, float *dst_scale, int lane)
{
    const int nch = cols / QZ_VEC;
    float v[QZ_VEC];
    float amax = 0.0f;
    if (lane < nch) {
        Chunk8<In>::load(src + lane * QZ_VEC, v);
#pragma unroll
        for (int j = 0; j < QZ_VEC; ++j) amax = fmaxf(amax, fabsf(v[j]));
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float s = e4m3_scale_of(amax);
    bool r_ok;
    const float rs = e4m3_recip(s, r_ok);
    if (lane < nch) *reinterpret_cast<uint2 *>(dst + lane * QZ_VEC) = e4m3_codes8(v, s, rs, r_ok);
    if (lane == 0) *dst_scale = s;
}

// One warp per new token: quantise its index key (d_I values, at most 256)
// into the FP8 cache slot, and copy its bf16 K and V rows (d values each), or
// with KV8 quantise them too (d at most 256) into FP8 K/V caches with scales.
template <typename In, bool KV8>
__global__ void __launch_bounds__(QZ_THREADS)
cache_append_kernel(const In *__restrict__ kidx_new, const uint16_t *__restrict__ k_new,
                    const uint16_t *__restrict__ v_new, const int32_t *__restrict__ seq,
                    const int32_t *__restrict__ pos, int64_t N, int B, const int32_t *__restrict__ bt,
                    int max_pages, int64_t num_pages, int ps, int d_I, int d, uint8_t *kidx_cache,
                    float *kscale_cache, void *k_cache, void *v_cache, float *k_cache_scale,
                    float *v_cache_scale, uint32_t *status)
{
    const int lane = threadIdx.x & 31;
    const int64_t warps = (int64_t)gridDim.x * (QZ_THREADS / 32);
    for (int64_t i = (int64_t)blockIdx.x * (QZ_THREADS / 32) + (threadIdx.x >> 5); i < N; i += warps) {
        const int b = __ldg(seq + i);
        const int64_t p = __ldg(pos + i);
        int64_t page = -1;
        if (b >= 0 && b < B && p >= 0 && p < (int64_t)max_pages * ps) page = __ldg(bt + (int64_t)b * max_pages + p / ps);
        if (page < 0 || page >= num_pages) {         // warp-uniform: every lane read the same token
            if (lane == 0 && status) atomicCAS(status, (uint32_t)DSA_OK, (uint32_t)DSA_ERR_INVALID_ARG);
            continue;
        }
        const int64_t slot = page * ps + p % ps;
        warp_quantize_row(kidx_new + i * d_I, d_I, kidx_cache + slot * d_I, kscale_cache + slot, lane);
        if constexpr (KV8) {
            warp_quantize_row(k_new + i * d, d, static_cast<uint8_t *>(k_cache) + slot * d, k_cache_scale + slot, lane);
            warp_quantize_row(v_new + i * d, d, static_cast<uint8_t *>(v_cache) + slot * d, v_cache_scale + slot, lane);
        } else {
            // K and V rows: 16-byte chunks
            const int vch = d / 8;
            for (int c = lane; c < 2 * vch; c += 32) {
                const bool is_v = c >= vch;
                const int cc = is_v ? c - vch : c;
                const uint4 val = __ldg(reinterpret_cast<const uint4 *>((is_v ? v_new : k_new) + i * d) + cc);
                reinterpret_cast<uint4 *>(static_cast<uint16_t *>(is_v ? v_cache : k_cache) + slot * d)[cc] = val;
            }
        }
    }
}

}  // namespace

cudaError_t launch_quantize_e4m3(const void *x, bool bf16_in, int64_t rows, int cols, uint8_t *codes,
                                 float *scale, cudaStream_t st)
{
    if (rows <= 0) return cudaSuccess;
    if (bf16_in) return launch_quantize_in(static_cast<const uint16_t *>(x), rows, cols, codes, scale, st);
    return launch_quantize_in(static_cast<const float *>(x), rows, cols, codes, scale, st);
}

cudaError_t launch_cache_append(const void *kidx_new, bool bf16_in, const uint16_t *k_new,
                                const uint16_t *v_new, const int32_t *seq, const int32_t *pos, int64_t N,
                                int B, const int32_t *bt, int max_pages, int64_t num_pages, int ps,
                                int d_I, int d, uint8_t *kidx_cache, float *kscale_cache,
                                void *k_cache, void *v_cache, float *k_cache_scale, float *v_cache_scale,
                                uint32_t *status, cudaStream_t st)
{
    if (N <= 0) return cudaSuccess;
    const int64_t need = ceil_div(N, QZ_THREADS / 32);
    const unsigned grid = (unsigned)(need < 148 * 8 ? need : 148 * 8);
    const bool kv8 = k_cache_scale != nullptr;
#define DSA_APPEND(IN, KV)                                                                                     \
    cache_append_kernel<IN, KV><<<grid, QZ_THREADS, 0, st>>>(                                                  \
        static_cast<const IN *>(kidx_new), k_new, v_new, seq, pos, N, B, bt, max_pages, num_pages, ps, d_I, d, \
        kidx_cache, kscale_cache, k_cache, v_cache, k_cache_scale, v_cache_scale, status)
    if (bf16_in) {
        if (kv8) DSA_APPEND(uint16_t, true); else DSA_APPEND(uint16_t, false);
    } else {
        if (kv8) DSA_APPEND(float, true); else DSA_APPEND(float, false);
    }
#undef DSA_APPEND
    return cudaGetLastError();
}

}  // namespace dsa
