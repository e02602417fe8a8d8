// Lightning-indexer scores, stage kernels.
//
// I[t,s] = sk[s] * sum_h (w[t,h] * sq[t]) * ReLU(q8[t,h,:] . k8[s,:])
// -- the indexer of "DeepSeek-V3.2-Exp DSA 技术深度解析", section 1 (few heads,
// index_head_dim 128, FP8, ReLU), with both per-token scales factored out of
// the ReLU: they are positive, and ReLU(a*x) = a*ReLU(x) for a > 0.
//
// index_fp8_mma_kernel: FP8 E4M3 tensor-core (mma.sync m16n8k32) version used
// for row-chunked stage output.  A CTA owns 64 query rows x 256 keys; the key
// tile stays in shared memory for all heads while the per-head query tiles
// stream through a 3-stage cp.async ring.  Each head's 64x256 fp32 product is
// folded into the running score with one max + one FMA per element, so the
// per-head products never leave registers.
#include "kernels.h"

namespace dsa {
namespace {

constexpr int IDX_BM = 64;     // query rows per CTA
constexpr int IDX_BN = 256;    // keys per CTA
constexpr int IDX_D = 128;     // index head dim (bytes per row)
constexpr int IDX_STAGES = 3;
constexpr int IDX_THREADS = 256;

// byte offset of 16-byte chunk `c` of row `r` in a 128-byte-row tile (XOR swizzle)
__device__ __forceinline__ int swz(int r, int c) { return r * 128 + ((c ^ (r & 7)) << 4); }

__global__ void __launch_bounds__(IDX_THREADS, 1)
index_fp8_mma_kernel(const uint8_t *__restrict__ q8, const float *__restrict__ sq,
                     const uint8_t *__restrict__ k8, const float *__restrict__ sk,
                     const uint16_t *__restrict__ w, int64_t T, int H, int64_t row_begin,
                     int64_t row_count, float *__restrict__ out, int64_t ld, int write_upper)
{
    extern __shared__ __align__(128) uint8_t smem[];
    uint8_t *Ks = smem;                                   // 256 x 128 B
    uint8_t *Qs = Ks + IDX_BN * IDX_D;                    // 3 x 64 x 128 B
    float *Cs = reinterpret_cast<float *>(Qs + IDX_STAGES * IDX_BM * IDX_D);  // [64][H]
    float *Sk = Cs + IDX_BM * H;                          // [256]

    const int tid = threadIdx.x;
    const int lane = tid & 31, warp = tid >> 5;
    const int warp_m = warp >> 2, warp_n = warp & 3;
    const int g = lane >> 2, tig = lane & 3;

    const int64_t r_lo = row_begin + (int64_t)blockIdx.y * IDX_BM;          // first query position
    const int64_t r_end = min(row_begin + row_count, r_lo + IDX_BM);         // one past last
    const int64_t s0 = (int64_t)blockIdx.x * IDX_BN;
    const int nrows = (int)(r_end - r_lo);

    if (s0 > r_end - 1) {       // tile entirely above the diagonal
        if (write_upper) {
            for (int i = tid; i < nrows * IDX_BN; i += IDX_THREADS) {
                int r = i / IDX_BN, c = i % IDX_BN;
                int64_t s = s0 + c;
                if (s < T) out[(r_lo + r - row_begin) * ld + s] = -INFINITY;
            }
        }
        return;
    }

    // ---- async loads: key tile + first two query-head tiles ----
    for (int i = tid; i < IDX_BN * 8; i += IDX_THREADS) {
        int r = i >> 3, c = i & 7;
        int64_t s = s0 + r;
        bool ok = s < T;
        cp_async_16(Ks + swz(r, c), k8 + (ok ? s : 0) * IDX_D + c * 16, ok);
    }
    auto load_q = [&](int h, int stage) {
        uint8_t *dst = Qs + stage * IDX_BM * IDX_D;
        for (int i = tid; i < IDX_BM * 8; i += IDX_THREADS) {
            int r = i >> 3, c = i & 7;
            bool ok = r < nrows;
            int64_t t = ok ? r_lo + r : 0;
            cp_async_16(dst + swz(r, c), q8 + (t * H + h) * IDX_D + c * 16, ok);
        }
    };
    load_q(0, 0);
    cp_async_commit();
    if (H > 1) load_q(1, 1);
    cp_async_commit();

    // combined per-row head weights c[t,h] = w[t,h] * sq[t] and key scales
    for (int i = tid; i < IDX_BM * H; i += IDX_THREADS) {
        int r = i / H, h = i % H;
        float c = 0.f;
        if (r < nrows) c = bf16_to_f32(w[(r_lo + r) * H + h]) * sq[r_lo + r];
        Cs[i] = c;
    }
    for (int i = tid; i < IDX_BN; i += IDX_THREADS) {
        int64_t s = s0 + i;
        Sk[i] = s < T ? sk[s] : 0.f;
    }

    float score[2][8][4];
#pragma unroll
    for (int a = 0; a < 2; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b)
#pragma unroll
            for (int c = 0; c < 4; ++c) score[a][b][c] = 0.f;

    const int wrow = warp_m * 32, wcol = warp_n * 64;

    for (int h = 0; h < H; ++h) {
        cp_async_wait<1>();
        __syncthreads();
        if (h + 2 < H) load_q(h + 2, (h + 2) % IDX_STAGES);
        cp_async_commit();

        const uint8_t *Qh = Qs + (h % IDX_STAGES) * IDX_BM * IDX_D;
        float acc[2][8][4];
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int b = 0; b < 8; ++b)
#pragma unroll
                for (int c = 0; c < 4; ++c) acc[a][b][c] = 0.f;

#pragma unroll
        for (int ks = 0; ks < 4; ++ks) {
            uint32_t af[2][4];
#pragma unroll
            for (int mt = 0; mt < 2; ++mt) {
                int mi = lane >> 3;
                int row = wrow + mt * 16 + (mi & 1) * 8 + (lane & 7);
                int chunk = ks * 2 + (mi >> 1);
                ldmatrix_x4(af[mt][0], af[mt][1], af[mt][2], af[mt][3], Qh + swz(row, chunk));
            }
            uint32_t bf[8][2];
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                int mi = lane >> 3;
                int key = wcol + np * 16 + (mi >> 1) * 8 + (lane & 7);
                int chunk = ks * 2 + (mi & 1);
                ldmatrix_x4(bf[2 * np][0], bf[2 * np][1], bf[2 * np + 1][0], bf[2 * np + 1][1],
                            Ks + swz(key, chunk));
            }
#pragma unroll
            for (int mt = 0; mt < 2; ++mt)
#pragma unroll
                for (int nt = 0; nt < 8; ++nt) mma_e4m3_16832(acc[mt][nt], af[mt], bf[nt][0], bf[nt][1]);
        }
        // fold this head in: score += c[t,h] * ReLU(acc)
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
            float c_lo = Cs[(wrow + mt * 16 + g) * H + h];
            float c_hi = Cs[(wrow + mt * 16 + 8 + g) * H + h];
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
                score[mt][nt][0] = fmaf(c_lo, fmaxf(acc[mt][nt][0], 0.f), score[mt][nt][0]);
                score[mt][nt][1] = fmaf(c_lo, fmaxf(acc[mt][nt][1], 0.f), score[mt][nt][1]);
                score[mt][nt][2] = fmaf(c_hi, fmaxf(acc[mt][nt][2], 0.f), score[mt][nt][2]);
                score[mt][nt][3] = fmaf(c_hi, fmaxf(acc[mt][nt][3], 0.f), score[mt][nt][3]);
            }
        }
    }
    cp_async_wait<0>();

    // ---- epilogue: key scale, causal mask, store ----
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            int r = wrow + mt * 16 + half * 8 + g;
            if (r >= nrows) continue;
            int64_t t = r_lo + r;
            float *orow = out + (t - row_begin) * ld;
#pragma unroll
            for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    int c = wcol + nt * 8 + tig * 2 + e;
                    int64_t s = s0 + c;
                    if (s >= T) continue;
                    if (s <= t) orow[s] = score[mt][nt][half * 2 + e] * Sk[c];
                    else if (write_upper) orow[s] = -INFINITY;
                }
            }
        }
    }
}

// fp32 indexer for small shapes: one thread per (query row, key).
__global__ void index_f32_kernel(const float *__restrict__ q, const float *__restrict__ k,
                                 const float *__restrict__ w, int64_t T, int H, int D,
                                 int64_t row_begin, float *__restrict__ out, int64_t ld,
                                 int write_upper)
{
    extern __shared__ float qs[];            // [H*D] query row, then [H] weights
    float *ws = qs + H * D;
    const int64_t t = row_begin + blockIdx.y;
    for (int i = threadIdx.x; i < H * D; i += blockDim.x) qs[i] = q[t * H * D + i];
    for (int i = threadIdx.x; i < H; i += blockDim.x) ws[i] = w[t * H + i];
    __syncthreads();
    const int64_t s = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= T) return;
    float *orow = out + (int64_t)blockIdx.y * ld;
    if (s > t) {
        if (write_upper) orow[s] = -INFINITY;
        return;
    }
    const float *kr = k + s * D;
    float total = 0.f;
    for (int h = 0; h < H; ++h) {
        float dot = 0.f;
        for (int j = 0; j < D; ++j) dot = fmaf(qs[h * D + j], kr[j], dot);
        total = fmaf(ws[h], fmaxf(dot, 0.f), total);
    }
    orow[s] = total;
}

}  // namespace

cudaError_t launch_index_fp8(const uint8_t *q8, const float *sq, const uint8_t *k8,
                             const float *sk, const uint16_t *w, int64_t T, int H,
                             int64_t row_begin, int64_t row_count, float *out, int64_t ld,
                             bool write_upper, cudaStream_t st)
{
    if (row_count <= 0) return cudaSuccess;
    size_t smem = IDX_BN * IDX_D + IDX_STAGES * IDX_BM * IDX_D + sizeof(float) * (IDX_BM * H + IDX_BN);
    cudaError_t e = cudaFuncSetAttribute(index_fp8_mma_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    // only key tiles that can hold a causal key of this row block are visited,
    // unless the upper triangle must be written out
    int64_t kt = write_upper ? ceil_div(T, IDX_BN) : ceil_div(row_begin + row_count, IDX_BN);
    dim3 grid((unsigned)kt, (unsigned)ceil_div(row_count, IDX_BM));
    index_fp8_mma_kernel<<<grid, IDX_THREADS, smem, st>>>(q8, sq, k8, sk, w, T, H, row_begin,
                                                          row_count, out, ld, write_upper);
    return cudaGetLastError();
}

cudaError_t launch_index_f32(const float *q, const float *k, const float *w, int64_t T, int H,
                             int D, int64_t row_begin, int64_t row_count, float *out,
                             int64_t ld, bool write_upper, cudaStream_t st)
{
    if (row_count <= 0) return cudaSuccess;
    size_t smem = sizeof(float) * (H * D + H);
    if (smem > 48 * 1024) {
        cudaError_t e = cudaFuncSetAttribute(index_f32_kernel,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
    }
    for (int64_t r0 = 0; r0 < row_count; r0 += 65535) {      // gridDim.y limit
        int64_t n = min(row_count - r0, (int64_t)65535);
        int64_t cols = write_upper ? T : (row_begin + r0 + n);
        dim3 grid((unsigned)ceil_div(cols, 128), (unsigned)n);
        index_f32_kernel<<<grid, 128, smem, st>>>(q, k, w, T, H, D, row_begin + r0,
                                                  out + r0 * ld, ld, write_upper);
    }
    return cudaGetLastError();
}

}  // namespace dsa
