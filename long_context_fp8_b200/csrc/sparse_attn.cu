// Sparse main attention over the selected KV rows ("DeepSeek-V3.2-Exp DSA
// 技术深度解析", section 1: the main attention looks only at the selected
// subset, O(n^2) -> O(n k)).  One shared K/V head (MQA): every query head of a
// token attends to the same selected rows, so a CTA gathers each selected
// K/V row once into shared memory and reuses it for all of its query heads.
//
// CTA = one query token x up to 128 query heads (one warp per 16 heads).
// Selected rows are gathered 64 at a time with 16-byte cp.async into a
// double-buffered, XOR-swizzled tile; S = Q K^T and O += P V run on bf16
// tensor cores (mma.sync m16n8k16) with an online softmax in fp32 (base 2,
// log2(e) folded into the scale).  Decode uses the same kernel with K/V read
// through the page table, and may split the index list over several CTAs
// whose normalised partial outputs and log-sum-exps are merged afterwards.
#include "kernels.h"

namespace dsa {
namespace {

constexpr int AT_BK = 64;                 // selected rows per block
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct AttnArgs {
    const uint16_t *q;        // [rows, H, D]
    const uint16_t *k;        // contiguous [T, D] (paged: unused)
    const uint16_t *v;
    int64_t T;
    PagedKV kv;               // paged K/V (decode)
    const int32_t *idx;       // [rows, ksel]
    int H, ksel;
    float scale_log2;         // sm_scale * log2(e)
    uint16_t *out;            // [rows, H, D]
    float *lse;               // [rows, H] or null
    float *part;              // split partials (splits > 1)
    int splits, chunk;        // index-list entries per split (multiple of AT_BK)
    WsHeader *hdr;
};

template <int D>
__device__ __forceinline__ int aswz(int r, int c)   // byte offset of chunk c (16 B) of row r
{
    return r * (D * 2) + ((c ^ (r & 7)) << 4);
}

template <int D, bool PAGED>
__global__ void __launch_bounds__(256, 1)
sparse_attn_bf16_kernel(const AttnArgs a)
{
    constexpr int CPR = D / 8;            // 16-byte chunks per row
    constexpr int ROWB = D * 2;           // bytes per row
    extern __shared__ __align__(128) uint8_t smem[];
    const int nw = blockDim.x >> 5;
    const int hrows = nw * 16;            // query heads handled by this CTA
    uint8_t *Qs = smem;                                   // [hrows][D]
    uint8_t *Ks = Qs + hrows * ROWB;                      // [2][64][D]
    uint8_t *Vs = Ks + 2 * AT_BK * ROWB;                  // [2][64][D]
    int *valid = reinterpret_cast<int *>(Vs + 2 * AT_BK * ROWB);  // [2][64]

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, tig = lane & 3;
    const int64_t row = blockIdx.x;
    const int h0 = blockIdx.y * 128;
    const int split = blockIdx.z;
    const int e_begin = split * a.chunk;
    const int e_end = min(a.ksel, e_begin + a.chunk);
    const int nblk = e_end > e_begin ? (e_end - e_begin + AT_BK - 1) / AT_BK : 0;

    int ctx = 0;
    if constexpr (PAGED) {
        ctx = a.kv.context_lens[row];
        if (ctx < 0 || (int64_t)ctx > (int64_t)a.kv.max_pages * a.kv.page_size) ctx = 0;
    }

    // ---- Q tile ----
    for (int i = tid; i < hrows * CPR; i += blockDim.x) {
        int r = i / CPR, c = i % CPR;
        int h = h0 + r;
        bool ok = h < a.H;
        cp_async_16(Qs + aswz<D>(r, c), a.q + ((row * a.H + (ok ? h : 0)) * D) + c * 8, ok);
    }
    cp_async_commit();

    auto gather = [&](int blk, int stage) {
        uint8_t *kd = Ks + stage * AT_BK * ROWB;
        uint8_t *vd = Vs + stage * AT_BK * ROWB;
        for (int i = tid; i < AT_BK * CPR; i += blockDim.x) {
            int r = i / CPR, c = i % CPR;
            int e = e_begin + blk * AT_BK + r;
            int p = e < e_end ? a.idx[row * a.ksel + e] : -1;
            const uint16_t *ksrc = a.k, *vsrc = a.v;
            bool ok;
            if constexpr (PAGED) {
                ok = p >= 0 && p < ctx;
                if (ok) {
                    int page = a.kv.block_table[row * a.kv.max_pages + p / a.kv.page_size];
                    if (page < 0 || page >= a.kv.num_pages) {
                        if (c == 0) record_error(a.hdr, DSA_ERR_INVALID_ARG, (unsigned)row);
                        ok = false;
                    } else {
                        int64_t off = ((int64_t)page * a.kv.page_size + p % a.kv.page_size) * D;
                        ksrc = a.kv.k_cache + off;
                        vsrc = a.kv.v_cache + off;
                    }
                }
            } else {
                ok = p >= 0 && p < a.T;
                if (ok) {
                    ksrc = a.k + (int64_t)p * D;
                    vsrc = a.v + (int64_t)p * D;
                }
            }
            if (!ok) { ksrc = a.q; vsrc = a.q; }       // any valid address; zero-filled
            cp_async_16(kd + aswz<D>(r, c), ksrc + c * 8, ok);
            cp_async_16(vd + aswz<D>(r, c), vsrc + c * 8, ok);
            if (c == 0) valid[stage * AT_BK + r] = ok;
        }
    };
    if (nblk > 0) gather(0, 0);
    cp_async_commit();

    cp_async_wait<1>();
    __syncthreads();
    uint32_t qf[D / 16][4];
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
        int mi = lane >> 3;
        int r = warp * 16 + (mi & 1) * 8 + (lane & 7);
        int c = 2 * kk + (mi >> 1);
        ldmatrix_x4(qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], Qs + aswz<D>(r, c));
    }

    float o[D / 8][4];
#pragma unroll
    for (int i = 0; i < D / 8; ++i) o[i][0] = o[i][1] = o[i][2] = o[i][3] = 0.f;
    float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;

    for (int j = 0; j < nblk; ++j) {
        __syncthreads();                                  // stage (j+1)&1 is free again
        if (j + 1 < nblk) gather(j + 1, (j + 1) & 1);
        cp_async_commit();
        cp_async_wait<1>();
        __syncthreads();
        const uint8_t *Kb = Ks + (j & 1) * AT_BK * ROWB;
        const uint8_t *Vb = Vs + (j & 1) * AT_BK * ROWB;
        const int *vb = valid + (j & 1) * AT_BK;

        float s[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
#pragma unroll
            for (int np = 0; np < 4; ++np) {
                int mi = lane >> 3;
                int key = np * 16 + (mi >> 1) * 8 + (lane & 7);
                int c = 2 * kk + (mi & 1);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(b0, b1, b2, b3, Kb + aswz<D>(key, c));
                mma_bf16_16816(s[2 * np], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b0, b1);
                mma_bf16_16816(s[2 * np + 1], qf[kk][0], qf[kk][1], qf[kk][2], qf[kk][3], b2, b3);
            }
        }
        // scale (log2 domain), mask, row max
        float mx_lo = m_lo, mx_hi = m_hi;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                bool ok = vb[nt * 8 + tig * 2 + e];
                s[nt][e] = ok ? s[nt][e] * a.scale_log2 : -INFINITY;
                s[nt][2 + e] = ok ? s[nt][2 + e] * a.scale_log2 : -INFINITY;
                mx_lo = fmaxf(mx_lo, s[nt][e]);
                mx_hi = fmaxf(mx_hi, s[nt][2 + e]);
            }
        }
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
        mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
        mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
        const float base_lo = mx_lo == -INFINITY ? 0.f : mx_lo;
        const float base_hi = mx_hi == -INFINITY ? 0.f : mx_hi;
        const float al_lo = exp2f(m_lo - base_lo), al_hi = exp2f(m_hi - base_hi);
        m_lo = mx_lo;
        m_hi = mx_hi;
        float rs_lo = 0.f, rs_hi = 0.f;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
            s[nt][0] = exp2f(s[nt][0] - base_lo);
            s[nt][1] = exp2f(s[nt][1] - base_lo);
            s[nt][2] = exp2f(s[nt][2] - base_hi);
            s[nt][3] = exp2f(s[nt][3] - base_hi);
            rs_lo += s[nt][0] + s[nt][1];
            rs_hi += s[nt][2] + s[nt][3];
        }
        l_lo = l_lo * al_lo + rs_lo;
        l_hi = l_hi * al_hi + rs_hi;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            o[i][0] *= al_lo; o[i][1] *= al_lo;
            o[i][2] *= al_hi; o[i][3] *= al_hi;
        }
        // O += P V
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            uint32_t p0 = pack_bf16x2(s[2 * kk][0], s[2 * kk][1]);
            uint32_t p1 = pack_bf16x2(s[2 * kk][2], s[2 * kk][3]);
            uint32_t p2 = pack_bf16x2(s[2 * kk + 1][0], s[2 * kk + 1][1]);
            uint32_t p3 = pack_bf16x2(s[2 * kk + 1][2], s[2 * kk + 1][3]);
#pragma unroll
            for (int dp = 0; dp < D / 16; ++dp) {
                int mi = lane >> 3;
                int key = kk * 16 + (mi & 1) * 8 + (lane & 7);
                int c = 2 * dp + (mi >> 1);
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(b0, b1, b2, b3, Vb + aswz<D>(key, c));
                mma_bf16_16816(o[2 * dp], p0, p1, p2, p3, b0, b1);
                mma_bf16_16816(o[2 * dp + 1], p0, p1, p2, p3, b2, b3);
            }
        }
    }
    cp_async_wait<0>();

    // ---- epilogue ----
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 1);
    l_lo += __shfl_xor_sync(0xffffffffu, l_lo, 2);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 1);
    l_hi += __shfl_xor_sync(0xffffffffu, l_hi, 2);
    const float inv_lo = l_lo > 0.f ? 1.f / l_lo : 0.f;
    const float inv_hi = l_hi > 0.f ? 1.f / l_hi : 0.f;
    const float lse_lo = l_lo > 0.f ? m_lo * kLn2 + logf(l_lo) : -INFINITY;
    const float lse_hi = l_hi > 0.f ? m_hi * kLn2 + logf(l_hi) : -INFINITY;
    const int hl = h0 + warp * 16 + g, hh = hl + 8;
    if (a.splits == 1) {
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            int d = i * 8 + tig * 2;
            if (hl < a.H)
                *reinterpret_cast<uint32_t *>(a.out + (row * a.H + hl) * D + d) =
                    pack_bf16x2(o[i][0] * inv_lo, o[i][1] * inv_lo);
            if (hh < a.H)
                *reinterpret_cast<uint32_t *>(a.out + (row * a.H + hh) * D + d) =
                    pack_bf16x2(o[i][2] * inv_hi, o[i][3] * inv_hi);
        }
        if (a.lse && tig == 0) {
            if (hl < a.H) a.lse[row * a.H + hl] = lse_lo;
            if (hh < a.H) a.lse[row * a.H + hh] = lse_hi;
        }
    } else {
        // partials: o_part [rows, splits, H, D] then lse_part [rows, splits, H]
        float *po = a.part + ((row * a.splits + split) * a.H) * (int64_t)D;
        float *pl = a.part + (int64_t)gridDim.x * a.splits * a.H * D + (row * a.splits + split) * a.H;
#pragma unroll
        for (int i = 0; i < D / 8; ++i) {
            int d = i * 8 + tig * 2;
            if (hl < a.H) {
                po[hl * D + d] = o[i][0] * inv_lo;
                po[hl * D + d + 1] = o[i][1] * inv_lo;
            }
            if (hh < a.H) {
                po[hh * D + d] = o[i][2] * inv_hi;
                po[hh * D + d + 1] = o[i][3] * inv_hi;
            }
        }
        if (tig == 0) {
            if (hl < a.H) pl[hl] = lse_lo;
            if (hh < a.H) pl[hh] = lse_hi;
        }
    }
}

// Merge of split partials: o = sum_i exp(lse_i - lse) o_i, lse = logsumexp_i lse_i.
template <int D>
__global__ void merge_splits_kernel(const float *__restrict__ part, int rows, int splits, int H,
                                    uint16_t *__restrict__ out, float *__restrict__ lse)
{
    const int64_t row = blockIdx.x;
    const int h = blockIdx.y;
    const int d = threadIdx.x;
    const float *pl = part + (int64_t)rows * splits * H * D;
    float mx = -INFINITY;
    for (int i = 0; i < splits; ++i) mx = fmaxf(mx, pl[(row * splits + i) * H + h]);
    float acc = 0.f, den = 0.f;
    if (mx != -INFINITY) {
        for (int i = 0; i < splits; ++i) {
            float li = pl[(row * splits + i) * H + h];
            float wgt = li == -INFINITY ? 0.f : __expf(li - mx);
            den += wgt;
            acc += wgt * part[((row * splits + i) * H + h) * (int64_t)D + d];
        }
    }
    float val = den > 0.f ? acc / den : 0.f;
    __nv_bfloat16 b = __float2bfloat16_rn(val);
    out[(row * H + h) * D + d] = *reinterpret_cast<uint16_t *>(&b);
    if (lse && d == 0) lse[row * H + h] = den > 0.f ? mx + logf(den) : -INFINITY;
}

// The same merge for D = 128 with one warp per (row, head): lane l owns
// dimensions 4l .. 4l+3 (16-byte loads of each split's partial), eight heads
// per 256-thread block, so a decode step's merge is a few waves of blocks.
// Lane i holds split i's log-sum-exp and weight (32 splits a round), and the
// splits' partial rows are loaded eight at a time, all in flight together: the
// merge moves a few MB and is bound by memory latency.
__global__ void __launch_bounds__(256)
merge_splits_warp_kernel(const float *__restrict__ part, int rows, int splits, int H,
                         uint16_t *__restrict__ out, float *__restrict__ lse)
{
    constexpr int D = 128, U = 8;
    grid_dep_wait();                                 // the attention's partials
    const int64_t row = blockIdx.x;
    const int h = blockIdx.y * 8 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (h >= H) return;
    const float *pl = part + (int64_t)rows * splits * H * D + row * splits * H + h;
    const float *po = part + (row * splits * H + h) * (int64_t)D + lane * 4;
    float mx = -INFINITY;
    for (int i0 = 0; i0 < splits; i0 += 32)
        if (i0 + lane < splits) mx = fmaxf(mx, __ldg(pl + (int64_t)(i0 + lane) * H));
#pragma unroll
    for (int o = 16; o; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    float den = 0.f;                                 // this lane's splits' weights
    if (mx != -INFINITY) {
        for (int i0 = 0; i0 < splits; i0 += 32) {
            const float li = i0 + lane < splits ? __ldg(pl + (int64_t)(i0 + lane) * H) : -INFINITY;
            const float wl = li == -INFINITY ? 0.f : __expf(li - mx);
            den += wl;
            const int n = splits - i0 < 32 ? splits - i0 : 32;
            for (int j0 = 0; j0 < n; j0 += U) {
                float4 v[U];
#pragma unroll
                for (int u = 0; u < U; ++u)
                    v[u] = j0 + u < n
                               ? __ldg(reinterpret_cast<const float4 *>(po + (int64_t)(i0 + j0 + u) * H * D))
                               : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
                for (int u = 0; u < U; ++u) {
                    const float wgt = __shfl_sync(0xffffffffu, wl, (j0 + u) & 31);
                    if (j0 + u < n && wgt != 0.f) {  // an empty split's partial is not read into the sum
                        acc.x += wgt * v[u].x; acc.y += wgt * v[u].y;
                        acc.z += wgt * v[u].z; acc.w += wgt * v[u].w;
                    }
                }
            }
        }
    }
#pragma unroll
    for (int o = 16; o; o >>= 1) den += __shfl_xor_sync(0xffffffffu, den, o);
    const float inv = den > 0.f ? 1.f / den : 0.f;
    uint2 packed;
    packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2 *>(out + (row * H + h) * (int64_t)D + lane * 4) = packed;
    if (lse && lane == 0) lse[row * H + h] = den > 0.f ? mx + logf(den) : -INFINITY;
}

// fp32 attention for small shapes: one warp per (query row, head).
__global__ void sparse_attn_f32_kernel(const float *__restrict__ q, const float *__restrict__ k,
                                       const float *__restrict__ v, const int32_t *__restrict__ idx,
                                       int64_t T, int H, int D, int ksel, float sm_scale,
                                       float *__restrict__ out, float *__restrict__ lse)
{
    const int64_t row = blockIdx.x;
    const int h = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (h >= H) return;
    float qv[4], ov[4];
    for (int i = 0; i < 4; ++i) {
        int d = lane + 32 * i;
        qv[i] = d < D ? q[(row * H + h) * D + d] : 0.f;
        ov[i] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    for (int e = 0; e < ksel; ++e) {
        int p = idx[row * ksel + e];
        if (p < 0 || p >= T) continue;
        float dot = 0.f;
        for (int i = 0; i < 4; ++i) {
            int d = lane + 32 * i;
            if (d < D) dot = fmaf(qv[i], k[(int64_t)p * D + d], dot);
        }
        for (int o = 16; o > 0; o >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, o);
        float z = dot * sm_scale;
        float mn = fmaxf(m, z);
        float al = __expf(m - mn), pz = __expf(z - mn);
        l = l * al + pz;
        for (int i = 0; i < 4; ++i) {
            int d = lane + 32 * i;
            ov[i] = ov[i] * al + (d < D ? pz * v[(int64_t)p * D + d] : 0.f);
        }
        m = mn;
    }
    for (int i = 0; i < 4; ++i) {
        int d = lane + 32 * i;
        if (d < D) out[(row * H + h) * D + d] = l > 0.f ? ov[i] / l : 0.f;
    }
    if (lse && lane == 0) lse[row * H + h] = l > 0.f ? m + logf(l) : -INFINITY;
}

}  // namespace

cudaError_t launch_sparse_attn_bf16(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                    const int32_t *idx, int64_t rows, int64_t T, int H, int d,
                                    int ksel, float sm_scale, uint16_t *out, float *lse,
                                    cudaStream_t st)
{
    if (rows <= 0) return cudaSuccess;
    AttnArgs a{};
    a.q = q; a.k = k; a.v = v; a.T = T; a.idx = idx; a.H = H; a.ksel = ksel;
    a.scale_log2 = sm_scale * kLog2e; a.out = out; a.lse = lse;
    a.splits = 1; a.chunk = ksel;
    const int hg = H > 128 ? 128 : H;
    const int nw = (hg + 15) / 16;
    const size_t smem = (size_t)nw * 16 * d * 2 + 4 * AT_BK * d * 2 + 2 * AT_BK * sizeof(int);
    dim3 grid((unsigned)rows, (unsigned)((H + 127) / 128), 1);
    cudaError_t e;
    if (d == 128) {
        e = cudaFuncSetAttribute(sparse_attn_bf16_kernel<128, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        sparse_attn_bf16_kernel<128, false><<<grid, nw * 32, smem, st>>>(a);
    } else {
        e = cudaFuncSetAttribute(sparse_attn_bf16_kernel<64, false>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        sparse_attn_bf16_kernel<64, false><<<grid, nw * 32, smem, st>>>(a);
    }
    return cudaGetLastError();
}

// Index-list splits per decode sequence: as many as keep B x splits items
// within one wave of the B200's 148 SMs (a second, partial wave of items cost
// more than the smaller merge it saves).
int sparse_attn_paged_splits(int B, int ksel)
{
    int max_splits = (ksel + AT_BK - 1) / AT_BK;
    int want = 148 / B;
    int s = want < max_splits ? want : max_splits;
    return s < 1 ? 1 : s;
}

size_t sparse_attn_paged_part_bytes(int B, int H, int d, int splits)
{
    if (splits <= 1) return 0;
    return sizeof(float) * (size_t)B * splits * H * (d + 1);
}

cudaError_t launch_sparse_attn_paged_bf16(const uint16_t *q, const PagedKV &kv,
                                          const int32_t *idx, int B, int H, int d, int ksel,
                                          float sm_scale, uint16_t *out, float *lse,
                                          float *part, int splits, WsHeader *hdr,
                                          cudaStream_t st)
{
    if (B <= 0) return cudaSuccess;
    AttnArgs a{};
    a.q = q; a.kv = kv; a.idx = idx; a.H = H; a.ksel = ksel;
    a.scale_log2 = sm_scale * kLog2e; a.out = out; a.lse = lse; a.part = part;
    a.splits = splits;
    a.chunk = (int)(ceil_div(ceil_div(ksel, splits), AT_BK) * AT_BK);
    a.hdr = hdr;
    const int hg = H > 128 ? 128 : H;
    const int nw = (hg + 15) / 16;
    const size_t smem = (size_t)nw * 16 * d * 2 + 4 * AT_BK * d * 2 + 2 * AT_BK * sizeof(int);
    dim3 grid((unsigned)B, (unsigned)((H + 127) / 128), (unsigned)splits);
    cudaError_t e = cudaFuncSetAttribute(sparse_attn_bf16_kernel<128, true>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    sparse_attn_bf16_kernel<128, true><<<grid, nw * 32, smem, st>>>(a);
    if (splits > 1) {
        dim3 mg((unsigned)B, (unsigned)H);
        merge_splits_kernel<128><<<mg, 128, 0, st>>>(part, B, splits, H, out, lse);
    }
    return cudaGetLastError();
}

cudaError_t launch_merge_splits(const float *part, int rows, int splits, int H, int d, uint16_t *out,
                               float *lse, cudaStream_t st)
{
    if (rows <= 0 || splits <= 1) return cudaSuccess;
    if (d != 128) return cudaErrorNotSupported;
    dim3 mg((unsigned)rows, (unsigned)((H + 7) / 8));
    cudaError_t e = launch_chained(merge_splits_warp_kernel, mg, dim3(256), 0, st, part, rows, splits, H,
                                   out, lse);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

cudaError_t launch_sparse_attn_f32(const float *q, const float *k, const float *v,
                                   const int32_t *idx, int64_t T, int H, int d, int ksel,
                                   float sm_scale, float *out, float *lse, cudaStream_t st)
{
    if (T <= 0) return cudaSuccess;
    sparse_attn_f32_kernel<<<(unsigned)T, H * 32, 0, st>>>(q, k, v, idx, T, H, d, ksel,
                                                          sm_scale, out, lse);
    return cudaGetLastError();
}

}  // namespace dsa
