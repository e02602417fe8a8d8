// Decode-step lightning indexer on the 5th-generation tensor cores.
//
// One new query token per sequence scores every cached token s < n_b:
//   I[s] = ksc[s] * sum_h (w[h] * sq) * ReLU(q8[h,:] . k8[s,:])
// ("DeepSeek-V3.2-Exp 稀疏注意力机制(DSA)技术深度解析", sections 1 and 6: the
// decode path still runs the O(n) indexer per token over FP8 index keys).
//
// The keys are the MMA rows: a tile of 128 cached keys (one or more pages of
// the FP8 index-key cache, fetched by TMA into a 128-byte-swizzled shared
// tile) times the query's H heads gives a 128 x H fp32 accumulator in tensor
// memory (tcgen05.mma kind::f8f6f4, M = 128, N = H, K = 4 x 32).  Each
// epilogue thread owns one key (one TMEM lane), reads its H head products,
// and folds them as sum_h c_h * ReLU(.) with c_h = w[h] * sq, then applies
// the key's scale.  A 4-stage TMA ring keeps the HBM stream going while the
// epilogue of the previous tile runs.  Every mbarrier wait is bounded; on a
// timeout the CTA records DSA_ERR_TIMEOUT, drains its outstanding copies
// (again bounded), frees its tensor memory and returns.
#include "kernels.h"
#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr int DT_STAGES = 4;
constexpr int DT_TILE = 128;                 // keys per tile = UMMA M
constexpr int DT_TILE_BYTES = DT_TILE * 128;
constexpr int DT_TPC = 16;                   // tiles per CTA
constexpr int DT_THREADS = 128;
constexpr int DT_TMEM_COLS = 128;            // two 64-column accumulators

struct DecTcArgs {
    const float *sq;
    const uint16_t *w;
    const float *kscale;
    const int32_t *block_table;
    const int32_t *context_lens;
    int64_t num_pages;
    int max_pages;
    int page_size;
    int box_rows;            // rows per TMA box: min(page_size, 128)
    int64_t max_context;
    float *scores;
    int64_t ld;
    WsHeader *hdr;
};

constexpr size_t dt_smem_bytes()
{
    return 1024 /*align slack*/ + 8192 /*q*/ + (size_t)DT_STAGES * DT_TILE_BYTES + 64 * 4 /*c*/ +
           (DT_STAGES + 3) * 8 + 16;
}

template <int H>
__global__ void __launch_bounds__(DT_THREADS)
decode_index_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap qmap, const DecTcArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *qs = smem;                                         // H x 128 B
    uint8_t *ks = qs + 8192;                                    // stages x 128 x 128 B
    float *cw = reinterpret_cast<float *>(ks + DT_STAGES * DT_TILE_BYTES);
    uint64_t *full = reinterpret_cast<uint64_t *>(cw + 64);
    uint64_t *qbar = full + DT_STAGES;
    uint64_t *mbar = qbar + 1;                                  // [2]: one per accumulator
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(mbar + 2);

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int b = blockIdx.y;
    const int ps = a.page_size;
    const int64_t n = a.context_lens[b];
    if (n < 1 || n > a.max_context || n > (int64_t)a.max_pages * ps) {
        if (blockIdx.x == 0 && tid == 0) record_error(a.hdr, DSA_ERR_INVALID_ARG, (unsigned)b);
        return;
    }
    const int64_t tiles = (n + DT_TILE - 1) / DT_TILE;
    const int64_t t_begin = (int64_t)blockIdx.x * DT_TPC;
    if (t_begin >= tiles) return;
    const int nt = (int)min((int64_t)DT_TPC, tiles - t_begin);
    const int32_t *bt = a.block_table + (int64_t)b * a.max_pages;

    if (warp == 0) {
        tmem_alloc(tmem_slot, DT_TMEM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int s = 0; s < DT_STAGES; ++s) mbar_init(&full[s], 1);
        mbar_init(qbar, 1);
        mbar_init(&mbar[0], 1);
        mbar_init(&mbar[1], 1);
        fence_mbar_init();
    }
    if (tid < H) cw[tid] = bf16_to_f32(a.w[(int64_t)b * H + tid]) * a.sq[b];
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    // Producer (thread 0): one tile = 128 / box_rows TMA boxes, one per page segment.
    int issued = 0;
    auto issue_tile = [&](int j) {
        const int s = j % DT_STAGES;
        const int64_t p0 = (t_begin + j) * DT_TILE;
        const int nseg = DT_TILE / a.box_rows;
        uint32_t bytes = 0;
        for (int seg = 0; seg < nseg; ++seg) {
            int64_t pos = p0 + (int64_t)seg * a.box_rows;
            if (pos >= n) break;
            int page = bt[pos / ps];
            if (page >= 0 && page < a.num_pages) bytes += (uint32_t)a.box_rows * 128;
        }
        mbar_arrive_expect_tx(&full[s], bytes);
        for (int seg = 0; seg < nseg; ++seg) {
            int64_t pos = p0 + (int64_t)seg * a.box_rows;
            if (pos >= n) break;
            int page = bt[pos / ps];
            if (page < 0 || page >= a.num_pages) {
                record_error(a.hdr, DSA_ERR_INVALID_ARG, (unsigned)b);
                continue;
            }
            tma_load_2d(ks + s * DT_TILE_BYTES + seg * a.box_rows * 128, &kmap, &full[s], 0,
                        (int)((int64_t)page * ps + pos % ps));
        }
        ++issued;
    };
    if (tid == 0) {
        tma_prefetch_desc(&kmap);
        tma_prefetch_desc(&qmap);
        mbar_arrive_expect_tx(qbar, H * 128);
        tma_load_2d(qs, &qmap, qbar, 0, b * H);
        for (int j = 0; j < nt && j < DT_STAGES; ++j) issue_tile(j);
    }

    constexpr uint32_t idesc = umma_idesc_e4m3_f32(DT_TILE, H);
    const uint64_t bdesc = umma_desc_k_sw128(smem_u32(qs));
    // thread 0: wait for tile j's keys, then run its MMA into accumulator j & 1
    int consumed = 0, mma_issued = 0;
    auto mma_tile = [&](int j) -> bool {
        const int s = j % DT_STAGES;
        if (!mbar_wait(&full[s], (j / DT_STAGES) & 1)) return false;
        consumed = j + 1;
        tc_fence_after();
        const uint64_t adesc = umma_desc_k_sw128(smem_u32(ks + s * DT_TILE_BYTES));
        const uint32_t d = tmem + (uint32_t)((j & 1) * 64);
#pragma unroll
        for (int k = 0; k < 4; ++k) umma_f8f6f4(d, adesc + 2 * k, bdesc + 2 * k, idesc, k > 0);
        umma_commit(&mbar[j & 1]);
        mma_issued = j + 1;
        return true;
    };
    int bad = 0;
    if (tid == 0) bad = !(mbar_wait(qbar, 0) && mma_tile(0));
    bool failed = __syncthreads_or(bad);
    for (int j = 0; j < nt && !failed; ++j) {
        // this thread's key of tile j, and its scale, fetched while the MMA runs
        const int64_t pos = (t_begin + j) * DT_TILE + warp * 32 + lane;
        float ksc = 0.f;
        bool live = false;
        if (pos < n) {
            int page = bt[pos / ps];
            if (page >= 0 && page < a.num_pages) {
                ksc = a.kscale[(int64_t)page * ps + pos % ps];
                live = true;
            }
        }
        bad = 0;
        if (tid == 0 && j + 1 < nt) bad = !mma_tile(j + 1);
        bad |= !mbar_wait(&mbar[j & 1], (j >> 1) & 1);
        if (__syncthreads_or(bad)) { failed = true; break; }
        tc_fence_after();
        // tile j's MMA is done with its stage: refill it
        if (tid == 0 && j + DT_STAGES < nt) issue_tile(j + DT_STAGES);

        // epilogue: this thread's key = TMEM lane 32*warp + lane, accumulator j & 1
        const uint32_t trow = tmem + ((uint32_t)(warp * 32) << 16) + (uint32_t)((j & 1) * 64);
        float acc = 0.f;
        if constexpr (H % 32 == 0) {
#pragma unroll
            for (int c0 = 0; c0 < H; c0 += 32) {
                uint32_t v[32];
                tmem_ld32(trow + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) acc = fmaf(cw[c0 + i], fmaxf(__uint_as_float(v[i]), 0.f), acc);
            }
        } else {
#pragma unroll
            for (int c0 = 0; c0 < H; c0 += 16) {
                uint32_t v[16];
                tmem_ld16(trow + c0, v);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 16; ++i) acc = fmaf(cw[c0 + i], fmaxf(__uint_as_float(v[i]), 0.f), acc);
            }
        }
        if (live) a.scores[(int64_t)b * a.ld + pos] = acc * ksc;
        tc_fence_before();
        __syncthreads();          // accumulator j & 1 is free for tile j + 2
    }

    if (failed) {
        // wind down: let copies and MMAs already in flight land before the CTA's
        // shared and tensor memory are released (bounded again)
        if (tid == 0) {
            record_error(a.hdr, DSA_ERR_TIMEOUT, (unsigned)b);
            for (int j = consumed; j < issued; ++j) mbar_wait(&full[j % DT_STAGES], (j / DT_STAGES) & 1);
            for (int j = (mma_issued >= 2 ? mma_issued - 2 : 0); j < mma_issued; ++j)
                mbar_wait(&mbar[j & 1], (j >> 1) & 1);
        }
        tc_fence_before();
        __syncthreads();
    }
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, DT_TMEM_COLS);
}

}  // namespace

bool decode_index_tc_supported(int H, int page_size)
{
    bool h_ok = H == 16 || H == 32 || H == 48 || H == 64;
    bool p_ok = page_size == 16 || page_size == 32 || page_size == 64 || page_size == 128 ||
                (page_size > 128 && page_size % 128 == 0);
    return h_ok && p_ok;
}

cudaError_t launch_decode_index_tc(const uint8_t *q8, const float *sq, const uint16_t *w,
                                   const uint8_t *kidx, const float *kscale,
                                   const int32_t *block_table, const int32_t *context_lens,
                                   int64_t num_pages, int max_pages, int page_size, int B,
                                   int64_t max_context, int H, float *scores, int64_t ld,
                                   WsHeader *hdr, cudaStream_t st)
{
    if (B <= 0) return cudaSuccess;
    if (!decode_index_tc_supported(H, page_size)) return cudaErrorNotSupported;
    if ((int64_t)num_pages * page_size >= ((int64_t)1 << 31) || (int64_t)B * H >= ((int64_t)1 << 31))
        return cudaErrorNotSupported;
    CUtensorMap kmap, qmap;
    const int box_rows = page_size < DT_TILE ? page_size : DT_TILE;
    uint64_t kd[2] = {128, (uint64_t)num_pages * page_size}, kst[1] = {128};
    uint32_t kb[2] = {128, (uint32_t)box_rows};
    uint64_t qd[2] = {128, (uint64_t)B * H}, qst[1] = {128};
    uint32_t qb[2] = {128, (uint32_t)H};
    if (!make_tmap_u8(&kmap, kidx, 2, kd, kst, kb) || !make_tmap_u8(&qmap, q8, 2, qd, qst, qb))
        return cudaErrorNotSupported;
    DecTcArgs a{sq, w, kscale, block_table, context_lens, num_pages, max_pages, page_size, box_rows,
                max_context, scores, ld, hdr};
    const int64_t tiles = ceil_div(max_context, DT_TILE);
    dim3 grid((unsigned)ceil_div(tiles, DT_TPC), (unsigned)B);
    const size_t smem = dt_smem_bytes();
    cudaError_t e;
#define DT_CASE(HV)                                                                              \
    case HV:                                                                                     \
        e = cudaFuncSetAttribute(decode_index_tc_kernel<HV>,                                      \
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);        \
        if (e != cudaSuccess) return e;                                                          \
        decode_index_tc_kernel<HV><<<grid, DT_THREADS, smem, st>>>(kmap, qmap, a);               \
        break;
    switch (H) {
        DT_CASE(16) DT_CASE(32) DT_CASE(48) DT_CASE(64)
    default: return cudaErrorNotSupported;
    }
#undef DT_CASE
    return cudaGetLastError();
}

}  // namespace dsa
