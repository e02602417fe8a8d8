// Lightning-indexer scores on the 5th-generation tensor cores (tcgen05).
//
//   I[t,s] = sk[s] * sum_h c[t,h] * ReLU(q8[t,h,:] . k8[s,:]),  c[t,h] = w[t,h] * sq[t]
// ("DeepSeek-V3.2-Exp 稀疏注意力机制(DSA)技术深度解析", section 1: few heads,
// index_head_dim 128, FP8, ReLU; the indexer is O(n^2) but cheap per pair).
//
// Persistent, warp-specialised CTA (one per SM) sweeping the causal
// (128 query rows x 256 keys) work tiles:
//   warp 0    TMA producer: the key tile (256 x 128 B, kept for all heads,
//             double-buffered across work tiles) and one 128 x 128 B query
//             tile per head through a 4-stage ring (128-byte swizzle);
//   warp 1    MMA issuer (one thread): per head, 4 x tcgen05.mma kind::f8f6f4
//             (M = 128 query rows, N = 256 keys, K = 32) into one of two
//             256-column fp32 accumulators in tensor memory;
//   warps 4-11 epilogue: TMEM lane = query row; each warp reads half the
//             columns of its lane quarter and folds c[t,h] * ReLU(acc) into
//             128 running scores held in registers, so the per-head products
//             never leave the SM; after the last head the key scales are
//             applied and the causal part of the tile is stored.
// Three epilogue modes share the products and the fold:
//   scores  store the causal scores (the stage entry point, and the prefill's
//           repair of rows whose fused selection failed: then only the row
//           blocks flagged by the selection are visited, and nothing at all
//           when none was flagged);
//   sample  the same over a gathered sample of the keys (one per block of S
//           positions), for the per-row threshold of the fused selection;
//   select  the fused selection: each score of a competing position that is
//           at or above its row's threshold tau is appended, as (score bits,
//           position), to the row's candidate list; the scores themselves
//           never leave the SM.
// Every mbarrier wait is bounded; a timeout records DSA_ERR_TIMEOUT, makes
// every role stop at its next wait, and the CTA still frees its tensor memory.
#include <algorithm>
#include <cstring>

#include "kernels.h"
#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr int IT_BM = 128;                    // query rows per work tile (UMMA M)
constexpr int IT_BN = 256;                    // keys per work tile (UMMA N)
constexpr int IT_QSTAGES = 3;
constexpr int IT_KSTAGES = 2;
constexpr int IT_EPI_WARPS = 8;
constexpr int IT_THREADS = 32 * (4 + IT_EPI_WARPS);   // warpgroup 0: producer, MMA, 2 coefficient warps
// Register split (setmaxnreg): the kernel is built for 168 registers x 384
// threads = 64512; warpgroup 0 gives up to 56 and the two epilogue warpgroups
// take 224: 128 x 56 + 256 x 224 = 64512, the launch's own total.
constexpr int IT_LAUNCH_REGS = 168;
constexpr int IT_REGS_LOW = 56;
constexpr int IT_REGS_HIGH = 224;
static_assert(128 * IT_REGS_LOW + 256 * IT_REGS_HIGH <= IT_LAUNCH_REGS * IT_THREADS, "register split");
constexpr int IT_QBYTES = IT_BM * 128;        // 16 KB
constexpr int IT_KBYTES = IT_BN * 128;        // 32 KB
constexpr int IT_CS_STRIDE = IT_BM + 1;       // padded row of the c table (bank spread)
constexpr int IT_MAX_H = 64;

struct IdxTcArgs {
    const float *sq;
    const float *sk;             // key scales, [nkeys]
    const uint16_t *w;
    int64_t T;                   // positions of the sequence (keys of the scores epilogue)
    int64_t q_base;              // q8, sq and w hold positions [q_base, q_base + q rows)
    int64_t nkeys;               // keys of kmap and sk (T, or the sample count)
    int H;
    int mode;                    // IT_SCORES, IT_SAMPLE, IT_SELECT
    int window;                  // sample, select: positions past t - window do not compete
    int sample_stride;           // sample: S
    // select
    const float *tau;            // [row_count] thresholds
    uint2 *cand;                 // [row_count][cap] (score bits, position)
    uint32_t *cand_cnt;          // [row_count * kCandCntStride]
    int cap;
    // scores: visit only the row blocks whose rb_mask entry is set (nullable),
    // and nothing at all when *any is 0 (nullable)
    const uint32_t *rb_mask;
    const uint32_t *any;
    int64_t row_begin, row_count;
    int64_t n_rb;                // 128-row blocks in [row_begin, row_begin + row_count)
    float *out;
    int64_t ld;
    int vec_store;               // ld % 4 == 0 and out 16-byte aligned
    int tma_store;               // tiles wholly below the diagonal leave through TMA stores (omap)
    WsHeader *hdr;
    int stall_at;                // test hook: CTA 0's producer stops before query copy stall_at (-1: off)
};

struct SmemLayout {
    static constexpr size_t k_off = 0;
    static constexpr size_t q_off = k_off + (size_t)IT_KSTAGES * IT_KBYTES;
    static constexpr size_t stg_off = q_off + (size_t)IT_QSTAGES * IT_QBYTES;    // [8 warps] 32 x 32 fp32 store staging
    static constexpr size_t c_off = stg_off + (size_t)IT_EPI_WARPS * 4096;       // [2] c tables
    static constexpr size_t sk_off = c_off + 2 * sizeof(float) * IT_MAX_H * IT_CS_STRIDE;   // [2] key scales
    static constexpr size_t tau_off = sk_off + 2 * sizeof(float) * IT_BN;                // [2] row thresholds
    static constexpr size_t bar_off = tau_off + 2 * sizeof(float) * IT_BM;
    static constexpr int n_bars = 2 * IT_KSTAGES + 2 * IT_QSTAGES + 4 + 4;
    static constexpr size_t slot_off = bar_off + 8 * n_bars;
    static constexpr size_t total = slot_off + 16 + 1024;   // + alignment slack
};

// Keys [0, key_limit) of the key tensor that row t scores: s <= t for the
// scores; for the sample and the selection, the positions before the row's
// window, n_t = max(0, t + 1 - window): all of them (select) or the samples
// among them (sample).  Nondecreasing in t.
__host__ __device__ __forceinline__ int64_t key_limit(int mode, int window, int S, int64_t t)
{
    if (mode == IT_SCORES) return t + 1;
    const int64_t n = t + 1 - window > 0 ? t + 1 - window : 0;
    return mode == IT_SAMPLE ? sample_count(n, S) : n;
}

// Walks the causal work tiles of the row range in (row block, key tile) order.
template <int MODE>
struct TileWalk {
    int64_t rb = 0, kt = 0;
    __device__ __forceinline__ static int64_t tiles_of(const IdxTcArgs &a, int64_t rb)
    {
        if (MODE == IT_SCORES && a.rb_mask && a.rb_mask[rb] == 0u) return 0;
        int64_t last = min(a.row_begin + rb * IT_BM + IT_BM - 1, a.row_begin + a.row_count - 1);
        return ceil_div(key_limit(MODE, a.window, a.sample_stride, last), IT_BN);
    }
    __device__ __forceinline__ bool normalise(const IdxTcArgs &a)
    {
        while (rb < a.n_rb) {
            int64_t nk = tiles_of(a, rb);
            if (kt < nk) return true;
            kt -= nk;
            ++rb;
        }
        return false;
    }
    __device__ __forceinline__ bool start(const IdxTcArgs &a, int64_t idx) { rb = 0; kt = idx; return normalise(a); }
    __device__ __forceinline__ bool next(const IdxTcArgs &a, int64_t step) { kt += step; return normalise(a); }
};

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer_ns();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort = 1;
            return false;
        }
    }
}

// MODE: the epilogue (IT_SCORES, IT_SAMPLE, IT_SELECT), one instantiation each
// so that each carries only its own epilogue's registers.
template <int MODE>
__global__ void __launch_bounds__(IT_THREADS, 1)
index_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap omap, const IdxTcArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *Ks = smem + SmemLayout::k_off;
    uint8_t *Qs = smem + SmemLayout::q_off;
    float *Cs = reinterpret_cast<float *>(smem + SmemLayout::c_off);
    uint8_t *Stg = smem + SmemLayout::stg_off;
    float *Sk = reinterpret_cast<float *>(smem + SmemLayout::sk_off);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + SmemLayout::bar_off);
    uint64_t *kfull = bars, *kempty = bars + IT_KSTAGES;
    uint64_t *qfull = bars + 2 * IT_KSTAGES, *qempty = qfull + IT_QSTAGES;
    uint64_t *tfull = qempty + IT_QSTAGES, *tempty = tfull + 2;
    uint64_t *cfull = tempty + 2, *cempty = cfull + 2;     // per work tile: c table and key scales
    float *Tau = reinterpret_cast<float *>(smem + SmemLayout::tau_off);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + SmemLayout::slot_off);
    __shared__ volatile int abort_flag;
    // progress of the producer and the MMA issuer, for the wind-down after an abort
    __shared__ int q_issued, k_issued, q_consumed, k_consumed, mma_heads;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int H = a.H;
    const int64_t row_end = a.row_begin + a.row_count;
    if (a.any && *a.any == 0u) return;           // a repair launch with nothing to repair

    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < IT_KSTAGES; ++i) { mbar_init(&kfull[i], 1); mbar_init(&kempty[i], 1); }
        for (int i = 0; i < IT_QSTAGES; ++i) { mbar_init(&qfull[i], 1); mbar_init(&qempty[i], 1); }
        for (int i = 0; i < 2; ++i) { mbar_init(&tfull[i], 1); mbar_init(&tempty[i], IT_EPI_WARPS); }
        for (int i = 0; i < 2; ++i) { mbar_init(&cfull[i], 2); mbar_init(&cempty[i], IT_EPI_WARPS); }
        abort_flag = 0;
        q_issued = k_issued = q_consumed = k_consumed = mma_heads = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    if (warp < 4) {
        // warpgroup 0 (warps 0-3): producer, MMA issuer, two coefficient warps
        regs_dec<IT_REGS_LOW>();
        if (warp == 0) {
            // ------------------------------------------------ TMA producer
            if (lane == 0) {
                tma_prefetch_desc(&qmap);
                tma_prefetch_desc(&kmap);
                // The per-head path is kept to a few instructions (stage and phase
                // advance incrementally; progress is published once, at the end): this
                // warp shares its scheduler with two busy epilogue warps.
                TileWalk<MODE> tw;
                int lt = 0, qst = 0, qi = 0;
                uint32_t qph = 0;
                for (bool ok = tw.start(a, blockIdx.x); ok; ok = tw.next(a, gridDim.x), ++lt) {
                    const int kb = lt & 1;
                    if (!wait_or_abort(&kempty[kb], ((lt >> 1) & 1) ^ 1, &abort_flag)) break;
                    mbar_arrive_expect_tx(&kfull[kb], IT_KBYTES);
                    tma_load_2d(Ks + kb * IT_KBYTES, &kmap, &kfull[kb], 0, (int)(tw.kt * IT_BN));
                    k_issued = lt + 1;
                    const int tq = (int)(a.row_begin + tw.rb * IT_BM - a.q_base);
                    bool stop = false;
                    for (int h = 0; h < H; ++h) {
                        if (qi == a.stall_at && blockIdx.x == 0) { stop = true; break; }   // test hook
                        if (!wait_or_abort(&qempty[qst], qph ^ 1, &abort_flag)) { stop = true; break; }
                        mbar_arrive_expect_tx(&qfull[qst], IT_QBYTES);
                        tma_load_3d(Qs + qst * IT_QBYTES, &qmap, &qfull[qst], 0, h, tq);
                        ++qi;
                        if (++qst == IT_QSTAGES) { qst = 0; qph ^= 1; }
                    }
                    if (stop) break;
                }
                q_issued = qi;
            }
        } else if (warp == 1) {
            // ------------------------------------------------ MMA issuer
            if (lane == 0) {
                // Lean per-head path, as for the producer: stage, accumulator and
                // phases advance incrementally, the query-tile descriptors are
                // precomputed, and the progress for the abort drain is published once.
                constexpr uint32_t idesc = umma_idesc_e4m3_f32(IT_BM, IT_BN);
                const uint64_t qdesc0 = umma_desc_k_sw128(smem_u32(Qs));
                constexpr uint64_t kQStep = (uint64_t)(IT_QBYTES >> 4);   // descriptor address units
                TileWalk<MODE> tw;
                int lt = 0, qst = 0, acc = 0, qdone = 0, issued = 0;
                uint32_t qph = 0, aph = 0;
                for (bool ok = tw.start(a, blockIdx.x); ok; ok = tw.next(a, gridDim.x), ++lt) {
                    const int kb = lt & 1;
                    if (!wait_or_abort(&kfull[kb], (lt >> 1) & 1, &abort_flag)) break;
                    k_consumed = lt + 1;
                    const uint64_t bdesc = umma_desc_k_sw128(smem_u32(Ks + kb * IT_KBYTES));
                    bool stop = false;
                    for (int h = 0; h < H; ++h) {
                        if (!wait_or_abort(&qfull[qst], qph, &abort_flag)) { stop = true; break; }
                        ++qdone;
                        if (!wait_or_abort(&tempty[acc], aph ^ 1, &abort_flag)) { stop = true; break; }
                        tc_fence_after();
                        const uint64_t adesc = qdesc0 + (uint64_t)qst * kQStep;
                        const uint32_t d = tmem + (uint32_t)(acc * IT_BN);
                        umma_f8f6f4(d, adesc, bdesc, idesc, 0u);
    #pragma unroll
                        for (int k = 1; k < 4; ++k) umma_f8f6f4(d, adesc + 2 * k, bdesc + 2 * k, idesc, 1u);
                        umma_commit(&qempty[qst]);
                        umma_commit(&tfull[acc]);
                        ++issued;
                        if (++qst == IT_QSTAGES) { qst = 0; qph ^= 1; }
                        acc ^= 1;
                        aph ^= (uint32_t)(acc == 0);
                    }
                    if (stop) break;
                    umma_commit(&kempty[kb]);
                }
                q_consumed = qdone;
                mma_heads = issued;
            }
        } else {
            // ------------------------------------------------ coefficient warps (2, 3)
            // One work tile ahead of the epilogue: the c table c[t,h] = w[t,h] * sq[t]
            // of the tile's query rows and its 256 key scales, into one of two buffers.
            const int ct = tid - 64;                       // 0..63
            const bool wvec = (H % 8) == 0 && (reinterpret_cast<uintptr_t>(a.w) & 15u) == 0;
            TileWalk<MODE> tw;
            int lt = 0;
            for (bool ok = tw.start(a, blockIdx.x); ok; ok = tw.next(a, gridDim.x), ++lt) {
                const int cb = lt & 1;
                if (!__all_sync(0xffffffffu, wait_or_abort(&cempty[cb], ((lt >> 1) & 1) ^ 1, &abort_flag))) break;
                const int64_t t0 = a.row_begin + tw.rb * IT_BM;
                const int64_t s0 = tw.kt * IT_BN;
                float *cs = Cs + cb * IT_MAX_H * IT_CS_STRIDE;
                if (wvec) {
                    // thread = query row (two per thread): its H weights in 16-byte loads, four
                    // in flight at a time, so a table costs a few memory latencies
                    for (int r = ct; r < IT_BM; r += 64) {
                        const int64_t t = t0 + r;
                        const bool in = t < row_end;
                        const float sqv = in ? a.sq[t - a.q_base] : 0.f;
                        const uint4 *wr = reinterpret_cast<const uint4 *>(a.w + (in ? t - a.q_base : 0) * H);
                        for (int j0 = 0; j0 < H / 8; j0 += 4) {
                            uint4 u[4];
#pragma unroll
                            for (int j = 0; j < 4; ++j) u[j] = j0 + j < H / 8 && in ? __ldg(wr + j0 + j) : make_uint4(0, 0, 0, 0);
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                if (j0 + j >= H / 8) break;
                                const uint32_t wv[4] = {u[j].x, u[j].y, u[j].z, u[j].w};
#pragma unroll
                                for (int e = 0; e < 4; ++e) {
                                    const int h = (j0 + j) * 8 + 2 * e;
                                    cs[h * IT_CS_STRIDE + r] = __uint_as_float(wv[e] << 16) * sqv;
                                    cs[(h + 1) * IT_CS_STRIDE + r] = __uint_as_float(wv[e] & 0xffff0000u) * sqv;
                                }
                            }
                        }
                    }
                } else {
                    for (int i = ct; i < IT_BM * H; i += 64) {
                        const int r = i / H, h = i % H;
                        const int64_t t = t0 + r;
                        cs[h * IT_CS_STRIDE + r] =
                            t < row_end ? bf16_to_f32(a.w[(t - a.q_base) * H + h]) * a.sq[t - a.q_base] : 0.f;
                    }
                }
                for (int i = ct; i < IT_BN; i += 64) Sk[cb * IT_BN + i] = s0 + i < a.nkeys ? a.sk[s0 + i] : 0.f;
                if constexpr (MODE == IT_SELECT)
                    for (int i = ct; i < IT_BM; i += 64)
                        Tau[cb * IT_BM + i] = t0 + i < row_end ? a.tau[t0 + i - a.row_begin] : INFINITY;
                __syncwarp();
                if (lane == 0) mbar_arrive(&cfull[cb]);    // releases the tables to the epilogue
            }
        }
    } else {
        regs_inc<IT_REGS_HIGH>();
        // ------------------------------------------------ epilogue (8 warps)
        const int et = tid - 128;                    // 0..255
        const int quarter = warp & 3;                // TMEM lane quarter this warp may access
        const int half = (warp - 4) >> 2;            // column half: 0 for warps 4-7, 1 for 8-11
        const int row = quarter * 32 + lane;         // query row within the tile = TMEM lane
        const uint32_t tlane = tmem + ((uint32_t)(quarter * 32) << 16) + (uint32_t)(half * 128);
        TileWalk<MODE> tw;
        int lt = 0;
        bool dead = false;   // after an abort: stop (every wait below is bounded)
        for (bool ok = tw.start(a, blockIdx.x); ok && !dead; ok = tw.next(a, gridDim.x), ++lt) {
            const int64_t t0 = a.row_begin + tw.rb * IT_BM;
            const int64_t s0 = tw.kt * IT_BN;
            const int cb = lt & 1;
            if (!__all_sync(0xffffffffu, wait_or_abort(&cfull[cb], (lt >> 1) & 1, &abort_flag))) { dead = true; break; }
            const float *cs = Cs + cb * IT_MAX_H * IT_CS_STRIDE;

            uint64_t sc[64];                         // running scores, column pairs (2i, 2i+1)
#pragma unroll
            for (int i = 0; i < 64; ++i) sc[i] = 0ull;
            for (int h = 0; h < H; ++h) {
                const int g = lt * H + h, acc = g & 1;
                // warp-uniform outcome: the TMEM loads below are warp-collective
                const bool ok = wait_or_abort(&tfull[acc], (g >> 1) & 1, &abort_flag);
                if (!__all_sync(0xffffffffu, ok)) { dead = true; break; }
                tc_fence_after();
                // c = w[t,h] * sq[t]; the odd column of each pair takes the ReLU as
                // (x + |x|) = 2 ReLU(x), an add on the FMA pipe instead of a max on the
                // ALU pipe, with 0.5 c: 0.5c * 2r = c r exactly, one rounding as before
                const float c = cs[h * IT_CS_STRIDE + row];
                const uint64_t cc = f2_pack(c, 0.5f * c);
                const uint32_t base = tlane + (uint32_t)(acc * IT_BN);
                // 8 chunks of 16 columns; the load of chunk i+1 overlaps the math of chunk i
                uint32_t va[16], vb[16];
                tmem_ld16(base, va);
                tmem_wait_ld_dep16(va);
#pragma unroll
                for (int ch = 0; ch < 8; ch += 2) {
                    tmem_ld16(base + (uint32_t)((ch + 1) * 16), vb);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        sc[ch * 8 + i] = f2_fma(cc, f2_pack(fmaxf(__uint_as_float(va[2 * i]), 0.f),
                                                            __uint_as_float(va[2 * i + 1]) +
                                                                fabsf(__uint_as_float(va[2 * i + 1]))),
                                                sc[ch * 8 + i]);
                    tmem_wait_ld_dep16(vb);
                    if (ch + 2 < 8) tmem_ld16(base + (uint32_t)((ch + 2) * 16), va);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        sc[(ch + 1) * 8 + i] = f2_fma(cc, f2_pack(fmaxf(__uint_as_float(vb[2 * i]), 0.f),
                                                                  __uint_as_float(vb[2 * i + 1]) +
                                                                      fabsf(__uint_as_float(vb[2 * i + 1]))),
                                                      sc[(ch + 1) * 8 + i]);
                    if (ch + 2 < 8) tmem_wait_ld_dep16(va);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&tempty[acc]);
            }
            if (dead) break;
            // key scales, causal mask, store
            const int64_t t = t0 + row;
            if constexpr (MODE == IT_SELECT) {
                if (t < row_end) {
                    // the competing positions [0, kl) at or above the row's threshold
                    const int64_t kl = key_limit(IT_SELECT, a.window, 0, t);
                    const float tau = Tau[cb * IT_BM + row];
                    const int64_t sb = s0 + half * 128;
                    // columns [0, lim) of this thread's 128 compete
                    const int lim = (int)max((int64_t)0, min(kl - sb, (int64_t)128));
                    const uint32_t sb32 = (uint32_t)sb;
                    const float *skh = Sk + cb * IT_BN + half * 128;
                    uint32_t fl[4];
                    uint32_t n = 0;
#pragma unroll
                    for (int wd = 0; wd < 4; ++wd) {
                        uint32_t f = 0;
#pragma unroll
                        for (int i = 0; i < 16; ++i) {
                            const int j = wd * 16 + i;               // column pair 2j, 2j + 1
                            float v0, v1;
                            f2_unpack(sc[j], v0, v1);
                            v0 *= skh[2 * j];
                            v1 *= skh[2 * j + 1];
                            f |= (uint32_t)(v0 >= tau && 2 * j < lim) << (2 * i);
                            f |= (uint32_t)(v1 >= tau && 2 * j + 1 < lim) << (2 * i + 1);
                        }
                        fl[wd] = f;
                        n += (uint32_t)__popc(f);
                    }
                    if (n) {
                        const int64_t r = t - a.row_begin;
                        uint32_t slot = atomicAdd(a.cand_cnt + r * kCandCntStride, n);
                        uint2 *dst = a.cand + r * (int64_t)a.cap;
                        // each 32-column word with candidates: its scaled scores go to this
                        // lane's row of the warp's staging buffer (16-byte chunks swizzled
                        // by the lane), then the candidates are read back by bit position
                        uint8_t *mine = Stg + (warp - 4) * 4096 + lane * 128;
#pragma unroll
                        for (int wd = 0; wd < 4; ++wd) {
                            uint32_t f = fl[wd];
                            if (f == 0u) continue;
#pragma unroll
                            for (int q = 0; q < 8; ++q) {
                                float v0, v1, v2, v3;
                                f2_unpack(sc[wd * 16 + 2 * q], v0, v1);
                                f2_unpack(sc[wd * 16 + 2 * q + 1], v2, v3);
                                const float *kv = skh + wd * 32 + q * 4;
                                *reinterpret_cast<float4 *>(mine + ((q ^ (lane & 7)) << 4)) =
                                    make_float4(v0 * kv[0], v1 * kv[1], v2 * kv[2], v3 * kv[3]);
                            }
                            while (f) {
                                const int i = __ffs(f) - 1;
                                f &= f - 1;
                                const float v = *reinterpret_cast<const float *>(
                                    mine + (((i >> 2) ^ (lane & 7)) << 4) + (i & 3) * 4);
                                // past the capacity only the count grows: the row then fails
                                if (slot < (uint32_t)a.cap)
                                    dst[slot] = make_uint2(__float_as_uint(v), sb32 + (uint32_t)(wd * 32 + i));
                                ++slot;
                            }
                        }
                    }
                }
            } else if (MODE == IT_SCORES && a.tma_store && s0 + IT_BN - 1 <= t0) {
                // every key of the tile is at or below every row: the warp's 32 rows x 128
                // keys leave as four 32 x 32 tiles through shared memory and TMA stores
                // (coalesced, asynchronous; rows and keys past the ends are clipped)
                uint8_t *stg = Stg + (warp - 4) * 4096;
                const float *skh = Sk + cb * IT_BN + half * 128;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    if (lane == 0) bulk_wait_group_read<0>();   // the last store has read the staging
                    __syncwarp();
#pragma unroll
                    for (int j = 0; j < 8; ++j) {          // row `lane`, 16-byte chunk j, 128-byte swizzle
                        float v0, v1, v2, v3;
                        f2_unpack(sc[c * 16 + 2 * j], v0, v1);
                        f2_unpack(sc[c * 16 + 2 * j + 1], v2, v3);
                        const float *kv = skh + c * 32 + j * 4;
                        *reinterpret_cast<float4 *>(stg + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                            make_float4(v0 * kv[0], v1 * kv[1], v2 * kv[2], v3 * kv[3]);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tma_store_2d(&omap, stg, (int)(s0 + half * 128 + c * 32),
                                     (int)(t0 - a.row_begin + quarter * 32));
                        bulk_commit_group();
                    }
                }
            } else if (t < row_end) {
                // keys [0, kl) of this row: s <= t, or the samples before the window
                const int64_t kl = key_limit(MODE, a.window, a.sample_stride, t);
                float *orow = a.out + (t - a.row_begin) * a.ld;
                const int64_t sb = s0 + half * 128;
                const float *skh = Sk + cb * IT_BN + half * 128;
#pragma unroll
                for (int j4 = 0; j4 < 32; ++j4) {
                    const int64_t s = sb + j4 * 4;
                    float v0, v1, v2, v3;
                    f2_unpack(sc[2 * j4], v0, v1);
                    f2_unpack(sc[2 * j4 + 1], v2, v3);
                    v0 *= skh[j4 * 4]; v1 *= skh[j4 * 4 + 1]; v2 *= skh[j4 * 4 + 2]; v3 *= skh[j4 * 4 + 3];
                    if (a.vec_store && s + 3 < kl) {
                        *reinterpret_cast<float4 *>(orow + s) = make_float4(v0, v1, v2, v3);
                    } else {
                        if (s < kl) orow[s] = v0;
                        if (s + 1 < kl) orow[s + 1] = v1;
                        if (s + 2 < kl) orow[s + 2] = v2;
                        if (s + 3 < kl) orow[s + 3] = v3;
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&cempty[cb]);        // done with this tile's c table and key scales
        }
        if (lane == 0) bulk_wait_group<0>();               // stores complete before shared memory goes
    }

    tc_fence_before();
    __syncthreads();
    if (abort_flag && tid == 0) {
        record_error(a.hdr, DSA_ERR_TIMEOUT, blockIdx.x);
        // let the TMA copies and MMAs still in flight land before the shared and
        // tensor memory are released (each wait bounded)
        for (int g = q_consumed; g < q_issued; ++g) mbar_wait(&qfull[g % IT_QSTAGES], (g / IT_QSTAGES) & 1);
        for (int l = k_consumed; l < k_issued; ++l) mbar_wait(&kfull[l & 1], (l >> 1) & 1);
        if (mma_heads > 0) mbar_wait(&tfull[(mma_heads - 1) & 1], ((mma_heads - 1) >> 1) & 1);
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

// -inf above the diagonal of the stage output (s > t, s < T).
__global__ void fill_upper_kernel(float *out, int64_t ld, int64_t T, int64_t row_begin)
{
    const int64_t r = blockIdx.y;
    const int64_t t = row_begin + r;
    for (int64_t s = t + 1 + (int64_t)blockIdx.x * blockDim.x + threadIdx.x; s < T;
         s += (int64_t)gridDim.x * blockDim.x)
        out[r * ld + s] = -INFINITY;
}

// Sample j of the index keys (position sample_pos(j, S)) into row j of ks,
// its scale into sks[j]: one thread per 16-byte chunk of a 128-byte key.
__global__ void gather_samples_kernel(const uint4 *__restrict__ k8, const float *__restrict__ sk, int64_t M, int S,
                                      uint4 *__restrict__ ks, float *__restrict__ sks)
{
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    const int64_t j = i >> 3;
    const int c = (int)(i & 7);
    if (j >= M) return;
    const int64_t p = sample_pos(j, S);
    ks[j * 8 + c] = __ldg(k8 + p * 8 + c);
    if (c == 0) sks[j] = __ldg(sk + p);
}

}  // namespace

cudaError_t launch_gather_samples(const uint8_t *k8, const float *sk, int64_t M, int S, uint8_t *ks,
                                  float *sks, cudaStream_t st)
{
    if (M <= 0) return cudaSuccess;
    const int64_t threads = M * 8;
    gather_samples_kernel<<<(unsigned)ceil_div(threads, 256), 256, 0, st>>>(
        reinterpret_cast<const uint4 *>(k8), sk, M, S, reinterpret_cast<uint4 *>(ks), sks);
    return cudaGetLastError();
}

bool index_tc_supported(int H) { return H >= 1 && H <= IT_MAX_H; }

cudaError_t launch_index_tc(const uint8_t *q8, const float *sq, const uint8_t *k8, const float *sk,
                            const uint16_t *w, int64_t T, int H, int64_t row_begin,
                            int64_t row_count, float *out, int64_t ld, bool write_upper,
                            WsHeader *hdr, cudaStream_t st, const IndexTcOpts *opts)
{
    const IndexTcOpts o = opts ? *opts : IndexTcOpts{};
    if (row_count <= 0) return cudaSuccess;
    const int64_t nkeys = o.nkeys > 0 ? o.nkeys : T;
    if (!index_tc_supported(H) || T >= ((int64_t)1 << 31) || nkeys >= ((int64_t)1 << 31)) return cudaErrorNotSupported;
    if (o.mode == IT_SAMPLE && (o.sample_stride < 1 || (o.sample_stride & (o.sample_stride - 1)))) return cudaErrorInvalidValue;
    if (o.mode == IT_SELECT && (!o.tau || !o.cand || !o.cand_cnt || o.cap < 1)) return cudaErrorInvalidValue;
    CUtensorMap qmap, kmap;
    // q8/sq/w: positions [q_base, q_base + q_rows); the rows scored must lie inside
    const int64_t q_rows = o.q_rows > 0 ? o.q_rows : T - o.q_base;
    if (o.q_base < 0 || row_begin < o.q_base || row_begin + row_count > o.q_base + q_rows) return cudaErrorInvalidValue;
    uint64_t qd[3] = {128, (uint64_t)H, (uint64_t)q_rows}, qs[2] = {128, (uint64_t)H * 128};
    uint32_t qb[3] = {128, 1, (uint32_t)IT_BM};
    uint64_t kd[2] = {128, (uint64_t)nkeys}, ks[1] = {128};
    uint32_t kb[2] = {128, (uint32_t)IT_BN};
    if (!make_tmap_u8(&qmap, q8, 3, qd, qs, qb) || !make_tmap_u8(&kmap, k8, 2, kd, ks, kb))
        return cudaErrorNotSupported;
    IdxTcArgs a{};
    a.sq = sq; a.sk = sk; a.w = w; a.T = T; a.q_base = o.q_base; a.nkeys = nkeys; a.H = H;
    a.row_begin = row_begin; a.row_count = row_count;
    a.mode = o.mode; a.window = o.window; a.sample_stride = o.sample_stride;
    a.tau = o.tau; a.cand = o.cand; a.cand_cnt = o.cand_cnt; a.cap = o.cap;
    a.rb_mask = o.rb_mask; a.any = o.any;
    a.n_rb = ceil_div(row_count, IT_BM);
    a.out = out; a.ld = ld;
    a.vec_store = out && (ld % 4 == 0) && ((reinterpret_cast<uintptr_t>(out) & 15u) == 0);
    CUtensorMap omap;
    std::memset(&omap, 0, sizeof(omap));
    a.tma_store = o.mode == IT_SCORES && a.vec_store && row_count < ((int64_t)1 << 31) &&
                  make_tmap_f32_2d(&omap, out, (uint64_t)T, (uint64_t)row_count, (uint64_t)ld * 4, 32, 32);
    a.hdr = hdr;
    a.stall_at = -1;
    // number of work tiles, to size the persistent grid (a repair launch may visit fewer)
    int64_t tiles = 0;
    for (int64_t rb = 0; rb < a.n_rb; ++rb) {
        int64_t last = std::min(row_begin + rb * IT_BM + IT_BM - 1, row_begin + row_count - 1);
        tiles += ceil_div(key_limit(o.mode, o.window, o.sample_stride, last), IT_BN);
    }
    if (tiles == 0) return cudaSuccess;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const unsigned grid = (unsigned)std::min<int64_t>(tiles, sms);
    const size_t smem = SmemLayout::total;
    void (*kern)(const CUtensorMap, const CUtensorMap, const CUtensorMap, const IdxTcArgs) =
        o.mode == IT_SAMPLE ? index_tc_kernel<IT_SAMPLE>
                            : (o.mode == IT_SELECT ? index_tc_kernel<IT_SELECT> : index_tc_kernel<IT_SCORES>);
    // the warpgroups' register split adds up to the launch's total only if the
    // kernel was built for exactly IT_LAUNCH_REGS registers per thread
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return e;
    // (the build checks this too; a mismatch is an error, not a silent slower path)
    if (fa.numRegs != IT_LAUNCH_REGS) return cudaErrorInvalidKernelImage;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if (write_upper && o.mode == IT_SCORES) {
        for (int64_t r0 = 0; r0 < row_count; r0 += 65535) {
            int64_t n = std::min<int64_t>(row_count - r0, 65535);
            fill_upper_kernel<<<dim3(8, (unsigned)n), 256, 0, st>>>(out + r0 * ld, ld, T, row_begin + r0);
        }
    }
    if (consume_test_stall(0 /* prefill indexer */)) a.stall_at = 1;
    kern<<<grid, IT_THREADS, smem, st>>>(qmap, kmap, omap, a);
    return cudaGetLastError();
}

}  // namespace dsa
