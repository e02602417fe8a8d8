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
// the key's scale.  Persistent and warp-specialised: one CTA per SM takes a
// contiguous share of the (sequence, 256-key item) work; a producer warp
// keeps a 4-stage TMA ring of items in flight, one thread issues each item's
// two 128-key MMAs into one of two rotating TMEM accumulator pairs, and two
// groups of four epilogue warps (one per 128-key half) drain them.  Items of
// 256 keys halve the per-item hand-offs between the roles, which bound the
// throughput at 128-key items.  Every mbarrier wait is bounded; on a
// timeout every role stops, the CTA records DSA_ERR_TIMEOUT, waits (bounded)
// for its copies in flight, frees its tensor memory and returns.
#include <algorithm>

#include "kernels.h"
#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr int DT_TILE = 128;                 // keys per UMMA tile = UMMA M
constexpr int DT_TILE_BYTES = DT_TILE * 128;
constexpr int DT_SUB = 2;                    // UMMA tiles per item
constexpr int DT_ITEM = DT_TILE * DT_SUB;    // keys per item (one pipeline stage)
constexpr int DT_STAGE_BYTES = DT_ITEM * 128;
constexpr int DT_STAGES = 4;
constexpr int DT_MAXSEG = DT_ITEM / 16;      // page segments per item (pages hold >= 16 keys)
constexpr int DT_EPI_WARPS = 4 * DT_SUB;     // four warps (the 128 TMEM lanes) per UMMA tile
constexpr int DT_THREADS = 32 * (2 + DT_EPI_WARPS);
constexpr int DT_ACC = 2;                    // item accumulators (DT_SUB x 64 columns each) in rotation
constexpr int DT_TMEM_COLS = 64 * DT_SUB * DT_ACC;
constexpr int DT_MAX_B = 4096;               // sequences the per-CTA item table can hold
static_assert(DT_STAGE_BYTES % 1024 == 0, "stages keep the 1024-byte swizzle alignment");
static_assert(DT_TMEM_COLS >= 32 && DT_TMEM_COLS <= 512 && (DT_TMEM_COLS & (DT_TMEM_COLS - 1)) == 0,
              "tensor memory is allocated in powers of two columns");

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
    int B;
    int64_t max_context;
    float *scores;
    int64_t ld;
    WsHeader *hdr;
    int64_t stall_at;        // test hook: CTA 0's producer stops before its item stall_at (-1: off)
};

constexpr size_t dt_smem_bytes()
{
    return 1024 /*align slack*/ + 2 * 8192 /*q, double-buffered*/ + (size_t)DT_STAGES * DT_STAGE_BYTES +
           (size_t)DT_STAGES * (DT_ITEM + 1) * 4 /*key scales, segment masks*/ +
           64 * (DT_MAXSEG + 2) * 4 /*producer batches*/ +
           2 * 64 * 4 /*c*/ + (2 * DT_STAGES + 4 + 2 * DT_ACC) * 8 + 16 +
           (size_t)(2 * DT_MAX_B + 1) * 4 /*per-sequence lengths and tile prefix*/;
}
static_assert(dt_smem_bytes() <= 232448 - 64, "dynamic shared memory per CTA");
static_assert(((2 * DT_STAGES + 4 + 2 * DT_ACC) * 8 + 16) % 16 == 0,
              "the key-scale stages (bulk-copy targets) start 16-byte aligned");

// Context length of sequence b if valid, else 0 (the caller records the error).
__device__ __forceinline__ int64_t seq_len(const DecTcArgs &a, int b)
{
    int64_t n = a.context_lens[b];
    if (n < 1 || n > a.max_context || n > (int64_t)a.max_pages * a.page_size) return 0;
    return n;
}

// Per-CTA table of the sequences' lengths and of the prefix sums of their
// 256-key items (filled once from context_lens), so that locating an item is
// a binary search in shared memory.
struct SeqTable {
    const int32_t *n;        // [B]
    const int32_t *prefix;   // [B + 1]
    int B;
};

// Walks this CTA's contiguous share of the (sequence, 256-key item) work; `tile`
// is the item's index within its sequence.
struct ItemWalk {
    int b = 0;
    int64_t tile = 0, left = 0, n = 0;
    __device__ bool start(const SeqTable &t, int64_t first, int64_t count)
    {
        left = count;
        if (count <= 0 || first >= t.prefix[t.B]) return false;
        int lo = 0, hi = t.B - 1;                        // last b with prefix[b] <= first
        while (lo < hi) {
            int mid = (lo + hi + 1) >> 1;
            if (t.prefix[mid] <= first) lo = mid; else hi = mid - 1;
        }
        b = lo;
        tile = first - t.prefix[b];
        n = t.n[b];
        return true;
    }
    __device__ bool next(const SeqTable &t)
    {
        if (--left <= 0) return false;
        ++tile;
        while (b < t.B && tile >= t.prefix[b + 1] - t.prefix[b]) {
            tile = 0;
            if (++b < t.B) n = t.n[b];
        }
        return b < t.B;
    }
};

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

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, %0;" :: "n"(32 * DT_EPI_WARPS) : "memory"); }

template <int H>
__global__ void __launch_bounds__(DT_THREADS, 1)
decode_index_tc_kernel(const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap qmap, const DecTcArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *qs = smem;                                         // [2] x H x 128 B
    uint8_t *ks = qs + 2 * 8192;                                // stages x 256 x 128 B
    // the mbarriers first: they follow a 1024-byte-aligned region, so they stay
    // 8-byte aligned whatever the sizes of the 4-byte arrays after them
    uint64_t *kfull = reinterpret_cast<uint64_t *>(ks + DT_STAGES * DT_STAGE_BYTES);
    uint64_t *kempty = kfull + DT_STAGES;
    uint64_t *qfull = kempty + DT_STAGES, *qempty = qfull + 2;
    uint64_t *tfull = qempty + 2, *tempty = tfull + DT_ACC;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tempty + DT_ACC);
    float *kss = reinterpret_cast<float *>(tmem_slot + 4);                         // [stages][ITEM] key scales
    uint32_t *kmask = reinterpret_cast<uint32_t *>(kss + DT_STAGES * DT_ITEM);     // [stages] loaded segments
    int32_t *pt_b = reinterpret_cast<int32_t *>(kmask + DT_STAGES);               // producer's batches: [2][32] sequences
    uint32_t *pt_mask = reinterpret_cast<uint32_t *>(pt_b + 64);                   // [2][32] segment masks
    int32_t *pt_slot = reinterpret_cast<int32_t *>(pt_mask + 64);                  // [2][32][MAXSEG] segment cache rows
    float *cw = reinterpret_cast<float *>(pt_slot + 64 * DT_MAXSEG);               // [2][64]
    int32_t *tab_n = reinterpret_cast<int32_t *>(cw + 128);                        // [DT_MAX_B]
    int32_t *tab_prefix = tab_n + DT_MAX_B;                                         // [DT_MAX_B + 1]
    __shared__ volatile int abort_flag;
    __shared__ int k_issued, k_consumed, mma_items, q_issued, q_consumed;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int ps = a.page_size;
    grid_dep_trigger();                              // the top-k may be scheduled (it waits for the scores)

    // per-sequence lengths and tile prefix sums (warp 0: lane l scans a block of sequences)
    if (warp == 0) {
        const int per_lane = (a.B + 31) / 32;
        const int b0 = min(a.B, lane * per_lane), b1 = min(a.B, b0 + per_lane);
        int32_t local = 0;
        for (int b = b0; b < b1; ++b) {
            const int64_t n = seq_len(a, b);
            if (n == 0 && blockIdx.x == 0) record_error(a.hdr, DSA_ERR_INVALID_ARG, (unsigned)b);
            tab_n[b] = (int32_t)n;
            local += (int32_t)((n + DT_ITEM - 1) / DT_ITEM);
        }
        int32_t incl = local;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            int32_t y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        int32_t run = incl - local;
        for (int b = b0; b < b1; ++b) {
            tab_prefix[b] = run;
            run += (tab_n[b] + DT_ITEM - 1) / DT_ITEM;
        }
        if (lane == 31) tab_prefix[a.B] = incl;
    }
    __syncthreads();
    const SeqTable tab{tab_n, tab_prefix, a.B};
    const int64_t total = tab_prefix[a.B];
    const int64_t per = (total + gridDim.x - 1) / gridDim.x;
    const int64_t first = (int64_t)blockIdx.x * per;
    const int64_t count = min(per, total - first);
    if (count <= 0) return;

    if (warp == 0) {
        tmem_alloc(tmem_slot, DT_TMEM_COLS);
        tmem_relinquish();
    }
    if (tid == 0) {
        // a stage is free once its MMAs have completed and every epilogue warp has
        // read its key scales
        for (int s = 0; s < DT_STAGES; ++s) { mbar_init(&kfull[s], 1); mbar_init(&kempty[s], 1 + DT_EPI_WARPS); }
        for (int i = 0; i < 2; ++i) { mbar_init(&qfull[i], 1); mbar_init(&qempty[i], 1); }
        for (int i = 0; i < DT_ACC; ++i) { mbar_init(&tfull[i], 1); mbar_init(&tempty[i], DT_EPI_WARPS); }
        abort_flag = 0;
        k_issued = k_consumed = mma_items = q_issued = q_consumed = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------ TMA producer (whole warp)
        // The 32 lanes resolve the page ids of the 32 items of a batch at once,
        // one batch ahead, so that the block-table reads are in flight while the
        // current batch is issued.  Per item, lane 0 claims the stage and lane g
        // copies page segment g: its keys by tensor TMA, its scales by bulk copy.
        if (lane == 0) {
            tma_prefetch_desc(&kmap);
            tma_prefetch_desc(&qmap);
        }
        const int nseg = DT_ITEM / a.box_rows;           // <= DT_MAXSEG page segments per item
        int seg = -1, prev_b = -1;
        bool stop = false;
        ItemWalk mine;                                   // this lane's item of the batch being fetched
        bool have = false;
        int pgs[DT_MAXSEG];                              // its page ids, loads in flight
        auto fetch = [&](int64_t j0) {
            have = j0 + lane < count && mine.start(tab, first + j0 + lane, count - j0 - lane);
            const int64_t p0 = mine.tile * DT_ITEM;
#pragma unroll
            for (int g = 0; g < DT_MAXSEG; ++g) {
                const int64_t pos = p0 + (int64_t)g * a.box_rows;
                pgs[g] = have && g < nseg && pos < mine.n
                             ? __ldg(a.block_table + (int64_t)mine.b * a.max_pages + pos / ps) : -1;
            }
        };
        auto publish = [&](int t) {                      // batch table t <- this lane's item
            uint32_t m = 0;
            const int64_t p0 = mine.tile * DT_ITEM;
#pragma unroll
            for (int g = 0; g < DT_MAXSEG; ++g) {
                const int64_t pos = p0 + (int64_t)g * a.box_rows;
                int slot = 0;
                if (have && g < nseg && pos < mine.n) {
                    if (pgs[g] >= 0 && pgs[g] < a.num_pages) {
                        m |= 1u << g;
                        slot = (int)((int64_t)pgs[g] * ps + pos % ps);
                    } else {
                        record_error(a.hdr, DSA_ERR_INVALID_ARG, (unsigned)mine.b);
                    }
                }
                if (g < nseg) pt_slot[(t * 32 + lane) * DT_MAXSEG + g] = slot;
            }
            pt_b[t * 32 + lane] = have ? mine.b : -1;
            pt_mask[t * 32 + lane] = m;
        };
        fetch(0);
        int t = 0;
        for (int64_t j0 = 0; j0 < count && !stop; j0 += 32, t ^= 1) {
            publish(t);
            fetch(j0 + 32);
            __syncwarp();
            const int nb = (int)min((int64_t)32, count - j0);
            for (int i = 0; i < nb; ++i) {
                const int64_t j = j0 + i;
                if (j == a.stall_at && blockIdx.x == 0) {    // test hook: leave a copy unissued
                    stop = true;
                    break;
                }
                const int s = (int)(j % DT_STAGES);
                const uint32_t mask = pt_mask[t * 32 + i];
                bool ok = true;
                if (lane == 0) {
                    const int b = pt_b[t * 32 + i];
                    if (b != prev_b) {                       // a new sequence: its query heads
                        ++seg;
                        prev_b = b;
                        ok = wait_or_abort(&qempty[seg & 1], ((seg >> 1) & 1) ^ 1, &abort_flag);
                        if (ok) {
                            mbar_arrive_expect_tx(&qfull[seg & 1], H * 128);
                            tma_load_2d(qs + (seg & 1) * 8192, &qmap, &qfull[seg & 1], 0, b * H);
                            q_issued = seg + 1;
                        }
                    }
                    if (ok) ok = wait_or_abort(&kempty[s], (uint32_t)((j / DT_STAGES) & 1) ^ 1, &abort_flag);
                    if (ok) {
                        kmask[s] = mask;                     // published by the arrive below
                        mbar_arrive_expect_tx(&kfull[s], (uint32_t)__popc(mask) * a.box_rows * (128 + 4));
                    }
                }
                // after lane 0's claim of the stage (the shuffle orders the warp behind it)
                if (!__shfl_sync(0xffffffffu, ok, 0)) {
                    stop = true;
                    break;
                }
                __syncwarp();
                if (lane < nseg && ((mask >> lane) & 1u)) {
                    const int slot = pt_slot[(t * 32 + i) * DT_MAXSEG + lane];
                    tma_load_2d(ks + s * DT_STAGE_BYTES + lane * a.box_rows * 128, &kmap, &kfull[s], 0, slot);
                    bulk_load(kss + s * DT_ITEM + lane * a.box_rows, a.kscale + slot, (uint32_t)a.box_rows * 4,
                              &kfull[s]);
                }
                if (lane == 0) k_issued = (int)j + 1;
            }
            __syncwarp();                                    // batch table t is rewritten two batches on
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        if (lane == 0) {
            constexpr uint32_t idesc = umma_idesc_e4m3_f32(DT_TILE, H);
            ItemWalk it;
            int j = 0, seg = -1, prev_b = -1;
            uint64_t bdesc = 0;
            for (bool ok = it.start(tab, first, count); ok; ok = it.next(tab), ++j) {
                if (it.b != prev_b) {
                    if (seg >= 0) umma_commit(&qempty[seg & 1]);   // previous query heads are free
                    ++seg;
                    prev_b = it.b;
                    if (!wait_or_abort(&qfull[seg & 1], (seg >> 1) & 1, &abort_flag)) break;
                    q_consumed = seg + 1;
                    bdesc = umma_desc_k_sw128(smem_u32(qs + (seg & 1) * 8192));
                }
                const int s = j % DT_STAGES, acc = j % DT_ACC;
                if (!wait_or_abort(&kfull[s], (j / DT_STAGES) & 1, &abort_flag)) break;
                k_consumed = j + 1;
                if (!wait_or_abort(&tempty[acc], ((j / DT_ACC) & 1) ^ 1, &abort_flag)) break;
                tc_fence_after();
#pragma unroll
                for (int sub = 0; sub < DT_SUB; ++sub) {
                    const uint64_t adesc = umma_desc_k_sw128(smem_u32(ks + s * DT_STAGE_BYTES + sub * DT_TILE_BYTES));
                    const uint32_t d = tmem + (uint32_t)((acc * DT_SUB + sub) * 64);
#pragma unroll
                    for (int k = 0; k < 4; ++k) umma_f8f6f4(d, adesc + 2 * k, bdesc + 2 * k, idesc, k > 0);
                }
                umma_commit(&kempty[s]);
                umma_commit(&tfull[acc]);
                mma_items = j + 1;
            }
        }
    } else {
        // ------------------------------------------------ epilogue (4 warps per UMMA tile, one key per thread)
        const int q4 = warp & 3;                       // TMEM lane quarter
        const int et = tid - 64;
        const int sub = (warp - 2) >> 2;               // this warp's UMMA tile of every item
        const int r = sub * DT_TILE + q4 * 32 + lane;   // this thread's key within every item
        int j = 0, seg = -1, prev_b = -1;
        bool dead = false;
        uint64_t cpk[H / 2];                           // this sequence's c_h, packed in pairs
        ItemWalk it;
        for (bool ok = it.start(tab, first, count); ok; ok = it.next(tab), ++j) {
            if (it.b != prev_b) {                       // per-sequence head weights c_h = w[b,h] * sq[b]
                ++seg;
                prev_b = it.b;
                epi_sync();
                if (et < H) cw[(seg & 1) * 64 + et] = bf16_to_f32(a.w[(int64_t)it.b * H + et]) * a.sq[it.b];
                epi_sync();
#pragma unroll
                for (int i = 0; i < H / 2; ++i) cpk[i] = f2_pack(cw[(seg & 1) * 64 + 2 * i], cw[(seg & 1) * 64 + 2 * i + 1]);
            }
            if (dead) continue;
            const int s = j % DT_STAGES, acc = j % DT_ACC;
            const int64_t pos = it.tile * DT_ITEM + r;
            // warp-uniform outcome: the TMEM loads below are warp-collective
            if (!__all_sync(0xffffffffu, wait_or_abort(&tfull[acc], (j / DT_ACC) & 1, &abort_flag))) {
                dead = true;
                continue;
            }
            tc_fence_after();
            // the stage's copies landed before its MMAs ran: this wait only orders the
            // scale reads behind the copies
            if (!__all_sync(0xffffffffu, wait_or_abort(&kfull[s], (j / DT_STAGES) & 1, &abort_flag))) {
                dead = true;
                continue;
            }
            const bool live = pos < it.n && ((kmask[s] >> (r / a.box_rows)) & 1u);
            const float ksc = kss[s * DT_ITEM + r];
            __syncwarp();
            if (lane == 0) mbar_arrive(&kempty[s]);
            const uint32_t trow = tmem + ((uint32_t)(q4 * 32) << 16) + (uint32_t)((acc * DT_SUB + sub) * 64);
            // all of this key's H head products in one round trip, four independent sums
            uint64_t s4[4] = {0ull, 0ull, 0ull, 0ull};
            if constexpr (H == 64) {
                uint32_t va[32], vb[32];
                tmem_ld32(trow, va);
                tmem_ld32(trow + 32, vb);
                tmem_wait_ld_dep32(vb);
                tmem_wait_ld_dep32(va);
#pragma unroll
                for (int i = 0; i < 32; i += 2) {
                    s4[(i >> 1) & 3] = f2_fma(cpk[i >> 1],
                                              f2_pack(fmaxf(__uint_as_float(va[i]), 0.f), fmaxf(__uint_as_float(va[i + 1]), 0.f)),
                                              s4[(i >> 1) & 3]);
                    s4[(i >> 1) & 3] = f2_fma(cpk[16 + (i >> 1)],
                                              f2_pack(fmaxf(__uint_as_float(vb[i]), 0.f), fmaxf(__uint_as_float(vb[i + 1]), 0.f)),
                                              s4[(i >> 1) & 3]);
                }
            } else {
#pragma unroll
                for (int c0 = 0; c0 < H; c0 += 16) {
                    uint32_t v[16];
                    tmem_ld16(trow + c0, v);
                    tmem_wait_ld_dep16(v);
#pragma unroll
                    for (int i = 0; i < 16; i += 2)
                        s4[(i >> 1) & 3] = f2_fma(cpk[(c0 + i) >> 1],
                                                  f2_pack(fmaxf(__uint_as_float(v[i]), 0.f), fmaxf(__uint_as_float(v[i + 1]), 0.f)),
                                                  s4[(i >> 1) & 3]);
                }
            }
            float lo, hi, acc_sum = 0.f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                f2_unpack(s4[q], lo, hi);
                acc_sum += lo + hi;
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&tempty[acc]);
            if (live) a.scores[(int64_t)it.b * a.ld + pos] = acc_sum * ksc;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (abort_flag && tid == 0) {
        record_error(a.hdr, DSA_ERR_TIMEOUT, blockIdx.x);
        // let copies and MMAs still in flight land before shared and tensor memory go
        for (int j = k_consumed; j < k_issued; ++j) mbar_wait(&kfull[j % DT_STAGES], (j / DT_STAGES) & 1);
        for (int q = q_consumed; q < q_issued; ++q) mbar_wait(&qfull[q & 1], (q >> 1) & 1);
        if (mma_items > 0) mbar_wait(&tfull[(mma_items - 1) % DT_ACC], ((mma_items - 1) / DT_ACC) & 1);
    }
    __syncthreads();
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
    if (!decode_index_tc_supported(H, page_size) || B > DT_MAX_B) return cudaErrorNotSupported;
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
                B, max_context, scores, ld, hdr, consume_test_stall(1 /* decode indexer */) ? 0 : -1};
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t max_items = (int64_t)B * ceil_div(max_context, DT_ITEM);
    dim3 grid((unsigned)std::min<int64_t>(max_items, sms));
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
