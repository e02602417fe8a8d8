// Sparse main attention on the 5th-generation tensor cores (tcgen05).
//
// o[t,h] = sum_{j in S_t} softmax_j(sm * q[t,h] . K[j]) V[j]
// ("DeepSeek-V3.2-Exp 稀疏注意力机制(DSA)技术深度解析", section 1: the main
// attention runs only over the k selected KV entries, O(n^2) -> O(n k)).
//
// One shared K/V head (MQA): the 128 query heads of a token are the UMMA M
// dimension, so every gathered K/V row feeds 128 heads.  Persistent: each
// CTA (one per SM) takes a contiguous range of items -- a query token (or
// decode sequence), a group of 128 heads, a range of its index list -- and
// streams their selected rows in blocks of 64:
//   warps 4-5 producers: thread p resolves selected position p of a 64-row
//             block (through the page table for the paged caches) and copies
//             its K and V rows with 16-byte cp.async into the 128-byte-swizzled
//             tiles of a 5-stage ring (many small loads in flight per SM: the
//             rows are scattered); one thread also brings the next item's Q
//             with TMA into a second Q buffer;
//   warp 6    S issuer: S = Q K^T (kind::f16, M 128 heads, N 64 rows,
//             K = 128 = 8 x 16) into one of two TMEM buffers, as soon as the
//             K tile is in and the softmax has read that buffer's last S;
//   warp 7    PV issuer: O += P V (P from tensor memory, V read MN-major
//             straight from the gathered rows) into one of two TMEM O buffers
//             (per item), as soon as P is written.  Two issuing threads keep
//             the S MMAs from queueing behind the PV MMAs, which wait for the
//             softmax;
//   warps 0-3 softmax: thread = head row.  Reads its S row from TMEM, masks
//             unused slots, keeps the running max m and sum l in registers,
//             writes P (bf16 pairs) to tensor memory, the A operand of the PV
//             MMA (no shared-memory round trip, no proxy fence).  O is rescaled
//             (a TMEM round trip) only when the block max exceeds m by more
//             than 2^8 -- otherwise P <= 256 and m stays -- which is exact up
//             to rounding.  At the end O / l and the log-sum-exp are written.
// Every mbarrier wait is bounded (DSA_ERR_TIMEOUT on expiry).
#include <algorithm>

#include <cuda_fp8.h>

#include "kernels.h"
#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr int AT_HEADS = 128;          // UMMA M: query heads per item
constexpr int AT_D = 128;              // head dim
constexpr int AT_BLK = 64;             // selected rows per block (UMMA N of S, K of PV)
// K/V gather ring depth: a block holds its stage from the gather to the end of
// its PV product (about four block periods), so the ring bounds the block rate.
// Five stages fill the shared memory of the bf16 kernel; the KV8 kernel keeps
// four beside its staging buffers.
template <bool KV8> constexpr int at_stages() { return KV8 ? 2 : 5; }
constexpr int AT_NSTG = 4;             // KV8: staging buffers of E4M3 blocks (three blocks of lookahead)
constexpr int AT_THREADS = 384;        // 2 x 4 softmax warps, 2 producer warps, S and PV issuer warps
constexpr int AT_PRODUCERS = 64;       // producer threads: one selected row each per block
// Register split by warpgroup: producers and issuers (warps 4-7) give theirs to
// the two softmax sets (warps 0-3 and 8-11).  The split adds up to the launch's
// total only for a kernel built with exactly AT_LAUNCH_REGS per thread (checked
// before every launch).
constexpr int AT_LAUNCH_REGS = 168;
constexpr int AT_REGS_LOW = 96;
constexpr int AT_REGS_HIGH = 200;
static_assert(128 * AT_REGS_LOW + 256 * AT_REGS_HIGH <= AT_LAUNCH_REGS * 384, "register split");

constexpr int AT_QHALF = AT_HEADS * 128;     // one 64-column half of Q (16 KB)
constexpr int AT_QTILE = 2 * AT_QHALF;       // Q of one item (32 KB)
constexpr int AT_KHALF = AT_BLK * 128;       // one 64-column half of a 64-row K or V tile (8 KB)
constexpr int AT_KTILE = 2 * AT_KHALF;       // a 64 x 128 bf16 tile (16 KB)
constexpr int AT_STAGE = 2 * AT_KTILE;       // K + V of one block (32 KB)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.f;     // log2 units

struct AttnTcArgs {
    const uint16_t *k;       // K rows [kv_rows, D] (contiguous or paged cache)
    const uint16_t *v;
    // FP8 K/V (the KV8 kernel): E4M3 rows [kv_rows, D] and one fp32 scale per row
    const uint8_t *k8, *v8;
    const float *ks, *vs;
    const int32_t *idx;      // [rows, ksel]
    int ksel;
    int H;                   // query heads (multiple of 128)
    int64_t kv_rows;         // rows of the K/V tensor maps
    int64_t T;               // contiguous: positions must be < T
    // paged K/V (null block_table: contiguous)
    const int32_t *block_table;
    const int32_t *context_lens;
    int64_t num_pages;
    int max_pages, page_size;
    float scale_log2;
    uint16_t *out;           // [rows, H, D] (splits == 1)
    float *lse;              // [rows, H] or null
    float *part;             // split partials (splits > 1)
    int64_t rows;
    int splits, chunk;
    int64_t items;           // rows x head groups x splits
    WsHeader *hdr;
};

template <int NST>
struct AtSmemT {
    static constexpr size_t q_off = 0;                                   // [2] Q tiles
    static constexpr size_t kv_off = q_off + 2 * AT_QTILE;                // [stages] K, V tiles
    static constexpr size_t valid_off = kv_off + (size_t)NST * AT_STAGE;  // [stages][2] validity bits
    static constexpr size_t ml_off = valid_off + NST * 2 * 4;            // set 1's (m, l) per head
    static constexpr size_t bar_off = ml_off + 2 * AT_HEADS * 4;
    // qfull[2] qempty[2] kvfull[S] kvempty[S] sfull[2] sempty[2] pfull[2] pempty[2] ofull oempty mlfull mlempty
    static constexpr int n_bars = 2 * NST + 16;
    static constexpr size_t slot_off = bar_off + 8 * n_bars;
    static constexpr size_t total() { return slot_off + 16 + 1024; }
    // KV8: staging buffers of one block's E4M3 K and V rows (64 x 256 bytes), then
    // their K and V scales ([buf][2][64] floats) and validity words ([buf][2])
    static constexpr size_t stg_bytes = (size_t)AT_BLK * 2 * AT_D;
    static constexpr size_t stg_off = (slot_off + 16 + 127) / 128 * 128;
    static constexpr size_t stg_sc_off = stg_off + AT_NSTG * stg_bytes;
    static constexpr size_t stg_vw_off = stg_sc_off + AT_NSTG * 2 * AT_BLK * 4;
    static constexpr size_t total_kv8() { return stg_vw_off + AT_NSTG * 2 * 4 + 1024; }
};
using AtSmemBf16 = AtSmemT<at_stages<false>()>;
using AtSmemKv8 = AtSmemT<at_stages<true>()>;
static_assert(AtSmemBf16::total() + 64 <= 232448, "the bf16 kernel's ring fits the shared memory of a CTA");
static_assert(AtSmemKv8::total_kv8() + 64 <= 232448, "KV8 staging fits the shared memory of a CTA");

// Eight bf16 pairs of 16 E4M3 codes times a scale (code j in byte j of the 16).
__device__ __forceinline__ void e4m3x16_to_bf16_scaled(const uint4 &raw, float sc, uint32_t (&out)[8])
{
    const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const __nv_fp8x2_storage_t two = (__nv_fp8x2_storage_t)((w[i >> 1] >> (16 * (i & 1))) & 0xffffu);
        const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(two, __NV_E4M3);
        const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&hr));
        out[i] = pack_bf16x2(f.x * sc, f.y * sc);
    }
}

// 4-byte cp.async (zero-filled when !valid).
__device__ __forceinline__ void cp_async_4(void *smem, const void *gmem, bool valid)
{
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;\n"
                 :: "r"(smem_u32(smem)), "l"(gmem), "r"(valid ? 4u : 0u) : "memory");
}

__device__ __forceinline__ void st_shared_v4(void *p, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" :: "r"(smem_u32(p)), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

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

// 2^x by the SFU's approximate base-2 exponential (results below 2^-126 flush
// to zero; P is rounded to bf16 right after, so neither matters).
__device__ __forceinline__ float ex2_sfu(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// Decomposition of an item index and its block count.
struct Item {
    int64_t row;
    int hg, split, e0, e1, nblk;
    __device__ __forceinline__ void set(const AttnTcArgs &a, int64_t it)
    {
        split = (int)(it % a.splits);
        const int64_t rh = it / a.splits;
        const int hgs = a.H / AT_HEADS;
        hg = (int)(rh % hgs);
        row = rh / hgs;
        e0 = split * a.chunk;
        e1 = min(a.ksel, e0 + a.chunk);
        nblk = e1 > e0 ? (e1 - e0 + AT_BLK - 1) / AT_BLK : 0;
    }
};

// KV8: the K/V rows are FP8 E4M3 with a per-row scale (the paged decode
// caches); the producers stage a block's codes one block ahead with cp.async
// and widen them to bf16 (times the scale) into the same swizzled tiles, so
// the MMA and softmax roles are those of the bf16 kernel.
template <bool KV8>
__global__ void __launch_bounds__(AT_THREADS, 1)
sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap, const AttnTcArgs a)
{
    constexpr int AT_STAGES = at_stages<KV8>();
    using AtSmem = AtSmemT<AT_STAGES>;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *Qs = smem + AtSmem::q_off;
    uint8_t *KVs = smem + AtSmem::kv_off;
    uint32_t *valid = reinterpret_cast<uint32_t *>(smem + AtSmem::valid_off);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + AtSmem::bar_off);
    uint64_t *qfull = bars, *qempty = bars + 2, *kvfull = bars + 4, *kvempty = kvfull + AT_STAGES;
    uint64_t *sfull = kvempty + AT_STAGES, *sempty = sfull + 2, *pfull = sempty + 2, *pempty = pfull + 2;
    uint64_t *ofull = pempty + 2, *oempty = ofull + 1, *mlfull = oempty + 1, *mlempty = mlfull + 1;
    float *mls = reinterpret_cast<float *>(smem + AtSmem::ml_off);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + AtSmem::slot_off);
    __shared__ volatile int abort_flag;
    __shared__ int kv_issued, kv_consumed, q_issued, q_consumed, pv_last, s_last;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t per = (a.items + gridDim.x - 1) / gridDim.x;
    const int64_t it_begin = (int64_t)blockIdx.x * per;
    const int64_t it_end = min(a.items, it_begin + per);
    if (it_begin >= it_end) return;
    const bool paged = a.block_table != nullptr;

    if (warp == 0) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    if (tid == 0) {
        for (int i = 0; i < 2; ++i) {
            mbar_init(&qfull[i], 1); mbar_init(&qempty[i], 1);
            mbar_init(&sfull[i], 1); mbar_init(&sempty[i], 4);   // [x]: the 4 warps of softmax set x
            mbar_init(&pfull[i], 4); mbar_init(&pempty[i], 1);
        }
        mbar_init(ofull, 1); mbar_init(oempty, 4);                // oempty: set 0 read O_0 and O_1
        mbar_init(mlfull, 4); mbar_init(mlempty, 4);              // set 1 -> set 0 hand-off of (m, l)
        // kvfull: one asynchronous arrival per copying producer thread when its copies
        // land (bf16: the one warp of the block; KV8: both warps), plus two ordinary
        // arrivals publishing the validity bits
        for (int i = 0; i < AT_STAGES; ++i) { mbar_init(&kvfull[i], (KV8 ? AT_PRODUCERS : 32) + 2); mbar_init(&kvempty[i], 1); }
        abort_flag = 0;
        kv_issued = kv_consumed = q_issued = q_consumed = pv_last = s_last = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    grid_dep_wait();                                 // chained launch: the index lists of the kernel before
    grid_dep_trigger();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tO = tmem + 2 * AT_BLK;    // S [0,128), O [128,384)
    const uint32_t tP = tmem + 6 * AT_BLK;               // P [384,448): 32 columns of bf16 pairs per set

    if (warp >= 4 && warp < 8) {
        regs_dec<AT_REGS_LOW>();
        if (warp == 4 || warp == 5) {
            // ------------------------------------------------ producers (2 warps, one row per thread)
            // Thread p copies selected row p of each 64-row block (its K and V rows,
            // 16 x 16 bytes each) with cp.async into the 128-byte-swizzled tiles.
            // Each thread's copies signal the block's kvfull barrier asynchronously when
            // they land (cp.async.mbarrier.arrive.noinc); the MMA issuer fences the
            // generic-proxy writes for the tensor cores' async-proxy reads.
            const int pt = tid - 128;                     // 0..63: row of the block
            if (pt == 0) {
                tma_prefetch_desc(&qmap);
            }
            int qi = 0, g = 0;
            bool stop = false;
            for (int64_t it = it_begin; it < it_end && !stop; ++it) {
                Item item;
                item.set(a, it);
                if (item.nblk == 0) continue;
                int ctx = 0;
                if (paged) {
                    ctx = a.context_lens[item.row];
                    if (ctx < 0 || (int64_t)ctx > (int64_t)a.max_pages * a.page_size) ctx = 0;
                }
                if (pt == 0) {
                    const int qb = qi & 1;
                    if (!wait_or_abort(&qempty[qb], ((qi >> 1) & 1) ^ 1, &abort_flag)) stop = true;
                    else {
                        mbar_arrive_expect_tx(&qfull[qb], AT_QTILE);
                        const int qrow = (int)(item.row * a.H + item.hg * AT_HEADS);
                        tma_load_2d(Qs + qb * AT_QTILE, &qmap, &qfull[qb], 0, qrow);
                        tma_load_2d(Qs + qb * AT_QTILE + AT_QHALF, &qmap, &qfull[qb], 64, qrow);
                        q_issued = qi + 1;
                    }
                }
                stop = __shfl_sync(0xffffffffu, stop, 0) || __any_sync(0xffffffffu, stop);
                if (warp == 5) stop = stop || abort_flag;
                ++qi;
                const int32_t *irow = a.idx + item.row * a.ksel;
                // bf16: producer warp w = warp - 4 takes blocks b = w, w + 2, ... of the item
                // whole; lane l resolves rows l and 32 + l of its block (broadcast by shuffles)
                // and copies 16-byte chunk l % 16 of each row's K (l < 16) or V (l >= 16), so
                // one instruction moves one whole row pair (two 256-byte runs).  A warp's
                // loop runs at the latency of the index reads for its next block, so the
                // two warps taking alternate blocks issue a block in about half that time.
                // KV8: warp w copies rows 32 w .. 32 w + 31 of every block (below).
                const int rbase = (warp - 4) * 32;
                const int32_t *brow = paged ? a.block_table + item.row * a.max_pages : nullptr;
                const int chunk = lane & 15;
                const bool is_v = lane >= 16;
                // K/V row of selected position p (page pg): lane l resolves row
                // rbase + l of a block; out-of-range page ids are reported, not read.
                auto resolve = [&](int p, int pg, int &r, bool &v) {
                    r = 0;                                // K/V row (kv_rows < 2^31)
                    v = false;
                    if (paged) {
                        if (p >= 0 && p < ctx) {
                            if (pg >= 0 && pg < a.num_pages) {
                                r = pg * a.page_size + p % a.page_size;
                                v = true;
                            } else {
                                record_error(a.hdr, DSA_ERR_INVALID_ARG, (unsigned)item.row);
                            }
                        }
                    } else if (p >= 0 && p < a.T) {
                        r = p;
                        v = true;
                    }
                };
                // KV8: lane l copies (and later widens) 16-byte code chunk l % 16 -- K
                // for l % 16 < 8, V otherwise -- of rows l / 16, l / 16 + 2, ... of
                // the warp's 32, into staging buffer g % AT_NSTG, three blocks ahead;
                // lane l also copies row rbase + l's two scales, and lane 0 records the
                // block's validity word.  The positions run one block and the page ids
                // one block ahead of the staging.
                uint8_t *stg = smem + AtSmem::stg_off;
                float *stg_sc = reinterpret_cast<float *>(smem + AtSmem::stg_sc_off);
                uint32_t *stg_vw = reinterpret_cast<uint32_t *>(smem + AtSmem::stg_vw_off);
                auto pos_of = [&](int bb) -> int {
                    const int ee = item.e0 + bb * AT_BLK + rbase + lane;
                    return (bb < item.nblk && ee < item.e1) ? __ldg(irow + ee) : -1;
                };
                auto page_of = [&](int pp) -> int {
                    return paged && pp >= 0 && pp < ctx ? __ldg(brow + pp / a.page_size) : -1;
                };
                auto stage = [&](int gb, int pp, int pg) {
                    int r;
                    bool v;
                    resolve(pp, pg, r, v);
                    const unsigned vb = __ballot_sync(0xffffffffu, v);
                    const int buf = gb % AT_NSTG;
                    uint8_t *sb = stg + buf * AtSmem::stg_bytes + rbase * 2 * AT_D + chunk * 16;
                    const uint8_t *src = (chunk < 8 ? a.k8 : a.v8) + (chunk & 7) * 16;
#pragma unroll
                    for (int j = 0; j < 16; ++j) {
                        const int i = 2 * j + (lane >> 4);
                        const int ri = __shfl_sync(0xffffffffu, r, i);
                        cp_async_16(sb + i * 2 * AT_D, src + (int64_t)ri * AT_D, (vb >> i) & 1u);
                    }
                    cp_async_4(stg_sc + (buf * 2 + 0) * AT_BLK + rbase + lane, a.ks + r, v);
                    cp_async_4(stg_sc + (buf * 2 + 1) * AT_BLK + rbase + lane, a.vs + r, v);
                    if (lane == 0) stg_vw[buf * 2 + (warp - 4)] = vb;
                };
                int pnx = -1, pgnx = -1, pnx2 = -1;           // block b + 3's position and page, b + 4's position
                if constexpr (KV8) {
                    for (int bb = 0; bb < AT_NSTG - 1; ++bb) {
                        if (bb < item.nblk && !stop) {
                            const int pp = pos_of(bb);
                            stage(g + bb, pp, page_of(pp));
                        }
                        cp_async_commit();
                    }
                    pnx = pos_of(AT_NSTG - 1);
                    pgnx = page_of(pnx);
                    pnx2 = pos_of(AT_NSTG);
                }
                if constexpr (!KV8) {
                    const int w = warp - 4;
                    auto pos_at = [&](int bb, int row) -> int {
                        const int ee = item.e0 + bb * AT_BLK + row;
                        return (bb < item.nblk && ee < item.e1) ? __ldg(irow + ee) : -1;
                    };
                    // positions of the warp's block b (rows l, 32 + l) and of its next block
                    // b + 2, read one block of the warp ahead; paged: block b's page ids
                    int qa0 = pos_at(w, lane), qa1 = pos_at(w, 32 + lane);
                    int qb0 = pos_at(w + 2, lane), qb1 = pos_at(w + 2, 32 + lane);
                    int pga0 = page_of(qa0), pga1 = page_of(qa1);
                    for (int b = w; b < item.nblk && !stop; b += 2) {
                        const int gb = g + b, st = gb % AT_STAGES;
                        const int p0 = qa0, p1 = qa1, pg0 = pga0, pg1 = pga1;
                        qa0 = qb0;
                        qa1 = qb1;
                        pga0 = page_of(qa0);
                        pga1 = page_of(qa1);
                        qb0 = pos_at(b + 4, lane);
                        qb1 = pos_at(b + 4, 32 + lane);
                        // warp-uniform outcome: the ballots and shuffles below need every lane
                        const bool ok = __all_sync(0xffffffffu,
                                                   wait_or_abort(&kvempty[st], ((gb / AT_STAGES) & 1) ^ 1, &abort_flag));
                        if (!ok) { stop = true; break; }
                        int r0, r1;
                        bool v0, v1;
                        resolve(p0, pg0, r0, v0);
                        resolve(p1, pg1, r1, v1);
                        const unsigned vw0 = __ballot_sync(0xffffffffu, v0);
                        const unsigned vw1 = __ballot_sync(0xffffffffu, v1);
                        if (lane == 0) {
                            valid[st * 2] = vw0;
                            valid[st * 2 + 1] = vw1;
                            mbar_arrive(&kvfull[st]);      // releases the validity bits
                            mbar_arrive(&kvfull[st]);
                        }
                        uint8_t *tile = KVs + st * AT_STAGE + (is_v ? AT_KTILE : 0) + (chunk >> 3) * AT_KHALF;
                        const uint16_t *base = (is_v ? a.v : a.k) + chunk * 8;
#pragma unroll
                        for (int i = 0; i < 32; ++i) {    // rows i and 32 + i of the block
                            const int ri = __shfl_sync(0xffffffffu, r0, i);
                            cp_async_16(tile + i * 128 + (((chunk ^ i) & 7) << 4), base + (int64_t)ri * AT_D, (vw0 >> i) & 1u);
                        }
#pragma unroll
                        for (int i = 0; i < 32; ++i) {
                            const int ri = __shfl_sync(0xffffffffu, r1, i);
                            cp_async_16(tile + (32 + i) * 128 + (((chunk ^ i) & 7) << 4), base + (int64_t)ri * AT_D,
                                        (vw1 >> i) & 1u);
                        }
                        cp_async_arrive_noinc(&kvfull[st]);   // fires when this thread's copies land
                        if (lane == 0) atomicMax(&kv_issued, gb + 1);
                    }
                    g += item.nblk;
                } else {
                    for (int b = 0; b < item.nblk && !stop; ++b, ++g) {
                        const int st = g % AT_STAGES;
                        // warp-uniform outcome: the ballot and shuffles below need every lane
                        const bool ok = __all_sync(0xffffffffu,
                                                   wait_or_abort(&kvempty[st], ((g / AT_STAGES) & 1) ^ 1, &abort_flag));
                        if (!ok) { stop = true; break; }
                        cp_async_wait<AT_NSTG - 2>();     // this lane's copies of block g have landed
                        __syncwarp();                     // and every lane's (scales, validity word)
                        const int buf = g % AT_NSTG;
                        const unsigned vw = stg_vw[buf * 2 + (warp - 4)];
                        if (lane == 0) {
                            valid[st * 2 + (warp - 4)] = vw;
                            mbar_arrive(&kvfull[st]);      // releases the validity bits
                        }
                        const uint8_t *sb = stg + buf * AtSmem::stg_bytes + rbase * 2 * AT_D + chunk * 16;
                        const float *scl = stg_sc + (buf * 2 + (chunk < 8 ? 0 : 1)) * AT_BLK + rbase;
                        uint8_t *tile = KVs + st * AT_STAGE + (chunk < 8 ? 0 : AT_KTILE) + ((chunk & 7) >> 2) * AT_KHALF +
                                        rbase * 128;
                        const int c0 = 2 * (chunk & 7);   // bf16 chunks c0, c0 + 1 of the row
#pragma unroll 4
                        for (int j = 0; j < 16; ++j) {
                            const int i = 2 * j + (lane >> 4);
                            const uint4 raw = *reinterpret_cast<const uint4 *>(sb + i * 2 * AT_D);
                            uint32_t o[8];
                            e4m3x16_to_bf16_scaled(raw, scl[i], o);
                            uint8_t *row = tile + i * 128;
                            st_shared_v4(row + ((((c0) ^ i) & 7) << 4), o[0], o[1], o[2], o[3]);
                            st_shared_v4(row + ((((c0 + 1) ^ i) & 7) << 4), o[4], o[5], o[6], o[7]);
                        }
                        fence_proxy_async_smem();         // generic writes, read by the tensor cores
                        mbar_arrive(&kvfull[st]);
                        // refill buffer (g + 3) % AT_NSTG -- block g - 1's, converted last
                        // iteration -- with block b + 3, and run the lookahead on
                        if (b + AT_NSTG - 1 < item.nblk) stage(g + AT_NSTG - 1, pnx, pgnx);
                        cp_async_commit();
                        pnx = pnx2;
                        pgnx = page_of(pnx);
                        pnx2 = pos_of(b + AT_NSTG + 1);
                        if (pt == 0) kv_issued = g + 1;
                    }
                }
            }
            cp_async_wait<0>();                           // nothing in flight when the CTA retires
        } else if (warp == 6) {
            // ------------------------------------------------ S issuer: S(b) = Q K(b)^T
            // Block b of an item belongs to softmax set b % 2 and its S buffer; S(b)
            // waits only for its K tile and for that set to have read its last S.
            if (lane == 0) {
                constexpr uint32_t idesc_s = umma_idesc_bf16_f32(AT_HEADS, AT_BLK, false);
                int qi = 0, g = 0, cnt[2] = {0, 0};
                bool ok = true;
                for (int64_t it = it_begin; it < it_end && ok; ++it) {
                    Item item;
                    item.set(a, it);
                    if (item.nblk == 0) continue;
                    const int qb = qi & 1;
                    if (!wait_or_abort(&qfull[qb], (qi >> 1) & 1, &abort_flag)) { ok = false; break; }
                    q_consumed = qi + 1;
                    const uint32_t qa = smem_u32(Qs + qb * AT_QTILE);
                    for (int b = 0; b < item.nblk; ++b, ++g) {
                        const int st = g % AT_STAGES, x = b & 1, k = cnt[x]++;
                        if (!wait_or_abort(&kvfull[st], (g / AT_STAGES) & 1, &abort_flag) ||
                            !wait_or_abort(&sempty[x], (k & 1) ^ 1, &abort_flag)) { ok = false; break; }
                        kv_consumed = g + 1;
                        fence_proxy_async_smem();         // cp.async wrote the tiles; the MMA reads them
                        tc_fence_after();
                        const uint32_t ka = smem_u32(KVs + st * AT_STAGE);
#pragma unroll
                        for (int kk = 0; kk < AT_D / 16; ++kk) {
                            umma_f16(tS + x * AT_BLK,
                                     umma_desc_k_sw128_sbo(qa + (kk >> 2) * AT_QHALF + (kk & 3) * 32, 1024),
                                     umma_desc_k_sw128_sbo(ka + (kk >> 2) * AT_KHALF + (kk & 3) * 32, 1024),
                                     idesc_s, kk > 0 ? 1u : 0u);
                        }
                        umma_commit(&sfull[x]);
                        s_last = x | ((k & 1) << 1) | 4;
                    }
                    if (ok) umma_commit(&qempty[qb]);     // Q is read by this item's S MMAs only
                    ++qi;
                }
            }
        } else {
            // ------------------------------------------------ PV issuer: O_x += P(b) V(b), x = b % 2
            if (lane == 0) {
                constexpr uint32_t idesc_o = umma_idesc_bf16_f32(AT_HEADS, AT_D, true);
                int qi = 0, g = 0, cnt[2] = {0, 0};
                bool ok = true;
                for (int64_t it = it_begin; it < it_end && ok; ++it) {
                    Item item;
                    item.set(a, it);
                    if (item.nblk == 0) continue;
                    for (int b = 0; b < item.nblk; ++b, ++g) {
                        const int st = g % AT_STAGES, x = b & 1, k = cnt[x]++;
                        // kvfull (long complete) orders this thread's V reads behind the copies;
                        // oempty: the previous item's O_0 and O_1 have been read
                        if (!wait_or_abort(&pfull[x], k & 1, &abort_flag) ||
                            !wait_or_abort(&kvfull[st], (g / AT_STAGES) & 1, &abort_flag) ||
                            (b == 0 && !wait_or_abort(oempty, (qi & 1) ^ 1, &abort_flag))) {
                            ok = false;
                            break;
                        }
                        fence_proxy_async_smem();
                        tc_fence_after();
                        const uint32_t va = smem_u32(KVs + st * AT_STAGE + AT_KTILE);
#pragma unroll
                        for (int kk = 0; kk < AT_BLK / 16; ++kk) {
                            const uint64_t bd = umma_desc_mn_sw128(va + kk * 2048, AT_KHALF, 1024);
                            umma_f16_ts(tO + x * AT_D, tP + x * 32 + kk * 8, bd, idesc_o, (b > 1 || kk > 0) ? 1u : 0u);
                        }
                        umma_commit(&kvempty[st]);        // S(b) completed before P(b) existed
                        umma_commit(&pempty[x]);
                        if (b == item.nblk - 1) umma_commit(ofull);
                        pv_last = x | ((k & 1) << 1) | 4;
                    }
                    ++qi;
                }
            }
        }
    } else {
        regs_inc<AT_REGS_HIGH>();
        // ------------------------------------------------ softmax sets (thread = head row)
        // Set x (warps 0-3: x = 0; warps 8-11: x = 1) takes blocks b = x, x + 2, ...
        // of every item, with its own S, P and O buffers and its own running max m
        // and sum l; two sets keep two softmax warps on every SM sub-partition, so
        // one's TMEM and memory latencies hide behind the other's arithmetic.  At
        // the end of an item set 1 hands (m, l) to set 0, which merges O_0 and O_1:
        //   O = (2^(m0 - m) O_0 + 2^(m1 - m) O_1) / (2^(m0 - m) l0 + 2^(m1 - m) l1).
        const int x = warp >> 3;
        const int q4 = warp & 3;
        const int h = q4 * 32 + lane;
        const uint32_t trow = (uint32_t)(q4 * 32) << 16;
        const uint32_t tSx = tS + x * AT_BLK, tOx = tO + x * AT_D;
        int qi = 0, g = 0, k = 0, mi = 0;   // items, blocks before this item, this set's blocks, merged items
        bool dead = false;
        for (int64_t it = it_begin; it < it_end; ++it) {
            Item item;
            item.set(a, it);
            float m = -INFINITY, l = 0.f;
            for (int b = x; b < item.nblk && !dead; b += 2, ++k) {
                const int gb = g + b, st = gb % AT_STAGES;
                // kvfull: acquire the producer's validity bits; sfull: S of block b is in TMEM.
                // Outcomes are made warp-uniform: the TMEM accesses below are warp-collective.
                bool ok = wait_or_abort(&kvfull[st], (gb / AT_STAGES) & 1, &abort_flag) &&
                          wait_or_abort(&sfull[x], k & 1, &abort_flag);
                if (!__all_sync(0xffffffffu, ok)) { dead = true; break; }
                tc_fence_after();
                // both halves of the S row in one TMEM round trip
                uint32_t va[32], vb[32];
                tmem_ld32(tSx + trow, va);
                tmem_ld32(tSx + trow + 32, vb);
                tmem_wait_ld_dep32(va);
                tmem_wait_ld_dep32(vb);
                float sv[AT_BLK];                     // raw q.k; unused slots -inf
#pragma unroll
                for (int i = 0; i < 32; ++i) { sv[i] = __uint_as_float(va[i]); sv[32 + i] = __uint_as_float(vb[i]); }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sempty[x]);
                const uint32_t vw0 = valid[st * 2], vw1 = valid[st * 2 + 1];
                if ((vw0 & vw1) != 0xffffffffu) {     // block-uniform: only blocks with unused slots mask
#pragma unroll
                    for (int i = 0; i < 32; ++i) {
                        if (!((vw0 >> i) & 1u)) sv[i] = -INFINITY;
                        if (!((vw1 >> i) & 1u)) sv[32 + i] = -INFINITY;
                    }
                }
                float mx[8];                          // eight independent max chains
#pragma unroll
                for (int i = 0; i < 8; ++i) mx[i] = sv[i];
#pragma unroll
                for (int i = 8; i < AT_BLK; ++i) mx[i & 7] = fmaxf(mx[i & 7], sv[i]);
                const float mr = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                       fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
                const float mb = mr * a.scale_log2;   // the scale is positive: max commutes with it
                float m_new = m, alpha = 1.f;
                if (mb > m + kRescaleThreshold || (m == -INFINITY && mb != -INFINITY)) {
                    m_new = mb;
                    alpha = m == -INFINITY ? 0.f : exp2f(m - m_new);
                }
                const float base = m_new == -INFINITY ? 0.f : m_new;
                // p = 2^(s * scale - base): one packed FMA per pair for the exponent,
                // four packed partial sums
                const uint64_t sc2 = f2_pack(a.scale_log2, a.scale_log2), nb2 = f2_pack(-base, -base);
                const uint64_t one2 = f2_pack(1.f, 1.f);
                uint64_t rs2[4] = {0ull, 0ull, 0ull, 0ull};
                uint32_t pk[AT_BLK / 2];
#pragma unroll
                for (int i = 0; i < AT_BLK / 2; ++i) {
                    float x0, x1;
                    f2_unpack(f2_fma(f2_pack(sv[2 * i], sv[2 * i + 1]), sc2, nb2), x0, x1);
                    const float p0 = ex2_sfu(x0), p1 = ex2_sfu(x1);
                    rs2[i & 3] = f2_fma(f2_pack(p0, p1), one2, rs2[i & 3]);
                    pk[i] = pack_bf16(p0, p1);
                }
                float rsum = 0.f;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    float lo, hi;
                    f2_unpack(rs2[q], lo, hi);
                    rsum += lo + hi;
                }
                l = l * alpha + rsum;
                m = m_new;
                // P_x is free and O_x up to date once this set's previous PV has completed
                ok = wait_or_abort(&pempty[x], (k & 1) ^ 1, &abort_flag);
                if (!__all_sync(0xffffffffu, ok)) { dead = true; break; }
                // Rescale O_x rows whose max moved.  tcgen05.ld/st are warp-collective: the
                // whole warp takes the branch if any of its rows needs it, the others multiply by 1.
                const bool need = b > x && alpha != 1.f;
                if (__any_sync(0xffffffffu, need)) {
                    const float f = need ? alpha : 1.f;
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < AT_D / 32; ++c) {
                        uint32_t v[32];
                        tmem_ld32(tOx + trow + c * 32, v);
                        tmem_wait_ld_dep32(v);
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
                        tmem_st32(tOx + trow + c * 32, v);
                    }
                    tmem_wait_st();
                }
                // P row h into tensor memory: 64 keys as 32 columns of bf16 pairs
                tmem_st32(tP + x * 32 + trow, pk);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&pfull[x]);
            }
            g += item.nblk;
            if (item.nblk == 0 && x == 1) continue;
            const bool two = item.nblk >= 2;
            if (x == 1) {
                // ---- set 1: hand its running max and sum to set 0 ----
                if (two) {
                    bool ok = !dead && wait_or_abort(mlempty, (mi & 1) ^ 1, &abort_flag);
                    if (__all_sync(0xffffffffu, ok)) {
                        mls[h] = m;
                        mls[AT_HEADS + h] = l;
                        __syncwarp();
                        if (lane == 0) mbar_arrive(mlfull);
                    } else {
                        dead = true;
                    }
                    ++mi;
                }
                continue;
            }
            // ---- set 0: merge the two sets, O / l and the log-sum-exp ----
            bool have = item.nblk > 0;
            float m1 = -INFINITY, l1 = 0.f;
            if (two) {
                bool ok = !dead && wait_or_abort(mlfull, mi & 1, &abort_flag);
                if (__all_sync(0xffffffffu, ok)) {
                    m1 = mls[h];
                    l1 = mls[AT_HEADS + h];
                    __syncwarp();
                    if (lane == 0) mbar_arrive(mlempty);
                } else {
                    dead = true;
                }
                ++mi;
            }
            if (have) {
                bool ok = !dead && wait_or_abort(ofull, qi & 1, &abort_flag);
                have = __all_sync(0xffffffffu, ok);
                dead = dead || !have;
            }
            const float mt = fmaxf(m, m1);
            const float f0 = (have && m != -INFINITY) ? exp2f(m - mt) : 0.f;
            const float f1 = (have && m1 != -INFINITY) ? exp2f(m1 - mt) : 0.f;
            const float lt = l * f0 + l1 * f1;
            const float inv = lt > 0.f ? 1.f / lt : 0.f;
            const float lse = lt > 0.f ? mt * kLn2 + logf(lt) : -INFINITY;
            const float g0 = f0 * inv, g1 = f1 * inv;
            const int64_t hh = (int64_t)item.hg * AT_HEADS + h;
            if (have) tc_fence_after();
#pragma unroll
            for (int c = 0; c < AT_D / 32; ++c) {
                float o[32];
                if (have) {
                    uint32_t v0[32], v1[32];
                    tmem_ld32(tO + trow + c * 32, v0);
                    if (two) tmem_ld32(tO + AT_D + trow + c * 32, v1);
                    tmem_wait_ld_dep32(v0);
                    if (two) {
                        tmem_wait_ld_dep32(v1);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __uint_as_float(v0[i]) * g0 + __uint_as_float(v1[i]) * g1;
                    } else {
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __uint_as_float(v0[i]) * g0;
                    }
                } else {
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[i] = 0.f;
                }
                if (a.splits == 1) {
                    uint16_t *orow = a.out + (item.row * a.H + hh) * AT_D + c * 32;
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        *reinterpret_cast<uint4 *>(orow + u * 8) =
                            make_uint4(pack_bf16(o[u * 8], o[u * 8 + 1]), pack_bf16(o[u * 8 + 2], o[u * 8 + 3]),
                                       pack_bf16(o[u * 8 + 4], o[u * 8 + 5]), pack_bf16(o[u * 8 + 6], o[u * 8 + 7]));
                } else {
                    float *po = a.part + ((item.row * a.splits + item.split) * a.H + hh) * (int64_t)AT_D + c * 32;
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        *reinterpret_cast<float4 *>(po + u * 4) = make_float4(o[u * 4], o[u * 4 + 1], o[u * 4 + 2], o[u * 4 + 3]);
                }
            }
            if (have) {
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(oempty);
            }
            if (a.splits == 1) {
                if (a.lse) a.lse[item.row * a.H + hh] = lse;
            } else {
                a.part[a.rows * a.splits * (int64_t)a.H * AT_D + (item.row * a.splits + item.split) * a.H + hh] = lse;
            }
            if (item.nblk > 0) ++qi;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (abort_flag && tid == 0) {
        record_error(a.hdr, DSA_ERR_TIMEOUT, blockIdx.x);
        // let copies and MMAs in flight land before shared and tensor memory go
        for (int j = kv_consumed; j < kv_issued; ++j) mbar_wait(&kvfull[j % AT_STAGES], (j / AT_STAGES) & 1);
        for (int j = q_consumed; j < q_issued; ++j) mbar_wait(&qfull[j & 1], (j >> 1) & 1);
        if (pv_last & 4) mbar_wait(&pempty[pv_last & 1], (pv_last >> 1) & 1);
        if (s_last & 4) mbar_wait(&sfull[s_last & 1], (s_last >> 1) & 1);
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace

bool sparse_attn_tc_supported(int H, int d) { return d == AT_D && H % AT_HEADS == 0 && H / AT_HEADS <= 65535; }

namespace {

template <bool KV8>
cudaError_t launch_attn_tc_impl(const CUtensorMap &qmap, const CUtensorMap &kmap, const CUtensorMap &vmap,
                                const AttnTcArgs &a, cudaStream_t st, bool chained)
{
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t smem = KV8 ? AtSmemKv8::total_kv8() : AtSmemBf16::total();
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, sparse_attn_tc_kernel<KV8>);
    if (e != cudaSuccess) return e;
    // the register split assumes it (the build checks it too): an error, not a silent slower path
    if (fa.numRegs != AT_LAUNCH_REGS) return cudaErrorInvalidKernelImage;
    e = cudaFuncSetAttribute(sparse_attn_tc_kernel<KV8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)std::min<int64_t>(a.items, sms);
    if (chained) {
        e = launch_chained(sparse_attn_tc_kernel<KV8>, dim3(grid), dim3(AT_THREADS), smem, st, qmap, kmap, vmap, a);
        if (e != cudaSuccess) return e;
    } else {
        sparse_attn_tc_kernel<KV8><<<grid, AT_THREADS, smem, st>>>(qmap, kmap, vmap, a);
    }
    return cudaGetLastError();
}

void fill_common(AttnTcArgs &a, const int32_t *idx, int64_t rows, int H, int ksel, int64_t kv_rows, int64_t T,
                 const int32_t *block_table, const int32_t *context_lens, int64_t num_pages, int max_pages,
                 int page_size, float sm_scale, uint16_t *out, float *lse, float *part, int splits, WsHeader *hdr)
{
    a.idx = idx; a.ksel = ksel; a.H = H; a.kv_rows = kv_rows; a.T = T;
    a.block_table = block_table; a.context_lens = context_lens; a.num_pages = num_pages;
    a.max_pages = max_pages; a.page_size = page_size;
    a.scale_log2 = sm_scale * kLog2e;
    a.out = out; a.lse = lse; a.part = part; a.rows = rows;
    a.splits = splits;
    a.chunk = (int)(ceil_div(ceil_div(ksel, splits), AT_BLK) * AT_BLK);
    a.items = rows * (H / AT_HEADS) * splits;
    a.hdr = hdr;
}

}  // namespace

cudaError_t launch_sparse_attn_tc(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                  int64_t kv_rows, int64_t T, const int32_t *block_table,
                                  const int32_t *context_lens, int64_t num_pages, int max_pages,
                                  int page_size, const int32_t *idx, int64_t rows, int H, int d,
                                  int ksel, float sm_scale, uint16_t *out, float *lse, float *part,
                                  int splits, WsHeader *hdr, cudaStream_t st, bool chained)
{
    if (rows <= 0) return cudaSuccess;
    if (!sparse_attn_tc_supported(H, d) || kv_rows >= ((int64_t)1 << 31) ||
        rows * H >= ((int64_t)1 << 31))
        return cudaErrorNotSupported;
    CUtensorMap qmap, kmap, vmap;
    if (!make_tmap_bf16_2d(&qmap, q, AT_D, (uint64_t)rows * H, AT_D * 2, 64, AT_HEADS) ||
        !make_tmap_bf16_2d(&kmap, k, AT_D, (uint64_t)kv_rows, AT_D * 2, 64, 1) ||
        !make_tmap_bf16_2d(&vmap, v, AT_D, (uint64_t)kv_rows, AT_D * 2, 64, 1))
        return cudaErrorNotSupported;
    AttnTcArgs a{};
    a.k = k; a.v = v;
    fill_common(a, idx, rows, H, ksel, kv_rows, T, block_table, context_lens, num_pages, max_pages, page_size,
                sm_scale, out, lse, part, splits, hdr);
    return launch_attn_tc_impl<false>(qmap, kmap, vmap, a, st, chained);
}

cudaError_t launch_sparse_attn_tc_kv8(const uint16_t *q, const uint8_t *k8, const float *ks, const uint8_t *v8,
                                      const float *vs, int64_t kv_rows, const int32_t *block_table,
                                      const int32_t *context_lens, int64_t num_pages, int max_pages,
                                      int page_size, const int32_t *idx, int64_t rows, int H, int d, int ksel,
                                      float sm_scale, uint16_t *out, float *lse, float *part, int splits,
                                      WsHeader *hdr, cudaStream_t st, bool chained)
{
    if (rows <= 0) return cudaSuccess;
    if (!sparse_attn_tc_supported(H, d) || kv_rows >= ((int64_t)1 << 31) ||
        rows * H >= ((int64_t)1 << 31))
        return cudaErrorNotSupported;
    CUtensorMap qmap;
    if (!make_tmap_bf16_2d(&qmap, q, AT_D, (uint64_t)rows * H, AT_D * 2, 64, AT_HEADS)) return cudaErrorNotSupported;
    AttnTcArgs a{};
    a.k8 = k8; a.v8 = v8; a.ks = ks; a.vs = vs;
    fill_common(a, idx, rows, H, ksel, kv_rows, 0, block_table, context_lens, num_pages, max_pages, page_size,
                sm_scale, out, lse, part, splits, hdr);
    // the K/V maps are parameters of the bf16 kernel's signature only; the KV8
    // producers copy with cp.async, so the query map stands in for them
    return launch_attn_tc_impl<true>(qmap, qmap, qmap, a, st, chained);
}

}  // namespace dsa
