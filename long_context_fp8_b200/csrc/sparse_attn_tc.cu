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
//             tiles of a 4-stage ring (many small loads in flight per SM: the
//             rows are scattered); one thread also brings the next item's Q
//             with TMA into a second Q buffer;
//   warp 6    MMA issuer: S = Q K^T (kind::f16, M 128 heads, N 64 rows,
//             K = 128 = 8 x 16) into one of two TMEM buffers, then
//             O += P V of the previous block (V read MN-major straight from
//             the gathered rows) into one of two TMEM O buffers (per item);
//   warps 0-3 softmax: thread = head row.  Reads its S row from TMEM, masks
//             unused slots, keeps the running max m and sum l in registers,
//             writes P (bf16) to one of two shared buffers for the PV MMA.  O is rescaled
//             (a TMEM round trip) only when the block max exceeds m by more
//             than 2^8 -- otherwise P <= 256 and m stays -- which is exact up
//             to rounding.  At the end O / l and the log-sum-exp are written.
// Every mbarrier wait is bounded (DSA_ERR_TIMEOUT on expiry).
#include <algorithm>

#include "kernels.h"
#include "sm100.cuh"

namespace dsa {
namespace {

using namespace sm100;

constexpr int AT_HEADS = 128;          // UMMA M: query heads per item
constexpr int AT_D = 128;              // head dim
constexpr int AT_BLK = 64;             // selected rows per block (UMMA N of S, K of PV)
constexpr int AT_STAGES = 4;           // K/V gather ring depth
constexpr int AT_THREADS = 224;        // 4 softmax warps, 2 producer warps, MMA warp
constexpr int AT_PRODUCERS = 64;       // producer threads: one selected row each per block

constexpr int AT_QHALF = AT_HEADS * 128;     // one 64-column half of Q (16 KB)
constexpr int AT_QTILE = 2 * AT_QHALF;       // Q of one item (32 KB)
constexpr int AT_KHALF = AT_BLK * 128;       // one 64-column half of a 64-row K or V tile (8 KB)
constexpr int AT_KTILE = 2 * AT_KHALF;       // a 64 x 128 bf16 tile (16 KB)
constexpr int AT_STAGE = 2 * AT_KTILE;       // K + V of one block (32 KB)
constexpr int AT_PTILE = AT_HEADS * 128;     // P of one block: 128 rows x 64 bf16 (16 KB)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.f;     // log2 units

struct AttnTcArgs {
    const uint16_t *k;       // K rows [kv_rows, D] (contiguous or paged cache)
    const uint16_t *v;
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

struct AtSmem {
    static constexpr size_t q_off = 0;                                   // [2] Q tiles
    static constexpr size_t kv_off = q_off + 2 * AT_QTILE;                // [stages] K, V tiles
    static constexpr size_t p_off = kv_off + (size_t)AT_STAGES * AT_STAGE; // [2] P tiles
    static constexpr size_t valid_off = p_off + 2 * AT_PTILE;            // [stages][2] validity bits
    static constexpr size_t bar_off = valid_off + AT_STAGES * 2 * 4;
    // qfull[2] qempty[2] kvfull[S] kvempty[S] sfull[2] sempty[2] pfull[2] pempty[2] ofull[2] oempty[2]
    static constexpr int n_bars = 2 * AT_STAGES + 16;
    static constexpr size_t slot_off = bar_off + 8 * n_bars;
    static constexpr size_t total = slot_off + 16 + 1024;
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

__global__ void __launch_bounds__(AT_THREADS, 1)
sparse_attn_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap, const AttnTcArgs a)
{
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t *Qs = smem + AtSmem::q_off;
    uint8_t *KVs = smem + AtSmem::kv_off;
    uint8_t *Ps = smem + AtSmem::p_off;
    uint32_t *valid = reinterpret_cast<uint32_t *>(smem + AtSmem::valid_off);
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + AtSmem::bar_off);
    uint64_t *qfull = bars, *qempty = bars + 2, *kvfull = bars + 4, *kvempty = kvfull + AT_STAGES;
    uint64_t *sfull = kvempty + AT_STAGES, *sempty = sfull + 2, *pfull = sempty + 2, *pempty = pfull + 2;
    uint64_t *ofull = pempty + 2, *oempty = ofull + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + AtSmem::slot_off);
    __shared__ volatile int abort_flag;
    __shared__ int kv_issued, kv_consumed, q_issued, q_consumed, mma_blocks;

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
            mbar_init(&sfull[i], 1); mbar_init(&sempty[i], 4);
            mbar_init(&pfull[i], 4); mbar_init(&pempty[i], 1);
            mbar_init(&ofull[i], 1); mbar_init(&oempty[i], 4);
        }
        // kvfull: one asynchronous arrival per producer thread when its copies land,
        // plus one ordinary arrival per producer warp publishing the validity bits
        for (int i = 0; i < AT_STAGES; ++i) { mbar_init(&kvfull[i], AT_PRODUCERS + 2); mbar_init(&kvempty[i], 1); }
        abort_flag = 0;
        kv_issued = kv_consumed = q_issued = q_consumed = mma_blocks = 0;
        fence_mbar_init();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tO = tmem + 2 * AT_BLK;    // S [0,128), O [128,384)

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
            // warp (w - 4) copies rows 32 (w - 4) .. +31 of each block; lane l copies
            // 16-byte chunk l % 16 of the row's K (l < 16) or V (l >= 16), so one
            // instruction moves one whole row pair (two 256-byte runs).  Lane l also
            // resolves row 32 (w - 4) + l of the block, broadcast by shuffles.
            const int rbase = (warp - 4) * 32;
            int e = item.e0 + rbase + lane;
            int p_next = e < item.e1 ? __ldg(irow + e) : -1;
            const int chunk = lane & 15;
            const bool is_v = lane >= 16;
            for (int b = 0; b < item.nblk && !stop; ++b, ++g) {
                const int st = g % AT_STAGES;
                const int p = p_next;
                e += AT_BLK;                          // prefetch the next block's index
                p_next = (b + 1 < item.nblk && e < item.e1) ? __ldg(irow + e) : -1;
                // warp-uniform outcome: the ballot and shuffles below need every lane
                const bool ok = __all_sync(0xffffffffu,
                                           wait_or_abort(&kvempty[st], ((g / AT_STAGES) & 1) ^ 1, &abort_flag));
                if (!ok) { stop = true; break; }
                int64_t r = 0;
                bool v = false;
                if (paged) {
                    if (p >= 0 && p < ctx) {
                        const int page = a.block_table[item.row * a.max_pages + p / a.page_size];
                        if (page >= 0 && page < a.num_pages) {
                            r = (int64_t)page * a.page_size + p % a.page_size;
                            v = true;
                        } else {
                            record_error(a.hdr, DSA_ERR_INVALID_ARG, (unsigned)item.row);
                        }
                    }
                } else if (p >= 0 && p < a.T) {
                    r = p;
                    v = true;
                }
                const unsigned vw = __ballot_sync(0xffffffffu, v);
                if (lane == 0) {
                    valid[st * 2 + (warp - 4)] = vw;
                    mbar_arrive(&kvfull[st]);          // releases the validity bits
                }
                uint8_t *tile = KVs + st * AT_STAGE + (is_v ? AT_KTILE : 0);
                const uint16_t *base = is_v ? a.v : a.k;
                const int coff = (chunk >> 3) * AT_KHALF;
#pragma unroll 4
                for (int i = 0; i < 32; ++i) {
                    const int j = rbase + i;          // row of the block
                    const int64_t ri = __shfl_sync(0xffffffffu, r, i);
                    const bool vi = (vw >> i) & 1u;
                    cp_async_16(tile + coff + j * 128 + (((chunk & 7) ^ (j & 7)) << 4),
                                base + ri * AT_D + chunk * 8, vi);
                }
                cp_async_arrive_noinc(&kvfull[st]);   // fires when this thread's copies land
                if (pt == 0) kv_issued = g + 1;
            }
        }
        cp_async_wait<0>();                           // nothing in flight when the CTA retires
    } else if (warp == 6) {
        // ------------------------------------------------ MMA issuer: S(g), then PV(g - 1)
        if (lane == 0) {
            constexpr uint32_t idesc_s = umma_idesc_bf16_f32(AT_HEADS, AT_BLK, false);
            constexpr uint32_t idesc_o = umma_idesc_bf16_f32(AT_HEADS, AT_D, true);
            // the pending PV: block gp of the item with Q/O buffer slot qp, first/last flags
            int gp = -1, qp = 0;
            bool p_first = false, p_last = false;
            auto issue_pv = [&]() -> bool {
                const int st = gp % AT_STAGES, pb = gp & 1, ob = qp & 1;
                if (!wait_or_abort(&pfull[pb], (gp >> 1) & 1, &abort_flag)) return false;
                if (p_first && !wait_or_abort(&oempty[ob], ((qp >> 1) & 1) ^ 1, &abort_flag)) return false;
                tc_fence_after();
                const uint32_t pa = smem_u32(Ps + pb * AT_PTILE);
                const uint32_t va = smem_u32(KVs + st * AT_STAGE + AT_KTILE);
#pragma unroll
                for (int kk = 0; kk < AT_BLK / 16; ++kk) {
                    const uint64_t ad = umma_desc_k_sw128_sbo(pa + kk * 32, 1024);
                    const uint64_t bd = umma_desc_mn_sw128(va + kk * 2048, AT_KHALF, 1024);
                    umma_f16(tO + ob * AT_D, ad, bd, idesc_o, (!p_first || kk > 0) ? 1u : 0u);
                }
                umma_commit(&kvempty[st]);
                umma_commit(&pempty[pb]);
                if (p_last) {
                    umma_commit(&ofull[ob]);
                    umma_commit(&qempty[ob]);
                }
                mma_blocks = gp + 1;
                return true;
            };
            int qi = 0, g = 0;
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
                    const int st = g % AT_STAGES, sb = g & 1;
                    if (!wait_or_abort(&kvfull[st], (g / AT_STAGES) & 1, &abort_flag) ||
                        !wait_or_abort(&sempty[sb], ((g >> 1) & 1) ^ 1, &abort_flag)) { ok = false; break; }
                    kv_consumed = g + 1;
                    fence_proxy_async_smem();         // cp.async wrote the tiles; the MMA reads them
                    tc_fence_after();
                    const uint32_t ka = smem_u32(KVs + st * AT_STAGE);
#pragma unroll
                    for (int kk = 0; kk < AT_D / 16; ++kk) {
                        umma_f16(tS + sb * AT_BLK,
                                 umma_desc_k_sw128_sbo(qa + (kk >> 2) * AT_QHALF + (kk & 3) * 32, 1024),
                                 umma_desc_k_sw128_sbo(ka + (kk >> 2) * AT_KHALF + (kk & 3) * 32, 1024),
                                 idesc_s, kk > 0 ? 1u : 0u);
                    }
                    umma_commit(&sfull[sb]);
                    if (gp >= 0 && !issue_pv()) { ok = false; break; }
                    gp = g; qp = qi; p_first = b == 0; p_last = b == item.nblk - 1;
                }
                ++qi;
            }
            if (ok && gp >= 0) issue_pv();
        }
    } else {
        // ------------------------------------------------ softmax (thread = head row)
        const int h = warp * 32 + lane;
        const uint32_t trow = (uint32_t)(warp * 32) << 16;
        int qi = 0, g = 0;
        bool dead = false;
        for (int64_t it = it_begin; it < it_end; ++it) {
            Item item;
            item.set(a, it);
            float m = -INFINITY, l = 0.f;
            const int ob = qi & 1;
            bool have = item.nblk > 0;
            for (int b = 0; b < item.nblk && !dead; ++b, ++g) {
                const int st = g % AT_STAGES, sb = g & 1;
                // kvfull: acquire the producer's validity bits; sfull: S of block g is in TMEM.
                // Outcomes are made warp-uniform: the TMEM accesses below are warp-collective.
                bool ok = wait_or_abort(&kvfull[st], (g / AT_STAGES) & 1, &abort_flag) &&
                          wait_or_abort(&sfull[sb], (g >> 1) & 1, &abort_flag);
                if (!__all_sync(0xffffffffu, ok)) { dead = true; break; }
                tc_fence_after();
                float sv[AT_BLK];
#pragma unroll
                for (int c = 0; c < AT_BLK / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld32(tS + trow + sb * AT_BLK + c * 32, v);
                    tmem_wait_ld_dep32(v);
                    const uint32_t vw = valid[st * 2 + c];
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        sv[c * 32 + i] = ((vw >> i) & 1u) ? __uint_as_float(v[i]) * a.scale_log2 : -INFINITY;
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&sempty[sb]);
                float mb = -INFINITY;
#pragma unroll
                for (int i = 0; i < AT_BLK; ++i) mb = fmaxf(mb, sv[i]);
                float m_new = m, alpha = 1.f;
                if (mb > m + kRescaleThreshold || (m == -INFINITY && mb != -INFINITY)) {
                    m_new = mb;
                    alpha = m == -INFINITY ? 0.f : exp2f(m - m_new);
                }
                const float base = m_new == -INFINITY ? 0.f : m_new;
                float rs = 0.f;
                uint32_t pk[AT_BLK / 2];
#pragma unroll
                for (int i = 0; i < AT_BLK / 2; ++i) {
                    const float p0 = exp2f(sv[2 * i] - base), p1 = exp2f(sv[2 * i + 1] - base);
                    rs += p0 + p1;
                    pk[i] = pack_bf16(p0, p1);
                }
                l = l * alpha + rs;
                m = m_new;
                // P buffer sb is free once PV(g - 2) has completed
                ok = wait_or_abort(&pempty[sb], ((g >> 1) & 1) ^ 1, &abort_flag);
                if (!__all_sync(0xffffffffu, ok)) { dead = true; break; }
                // Rescale O rows whose max moved (needs PV(g - 1) done).  tcgen05.ld/st are
                // warp-collective: the whole warp takes the branch if any of its rows needs
                // it, the others multiply by 1.
                const bool need = b > 0 && alpha != 1.f;
                if (__any_sync(0xffffffffu, need)) {
                    ok = wait_or_abort(&pempty[(g - 1) & 1], ((g - 1) >> 1) & 1, &abort_flag);
                    if (!__all_sync(0xffffffffu, ok)) { dead = true; break; }
                    const float f = need ? alpha : 1.f;
                    tc_fence_after();
#pragma unroll
                    for (int c = 0; c < AT_D / 32; ++c) {
                        uint32_t v[32];
                        tmem_ld32(tO + trow + ob * AT_D + c * 32, v);
                        tmem_wait_ld_dep32(v);
#pragma unroll
                        for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * f);
                        tmem_st32(tO + trow + ob * AT_D + c * 32, v);
                    }
                    tmem_wait_st();
                }
                // P row h: 64 keys = 128 bytes, 16-byte chunks swizzled by h % 8
                uint8_t *prow = Ps + sb * AT_PTILE + h * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<uint4 *>(prow + ((c ^ (h & 7)) << 4)) =
                        make_uint4(pk[c * 4], pk[c * 4 + 1], pk[c * 4 + 2], pk[c * 4 + 3]);
                fence_proxy_async_smem();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&pfull[sb]);
            }
            // ---- item epilogue: O / l and the log-sum-exp ----
            float o[AT_D];
            if (have) {
                bool ok = !dead && wait_or_abort(&ofull[ob], (qi >> 1) & 1, &abort_flag);
                have = __all_sync(0xffffffffu, ok);
                dead = dead || !have;
            }
            if (have) {
                tc_fence_after();
#pragma unroll
                for (int c = 0; c < AT_D / 32; ++c) {
                    uint32_t v[32];
                    tmem_ld32(tO + trow + ob * AT_D + c * 32, v);
                    tmem_wait_ld_dep32(v);
#pragma unroll
                    for (int i = 0; i < 32; ++i) o[c * 32 + i] = __uint_as_float(v[i]);
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&oempty[ob]);
            } else {
#pragma unroll
                for (int i = 0; i < AT_D; ++i) o[i] = 0.f;
            }
            if (item.nblk > 0) ++qi;
            const float inv = (have && l > 0.f) ? 1.f / l : 0.f;
            const float lse = (have && l > 0.f) ? m * kLn2 + logf(l) : -INFINITY;
            const int64_t hh = (int64_t)item.hg * AT_HEADS + h;
            if (a.splits == 1) {
                uint16_t *orow = a.out + (item.row * a.H + hh) * AT_D;
#pragma unroll
                for (int c = 0; c < AT_D / 8; ++c) {
                    uint4 w = make_uint4(pack_bf16(o[c * 8] * inv, o[c * 8 + 1] * inv),
                                         pack_bf16(o[c * 8 + 2] * inv, o[c * 8 + 3] * inv),
                                         pack_bf16(o[c * 8 + 4] * inv, o[c * 8 + 5] * inv),
                                         pack_bf16(o[c * 8 + 6] * inv, o[c * 8 + 7] * inv));
                    *reinterpret_cast<uint4 *>(orow + c * 8) = w;
                }
                if (a.lse) a.lse[item.row * a.H + hh] = lse;
            } else {
                float *po = a.part + ((item.row * a.splits + item.split) * a.H + hh) * (int64_t)AT_D;
                float *pl = a.part + a.rows * a.splits * (int64_t)a.H * AT_D +
                            (item.row * a.splits + item.split) * a.H + hh;
#pragma unroll
                for (int c = 0; c < AT_D / 4; ++c)
                    *reinterpret_cast<float4 *>(po + c * 4) =
                        make_float4(o[c * 4] * inv, o[c * 4 + 1] * inv, o[c * 4 + 2] * inv, o[c * 4 + 3] * inv);
                *pl = lse;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (abort_flag && tid == 0) {
        record_error(a.hdr, DSA_ERR_TIMEOUT, blockIdx.x);
        // let copies and MMAs in flight land before shared and tensor memory go
        for (int j = kv_consumed; j < kv_issued; ++j) mbar_wait(&kvfull[j % AT_STAGES], (j / AT_STAGES) & 1);
        for (int j = q_consumed; j < q_issued; ++j) mbar_wait(&qfull[j & 1], (j >> 1) & 1);
        if (mma_blocks > 0) mbar_wait(&pempty[(mma_blocks - 1) & 1], ((mma_blocks - 1) >> 1) & 1);
    }
    __syncthreads();
    tc_fence_after();
    if (warp == 0) tmem_dealloc(tmem, 512);
}

}  // namespace

bool sparse_attn_tc_supported(int H, int d) { return d == AT_D && H % AT_HEADS == 0 && H / AT_HEADS <= 65535; }

cudaError_t launch_sparse_attn_tc(const uint16_t *q, const uint16_t *k, const uint16_t *v,
                                  int64_t kv_rows, int64_t T, const int32_t *block_table,
                                  const int32_t *context_lens, int64_t num_pages, int max_pages,
                                  int page_size, const int32_t *idx, int64_t rows, int H, int d,
                                  int ksel, float sm_scale, uint16_t *out, float *lse, float *part,
                                  int splits, WsHeader *hdr, cudaStream_t st)
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
    a.idx = idx; a.ksel = ksel; a.H = H; a.kv_rows = kv_rows; a.T = T;
    a.block_table = block_table; a.context_lens = context_lens; a.num_pages = num_pages;
    a.max_pages = max_pages; a.page_size = page_size;
    a.scale_log2 = sm_scale * kLog2e;
    a.out = out; a.lse = lse; a.part = part; a.rows = rows;
    a.splits = splits;
    a.chunk = (int)(ceil_div(ceil_div(ksel, splits), AT_BLK) * AT_BLK);
    a.items = rows * (H / AT_HEADS) * splits;
    a.hdr = hdr;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const size_t smem = AtSmem::total;
    cudaError_t e = cudaFuncSetAttribute(sparse_attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const unsigned grid = (unsigned)std::min<int64_t>(a.items, sms);
    sparse_attn_tc_kernel<<<grid, AT_THREADS, smem, st>>>(qmap, kmap, vmap, a);
    return cudaGetLastError();
}

}  // namespace dsa
