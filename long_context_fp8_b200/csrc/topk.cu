// Top-k selector ("DeepSeek-V3.2-Exp 稀疏注意力机制(DSA)技术深度解析", section 1:
// keep only the k best-scoring KV per query token; the hotdry page's
// "fine-grained selector").  Exact: the min(k, n) largest scores of a row, ties
// toward the lower position, emitted in ascending position order.
//
// One CTA per row.  Scores are mapped to order-preserving uint32 keys (-0
// folded onto +0).  Normally one pass over the row: a threshold tau is guessed
// from 2048 evenly spaced samples (the sample rank that should leave about
// 1.5 k keys of the row at or above it), and an ordered compaction copies
// every (key, position) with key >= tau into shared memory.  If that yields at
// least k and at most the buffer's capacity, the selection is among them:
// an exact radix select over the candidates on chip and a last ordered
// compaction emit it in ascending position order (no sort needed).  Rows
// short enough to fit are copied whole.  Otherwise the row falls back to two
// passes: a histogram of the top 11 key bits (warp-aggregated atomics) fixes
// the bin holding the k-th largest key, the keys in or above it go on chip;
// and if even those do not fit, a radix select runs over the row in global
// memory.  Every path is exact; the guess only decides which one is taken.
//
// With a sliding window of W positions ("DeepSeek-V4 百万 token 上下文的工程实现",
// section on the sliding-window KV cache: the most recent tokens keep their
// full KV) only the positions before the window compete, and the W window
// positions follow the selected ones in the output row of k + W entries.
#include <algorithm>

#include "kernels.h"

namespace dsa {
namespace {

constexpr int TK_ITEMS = 8;                          // consecutive positions per thread per step

// Launch shape of a top-k kernel: NT threads per CTA, a shared-memory
// candidate buffer of CAP entries, NSAMP samples for the threshold guess,
// taken one by one at evenly spaced positions or (RUNS) as runs of 8
// consecutive positions (one 32-byte sector each, instead of a sector per
// sample), kept in the candidate buffer, which is free until the guess is made.
template <int NT_, int CAP_, int NSAMP_, bool RUNS_>
struct TopkCfg {
    static constexpr int NT = NT_;
    static constexpr int WARPS = NT_ / 32;
    static constexpr int STEP = NT_ * TK_ITEMS;      // positions per block-wide step
    static constexpr int CAP = CAP_;
    static constexpr int WCAP = CAP_ / WARPS;        // candidate slots per warp
    static constexpr int NSAMP = NSAMP_;
    static constexpr bool RUNS = RUNS_;
    static_assert(!RUNS_ || (NSAMP_ <= CAP_ && NSAMP_ % (8 * NT_) == 0), "sample runs must fit the buffer");
};
// Causal prefill rows: two 512-thread CTAs per SM; 4096 threshold samples in
// runs of 8 (a sector each) kept in the candidate buffer.
using RowsCfg = TopkCfg<512, 8192, 4096, true>;
// Decode rows split over CTAs (and the final join of their candidates).
using SplitCfg = TopkCfg<512, 8192, 2048, false>;

template <class C>
struct TopkSmem {
    uint32_t hist[2048];
    uint32_t warp_buf[32];
    uint32_t sh_bin, sh_above, sh_count, sh_overflow, sh_diff;
    uint32_t wcnt[C::WARPS], wbefore[C::WARPS + 1];
    uint32_t sample_store[C::RUNS ? 1 : C::NSAMP];
    uint32_t ckey[C::CAP];
    int32_t cpos[C::CAP];
    __device__ __forceinline__ uint32_t *sample() { return C::RUNS ? ckey : sample_store; }
};

// Exclusive block-wide prefix sum of `v`; the block total goes to *total.
template <class C>
__device__ __forceinline__ uint32_t block_excl_scan(uint32_t v, uint32_t *warp_buf, uint32_t *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) warp_buf[warp] = x;
    __syncthreads();
    if (warp == 0) {
        uint32_t s = lane < C::WARPS ? warp_buf[lane] : 0u;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            uint32_t y = __shfl_up_sync(0xffffffffu, s, o);
            if (lane >= o) s += y;
        }
        if (lane < C::WARPS) warp_buf[lane] = s;
    }
    __syncthreads();
    uint32_t before = (warp > 0 ? warp_buf[warp - 1] : 0u) + x - v;
    *total = warp_buf[C::WARPS - 1];
    __syncthreads();
    return before;
}

// Raw scores of positions [s, s + 8) of a row (0 past n).  Kept apart from
// the key conversion so that a loop can issue the next step's loads before it
// works on the current step's values.
__device__ __forceinline__ void load_raw8(const float *row, int64_t n, int64_t s, bool vec, float (&v)[TK_ITEMS])
{
    if (vec && s + TK_ITEMS <= n) {
        const float4 a = __ldg(reinterpret_cast<const float4 *>(row + s));
        const float4 b = __ldg(reinterpret_cast<const float4 *>(row + s + 4));
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w; v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
    } else {
#pragma unroll
        for (int i = 0; i < TK_ITEMS; ++i) v[i] = s + i < n ? row[s + i] : 0.f;
    }
}

// Keys of raw scores of positions [s, s + 8) (bit i of *valid set when s + i < n).
__device__ __forceinline__ void keys_of(const float (&v)[TK_ITEMS], int64_t n, int64_t s,
                                        uint32_t (&key)[TK_ITEMS], uint32_t &valid)
{
    valid = 0;
#pragma unroll
    for (int i = 0; i < TK_ITEMS; ++i) {
        key[i] = float_key(v[i]);
        if (s + i < n) valid |= 1u << i;
    }
}

// Keys of positions [s, s + 8) of a row (bit i of *valid set when s + i < n).
__device__ __forceinline__ void load8(const float *row, int64_t n, int64_t s, bool vec,
                                      uint32_t (&key)[TK_ITEMS], uint32_t &valid)
{
    float v[TK_ITEMS];
    load_raw8(row, n, s, vec, v);
    keys_of(v, n, s, key, valid);
}

// Bin holding the `remaining`-th largest count (from the top), and how many
// counts lie strictly above it.  All threads call it; results in smem.
template <class C>
__device__ __forceinline__ void find_bin(TopkSmem<C> &sm, int nb, uint32_t remaining)
{
    const int tid = threadIdx.x;
    const int bpt = nb > C::NT ? nb / C::NT : 1;     // nb: a power of two
    uint32_t local = 0;
    for (int j = 0; j < bpt; ++j) {
        const int b = nb - 1 - (tid * bpt + j);
        if (b >= 0) local += sm.hist[b];
    }
    uint32_t tot;
    uint32_t cum = block_excl_scan<C>(local, sm.warp_buf, &tot);
    for (int j = 0; j < bpt; ++j) {
        const int b = nb - 1 - (tid * bpt + j);
        if (b < 0) break;
        uint32_t c = sm.hist[b];
        if (cum < remaining && remaining <= cum + c) { sm.sh_bin = (uint32_t)b; sm.sh_above = cum; }
        cum += c;
    }
    __syncthreads();
}

// Ordered compaction of a key sequence given by get(i) for i in [0, n):
// emits pos(i) for keys above thr and for the first `need` keys equal to thr.
template <class C, class GetKey, class GetPos>
__device__ __forceinline__ void emit_selected(TopkSmem<C> &sm, int64_t n, uint32_t thr, uint32_t need,
                                              int k, int32_t *out, GetKey get, GetPos pos_of)
{
    const int tid = threadIdx.x;
    uint32_t base_gt = 0, base_eq = 0;
    for (int64_t c0 = 0; c0 < n; c0 += C::STEP) {
        const int64_t i0 = c0 + (int64_t)tid * TK_ITEMS;
        uint32_t flags_gt = 0, flags_eq = 0, n_gt = 0, n_eq = 0;
        uint32_t keys[TK_ITEMS], valid;
        get(i0, keys, valid);
#pragma unroll
        for (int i = 0; i < TK_ITEMS; ++i) {
            if ((valid >> i) & 1u) {
                if (keys[i] > thr) { flags_gt |= 1u << i; ++n_gt; }
                else if (keys[i] == thr) { flags_eq |= 1u << i; ++n_eq; }
            }
        }
        uint32_t tot;
        uint32_t ex = block_excl_scan<C>((n_gt << 16) | n_eq, sm.warp_buf, &tot);
        uint32_t gt_before = base_gt + (ex >> 16), eq_before = base_eq + (ex & 0xffffu);
#pragma unroll
        for (int i = 0; i < TK_ITEMS; ++i) {
            bool gt = (flags_gt >> i) & 1u, eq = (flags_eq >> i) & 1u;
            if (gt || (eq && eq_before < need)) {
                uint32_t p = gt_before + min(eq_before, need);
                if (p < (uint32_t)k) out[p] = pos_of(i0 + i);
            }
            gt_before += gt;
            eq_before += eq;
        }
        base_gt += tot >> 16;
        base_eq += tot & 0xffffu;
    }
}

// Given the candidates (every key whose top 11 bits are >= b1, in ascending
// position order) in shared memory, resolve the remaining 21 bits of the
// threshold on chip and emit the selection in position order.
template <class C>
__device__ __noinline__ void select_on_chip(TopkSmem<C> &sm, uint32_t ncand, uint32_t b1, uint32_t remaining, int k,
                               int32_t *out)
{
    const int tid = threadIdx.x;
    uint32_t prefix = b1 << 21, pmask = 0x7FFu << 21;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const int shift = pass == 0 ? 10 : 0;
        const int nb = pass == 0 ? 2048 : 1024;
        const uint32_t bmask = (uint32_t)nb - 1u;
        for (int i = tid; i < nb; i += C::NT) sm.hist[i] = 0u;
        __syncthreads();
        for (uint32_t j = tid; j < ncand; j += C::NT) {
            uint32_t key = sm.ckey[j];
            if ((key & pmask) == prefix) atomicAdd(&sm.hist[(key >> shift) & bmask], 1u);
        }
        __syncthreads();
        find_bin(sm, nb, remaining);
        remaining -= sm.sh_above;
        prefix |= sm.sh_bin << shift;
        pmask |= bmask << shift;
        __syncthreads();
    }
    emit_selected(
        sm, ncand, prefix, remaining, k, out,
        [&](int64_t i0, uint32_t (&keys)[TK_ITEMS], uint32_t &valid) {
            valid = 0;
#pragma unroll
            for (int i = 0; i < TK_ITEMS; ++i) {
                keys[i] = 0;
                if (i0 + i < (int64_t)ncand) { keys[i] = sm.ckey[i0 + i]; valid |= 1u << i; }
            }
        },
        [&](int64_t i) { return sm.cpos[i]; });
}

// Radix select over keys[0..n) in shared memory (n >= 1): the `rank`-th
// largest key (*thr) and how many keys equal to it rank within the first
// `rank` (*need).  The digits start below the bits that all keys share (found
// by an OR-reduction of key ^ keys[0]), so that the first histogram spreads
// over the keys' actual range instead of piling onto one bin of the top bits.
// With passes = 3 the result is exact; with fewer, the bits not yet resolved
// are zero in *thr (a threshold at or below the exact key).  refine = false
// skips the direct search among a small last bin (for a threshold guess, the
// bin's lower bound serves as well and saves its barriers).
template <class C>
__device__ void radix_select_smem(TopkSmem<C> &sm, const uint32_t *keys, uint32_t n, uint32_t rank,
                                  uint32_t *thr, uint32_t *need, int passes = 3, bool refine = true)
{
    const int tid = threadIdx.x;
    const uint32_t first = keys[0];
    if (tid == 0) sm.sh_diff = 0u;
    __syncthreads();
    uint32_t diff = 0;
    for (uint32_t j = tid; j < n; j += C::NT) diff |= keys[j] ^ first;
    diff = __reduce_or_sync(0xffffffffu, diff);
    if ((tid & 31) == 0 && diff) atomicOr(&sm.sh_diff, diff);
    __syncthreads();
    diff = sm.sh_diff;
    uint32_t remaining = rank;
    if (diff == 0u) {                                     // every key equal
        *thr = first;
        *need = remaining;
        return;
    }
    int lo = 32 - __clz(diff);                            // bits [0, lo) still to resolve
    uint32_t pmask = lo == 32 ? 0u : ~((1u << lo) - 1u);
    uint32_t prefix = first & pmask;
#pragma unroll 1
    for (int pass = 0; pass < passes && lo > 0; ++pass) {
        const int width = lo < 11 ? lo : 11;
        const int shift = lo - width;
        const int nb = 1 << width;
        const uint32_t bmask = (uint32_t)nb - 1u;
        for (int i = tid; i < nb; i += C::NT) sm.hist[i] = 0u;
        __syncthreads();
        for (uint32_t j = tid; j < n; j += C::NT) {
            const uint32_t key = keys[j];
            if ((key & pmask) == prefix) atomicAdd(&sm.hist[(key >> shift) & bmask], 1u);
        }
        __syncthreads();
        find_bin(sm, nb, remaining);
        remaining -= sm.sh_above;
        const uint32_t in_bin = sm.hist[sm.sh_bin];
        prefix |= sm.sh_bin << shift;
        pmask |= bmask << shift;
        lo = shift;
        __syncthreads();
        if (refine && lo > 0 && in_bin <= 64) {
            // Few keys share the bin of the rank-th key: gather them (their order does
            // not matter) and find it among them directly, instead of more passes:
            // it is the x with  #{y > x} < remaining <= #{y >= x}.
            uint32_t *bk = sm.hist;
            if (tid == 0) sm.sh_count = 0u;
            __syncthreads();
            for (uint32_t j = tid; j < n; j += C::NT) {
                const uint32_t key = keys[j];
                if ((key & pmask) == prefix) bk[atomicAdd(&sm.sh_count, 1u)] = key;
            }
            __syncthreads();
            if (tid < 32) {
                const uint32_t m = sm.sh_count;
                for (uint32_t i = tid; i < m; i += 32) {
                    const uint32_t x = bk[i];
                    uint32_t gt = 0, ge = 0;
                    for (uint32_t u = 0; u < m; ++u) { gt += bk[u] > x; ge += bk[u] >= x; }
                    if (gt < remaining && remaining <= ge) { sm.sh_bin = x; sm.sh_above = remaining - gt; }
                }
            }
            __syncthreads();
            *thr = sm.sh_bin;
            *need = sm.sh_above;
            __syncthreads();
            return;
        }
    }
    *thr = prefix;
    *need = remaining;
}

// Exact select among the candidates in shared memory (every key that could
// be selected, in ascending position order), emitted in position order.
template <class C>
__device__ void select_candidates(TopkSmem<C> &sm, uint32_t ncand, int k, int32_t *out)
{
    uint32_t thr, need;
    radix_select_smem(sm, sm.ckey, ncand, (uint32_t)k, &thr, &need);
    emit_selected(
        sm, ncand, thr, need, k, out,
        [&](int64_t i0, uint32_t (&keys)[TK_ITEMS], uint32_t &valid) {
            valid = 0;
#pragma unroll
            for (int i = 0; i < TK_ITEMS; ++i) {
                keys[i] = 0;
                if (i0 + i < (int64_t)ncand) { keys[i] = sm.ckey[i0 + i]; valid |= 1u << i; }
            }
        },
        [&](int64_t i) { return sm.cpos[i]; });
}

// Ordered copy of every key of the row that passes `keep` into the candidate
// buffer; returns the total count (entries past C::CAP are counted, not
// stored).  Each thread takes 8 consecutive positions per step (two 16-byte
// loads), one block scan per 4K positions.
template <class C, class Keep>
__device__ uint32_t collect_candidates(TopkSmem<C> &sm, const float *row, int64_t n, bool vec, Keep keep)
{
    constexpr int D = 2;                                   // steps of loads in flight
    const int tid = threadIdx.x;
    uint32_t base = 0;
    float ring[D][TK_ITEMS];
#pragma unroll
    for (int q = 0; q < D; ++q)
        if ((int64_t)q * C::STEP < n) load_raw8(row, n, (int64_t)q * C::STEP + (int64_t)tid * TK_ITEMS, vec, ring[q]);
    for (int64_t c0 = 0; c0 < n; c0 += (int64_t)D * C::STEP) {
#pragma unroll
        for (int q = 0; q < D; ++q) {
            const int64_t cq = c0 + (int64_t)q * C::STEP;
            if (cq >= n) break;                            // block-uniform
            const int64_t s0 = cq + (int64_t)tid * TK_ITEMS;
            uint32_t keys[TK_ITEMS], valid;
            keys_of(ring[q], n, s0, keys, valid);
            if (cq + (int64_t)D * C::STEP < n) load_raw8(row, n, s0 + (int64_t)D * C::STEP, vec, ring[q]);
            uint32_t flags = 0, cnt = 0;
#pragma unroll
            for (int i = 0; i < TK_ITEMS; ++i)
                if (((valid >> i) & 1u) && keep(keys[i])) { flags |= 1u << i; ++cnt; }
            uint32_t tot;
            uint32_t off = base + block_excl_scan<C>(cnt, sm.warp_buf, &tot);
#pragma unroll
            for (int i = 0; i < TK_ITEMS; ++i) {
                if ((flags >> i) & 1u) {
                    if (off < C::CAP) { sm.ckey[off] = keys[i]; sm.cpos[off] = (int32_t)(s0 + i); }
                    ++off;
                }
            }
            base += tot;
        }
    }
    return base;
}

// Float of an order-preserving key (the inverse of float_key on non-negative
// zero): x >= key_float(t) exactly when float_key(x) >= t, for every non-NaN x.
__device__ __forceinline__ float key_float(uint32_t key)
{
    return __uint_as_float((key & 0x80000000u) ? (key & 0x7fffffffu) : ~key);
}


// Candidates x >= tau_f of the row, in ascending position order, into
// sm.ckey / sm.cpos[0, count).  Each warp scans its own contiguous chunk of
// the row (two steps of 512 scores in flight, warp-level ordered
// compaction, no block barrier) into its own WCAP slots; one barrier, then
// the warps' lists are packed in warp order.  The scan is issue-bound, so it
// keeps per-score work minimal: full steps skip the bounds test, positions
// are 32-bit (rows are shorter than 2^31), and the slots hold the raw score
// bits, turned into keys by the pack pass, which touches every candidate
// anyway.  Returns the count, or 0xffffffff if a warp's chunk held more than
// WCAP candidates (the caller falls back).
// Raw scores of positions [s, s + 16) of a row (0 past n): four 16-byte loads.
__device__ __forceinline__ void load_raw16(const float *row, int n, int s, bool vec, float (&v)[16])
{
    if (vec && s + 16 <= n) {
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const float4 a = __ldg(reinterpret_cast<const float4 *>(row + s + 4 * j));
            v[4 * j] = a.x; v[4 * j + 1] = a.y; v[4 * j + 2] = a.z; v[4 * j + 3] = a.w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = s + i < n ? row[s + i] : 0.f;
    }
}

template <class C>
__device__ uint32_t collect_above_warp(TopkSmem<C> &sm, const float *row, int64_t n_, bool vec, float tau_f)
{
    // Steps of 512 scores per warp (16 per lane), two in flight: the per-step
    // cost (ordered prefix over the lanes, candidate writes) is paid once per
    // 2 KB, which measured markedly faster than 1 KB steps four deep.
    constexpr int D = 2, IT = 16, SW = 32 * IT;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n = (int)n_;
    const int per = ((n + C::WARPS - 1) / C::WARPS + SW - 1) / SW * SW;
    const int w0 = warp * per, w1 = min(n, w0 + per);
    uint32_t *wk = sm.ckey + warp * C::WCAP;
    int32_t *wp = sm.cpos + warp * C::WCAP;
    uint32_t cnt = 0;                                      // warp-uniform
    float ring[D][IT];
#pragma unroll
    for (int q = 0; q < D; ++q)
        if (w0 + q * SW < w1) load_raw16(row, w1, w0 + q * SW + lane * IT, vec, ring[q]);
    for (int c0 = w0; c0 < w1; c0 += D * SW) {
#pragma unroll
        for (int q = 0; q < D; ++q) {
            const int cq = c0 + q * SW;
            if (cq >= w1) break;                           // warp-uniform
            const int s0 = cq + lane * IT;
            float v[IT];
#pragma unroll
            for (int i = 0; i < IT; ++i) v[i] = ring[q][i];
            if (cq + D * SW < w1) load_raw16(row, w1, s0 + D * SW, vec, ring[q]);
            uint32_t flags = 0;
            if (cq + SW <= w1) {                           // warp-uniform: a full step
#pragma unroll
                for (int i = 0; i < IT; ++i) flags |= (uint32_t)(v[i] >= tau_f) << i;
            } else {
#pragma unroll
                for (int i = 0; i < IT; ++i) flags |= (uint32_t)(s0 + i < w1 && v[i] >= tau_f) << i;
            }
            const uint32_t c = (uint32_t)__popc(flags);
            uint32_t x = c;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
                if (lane >= o) x += y;
            }
            uint32_t off = cnt + x - c;
            while (flags) {
                const int i = __ffs(flags) - 1;
                flags &= flags - 1;
                if (off < C::WCAP) { wk[off] = __float_as_uint(v[i]); wp[off] = s0 + i; }
                ++off;
            }
            cnt += __shfl_sync(0xffffffffu, x, 31);
        }
    }
    if (lane == 0) sm.wcnt[warp] = cnt;
    __syncthreads();
    if (warp == 0) {                                       // exclusive prefix of the warps' counts
        const uint32_t c = lane < C::WARPS ? sm.wcnt[lane] : 0u;
        uint32_t x = c;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
            if (lane >= o) x += y;
        }
        const bool over = __any_sync(0xffffffffu, c > C::WCAP);
        if (lane <= C::WARPS) sm.wbefore[lane] = over ? 0xffffffffu : x - c;
    }
    __syncthreads();
    const uint32_t total = sm.wbefore[C::WARPS];
    if (total == 0xffffffffu) return total;                // a warp overflowed (block-uniform)
    // Pack in rounds of NT * 4 entries in increasing order: an entry only moves
    // down, so a round's targets never hold a later round's sources; each round
    // reads all its sources before it writes.  Raw score bits become keys here.
    for (uint32_t r0 = 0; r0 < total; r0 += C::NT * 4) {
        uint32_t kk[4];
        int32_t pp[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t i = r0 + tid + q * C::NT;
            if (i < total) {
                int w = 0;                                 // last warp with wbefore[w] <= i
#pragma unroll
                for (int step = C::WARPS / 2; step > 0; step >>= 1)
                    if (sm.wbefore[w + step] <= i) w += step;
                const uint32_t src = w * C::WCAP + (i - sm.wbefore[w]);
                kk[q] = float_key(__uint_as_float(sm.ckey[src]));
                pp[q] = sm.cpos[src];
            }
        }
        __syncthreads();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const uint32_t i = r0 + tid + q * C::NT;
            if (i < total) { sm.ckey[i] = kk[q]; sm.cpos[i] = pp[q]; }
        }
        __syncthreads();
    }
    return total;
}

// Radix select run over the whole row in global memory (candidates did not fit).
template <class C>
__device__ __noinline__ void select_global(TopkSmem<C> &sm, const float *row, int64_t n, bool vec, int k, int32_t *out)
{
    const int tid = threadIdx.x;
    auto row_keys = [&](int64_t s, uint32_t (&keys)[TK_ITEMS], uint32_t &valid) {
        load8(row, n, s, vec, keys, valid);
    };
    uint32_t prefix = 0, pmask = 0, remaining = (uint32_t)k;
#pragma unroll 1
    for (int pass = 0; pass < 3; ++pass) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const int nb = pass == 2 ? 1024 : 2048;
        const uint32_t bmask = (uint32_t)nb - 1u;
        for (int i = tid; i < nb; i += C::NT) sm.hist[i] = 0u;
        __syncthreads();
        for (int64_t c0 = 0; c0 < n; c0 += C::STEP) {
            uint32_t keys[TK_ITEMS], valid;
            row_keys(c0 + (int64_t)tid * TK_ITEMS, keys, valid);
#pragma unroll
            for (int i = 0; i < TK_ITEMS; ++i)
                if (((valid >> i) & 1u) && (keys[i] & pmask) == prefix)
                    atomicAdd(&sm.hist[(keys[i] >> shift) & bmask], 1u);
        }
        __syncthreads();
        find_bin(sm, nb, remaining);
        remaining -= sm.sh_above;
        prefix |= sm.sh_bin << shift;
        pmask |= bmask << shift;
        __syncthreads();
    }
    emit_selected(sm, n, prefix, remaining, k, out, row_keys, [&](int64_t i) { return (int32_t)i; });
}

// Warp-aggregated histogram of the top 11 bits of keys[valid].
__device__ __forceinline__ void hist_top11(uint32_t *hist, const uint32_t (&keys)[TK_ITEMS], uint32_t valid)
{
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int i = 0; i < TK_ITEMS; ++i) {
        const bool v = (valid >> i) & 1u;
        const unsigned act = __ballot_sync(0xffffffffu, v);
        if (v) {
            const uint32_t bin = keys[i] >> 21;
            const unsigned same = __match_any_sync(act, bin);
            if (lane == __ffs(same) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(same));
        }
    }
}

// Threshold guess for a long row: the key of rank ~1.5 k (scaled to the
// sample, at least 8) among NSAMP samples spread evenly over the row, resolved
// by one radix pass (a threshold at or below it).  Every thread calls it;
// every CTA working on the same row computes the same value.  With RUNS the
// samples are runs of 8 consecutive positions starting at multiples of 8
// (n > CAP >= NSAMP, so the runs do not overlap and stay inside the row).
template <class C>
__device__ uint32_t sampled_threshold(TopkSmem<C> &sm, const float *row, int64_t n, int k, bool vec)
{
    const int tid = threadIdx.x;
    uint32_t *smp = sm.sample();
    if constexpr (C::RUNS) {
        constexpr int NRUN = C::NSAMP / 8, RPT = NRUN / C::NT;
        float sv[RPT][TK_ITEMS];                          // all loads issued before any is used
#pragma unroll
        for (int q = 0; q < RPT; ++q) {
            const int64_t j = tid + q * C::NT;
            load_raw8(row, n, (j * n / NRUN) & ~(int64_t)7, vec, sv[q]);
        }
#pragma unroll
        for (int q = 0; q < RPT; ++q)
#pragma unroll
            for (int i = 0; i < TK_ITEMS; ++i) smp[(tid + q * C::NT) * TK_ITEMS + i] = float_key(sv[q][i]);
    } else {
        float sv[C::NSAMP / C::NT];
#pragma unroll
        for (int q = 0; q < C::NSAMP / C::NT; ++q)
            sv[q] = __ldg(row + (int64_t)(tid + q * C::NT) * n / C::NSAMP);
#pragma unroll
        for (int q = 0; q < C::NSAMP / C::NT; ++q) smp[tid + q * C::NT] = float_key(sv[q]);
    }
    __syncthreads();
    // lam = k * NSAMP / n samples are expected above the k-th largest key, about
    // Poisson-distributed; the guess falls short of k when lam's count reaches the
    // chosen rank.  1.5 lam leaves a wide margin for large lam, but for few samples
    // (short shards of long rows, small k: lam = 8 fails about one row in ten at
    // rank 12) the rank needs lam + 4 sqrt(lam) + 2 (a miss rate near 1e-4 at lam
    // = 8), and at least 8.
    const double lam = (double)k * C::NSAMP / (double)n;
    const double want = fmax(1.5 * lam, lam + 4.0 * sqrt(lam) + 2.0);
    const uint32_t rank = (uint32_t)min((double)C::NSAMP, max(8.0, ceil(want)));
    uint32_t tau, unused;
    radix_select_smem(sm, smp, C::NSAMP, rank, &tau, &unused, 1, false);
    return tau;
}

// Exact top-k of a row without a threshold guess: a histogram of the top 11
// key bits fixes the bin of the k-th largest key; the keys in or above it go
// on chip (or, if too many, a radix select runs over the row in global memory).
template <class C>
__device__ __noinline__ void topk_row_histogram(TopkSmem<C> &sm, const float *row, int64_t n, bool vec, int k,
                                                int32_t *out)
{
    const int tid = threadIdx.x;
    for (int i = tid; i < 2048; i += C::NT) sm.hist[i] = 0u;
    __syncthreads();
    for (int64_t c0 = 0; c0 < n; c0 += C::STEP) {
        uint32_t keys[TK_ITEMS], valid;
        load8(row, n, c0 + (int64_t)tid * TK_ITEMS, vec, keys, valid);
        hist_top11(sm.hist, keys, valid);
    }
    __syncthreads();
    find_bin(sm, 2048, (uint32_t)k);
    const uint32_t b1 = sm.sh_bin;
    const uint32_t remaining = (uint32_t)k - sm.sh_above;
    const uint32_t ncand = collect_candidates(sm, row, n, vec, [b1](uint32_t key) { return (key >> 21) >= b1; });
    if (ncand <= C::CAP) select_on_chip(sm, ncand, b1, remaining, k, out);
    else select_global(sm, row, n, vec, k, out);
}

// Row of n_all causal positions with a window of W: positions [0, n) compete
// (n = n_all - W, or 0), [n, n_all) are always taken.  When n <= k the whole
// row is selected, so out[i] = i for i < n_all, then -1 up to k + W.
// Otherwise the top-k part fills out[0, k) and the window out[k, k + W).
template <class C>
__device__ __forceinline__ void emit_window(int32_t *out, int k, int window, int64_t n)
{
    for (int i = threadIdx.x; i < window; i += C::NT) out[k + i] = (int32_t)(n + i);
}

template <class C>
__device__ __forceinline__ bool emit_whole_row(int32_t *out, int k, int window, int64_t n, int64_t n_all)
{
    if (n > k) return false;
    for (int i = threadIdx.x; i < k + window; i += C::NT) out[i] = i < n_all ? i : -1;
    return true;
}

// The exact top-k of one row of n_all causal positions (the last `window`
// of them always selected) into out[k + window].
__device__ __forceinline__ void topk_one_row(TopkSmem<RowsCfg> &sm, const float *row, int64_t n_all, int k,
                                             int window, int32_t *out, bool vec)
{
    using C = RowsCfg;
    const int tid = threadIdx.x;
    const int64_t n = n_all > window ? n_all - window : 0;     // positions before the window
    if (emit_whole_row<C>(out, k, window, n, n_all)) return;
    emit_window<C>(out, k, window, n);
    if (tid == 0) { sm.sh_count = 0; sm.sh_overflow = 0; }

    // ---- short rows: every key is a candidate ----
    if (n <= C::CAP) {
        const uint32_t c = collect_candidates(sm, row, n, vec, [](uint32_t) { return true; });
        select_candidates(sm, c, k, out);
        return;
    }

    // ---- guess a threshold from evenly spaced samples: about 1.5 k keys of the
    // row should lie at or above it; then one ordered pass collects them ----
    {
        const uint32_t tau = sampled_threshold(sm, row, n, k, vec);
        const uint32_t c = collect_above_warp(sm, row, n, vec, key_float(tau));
        if (c >= (uint32_t)k && c <= C::CAP) {        // the selection lies among the candidates
            select_candidates(sm, c, k, out);
            return;
        }
    }
    // ---- fallback: the exact histogram path ----
    topk_row_histogram(sm, row, n, vec, k, out);
}

__global__ void __launch_bounds__(RowsCfg::NT, 2)
topk_rows_kernel(const float *__restrict__ scores, int64_t ld, int64_t row_begin,
                 const int32_t *__restrict__ lens, int64_t max_len, int k, int window,
                 int32_t *__restrict__ idx, WsHeader *hdr, int vec_ok)
{
    using C = RowsCfg;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TopkSmem<C> &sm = *reinterpret_cast<TopkSmem<C> *>(smem_raw);

    const int64_t r = blockIdx.x;
    const int tid = threadIdx.x;
    const float *row = scores + r * ld;
    int32_t *out = idx + r * (int64_t)(k + window);
    int64_t n_all;
    if (lens) {
        n_all = lens[r];
        if (n_all < 1 || n_all > max_len) {
            if (tid == 0) record_error(hdr, DSA_ERR_INVALID_ARG, (unsigned)r);
            for (int i = tid; i < k + window; i += C::NT) out[i] = -1;
            return;
        }
    } else {
        n_all = row_begin + r + 1;
    }
    const int64_t n = n_all > window ? n_all - window : 0;     // positions before the window
    if (emit_whole_row<C>(out, k, window, n, n_all)) return;
    emit_window<C>(out, k, window, n);
    const bool vec = vec_ok != 0;
    if (tid == 0) { sm.sh_count = 0; sm.sh_overflow = 0; }

    // ---- short rows: every key is a candidate ----
    if (n <= C::CAP) {
        const uint32_t c = collect_candidates(sm, row, n, vec, [](uint32_t) { return true; });
        select_candidates(sm, c, k, out);
        return;
    }

    // ---- guess a threshold from evenly spaced samples: about 1.5 k keys of the
    // row should lie at or above it; then one ordered pass collects them ----
    {
        const uint32_t tau = sampled_threshold(sm, row, n, k, vec);
        const uint32_t c = collect_above_warp(sm, row, n, vec, key_float(tau));
        if (c >= (uint32_t)k && c <= C::CAP) {        // the selection lies among the candidates
            select_candidates(sm, c, k, out);
            return;
        }
    }
    // ---- fallback: the exact histogram path ----
    topk_row_histogram(sm, row, n, vec, k, out);
}

// The rows listed in list[0, *count) (pass-relative, position row_begin + r),
// shared out over a persistent grid: the prefill's repair of rows whose fused
// selection failed, which is usually an empty list.
__global__ void __launch_bounds__(RowsCfg::NT, 2)
topk_rows_list_kernel(const float *__restrict__ scores, int64_t ld, int64_t row_begin, int k, int window,
                      int32_t *__restrict__ idx, int vec_ok, const uint32_t *__restrict__ list,
                      const uint32_t *__restrict__ count)
{
    using C = RowsCfg;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TopkSmem<C> &sm = *reinterpret_cast<TopkSmem<C> *>(smem_raw);
    const uint32_t n = *count;
    for (uint32_t i = blockIdx.x; i < n; i += gridDim.x) {
        __syncthreads();                              // the previous row is done with shared memory
        const int64_t r = list[i];
        topk_one_row(sm, scores + r * ld, row_begin + r + 1, k, window, idx + r * (int64_t)(k + window),
                     vec_ok != 0);
    }
}


// ---------------------------------------------------------------- long rows, split over CTAs
// For few long rows (decode): every CTA of a row computes the same sampled
// threshold, collects the candidates of its chunk of the row into a fixed
// slot in global memory; one CTA per row then joins the slots in chunk order
// (so in position order) and finishes the exact select on chip.  Rows whose
// candidates do not fit (or fall short of k) take the exact histogram path.
// Workspace per row: cnt[chunks], then per chunk a slot of TS_SLOT
// (key, position) candidates.

constexpr int TS_CHUNK = 16384;            // positions per CTA
constexpr int TS_SLOT = 2048;              // candidate slot per chunk (more: the row falls back)

struct SplitWs {
    uint32_t *cnt;       // [rows][chunks]: candidates of the chunk, 0xffffffff: a warp overflowed
    uint32_t *ckey;      // [rows][chunks][TS_SLOT]
    int32_t *cpos;       // [rows][chunks][TS_SLOT]
    int chunks;
};

__device__ __forceinline__ int64_t split_len(const int32_t *lens, int64_t max_len, int64_t r)
{
    int64_t n = lens[r];
    return (n < 1 || n > max_len) ? -1 : n;
}

// Positions of a row of n_all (>= 0) that compete for the k slots.
__device__ __forceinline__ int64_t before_window(int64_t n_all, int window)
{
    return n_all > window ? n_all - window : 0;
}

__global__ void __launch_bounds__(SplitCfg::NT, 2)
topk_split_collect_kernel(const float *__restrict__ scores, int64_t ld, const int32_t *__restrict__ lens,
                          int64_t max_len, int k, int window, SplitWs ws, int vec_ok)
{
    using C = SplitCfg;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TopkSmem<C> &sm = *reinterpret_cast<TopkSmem<C> *>(smem_raw);
    grid_dep_wait();                                 // the scores of the kernel before
    grid_dep_trigger();
    const int64_t r = blockIdx.y;
    const int64_t n_all = split_len(lens, max_len, r);
    const int64_t n = n_all < 0 ? -1 : before_window(n_all, window);
    const int64_t c0 = (int64_t)blockIdx.x * TS_CHUNK;
    if (n <= C::CAP || c0 >= n) return;              // short or invalid rows: the final kernel alone
    const int64_t c1 = min(n, c0 + TS_CHUNK);
    const float *row = scores + r * ld;
    const uint32_t tau = sampled_threshold(sm, row, n, k, vec_ok != 0);
    const uint32_t c = collect_above_warp(sm, row + c0, c1 - c0, vec_ok != 0, key_float(tau));
    const int64_t slot = (r * ws.chunks + blockIdx.x) * (int64_t)TS_SLOT;
    if (c != 0xffffffffu)
        for (uint32_t i = threadIdx.x; i < min(c, (uint32_t)TS_SLOT); i += C::NT) {
            ws.ckey[slot + i] = sm.ckey[i];
            ws.cpos[slot + i] = (int32_t)(sm.cpos[i] + c0);
        }
    if (threadIdx.x == 0) ws.cnt[r * ws.chunks + blockIdx.x] = c;
}

__global__ void __launch_bounds__(SplitCfg::NT)
topk_split_final_kernel(const float *__restrict__ scores, int64_t ld, const int32_t *__restrict__ lens,
                        int64_t max_len, int k, int window, SplitWs ws, int32_t *__restrict__ idx,
                        WsHeader *hdr, int vec_ok)
{
    using C = SplitCfg;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TopkSmem<C> &sm = *reinterpret_cast<TopkSmem<C> *>(smem_raw);
    grid_dep_wait();                                 // the collect kernel's slots
    grid_dep_trigger();
    const int64_t r = blockIdx.x;
    const int tid = threadIdx.x;
    int32_t *out = idx + r * (int64_t)(k + window);
    const int64_t n_all = split_len(lens, max_len, r);
    if (n_all < 0) {
        if (tid == 0) record_error(hdr, DSA_ERR_INVALID_ARG, (unsigned)r);
        for (int i = tid; i < k + window; i += C::NT) out[i] = -1;
        return;
    }
    const int64_t n = before_window(n_all, window);
    if (emit_whole_row<C>(out, k, window, n, n_all)) return;
    emit_window<C>(out, k, window, n);
    const float *row = scores + r * ld;
    const bool vec = vec_ok != 0;
    if (n <= C::CAP) {                               // short rows: every key is a candidate
        const uint32_t c = collect_candidates(sm, row, n, vec, [](uint32_t) { return true; });
        select_candidates(sm, c, k, out);
        return;
    }
    const int nch = (int)((n + TS_CHUNK - 1) / TS_CHUNK);
    bool use = nch <= C::NSAMP;                     // counts and offsets fit the scratch arrays
    if (use) {
        // chunk counts (sm.sample) and their exclusive prefix (sm.hist), in parallel
        const int cpt = (nch + C::NT - 1) / C::NT;
        uint32_t msum = 0;
        bool fit = true;
        for (int u = 0; u < cpt; ++u) {
            const int c = tid * cpt + u;
            if (c < nch) {
                const uint32_t m = ws.cnt[r * ws.chunks + c];
                fit = fit && m <= TS_SLOT;
                sm.sample()[c] = m <= TS_SLOT ? m : 0u;
                msum += m <= TS_SLOT ? m : 0u;
            }
        }
        use = __syncthreads_and(fit) != 0;
        uint32_t total;
        uint32_t run = block_excl_scan<C>(msum, sm.warp_buf, &total);
        for (int u = 0; u < cpt; ++u) {
            const int c = tid * cpt + u;
            if (c < nch) { sm.hist[c] = run; run += sm.sample()[c]; }
        }
        __syncthreads();
        use = use && total >= (uint32_t)k && total <= C::CAP;
        if (use) {
            // Every thread copies joined entries tid, tid + 512, ... with four
            // entries' loads in flight: entry i comes from the last chunk c whose
            // offset hist[c] <= i (that chunk is never empty), at i - hist[c].
            for (uint32_t base = 0; base < total; base += C::NT * 4) {
                uint32_t kk[4];
                int32_t pp[4];
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t i = base + (uint32_t)(q * C::NT + tid);
                    if (i < total) {
                        int lo = 0, hi = nch - 1;
                        while (lo < hi) {
                            const int mid = (lo + hi + 1) >> 1;
                            if (sm.hist[mid] <= i) lo = mid; else hi = mid - 1;
                        }
                        const int64_t src = (r * ws.chunks + lo) * (int64_t)TS_SLOT + (i - sm.hist[lo]);
                        kk[q] = ws.ckey[src];
                        pp[q] = ws.cpos[src];
                    }
                }
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    const uint32_t i = base + (uint32_t)(q * C::NT + tid);
                    if (i < total) { sm.ckey[i] = kk[q]; sm.cpos[i] = pp[q]; }
                }
            }
            __syncthreads();
            select_candidates(sm, total, k, out);
        }
    }
    if (!use) {
        topk_row_histogram(sm, row, n, vec, k, out);
    }
}

// ---------------------------------------------------------------- fused prefill selection
// The prefill indexer's select epilogue appends, for each query row, every
// competing position whose score is at or above the row's threshold tau, as
// (score bits, position), in no particular order.  tau comes from the scores
// of a sample of the keys (one pseudo-random position per S): with m samples
// before the row's window and n competing positions, lam = k m / n samples
// are expected above the k-th largest score, and tau is the sample of rank
// lam + 6 sqrt(lam) + 2, which leaves about that many times S candidates
// and falls short of k only with probability near 2e-8 per row.  A row
// whose count lies outside [k, cap] is flagged; the caller then recomputes
// its scores and runs the stand-alone select on it, so every row is exact.

// Rank of tau among the m samples of a row of n competing positions.
__host__ __device__ inline uint32_t tau_rank(int k, int64_t m, int64_t n)
{
    const double lam = (double)k * (double)m / (double)n;
    double r = ceil(lam + 6.0 * sqrt(lam) + 2.0);
    if (r > (double)m) r = (double)m;
    return r < 1.0 ? 1u : (uint32_t)r;
}

// One warp per row: tau (+inf when the whole row is selected without scores,
// -inf when every competing position fits the candidate list), and the
// row's candidate counter and repair state cleared for the select pass.
// The rank-th largest sample key: each lane keeps its own J = ceil(rank/32)
// largest keys; the smallest of the lanes' J-th largest, L, has at least
// 32 J >= rank keys at or above it, so only those are compacted (usually a
// tenth of the samples) and searched by bisection over the key range [L, max].
// Rows with more samples than the registers hold bisect over all of them.
constexpr int TAU_WARPS = 8;
constexpr int TAU_REG = 64;                      // keys per lane held in registers
constexpr int TAU_TOP = 4;                       // per-lane top list: ranks up to 128
constexpr int TAU_LIST = 1024;                   // compacted keys per warp

__device__ __forceinline__ uint32_t warp_count_ge(const uint32_t *list, uint32_t n, uint32_t mid)
{
    uint32_t c = 0;
    for (uint32_t j = threadIdx.x & 31; j < n; j += 32) c += list[j] >= mid;
    return __reduce_add_sync(0xffffffffu, c);
}

__global__ void __launch_bounds__(TAU_WARPS * 32)
prefill_tau_kernel(const float *__restrict__ ss, int64_t ld, int64_t row_begin, int64_t rows, int k, int window,
                   int S, int cap, float *__restrict__ tau, uint32_t *__restrict__ cnt,
                   uint32_t *__restrict__ rb_fail, uint32_t *__restrict__ fail_cnt)
{
    __shared__ uint32_t lists[TAU_WARPS][TAU_LIST];
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int64_t r = (int64_t)blockIdx.x * TAU_WARPS + wid;
    if (r >= rows) return;
    const int64_t t = row_begin + r;
    const int64_t n = t + 1 - window > 0 ? t + 1 - window : 0;
    float tv;
    if (n <= k) {
        tv = INFINITY;
    } else if (n <= cap) {
        tv = -INFINITY;
    } else {
        const int64_t m = sample_count(n, S);
        const uint32_t rank = tau_rank(k, m, n);
        const float *row = ss + r * ld;
        uint32_t lo = 0u, hi = 0xffffffffu;              // count(key >= lo) >= rank throughout
        if (m <= 32 * TAU_REG && rank <= 32 * TAU_TOP) {
            uint32_t kv[TAU_REG];
#pragma unroll
            for (int i = 0; i < TAU_REG; ++i) {
                const int64_t j = lane + 32 * i;
                kv[i] = j < m ? float_key(row[j]) : 0u;      // key 0 is no score's key
            }
            // this lane's TAU_TOP largest keys, descending
            uint32_t top[TAU_TOP];
#pragma unroll
            for (int q = 0; q < TAU_TOP; ++q) top[q] = 0u;
            uint32_t mx = 0u;
#pragma unroll
            for (int i = 0; i < TAU_REG; ++i) {
                uint32_t x = kv[i];
                mx = max(mx, x);
#pragma unroll
                for (int q = 0; q < TAU_TOP; ++q) {
                    const uint32_t hiq = max(top[q], x);
                    x = min(top[q], x);
                    top[q] = hiq;
                }
            }
            const int J = (int)((rank + 31) / 32);
            uint32_t lj = top[0];
#pragma unroll
            for (int q = 1; q < TAU_TOP; ++q)
                if (q == J - 1) lj = top[q];
            const uint32_t L = __reduce_min_sync(0xffffffffu, lj);
            const uint32_t M = __reduce_max_sync(0xffffffffu, mx);
            // compact the keys >= L (a key of 0 is padding and never counted)
            uint32_t *list = lists[wid];
            uint32_t base = 0;
            const uint32_t lt = (1u << lane) - 1u;
            bool fits = true;
#pragma unroll
            for (int i = 0; i < TAU_REG; ++i) {
                const bool p = kv[i] >= L && kv[i] != 0u;
                const uint32_t bal = __ballot_sync(0xffffffffu, p);
                if (p && base + __popc(bal & lt) < (uint32_t)TAU_LIST) list[base + __popc(bal & lt)] = kv[i];
                base += __popc(bal);
            }
            fits = base <= (uint32_t)TAU_LIST;
            __syncwarp();
            lo = L;
            hi = M;
            if (fits) {
                while (lo < hi) {
                    const uint32_t mid = lo + ((hi - lo) >> 1) + 1u;
                    if (warp_count_ge(list, base, mid) >= rank) lo = mid; else hi = mid - 1u;
                }
            } else {
                while (lo < hi) {
                    const uint32_t mid = lo + ((hi - lo) >> 1) + 1u;
                    uint32_t c = 0;
#pragma unroll
                    for (int i = 0; i < TAU_REG; ++i) c += kv[i] >= mid;
                    c = __reduce_add_sync(0xffffffffu, c);
                    if (c >= rank) lo = mid; else hi = mid - 1u;
                }
            }
        } else {
            while (lo < hi) {
                const uint32_t mid = lo + ((hi - lo) >> 1) + 1u;
                uint32_t c = 0;
                for (int64_t j = lane; j < m; j += 32) c += float_key(row[j]) >= mid;
                c = __reduce_add_sync(0xffffffffu, c);
                if (c >= rank) lo = mid; else hi = mid - 1u;
            }
        }
        tv = key_float(lo);
    }
    if (lane == 0) {
        tau[r] = tv;
        cnt[r * kCandCntStride] = 0u;
        if ((r & 127) == 0) rb_fail[r >> 7] = 0u;
        if (r == 0) *fail_cnt = 0u;
    }
}

// One CTA per row: the exact top-k of the row's candidates, emitted in
// ascending position order (the window, if any, after them).  The k-th
// largest key thr and the number `need` of keys equal to thr that rank within
// the top k come from the radix select over the keys in shared memory.  When
// more keys than `need` equal thr, the lowest positions win: a bisection over
// positions finds the cut.  The emit then marks the selected positions in a
// bitmap of 65536 positions at a time and writes them in order through one
// block-wide prefix count per window.  Positions are read again from the
// candidate list (L2) where needed rather than held in registers: the kernel
// is bound by its barriers and latencies, so the registers buy more resident
// rows (five CTAs per SM) instead.
constexpr int FIN_NT = 256;
using FinCfg = TopkCfg<FIN_NT, 256, 8, false>;
constexpr int FIN_WIN_WORDS = 2048;                  // 65536 positions per emit window (the histogram's words)

__host__ __device__ inline size_t finish_smem_bytes(int cap)
{
    return align_up(sizeof(TopkSmem<FinCfg>), 16) + sizeof(uint32_t) * (size_t)cap;
}

template <int PER>                                   // candidates per thread: cap <= PER * FIN_NT
__global__ void __launch_bounds__(FIN_NT, PER <= 32 ? 5 : 4)
prefill_finish_kernel(const uint2 *__restrict__ cand, int cap, const uint32_t *__restrict__ cnt, int64_t row_begin,
                      int k, int window, int32_t *__restrict__ idx, uint32_t *__restrict__ rb_fail,
                      uint32_t *__restrict__ fail_cnt, uint32_t *__restrict__ fail_list)
{
    using C = FinCfg;
    extern __shared__ __align__(16) uint8_t smem_raw[];
    TopkSmem<C> &sm = *reinterpret_cast<TopkSmem<C> *>(smem_raw);
    uint32_t *keys = reinterpret_cast<uint32_t *>(smem_raw + align_up(sizeof(TopkSmem<C>), 16));
    uint32_t *bm = sm.hist;                          // free once the select is done
    static_assert(sizeof(sm.hist) / sizeof(uint32_t) == FIN_WIN_WORDS, "bitmap window");

    const int tid = threadIdx.x;
    const int64_t r = blockIdx.x;
    const int64_t n_all = row_begin + r + 1;
    const int64_t n = before_window(n_all, window);
    int32_t *out = idx + r * (int64_t)(k + window);
    if (emit_whole_row<C>(out, k, window, n, n_all)) return;
    emit_window<C>(out, k, window, n);
    const uint32_t c = cnt[r * kCandCntStride];
    if (c < (uint32_t)k || c > (uint32_t)cap) {
        if (tid == 0) {                              // the repair pass takes this row
            fail_list[atomicAdd(fail_cnt, 1u)] = (uint32_t)r;
            atomicOr(rb_fail + (r >> 7), 1u);
        }
        return;
    }
    const uint2 *cr = cand + r * (int64_t)cap;
#pragma unroll 8
    for (int j = 0; j < PER; ++j) {
        const uint32_t i = tid + j * FIN_NT;
        if (i < c) keys[i] = float_key(__uint_as_float(cr[i].x));
    }
    __syncthreads();
    uint32_t thr, need;
    radix_select_smem(sm, keys, c, (uint32_t)k, &thr, &need);
    __syncthreads();

    // ties at thr: the lowest `need` positions among them
    uint32_t ecnt = 0;
#pragma unroll
    for (int j = 0; j < PER; ++j) {
        const uint32_t i = tid + j * FIN_NT;
        ecnt += i < c && keys[i] == thr;
    }
    uint32_t etot;
    block_excl_scan<C>(ecnt, sm.warp_buf, &etot);
    uint32_t pcut = 0xffffffffu;                     // every key equal to thr is taken
    if (etot > need) {                               // block-uniform
        uint32_t lo = 0, hi = (uint32_t)(n - 1);     // smallest p with count(eq, pos <= p) >= need
        while (lo < hi) {
            const uint32_t mid = lo + (hi - lo) / 2;
            uint32_t e = 0;
#pragma unroll 4
            for (int j = 0; j < PER; ++j) {
                const uint32_t i = tid + j * FIN_NT;
                e += i < c && keys[i] == thr && __ldg(&cr[i].y) <= mid;
            }
            uint32_t tot;
            block_excl_scan<C>(e, sm.warp_buf, &tot);
            if (tot >= need) hi = mid; else lo = mid + 1;
        }
        pcut = lo;
    }

    uint32_t out_base = 0;                           // block-uniform
    for (int64_t w0 = 0; w0 < n; w0 += 32 * FIN_WIN_WORDS) {
        for (int i = tid; i < FIN_WIN_WORDS; i += FIN_NT) bm[i] = 0u;
        __syncthreads();
#pragma unroll 4
        for (int j = 0; j < PER; ++j) {
            const uint32_t i = tid + j * FIN_NT;
            if (i < c) {
                const uint32_t key = keys[i];
                if (key >= thr) {
                    const uint32_t p = __ldg(&cr[i].y);
                    const int64_t off = (int64_t)p - w0;
                    if ((key > thr || p <= pcut) && off >= 0 && off < 32 * FIN_WIN_WORDS)
                        atomicOr(bm + (off >> 5), 1u << (off & 31));
                }
            }
        }
        __syncthreads();
        constexpr int WPT = FIN_WIN_WORDS / FIN_NT;  // words per thread, consecutive
        uint32_t g[WPT], scnt = 0;
#pragma unroll
        for (int q = 0; q < WPT; ++q) {
            g[q] = bm[tid * WPT + q];
            scnt += (uint32_t)__popc(g[q]);
        }
        uint32_t stot;
        uint32_t o = out_base + block_excl_scan<C>(scnt, sm.warp_buf, &stot);
#pragma unroll
        for (int q = 0; q < WPT; ++q) {
            uint32_t x = g[q];
            while (x) {
                const int b = __ffs(x) - 1;
                x &= x - 1;
                if (o < (uint32_t)k) out[o] = (int32_t)(w0 + (int64_t)(tid * WPT + q) * 32 + b);
                ++o;
            }
        }
        out_base += stot;
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_topk_rows(const float *scores, int64_t ld, int64_t row_begin,
                             const int32_t *lens, int64_t max_len, int64_t row_count, int k,
                             int32_t *idx, WsHeader *hdr, cudaStream_t st, int window)
{
    if (row_count <= 0) return cudaSuccess;
    const size_t smem = sizeof(TopkSmem<RowsCfg>);
    cudaError_t e = cudaFuncSetAttribute(topk_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    const int vec_ok = (ld % 4 == 0) && ((reinterpret_cast<uintptr_t>(scores) & 15u) == 0);
    topk_rows_kernel<<<(unsigned)row_count, RowsCfg::NT, smem, st>>>(scores, ld, row_begin, lens,
                                                                     max_len, k, window, idx, hdr, vec_ok);
    return cudaGetLastError();
}

size_t topk_split_ws_bytes(int64_t rows, int64_t max_len)
{
    const int64_t chunks = ceil_div(max_len, TS_CHUNK);
    return align_up(sizeof(uint32_t) * (size_t)rows * chunks, 256) +
           2 * align_up(sizeof(uint32_t) * (size_t)rows * chunks * TS_SLOT, 256);
}

cudaError_t launch_topk_split(const float *scores, int64_t ld, const int32_t *lens, int64_t max_len,
                              int64_t rows, int k, int32_t *idx, void *ws_base, WsHeader *hdr,
                              cudaStream_t st, int window)
{
    if (rows <= 0) return cudaSuccess;
    const int64_t chunks = ceil_div(max_len, TS_CHUNK);
    uint8_t *p = static_cast<uint8_t *>(ws_base);
    SplitWs ws;
    ws.chunks = (int)chunks;
    ws.cnt = reinterpret_cast<uint32_t *>(p);
    p += align_up(sizeof(uint32_t) * (size_t)rows * chunks, 256);
    ws.ckey = reinterpret_cast<uint32_t *>(p);
    p += align_up(sizeof(uint32_t) * (size_t)rows * chunks * TS_SLOT, 256);
    ws.cpos = reinterpret_cast<int32_t *>(p);
    const int vec_ok = (ld % 4 == 0) && ((reinterpret_cast<uintptr_t>(scores) & 15u) == 0);
    const size_t smem = sizeof(TopkSmem<SplitCfg>);
    cudaError_t e = cudaFuncSetAttribute(topk_split_collect_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(topk_split_final_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((unsigned)chunks, (unsigned)rows);
    e = launch_chained(topk_split_collect_kernel, grid, dim3(SplitCfg::NT), smem, st, scores, ld, lens,
                       max_len, k, window, ws, vec_ok);
    if (e != cudaSuccess) return e;
    e = launch_chained(topk_split_final_kernel, dim3((unsigned)rows), dim3(SplitCfg::NT), smem, st, scores,
                       ld, lens, max_len, k, window, ws, idx, hdr, vec_ok);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}


cudaError_t launch_prefill_tau(const float *ss, int64_t ld, int64_t row_begin, int64_t rows, int k, int window,
                               int S, int cap, float *tau, uint32_t *cnt, uint32_t *rb_fail, uint32_t *fail_cnt,
                               cudaStream_t st)
{
    if (rows <= 0) return cudaSuccess;
    prefill_tau_kernel<<<(unsigned)ceil_div(rows, TAU_WARPS), TAU_WARPS * 32, 0, st>>>(
        ss, ld, row_begin, rows, k, window, S, cap, tau, cnt, rb_fail, fail_cnt);
    return cudaGetLastError();
}

size_t prefill_finish_smem(int cap) { return finish_smem_bytes(cap); }

template <int PER>
static cudaError_t launch_finish_per(const uint2 *cand, int cap, const uint32_t *cnt, int64_t row_begin, int64_t rows,
                                     int k, int window, int32_t *idx, uint32_t *rb_fail, uint32_t *fail_cnt,
                                     uint32_t *fail_list, cudaStream_t st)
{
    const size_t smem = finish_smem_bytes(cap);
    cudaError_t e = cudaFuncSetAttribute(prefill_finish_kernel<PER>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    prefill_finish_kernel<PER><<<(unsigned)rows, FIN_NT, smem, st>>>(cand, cap, cnt, row_begin, k, window, idx,
                                                                     rb_fail, fail_cnt, fail_list);
    return cudaGetLastError();
}

cudaError_t launch_prefill_finish(const uint2 *cand, int cap, const uint32_t *cnt, int64_t row_begin, int64_t rows,
                                  int k, int window, int32_t *idx, uint32_t *rb_fail, uint32_t *fail_cnt,
                                  uint32_t *fail_list, cudaStream_t st)
{
    if (rows <= 0) return cudaSuccess;
    if (cap <= 16 * FIN_NT)
        return launch_finish_per<16>(cand, cap, cnt, row_begin, rows, k, window, idx, rb_fail, fail_cnt, fail_list, st);
    if (cap <= 32 * FIN_NT)
        return launch_finish_per<32>(cand, cap, cnt, row_begin, rows, k, window, idx, rb_fail, fail_cnt, fail_list, st);
    if (cap <= 64 * FIN_NT)
        return launch_finish_per<64>(cand, cap, cnt, row_begin, rows, k, window, idx, rb_fail, fail_cnt, fail_list, st);
    return cudaErrorInvalidValue;
}

cudaError_t launch_topk_rows_list(const float *scores, int64_t ld, int64_t row_begin, int64_t rows, int k,
                                  int32_t *idx, cudaStream_t st, int window, const uint32_t *list,
                                  const uint32_t *count)
{
    if (rows <= 0) return cudaSuccess;
    const size_t smem = sizeof(TopkSmem<RowsCfg>);
    cudaError_t e = cudaFuncSetAttribute(topk_rows_list_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const unsigned grid = (unsigned)std::min<int64_t>(rows, 2 * (int64_t)sms);
    const int vec_ok = (ld % 4 == 0) && ((reinterpret_cast<uintptr_t>(scores) & 15u) == 0);
    topk_rows_list_kernel<<<grid, RowsCfg::NT, smem, st>>>(scores, ld, row_begin, k, window, idx, vec_ok, list,
                                                          count);
    return cudaGetLastError();
}

}  // namespace dsa
