// C entry points: argument validation, workspace carving, stage sequencing.
// Everything numeric happens in the kernels; this file only checks and launches.
#include <atomic>
#include <cmath>
#include <mutex>
#include <vector>

#include "kernels.h"

using namespace dsa;

namespace {

inline bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t as_stream(void *s) { return reinterpret_cast<cudaStream_t>(s); }
inline dsa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

// Row block of the prefill indexer pass: as many rows as the score buffer holds.
constexpr int64_t kPrefillRowsDefault = 8192;
constexpr size_t kPrefillScoreBudget = size_t(4) << 30;

inline int64_t prefill_rows_default(int64_t T)
{
    int64_t r = (int64_t)(kPrefillScoreBudget / (sizeof(float) * (size_t)(T > 0 ? T : 1)));
    r = r < kPrefillRowsDefault ? r : kPrefillRowsDefault;
    r = r / 64 * 64;
    if (r < 64) r = 64;
    int64_t tr = ceil_div(T, 64) * 64;
    return r < tr ? r : tr;
}

inline size_t idx_bytes(int64_t rows, int k) { return align_up(sizeof(int32_t) * (size_t)rows * k, 256); }

// ---- stage timing (dsa_profile_enable / dsa_profile_read)
struct ProfRec {
    int stage;
    cudaEvent_t a, b;
};
struct Profiler {
    std::mutex mu;
    std::atomic<bool> on{false};
    std::vector<ProfRec> recs;
};
Profiler &profiler()
{
    static Profiler p;
    return p;
}
// Records an event pair on `st` around its scope when timing is enabled.
class StageTimer {
public:
    StageTimer(int stage, cudaStream_t st) : stage_(stage), st_(st)
    {
        if (!profiler().on.load(std::memory_order_relaxed)) return;
        if (cudaEventCreate(&a_) != cudaSuccess) { a_ = nullptr; return; }
        if (cudaEventCreate(&b_) != cudaSuccess || cudaEventRecord(a_, st_) != cudaSuccess) {
            cudaEventDestroy(a_);
            if (b_) cudaEventDestroy(b_);
            a_ = b_ = nullptr;
        }
    }
    ~StageTimer()
    {
        if (!a_) return;
        if (cudaEventRecord(b_, st_) != cudaSuccess) {
            cudaEventDestroy(a_);
            cudaEventDestroy(b_);
            return;
        }
        std::lock_guard<std::mutex> g(profiler().mu);
        profiler().recs.push_back({stage_, a_, b_});
    }
    StageTimer(const StageTimer &) = delete;
    StageTimer &operator=(const StageTimer &) = delete;

private:
    int stage_;
    cudaStream_t st_;
    cudaEvent_t a_ = nullptr, b_ = nullptr;
};

// Largest sliding window (positions) the window entry points accept.
constexpr int kMaxWindow = 1 << 24;

// ---- fused prefill selection (the FP8 tcgen05 indexer with its select epilogue)
// A pass of R query rows: sample scores -> per-row tau -> select epilogue
// (candidates at or above tau) -> exact finish; rows whose candidate count
// fell outside [k, cap] are recomputed by the score epilogue (only their row
// blocks) and selected by the stand-alone top-k.  The repair's score rows
// bound R: kRepairBudget bytes of them by default.
constexpr int kSampleStride = 64;               // one sampled key per 64 positions
constexpr int kFusedMaxK = 4096;                // larger k: the stand-alone top-k path
constexpr size_t kRepairBudget = size_t(1) << 30;
// Sample scores of up to kSampleBudget bytes of query rows are computed in one
// launch (several passes' worth), which keeps that small launch's grid full.
constexpr size_t kSampleBudget = size_t(128) << 20;

inline bool fused_ok(dsa_dtype dtype, int H_I, int64_t T, int k)
{
    return dtype == DSA_E4M3 && index_tc_supported(H_I) && T < ((int64_t)1 << 31) && k >= 1 && k <= kFusedMaxK;
}
inline int fused_cap(int k) { return 4 * k > 4096 ? 4 * k : 4096; }

// The fused scratch for passes of R rows, carved after `base` bytes.
struct FusedLayout {
    int S = kSampleStride, cap = 0;
    int64_t T = 0, M = 0, ldM = 0, R = 0, SG = 0;   // SG: rows of sample scores held (a multiple of R)
    size_t ks = 0, sks = 0, fail_cnt = 0, ss = 0, tau = 0, cnt = 0, fail_list = 0, rb_fail = 0, cand = 0,
           scores = 0, end = 0;
    FusedLayout(int64_t T_, int k, int64_t R_, size_t base) : cap(fused_cap(k)), T(T_), R(R_)
    {
        M = sample_count(T, S);
        ldM = (M + 3) / 4 * 4;
        if (ldM < 4) ldM = 4;
        SG = R;
        if (R > 0) {
            const int64_t groups = (int64_t)(kSampleBudget / (sizeof(float) * (size_t)ldM)) / R;
            const int64_t need = ceil_div(T, R);
            SG = R * (groups < 1 ? 1 : (groups < need ? groups : need));
        }
        size_t off = base;
        auto take = [&](size_t bytes) { size_t o = off; off += align_up(bytes > 0 ? bytes : 1, 256); return o; };
        ks = take((size_t)M * 128);
        sks = take(sizeof(float) * (size_t)M);
        fail_cnt = take(sizeof(uint32_t));
        ss = take(sizeof(float) * (size_t)SG * ldM);
        tau = take(sizeof(float) * (size_t)R);
        cnt = take(sizeof(uint32_t) * (size_t)R * kCandCntStride);
        fail_list = take(sizeof(uint32_t) * (size_t)R);
        rb_fail = take(sizeof(uint32_t) * (size_t)ceil_div(R, 128));
        cand = take(sizeof(uint2) * (size_t)R * cap);
        scores = take(sizeof(float) * (size_t)R * T);
        end = off;
    }
};

inline int64_t fused_rows_max(int64_t T) { return ceil_div(T, 128) * 128; }
// Default pass: at most kFusedRowsMax rows (the candidate lists take 32 KB
// a row at k 2048) and kRepairBudget bytes of repair score rows.
constexpr int64_t kFusedRowsMax = 4096;
inline int64_t fused_rows_default(int64_t T)
{
    int64_t r = (int64_t)(kRepairBudget / (sizeof(float) * (size_t)T)) / 128 * 128;
    if (r < 128) r = 128;
    if (r > kFusedRowsMax) r = kFusedRowsMax;
    return r < fused_rows_max(T) ? r : fused_rows_max(T);
}
// The host-memory prefill's pass: twice the repair budget of the default (so, at
// 128K positions, 4096 rows instead of 2048), since its workspace already mirrors
// every input and output; fewer passes mean fewer small sample launches.
inline int64_t fused_rows_host(int64_t T)
{
    int64_t r = (int64_t)(2 * kRepairBudget / (sizeof(float) * (size_t)T)) / 128 * 128;
    if (r < 128) r = 128;
    if (r > kFusedRowsMax) r = kFusedRowsMax;
    return r < fused_rows_max(T) ? r : fused_rows_max(T);
}
// Largest R (a multiple of 128, at most T rounded up) whose layout fits ws_bytes; 0 if none.
inline int64_t fused_rows_fitting(int64_t T, int k, size_t base, size_t ws_bytes)
{
    int64_t lo = 0, hi = fused_rows_max(T) / 128;        // in units of 128 rows
    while (lo < hi) {
        const int64_t mid = (lo + hi + 1) / 2;
        if (FusedLayout(T, k, mid * 128, base).end <= ws_bytes) lo = mid; else hi = mid - 1;
    }
    return lo * 128;
}

// The sampled keys, once per sequence.
cudaError_t fused_gather(const FusedLayout &L, uint8_t *ws, const void *k_idx, const float *k_scale, cudaStream_t st)
{
    return launch_gather_samples((const uint8_t *)k_idx, k_scale, L.M, L.S, ws + L.ks, (float *)(ws + L.sks), st);
}

// Sample scores of query rows [g0, g0 + gn) (gn <= L.SG) into the sample-score
// rows 0.. of the workspace, when any of those rows has more competing
// positions than the candidate list holds (the others never read theirs).
cudaError_t fused_sample(const FusedLayout &L, uint8_t *ws, const void *q_idx, const float *q_scale, const void *w,
                         int64_t T, int H_I, int window, int64_t g0, int64_t gn, WsHeader *hdr, cudaStream_t st,
                         int64_t q_base, int64_t q_rows)
{
    if (g0 + gn - window <= L.cap) return cudaSuccess;
    StageTimer tm(DSA_STAGE_SAMPLE, st);
    IndexTcOpts o;
    o.mode = IT_SAMPLE;
    o.q_base = q_base;
    o.q_rows = q_rows;
    o.nkeys = L.M;
    o.window = window;
    o.sample_stride = L.S;
    return launch_index_tc((const uint8_t *)q_idx, q_scale, ws + L.ks, (const float *)(ws + L.sks),
                           (const uint16_t *)w, T, H_I, g0, gn, (float *)(ws + L.ss), L.ldM, false, hdr, st, &o);
}

// Selection of query rows [r0, r0 + n) (n <= L.R) into idx_rows (row r0 first,
// k + window wide).  q_idx, q_scale and w hold positions [q_base, q_base +
// q_rows) of the sequence; the key side holds positions [0, T).
cudaError_t fused_select_pass(const FusedLayout &L, uint8_t *ws, const void *q_idx, const float *q_scale,
                              const void *k_idx, const float *k_scale, const void *w, int64_t T, int H_I, int k,
                              int window, int64_t r0, int64_t n, int32_t *idx_rows, WsHeader *hdr, cudaStream_t st,
                              int64_t q_base, int64_t q_rows, int64_t ss_row0)
{
    float *ss = (float *)(ws + L.ss), *tau = (float *)(ws + L.tau), *scores = (float *)(ws + L.scores);
    uint32_t *cnt = (uint32_t *)(ws + L.cnt), *fail_list = (uint32_t *)(ws + L.fail_list);
    uint32_t *rb_fail = (uint32_t *)(ws + L.rb_fail), *fail_cnt = (uint32_t *)(ws + L.fail_cnt);
    uint2 *cand = (uint2 *)(ws + L.cand);
    const uint8_t *q8 = (const uint8_t *)q_idx, *k8 = (const uint8_t *)k_idx;
    const uint16_t *wb = (const uint16_t *)w;
    cudaError_t e = cudaSuccess;
    {
        StageTimer tm(DSA_STAGE_TAU, st);
        e = launch_prefill_tau(ss + ss_row0 * L.ldM, L.ldM, r0, n, k, window, L.S, L.cap, tau, cnt, rb_fail,
                               fail_cnt, st);
        if (e != cudaSuccess) return e;
    }
    {
        StageTimer tm(DSA_STAGE_SELECT, st);
        IndexTcOpts o;
        o.mode = IT_SELECT;
        o.q_base = q_base;
        o.q_rows = q_rows;
        o.window = window;
        o.tau = tau;
        o.cand = cand;
        o.cand_cnt = cnt;
        o.cap = L.cap;
        e = launch_index_tc(q8, q_scale, k8, k_scale, wb, T, H_I, r0, n, nullptr, 0, false, hdr, st, &o);
        if (e != cudaSuccess) return e;
    }
    {
        StageTimer tm(DSA_STAGE_FINISH, st);
        e = launch_prefill_finish(cand, L.cap, cnt, r0, n, k, window, idx_rows, rb_fail, fail_cnt, fail_list, st);
        if (e != cudaSuccess) return e;
    }
    // repair: scores of the flagged row blocks (nothing when none), stand-alone select of the flagged rows
    StageTimer tm(DSA_STAGE_REPAIR, st);
    {
        IndexTcOpts o;
        o.mode = IT_SCORES;
        o.q_base = q_base;
        o.q_rows = q_rows;
        o.rb_mask = rb_fail;
        o.any = fail_cnt;
        e = launch_index_tc(q8, q_scale, k8, k_scale, wb, T, H_I, r0, n, scores, T, false, hdr, st, &o);
        if (e != cudaSuccess) return e;
    }
    return launch_topk_rows_list(scores, T, r0, n, k, idx_rows, st, window, fail_list, fail_cnt);
}

dsa_status check_index_args(const void *q_idx, const float *q_scale, const void *k_idx,
                            const float *k_scale, const void *w, int64_t T, int H_I, int d_I,
                            dsa_dtype dtype)
{
    if (!q_idx || !k_idx || !w || T <= 0 || H_I <= 0 || d_I <= 0) return DSA_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(k_idx)) return DSA_ERR_INVALID_ARG;
    if (dtype == DSA_E4M3) {
        if (!q_scale || !k_scale) return DSA_ERR_INVALID_ARG;
        if (d_I != 128 || H_I > 128) return DSA_ERR_UNSUPPORTED;
    } else if (dtype == DSA_F32) {
        if (q_scale || k_scale) return DSA_ERR_INVALID_ARG;
        if (d_I > 256 || H_I > 64) return DSA_ERR_UNSUPPORTED;
    } else {
        return DSA_ERR_UNSUPPORTED;
    }
    return DSA_OK;
}

dsa_status check_attn_args(const void *q, const void *k, const void *v, const int32_t *idx,
                           int64_t T, int H_q, int d, int k_sel, const void *out, dsa_dtype dtype)
{
    if (!q || !k || !v || !idx || !out || T <= 0 || H_q <= 0 || d <= 0 || k_sel <= 0)
        return DSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
    if (dtype == DSA_F32) {
        if (d > 128 || H_q > 32) return DSA_ERR_UNSUPPORTED;
    } else if (dtype == DSA_BF16 || dtype == DSA_E4M3) {
        if (d != 128 && d != 64) return DSA_ERR_UNSUPPORTED;
        if (H_q > 128 && H_q % 128 != 0) return DSA_ERR_UNSUPPORTED;
        if (H_q > 65535 * 128) return DSA_ERR_UNSUPPORTED;
    } else {
        return DSA_ERR_UNSUPPORTED;
    }
    return DSA_OK;
}

cudaError_t run_attn(const void *q, const void *k, const void *v, const int32_t *idx, int64_t T,
                     int H_q, int d, int k_sel, float sm_scale, void *out, float *lse,
                     dsa_dtype dtype, cudaStream_t st)
{
    if (dtype == DSA_F32)
        return launch_sparse_attn_f32((const float *)q, (const float *)k, (const float *)v, idx,
                                      T, H_q, d, k_sel, sm_scale, (float *)out, lse, st);
    if (sparse_attn_tc_supported(H_q, d)) {
        // tcgen05 kernel: the 128 query heads of a token are the MMA's M dimension
        cudaError_t e = launch_sparse_attn_tc((const uint16_t *)q, (const uint16_t *)k,
                                              (const uint16_t *)v, T, T, nullptr, nullptr, 0, 0, 0,
                                              idx, T, H_q, d, k_sel, sm_scale, (uint16_t *)out, lse,
                                              nullptr, 1, nullptr, st);
        if (e != cudaErrorNotSupported) return e;
    }
    return launch_sparse_attn_bf16((const uint16_t *)q, (const uint16_t *)k, (const uint16_t *)v,
                                   idx, T, T, H_q, d, k_sel, sm_scale, (uint16_t *)out, lse, st);
}

// Attention of `rows` query rows (q, idx, out, lse already offset to the first
// row) against the whole contiguous K/V of T rows; bf16, for dsa_prefill_host.
cudaError_t run_attn_rows(const void *q, const void *k, const void *v, const int32_t *idx, int64_t T,
                          int64_t rows, int H_q, int d, int k_sel, float sm_scale, void *out, float *lse,
                          cudaStream_t st)
{
    if (sparse_attn_tc_supported(H_q, d)) {
        cudaError_t e = launch_sparse_attn_tc((const uint16_t *)q, (const uint16_t *)k, (const uint16_t *)v,
                                              T, T, nullptr, nullptr, 0, 0, 0, idx, rows, H_q, d, k_sel,
                                              sm_scale, (uint16_t *)out, lse, nullptr, 1, nullptr, st);
        if (e != cudaErrorNotSupported) return e;
    }
    return launch_sparse_attn_bf16((const uint16_t *)q, (const uint16_t *)k, (const uint16_t *)v, idx, rows, T,
                                   H_q, d, k_sel, sm_scale, (uint16_t *)out, lse, st);
}

cudaError_t run_index(const void *q_idx, const float *q_scale, const void *k_idx,
                      const float *k_scale, const void *w, int64_t T, int H_I, int d_I,
                      int64_t row_begin, int64_t row_count, float *out, int64_t ld,
                      bool write_upper, dsa_dtype dtype, cudaStream_t st)
{
    if (dtype == DSA_E4M3) {
        // tcgen05 tensor-core indexer where the shape allows, else mma.sync
        if (index_tc_supported(H_I) && T < ((int64_t)1 << 31)) {
            cudaError_t e = launch_index_tc((const uint8_t *)q_idx, q_scale, (const uint8_t *)k_idx,
                                            k_scale, (const uint16_t *)w, T, H_I, row_begin,
                                            row_count, out, ld, write_upper, nullptr, st);
            if (e != cudaErrorNotSupported) return e;
        }
        return launch_index_fp8((const uint8_t *)q_idx, q_scale, (const uint8_t *)k_idx, k_scale,
                                (const uint16_t *)w, T, H_I, row_begin, row_count, out, ld,
                                write_upper, st);
    }
    return launch_index_f32((const float *)q_idx, (const float *)k_idx, (const float *)w, T, H_I,
                            d_I, row_begin, row_count, out, ld, write_upper, st);
}

// Device mirrors of a prefill's inputs and outputs plus the prefill scratch,
// carved from one workspace (E4M3 layouts), for dsa_prefill_host.
struct HostPrefillLayout {
    size_t q_idx, q_scale, w, q, k_idx, k_scale, k, v, out, lse, idx, scores, total;
    int64_t R;
    bool fused;                  // the fused selection's scratch follows the mirrors
    FusedLayout F;
    HostPrefillLayout(int64_t T, int H_I, int d_I, int H_q, int d, int k_sel)
        : fused(fused_ok(DSA_E4M3, H_I, T, k_sel)), F(1, 1, 0, 0)
    {
        R = fused ? fused_rows_host(T) : prefill_rows_default(T);
        size_t off = kWsHeader;
        auto take = [&](size_t bytes) { size_t o = off; off += align_up(bytes, 256); return o; };
        q_idx = take((size_t)T * H_I * d_I);
        q_scale = take(sizeof(float) * (size_t)T);
        w = take(2 * (size_t)T * H_I);
        q = take(2 * (size_t)T * H_q * d);
        k_idx = take((size_t)T * d_I);
        k_scale = take(sizeof(float) * (size_t)T);
        k = take(2 * (size_t)T * d);
        v = take(2 * (size_t)T * d);
        out = take(2 * (size_t)T * H_q * d);
        lse = take(sizeof(float) * (size_t)T * H_q);
        idx = take(sizeof(int32_t) * (size_t)T * k_sel);
        if (fused) {
            F = FusedLayout(T, k_sel, R, off);
            scores = F.scores;
            total = F.end;
        } else {
            scores = take(sizeof(float) * (size_t)R * T);
            total = off;
        }
    }
};

// Per-device copy streams and events for dsa_prefill_host, created on first
// use and kept for the life of the process.
struct CopyEngine {
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, in = nullptr, in_attn = nullptr, out = nullptr, done = nullptr;
    bool ok = false;
};

CopyEngine *copy_engine()
{
    static CopyEngine engines[64];
    static std::once_flag once[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    std::call_once(once[dev], [dev] {
        CopyEngine &c = engines[dev];
        c.ok = cudaStreamCreateWithFlags(&c.h2d, cudaStreamNonBlocking) == cudaSuccess &&
               cudaStreamCreateWithFlags(&c.d2h, cudaStreamNonBlocking) == cudaSuccess &&
               cudaEventCreateWithFlags(&c.start, cudaEventDisableTiming) == cudaSuccess &&
               cudaEventCreateWithFlags(&c.in, cudaEventDisableTiming) == cudaSuccess &&
               cudaEventCreateWithFlags(&c.in_attn, cudaEventDisableTiming) == cudaSuccess &&
               cudaEventCreateWithFlags(&c.out, cudaEventDisableTiming) == cudaSuccess &&
               cudaEventCreateWithFlags(&c.done, cudaEventDisableTiming) == cudaSuccess;
    });
    return engines[dev].ok ? &engines[dev] : nullptr;
}

// The fused prefill of query rows [row_begin, row_begin + rows) of a sequence
// whose key side (k_idx, k_scale, k, v) holds positions [0, T): the query side
// (q_idx, q_scale, w, q) and the outputs (out, lse, idx) hold those rows only.
cudaError_t prefill_fused_rows(const FusedLayout &L, uint8_t *ws, const void *q_idx, const float *q_scale,
                               const void *k_idx, const float *k_scale, const void *w, const void *q,
                               const void *k, const void *v, int64_t T, int64_t row_begin, int64_t rows, int H_I,
                               int H_q, int d, int k_sel, int window, float sm_scale, void *out, float *lse_out,
                               int32_t *idx, WsHeader *hdr, cudaStream_t st)
{
    const int kw = k_sel + window;
    cudaError_t e = fused_gather(L, ws, k_idx, k_scale, st);
    for (int64_t r = 0; e == cudaSuccess && r < rows; r += L.R) {
        const int64_t n = rows - r < L.R ? rows - r : L.R;
        if (r % L.SG == 0) {                         // the sample scores of the next group of passes
            e = fused_sample(L, ws, q_idx, q_scale, w, T, H_I, window, row_begin + r,
                             rows - r < L.SG ? rows - r : L.SG, hdr, st, row_begin, rows);
            if (e != cudaSuccess) break;
        }
        e = fused_select_pass(L, ws, q_idx, q_scale, k_idx, k_scale, w, T, H_I, k_sel, window, row_begin + r, n,
                              idx + r * (int64_t)kw, hdr, st, row_begin, rows, r % L.SG);
    }
    if (e == cudaSuccess) {
        StageTimer tm(DSA_STAGE_ATTN, st);
        e = run_attn_rows(q, k, v, idx, T, rows, H_q, d, kw, sm_scale, out, lse_out, st);
    }
    return e;
}

std::atomic<int> g_test_stall{0};               // 0: off, else 1 + the armed target

}  // namespace

bool dsa::consume_test_stall(int target)
{
    int want = target + 1;
    return g_test_stall.load(std::memory_order_relaxed) == want &&
           g_test_stall.compare_exchange_strong(want, 0);
}

extern "C" {

dsa_status dsa_test_stall_next(dsa_stall_target target)
{
    if (target == DSA_STALL_NONE) { g_test_stall.store(0); return DSA_OK; }
    if (target != DSA_STALL_PREFILL_INDEXER && target != DSA_STALL_DECODE_INDEXER) return DSA_ERR_INVALID_ARG;
    g_test_stall.store(target == DSA_STALL_PREFILL_INDEXER ? 1 : 2);
    return DSA_OK;
}

const char *dsa_status_string(dsa_status s)
{
    switch (s) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
    case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT";
    }
    return "DSA_ERR_UNKNOWN";
}

int dsa_version(void) { return (DSA_VERSION_MAJOR << 16) | DSA_VERSION_MINOR; }

dsa_status dsa_index_scores(const void *q_idx, const float *q_scale, const void *k_idx,
                            const float *k_scale, const void *w, int64_t T, int H_I, int d_I,
                            int64_t q_row_begin, int64_t q_row_count, float *scores_out,
                            int64_t ld_scores, int fill_upper, dsa_dtype dtype, void *stream)
{
    dsa_status s = check_index_args(q_idx, q_scale, k_idx, k_scale, w, T, H_I, d_I, dtype);
    if (s != DSA_OK) return s;
    if (q_row_begin < 0 || q_row_count < 0 || q_row_begin + q_row_count > T) return DSA_ERR_INVALID_ARG;
    if (q_row_count == 0) return DSA_OK;
    if (!scores_out || ld_scores < T) return DSA_ERR_INVALID_ARG;
    return cuda_status(run_index(q_idx, q_scale, k_idx, k_scale, w, T, H_I, d_I, q_row_begin,
                                 q_row_count, scores_out, ld_scores, fill_upper != 0, dtype,
                                 as_stream(stream)));
}

size_t dsa_topk_workspace_size(int64_t row_count, int64_t T, int k)
{
    (void)row_count; (void)T; (void)k;
    return 0;
}

dsa_status dsa_topk(const float *scores, int64_t ld_scores, int64_t row_begin,
                    int64_t row_count, int64_t T, int k, int32_t *idx_out, void *workspace,
                    size_t ws_bytes, void *stream)
{
    (void)workspace; (void)ws_bytes;
    if (!scores || !idx_out || T <= 0 || k < 1 || k > 65536) return DSA_ERR_INVALID_ARG;
    if (row_begin < 0 || row_count < 0 || row_begin + row_count > T || ld_scores < T)
        return DSA_ERR_INVALID_ARG;
    if (row_count == 0) return DSA_OK;
    return cuda_status(launch_topk_rows(scores, ld_scores, row_begin, nullptr, T, row_count, k,
                                        idx_out, nullptr, as_stream(stream)));
}

dsa_status dsa_topk_window(const float *scores, int64_t ld_scores, int64_t row_begin,
                           int64_t row_count, int64_t T, int k, int window, int32_t *idx_out,
                           void *workspace, size_t ws_bytes, void *stream)
{
    (void)workspace; (void)ws_bytes;
    if (!scores || !idx_out || T <= 0 || k < 1 || k > 65536 || window < 0 || window > kMaxWindow)
        return DSA_ERR_INVALID_ARG;
    if (row_begin < 0 || row_count < 0 || row_begin + row_count > T || ld_scores < T)
        return DSA_ERR_INVALID_ARG;
    if (row_count == 0) return DSA_OK;
    return cuda_status(launch_topk_rows(scores, ld_scores, row_begin, nullptr, T, row_count, k,
                                        idx_out, nullptr, as_stream(stream), window));
}

dsa_status dsa_sparse_attn(const void *q, const void *k, const void *v, const int32_t *idx,
                           int64_t T, int H_q, int d, int k_sel, float sm_scale, void *out,
                           float *lse_out, dsa_dtype dtype, void *stream)
{
    dsa_status s = check_attn_args(q, k, v, idx, T, H_q, d, k_sel, out, dtype);
    if (s != DSA_OK) return s;
    if (!std::isfinite(sm_scale)) return DSA_ERR_INVALID_ARG;
    return cuda_status(run_attn(q, k, v, idx, T, H_q, d, k_sel, sm_scale, out, lse_out, dtype,
                                as_stream(stream)));
}

size_t dsa_prefill_workspace_size(int64_t T, int H_I, int d_I, int H_q, int d, int k_sel,
                                  dsa_dtype dtype)
{
    (void)d_I; (void)H_q; (void)d;
    if (T <= 0 || k_sel <= 0) return 0;
    if (fused_ok(dtype, H_I, T, k_sel))
        return FusedLayout(T, k_sel, fused_rows_default(T), kWsHeader + idx_bytes(T, k_sel)).end;
    int64_t R = prefill_rows_default(T);
    return kWsHeader + idx_bytes(T, k_sel) + align_up(sizeof(float) * (size_t)R * T, 256);
}

}  // extern "C"

namespace {

// dsa_prefill with a sliding window of `window` positions (0: none); the
// selection rows are k_sel + window wide.
dsa_status prefill_impl(const void *q_idx, const float *q_scale, const void *k_idx,
                        const float *k_scale, const void *w, const void *q, const void *k,
                        const void *v, int64_t T, int H_I, int d_I, int H_q, int d, int k_sel,
                        int window, float sm_scale, void *out, float *lse_out, int32_t *idx_out,
                        dsa_dtype dtype, void *workspace, size_t ws_bytes, void *stream)
{
    if (dtype != DSA_E4M3 && dtype != DSA_F32) return DSA_ERR_UNSUPPORTED;
    dsa_status s = check_index_args(q_idx, q_scale, k_idx, k_scale, w, T, H_I, d_I, dtype);
    if (s != DSA_OK) return s;
    // any non-null placeholder for idx: only the other attention arguments are checked here
    s = check_attn_args(q, k, v, reinterpret_cast<const int32_t *>(q), T, H_q, d, k_sel, out, dtype);
    if (s != DSA_OK) return s;
    if (k_sel > 65536 || window < 0 || window > kMaxWindow || !std::isfinite(sm_scale))
        return DSA_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DSA_ERR_WORKSPACE;
    const int kw = k_sel + window;                    // selection row width
    size_t fixed = kWsHeader + (idx_out ? 0 : idx_bytes(T, kw));
    if (fused_ok(dtype, H_I, T, k_sel)) {
        const int64_t R = fused_rows_fitting(T, k_sel, fixed, ws_bytes);
        if (R < 128) return DSA_ERR_WORKSPACE;
        const FusedLayout L(T, k_sel, R, fixed);
        cudaStream_t st = as_stream(stream);
        uint8_t *ws = static_cast<uint8_t *>(workspace);
        WsHeader *hdr = reinterpret_cast<WsHeader *>(ws);
        int32_t *idx = idx_out ? idx_out : reinterpret_cast<int32_t *>(ws + kWsHeader);
        cudaError_t e = cudaMemsetAsync(hdr, 0, sizeof(WsHeader), st);
        if (e == cudaSuccess)
            e = prefill_fused_rows(L, ws, q_idx, q_scale, k_idx, k_scale, w, q, k, v, T, 0, T, H_I, H_q, d, k_sel,
                                   window, sm_scale, out, lse_out, idx, hdr, st);
        return cuda_status(e);
    }
    if (ws_bytes < fixed + sizeof(float) * 64 * (size_t)T) return DSA_ERR_WORKSPACE;
    int64_t R = (int64_t)((ws_bytes - fixed) / (sizeof(float) * (size_t)T)) / 64 * 64;
    R = R < T ? R : ceil_div(T, 64) * 64;

    cudaStream_t st = as_stream(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    WsHeader *hdr = reinterpret_cast<WsHeader *>(ws);
    int32_t *idx = idx_out ? idx_out : reinterpret_cast<int32_t *>(ws + kWsHeader);
    float *scores = reinterpret_cast<float *>(ws + fixed);
    cudaError_t e = cudaMemsetAsync(hdr, 0, sizeof(WsHeader), st);
    for (int64_t r0 = 0; e == cudaSuccess && r0 < T; r0 += R) {
        int64_t n = T - r0 < R ? T - r0 : R;
        {
            StageTimer tm(DSA_STAGE_SCORES, st);
            e = run_index(q_idx, q_scale, k_idx, k_scale, w, T, H_I, d_I, r0, n, scores, T, false,
                          dtype, st);
        }
        if (e == cudaSuccess) {
            StageTimer tm(DSA_STAGE_TOPK, st);
            e = launch_topk_rows(scores, T, r0, nullptr, T, n, k_sel, idx + r0 * (int64_t)kw,
                                 hdr, st, window);
        }
    }
    if (e == cudaSuccess) {
        StageTimer tm(DSA_STAGE_ATTN, st);
        e = run_attn(q, k, v, idx, T, H_q, d, kw, sm_scale, out, lse_out, dtype, st);
    }
    return cuda_status(e);
}

}  // namespace

extern "C" {

dsa_status dsa_prefill(const void *q_idx, const float *q_scale, const void *k_idx,
                       const float *k_scale, const void *w, const void *q, const void *k,
                       const void *v, int64_t T, int H_I, int d_I, int H_q, int d, int k_sel,
                       float sm_scale, void *out, float *lse_out, int32_t *idx_out,
                       dsa_dtype dtype, void *workspace, size_t ws_bytes, void *stream)
{
    return prefill_impl(q_idx, q_scale, k_idx, k_scale, w, q, k, v, T, H_I, d_I, H_q, d, k_sel, 0,
                        sm_scale, out, lse_out, idx_out, dtype, workspace, ws_bytes, stream);
}

dsa_status dsa_prefill_window(const void *q_idx, const float *q_scale, const void *k_idx,
                              const float *k_scale, const void *w, const void *q, const void *k,
                              const void *v, int64_t T, int H_I, int d_I, int H_q, int d, int k_sel,
                              int window, float sm_scale, void *out, float *lse_out,
                              int32_t *idx_out, dsa_dtype dtype, void *workspace, size_t ws_bytes,
                              void *stream)
{
    return prefill_impl(q_idx, q_scale, k_idx, k_scale, w, q, k, v, T, H_I, d_I, H_q, d, k_sel,
                        window, sm_scale, out, lse_out, idx_out, dtype, workspace, ws_bytes, stream);
}

size_t dsa_prefill_rows_workspace_size(int64_t T, int64_t row_count, int H_I, int d_I, int H_q, int d,
                                       int k_sel, dsa_dtype dtype)
{
    (void)d_I; (void)H_q; (void)d;
    if (T <= 0 || row_count <= 0 || row_count > T || !fused_ok(dtype, H_I, T, k_sel)) return 0;
    const int64_t rmax = ceil_div(row_count, 128) * 128;
    const int64_t R = fused_rows_default(T) < rmax ? fused_rows_default(T) : rmax;
    return FusedLayout(T, k_sel, R, kWsHeader + idx_bytes(row_count, k_sel)).end;
}

dsa_status dsa_prefill_rows(const void *q_idx, const float *q_scale, const void *k_idx, const float *k_scale,
                            const void *w, const void *q, const void *k, const void *v, int64_t T,
                            int64_t row_begin, int64_t row_count, int H_I, int d_I, int H_q, int d, int k_sel,
                            float sm_scale, void *out, float *lse_out, int32_t *idx_out, dsa_dtype dtype,
                            void *workspace, size_t ws_bytes, void *stream)
{
    if (dtype != DSA_E4M3) return DSA_ERR_UNSUPPORTED;
    if (row_begin < 0 || row_count < 0 || row_begin + row_count > T) return DSA_ERR_INVALID_ARG;
    // the q-side arrays hold row_count rows: check them as a sequence of that length
    dsa_status s = check_index_args(q_idx, q_scale, k_idx, k_scale, w, T, H_I, d_I, dtype);
    if (s != DSA_OK) return s;
    s = check_attn_args(q, k, v, reinterpret_cast<const int32_t *>(q), T, H_q, d, k_sel, out, dtype);
    if (s != DSA_OK) return s;
    if (k_sel > 65536 || !std::isfinite(sm_scale)) return DSA_ERR_INVALID_ARG;
    if (!fused_ok(dtype, H_I, T, k_sel)) return DSA_ERR_UNSUPPORTED;
    if (row_count == 0) return DSA_OK;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DSA_ERR_WORKSPACE;
    const size_t fixed = kWsHeader + (idx_out ? 0 : idx_bytes(row_count, k_sel));
    int64_t R = fused_rows_fitting(T, k_sel, fixed, ws_bytes);
    const int64_t rmax = ceil_div(row_count, 128) * 128;
    if (R > rmax) R = rmax;
    if (R < 128) return DSA_ERR_WORKSPACE;
    const FusedLayout L(T, k_sel, R, fixed);
    cudaStream_t st = as_stream(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    WsHeader *hdr = reinterpret_cast<WsHeader *>(ws);
    int32_t *idx = idx_out ? idx_out : reinterpret_cast<int32_t *>(ws + kWsHeader);
    cudaError_t e = cudaMemsetAsync(hdr, 0, sizeof(WsHeader), st);
    if (e == cudaSuccess)
        e = prefill_fused_rows(L, ws, q_idx, q_scale, k_idx, k_scale, w, q, k, v, T, row_begin, row_count, H_I,
                               H_q, d, k_sel, 0, sm_scale, out, lse_out, idx, hdr, st);
    return cuda_status(e);
}

size_t dsa_prefill_host_workspace_size(int64_t T, int H_I, int d_I, int H_q, int d, int k_sel,
                                       dsa_dtype dtype)
{
    if (dtype != DSA_E4M3 || T <= 0 || H_I <= 0 || d_I <= 0 || H_q <= 0 || d <= 0 || k_sel <= 0) return 0;
    return HostPrefillLayout(T, H_I, d_I, H_q, d, k_sel).total;
}

dsa_status dsa_prefill_host(const void *q_idx, const float *q_scale, const void *k_idx,
                            const float *k_scale, const void *w, const void *q, const void *k,
                            const void *v, int64_t T, int H_I, int d_I, int H_q, int d, int k_sel,
                            float sm_scale, void *out, float *lse_out, int32_t *idx_out,
                            dsa_dtype dtype, void *workspace, size_t ws_bytes, void *stream)
{
    if (dtype != DSA_E4M3) return DSA_ERR_UNSUPPORTED;
    if (!q_idx || !q_scale || !k_idx || !k_scale || !w || !q || !k || !v || !out) return DSA_ERR_INVALID_ARG;
    if (T <= 0 || H_I <= 0 || d_I <= 0 || H_q <= 0 || d <= 0 || k_sel <= 0 || k_sel > 65536 ||
        !std::isfinite(sm_scale))
        return DSA_ERR_INVALID_ARG;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DSA_ERR_WORKSPACE;
    const HostPrefillLayout L(T, H_I, d_I, H_q, d, k_sel);
    if (ws_bytes < L.total) return DSA_ERR_WORKSPACE;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    // the device mirrors must pass the same checks as dsa_prefill's arguments
    dsa_status s = check_index_args(ws + L.q_idx, (const float *)(ws + L.q_scale), ws + L.k_idx,
                                    (const float *)(ws + L.k_scale), ws + L.w, T, H_I, d_I, dtype);
    if (s != DSA_OK) return s;
    s = check_attn_args(ws + L.q, ws + L.k, ws + L.v, (const int32_t *)(ws + L.idx), T, H_q, d, k_sel,
                        ws + L.out, dtype);
    if (s != DSA_OK) return s;
    // Passes run from the last rows to the first: late rows carry the most work per
    // copied byte (their causal rows are longest), so the copies stay ahead of the
    // computation.  The first pass and the last are at most kHostEdgeRows rows: the
    // computation starts as soon as that few query rows have landed, and the outputs
    // left to copy after it has ended are that few rows'.
    constexpr int64_t kHostEdgeRows = 512;
    std::vector<std::pair<int64_t, int64_t>> passes;   // (first row, rows), in processing order
    {
        const int64_t edge = L.R < kHostEdgeRows ? L.R : kHostEdgeRows;
        int64_t top = T;
        const int64_t n0 = edge < top ? edge : top;
        passes.emplace_back(top - n0, n0);
        top -= n0;
        const int64_t bottom = edge < top ? edge : top;
        while (top > bottom) {
            const int64_t n = L.R < top - bottom ? L.R : top - bottom;
            passes.emplace_back(top - n, n);
            top -= n;
        }
        if (bottom > 0) passes.emplace_back(0, bottom);
    }
    CopyEngine *ce = copy_engine();
    if (!ce) return DSA_ERR_CUDA;
    cudaStream_t st = as_stream(stream);
    WsHeader *hdr = reinterpret_cast<WsHeader *>(ws);
    float *scores = reinterpret_cast<float *>(ws + L.scores);
    int32_t *idx = reinterpret_cast<int32_t *>(ws + L.idx);
    const size_t qi_row = (size_t)H_I * d_I, q_row = 2 * (size_t)H_q * d;
    auto h2d = [&](size_t off, const void *src, size_t bytes) {
        return cudaMemcpyAsync(ws + off, src, bytes, cudaMemcpyHostToDevice, ce->h2d);
    };
    auto d2h = [&](void *dst, size_t off, size_t bytes) {
        return cudaMemcpyAsync(dst, ws + off, bytes, cudaMemcpyDeviceToHost, ce->d2h);
    };
    // The copy streams start behind the caller's stream's earlier work; inputs move
    // pass by pass ahead of the compute, and each pass's outputs leave while the next
    // pass computes.
    cudaError_t e = cudaMemsetAsync(hdr, 0, sizeof(WsHeader), st);
    if (e == cudaSuccess) e = cudaEventRecord(ce->start, st);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ce->h2d, ce->start, 0);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(ce->d2h, ce->start, 0);
    // The selection needs only the index keys, their scales, the query scales and
    // the head weights: they go first, and K and V follow while the first pass
    // selects.
    if (e == cudaSuccess) e = h2d(L.k_idx, k_idx, (size_t)T * d_I);
    if (e == cudaSuccess) e = h2d(L.k_scale, k_scale, sizeof(float) * (size_t)T);
    if (e == cudaSuccess) e = h2d(L.q_scale, q_scale, sizeof(float) * (size_t)T);
    if (e == cudaSuccess) e = h2d(L.w, w, 2 * (size_t)T * H_I);
    if (e == cudaSuccess) e = cudaEventRecord(ce->in, ce->h2d);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ce->in, 0);
    if (e == cudaSuccess && L.fused)          // the sampled keys, once the keys have landed
        e = fused_gather(L.F, ws, ws + L.k_idx, (const float *)(ws + L.k_scale), st);
    // the first pass's index queries go ahead of K and V (the h2d stream is in order)
    if (e == cudaSuccess)
        e = h2d(L.q_idx + passes[0].first * qi_row, static_cast<const uint8_t *>(q_idx) + passes[0].first * qi_row,
                passes[0].second * qi_row);
    if (e == cudaSuccess) e = cudaEventRecord(ce->in, ce->h2d);
    if (e == cudaSuccess) e = h2d(L.k, k, 2 * (size_t)T * d);
    if (e == cudaSuccess) e = h2d(L.v, v, 2 * (size_t)T * d);
    for (size_t pi = 0; e == cudaSuccess && pi < passes.size(); ++pi) {
        const int64_t r0 = passes[pi].first, n = passes[pi].second;
        // the pass's index queries for its selection (the first pass's went ahead of K
        // and V), then its queries for its attention
        if (pi > 0) {
            e = h2d(L.q_idx + r0 * qi_row, static_cast<const uint8_t *>(q_idx) + r0 * qi_row, n * qi_row);
            if (e == cudaSuccess) e = cudaEventRecord(ce->in, ce->h2d);
        }
        if (e == cudaSuccess) e = h2d(L.q + r0 * q_row, static_cast<const uint8_t *>(q) + r0 * q_row, n * q_row);
        if (e == cudaSuccess) e = cudaEventRecord(ce->in_attn, ce->h2d);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ce->in, 0);
        if (e == cudaSuccess && L.fused) {
            // one pass's sample scores at a time
            e = fused_sample(L.F, ws, ws + L.q_idx, (const float *)(ws + L.q_scale), ws + L.w, T, H_I, 0, r0, n,
                             hdr, st, 0, T);
            if (e == cudaSuccess)
                e = fused_select_pass(L.F, ws, ws + L.q_idx, (const float *)(ws + L.q_scale), ws + L.k_idx,
                                      (const float *)(ws + L.k_scale), ws + L.w, T, H_I, k_sel, 0, r0, n,
                                      idx + r0 * (int64_t)k_sel, hdr, st, 0, T, 0);
        } else {
            if (e == cudaSuccess) {
                StageTimer tm(DSA_STAGE_SCORES, st);
                e = run_index(ws + L.q_idx, (const float *)(ws + L.q_scale), ws + L.k_idx,
                              (const float *)(ws + L.k_scale), ws + L.w, T, H_I, d_I, r0, n, scores, T, false,
                              dtype, st);
            }
            if (e == cudaSuccess) {
                StageTimer tm(DSA_STAGE_TOPK, st);
                e = launch_topk_rows(scores, T, r0, nullptr, T, n, k_sel, idx + r0 * (int64_t)k_sel, hdr, st);
            }
        }
        // the attention also needs K and V, copied before any pass's queries
        if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ce->in_attn, 0);
        if (e == cudaSuccess) {
            StageTimer tm(DSA_STAGE_ATTN, st);
            e = run_attn_rows(ws + L.q + r0 * q_row, ws + L.k, ws + L.v, idx + r0 * (int64_t)k_sel, T, n, H_q,
                              d, k_sel, sm_scale, ws + L.out + r0 * q_row,
                              reinterpret_cast<float *>(ws + L.lse) + r0 * H_q, st);
        }
        if (e == cudaSuccess) e = cudaEventRecord(ce->out, st);
        if (e == cudaSuccess) e = cudaStreamWaitEvent(ce->d2h, ce->out, 0);
        if (e == cudaSuccess)
            e = d2h(static_cast<uint8_t *>(out) + r0 * q_row, L.out + r0 * q_row, n * q_row);
        if (e == cudaSuccess && lse_out)
            e = d2h(lse_out + r0 * H_q, L.lse + sizeof(float) * r0 * H_q, sizeof(float) * n * H_q);
        if (e == cudaSuccess && idx_out)
            e = d2h(idx_out + r0 * (int64_t)k_sel, L.idx + sizeof(int32_t) * r0 * k_sel,
                    sizeof(int32_t) * n * k_sel);
    }
    // the caller's stream completes only once the last outputs are on the host
    if (e == cudaSuccess) e = cudaEventRecord(ce->done, ce->d2h);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st, ce->done, 0);
    return cuda_status(e);
}

size_t dsa_decode_workspace_size(int B, int64_t max_context, int H_q, int d, int k_sel)
{
    if (B <= 0 || max_context <= 0 || k_sel <= 0) return 0;
    int splits = sparse_attn_paged_splits(B, k_sel);
    return kWsHeader + align_up(sizeof(float) * (size_t)B * max_context, 256) + idx_bytes(B, k_sel) +
           align_up(sparse_attn_paged_part_bytes(B, H_q, d, splits), 256) +
           align_up(topk_split_ws_bytes(B, max_context), 256);
}

}  // extern "C"

namespace {

// The decode indexer's scores [B, max_context] and each row's top-k (plus the
// window) into idx [B, k_sel + window].
cudaError_t run_decode_select(const void *q_idx, const float *q_scale, const void *w, const void *kidx_cache,
                              const float *kscale_cache, const int32_t *block_table, const int32_t *context_lens,
                              int64_t num_pages, int max_pages_per_seq, int page_size, int B,
                              int64_t max_context, int H_I, int k_sel, int window, float *scores, int32_t *idx,
                              void *topk_ws, WsHeader *hdr, cudaStream_t st)
{
    cudaError_t e;
    // tensor-core (tcgen05 + TMA) indexer where the shape allows, else mma.sync
    if (decode_index_tc_supported(H_I, page_size) && B <= 4096 &&
        (int64_t)num_pages * page_size < ((int64_t)1 << 31) && aligned16(kscale_cache))
        e = launch_decode_index_tc((const uint8_t *)q_idx, q_scale, (const uint16_t *)w,
                                   (const uint8_t *)kidx_cache, kscale_cache, block_table, context_lens,
                                   num_pages, max_pages_per_seq, page_size, B, max_context, H_I, scores,
                                   max_context, hdr, st);
    else
        e = launch_decode_index((const uint8_t *)q_idx, q_scale, (const uint16_t *)w,
                                (const uint8_t *)kidx_cache, kscale_cache, block_table, context_lens,
                                num_pages, max_pages_per_seq, page_size, B, max_context, H_I, scores,
                                max_context, hdr, st);
    if (e == cudaSuccess)   // each row split over 16K-position chunks (CTAs), then one CTA per row
        e = launch_topk_split(scores, max_context, context_lens, max_context, B, k_sel, idx, topk_ws, hdr, st,
                              window);
    return e;
}

// The paged attention of B single-token queries over idx [B, kw] (tcgen05
// kernel where the shape allows, else the mma.sync one; FP8 K/V when
// k_cache_scale is given), split over the index list and merged.
cudaError_t run_decode_attend(const void *q, const void *k_cache, const void *v_cache, const float *k_cache_scale,
                              const float *v_cache_scale, const int32_t *block_table, const int32_t *context_lens,
                              int64_t num_pages, int max_pages_per_seq, int page_size, int B, int H_q, int d,
                              int kw, float sm_scale, const int32_t *idx, void *out, float *lse_out, float *part,
                              WsHeader *hdr, cudaStream_t st)
{
    const int splits = sparse_attn_paged_splits(B, kw);
    const int chunk = (int)(ceil_div(ceil_div(kw, splits), 128) * 128);
    const int tc_splits = (int)ceil_div(kw, chunk);
    cudaError_t e;
    if (k_cache_scale) {
        // tcgen05 kernel over the FP8 caches, the index list split in 128-row blocks
        if ((int64_t)num_pages * page_size >= ((int64_t)1 << 31)) return cudaErrorNotSupported;
        e = launch_sparse_attn_tc_kv8((const uint16_t *)q, (const uint8_t *)k_cache, k_cache_scale,
                                      (const uint8_t *)v_cache, v_cache_scale, num_pages * page_size, block_table,
                                      context_lens, num_pages, max_pages_per_seq, page_size, idx, B, H_q, d, kw,
                                      sm_scale, (uint16_t *)out, lse_out, part, tc_splits, hdr, st,
                                      /*chained=*/true);
        if (e == cudaSuccess) e = launch_merge_splits(part, B, tc_splits, H_q, d, (uint16_t *)out, lse_out, st);
        return e;
    }
    if (sparse_attn_tc_supported(H_q, d) && (int64_t)num_pages * page_size < ((int64_t)1 << 31)) {
        // tcgen05 kernel over the paged caches, the index list split in 128-row blocks
        e = launch_sparse_attn_tc((const uint16_t *)q, (const uint16_t *)k_cache, (const uint16_t *)v_cache,
                                  num_pages * page_size, 0, block_table, context_lens, num_pages,
                                  max_pages_per_seq, page_size, idx, B, H_q, d, kw, sm_scale, (uint16_t *)out,
                                  lse_out, part, tc_splits, hdr, st, /*chained=*/true);
        if (e == cudaSuccess) e = launch_merge_splits(part, B, tc_splits, H_q, d, (uint16_t *)out, lse_out, st);
        if (e != cudaErrorNotSupported) return e;
    }
    PagedKV kv{(const uint16_t *)k_cache, (const uint16_t *)v_cache, block_table, context_lens,
               num_pages, max_pages_per_seq, page_size};
    return launch_sparse_attn_paged_bf16((const uint16_t *)q, kv, idx, B, H_q, d, kw, sm_scale, (uint16_t *)out,
                                         lse_out, part, splits, hdr, st);
}

// dsa_decode with a sliding window of `window` positions (0: none); the
// selection rows (and the attention's index lists) are k_sel + window wide.
// k_cache_scale / v_cache_scale non-null: the K/V caches hold E4M3 codes with
// one fp32 scale per cached token (tcgen05 attention only).
dsa_status decode_impl(const void *q_idx, const float *q_scale, const void *w, const void *q,
                       const void *kidx_cache, const float *kscale_cache, const void *k_cache,
                       const void *v_cache, const int32_t *block_table,
                       const int32_t *context_lens, int64_t num_pages, int max_pages_per_seq,
                       int page_size, int B, int64_t max_context, int H_I, int d_I, int H_q,
                       int d, int k_sel, int window, float sm_scale, void *out, float *lse_out,
                       int32_t *idx_out, void *workspace, size_t ws_bytes, void *stream,
                       const float *k_cache_scale = nullptr, const float *v_cache_scale = nullptr)
{
    const bool kv8 = k_cache_scale != nullptr;
    if (kv8 && (!v_cache_scale || (reinterpret_cast<uintptr_t>(k_cache_scale) & 3u) ||
                (reinterpret_cast<uintptr_t>(v_cache_scale) & 3u)))
        return DSA_ERR_INVALID_ARG;
    if (kv8 && !sparse_attn_tc_supported(H_q, d)) return DSA_ERR_UNSUPPORTED;
    if (window < 0 || window > kMaxWindow || k_sel > 65536) return DSA_ERR_INVALID_ARG;
    const int kw = k_sel + window;                    // selection row width
    if (!q_idx || !q_scale || !w || !q || !kidx_cache || !kscale_cache || !k_cache || !v_cache ||
        !block_table || !context_lens || !out)
        return DSA_ERR_INVALID_ARG;
    if (B <= 0 || max_context <= 0 || num_pages <= 0 || max_pages_per_seq <= 0 || page_size <= 0 ||
        H_I <= 0 || H_q <= 0 || k_sel <= 0 || k_sel > 65536 || !std::isfinite(sm_scale))
        return DSA_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(q) || !aligned16(kidx_cache) || !aligned16(k_cache) ||
        !aligned16(v_cache) || !aligned16(out))
        return DSA_ERR_INVALID_ARG;
    if (d_I != 128 || d != 128 || H_I > 64 || H_I % 8 != 0 || page_size % 16 != 0)
        return DSA_ERR_UNSUPPORTED;
    if (H_q > 128 && H_q % 128 != 0) return DSA_ERR_UNSUPPORTED;
    if (B > 65535) return DSA_ERR_UNSUPPORTED;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DSA_ERR_WORKSPACE;
    if (ws_bytes < dsa_decode_workspace_size(B, max_context, H_q, d, kw)) return DSA_ERR_WORKSPACE;

    cudaStream_t st = as_stream(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    WsHeader *hdr = reinterpret_cast<WsHeader *>(ws);
    size_t off = kWsHeader;
    float *scores = reinterpret_cast<float *>(ws + off);
    off += align_up(sizeof(float) * (size_t)B * max_context, 256);
    int32_t *idx = reinterpret_cast<int32_t *>(ws + off);
    off += idx_bytes(B, kw);
    float *part = reinterpret_cast<float *>(ws + off);
    off += align_up(sparse_attn_paged_part_bytes(B, H_q, d, sparse_attn_paged_splits(B, kw)), 256);
    void *topk_ws = ws + off;
    if (idx_out) idx = idx_out;

    cudaError_t e = cudaMemsetAsync(hdr, 0, sizeof(WsHeader), st);
    if (e == cudaSuccess)
        e = run_decode_select(q_idx, q_scale, w, kidx_cache, kscale_cache, block_table, context_lens, num_pages,
                              max_pages_per_seq, page_size, B, max_context, H_I, k_sel, window, scores, idx,
                              topk_ws, hdr, st);
    if (e == cudaSuccess) {
        e = run_decode_attend(q, k_cache, v_cache, k_cache_scale, v_cache_scale, block_table, context_lens,
                              num_pages, max_pages_per_seq, page_size, B, H_q, d, kw, sm_scale, idx, out, lse_out,
                              part, hdr, st);
        if (e == cudaErrorNotSupported) return DSA_ERR_UNSUPPORTED;
    }
    return cuda_status(e);
}

}  // namespace

extern "C" {

dsa_status dsa_decode(const void *q_idx, const float *q_scale, const void *w, const void *q,
                      const void *kidx_cache, const float *kscale_cache, const void *k_cache,
                      const void *v_cache, const int32_t *block_table,
                      const int32_t *context_lens, int64_t num_pages, int max_pages_per_seq,
                      int page_size, int B, int64_t max_context, int H_I, int d_I, int H_q,
                      int d, int k_sel, float sm_scale, void *out, float *lse_out,
                      int32_t *idx_out, void *workspace, size_t ws_bytes, void *stream)
{
    return decode_impl(q_idx, q_scale, w, q, kidx_cache, kscale_cache, k_cache, v_cache, block_table,
                       context_lens, num_pages, max_pages_per_seq, page_size, B, max_context, H_I, d_I,
                       H_q, d, k_sel, 0, sm_scale, out, lse_out, idx_out, workspace, ws_bytes, stream);
}

dsa_status dsa_decode_window(const void *q_idx, const float *q_scale, const void *w, const void *q,
                             const void *kidx_cache, const float *kscale_cache, const void *k_cache,
                             const void *v_cache, const int32_t *block_table,
                             const int32_t *context_lens, int64_t num_pages, int max_pages_per_seq,
                             int page_size, int B, int64_t max_context, int H_I, int d_I, int H_q,
                             int d, int k_sel, int window, float sm_scale, void *out, float *lse_out,
                             int32_t *idx_out, void *workspace, size_t ws_bytes, void *stream)
{
    return decode_impl(q_idx, q_scale, w, q, kidx_cache, kscale_cache, k_cache, v_cache, block_table,
                       context_lens, num_pages, max_pages_per_seq, page_size, B, max_context, H_I, d_I,
                       H_q, d, k_sel, window, sm_scale, out, lse_out, idx_out, workspace, ws_bytes,
                       stream);
}

dsa_status dsa_decode_kv8(const void *q_idx, const float *q_scale, const void *w, const void *q,
                          const void *kidx_cache, const float *kscale_cache, const void *k_cache,
                          const float *k_cache_scale, const void *v_cache, const float *v_cache_scale,
                          const int32_t *block_table, const int32_t *context_lens, int64_t num_pages,
                          int max_pages_per_seq, int page_size, int B, int64_t max_context, int H_I,
                          int d_I, int H_q, int d, int k_sel, int window, float sm_scale, void *out,
                          float *lse_out, int32_t *idx_out, void *workspace, size_t ws_bytes, void *stream)
{
    if (!k_cache_scale || !v_cache_scale) return DSA_ERR_INVALID_ARG;
    return decode_impl(q_idx, q_scale, w, q, kidx_cache, kscale_cache, k_cache, v_cache, block_table,
                       context_lens, num_pages, max_pages_per_seq, page_size, B, max_context, H_I, d_I,
                       H_q, d, k_sel, window, sm_scale, out, lse_out, idx_out, workspace, ws_bytes,
                       stream, k_cache_scale, v_cache_scale);
}

size_t dsa_split_workspace_size(int G, int B, int64_t max_context, int H_q, int d, int k_sel)
{
    if (G <= 0 || B <= 0 || max_context <= 0 || H_q <= 0 || d <= 0 || k_sel <= 0) return 0;
    const size_t select = align_up(sizeof(float) * (size_t)B * max_context, 256) + idx_bytes(B, k_sel) +
                          align_up(topk_split_ws_bytes(B, max_context), 256);
    const size_t attend = idx_bytes(B, k_sel) +
                          align_up(sparse_attn_paged_part_bytes(B, H_q, d, sparse_attn_paged_splits(B, k_sel)), 256);
    const size_t merge = align_up(merge_selections_ws_bytes(B, G, k_sel), 256);
    size_t m = select > attend ? select : attend;
    m = m > merge ? m : merge;
    return kWsHeader + m;
}

dsa_status dsa_decode_select(const void *q_idx, const float *q_scale, const void *w, const void *kidx_cache,
                             const float *kscale_cache, const int32_t *block_table, const int32_t *context_lens,
                             const int32_t *pos_base, int64_t num_pages, int max_pages_per_seq, int page_size,
                             int B, int64_t max_context, int H_I, int d_I, int k_sel, int32_t *cand_pos_out,
                             float *cand_score_out, void *workspace, size_t ws_bytes, void *stream)
{
    if (!q_idx || !q_scale || !w || !kidx_cache || !kscale_cache || !block_table || !context_lens || !pos_base ||
        !cand_pos_out || !cand_score_out)
        return DSA_ERR_INVALID_ARG;
    if (B <= 0 || max_context <= 0 || max_context > INT32_MAX || num_pages <= 0 || max_pages_per_seq <= 0 ||
        page_size <= 0 || H_I <= 0 || k_sel <= 0 || k_sel > 65536)
        return DSA_ERR_INVALID_ARG;
    if (!aligned16(q_idx) || !aligned16(kidx_cache)) return DSA_ERR_INVALID_ARG;
    if (d_I != 128 || H_I > 64 || H_I % 8 != 0 || page_size % 16 != 0) return DSA_ERR_UNSUPPORTED;
    if (B > 65535) return DSA_ERR_UNSUPPORTED;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DSA_ERR_WORKSPACE;
    const size_t need = kWsHeader + align_up(sizeof(float) * (size_t)B * max_context, 256) + idx_bytes(B, k_sel) +
                        align_up(topk_split_ws_bytes(B, max_context), 256);
    if (ws_bytes < need) return DSA_ERR_WORKSPACE;

    cudaStream_t st = as_stream(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    WsHeader *hdr = reinterpret_cast<WsHeader *>(ws);
    size_t off = kWsHeader;
    float *scores = reinterpret_cast<float *>(ws + off);
    off += align_up(sizeof(float) * (size_t)B * max_context, 256);
    int32_t *idx_local = reinterpret_cast<int32_t *>(ws + off);
    off += idx_bytes(B, k_sel);
    cudaError_t e = cudaMemsetAsync(hdr, 0, sizeof(WsHeader), st);
    if (e == cudaSuccess)
        e = run_decode_select(q_idx, q_scale, w, kidx_cache, kscale_cache, block_table, context_lens, num_pages,
                              max_pages_per_seq, page_size, B, max_context, H_I, k_sel, 0, scores, idx_local,
                              ws + off, hdr, st);
    if (e == cudaSuccess)
        e = launch_gather_selected(scores, max_context, idx_local, pos_base, B, k_sel, cand_pos_out, cand_score_out,
                                   hdr, st);
    return cuda_status(e);
}

dsa_status dsa_merge_selections(const int32_t *cand_pos, const float *cand_score, int64_t list_stride, int G,
                                int B, int k_sel, int32_t *idx_out, void *workspace, size_t ws_bytes, void *stream)
{
    if (!cand_pos || !cand_score || !idx_out || G <= 0 || B <= 0 || k_sel <= 0 || k_sel > 65536)
        return DSA_ERR_INVALID_ARG;
    if (list_stride == 0) list_stride = (int64_t)B * k_sel;
    if (list_stride < (int64_t)B * k_sel && G > 1) return DSA_ERR_INVALID_ARG;
    if ((int64_t)G * k_sel > INT32_MAX / 2 || B > 65535) return DSA_ERR_UNSUPPORTED;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DSA_ERR_WORKSPACE;
    if (ws_bytes < kWsHeader + align_up(merge_selections_ws_bytes(B, G, k_sel), 256)) return DSA_ERR_WORKSPACE;
    cudaStream_t st = as_stream(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    WsHeader *hdr = reinterpret_cast<WsHeader *>(ws);
    cudaError_t e = cudaMemsetAsync(hdr, 0, sizeof(WsHeader), st);
    if (e == cudaSuccess)
        e = launch_merge_selections(cand_pos, cand_score, list_stride, B, G, k_sel, idx_out, ws + kWsHeader, hdr,
                                    st);
    return cuda_status(e);
}

dsa_status dsa_decode_attend(const void *q, const void *k_cache, const float *k_cache_scale, const void *v_cache,
                             const float *v_cache_scale, const int32_t *block_table, const int32_t *context_lens,
                             const int32_t *pos_base, int64_t num_pages, int max_pages_per_seq, int page_size, int B,
                             int H_q, int d, int k_sel, const int32_t *idx, float sm_scale, void *out,
                             float *lse_out, void *workspace, size_t ws_bytes, void *stream)
{
    const bool kv8 = k_cache_scale != nullptr;
    if (kv8 != (v_cache_scale != nullptr)) return DSA_ERR_INVALID_ARG;
    if (kv8 && ((reinterpret_cast<uintptr_t>(k_cache_scale) & 3u) || (reinterpret_cast<uintptr_t>(v_cache_scale) & 3u)))
        return DSA_ERR_INVALID_ARG;
    if (!q || !k_cache || !v_cache || !block_table || !context_lens || !pos_base || !idx || !out || !lse_out)
        return DSA_ERR_INVALID_ARG;
    if (B <= 0 || num_pages <= 0 || max_pages_per_seq <= 0 || page_size <= 0 || H_q <= 0 || k_sel <= 0 ||
        k_sel > 65536 || !std::isfinite(sm_scale))
        return DSA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out)) return DSA_ERR_INVALID_ARG;
    if (d != 128 || page_size % 16 != 0 || B > 65535) return DSA_ERR_UNSUPPORTED;
    if (H_q > 128 && H_q % 128 != 0) return DSA_ERR_UNSUPPORTED;
    if (kv8 && !sparse_attn_tc_supported(H_q, d)) return DSA_ERR_UNSUPPORTED;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & 255u)) return DSA_ERR_WORKSPACE;
    const size_t part_bytes = sparse_attn_paged_part_bytes(B, H_q, d, sparse_attn_paged_splits(B, k_sel));
    if (ws_bytes < kWsHeader + idx_bytes(B, k_sel) + align_up(part_bytes, 256)) return DSA_ERR_WORKSPACE;

    cudaStream_t st = as_stream(stream);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    WsHeader *hdr = reinterpret_cast<WsHeader *>(ws);
    int32_t *idx_local = reinterpret_cast<int32_t *>(ws + kWsHeader);
    float *part = reinterpret_cast<float *>(ws + kWsHeader + idx_bytes(B, k_sel));
    cudaError_t e = cudaMemsetAsync(hdr, 0, sizeof(WsHeader), st);
    if (e == cudaSuccess) e = launch_local_idx(idx, pos_base, context_lens, B, k_sel, idx_local, st);
    if (e == cudaSuccess) {
        e = run_decode_attend(q, k_cache, v_cache, k_cache_scale, v_cache_scale, block_table, context_lens,
                              num_pages, max_pages_per_seq, page_size, B, H_q, d, k_sel, sm_scale, idx_local, out,
                              lse_out, part, hdr, st);
        if (e == cudaErrorNotSupported) return DSA_ERR_UNSUPPORTED;
    }
    return cuda_status(e);
}

dsa_status dsa_merge_partials(const void *part_out, int64_t out_stride, const float *part_lse, int64_t lse_stride,
                              int G, int B, int H_q, int d, void *out, float *lse_out, void *stream)
{
    if (!part_out || !part_lse || !out || G <= 0 || B <= 0 || H_q <= 0) return DSA_ERR_INVALID_ARG;
    if (!aligned16(part_out) || !aligned16(out) || (reinterpret_cast<uintptr_t>(part_lse) & 3u))
        return DSA_ERR_INVALID_ARG;
    if (d != 128 || (int64_t)ceil_div(H_q, 8) > 65535) return DSA_ERR_UNSUPPORTED;
    const int64_t n_out = (int64_t)B * H_q * d, n_lse = (int64_t)B * H_q;
    if (out_stride == 0) out_stride = n_out;
    if (lse_stride == 0) lse_stride = n_lse;
    if (G > 1 && (out_stride < n_out || lse_stride < n_lse)) return DSA_ERR_INVALID_ARG;
    if (out_stride % 8 != 0) return DSA_ERR_INVALID_ARG;          // keeps every partial 16-byte aligned
    return cuda_status(launch_merge_partials((const uint16_t *)part_out, out_stride, part_lse, lse_stride, G, B, H_q,
                                             d, (uint16_t *)out, lse_out, as_stream(stream)));
}

dsa_status dsa_quantize_e4m3(const void *x, dsa_dtype x_dtype, int64_t rows, int64_t cols,
                             uint8_t *codes_out, float *scale_out, void *stream)
{
    if (x_dtype != DSA_BF16 && x_dtype != DSA_F32) return DSA_ERR_UNSUPPORTED;
    if (rows < 0 || cols <= 0) return DSA_ERR_INVALID_ARG;
    if (rows == 0) return DSA_OK;
    if (!x || !codes_out || !scale_out || !aligned16(x) || (reinterpret_cast<uintptr_t>(codes_out) & 7u))
        return DSA_ERR_INVALID_ARG;
    if (cols % 8 != 0 || cols > 16384) return DSA_ERR_UNSUPPORTED;
    return cuda_status(launch_quantize_e4m3(x, x_dtype == DSA_BF16, rows, (int)cols, codes_out, scale_out,
                                            as_stream(stream)));
}

dsa_status dsa_cache_append(const void *kidx_new, dsa_dtype kidx_dtype, const void *k_new,
                            const void *v_new, const int32_t *seq_ids, const int32_t *positions,
                            int64_t N, int B, const int32_t *block_table, int max_pages_per_seq,
                            int64_t num_pages, int page_size, int d_I, int d, void *kidx_cache,
                            float *kscale_cache, void *k_cache, void *v_cache, uint32_t *status,
                            void *stream)
{
    if (kidx_dtype != DSA_BF16 && kidx_dtype != DSA_F32) return DSA_ERR_UNSUPPORTED;
    if (N < 0) return DSA_ERR_INVALID_ARG;
    if (N == 0) return DSA_OK;
    if (!kidx_new || !k_new || !v_new || !seq_ids || !positions || !block_table || !kidx_cache ||
        !kscale_cache || !k_cache || !v_cache)
        return DSA_ERR_INVALID_ARG;
    if (B <= 0 || max_pages_per_seq <= 0 || num_pages <= 0 || page_size <= 0 || d_I <= 0 || d <= 0)
        return DSA_ERR_INVALID_ARG;
    if (!aligned16(kidx_new) || !aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) ||
        !aligned16(v_cache) || (reinterpret_cast<uintptr_t>(kidx_cache) & 7u) ||
        (reinterpret_cast<uintptr_t>(status) & 3u))
        return DSA_ERR_INVALID_ARG;
    if (d_I % 8 != 0 || d_I > 256 || d % 8 != 0) return DSA_ERR_UNSUPPORTED;
    return cuda_status(launch_cache_append(kidx_new, kidx_dtype == DSA_BF16, (const uint16_t *)k_new,
                                           (const uint16_t *)v_new, seq_ids, positions, N, B, block_table,
                                           max_pages_per_seq, num_pages, page_size, d_I, d,
                                           (uint8_t *)kidx_cache, kscale_cache, k_cache, v_cache, nullptr,
                                           nullptr, status, as_stream(stream)));
}

dsa_status dsa_cache_append_kv8(const void *kidx_new, dsa_dtype kidx_dtype, const void *k_new,
                                const void *v_new, const int32_t *seq_ids, const int32_t *positions,
                                int64_t N, int B, const int32_t *block_table, int max_pages_per_seq,
                                int64_t num_pages, int page_size, int d_I, int d, void *kidx_cache,
                                float *kscale_cache, void *k_cache, float *k_cache_scale, void *v_cache,
                                float *v_cache_scale, uint32_t *status, void *stream)
{
    if (kidx_dtype != DSA_BF16 && kidx_dtype != DSA_F32) return DSA_ERR_UNSUPPORTED;
    if (N < 0) return DSA_ERR_INVALID_ARG;
    if (N == 0) return DSA_OK;
    if (!kidx_new || !k_new || !v_new || !seq_ids || !positions || !block_table || !kidx_cache ||
        !kscale_cache || !k_cache || !k_cache_scale || !v_cache || !v_cache_scale)
        return DSA_ERR_INVALID_ARG;
    if (B <= 0 || max_pages_per_seq <= 0 || num_pages <= 0 || page_size <= 0 || d_I <= 0 || d <= 0)
        return DSA_ERR_INVALID_ARG;
    if (!aligned16(kidx_new) || !aligned16(k_new) || !aligned16(v_new) ||
        (reinterpret_cast<uintptr_t>(kidx_cache) & 7u) || (reinterpret_cast<uintptr_t>(k_cache) & 7u) ||
        (reinterpret_cast<uintptr_t>(v_cache) & 7u) || (reinterpret_cast<uintptr_t>(status) & 3u))
        return DSA_ERR_INVALID_ARG;
    if (d_I % 8 != 0 || d_I > 256 || d % 8 != 0 || d > 256) return DSA_ERR_UNSUPPORTED;
    return cuda_status(launch_cache_append(kidx_new, kidx_dtype == DSA_BF16, (const uint16_t *)k_new,
                                           (const uint16_t *)v_new, seq_ids, positions, N, B, block_table,
                                           max_pages_per_seq, num_pages, page_size, d_I, d,
                                           (uint8_t *)kidx_cache, kscale_cache, k_cache, v_cache, k_cache_scale,
                                           v_cache_scale, status, as_stream(stream)));
}

dsa_status dsa_profile_enable(int on)
{
    profiler().on.store(on != 0);
    return DSA_OK;
}

dsa_status dsa_profile_read(double *ms_out, int64_t *launches_out)
{
    if (!ms_out) return DSA_ERR_INVALID_ARG;
    std::vector<ProfRec> recs;
    {
        std::lock_guard<std::mutex> g(profiler().mu);
        recs.swap(profiler().recs);
    }
    dsa_status s = DSA_OK;
    for (const ProfRec &r : recs) {
        float ms = 0.f;
        if (s == DSA_OK && (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess))
            s = DSA_ERR_CUDA;
        if (s == DSA_OK && r.stage >= 0 && r.stage < DSA_STAGE_COUNT) {
            ms_out[r.stage] += ms;
            if (launches_out) launches_out[r.stage] += 1;
        }
        cudaEventDestroy(r.a);
        cudaEventDestroy(r.b);
    }
    return s;
}

dsa_status dsa_stream_status(void *workspace, void *stream)
{
    if (!workspace) return DSA_ERR_INVALID_ARG;
    cudaStream_t st = as_stream(stream);
    WsHeader h;
    if (cudaMemcpyAsync(&h, workspace, sizeof(WsHeader), cudaMemcpyDeviceToHost, st) != cudaSuccess)
        return DSA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaMemsetAsync(workspace, 0, sizeof(WsHeader), st) != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
    return (dsa_status)h.status;
}

}  // extern "C"
