// Allocation-free decode entry point.
//
// Some callers cannot give the library a workspace: a plugin whose host
// process has reserved all device memory in its own pool, or code on a
// latency-critical path where a device allocation (which can synchronise the
// device) is not allowed.  dsa_decode_noalloc runs the same kernels as
// dsa_decode, with the scratch in a fixed, file-scope device array.
//
// CUDA loads modules lazily, so the array is backed by device memory when its
// module is first needed on a device: the first call's address lookup below.
// That first call therefore reserves the 64 MiB (and can fail with
// DSA_ERR_CUDA when the device is full); later calls reserve nothing.  The
// reservation lasts as long as the context that loaded the module.
#include <cudaTypedefs.h>

#include <mutex>

#include "kernels.h"

namespace {

static __device__ __align__(256) unsigned char dsa_decode_scratch[DSA_DECODE_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 256;
std::mutex g_scratch_mu;
struct ScratchSlot {
    CUcontext ctx;       // the context the address belongs to
    void *addr;
};
ScratchSlot g_scratch[kMaxDevices];

PFN_cuCtxGetCurrent_v4000 ctx_get_current_fn()
{
    static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    });
    return fn;
}

// Device address of the scratch array on the current device.  The symbol's
// host-side name is not a device address, so the address is looked up with
// the device current and cached together with the context it belongs to: a
// device reset (or a released and recreated primary context) loads the
// module again, possibly at another address, and the lookup is redone.
dsa_status scratch_on_current_device(void **out)
{
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return DSA_ERR_UNSUPPORTED;
    PFN_cuCtxGetCurrent_v4000 get_ctx = ctx_get_current_fn();
    if (!get_ctx) return DSA_ERR_CUDA;
    CUcontext ctx = nullptr;
    if (get_ctx(&ctx) != CUDA_SUCCESS) return DSA_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    ScratchSlot &slot = g_scratch[dev];
    if (ctx == nullptr || slot.addr == nullptr || slot.ctx != ctx) {
        // (no context yet: the lookup makes the runtime create the device's primary one)
        void *p = nullptr;
        cudaError_t e = cudaGetSymbolAddress(&p, dsa_decode_scratch);
        if (e != cudaSuccess || p == nullptr) {
            (void)cudaGetLastError();        // reported through the return value, not left sticky
            return DSA_ERR_CUDA;
        }
        if (ctx == nullptr && (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr)) return DSA_ERR_CUDA;
        slot.ctx = ctx;
        slot.addr = p;
    }
    *out = slot.addr;
    return DSA_OK;
}

}  // namespace

extern "C" dsa_status dsa_decode_noalloc(
    const void *q_idx, const float *q_scale, const void *w, const void *q, const void *kidx_cache,
    const float *kscale_cache, const void *k_cache, const void *v_cache,
    const int32_t *block_table, const int32_t *context_lens, int64_t num_pages,
    int max_pages_per_seq, int page_size, int B, int64_t max_context, int H_I, int d_I, int H_q,
    int d, int k_sel, float sm_scale, void *out, float *lse_out, int32_t *idx_out,
    uint32_t *status_out, void *stream)
{
    const size_t need = dsa_decode_workspace_size(B, max_context, H_q, d, k_sel);
    if (need > (size_t)DSA_DECODE_NOALLOC_SCRATCH_BYTES) return DSA_ERR_WORKSPACE;
    void *scratch = nullptr;
    dsa_status s = scratch_on_current_device(&scratch);
    if (s != DSA_OK) return s;
    s = dsa_decode(q_idx, q_scale, w, q, kidx_cache, kscale_cache, k_cache, v_cache, block_table,
                   context_lens, num_pages, max_pages_per_seq, page_size, B, max_context, H_I,
                   d_I, H_q, d, k_sel, sm_scale, out, lse_out, idx_out, scratch,
                   (size_t)DSA_DECODE_NOALLOC_SCRATCH_BYTES, stream);
    if (s == DSA_OK && status_out) {
        // the device status word sits at the start of the scratch
        if (cudaMemcpyAsync(status_out, scratch, sizeof(uint32_t), cudaMemcpyDeviceToDevice,
                            reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
            return DSA_ERR_CUDA;
    }
    return s;
}
