// Shared device helpers of the DSA library (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "dsa.h"

namespace dsa {

constexpr size_t kWsHeader = 256;   // bytes reserved at the start of every workspace

// First 256 bytes of a workspace.  `status` holds a dsa_status recorded on
// the device; `detail` a free-form code (e.g. the offending row) for it.
struct WsHeader {
    unsigned int status;
    unsigned int detail;
    unsigned int pad[62];
};

__host__ __device__ inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
__host__ __device__ inline size_t align_up(size_t a, size_t b) { return (a + b - 1) / b * b; }

__device__ __forceinline__ void record_error(WsHeader *h, dsa_status s, unsigned int detail)
{
    if (h) {
        if (atomicCAS(&h->status, (unsigned int)DSA_OK, (unsigned int)s) == DSA_OK)
            h->detail = detail;
    }
}

// Programmatic dependent launch.  A kernel launched with launch_chained() may
// be scheduled while the kernel before it on the stream is still running; it
// calls grid_dep_wait() before it reads what that kernel wrote or writes
// anything that kernel might still read (the wait returns once the earlier
// grid has completed and its writes are visible; without the launch
// attribute it returns at once).  grid_dep_trigger() lets the next chained
// kernel be scheduled before this one ends.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void grid_dep_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// Launches kernel<<<grid, block, smem, st>>>(args...) so that it may start
// while the previous kernel on `st` finishes (see grid_dep_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                                  cudaStream_t st, Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// Sampled key positions of the fused prefill selection's threshold estimate:
// sample j sits at position j * S + (hash(j) mod S) (S a power of two), one
// pseudo-random point of each block of S positions, so that no periodic
// pattern in the keys lines up with the samples.  The hash is the 32-bit
// finaliser of MurmurHash3 (Appleby), applied to j.
__host__ __device__ inline uint32_t sample_hash(uint32_t j)
{
    j ^= j >> 16;
    j *= 0x85ebca6bu;
    j ^= j >> 13;
    j *= 0xc2b2ae35u;
    j ^= j >> 16;
    return j;
}
__host__ __device__ inline int64_t sample_pos(int64_t j, int S)
{
    return j * S + (int64_t)(sample_hash((uint32_t)j) & (uint32_t)(S - 1));
}
// Number of samples at positions < n (positions increase with j).
__host__ __device__ inline int64_t sample_count(int64_t n, int S)
{
    if (n <= 0) return 0;
    const int64_t j = (n - 1) / S;
    return j + ((int64_t)(sample_hash((uint32_t)j) & (uint32_t)(S - 1)) <= n - 1 - j * S ? 1 : 0);
}

__device__ __forceinline__ float bf16_to_f32(uint16_t b)
{
    return __uint_as_float(((uint32_t)b) << 16);
}

// Order-preserving map of a (non-NaN) fp32 value to uint32; -0 maps like +0.
__device__ __forceinline__ uint32_t float_key(float f)
{
    uint32_t u = __float_as_uint(f);
    if (u == 0x80000000u) u = 0u;
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint32_t smem_u32(const void *p)
{
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void cp_async_16(void *smem, const void *gmem, bool valid)
{
    // Copies 16 bytes, or writes 16 zero bytes when !valid (src-size 0).
    unsigned n = valid ? 16u : 0u;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n"
                 :: "r"(smem_u32(smem)), "l"(gmem), "r"(n) : "memory");
}
// Arrive on `bar` (asynchronously) once every cp.async this thread issued so
// far has completed; counts toward the barrier's expected arrivals.
__device__ __forceinline__ void cp_async_arrive_noinc(uint64_t *bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];\n" :: "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" :: "n"(N) : "memory"); }

__device__ __forceinline__ void ldmatrix_x4(uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3,
                                            const void *smem)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(smem_u32(smem)));
}
__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t &r0, uint32_t &r1, uint32_t &r2,
                                                  uint32_t &r3, const void *smem)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(smem_u32(smem)));
}

// D += A(16x32 e4m3, row) * B(32x8 e4m3, col), fp32 accumulate.
__device__ __forceinline__ void mma_e4m3_16832(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// D += A(16x16 bf16, row) * B(16x8 bf16, col), fp32 accumulate.
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1,
                                               uint32_t a2, uint32_t a3, uint32_t b0, uint32_t b1)
{
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
        "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi)
{
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

}  // namespace dsa
