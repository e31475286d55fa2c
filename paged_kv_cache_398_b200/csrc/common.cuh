// Internal device helpers shared by the library's kernels (not part of the ABI).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "paged_kv.h"

#include <nvtx3/nvToolsExt.h>  // header-only; inert unless a profiler injects NVTX

namespace pkv {

// NVTX range over one C-ABI call (host side: argument checks and launches),
// so profilers that trace NVTX (ncu --nvtx, nsys) can filter and label the
// library's kernels by entry point.  A few nanoseconds when none is attached.
struct NvtxRange {
    explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
    ~NvtxRange() { nvtxRangePop(); }
    NvtxRange(const NvtxRange&) = delete;
    NvtxRange& operator=(const NvtxRange&) = delete;
};

// ---- host side -----------------------------------------------------------

// Device address of this device's sticky status word (status.cu).  Returns
// nullptr and records the CUDA error if the address cannot be obtained.
int* status_word_for_current_device();

// Remember a CUDA error for pkv_last_cuda_error (thread-local).
void record_cuda_error(cudaError_t e);

// Check the launch that was just made.
inline int check_launch()
{
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) {
        record_cuda_error(e);
        return PKV_ERR_CUDA;
    }
    return PKV_OK;
}

inline bool aligned16(const void* p) { return ((uintptr_t)p & 15u) == 0; }

inline size_t dtype_bytes(int32_t dtype)
{
    return dtype == PKV_F32 ? 4 : (dtype == PKV_F16 || dtype == PKV_BF16) ? 2 : 0;
}

// Launch configuration whose kernel may be staged while the previous kernel
// on the stream finishes (programmatic dependent launch).  The kernel must
// call grid_dependency_wait() before it reads anything the previous kernel
// writes.  After a non-kernel stream operation the launch simply waits, as an
// ordinary one would.  The previous kernel releases it at the exit of its
// last CTA, or earlier where that kernel calls grid_dependency_launch(); the
// partition kernels call it only after their own grid_dependency_wait(), so
// whatever was written before them is complete, and visible at L2, by the
// time a kernel they release starts.
inline cudaLaunchConfig_t pdl_config(dim3 grid, dim3 block, size_t smem, cudaStream_t stream)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    return cfg;
}

// Under stream capture (CUDA graphs) the attribute is left out: capture
// does not accept it here, and an ordinary launch is always correct.
inline void pdl_attribute(cudaLaunchConfig_t* cfg, cudaLaunchAttribute* attr)
{
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(cfg->stream, &cs) != cudaSuccess) {
        cudaGetLastError();  // clear; fall back to an ordinary launch
        cs = cudaStreamCaptureStatusActive;
    }
    if (cs != cudaStreamCaptureStatusNone) {
        cfg->attrs = nullptr;
        cfg->numAttrs = 0;
        return;
    }
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg->attrs = attr;
    cfg->numAttrs = 1;
}

// ---- device side ---------------------------------------------------------

// Wait until the grids this one depends on have completed and their memory
// is visible (a no-op when the kernel was not launched as a dependent).
__device__ __forceinline__ void grid_dependency_wait()
{
    asm volatile("griddepcontrol.wait;" ::: "memory");
}

// Allow the next kernel on the stream, when it was launched as a dependent,
// to start before this grid ends (its grid_dependency_wait() still waits for
// this grid's completion).  Once every CTA has called it or exited, that
// kernel's CTAs can take SM slots this grid's tail leaves free.
__device__ __forceinline__ void grid_dependency_launch()
{
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// A read-only 32-bit global load kept where it is written (volatile asm): a
// kernel issues it ahead of the branches that decide whether the value is
// used, so independent loads travel together.
__device__ __forceinline__ int32_t ld_early(const int32_t* p)
{
    int32_t v;
    asm volatile("ld.global.nc.b32 %0, [%1];" : "=r"(v) : "l"(p));
    return v;
}

__device__ __forceinline__ void raise_flag(int* status, int flag)
{
    if (status) atomicOr(status, flag);
}

__device__ __forceinline__ uint32_t smem_addr(const void* p)
{
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

// Make mbarrier initialisation visible to the async (bulk copy) proxy.
__device__ __forceinline__ void fence_mbar_init()
{
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)),
                 "r"(bytes)
                 : "memory");
}

// 1-D bulk copy global -> this CTA's shared memory, completing on `bar`.
// Both addresses 16-byte aligned, bytes a multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                          uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1], %2, [%3], %4;" ::"r"(smem_addr(dst)),
        "l"(src), "r"(bytes), "r"(smem_addr(bar)), "l"(policy)
        : "memory");
}

// L2 policy for data read exactly once: evict first.
__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// Keep-in-L2 policy for data the next kernel reads back soon (split-K
// records), so the cache stream of the partition kernel does not push them
// out to DRAM first.
__device__ __forceinline__ uint64_t policy_evict_last()
{
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}

__device__ __forceinline__ void st_global_hint(float* ptr, float v, uint64_t policy)
{
    asm volatile("st.global.L2::cache_hint.f32 [%0], %1, %2;" ::"l"(ptr), "f"(v), "l"(policy) : "memory");
}

__device__ __forceinline__ void st_global_hint(float2* ptr, float2 v, uint64_t policy)
{
    asm volatile("st.global.L2::cache_hint.v2.f32 [%0], {%1, %2}, %3;" ::"l"(ptr), "f"(v.x), "f"(v.y), "l"(policy)
                 : "memory");
}

__device__ __forceinline__ void st_global_hint(float4* ptr, float4 v, uint64_t policy)
{
    asm volatile("st.global.L2::cache_hint.v4.f32 [%0], {%1, %2, %3, %4}, %5;" ::"l"(ptr), "f"(v.x), "f"(v.y),
                 "f"(v.z), "f"(v.w), "l"(policy)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_addr(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

__device__ __forceinline__ uint64_t global_ns()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Wait for phase `parity` of `bar` to complete, giving up after about
// `limit_ns` nanoseconds.  Returns false on timeout.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns)
{
    if (mbar_try_wait(bar, parity)) return true;
    uint64_t t0 = global_ns();
    for (;;) {
        if (mbar_try_wait(bar, parity)) return true;
        if (global_ns() - t0 > limit_ns) return false;
    }
}

// 2^x by the hardware approximation (PTX ex2.approx.ftz.f32: relative error
// about 2^-22; 2^-inf = +0).
__device__ __forceinline__ float fast_exp2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// ---- element conversion --------------------------------------------------

template <typename T>
struct Elem;

template <>
struct Elem<float> {
    // 16 bytes = 4 elements
    static constexpr int kVec = 4;
    __device__ __forceinline__ static void to_float(const uint4& v, float* f)
    {
        f[0] = __uint_as_float(v.x);
        f[1] = __uint_as_float(v.y);
        f[2] = __uint_as_float(v.z);
        f[3] = __uint_as_float(v.w);
    }
};

template <>
struct Elem<__half> {
    static constexpr int kVec = 8;
    __device__ __forceinline__ static void to_float(const uint4& v, float* f)
    {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            __half2 h = *reinterpret_cast<const __half2*>(&w[i]);
            float2 p = __half22float2(h);
            f[2 * i] = p.x;
            f[2 * i + 1] = p.y;
        }
    }
};

template <>
struct Elem<__nv_bfloat16> {
    static constexpr int kVec = 8;
    // A bfloat16 is the top half of a binary32: widening is a shift / mask.
    __device__ __forceinline__ static void to_float(const uint4& v, float* f)
    {
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            f[2 * i] = __uint_as_float(w[i] << 16);
            f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
        }
    }
};

__device__ __forceinline__ void store_out(float* p, float x) { *p = x; }
__device__ __forceinline__ void store_out(__half* p, float x) { *p = __float2half_rn(x); }
__device__ __forceinline__ void store_out(__nv_bfloat16* p, float x) { *p = __float2bfloat16_rn(x); }

}  // namespace pkv
