// swap_blocks_out / swap_blocks_in: move whole physical blocks (keys and
// values, every kv head) between the device cache and host memory, so a
// preempted sequence can give its blocks back and later resume.
// ("PagedAttention: How vLLM Serves AI Like an Operating System", "vLLM
// Architecture": the scheduler preempts low-priority requests by swapping
// their blocks to CPU memory.)
//
// The host buffers are pinned (page-locked) and mapped into the device's
// address space, so one kernel launch gathers (out) or scatters (in) any
// list of blocks over the host link: no staging buffer, no allocation, one
// launch per 1024 blocks.  Host slot i holds the block named by ids[i].
// Block ids are checked on the host and passed by value.  Consecutive
// threads move consecutive 16-byte chunks of a block, and each thread issues
// its loads before its stores.
#include <algorithm>
#include <vector>

#include "common.cuh"

namespace {

constexpr int kIdsPerLaunch = 1024;
constexpr int kThreads = 256;
constexpr int kUnroll = 4;

struct IdList {
    int32_t id[kIdsPerLaunch];
};

// to_host = true: dev block ids[i] -> host slot i; false: host slot i -> dev block ids[i]
__global__ void __launch_bounds__(kThreads) swap_kernel(uint4* __restrict__ k_dev, uint4* __restrict__ v_dev,
                                                        uint4* __restrict__ k_host, uint4* __restrict__ v_host,
                                                        const __grid_constant__ IdList ids, int32_t first_slot,
                                                        int64_t block_chunks, bool to_host)
{
    uint4* dev = blockIdx.z == 0 ? k_dev : v_dev;
    uint4* host = blockIdx.z == 0 ? k_host : v_host;
    uint4* d = dev + (int64_t)ids.id[blockIdx.y] * block_chunks;
    uint4* hst = host + (int64_t)(first_slot + blockIdx.y) * block_chunks;
    const uint4* src = to_host ? d : hst;
    uint4* dst = to_host ? hst : d;
    const int64_t base = (int64_t)blockIdx.x * (kThreads * kUnroll) + threadIdx.x;
    uint4 r[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * kThreads;
        if (i < block_chunks) r[u] = src[i];
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * kThreads;
        if (i < block_chunks) dst[i] = r[u];
    }
}

// Device address of a pinned, mapped host buffer, or null.
void* mapped_device_pointer(const void* host)
{
    cudaPointerAttributes attr;
    if (cudaPointerGetAttributes(&attr, host) != cudaSuccess) {
        cudaGetLastError();  // clear the non-sticky error
        return nullptr;
    }
    if (attr.type != cudaMemoryTypeHost || !attr.devicePointer) return nullptr;
    return attr.devicePointer;
}

int swap_blocks(void* k_cache, void* v_cache, const int64_t* block_ids, int32_t n, void* host_k, void* host_v,
                int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks, int32_t dtype,
                void* stream, bool to_host)
{
    const size_t eb = pkv::dtype_bytes(dtype);
    if (eb == 0) return PKV_ERR_UNSUPPORTED;
    if (n < 0 || num_kv_heads < 1 || head_dim < 1 || block_size < 1 || num_blocks < 0) return PKV_ERR_INVALID_ARG;
    const size_t block_bytes = (size_t)num_kv_heads * block_size * head_dim * eb;
    if (block_bytes % 16 != 0) return PKV_ERR_UNSUPPORTED;
    if (n == 0) return PKV_OK;
    if (!k_cache || !v_cache || !block_ids || !host_k || !host_v) return PKV_ERR_INVALID_ARG;
    if (!pkv::aligned16(k_cache) || !pkv::aligned16(v_cache) || !pkv::aligned16(host_k) || !pkv::aligned16(host_v))
        return PKV_ERR_INVALID_ARG;
    for (int32_t i = 0; i < n; ++i) {
        if (block_ids[i] < 0 || block_ids[i] >= num_blocks) return PKV_ERR_INVALID_ARG;
    }
    if (!to_host) {  // two host slots into one block: order-dependent.  Sorted, in time of n, not of the pool.
        std::vector<int64_t> ids;
        try {
            ids.assign(block_ids, block_ids + n);
        } catch (...) {  // no C++ exception leaves a C call
            return PKV_ERR_HOST_MEMORY;
        }
        std::sort(ids.begin(), ids.end());
        if (std::adjacent_find(ids.begin(), ids.end()) != ids.end()) return PKV_ERR_INVALID_ARG;
    }
    void* dk = mapped_device_pointer(host_k);
    void* dv = mapped_device_pointer(host_v);
    if (!dk || !dv) return PKV_ERR_INVALID_ARG;  // not pinned, device-mapped host memory
    const int64_t block_chunks = (int64_t)(block_bytes / 16);
    const unsigned gx = (unsigned)((block_chunks + kThreads * kUnroll - 1) / (kThreads * kUnroll));
    for (int32_t first = 0; first < n; first += kIdsPerLaunch) {
        const int32_t m = n - first < kIdsPerLaunch ? n - first : kIdsPerLaunch;
        IdList list;
        for (int32_t i = 0; i < m; ++i) list.id[i] = (int32_t)block_ids[first + i];
        swap_kernel<<<dim3(gx, (unsigned)m, 2), kThreads, 0, (cudaStream_t)stream>>>(
            (uint4*)k_cache, (uint4*)v_cache, (uint4*)dk, (uint4*)dv, list, first, block_chunks, to_host);
        const int rc = pkv::check_launch();
        if (rc != PKV_OK) return rc;
    }
    return PKV_OK;
}

}  // namespace

extern "C" int swap_blocks_out(const void* k_cache, const void* v_cache, const int64_t* block_ids, int32_t n,
                               void* host_k, void* host_v, int32_t num_kv_heads, int32_t head_dim,
                               int32_t block_size, int32_t num_blocks, int32_t dtype, void* stream)
{
    const pkv::NvtxRange nvtx("swap_blocks_out");
    return swap_blocks(const_cast<void*>(k_cache), const_cast<void*>(v_cache), block_ids, n, host_k, host_v,
                       num_kv_heads, head_dim, block_size, num_blocks, dtype, stream, true);
}

extern "C" int swap_blocks_in(void* k_cache, void* v_cache, const int64_t* block_ids, int32_t n, const void* host_k,
                              const void* host_v, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                              int32_t num_blocks, int32_t dtype, void* stream)
{
    const pkv::NvtxRange nvtx("swap_blocks_in");
    return swap_blocks(k_cache, v_cache, block_ids, n, const_cast<void*>(host_k), const_cast<void*>(host_v),
                       num_kv_heads, head_dim, block_size, num_blocks, dtype, stream, false);
}
