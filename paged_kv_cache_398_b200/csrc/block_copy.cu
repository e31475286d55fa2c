// block_copy: copy-on-write block copies.  For each (src, dst) pair, the
// whole physical block dst -- keys and values of every kv head -- becomes a
// copy of block src.  ("PagedAttention: How vLLM Serves AI Like an Operating
// System", "Copy-on-Write: Sharing KV Cache".)
//
// The pair list comes from the host allocator, so it is validated on the
// host and passed to the kernel by value (no device staging buffer, no
// allocation).  A launch carries up to kPairsPerLaunch pairs; grid.y walks
// the pairs, grid.z picks the key or the value cache, and each thread moves
// kUnroll 16-byte chunks with all loads issued before the stores.
#include <algorithm>
#include <vector>

#include "common.cuh"

namespace {

constexpr int kPairsPerLaunch = 1024;
constexpr int kThreads = 256;
constexpr int kUnroll = 4;

struct PairList {
    int2 p[kPairsPerLaunch];  // (src, dst); 8 KiB of kernel parameters
};

__global__ void __launch_bounds__(kThreads) block_copy_kernel(uint4* __restrict__ k_cache,
                                                              uint4* __restrict__ v_cache,
                                                              const __grid_constant__ PairList pairs,
                                                              int64_t block_chunks)
{
    uint4* cache = blockIdx.z == 0 ? k_cache : v_cache;
    const int2 pr = pairs.p[blockIdx.y];
    const uint4* src = cache + (int64_t)pr.x * block_chunks;
    uint4* dst = cache + (int64_t)pr.y * block_chunks;
    const int64_t base = (int64_t)blockIdx.x * (kThreads * kUnroll) + threadIdx.x;
    uint4 r[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * kThreads;
        if (i < block_chunks) r[u] = __ldg(src + i);
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
        const int64_t i = base + u * kThreads;
        if (i < block_chunks) dst[i] = r[u];
    }
}

}  // namespace

extern "C" int block_copy(void* k_cache, void* v_cache, const int64_t* pairs, int32_t num_pairs,
                          int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                          int32_t num_blocks, int32_t dtype, void* stream)
{
    const pkv::NvtxRange nvtx("block_copy");
    const size_t eb = pkv::dtype_bytes(dtype);
    if (eb == 0) return PKV_ERR_UNSUPPORTED;
    if (num_pairs < 0 || num_kv_heads < 1 || head_dim < 1 || block_size < 1 || num_blocks < 0)
        return PKV_ERR_INVALID_ARG;
    const size_t block_bytes = (size_t)num_kv_heads * block_size * head_dim * eb;
    if (block_bytes % 16 != 0) return PKV_ERR_UNSUPPORTED;
    if (num_pairs == 0) return PKV_OK;
    if (!k_cache || !v_cache || !pairs) return PKV_ERR_INVALID_ARG;
    if (!pkv::aligned16(k_cache) || !pkv::aligned16(v_cache)) return PKV_ERR_INVALID_ARG;

    // Reject every list whose result would depend on the copy order: a dst
    // named twice, or a dst that is also a src.  Sorting the ids keeps the
    // check's cost in the number of pairs, not the size of the pool.
    std::vector<int64_t> srcs, dsts;
    try {
        srcs.resize((size_t)num_pairs);
        dsts.resize((size_t)num_pairs);
    } catch (...) {  // no C++ exception leaves a C call
        return PKV_ERR_HOST_MEMORY;
    }
    for (int32_t i = 0; i < num_pairs; ++i) {
        const int64_t s = pairs[2 * i], d = pairs[2 * i + 1];
        if (s < 0 || s >= num_blocks || d < 0 || d >= num_blocks || s == d) return PKV_ERR_INVALID_ARG;
        srcs[i] = s;
        dsts[i] = d;
    }
    std::sort(srcs.begin(), srcs.end());
    std::sort(dsts.begin(), dsts.end());
    if (std::adjacent_find(dsts.begin(), dsts.end()) != dsts.end()) return PKV_ERR_INVALID_ARG;
    for (size_t i = 0, j = 0; i < dsts.size(); ++i) {  // merge walk: is any dst also a src?
        while (j < srcs.size() && srcs[j] < dsts[i]) ++j;
        if (j < srcs.size() && srcs[j] == dsts[i]) return PKV_ERR_INVALID_ARG;
    }

    const int64_t block_chunks = (int64_t)(block_bytes / 16);
    const unsigned gx = (unsigned)((block_chunks + kThreads * kUnroll - 1) / (kThreads * kUnroll));
    for (int32_t first = 0; first < num_pairs; first += kPairsPerLaunch) {
        const int32_t n = num_pairs - first < kPairsPerLaunch ? num_pairs - first : kPairsPerLaunch;
        PairList list;
        for (int32_t i = 0; i < n; ++i) {
            list.p[i] = make_int2((int)pairs[2 * (first + i)], (int)pairs[2 * (first + i) + 1]);
        }
        block_copy_kernel<<<dim3(gx, (unsigned)n, 2), kThreads, 0, (cudaStream_t)stream>>>(
            (uint4*)k_cache, (uint4*)v_cache, list, block_chunks);
        const int rc = pkv::check_launch();
        if (rc != PKV_OK) return rc;
    }
    return PKV_OK;
}
