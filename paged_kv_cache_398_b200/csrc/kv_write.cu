// paged_kv_write: store each new token's key and value rows (every kv head)
// in its slot of the paged cache.  ("PagedAttention: How vLLM Serves AI Like
// an Operating System", "How It Works" / "The Magic: No Pre-allocation":
// blocks are filled as tokens arrive.)
//
// Pure data movement, bit-exact.  One thread moves one 16-byte chunk of a
// key row and the matching chunk of the value row; consecutive threads take
// consecutive chunks of a row, so both the read of k_new/v_new and the write
// into the cache tile are fully coalesced.
#include "common.cuh"

namespace {

__global__ void __launch_bounds__(256) kv_write_kernel(const uint4* __restrict__ k_new,
                                                       const uint4* __restrict__ v_new,
                                                       uint4* __restrict__ k_cache,
                                                       uint4* __restrict__ v_cache,
                                                       const int64_t* __restrict__ slot_mapping,
                                                       int64_t total_chunks, int32_t num_kv_heads,
                                                       int32_t row_chunks, int32_t block_size,
                                                       int64_t num_slots, int* status)
{
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total_chunks; i += stride) {
        const int64_t row = i / row_chunks;          // (token, head)
        const int32_t c = (int32_t)(i - row * row_chunks);
        const int64_t t = row / num_kv_heads;
        const int32_t h = (int32_t)(row - t * num_kv_heads);
        const int64_t slot = __ldg(slot_mapping + t);
        if (slot < 0) continue;
        if (slot >= num_slots) {
            if (c == 0 && h == 0) pkv::raise_flag(status, PKV_DEV_BAD_SLOT);
            continue;
        }
        const int64_t blk = slot / block_size;
        const int64_t off = slot - blk * block_size;
        const int64_t dst = ((blk * num_kv_heads + h) * block_size + off) * row_chunks + c;
        const uint4 kv = __ldg(k_new + i);
        const uint4 vv = __ldg(v_new + i);
        k_cache[dst] = kv;
        v_cache[dst] = vv;
    }
}

}  // namespace

extern "C" int paged_kv_write(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                              const int64_t* slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
                              int32_t head_dim, int32_t block_size, int32_t num_blocks,
                              int32_t dtype, void* stream)
{
    const pkv::NvtxRange nvtx("paged_kv_write");
    const size_t eb = pkv::dtype_bytes(dtype);
    if (eb == 0) return PKV_ERR_UNSUPPORTED;
    if (num_tokens < 0 || num_kv_heads < 1 || head_dim < 1 || block_size < 1 || num_blocks < 0)
        return PKV_ERR_INVALID_ARG;
    if (((size_t)head_dim * eb) % 16 != 0) return PKV_ERR_UNSUPPORTED;
    if (num_tokens == 0) return PKV_OK;
    if (!k_new || !v_new || !k_cache || !v_cache || !slot_mapping) return PKV_ERR_INVALID_ARG;
    if (!pkv::aligned16(k_new) || !pkv::aligned16(v_new) || !pkv::aligned16(k_cache) ||
        !pkv::aligned16(v_cache) || ((uintptr_t)slot_mapping & 7u))
        return PKV_ERR_INVALID_ARG;
    int* status = pkv::status_word_for_current_device();
    if (!status) return PKV_ERR_CUDA;

    const int32_t row_chunks = (int32_t)((size_t)head_dim * eb / 16);
    const int64_t total = (int64_t)num_tokens * num_kv_heads * row_chunks;
    const int threads = 256;
    int64_t blocks = (total + threads - 1) / threads;
    if (blocks > 148 * 32) blocks = 148 * 32;
    kv_write_kernel<<<(unsigned)blocks, threads, 0, (cudaStream_t)stream>>>(
        (const uint4*)k_new, (const uint4*)v_new, (uint4*)k_cache, (uint4*)v_cache, slot_mapping,
        total, num_kv_heads, row_chunks, block_size, (int64_t)num_blocks * block_size, status);
    return pkv::check_launch();
}
