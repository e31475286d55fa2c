// Pieces of the decode path shared by its translation units (decode.cu,
// decode_shared.cu): launch constants, tile and sequence-range helpers, the
// split-K reduce kernel and the host-side launch helpers.  Internal: not part
// of the ABI.  Everything sits in an anonymous namespace, so each unit that
// includes it has its own copy.
#pragma once

#include <math.h>

#include <cudaTypedefs.h>

#include <atomic>
#include <mutex>
#include <type_traits>

#include "common.cuh"

namespace {


constexpr int kTile = 16;                          // tokens per compute tile
constexpr int kPartTokens = PKV_PARTITION_TOKENS;          // partition of an ordinary launch
constexpr int kLongPartTokens = PKV_PARTITION_TOKENS_LONG;  // 16-row launches that are not large batches
constexpr int kWidePartTokens = PKV_PARTITION_TOKENS_WIDE;  // large batches (fp16 / bf16)
constexpr int kPartTiles = kPartTokens / kTile;             // tiles per ordinary partition
constexpr int kMaxPartBlocks = kWidePartTokens / 8;         // blocks per partition, at most
constexpr int kWarps = 4;
constexpr int kStages = 2;
constexpr uint64_t kWaitLimitNs = 1000000000ull;

// What a tensor-core partition CTA computes (template parameter kPlan).
constexpr int kPlanNone = 0;   // an ordinary launch: partition p of sequence s
constexpr int kPlanGroup = 1;  // shared-prefix pass: partition p of a group's common positions [0, x)
constexpr int kPlanOwn = 2;    // a sequence's own positions [x, ctx) past the prefix its group shares

// A compute tile is 16 consecutive token positions of a sequence.  With
// block size B it is one block (B = 16), half of one (B = 32) or two
// consecutive ones (B = 8).  tile_rows gives the cache rows, in units of
// one token of one kv head (row = (block * Hkv + h) * B + offset), where the
// tile's first and second 8 tokens start.  For B = 16 and 32 the second half
// follows the first (r1 = r0 + 8).  nbp is the number of blocks this
// partition has, and a missing second block of a B = 8 tile reads the last
// one again (those positions are past the length and masked).
template <int B>
__device__ __forceinline__ void tile_rows(const int32_t* s_blk, int nbp, int tile, int num_kv_heads, int h,
                                          int& r0, int& r1)
{
    static_assert(B == 8 || B == 16 || B == 32, "block size 8, 16 or 32");
    if constexpr (B == 16) {
        r0 = (max(s_blk[tile], 0) * num_kv_heads + h) * 16;
        r1 = r0 + 8;
    } else if constexpr (B == 32) {
        r0 = (max(s_blk[tile / 2], 0) * num_kv_heads + h) * 32 + (tile % 2) * 16;
        r1 = r0 + 8;
    } else {
        const int bb = min(2 * tile + 1, nbp - 1);
        r0 = (max(s_blk[2 * tile], 0) * num_kv_heads + h) * 8;
        r1 = (max(s_blk[bb], 0) * num_kv_heads + h) * 8;
    }
}

struct SeqRange {
    int ctx;       // tokens attended (after clamping)
    int nparts;    // partitions of this sequence
    bool bad;      // context length < 1
};

// Checks and clamps a sequence's context length (ctx as loaded); the
// sequence splits into partitions of part_tokens tokens.
__device__ __forceinline__ SeqRange seq_range_of(int ctx, int mb, int block_size, int max_ctx, int part_tokens,
                                                 bool report, int* status)
{
    SeqRange r;
    int flag = 0;
    if (ctx < 1) {
        flag = 1;
        ctx = 0;
    }
    if ((int64_t)ctx > (int64_t)mb * block_size) {
        flag = 1;
        ctx = mb * block_size;
    }
    if (ctx > max_ctx) {
        flag = 1;
        ctx = max_ctx;
    }
    if (flag && report) pkv::raise_flag(status, PKV_DEV_BAD_CONTEXT);
    r.ctx = ctx;
    r.nparts = (ctx + part_tokens - 1) / part_tokens;
    r.bad = ctx < 1;
    return r;
}

__device__ __forceinline__ SeqRange seq_range(const int32_t* context_lens, int s, int mb, int block_size,
                                              int max_ctx, int part_tokens, bool report, int* status)
{
    return seq_range_of(__ldg(context_lens + s), mb, block_size, max_ctx, part_tokens, report, status);
}

// paged_attention_decode_shared: a sequence whose shared length x is a
// positive multiple of the block size below its context length has positions
// [0, x) attended by its group's pass and [x, ctx) by its own pass; any other
// x means the sequence is attended whole by its own pass (x = 0).
__device__ __forceinline__ int shared_split(int x, int ctx, int block_size)
{
    return x > 0 && x % block_size == 0 && x < ctx ? x : 0;
}

// Partitions of a sequence split at x: the group pass's ceil(x / pt) come
// first (records 0, 1, ...), then the sequence's own ceil((ctx - x) / pt).
__device__ __forceinline__ int split_parts(int x, int ctx, int part_tokens)
{
    return (x + part_tokens - 1) / part_tokens + (ctx - x + part_tokens - 1) / part_tokens;
}

// Merge the partitions of every (sequence, query head) that has more than
// one: out = sum_p acc_p 2^(m_p - M) / sum_p l_p 2^(m_p - M), M = max_p m_p,
// in partition order (shared_lens: see shared_split; null for an ordinary
// launch).  One warp per (sequence, query head); each lane owns
// head_dim / 32 consecutive outputs and issues the vector loads of up to 8
// partitions before it consumes them.
//
// The tensor-core partition kernels release this kernel early
// (grid_dependency_launch), so a warp decides whether its row needs a merge
// before it waits for them: the lengths are inputs of the call, complete
// before the partition kernel started, and are read at L2.  Rows that fit
// one partition (most of them in a batch of short contexts) then cost
// nothing after the partition grid ends.  CTA 0 waits in any case, so that
// this grid never completes before the partition grid does: a kernel that
// waits for this one also waits for that one.
template <typename T, int D>
__global__ void __launch_bounds__(128)
    decode_reduce_kernel(T* __restrict__ out, const float* __restrict__ ws_acc,
                         const float* __restrict__ ws_ml, const int32_t* __restrict__ context_lens,
                         int32_t num_seqs, int32_t q_len, int32_t num_q_heads, int32_t mb, int32_t block_size,
                         int32_t max_ctx, int32_t part_tokens, int32_t max_parts,
                         const int32_t* __restrict__ shared_lens)
{
    constexpr int kPer = D / 32;
    using Vec = typename std::conditional<kPer == 4, float4, float2>::type;
    constexpr int kUnroll = 8;
    if (blockIdx.x == 0) pkv::grid_dependency_wait();
    const int lane = threadIdx.x & 31;
    const int64_t row = (int64_t)blockIdx.x * 4 + (threadIdx.x >> 5);
    if (row >= (int64_t)num_seqs * q_len * num_q_heads) return;   // row = (s * q_len + j) * Hq + i
    const int s = (int)(row / ((int64_t)q_len * num_q_heads));
    const SeqRange sr = seq_range_of(__ldcg(context_lens + s), mb, block_size, max_ctx, part_tokens, false, nullptr);
    if (sr.bad || sr.ctx < q_len) return;   // zero rows: written
    // partitions: ceil(ctx / pt), or the group's and the sequence's own when
    // its positions are split (paged_attention_decode_shared)
    const int nparts =
        shared_lens ? split_parts(shared_split(__ldcg(shared_lens + s), sr.ctx, block_size), sr.ctx, part_tokens)
                    : sr.nparts;
    if (nparts <= 1) return;   // single partition: written by the partition kernel
    pkv::grid_dependency_wait();  // the partition kernel's results are visible after this
    const float* ml = ws_ml + row * max_parts * 2;
    const Vec* acc = reinterpret_cast<const Vec*>(ws_acc + row * max_parts * D) + lane;
    constexpr int kStride = D / kPer;  // Vec elements per partition

    if (nparts <= kUnroll) {
        // every record load of the row is issued before any is used: one
        // round trip to L2 (the same arithmetic, in the same order, as below)
        Vec a[kUnroll];
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            if (u < nparts) a[u] = acc[(int64_t)u * kStride];
        }
        const float m = lane < nparts ? ml[lane * 2] : -INFINITY;
        const float lv = lane < nparts ? ml[lane * 2 + 1] : 0.0f;
        float M = m;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
        M = fmaxf(-INFINITY, M);
        if (M == INFINITY) return;  // a poison record: see below
        float w = 0.0f, lw = 0.0f;
        if (lane < nparts) {
            w = exp2f(m - M);
            lw = lv * w;
        }
        float L = 0.0f;
        float o[kPer];
#pragma unroll
        for (int e = 0; e < kPer; ++e) o[e] = 0.0f;
#pragma unroll
        for (int u = 0; u < kUnroll; ++u) {
            if (u < nparts) {  // warp-uniform
                const float wj = __shfl_sync(0xffffffffu, w, u);
                L += __shfl_sync(0xffffffffu, lw, u);
                const float* av = reinterpret_cast<const float*>(&a[u]);
#pragma unroll
                for (int e = 0; e < kPer; ++e) o[e] = fmaf(av[e], wj, o[e]);
            }
        }
        const float inv = 1.0f / L;
#pragma unroll
        for (int e = 0; e < kPer; ++e) pkv::store_out(out + row * D + lane * kPer + e, o[e] * inv);
        return;
    }
    float M = -INFINITY;
    for (int p0 = 0; p0 < nparts; p0 += 32) {
        const int pp = p0 + lane;
        float m = pp < nparts ? ml[pp * 2] : -INFINITY;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        M = fmaxf(M, m);
    }
    // a poison record (m = +inf, written by the shared-prefix group pass for
    // a member whose table broke the plan's promise): leave the row unwritten
    if (M == INFINITY) return;
    float L = 0.0f;
    float o[kPer];
#pragma unroll
    for (int e = 0; e < kPer; ++e) o[e] = 0.0f;
    for (int p0 = 0; p0 < nparts; p0 += 32) {
        const int pp = p0 + lane;
        float w = 0.0f, lw = 0.0f;
        if (pp < nparts) {
            w = exp2f(ml[pp * 2] - M);
            lw = ml[pp * 2 + 1] * w;
        }
        const int n = min(32, nparts - p0);
        for (int j0 = 0; j0 < n; j0 += kUnroll) {
            Vec a[kUnroll];
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                if (j0 + u < n) a[u] = acc[(int64_t)(p0 + j0 + u) * kStride];
            }
#pragma unroll
            for (int u = 0; u < kUnroll; ++u) {
                if (j0 + u < n) {  // warp-uniform
                    const float wj = __shfl_sync(0xffffffffu, w, j0 + u);
                    L += __shfl_sync(0xffffffffu, lw, j0 + u);
                    const float* av = reinterpret_cast<const float*>(&a[u]);
#pragma unroll
                    for (int e = 0; e < kPer; ++e) o[e] = fmaf(av[e], wj, o[e]);
                }
            }
        }
    }
    const float inv = 1.0f / L;
#pragma unroll
    for (int e = 0; e < kPer; ++e) pkv::store_out(out + row * D + lane * kPer + e, o[e] * inv);
}

// cuTensorMapEncodeTiled, fetched from the driver through the runtime once.
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder()
{
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &qr) ==
                cudaSuccess &&
            qr == cudaDriverEntryPointSuccess) {
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        }
    });
    return fn;
}

// Tensor map over a cache viewed as [num_blocks * Hkv * block_size rows][D]
// 16-bit elements, in boxes of box_rows x 64 elements with the 128-byte
// swizzle (box_rows 16, or 8 for block size 8).
template <typename T>
int encode_cache_map(CUtensorMap* map, const void* cache, int64_t rows, int D, int box_rows)
{
    PFN_cuTensorMapEncodeTiled_v12000 enc = tensor_map_encoder();
    if (!enc) {
        pkv::record_cuda_error(cudaErrorNotSupported);
        return PKV_ERR_CUDA;
    }
    const cuuint64_t gdim[2] = {(cuuint64_t)D, (cuuint64_t)rows};
    const cuuint64_t gstride[1] = {(cuuint64_t)D * sizeof(T)};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estride[2] = {1, 1};
    const CUtensorMapDataType ty =
        sizeof(T) == 2 && std::is_same<T, __nv_bfloat16>::value ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                                                 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16;
    const CUresult r = enc(map, ty, 2, const_cast<void*>(cache), gdim, gstride, box, estride,
                           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        pkv::record_cuda_error(cudaErrorInvalidValue);
        return PKV_ERR_CUDA;
    }
    return PKV_OK;
}

// Once per device and kernel instantiation: allow more than 48 KiB of
// dynamic shared memory.
template <typename K>
int allow_smem(K kernel, int bytes, std::atomic<bool>* configured)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        pkv::record_cuda_error(e == cudaSuccess ? cudaErrorInvalidDevice : e);
        return PKV_ERR_CUDA;
    }
    if (!configured[dev].load(std::memory_order_acquire)) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
        if (e != cudaSuccess) {
            pkv::record_cuda_error(e);
            return PKV_ERR_CUDA;
        }
        configured[dev].store(true, std::memory_order_release);  // setting it twice is harmless
    }
    return PKV_OK;
}

// Resident CTAs per SM of `kernel` with `smem` bytes of dynamic shared memory.
template <typename K>
int occupancy_of(K kernel, int smem, std::atomic<bool>* configured, int* out)
{
    int rc = allow_smem(kernel, smem, configured);
    if (rc != PKV_OK) return rc;
    const cudaError_t e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(out, kernel, kWarps * 32, smem);
    if (e != cudaSuccess) {
        pkv::record_cuda_error(e);
        return PKV_ERR_CUDA;
    }
    return PKV_OK;
}

// Multiprocessor count of the current device, read once per device.
int sm_count(int* out)
{
    static std::atomic<int> cached[64] = {};  // 0: not read yet
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        pkv::record_cuda_error(e == cudaSuccess ? cudaErrorInvalidDevice : e);
        return PKV_ERR_CUDA;
    }
    if (cached[dev].load(std::memory_order_relaxed) == 0) {
        int n = 0;
        e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess || n < 1) {
            pkv::record_cuda_error(e == cudaSuccess ? cudaErrorInvalidValue : e);
            return PKV_ERR_CUDA;
        }
        cached[dev].store(n, std::memory_order_relaxed);
    }
    *out = cached[dev].load(std::memory_order_relaxed);
    return PKV_OK;
}

// A batch whose (sequence, kv head) pairs alone fill every SM several times
// over keeps the GPU busy with long partitions.
int large_batch(int32_t num_seqs, int32_t num_kv_heads, bool* out)
{
    int sms = 0;
    const int rc = sm_count(&sms);
    if (rc != PKV_OK) return rc;
    *out = (int64_t)num_seqs * num_kv_heads >= (int64_t)PKV_LONG_MIN_PAIRS_PER_SM * sms;
    return PKV_OK;
}

// Partition size of a launch.  A partition CTA has a fixed cost besides its
// stream of tiles: the prologue, the merge of its warps, its split-K record,
// and the CTAs past a shorter sequence's end that start only to exit.  On a
// large batch of long contexts, partitions of kWidePartTokens cut the CTA
// count and that cost, and contexts of at least PKV_LONG_MIN_CONTEXT tokens
// still split into several partitions.  Smaller or shorter batches keep
// kPartTokens for parallelism and a short tail.  The choice depends only on
// the launch shape, so it is the same for every call with that shape
// (bitwise-repeatable results).  fp32 keeps kPartTokens.
int part_tokens_for(int32_t dtype, int32_t num_seqs, int32_t num_kv_heads, int32_t max_context_len, int* out)
{
    *out = kPartTokens;
    if (dtype == PKV_F32 || max_context_len < PKV_LONG_MIN_CONTEXT) return PKV_OK;
    bool large = false;
    const int rc = large_batch(num_seqs, num_kv_heads, &large);
    if (rc != PKV_OK) return rc;
    if (large) *out = kWidePartTokens;
    return PKV_OK;
}

// The same for a launch of `rows` query rows per kv head (q_len x G).  More
// than 8 (the 16-row form): kWidePartTokens on a large batch of any context
// length, else kLongPartTokens (every partition ends with 16 rows of output
// or records, so even a small batch splits into fewer, longer partitions).
inline int mq_part_tokens_for(int32_t dtype, int32_t num_seqs, int32_t rows, int32_t num_kv_heads,
                              int32_t max_context_len, int* out)
{
    if (dtype != PKV_F32 && rows > 8) {
        bool large = false;
        const int rc = large_batch(num_seqs, num_kv_heads, &large);
        if (rc != PKV_OK) return rc;
        *out = large ? kWidePartTokens : kLongPartTokens;
        return PKV_OK;
    }
    return part_tokens_for(dtype, num_seqs, num_kv_heads, max_context_len, out);
}

}  // namespace
