// paged_attention_decode_shared: a decode step that reads the blocks a group
// of sequences shares once for the whole group.  ("PagedAttention: How vLLM
// Serves AI Like an Operating System", "Copy-on-Write: Sharing KV Cache",
// "Parallel Sampling" and "Prefix Caching": samples of one prompt hold the
// same physical blocks for the prompt.)
//
// Two launches on the caller's stream, the second staged behind the first by
// programmatic dependent launch:
//  1. decode_shared_tc_kernel, one CTA per (work item, kv head).  The host's
//     work list names every partition of both passes, longest first:
//     - group pass (partition p of [0, x) of group g): the tensor-core body
//       of decode_tc.cuh in its 16-row form, with the members' query heads
//       as its rows (kPlanGroup).  Each K/V tile of the shared positions
//       crosses HBM once for the whole group;
//     - own pass (partition p of [x, ctx) of sequence s): the one-query
//       form, fused with the new token's slot write (kPlanOwn).
//     One launch for both keeps the SMs busy across the passes, and the list
//     holds no partition that starts only to exit.
//  2. split-K reduce over the group's partitions followed by the
//     sequence's own (decode_reduce_kernel with shared_lens).
// The workspace has one record slot per row beyond ceil(max_ctx / PT),
// because a split at x can add one partition.
#include "decode_common.cuh"
#include "decode_tc.cuh"

namespace {

struct SharedArgs {
    void* out;
    const void* q;
    const void* k_new;
    const void* v_new;
    void* k_cache;
    void* v_cache;
    const int32_t* bt;
    int32_t mb;
    const int32_t* cl;
    int32_t S;
    int32_t max_ctx;
    const int32_t* groups;
    int32_t num_groups;
    const int32_t* shared_lens;
    const int32_t* work;
    int32_t num_work;
    int32_t Hq;
    int32_t Hkv;
    int32_t NB;
    int32_t block_size;
    int32_t part_tokens;
    float scale;
    void* ws;
    cudaStream_t stream;
    int* status;
    int* occupancy_out = nullptr;  // set: report the shared kernel's CTAs per SM, launch nothing
};

// Record slots per (sequence, query head) row.
inline int shared_record_slots(int max_ctx, int part_tokens) { return (max_ctx + part_tokens - 1) / part_tokens + 1; }

template <typename T, int D, int G, int B>
int launch_shared(const SharedArgs& a)
{
    using C = TcCfg<D>;
    const bool wide = a.part_tokens == kWidePartTokens;  // part_tokens_for: kPartTokens or kWidePartTokens
    if (!wide && a.part_tokens != kPartTokens) return PKV_ERR_UNSUPPORTED;
    const int smem = C::smem_bytes(0);  // neither pass stages new tokens' rows
    static std::atomic<bool> cfg_n[64] = {}, cfg_w[64] = {};
    if (a.occupancy_out) {
        return wide ? occupancy_of(decode_shared_tc_kernel<T, D, G, B, kWidePartTokens>, smem, cfg_w, a.occupancy_out)
                    : occupancy_of(decode_shared_tc_kernel<T, D, G, B, kPartTokens>, smem, cfg_n, a.occupancy_out);
    }
    const int slots = shared_record_slots(a.max_ctx, a.part_tokens);
    const int64_t qrows = (int64_t)a.S * a.Hq;
    float* ws_acc = static_cast<float*>(a.ws);
    float* ws_ml = ws_acc + (size_t)qrows * slots * D;
    const float scale_log2 = (float)((double)a.scale * 1.4426950408889634);
    const int64_t rows = (int64_t)a.NB * a.Hkv * B;
    if (rows > INT32_MAX) return PKV_ERR_UNSUPPORTED;  // TMA row coordinates are 32-bit
    CUtensorMap tm_k, tm_v;
    int rc;
    if ((rc = encode_cache_map<T>(&tm_k, a.k_cache, rows, D, B == 8 ? 8 : 16)) != PKV_OK) return rc;
    if ((rc = encode_cache_map<T>(&tm_v, a.v_cache, rows, D, B == 8 ? 8 : 16)) != PKV_OK) return rc;

    // 1. both passes
    auto run = [&](auto kernel, std::atomic<bool>* configured) {
        int r = allow_smem(kernel, smem, configured);
        if (r != PKV_OK) return r;
        cudaLaunchConfig_t cfg =
            pkv::pdl_config(dim3((unsigned)((int64_t)a.num_work * a.Hkv)), dim3(kWarps * 32), smem, a.stream);
        cudaLaunchAttribute attr[1];
        pkv::pdl_attribute(&cfg, attr);
        const cudaError_t e = cudaLaunchKernelEx(
            &cfg, kernel, tm_k, tm_v, static_cast<T*>(a.out), ws_acc, ws_ml, static_cast<const T*>(a.q),
            static_cast<const T*>(a.k_new), static_cast<const T*>(a.v_new), static_cast<T*>(a.k_cache),
            static_cast<T*>(a.v_cache), a.bt, a.mb, a.cl, a.max_ctx, a.Hq, a.Hkv, a.NB, scale_log2, slots, a.status,
            a.groups, a.num_groups, a.shared_lens, a.S, reinterpret_cast<const int2*>(a.work));
        if (e != cudaSuccess) {
            pkv::record_cuda_error(e);
            return PKV_ERR_CUDA;
        }
        return pkv::check_launch();
    };
    rc = wide ? run(decode_shared_tc_kernel<T, D, G, B, kWidePartTokens>, cfg_w)
              : run(decode_shared_tc_kernel<T, D, G, B, kPartTokens>, cfg_n);
    if (rc != PKV_OK) return rc;
    // 2. merge (always: a sequence split at x has records only)
    cudaLaunchConfig_t cfg = pkv::pdl_config(dim3((unsigned)((qrows + 3) / 4)), dim3(128), 0, a.stream);
    cudaLaunchAttribute attr[1];
    pkv::pdl_attribute(&cfg, attr);
    const cudaError_t e = cudaLaunchKernelEx(&cfg, decode_reduce_kernel<T, D>, static_cast<T*>(a.out),
                                             (const float*)ws_acc, (const float*)ws_ml, a.cl, a.S, 1, a.Hq, a.mb,
                                             B, a.max_ctx, a.part_tokens, slots, a.shared_lens);
    if (e != cudaSuccess) {
        pkv::record_cuda_error(e);
        return PKV_ERR_CUDA;
    }
    return pkv::check_launch();
}

template <typename T, int D, int G>
int shared_b(const SharedArgs& a)
{
    switch (a.block_size) {
        case 8: return launch_shared<T, D, G, 8>(a);
        case 16: return launch_shared<T, D, G, 16>(a);
        case 32: return launch_shared<T, D, G, 32>(a);
        default: return PKV_ERR_UNSUPPORTED;
    }
}

template <typename T, int D>
int shared_g(int G, const SharedArgs& a)
{
    switch (G) {
        case 1: return shared_b<T, D, 1>(a);
        case 2: return shared_b<T, D, 2>(a);
        case 4: return shared_b<T, D, 4>(a);
        case 8: return shared_b<T, D, 8>(a);
        default: return PKV_ERR_UNSUPPORTED;
    }
}

template <typename T>
int shared_d(int D, int G, const SharedArgs& a)
{
    if (D == 64) return shared_g<T, 64>(G, a);
    if (D == 128) return shared_g<T, 128>(G, a);
    return PKV_ERR_UNSUPPORTED;
}

}  // namespace

extern "C" size_t paged_attention_shared_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                                         int32_t max_context_len)
{
    if (num_seqs <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len <= 0) return 0;
    // sized for the shorter partition, which has the most slots
    const size_t slots = (size_t)shared_record_slots(max_context_len, kPartTokens);
    return (size_t)num_seqs * num_q_heads * slots * ((size_t)head_dim + 2) * sizeof(float);
}

extern "C" int paged_attention_decode_shared(void* out, const void* q, const void* k_new, const void* v_new,
                                             void* k_cache, void* v_cache, const int32_t* block_tables,
                                             int32_t max_blocks_per_seq, const int32_t* context_lens,
                                             int32_t num_seqs, int32_t max_context_len, const int32_t* groups,
                                             int32_t num_groups, const int32_t* shared_lens, const int32_t* work,
                                             int32_t num_work, int32_t work_part_tokens, int32_t num_q_heads,
                                             int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                             int32_t num_blocks, float scale, int32_t dtype, void* workspace,
                                             size_t workspace_bytes, void* stream)
{
    const pkv::NvtxRange nvtx("paged_attention_decode_shared");
    if (pkv::dtype_bytes(dtype) == 0) return PKV_ERR_UNSUPPORTED;
    if (num_seqs < 0 || num_q_heads < 1 || num_kv_heads < 1 || num_q_heads % num_kv_heads != 0 || num_blocks < 1 ||
        max_blocks_per_seq < 1 || !isfinite(scale) || (!k_new) != (!v_new) || num_groups < 0)
        return PKV_ERR_INVALID_ARG;
    if ((block_size != 8 && block_size != 16 && block_size != 32) || (head_dim != 64 && head_dim != 128))
        return PKV_ERR_UNSUPPORTED;
    const int G = num_q_heads / num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return PKV_ERR_UNSUPPORTED;
    if (dtype == PKV_F32) return PKV_ERR_UNSUPPORTED;  // the tensor-core kernel takes 16-bit inputs
    if (num_seqs == 0) return PKV_OK;
    if (max_context_len < 1 || num_seqs > 65535 || num_kv_heads > 65535 || num_groups > num_seqs)
        return PKV_ERR_INVALID_ARG;
    if (num_work < 1 || (int64_t)num_work * num_kv_heads > INT32_MAX) return PKV_ERR_INVALID_ARG;
    if (num_groups > 0 && (!groups || ((uintptr_t)groups & 3u))) return PKV_ERR_INVALID_ARG;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens || !shared_lens || !work ||
        !workspace || ((uintptr_t)work & 7u))
        return PKV_ERR_INVALID_ARG;
    if (!pkv::aligned16(q) || !pkv::aligned16(k_cache) || !pkv::aligned16(v_cache) ||
        ((uintptr_t)out % pkv::dtype_bytes(dtype)) || ((uintptr_t)block_tables & 3u) ||
        ((uintptr_t)context_lens & 3u) || ((uintptr_t)shared_lens & 3u) ||
        (k_new && (!pkv::aligned16(k_new) || !pkv::aligned16(v_new))))
        return PKV_ERR_INVALID_ARG;
    const size_t need = paged_attention_shared_workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len);
    if (workspace_bytes < need || ((uintptr_t)workspace & 255u)) return PKV_ERR_INVALID_ARG;
    int* status = pkv::status_word_for_current_device();
    if (!status) return PKV_ERR_CUDA;
    int part_tokens = kPartTokens;
    const int rc = part_tokens_for(dtype, num_seqs, num_kv_heads, max_context_len, &part_tokens);
    if (rc != PKV_OK) return rc;
    if (work_part_tokens != part_tokens) return PKV_ERR_INVALID_ARG;  // the list was made for another split
    const SharedArgs a{out,          q,           k_new,           v_new,          k_cache,
                       v_cache,      block_tables, max_blocks_per_seq, context_lens, num_seqs,
                       max_context_len, num_groups > 0 ? groups : nullptr, num_groups, shared_lens,
                       work,         num_work,    num_q_heads,     num_kv_heads,   num_blocks,
                       block_size,   part_tokens, scale,           workspace,      (cudaStream_t)stream,
                       status};
    if (dtype == PKV_F16) return shared_d<__half>(head_dim, G, a);
    return shared_d<__nv_bfloat16>(head_dim, G, a);
}

extern "C" int pkv_debug_shared_occupancy(int32_t dtype, int32_t head_dim, int32_t group, int32_t block_size,
                                          int32_t long_partitions, int32_t* ctas_per_sm)
{
    if (!ctas_per_sm) return PKV_ERR_INVALID_ARG;
    if ((block_size != 8 && block_size != 16 && block_size != 32) || (head_dim != 64 && head_dim != 128) ||
        (group != 1 && group != 2 && group != 4 && group != 8) || (dtype != PKV_F16 && dtype != PKV_BF16))
        return PKV_ERR_UNSUPPORTED;
    *ctas_per_sm = 0;
    SharedArgs a{};
    a.S = 1;
    a.max_ctx = long_partitions ? kWidePartTokens : kPartTokens;
    a.Hq = group;
    a.Hkv = 1;
    a.NB = 1;
    a.block_size = block_size;
    a.part_tokens = long_partitions ? kWidePartTokens : kPartTokens;
    a.scale = 1.0f;
    a.occupancy_out = ctas_per_sm;
    if (dtype == PKV_F16) return shared_d<__half>(head_dim, group, a);
    return shared_d<__nv_bfloat16>(head_dim, group, a);
}
