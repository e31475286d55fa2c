// paged_attention_decode: one decode step of attention whose keys and values
// sit in fixed-size, non-contiguous physical blocks reached through
// per-sequence block tables.  ("PagedAttention: How vLLM Serves AI Like an
// Operating System", "How It Works" and "PagedAttention Memory Layout"; the
// result is ordinary softmax attention -- "Throughput Impact: The Numbers":
// no approximations.)
//
// Design (B200, sm_100a):
//  * Work unit = (partition p, kv head h, sequence s): one CTA.  A partition
//    is PKV_PARTITION_TOKENS tokens, or PKV_PARTITION_TOKENS_WIDE on large
//    batches of long contexts; launches of more than 8 query rows per kv
//    head take PKV_PARTITION_TOKENS_WIDE on large batches and
//    PKV_PARTITION_TOKENS_LONG otherwise (mq_part_tokens_for).  The G = Hq / Hkv query
//    heads that share kv head h are computed together, so each K/V block is
//    read from HBM once per kv head, not once per query head.
//  * fp16 / bf16 run the tensor-core kernel of decode_tc.cuh (tiled TMA,
//    mma.sync).  This file holds the fp32 kernel, the launcher and the entry
//    points; the split-K reduce and the launch helpers are in
//    decode_common.cuh, shared with decode_shared.cu.
//  * fp32: each (block, kv head) tile is one contiguous block_size x
//    head_dim run in the cache layout, so it is fetched with 1-D bulk copies
//    (K and V; TMA engine, no tensor map, no multicast) into shared memory,
//    completing on an mbarrier.  Every warp owns a ring of kStages tile
//    pairs and walks its share of the partition's blocks (round-robin) with
//    its own pipeline.  All waits are bounded (about 1 s) and report a
//    timeout through the status word instead of hanging.
//  * fp32 Q.K: each lane holds 16 bytes of the head dimension of one token
//    for all G query heads (fp32, pre-scaled by scale * log2 e).  The partial
//    dot products of a whole block are summed across the lanes of a token
//    by a transposed shuffle reduction: each level halves the values a
//    lane keeps.
//  * Online softmax in fp32 (exp2), masked to the sequence's length, then
//    P.V with fp32 accumulators.  Warps are merged in shared memory.  A
//    sequence longer than one partition writes (max, sum, partial output)
//    to the workspace, and a second kernel merges its partitions in a fixed
//    order.
//  * Partitioning depends only on the context length and the launch shape,
//    so the result is bit-identical under any permutation of the physical
//    placement.
#include "decode_common.cuh"

namespace {

template <typename T, int D, int G>
struct Cfg {
    static constexpr int kVec = 16 / (int)sizeof(T);   // elements per 16 bytes
    static constexpr int kLpt = D / kVec;              // lanes per token row
    static constexpr int kTpi = 32 / kLpt;             // tokens per warp iteration
    static constexpr int kIters = kTile / kTpi;        // iterations per tile
    static constexpr int kTileBytes = kTile * D * (int)sizeof(T);
    static constexpr int kNv = kIters * G;             // partial dots per lane per tile
    static constexpr int kItems = kTile * G;           // scores per tile
    static constexpr int kItemsPerLane = (kItems + 31) / 32;
    static_assert(kLpt >= 1 && kLpt <= 32 && 32 % kLpt == 0, "bad row split");
    static_assert(32 % G == 0, "G must divide the warp");
    // shared memory carve-up (bytes)
    static constexpr int kTilesBytes = kWarps * kStages * 2 * kTileBytes;
    static constexpr int kBarOff = kTilesBytes;
    static constexpr int kScoreOff = kBarOff + kWarps * kStages * 8;
    static constexpr int kBlkOff = kScoreOff + kWarps * kItems * 4;
    static constexpr int kSmemBytes = kBlkOff + kMaxPartBlocks * 4;
    // the cross-warp merge reuses the tile area
    static constexpr int kMergeBytes = kWarps * G * (D + 2) * 4;
    static_assert(kMergeBytes <= kTilesBytes, "merge area does not fit");
};

// Transposed butterfly: sum N values across the lane bits MASK, MASK/2, .., 1.
// While N >= 2 each level keeps half of the values (the half selected by the
// lane's bit) and adds the partner's copy of that half; once one value is
// left the remaining levels are plain butterflies.
template <int N, int MASK>
__device__ __forceinline__ void treduce(float* v, int lane)
{
    if constexpr (MASK > 0) {
        if constexpr (N >= 2) {
            constexpr int H = N / 2;
            const bool up = (lane & MASK) != 0;
#pragma unroll
            for (int k = 0; k < H; ++k) {
                const float send = up ? v[k] : v[k + H];
                const float keep = up ? v[k + H] : v[k];
                v[k] = keep + __shfl_xor_sync(0xffffffffu, send, MASK);
            }
            treduce<H, MASK / 2>(v, lane);
        } else {
            v[0] += __shfl_xor_sync(0xffffffffu, v[0], MASK);
            treduce<1, MASK / 2>(v, lane);
        }
    }
}

// Index (into the original N values) of the first value a lane keeps.
template <int N, int MASK>
__device__ __forceinline__ int treduce_base(int lane)
{
    if constexpr (MASK > 0 && N >= 2) {
        return ((lane & MASK) ? N / 2 : 0) + treduce_base<N / 2, MASK / 2>(lane);
    } else {
        return 0;
    }
}

// Lane bits on which values are duplicated (plain butterfly levels).
template <int N, int MASK>
__host__ __device__ constexpr int treduce_dup_mask()
{
    if constexpr (MASK == 0) {
        return 0;
    } else if constexpr (N >= 2) {
        return treduce_dup_mask<N / 2, MASK / 2>();
    } else {
        return MASK | treduce_dup_mask<1, MASK / 2>();
    }
}

// Lane 0 of a warp: fetch the K and V rows of one tile (16 tokens x D) into
// the tile pair at `dst` (K then V), completing on `bar`.
template <int kTileBytes, typename T>
__device__ __forceinline__ void issue_tile_pair(uint8_t* dst, uint64_t* bar, const T* k_cache,
                                                const T* v_cache, int64_t row0, int64_t row1, bool split,
                                                int D, uint64_t policy)
{
    // order this warp's earlier generic reads of the tiles before the async writes
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    pkv::mbar_arrive_expect_tx(bar, 2 * kTileBytes);
    if (!split) {
        pkv::bulk_load(dst, k_cache + row0 * D, kTileBytes, bar, policy);
        pkv::bulk_load(dst + kTileBytes, v_cache + row0 * D, kTileBytes, bar, policy);
    } else {
        constexpr int kHalf = kTileBytes / 2;
        pkv::bulk_load(dst, k_cache + row0 * D, kHalf, bar, policy);
        pkv::bulk_load(dst + kHalf, k_cache + row1 * D, kHalf, bar, policy);
        pkv::bulk_load(dst + kTileBytes, v_cache + row0 * D, kHalf, bar, policy);
        pkv::bulk_load(dst + kTileBytes + kHalf, v_cache + row1 * D, kHalf, bar, policy);
    }
}

template <typename T, int D, int G, int B>
__global__ void __launch_bounds__(kWarps * 32)
    decode_partition_kernel(T* __restrict__ out, float* __restrict__ ws_acc, float* __restrict__ ws_ml,
                            const T* __restrict__ q, const T* __restrict__ k_cache,
                            const T* __restrict__ v_cache, const int32_t* __restrict__ block_tables,
                            int32_t mb, const int32_t* __restrict__ context_lens, int32_t max_ctx,
                            int32_t num_q_heads, int32_t num_kv_heads, int32_t num_blocks,
                            float scale_log2, int32_t max_parts, int* status)
{
    using C = Cfg<T, D, G>;
    extern __shared__ __align__(128) uint8_t smem[];
    pkv::grid_dependency_wait();  // inputs written by the previous kernel are visible after this
    const int p = blockIdx.x, h = blockIdx.y, s = blockIdx.z;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    const SeqRange sr =
        seq_range(context_lens, s, mb, B, max_ctx, kPartTokens, p == 0 && h == 0 && threadIdx.x == 0, status);
    if (sr.bad) {
        // nothing to attend to: a zero row (flagged above)
        if (p == 0) {
            for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
                pkv::store_out(out + ((int64_t)s * num_q_heads + h * G) * D + i, 0.0f);
            }
        }
        return;
    }
    if (p >= sr.nparts) return;

    constexpr int kPartBlocks = kPartTokens / B;
    const int nblk_seq = (sr.ctx + B - 1) / B;
    const int blk0 = p * kPartBlocks;
    const int nbp = min(kPartBlocks, nblk_seq - blk0);                 // blocks of this partition
    const int nb = min(kPartTiles, (sr.ctx - p * kPartTokens + kTile - 1) / kTile);  // its tiles

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff) + warp * kStages;
    float* s_sc = reinterpret_cast<float*>(smem + C::kScoreOff) + warp * C::kItems;
    int32_t* s_blk = reinterpret_cast<int32_t*>(smem + C::kBlkOff);
    uint8_t* my_tiles = smem + warp * (kStages * 2 * C::kTileBytes);

    for (int i = threadIdx.x; i < nbp; i += blockDim.x) {
        int b = __ldg(block_tables + (int64_t)s * mb + blk0 + i);
        if (b < 0 || b >= num_blocks) {
            pkv::raise_flag(status, PKV_DEV_BAD_BLOCK_ID);
            b = 0;
        }
        s_blk[i] = b;
    }
    if (lane == 0) {
#pragma unroll
        for (int st = 0; st < kStages; ++st) pkv::mbar_init(&bars[st], 1);
        pkv::fence_mbar_init();
    }
    __syncthreads();

    // this warp's tiles: warp + k * kWarps, k < nw
    const int nw = nb > warp ? (nb - warp + kWarps - 1) / kWarps : 0;
    uint64_t policy = 0;
    if (lane == 0) policy = pkv::policy_evict_first();

    if (lane == 0) {
        for (int k = 0; k < nw && k < kStages; ++k) {
            int r0, r1;
            tile_rows<B>(s_blk, nbp, warp + k * kWarps, num_kv_heads, h, r0, r1);
            issue_tile_pair<C::kTileBytes>(my_tiles + (k % kStages) * 2 * C::kTileBytes, &bars[k % kStages],
                                           k_cache, v_cache, r0, r1, B == 8, D, policy);
        }
    }

    // this lane's slice of the G query vectors, in the log2 domain
    const int c = lane % C::kLpt;
    const int tsub = lane / C::kLpt;
    float qf[G][C::kVec];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        const uint4 raw = *reinterpret_cast<const uint4*>(
            q + ((int64_t)s * num_q_heads + h * G + g) * D + c * C::kVec);
        pkv::Elem<T>::to_float(raw, qf[g]);
#pragma unroll
        for (int e = 0; e < C::kVec; ++e) qf[g][e] *= scale_log2;
    }

    // which (token, head) each reduced value stands for
    constexpr int kR = C::kNv >= C::kLpt ? C::kNv / C::kLpt : 1;
    const int jbase = treduce_base<C::kNv, C::kLpt / 2>(lane);
    constexpr int kDup = treduce_dup_mask<C::kNv, C::kLpt / 2>();
    const bool owner = (lane & kDup) == 0;
    const int g_lane = lane % G;  // the head of this lane's softmax items

    float m_run[G];
    float acc[G][C::kVec];
#pragma unroll
    for (int g = 0; g < G; ++g) {
        m_run[g] = -INFINITY;
#pragma unroll
        for (int e = 0; e < C::kVec; ++e) acc[g][e] = 0.0f;
    }
    float l_part = 0.0f;   // this lane's share of the softmax sum of head g_lane
    bool timed_out = false;
    int consumed = 0;

    for (int k = 0; k < nw; ++k) {
        const int st = k % kStages;
        if (!pkv::mbar_wait(&bars[st], (k / kStages) & 1, kWaitLimitNs)) {
            timed_out = true;
            break;
        }
        const T* sk = reinterpret_cast<const T*>(my_tiles + st * 2 * C::kTileBytes);
        const T* sv = reinterpret_cast<const T*>(my_tiles + st * 2 * C::kTileBytes + C::kTileBytes);
        const int valid = min(kTile, sr.ctx - (p * kPartTokens + (warp + k * kWarps) * kTile));

        // ---- Q.K for the block's 16 tokens -----------------------------
        float part[C::kNv];
#pragma unroll
        for (int it = 0; it < C::kIters; ++it) {
            const int t = it * C::kTpi + tsub;
            const uint4 raw = *reinterpret_cast<const uint4*>(sk + t * D + c * C::kVec);
            float kf[C::kVec];
            pkv::Elem<T>::to_float(raw, kf);
#pragma unroll
            for (int g = 0; g < G; ++g) {
                float d0 = 0.0f;
#pragma unroll
                for (int e = 0; e < C::kVec; ++e) d0 = fmaf(qf[g][e], kf[e], d0);
                part[it * G + g] = d0;
            }
        }
        treduce<C::kNv, C::kLpt / 2>(part, lane);
        if (owner) {
#pragma unroll
            for (int r = 0; r < kR; ++r) {
                const int j = jbase + r;
                const int t = (j / G) * C::kTpi + tsub;
                s_sc[t * G + (j % G)] = part[r];
            }
        }
        __syncwarp();

        // ---- online softmax ----------------------------------------------
        float x[C::kItemsPerLane];
        float mx = -INFINITY;
#pragma unroll
        for (int u = 0; u < C::kItemsPerLane; ++u) {
            const int idx = lane + 32 * u;
            x[u] = -INFINITY;
            if (idx < C::kItems && idx / G < valid) x[u] = s_sc[idx];
            mx = fmaxf(mx, x[u]);
        }
#pragma unroll
        for (int o = G; o < 32; o <<= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        float alpha[G];
        bool rescale = false;
#pragma unroll
        for (int g = 0; g < G; ++g) {
            const float bm = __shfl_sync(0xffffffffu, mx, g);
            const float mn = fmaxf(m_run[g], bm);
            alpha[g] = exp2f(m_run[g] - mn);
            rescale |= (mn != m_run[g]);
            m_run[g] = mn;
        }
        float m_mine = m_run[0], a_mine = alpha[0];  // values of head g_lane (no local memory)
#pragma unroll
        for (int g = 1; g < G; ++g) {
            if (g == g_lane) {
                m_mine = m_run[g];
                a_mine = alpha[g];
            }
        }
        float psum = 0.0f;
#pragma unroll
        for (int u = 0; u < C::kItemsPerLane; ++u) {
            const int idx = lane + 32 * u;
            const float pr = exp2f(x[u] - m_mine);
            if (idx < C::kItems) s_sc[idx] = pr;
            psum += pr;
        }
        l_part = l_part * a_mine + psum;
        if (rescale) {
#pragma unroll
            for (int g = 0; g < G; ++g)
#pragma unroll
                for (int e = 0; e < C::kVec; ++e) acc[g][e] *= alpha[g];
        }
        __syncwarp();

        // ---- P.V ----------------------------------------------------------
#pragma unroll
        for (int it = 0; it < C::kIters; ++it) {
            const int t = it * C::kTpi + tsub;
            if (t < valid) {
                const uint4 raw = *reinterpret_cast<const uint4*>(sv + t * D + c * C::kVec);
                float vf[C::kVec];
                pkv::Elem<T>::to_float(raw, vf);
                float pg[G];
#pragma unroll
                for (int g = 0; g < G; ++g) pg[g] = s_sc[t * G + g];
#pragma unroll
                for (int g = 0; g < G; ++g)
#pragma unroll
                    for (int e = 0; e < C::kVec; ++e) acc[g][e] = fmaf(pg[g], vf[e], acc[g][e]);
            }
        }
        __syncwarp();
        ++consumed;
        if (lane == 0 && k + kStages < nw) {
            int r0, r1;
            tile_rows<B>(s_blk, nbp, warp + (k + kStages) * kWarps, num_kv_heads, h, r0, r1);
            issue_tile_pair<C::kTileBytes>(my_tiles + st * 2 * C::kTileBytes, &bars[st], k_cache, v_cache, r0, r1,
                                           B == 8, D, policy);
        }
    }

    if (timed_out) {
        if (lane == 0) pkv::raise_flag(status, PKV_DEV_WAIT_TIMEOUT);
        // let the copies still in flight land before the smem is reused
        for (int k = consumed; k < nw && k < consumed + kStages; ++k) {
            pkv::mbar_wait(&bars[k % kStages], (k / kStages) & 1, kWaitLimitNs);
        }
    }

    // ---- merge the lanes of this warp ------------------------------------
#pragma unroll
    for (int o = G; o < 32; o <<= 1) l_part += __shfl_xor_sync(0xffffffffu, l_part, o);
#pragma unroll
    for (int o = C::kLpt; o < 32; o <<= 1)
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < C::kVec; ++e) acc[g][e] += __shfl_xor_sync(0xffffffffu, acc[g][e], o);

    __syncthreads();  // every warp is done with its tiles: reuse them for the merge
    float* mg = reinterpret_cast<float*>(smem);  // [kWarps][G][D + 2]: m, l, acc[D]
    float* mine = mg + warp * G * (D + 2);
#pragma unroll
    for (int g = 0; g < G; ++g) {
        if (lane == g) {
            mine[g * (D + 2)] = m_run[g];
            mine[g * (D + 2) + 1] = l_part;  // lane g holds the full sum of head g
        }
    }
    if (tsub == 0) {
#pragma unroll
        for (int g = 0; g < G; ++g)
#pragma unroll
            for (int e = 0; e < C::kVec; ++e) mine[g * (D + 2) + 2 + c * C::kVec + e] = acc[g][e];
    }
    __syncthreads();

    const int hq0 = h * G;
    for (int i = threadIdx.x; i < G * D; i += blockDim.x) {
        const int g = i / D, d = i % D;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, mg[(w * G + g) * (D + 2)]);
        float L = 0.0f, O = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float* rec = mg + (w * G + g) * (D + 2);
            const float wgt = exp2f(rec[0] - M);  // empty warp: m = -inf -> 0
            L = fmaf(rec[1], wgt, L);
            O = fmaf(rec[2 + d], wgt, O);
        }
        const int64_t row = (int64_t)s * num_q_heads + hq0 + g;
        if (sr.nparts == 1) {
            pkv::store_out(out + row * D + d, O / L);
        } else {
            ws_acc[(row * max_parts + p) * D + d] = O;
            if (d == 0) {
                ws_ml[(row * max_parts + p) * 2] = M;
                ws_ml[(row * max_parts + p) * 2 + 1] = L;
            }
        }
    }
}

}  // namespace

#include "decode_tc.cuh"

namespace {

struct DecodeArgs {
    void* out;
    const void* q;
    const void* k_new;  // fused slot write: [S][q_len][Hkv][D], or null
    const void* v_new;
    void* k_cache;
    void* v_cache;
    const int32_t* bt;
    int32_t mb;
    const int32_t* cl;
    int32_t S;
    int32_t q_len;
    int32_t max_ctx;
    int32_t Hq;
    int32_t Hkv;
    int32_t NB;
    int32_t block_size;
    int32_t part_tokens;  // mq_part_tokens_for
    float scale;
    void* ws;
    cudaStream_t stream;
    int* status;
    int* occupancy_out = nullptr;  // set: report the partition kernel's CTAs per SM, launch nothing
};


template <typename T, int D, int G, int B>
int launch(const DecodeArgs& a)
{
    const int max_parts = (a.max_ctx + a.part_tokens - 1) / a.part_tokens;
    const int64_t qrows = (int64_t)a.S * a.q_len * a.Hq;  // (sequence, new token, query head) rows
    float* ws_acc = static_cast<float*>(a.ws);
    float* ws_ml = ws_acc ? ws_acc + (size_t)qrows * max_parts * D : nullptr;
    const float scale_log2 = (float)((double)a.scale * 1.4426950408889634);
    dim3 grid((unsigned)max_parts, (unsigned)a.Hkv, (unsigned)a.S);
    int rc;
    cudaError_t launch_err = cudaSuccess;
    if constexpr (sizeof(T) == 2) {
        // fp16 / bf16: tensor-core kernel fed by tiled TMA; one instantiation
        // per (multi-query, partition size), each setting its shared-memory
        // limit once per device
        using C = TcCfg<D>;
        // the 8-column form takes kPartTokens or kWidePartTokens, the 16-row form
        // (past 8 rows) kLongPartTokens or kWidePartTokens (mq_part_tokens_for)
        const bool mq = a.q_len * G > 8, wide = a.part_tokens == kWidePartTokens;
        if (!wide && a.part_tokens != (mq ? kLongPartTokens : kPartTokens)) return PKV_ERR_UNSUPPORTED;
        const int smem = C::smem_bytes(mq ? 16 : 0);  // staging room for several new tokens' rows
        static std::atomic<bool> cfg_s[64] = {}, cfg_sw[64] = {}, cfg_m[64] = {}, cfg_mw[64] = {};
        auto with_kernel = [&](auto&& f) {
            if (!mq && !wide) return f(decode_partition_tc_kernel<T, D, G, false, B, kPartTokens>, cfg_s);
            if (!mq) return f(decode_partition_tc_kernel<T, D, G, false, B, kWidePartTokens>, cfg_sw);
            if (!wide) return f(decode_partition_tc_kernel<T, D, G, true, B, kLongPartTokens>, cfg_m);
            return f(decode_partition_tc_kernel<T, D, G, true, B, kWidePartTokens>, cfg_mw);
        };
        if (a.occupancy_out) {
            return with_kernel(
                [&](auto kernel, std::atomic<bool>* configured) { return occupancy_of(kernel, smem, configured, a.occupancy_out); });
        }
        const int64_t rows = (int64_t)a.NB * a.Hkv * B;
        if (rows > INT32_MAX) return PKV_ERR_UNSUPPORTED;  // TMA row coordinates are 32-bit
        CUtensorMap tm_k, tm_v;
        if ((rc = encode_cache_map<T>(&tm_k, a.k_cache, rows, D, B == 8 ? 8 : 16)) != PKV_OK) return rc;
        if ((rc = encode_cache_map<T>(&tm_v, a.v_cache, rows, D, B == 8 ? 8 : 16)) != PKV_OK) return rc;
        cudaLaunchConfig_t cfg = pkv::pdl_config(grid, dim3(kWarps * 32), smem, a.stream);
        cudaLaunchAttribute attr[1];
        pkv::pdl_attribute(&cfg, attr);
        auto args = [&](auto kernel) {
            return cudaLaunchKernelEx(&cfg, kernel, tm_k, tm_v, static_cast<T*>(a.out), ws_acc, ws_ml,
                                      static_cast<const T*>(a.q), static_cast<const T*>(a.k_new),
                                      static_cast<const T*>(a.v_new), static_cast<T*>(a.k_cache),
                                      static_cast<T*>(a.v_cache), a.bt, a.mb, a.cl, a.max_ctx, a.q_len, a.Hq, a.Hkv,
                                      a.NB, scale_log2, max_parts, a.status);
        };
        rc = with_kernel([&](auto kernel, std::atomic<bool>* configured) {
            const int r = allow_smem(kernel, smem, configured);
            if (r == PKV_OK) launch_err = args(kernel);
            return r;
        });
        if (rc != PKV_OK) return rc;
    } else {
        // fp32: CUDA-core kernel fed by 1-D bulk copies (one query, no fused write)
        if (a.q_len != 1 || a.k_new || a.part_tokens != kPartTokens) return PKV_ERR_UNSUPPORTED;
        using C = Cfg<T, D, G>;
        static std::atomic<bool> configured[64] = {};
        if (a.occupancy_out)
            return occupancy_of(decode_partition_kernel<T, D, G, B>, C::kSmemBytes, configured, a.occupancy_out);
        rc = allow_smem(decode_partition_kernel<T, D, G, B>, C::kSmemBytes, configured);
        if (rc != PKV_OK) return rc;
        cudaLaunchConfig_t cfg = pkv::pdl_config(grid, dim3(kWarps * 32), C::kSmemBytes, a.stream);
        cudaLaunchAttribute attr[1];
        pkv::pdl_attribute(&cfg, attr);
        launch_err = cudaLaunchKernelEx(&cfg, decode_partition_kernel<T, D, G, B>, static_cast<T*>(a.out), ws_acc,
                                        ws_ml, static_cast<const T*>(a.q), static_cast<const T*>(a.k_cache),
                                        static_cast<const T*>(a.v_cache), a.bt, a.mb, a.cl, a.max_ctx, a.Hq,
                                        a.Hkv, a.NB, scale_log2, max_parts, a.status);
    }
    if (launch_err != cudaSuccess) {
        pkv::record_cuda_error(launch_err);
        return PKV_ERR_CUDA;
    }
    rc = pkv::check_launch();
    if (rc != PKV_OK || max_parts == 1) return rc;
    cudaLaunchConfig_t cfg = pkv::pdl_config(dim3((unsigned)((qrows + 3) / 4)), dim3(128), 0, a.stream);
    cudaLaunchAttribute attr[1];
    pkv::pdl_attribute(&cfg, attr);
    const cudaError_t reduce_err =
        cudaLaunchKernelEx(&cfg, decode_reduce_kernel<T, D>, static_cast<T*>(a.out), (const float*)ws_acc,
                           (const float*)ws_ml, a.cl, a.S, a.q_len, a.Hq, a.mb, B, a.max_ctx, a.part_tokens,
                           max_parts, nullptr);
    if (reduce_err != cudaSuccess) {
        pkv::record_cuda_error(reduce_err);
        return PKV_ERR_CUDA;
    }
    return pkv::check_launch();
}

template <typename T, int D, int G>
int dispatch_b(const DecodeArgs& a)
{
    switch (a.block_size) {
        case 8: return launch<T, D, G, 8>(a);
        case 16: return launch<T, D, G, 16>(a);
        case 32: return launch<T, D, G, 32>(a);
        default: return PKV_ERR_UNSUPPORTED;
    }
}

template <typename T, int D>
int dispatch_g(int G, const DecodeArgs& a)
{
    switch (G) {
        case 1: return dispatch_b<T, D, 1>(a);
        case 2: return dispatch_b<T, D, 2>(a);
        case 4: return dispatch_b<T, D, 4>(a);
        case 8: return dispatch_b<T, D, 8>(a);
        default: return PKV_ERR_UNSUPPORTED;
    }
}

template <typename T>
int dispatch_d(int D, int G, const DecodeArgs& a)
{
    if (D == 64) return dispatch_g<T, 64>(G, a);
    if (D == 128) return dispatch_g<T, 128>(G, a);
    return PKV_ERR_UNSUPPORTED;
}

// Host-side checks of a decode call's shape and pointers (everything but
// the workspace), shared by the decode entry points.  PKV_OK with
// num_seqs == 0 means there is nothing to launch.
int decode_check(const void* out, const void* q, const void* k_new, const void* v_new, const void* k_cache,
                 const void* v_cache, const int32_t* block_tables, int32_t max_blocks_per_seq,
                 const int32_t* context_lens, int32_t num_seqs, int32_t q_len, int32_t max_context_len,
                 int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                 int32_t num_blocks, float scale, int32_t dtype)
{
    if (pkv::dtype_bytes(dtype) == 0) return PKV_ERR_UNSUPPORTED;
    if (num_seqs < 0 || q_len < 1 || num_q_heads < 1 || num_kv_heads < 1 || num_q_heads % num_kv_heads != 0 ||
        num_blocks < 1 || max_blocks_per_seq < 1 || !isfinite(scale) || (!k_new) != (!v_new))
        return PKV_ERR_INVALID_ARG;
    if ((block_size != 8 && block_size != 16 && block_size != 32) || (head_dim != 64 && head_dim != 128))
        return PKV_ERR_UNSUPPORTED;
    const int G = num_q_heads / num_kv_heads;
    if (G != 1 && G != 2 && G != 4 && G != 8) return PKV_ERR_UNSUPPORTED;
    if (q_len * G > 16) return PKV_ERR_UNSUPPORTED;  // the query rows fill one 16-row tensor-core operand
    if (dtype == PKV_F32 && (q_len != 1 || k_new)) return PKV_ERR_UNSUPPORTED;
    if (num_seqs == 0) return PKV_OK;
    if (max_context_len < 1 || num_seqs > 65535 || num_kv_heads > 65535) return PKV_ERR_INVALID_ARG;
    if (!out || !q || !k_cache || !v_cache || !block_tables || !context_lens) return PKV_ERR_INVALID_ARG;
    if (!pkv::aligned16(q) || !pkv::aligned16(k_cache) || !pkv::aligned16(v_cache) ||
        ((uintptr_t)out % pkv::dtype_bytes(dtype)) || ((uintptr_t)block_tables & 3u) ||
        ((uintptr_t)context_lens & 3u) || (k_new && (!pkv::aligned16(k_new) || !pkv::aligned16(v_new))))
        return PKV_ERR_INVALID_ARG;
    return PKV_OK;
}

// Host-side checks and dispatch shared by the decode entry points.
int decode_entry(void* out, const void* q, const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                 const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                 int32_t num_seqs, int32_t q_len, int32_t max_context_len, int32_t num_q_heads,
                 int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale,
                 int32_t dtype, void* workspace, size_t workspace_bytes, void* stream)
{
    const int checked = decode_check(out, q, k_new, v_new, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                     context_lens, num_seqs, q_len, max_context_len, num_q_heads, num_kv_heads,
                                     head_dim, block_size, num_blocks, scale, dtype);
    if (checked != PKV_OK || num_seqs == 0) return checked;
    const int G = num_q_heads / num_kv_heads;
    const size_t need =
        paged_attention_mq_workspace_bytes(num_seqs, q_len, num_q_heads, head_dim, max_context_len);
    if (need > 0 && (!workspace || workspace_bytes < need || ((uintptr_t)workspace & 255u)))
        return PKV_ERR_INVALID_ARG;
    int* status = pkv::status_word_for_current_device();
    if (!status) return PKV_ERR_CUDA;
    int part_tokens = kPartTokens;
    const int rc = mq_part_tokens_for(dtype, num_seqs, q_len * G, num_kv_heads, max_context_len, &part_tokens);
    if (rc != PKV_OK) return rc;
    const DecodeArgs a{out,           q,        k_new,          v_new,        k_cache,      v_cache,
                       block_tables,  max_blocks_per_seq,       context_lens, num_seqs,     q_len,
                       max_context_len, num_q_heads, num_kv_heads, num_blocks, block_size, part_tokens, scale,
                       workspace,     (cudaStream_t)stream,     status};
    switch (dtype) {
        case PKV_F32: return dispatch_d<float>(head_dim, G, a);
        case PKV_F16: return dispatch_d<__half>(head_dim, G, a);
        default: return dispatch_d<__nv_bfloat16>(head_dim, G, a);
    }
}

}  // namespace

extern "C" size_t paged_attention_mq_workspace_bytes(int32_t num_seqs, int32_t q_len, int32_t num_q_heads,
                                                     int32_t head_dim, int32_t max_context_len)
{
    if (num_seqs <= 0 || q_len <= 0 || num_q_heads <= 0 || head_dim <= 0 || max_context_len <= 0) return 0;
    const size_t parts = ((size_t)max_context_len + kPartTokens - 1) / kPartTokens;
    if (parts <= 1) return 0;
    return (size_t)num_seqs * q_len * num_q_heads * parts * ((size_t)head_dim + 2) * sizeof(float);
}

extern "C" int32_t paged_attention_mq_partition_tokens(int32_t num_seqs, int32_t q_len, int32_t num_q_heads,
                                                       int32_t num_kv_heads, int32_t max_context_len, int32_t dtype)
{
    if (num_seqs < 0 || q_len < 1 || num_q_heads < 1 || num_kv_heads < 1 || num_q_heads % num_kv_heads != 0 ||
        max_context_len < 1)
        return PKV_ERR_INVALID_ARG;
    if (dtype != PKV_F32 && dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
    int part_tokens = kPartTokens;
    const int rc = mq_part_tokens_for(dtype, num_seqs, q_len * (num_q_heads / num_kv_heads), num_kv_heads,
                                      max_context_len, &part_tokens);
    return rc != PKV_OK ? rc : part_tokens;
}

extern "C" int32_t paged_attention_partition_tokens(int32_t num_seqs, int32_t num_kv_heads, int32_t max_context_len,
                                                    int32_t dtype)
{
    if (num_seqs < 0 || num_kv_heads < 1 || max_context_len < 1) return PKV_ERR_INVALID_ARG;
    if (dtype != PKV_F32 && dtype != PKV_F16 && dtype != PKV_BF16) return PKV_ERR_UNSUPPORTED;
    int part_tokens = kPartTokens;
    const int rc = part_tokens_for(dtype, num_seqs, num_kv_heads, max_context_len, &part_tokens);
    return rc != PKV_OK ? rc : part_tokens;
}

extern "C" int pkv_debug_decode_occupancy(int32_t dtype, int32_t head_dim, int32_t group, int32_t q_len,
                                          int32_t block_size, int32_t long_partitions, int32_t* ctas_per_sm)
{
    if (!ctas_per_sm || q_len < 1) return PKV_ERR_INVALID_ARG;
    if ((block_size != 8 && block_size != 16 && block_size != 32) || (head_dim != 64 && head_dim != 128) ||
        (group != 1 && group != 2 && group != 4 && group != 8) || q_len * group > 16 ||
        (dtype != PKV_F32 && dtype != PKV_F16 && dtype != PKV_BF16) ||
        (dtype == PKV_F32 && (q_len != 1 || long_partitions)))
        return PKV_ERR_UNSUPPORTED;
    *ctas_per_sm = 0;
    DecodeArgs a{};
    a.S = 1;
    a.q_len = q_len;
    a.part_tokens = long_partitions ? kWidePartTokens : q_len * group > 8 ? kLongPartTokens : kPartTokens;
    a.max_ctx = a.part_tokens;
    a.Hq = group;
    a.Hkv = 1;
    a.NB = 1;
    a.block_size = block_size;
    a.scale = 1.0f;
    a.occupancy_out = ctas_per_sm;
    switch (dtype) {
        case PKV_F32: return dispatch_d<float>(head_dim, group, a);
        case PKV_F16: return dispatch_d<__half>(head_dim, group, a);
        default: return dispatch_d<__nv_bfloat16>(head_dim, group, a);
    }
}

extern "C" size_t paged_attention_workspace_bytes(int32_t num_seqs, int32_t num_q_heads,
                                                  int32_t head_dim, int32_t max_context_len)
{
    return paged_attention_mq_workspace_bytes(num_seqs, 1, num_q_heads, head_dim, max_context_len);
}

extern "C" int paged_attention_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                                      const int32_t* block_tables, int32_t max_blocks_per_seq,
                                      const int32_t* context_lens, int32_t num_seqs,
                                      int32_t max_context_len, int32_t num_q_heads, int32_t num_kv_heads,
                                      int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale,
                                      int32_t dtype, void* workspace, size_t workspace_bytes, void* stream)
{
    const pkv::NvtxRange nvtx("paged_attention_decode");
    // read-only caches: the const is cast away only for the shared launcher
    return decode_entry(out, q, nullptr, nullptr, const_cast<void*>(k_cache), const_cast<void*>(v_cache),
                        block_tables, max_blocks_per_seq, context_lens, num_seqs, 1, max_context_len,
                        num_q_heads, num_kv_heads, head_dim, block_size, num_blocks, scale, dtype, workspace,
                        workspace_bytes, stream);
}

extern "C" int paged_attention_decode_mq(void* out, const void* q, const void* k_new, const void* v_new,
                                         void* k_cache, void* v_cache, const int32_t* block_tables,
                                         int32_t max_blocks_per_seq, const int32_t* context_lens,
                                         int32_t num_seqs, int32_t q_len, int32_t max_context_len,
                                         int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                         int32_t block_size, int32_t num_blocks, float scale, int32_t dtype,
                                         void* workspace, size_t workspace_bytes, void* stream)
{
    const pkv::NvtxRange nvtx("paged_attention_decode_mq");
    return decode_entry(out, q, k_new, v_new, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                        num_seqs, q_len, max_context_len, num_q_heads, num_kv_heads, head_dim, block_size,
                        num_blocks, scale, dtype, workspace, workspace_bytes, stream);
}

// ---------------------------------------------------------------------------
// Allocation-free variant.  Callers that cannot allocate device memory when
// they decode get the split-K scratch from this fixed array instead of a
// workspace of their own.  See paged_attention_decode_noalloc in paged_kv.h.
// ---------------------------------------------------------------------------
static __device__ __align__(256) unsigned char g_noalloc_scratch[PKV_NOALLOC_SCRATCH_BYTES];

namespace {

constexpr int kNoallocMaxDevices = 64;
void* g_noalloc_ptr[kNoallocMaxDevices] = {};
std::mutex g_noalloc_mu;

// Device address of the array on the current device, resolved once per device.
// In host code `g_noalloc_scratch` names a host-side stand-in, not device memory,
// so it must never be handed to a kernel directly.
int noalloc_scratch(void** out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kNoallocMaxDevices) {
        pkv::record_cuda_error(e == cudaSuccess ? cudaErrorInvalidDevice : e);
        return PKV_ERR_CUDA;
    }
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess || !p) {
            pkv::record_cuda_error(e == cudaSuccess ? cudaErrorInvalidSymbol : e);
            return PKV_ERR_CUDA;
        }
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return PKV_OK;
}

}  // namespace

extern "C" int paged_attention_decode_noalloc(void* out, const void* q, const void* k_cache,
                                              const void* v_cache, const int32_t* block_tables,
                                              int32_t max_blocks_per_seq, const int32_t* context_lens,
                                              int32_t num_seqs, int32_t max_context_len, int32_t num_q_heads,
                                              int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                              int32_t num_blocks, float scale, int32_t dtype, void* stream)
{
    const pkv::NvtxRange nvtx("paged_attention_decode_noalloc");
    // a call that is invalid for any workspace gets the same code as from paged_attention_decode
    const int checked = decode_check(out, q, nullptr, nullptr, k_cache, v_cache, block_tables, max_blocks_per_seq,
                                     context_lens, num_seqs, 1, max_context_len, num_q_heads, num_kv_heads,
                                     head_dim, block_size, num_blocks, scale, dtype);
    if (checked != PKV_OK || num_seqs == 0) return checked;
    const size_t need = paged_attention_workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len);
    if (need > (size_t)PKV_NOALLOC_SCRATCH_BYTES) return PKV_ERR_SCRATCH_LIMIT;
    void* scratch = nullptr;
    const int rc = noalloc_scratch(&scratch);
    if (rc != PKV_OK) return rc;
    return paged_attention_decode(out, q, k_cache, v_cache, block_tables, max_blocks_per_seq, context_lens,
                                  num_seqs, max_context_len, num_q_heads, num_kv_heads, head_dim, block_size,
                                  num_blocks, scale, dtype, scratch, (size_t)PKV_NOALLOC_SCRATCH_BYTES, stream);
}
