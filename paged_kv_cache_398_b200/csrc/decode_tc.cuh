// Tensor-core partition kernels of the decode entry points for 16-bit inputs
// (fp16 / bf16): the body of one partition CTA (partition_tc), the ordinary
// grid kernel that wraps it, and the shared-prefix kernel that runs it over a
// work list.  Included by decode.cu and decode_shared.cu, which own the
// launchers; the split-K reduce is in decode_common.cuh.
//
// Per (partition, kv head, sequence) CTA, as in the CUDA-core kernel:
// 4 warps, each walking its share of the partition's 16-token blocks with
// its own 2-stage pipeline of (K tile, V tile) pairs.  The differences:
//
//  * Tiles arrive by 2-D tiled TMA (cp.async.bulk.tensor, no multicast) from
//    a tensor map over the cache viewed as [num_blocks * Hkv * B][head_dim],
//    in boxes of 16 (or, at block size 8, two of 8) rows x 64 elements with
//    the 128-byte swizzle.  The swizzle makes the ldmatrix reads below free
//    of shared-memory bank conflicts.
//  * The products run on the tensor cores as mma.sync m16n8k16 with fp32
//    accumulation.  One query per sequence (G <= 8 query heads): S^T = K Q^T
//    and O^T += V^T P^T, the block's 16 tokens or 16 head-dim entries as the
//    MMA rows and the query heads as its 8 columns, so no row is padding: per
//    block at head_dim 128, 8 MMAs for the scores and 8 for the output.
//    Multi-query (up to 16 query rows): S = Q K^T and O += P V with the rows
//    as the 16-row A operand, 16 + 16 MMAs per block.
//  * Q stays in registers as MMA fragments (exact 16-bit inputs, scaled
//    after the product in fp32).  The probabilities go from the score
//    accumulators into the output MMA's operand (for P^T, transposed in
//    registers by movmatrix).  For fp16 they are rounded to fp16 (11
//    significant bits).  For bf16 they are split into a bf16 pair hi + lo
//    (about 16 bits) and multiplied by two MMAs, because one bf16 rounding
//    (8 bits) can cost 5e-3 on a short, cancelling sum.
//  * In the sequence's last, partial block, the V operand rows of tokens past
//    the length are zeroed, and their scores are set to -inf, so whatever
//    the unused slots hold cannot reach the result.
#pragma once

#include <cuda.h>

namespace {

template <typename T>
struct Mma;

template <>
struct Mma<__nv_bfloat16> {
    __device__ __forceinline__ static void run(float* d, const uint32_t* a, uint32_t b0, uint32_t b1)
    {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    __device__ __forceinline__ static uint32_t pack(float lo, float hi)
    {
        __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&v);
    }
    // bf16 keeps only 8 significant bits, too few for the probabilities of a
    // short, cancelling sum; P is sent as hi + lo, two bf16 pairs holding
    // about 16 bits, through two MMAs on the same V fragments.
    static constexpr bool kSplitP = true;
    __device__ __forceinline__ static uint32_t residual(float lo, float hi, uint32_t packed)
    {
        return pack(lo - __uint_as_float(packed << 16), hi - __uint_as_float(packed & 0xffff0000u));
    }
};

template <>
struct Mma<__half> {
    __device__ __forceinline__ static void run(float* d, const uint32_t* a, uint32_t b0, uint32_t b1)
    {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
            "{%0,%1,%2,%3};"
            : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
    __device__ __forceinline__ static uint32_t pack(float lo, float hi)
    {
        __half2 v = __floats2half2_rn(lo, hi);
        return *reinterpret_cast<uint32_t*>(&v);
    }
    // fp16 keeps 11 significant bits: one MMA per P.V tile is accurate enough
    static constexpr bool kSplitP = false;
    __device__ __forceinline__ static uint32_t residual(float, float, uint32_t) { return 0u; }
};

__device__ __forceinline__ void ldsm_x4(uint32_t* r, uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}

__device__ __forceinline__ void ldsm_x4_trans(uint32_t* r, uint32_t addr)
{
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}

// 2-D tiled TMA load of one box into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar,
                                            uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar), "l"(policy)
        : "memory");
}

constexpr int kTcBoxBytes = 16 * 128;  // 16 rows x 64 16-bit elements

template <int D>
struct TcCfg {
    static constexpr int kBoxes = D / 64;                     // boxes per tile
    static constexpr int kTileBytes = kBoxes * kTcBoxBytes;   // one K (or V) tile
    static constexpr int kStageBytes = 2 * kTileBytes;        // K then V
    static constexpr int kKSteps = D / 16;                    // Q.K k-steps
    static constexpr int kNTiles = D / 8;                     // P.V n-tiles
    static constexpr int kTilesBytes = kWarps * kStages * kStageBytes;
    static constexpr int kBarOff = kTilesBytes;
    static constexpr int kNewBarOff = kBarOff + kWarps * kStages * 8;  // staged new-token rows have landed
    static constexpr int kBlkOff = kNewBarOff + 8;
    static constexpr int kNewOff = (kBlkOff + kMaxPartBlocks * 4 + 15) & ~15;  // staged new-token rows
    static constexpr int kNewRowBytes = 2 * D * 2;                        // one token's K and V rows
    // dynamic shared memory of a launch whose CTAs stage up to new_rows new tokens
    static constexpr int smem_bytes(int new_rows) { return 1024 /* alignment slack */ + kNewOff + new_rows * kNewRowBytes; }
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
};

// Lane 0 of a warp: fetch the K and V rows of one 16-token tile into the
// stage at `dst` (K boxes, then V boxes), completing on `bar`.  Unsplit:
// cache rows [r0, r0 + 16) as 16-row boxes.  Split (block size 8): rows
// [r0, r0 + 8) and [r1, r1 + 8) as 8-row boxes into the two 1 KiB halves of
// each 16-row box, which gives the same swizzled layout, since the 128-byte
// swizzle repeats every 8 rows.
template <int D>
__device__ __forceinline__ void tc_issue(uint32_t dst, uint64_t* bar, const CUtensorMap* tm_k,
                                         const CUtensorMap* tm_v, int r0, int r1, bool split, uint64_t policy)
{
    using C = TcCfg<D>;
    const uint32_t b = pkv::smem_addr(bar);
    // order this warp's earlier generic reads of the stage before the async writes
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    pkv::mbar_arrive_expect_tx(bar, C::kStageBytes);
#pragma unroll
    for (int bx = 0; bx < C::kBoxes; ++bx) {
        const uint32_t kd = dst + bx * kTcBoxBytes, vd = dst + C::kTileBytes + bx * kTcBoxBytes;
        tma_load_2d(kd, tm_k, bx * 64, r0, b, policy);
        tma_load_2d(vd, tm_v, bx * 64, r0, b, policy);
        if (split) {
            tma_load_2d(kd + kTcBoxBytes / 2, tm_k, bx * 64, r1, b, policy);
            tma_load_2d(vd + kTcBoxBytes / 2, tm_v, bx * 64, r1, b, policy);
        }
    }
}

// Transpose an 8x8 matrix of 16-bit values held as MMA fragments (lane l
// holds row l / 4, columns 2 (l % 4) and 2 (l % 4) + 1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x)
{
    uint32_t y;
    asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
    return y;
}

__device__ __forceinline__ uint4 ld_shared_v4(uint32_t addr)
{
    uint4 v;
    asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr)
                 : "memory");
    return v;
}

// 16 bytes global -> shared (cp.async, cached in L2 only), completing on the
// issuing thread's cp.async tracking.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}

// Arrive on `bar` once every cp.async this thread issued before has landed
// (the barrier's count includes this arrival).
__device__ __forceinline__ void cp_async_arrive(uint64_t* bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(pkv::smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, const uint4& v)
{
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// The reference max of a score row moves only when a block's max passes it
// by more than kLazyLog2 (log2 units).  Probabilities then stay below
// 2^kLazyLog2, so neither the fp32 sums nor the 16-bit P operand can
// overflow, and the running sums are rescaled on few blocks instead of on
// every block that raises the max.  The result is the same softmax: the
// reference cancels in out = acc / l.
constexpr float kLazyLog2 = 8.0f;

// Online-softmax update of one score row held by a lane quad.  x: this
// lane's 4 scores (log2 domain, -inf where masked); m / l: the row's
// reference max and this lane's share of the running sum.  Returns the
// factor by which earlier partial outputs must be scaled.  A row that has
// seen no visible token yet keeps m = -inf, and every factor stays finite.

__device__ __forceinline__ float softmax_row(float* x, float& m, float& l)
{
    float mx = fmaxf(fmaxf(x[0], x[1]), fmaxf(x[2], x[3]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    float alpha = 1.0f;
    if (mx > m + kLazyLog2) {  // never while the row has seen nothing (mx = m = -inf)
        alpha = pkv::fast_exp2(m - mx);
        m = mx;
    }
    const float mu = m == -INFINITY ? 0.0f : m;
#pragma unroll
    for (int i = 0; i < 4; ++i) x[i] = pkv::fast_exp2(x[i] - mu);
    l = l * alpha + ((x[0] + x[1]) + (x[2] + x[3]));
    return alpha;
}

// The work of one CTA: partition p, kv head h, and z = sequence s (or, in
// the group pass, group g).  q_len new tokens per sequence: query row r = j * G + g is query head h*G + g of new token j,
// which sits at position ctx - q_len + j and sees positions up to its own
// (q_len = 1: the whole context).
//  kMQ = false: q_len * G <= 8 rows, the transposed products S^T = K Q^T and
//               O^T += V^T P^T with the rows as the MMA's 8 columns.
//  kMQ = true : 9..16 rows, S = Q K^T and O += P V with the rows as the
//               16-row A operand.
// k_new / v_new non-null: the new tokens' K/V rows [S][q_len][Hkv][D] are
// written to their slots (through the block table) by the CTA whose
// partition holds them, and patched into the staged tiles before use.
// PT: partition size in tokens (kPartTokens, kLongPartTokens or
// kWidePartTokens: part_tokens_for / mq_part_tokens_for).
// kPlan (paged_attention_decode_shared; kPlanNone otherwise):
//  kPlanGroup: z is group g of plan_groups = (first sequence, n).
//              Its members' queries (one new token each, q_len = 1) are
//              rows j * G + g of the 16-row operand, and the CTA attends
//              partition p of the positions [0, x) that their block tables
//              share (x = shared_lens[first]), through the first member's
//              table, with no new tokens and no causal limit.  A member is
//              covered when its own shared_lens entry is x and x is below its
//              length (shared_split); rows of other members stay empty.
//              Every covered row writes a split-K record at slot p.
//  kPlanOwn:   partition p of sequence s covers its positions from its
//              shared length x (shared_split) on; its records follow the
//              group pass's ceil(x / PT).
// The kernels below run it for one work item each.
template <typename T, int D, int G, bool kMQ, int B, int PT, int kPlan>
__device__ __forceinline__ void partition_tc(const CUtensorMap* tm_k, const CUtensorMap* tm_v, T* __restrict__ out,
                                             float* __restrict__ ws_acc, float* __restrict__ ws_ml,
                                             const T* __restrict__ q, const T* __restrict__ k_new,
                                             const T* __restrict__ v_new, T* __restrict__ k_cache_w,
                                             T* __restrict__ v_cache_w, const int32_t* __restrict__ block_tables,
                                             int32_t mb, const int32_t* __restrict__ context_lens, int32_t max_ctx,
                                             int32_t q_len, int32_t num_q_heads, int32_t num_kv_heads,
                                             int32_t num_blocks, float scale_log2, int32_t max_parts, int* status,
                                             const int32_t* __restrict__ plan_groups,
                                             const int32_t* __restrict__ shared_lens, int32_t num_seqs, const int p,
                                             const int h, const int z)
{
    using C = TcCfg<D>;
    constexpr int part_tokens = PT;
    static_assert(PT == kPartTokens || PT == kLongPartTokens || PT == kWidePartTokens, "partition sizes");
    static_assert(kPlan != kPlanOwn || !kMQ, "a sequence's own pass has one query");
    static_assert(G >= 1 && G <= 8, "G query heads fill rows 0..G-1 of the 16-row operand");
    constexpr int kRows = kMQ ? 16 : 8;  // operand rows that can hold queries
    constexpr int kChunks = D / 8;       // 16-byte chunks per K or V row
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    pkv::grid_dependency_wait();  // inputs written by the previous kernel are visible after this
    // the split-K reduce may launch now: its CTAs whose rows need no merge
    // finish inside this grid's tail (after this grid's own wait, so the
    // lengths they read before theirs are complete)
    pkv::grid_dependency_launch();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const bool report = p == 0 && h == 0 && threadIdx.x == 0;
    constexpr int part_blocks = part_tokens / B;
    constexpr int kEntries = (part_blocks + kWarps * 32 - 1) / (kWarps * 32);  // table entries per thread
    static_assert(kEntries <= 2 && part_blocks <= kMaxPartBlocks, "at most two table entries per thread");

    // s: the sequence whose block table the CTA walks; row0: the query /
    // output row of its first query token; ctx: positions attended (the
    // shared length x in the group pass); part0 / blk0: the partition's first
    // position / table entry; slot: its split-K record; nparts: the
    // sequence's partitions in all.  In the group pass, cover bit j marks
    // member j as computed here.
    int s, row0, nq, ctx, part0, blk0, slot, nparts, x_own = 0;
    uint32_t cover = 0u;
    int32_t blk_raw[kEntries];  // this thread's entries of the partition's table slice
#pragma unroll
    for (int e = 0; e < kEntries; ++e) blk_raw[e] = -1;
    if constexpr (kPlan == kPlanGroup) {
        const int g = z;
        const int first = pkv::ld_early(plan_groups + 2 * (int64_t)g);
        const int n = pkv::ld_early(plan_groups + 2 * (int64_t)g + 1);
        if (first < 0 || n < 1 || n * G > kRows || first > num_seqs - n) {
            if (report) pkv::raise_flag(status, PKV_DEV_BAD_PLAN);
            return;
        }
        const int x = pkv::ld_early(shared_lens + first);
        if (x < 1 || x % B != 0 || x > max_ctx || (int64_t)x > (int64_t)mb * B) {
            if (report) pkv::raise_flag(status, PKV_DEV_BAD_PLAN);
            return;
        }
        if (p * part_tokens >= x) return;
        s = first;
        row0 = first;
        nq = n;
        ctx = x;
        part0 = p * part_tokens;
        blk0 = p * part_blocks;
        slot = p;
        nparts = 2;  // records, never the final output
#pragma unroll
        for (int e = 0; e < kEntries; ++e) {
            const int i = (int)threadIdx.x + e * kWarps * 32;
            if (i < part_blocks && blk0 + i < mb) blk_raw[e] = pkv::ld_early(block_tables + (int64_t)s * mb + blk0 + i);
        }
        // members: covered when their own split is x (warp 0, one lane each)
        if (warp == 0) {
            bool cov = false, stray = false;
            if (lane < n) {
                const int cj = pkv::ld_early(context_lens + first + lane);
                const int xj = pkv::ld_early(shared_lens + first + lane);
                cov = xj == x && cj >= 1 && cj <= max_ctx && (int64_t)cj <= (int64_t)mb * B &&
                      shared_split(xj, cj, B) == x;
                stray = !cov;
            }
            cover = __ballot_sync(0xffffffffu, cov);
            const uint32_t strays = __ballot_sync(0xffffffffu, stray);  // the whole warp votes
            if (report && strays != 0u) pkv::raise_flag(status, PKV_DEV_BAD_PLAN);
        }
    } else if constexpr (kPlan == kPlanOwn) {
        s = z;
        const int x_raw = pkv::ld_early(shared_lens + s);
        SeqRange sr = seq_range_of(pkv::ld_early(context_lens + s), mb, B, max_ctx, part_tokens, report, status);
        if (!sr.bad && sr.ctx < q_len) {
            if (report) pkv::raise_flag(status, PKV_DEV_BAD_CONTEXT);
            sr.bad = true;
        }
        if (sr.bad) {
            if (p == 0) {
                for (int i = threadIdx.x; i < q_len * G * D; i += blockDim.x) {
                    const int r = i / D;
                    const int64_t orow = ((int64_t)s * q_len + r / G) * num_q_heads + h * G + r % G;
                    pkv::store_out(out + orow * D + i % D, 0.0f);
                }
            }
            return;
        }
        const int x = shared_split(x_raw, sr.ctx, B);
        const int own_parts = (sr.ctx - x + part_tokens - 1) / part_tokens;
        if (report && x_raw != 0 && x == 0) pkv::raise_flag(status, PKV_DEV_BAD_PLAN);
        if (p >= own_parts) return;
        row0 = s * q_len;
        nq = q_len;
        ctx = sr.ctx;
        part0 = x + p * part_tokens;
        blk0 = part0 / B;
        x_own = x;  // slot and nparts follow from it after the loop
        slot = nparts = 0;
#pragma unroll
        for (int e = 0; e < kEntries; ++e) {
            const int i = (int)threadIdx.x + e * kWarps * 32;
            if (i < part_blocks && blk0 + i < mb) blk_raw[e] = pkv::ld_early(block_tables + (int64_t)s * mb + blk0 + i);
        }
    } else {
        // The context length and this thread's entry of the partition's table
        // slice are loaded together: the entry depends only on (s, p), so the
        // slice does not wait for the length (one memory round trip before
        // the first tile copies instead of two).  Entries past the sequence's
        // own blocks are loaded but never used.
        s = z;
        blk0 = p * part_blocks;
#pragma unroll
        for (int e = 0; e < kEntries; ++e) {
            const int i = (int)threadIdx.x + e * kWarps * 32;
            if (i < part_blocks && blk0 + i < mb) blk_raw[e] = pkv::ld_early(block_tables + (int64_t)s * mb + blk0 + i);
        }
        SeqRange sr = seq_range_of(pkv::ld_early(context_lens + s), mb, B, max_ctx, part_tokens,
                                   p == 0 && h == 0 && threadIdx.x == 0, status);
        if (!sr.bad && sr.ctx < q_len) {
            if (p == 0 && h == 0 && threadIdx.x == 0) pkv::raise_flag(status, PKV_DEV_BAD_CONTEXT);
            sr.bad = true;
        }
        if (sr.bad) {
            if (p == 0) {
                for (int i = threadIdx.x; i < q_len * G * D; i += blockDim.x) {
                    const int r = i / D;
                    const int64_t orow = ((int64_t)s * q_len + r / G) * num_q_heads + h * G + r % G;
                    pkv::store_out(out + orow * D + i % D, 0.0f);
                }
            }
            return;
        }
        if (p >= sr.nparts) return;
        row0 = s * q_len;
        nq = q_len;
        ctx = sr.ctx;
        part0 = p * part_tokens;
        slot = p;
        nparts = sr.nparts;
    }
    const int rows = nq * G;  // query rows

    const int nblk_seq = (ctx + B - 1) / B;
    const int nbp = min(part_blocks, nblk_seq - blk0);                          // blocks of this partition
    const int nb = min(part_tokens / kTile, (ctx - part0 + kTile - 1) / kTile);  // its 16-token tiles
    // position of the first new token (the group pass has none: its rows see all of [0, x))
    const int first_new = kPlan == kPlanGroup ? ctx - 1 : ctx - q_len;
    // Fused write: the new tokens that fall in this partition, as token
    // indices [jlo_p, jhi_p).  With up to 16 new tokens (kMQ), right after
    // the prologue every thread stages some of their K / V rows in shared
    // memory by cp.async, so the warp that writes and patches them later
    // never waits on global memory.  With at most 8 (kMQ false) the warp
    // loads them where it patches them, four 16-byte chunks in flight per lane.
    constexpr int kNewRows = kMQ ? 16 : 0;  // capacity of the staging area, in tokens
    const int jlo_p = max(0, part0 - first_new);
    const int jhi_p = min(q_len, part0 + part_tokens - first_new);
    const bool stage_new =
        kMQ && kPlan != kPlanGroup && k_new != nullptr && jhi_p > jlo_p;  // the same for the whole CTA
    uint64_t* new_bar = reinterpret_cast<uint64_t*>(smem + C::kNewBarOff);
    const uint32_t new_rows = pkv::smem_addr(smem + C::kNewOff);

    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kBarOff) + warp * kStages;
    int32_t* s_blk = reinterpret_cast<int32_t*>(smem + C::kBlkOff);
    const uint32_t tiles = pkv::smem_addr(smem + warp * (kStages * C::kStageBytes));

#pragma unroll
    for (int e = 0; e < kEntries; ++e) {
        const int i = (int)threadIdx.x + e * kWarps * 32;
        if (i < nbp) {  // nbp <= part_blocks, and blk0 + nbp <= mb
            int b = blk_raw[e];
            if (b < 0 || b >= num_blocks) {
                pkv::raise_flag(status, PKV_DEV_BAD_BLOCK_ID);
                b = -1;  // read block 0 in its place; never write through it
            }
            s_blk[i] = b;
        }
    }
    if (lane == 0) {
#pragma unroll
        for (int st = 0; st < kStages; ++st) pkv::mbar_init(&bars[st], 1);
        if (warp == 0 && stage_new) pkv::mbar_init(new_bar, kWarps * 32);  // one arrival per thread
        pkv::fence_mbar_init();
    }
    if constexpr (kPlan == kPlanGroup) {
        // the group pass stages nothing: the staging barrier's two words carry
        // the cover bits and the members whose tables disagree with the leader's
        if (threadIdx.x == 0) {
            reinterpret_cast<volatile uint32_t*>(new_bar)[0] = cover;
            reinterpret_cast<volatile uint32_t*>(new_bar)[1] = 0u;
        }
        __syncthreads();
        cover = *reinterpret_cast<volatile uint32_t*>(new_bar);
    } else {
        __syncthreads();
    }

    const int nw = nb > warp ? (nb - warp + kWarps - 1) / kWarps : 0;
    uint64_t policy = 0;
    if (lane == 0) {
        policy = pkv::policy_evict_first();
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm_k)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(tm_v)) : "memory");
        for (int k = 0; k < nw && k < kStages; ++k) {
            int r0, r1;
            tile_rows<B>(s_blk, nbp, warp + k * kWarps, num_kv_heads, h, r0, r1);
            tc_issue<D>(tiles + (k % kStages) * C::kStageBytes, &bars[k % kStages], tm_k, tm_v, r0, r1, B == 8,
                        policy);
        }
    }
    if (stage_new) {
        // staging layout [token - jlo_p][K or V][16-byte chunk], chunk index = it
        const int chunks = (jhi_p - jlo_p) * 2 * kChunks;  // <= kNewRows * 2 * kChunks
        for (int it = threadIdx.x; it < chunks; it += kWarps * 32) {
            const int c = it % kChunks, kv = (it / kChunks) & 1, jj = jlo_p + it / (2 * kChunks);
            cp_async_16(new_rows + it * 16,
                        (kv ? v_new : k_new) + (((int64_t)s * q_len + jj) * num_kv_heads + h) * D + c * 8);
        }
        cp_async_arrive(new_bar);
    }
    static_assert(kNewRows * C::kNewRowBytes == kNewRows * 2 * kChunks * 16, "staging row size");

    // ---- Q as A fragments: rows ra = lane / 4 (a0, a2) and rb = ra + 8 (a1, a3)
    const int ra = lane >> 2, rb = ra + 8;
    const int qd = 2 * (lane & 3);
    const bool live_a = ra < rows && (kPlan != kPlanGroup || ((cover >> (ra / G)) & 1u));
    const bool live_b = kMQ && rb < rows && (kPlan != kPlanGroup || ((cover >> (rb / G)) & 1u));
    uint32_t qa[C::kKSteps][4];
#pragma unroll
    for (int ks = 0; ks < C::kKSteps; ++ks) {
        qa[ks][0] = qa[ks][1] = qa[ks][2] = qa[ks][3] = 0u;
        if (live_a) {
            const T* qrow = q + (((int64_t)row0 + ra / G) * num_q_heads + h * G + ra % G) * D + 16 * ks + qd;
            qa[ks][0] = *reinterpret_cast<const uint32_t*>(qrow);
            qa[ks][2] = *reinterpret_cast<const uint32_t*>(qrow + 8);
        }
        if (live_b) {
            const T* qrow = q + (((int64_t)row0 + rb / G) * num_q_heads + h * G + rb % G) * D + 16 * ks + qd;
            qa[ks][1] = *reinterpret_cast<const uint32_t*>(qrow);
            qa[ks][3] = *reinterpret_cast<const uint32_t*>(qrow + 8);
        }
    }
    if constexpr (kPlan == kPlanGroup) {
        // The plan promises that every covered member's table holds the
        // leader's block ids over [0, x); a plan made before a table changed
        // (a copy-on-write repoint, an eviction) breaks that.  Check this
        // partition's slice of each member against the leader's (s_blk).
        // The loads go out after the first tile copies, so their latency
        // hides behind those.  A member that differs is marked; the merge
        // then gives it a poison record instead of its split-K record.
        uint32_t bad = 0u;
        const int checks = (nq - 1) * nbp;  // members 1..nq-1; blk0 + nbp <= ceil(x / B) <= mb
        for (int idx = threadIdx.x; idx < checks; idx += kWarps * 32) {
            const int j = 1 + idx / nbp, i = idx % nbp;
            if ((cover >> j) & 1u) {
                const int32_t b = pkv::ld_early(block_tables + (int64_t)(s + j) * mb + blk0 + i);
                if (b != s_blk[i]) bad |= 1u << j;
            }
        }
        bad = __reduce_or_sync(0xffffffffu, bad);
        if (lane == 0 && bad != 0u) atomicOr(reinterpret_cast<uint32_t*>(new_bar) + 1, bad);
    }

    // Multi-query: positions row ra (rb) may see are < lim_a (lim_b); a row
    // holding no query sees nothing.  (A single query sees the whole context,
    // so that path masks against ctx alone.)
    const int lim_a = live_a ? (kPlan == kPlanGroup ? ctx : first_new + ra / G + 1) : 0;
    const int lim_b = live_b ? (kPlan == kPlanGroup ? ctx : first_new + rb / G + 1) : 0;

    // ---- per-lane ldmatrix addressing (128-byte swizzle: chunk c of row r is at c ^ (r % 8))
    const int mi = lane >> 3, r8 = lane & 7;
    // K (non-transposed): matrix mi -> tokens (mi / 2) * 8 + r8, 16-byte chunk 2 * ks + (mi % 2)
    const uint32_t k_row_off = (uint32_t)(((mi >> 1) * 8 + r8) * 128);
    const uint32_t k_x = (uint32_t)(((mi & 1) ^ r8) << 4);
    // V (transposed): matrix mi -> tokens (mi % 2) * 8 + r8, chunk 2 * j + (mi / 2)
    const uint32_t v_row_off = (uint32_t)(((mi & 1) * 8 + r8) * 128);
    const uint32_t v_x = (uint32_t)(((mi >> 1) ^ r8) << 4);

    // Multi-query: O [16 rows][D] as n-tiles, rows ra (o[.][0..1]) and rb
    // (o[.][2..3]).  One query: O^T [D][8 rows] as m-tiles (ot), rows qd
    // (ot[.][0], ot[.][2]) and qd + 1 (ot[.][1], ot[.][3]), head-dim entries
    // 16 j + ra and 16 j + ra + 8; (m_a, l_a) belong to row qd and (m_b, l_b)
    // to row qd + 1.
    float o[kMQ ? C::kNTiles : 1][4];
    float ot[kMQ ? 1 : C::kNTiles / 2][4];
#pragma unroll
    for (int n = 0; n < (kMQ ? C::kNTiles : 1); ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.0f;
#pragma unroll
    for (int n = 0; n < (kMQ ? 1 : C::kNTiles / 2); ++n) ot[n][0] = ot[n][1] = ot[n][2] = ot[n][3] = 0.0f;
    float m_a = -INFINITY, l_a = 0.0f, m_b = -INFINITY, l_b = 0.0f;
    bool timed_out = false;
    int consumed = 0;

    for (int k = 0; k < nw; ++k) {
        const int st = k % kStages;
        if (!pkv::mbar_wait(&bars[st], (k / kStages) & 1, kWaitLimitNs)) {
            timed_out = true;
            break;
        }
        const uint32_t kbase = tiles + st * C::kStageBytes;
        const uint32_t vbase = kbase + C::kTileBytes;
        const int tile = warp + k * kWarps;
        const int pos0 = part0 + tile * kTile;

        // ---- fused slot write: this tile holds new tokens -> store and patch
        if (stage_new && pos0 + kTile > first_new) {
            if (!pkv::mbar_wait(new_bar, 0, kWaitLimitNs)) {
                timed_out = true;
                break;
            }
            const int jlo = max(0, pos0 - first_new);
            const int jhi = min(q_len, pos0 + kTile - first_new);
            const int items = (jhi - jlo) * 2 * kChunks;  // 16-byte chunks: (token, K or V, chunk)
            for (int it = lane; it < items; it += 32) {
                const int c = it % kChunks, kv = (it / kChunks) & 1, jj = jlo + it / (2 * kChunks);
                const int t = first_new + jj - pos0;  // row in the tile
                const int pos = first_new + jj;       // position in the sequence
                const int phys = s_blk[(pos - part0) / B];
                const uint4 val = ld_shared_v4(new_rows + (((jj - jlo_p) * 2 + kv) * kChunks + c) * 16);
                st_shared_v4(kbase + kv * C::kTileBytes + (c / 8) * kTcBoxBytes + t * 128 + (((c % 8) ^ (t & 7)) << 4),
                             val);
                if (phys >= 0) {
                    T* dst = (kv ? v_cache_w : k_cache_w) +
                             (((int64_t)phys * num_kv_heads + h) * B + pos % B) * D + c * 8;
                    *reinterpret_cast<uint4*>(dst) = val;
                }
            }
            __syncwarp();
        } else if (!kMQ && k_new != nullptr && pos0 + kTile > first_new) {
            // the new tokens of this block: loaded here, four 16-byte chunks in flight per lane
            const int jlo = max(0, pos0 - first_new);
            const int jhi = min(q_len, pos0 + kTile - first_new);
            const int items = (jhi - jlo) * 2 * kChunks;  // 16-byte chunks: (token, K or V, chunk)
            constexpr int kBatch = 4;
            for (int it0 = lane; it0 < items; it0 += 32 * kBatch) {
                uint4 val[kBatch];
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int it = it0 + 32 * u;
                    if (it < items) {
                        const int c = it % kChunks, kv = (it / kChunks) & 1, jj = jlo + it / (2 * kChunks);
                        const T* src = (kv ? v_new : k_new) + (((int64_t)s * q_len + jj) * num_kv_heads + h) * D + c * 8;
                        val[u] = __ldg(reinterpret_cast<const uint4*>(src));
                    }
                }
#pragma unroll
                for (int u = 0; u < kBatch; ++u) {
                    const int it = it0 + 32 * u;
                    if (it < items) {
                        const int c = it % kChunks, kv = (it / kChunks) & 1, jj = jlo + it / (2 * kChunks);
                        const int t = first_new + jj - pos0;  // row in the tile
                        const int pos = first_new + jj;       // position in the sequence
                        const int phys = s_blk[(pos - part0) / B];
                        st_shared_v4(kbase + kv * C::kTileBytes + (c / 8) * kTcBoxBytes + t * 128 +
                                         (((c % 8) ^ (t & 7)) << 4),
                                     val[u]);
                        if (phys >= 0) {
                            T* dst = (kv ? v_cache_w : k_cache_w) +
                                     (((int64_t)phys * num_kv_heads + h) * B + pos % B) * D + c * 8;
                            *reinterpret_cast<uint4*>(dst) = val[u];
                        }
                    }
                }
            }
            __syncwarp();
        }

        if constexpr (!kMQ) {
            // ---- one query: S^T = K Q^T, the block's 16 tokens as MMA rows and
            // the (at most 8) query heads as its columns, so the MMA carries no
            // padding rows.  The K fragments are the same ldmatrix tiles in A
            // order; Q's fragments serve as the B operand.
            float sa[4] = {0.f, 0.f, 0.f, 0.f}, sb[4] = {0.f, 0.f, 0.f, 0.f};  // even / odd k-steps
#pragma unroll
            for (int ks = 0; ks < C::kKSteps; ++ks) {
                uint32_t b[4];
                const uint32_t addr =
                    kbase + (ks / 4) * kTcBoxBytes + k_row_off + (((uint32_t)(2 * (ks % 4)) << 4) ^ k_x);
                ldsm_x4(b, addr);
                const uint32_t a[4] = {b[0], b[2], b[1], b[3]};
                Mma<T>::run(ks % 2 ? sb : sa, a, qa[ks][0], qa[ks][2]);
            }
            // this lane: tokens ra (x[0], x[1]) and ra + 8 (x[2], x[3]) of rows qd, qd + 1
            float x[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) x[i] = (sa[i] + sb[i]) * scale_log2;
            if (pos0 + kTile > first_new + 1) {
                // some token of this block lies past a row's last visible
                // position: ctx - 1 for one query, the row's own token's
                // position for several; padding rows keep ctx (finite scores)
                // (the group pass: every row sees all of [0, x) -- no causal limit)
                const int lim0 = kPlan != kPlanGroup && qd < rows ? first_new + qd / G + 1 : ctx;
                const int lim1 = kPlan != kPlanGroup && qd + 1 < rows ? first_new + (qd + 1) / G + 1 : ctx;
                if (pos0 + ra >= lim0) x[0] = -INFINITY;
                if (pos0 + ra >= lim1) x[1] = -INFINITY;
                if (pos0 + ra + 8 >= lim0) x[2] = -INFINITY;
                if (pos0 + ra + 8 >= lim1) x[3] = -INFINITY;
            }
            float mx0 = fmaxf(x[0], x[2]), mx1 = fmaxf(x[1], x[3]);
#pragma unroll
            for (int sh = 4; sh < 32; sh <<= 1) {
                mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, sh));
                mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, sh));
            }
            // A row moves its reference on its first visible token.  With
            // several new tokens a row can see nothing in this partition yet
            // (m = -inf): its scores are then all -inf and its weights 0.
            float alpha_a = 1.0f, alpha_b = 1.0f;
            if (mx0 > m_a + kLazyLog2) {
                alpha_a = pkv::fast_exp2(m_a - mx0);
                m_a = mx0;
            }
            if (mx1 > m_b + kLazyLog2) {
                alpha_b = pkv::fast_exp2(m_b - mx1);
                m_b = mx1;
            }
            const float mu_a = m_a == -INFINITY ? 0.0f : m_a, mu_b = m_b == -INFINITY ? 0.0f : m_b;
            x[0] = pkv::fast_exp2(x[0] - mu_a);
            x[2] = pkv::fast_exp2(x[2] - mu_a);
            x[1] = pkv::fast_exp2(x[1] - mu_b);
            x[3] = pkv::fast_exp2(x[3] - mu_b);
            l_a = l_a * alpha_a + (x[0] + x[2]);
            l_b = l_b * alpha_b + (x[1] + x[3]);
            // P^T as the B operand of O^T += V^T P^T: transpose each 8-token half
            const uint32_t h0 = Mma<T>::pack(x[0], x[1]), h1 = Mma<T>::pack(x[2], x[3]);
            const uint32_t pb0 = movmatrix_trans(h0), pb1 = movmatrix_trans(h1);
            uint32_t lb0 = 0u, lb1 = 0u;  // bf16: the residual (lo) of P
            if constexpr (Mma<T>::kSplitP) {
                lb0 = movmatrix_trans(Mma<T>::residual(x[0], x[1], h0));
                lb1 = movmatrix_trans(Mma<T>::residual(x[2], x[3], h1));
            }
            if (__any_sync(0xffffffffu, alpha_a != 1.0f || alpha_b != 1.0f)) {
#pragma unroll
                for (int j = 0; j < C::kNTiles / 2; ++j) {
                    ot[j][0] *= alpha_a;
                    ot[j][1] *= alpha_b;
                    ot[j][2] *= alpha_a;
                    ot[j][3] *= alpha_b;
                }
            }
            // ---- O^T += V^T P^T: 16 head-dim entries per MMA, the block's
            // tokens as k.  V rows of tokens at or past the sequence length are
            // zeroed: whatever the unused slots hold (even NaN) must not reach
            // the result.  This lane's V^T fragments hold tokens qd, qd + 1
            // (a0, a1) and qd + 8, qd + 9 (a2, a3).
            uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;
            if (pos0 + kTile > ctx) {
                const int t = pos0 + qd;
                keep_lo = (t < ctx ? 0x0000ffffu : 0u) | (t + 1 < ctx ? 0xffff0000u : 0u);
                keep_hi = (t + 8 < ctx ? 0x0000ffffu : 0u) | (t + 9 < ctx ? 0xffff0000u : 0u);
            }
#pragma unroll
            for (int j = 0; j < C::kNTiles / 2; ++j) {
                uint32_t v[4];
                const uint32_t addr =
                    vbase + (j / 4) * kTcBoxBytes + v_row_off + (((uint32_t)(2 * (j % 4)) << 4) ^ v_x);
                ldsm_x4_trans(v, addr);
                const uint32_t a[4] = {v[0] & keep_lo, v[2] & keep_lo, v[1] & keep_hi, v[3] & keep_hi};
                Mma<T>::run(ot[j], a, pb0, pb1);
                if constexpr (Mma<T>::kSplitP) Mma<T>::run(ot[j], a, lb0, lb1);
            }
        } else {
            // ---- multi-query: S = Q K^T, 16 query rows x the block's 16 tokens (two 8-token tiles)
            float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int ks = 0; ks < C::kKSteps; ++ks) {
                uint32_t b[4];
                const uint32_t addr =
                    kbase + (ks / 4) * kTcBoxBytes + k_row_off + (((uint32_t)(2 * (ks % 4)) << 4) ^ k_x);
                ldsm_x4(b, addr);
                Mma<T>::run(s0, qa[ks], b[0], b[1]);
                Mma<T>::run(s1, qa[ks], b[2], b[3]);
            }

            // ---- online softmax; this lane holds tokens qd, qd+1, qd+8, qd+9 of rows ra and rb
            const bool mask = pos0 + kTile > first_new + 1;  // some token of this tile is not visible to all rows
            float xa[4] = {s0[0] * scale_log2, s0[1] * scale_log2, s1[0] * scale_log2, s1[1] * scale_log2};
            float xb[4] = {s0[2] * scale_log2, s0[3] * scale_log2, s1[2] * scale_log2, s1[3] * scale_log2};
            const int tp[4] = {pos0 + qd, pos0 + qd + 1, pos0 + qd + 8, pos0 + qd + 9};
            if (mask) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (tp[i] >= lim_a) xa[i] = -INFINITY;
                    if (tp[i] >= lim_b) xb[i] = -INFINITY;
                }
            }
            const float alpha_a = softmax_row(xa, m_a, l_a);
            const float alpha_b = softmax_row(xb, m_b, l_b);
            uint32_t pa[4], pl[4];  // P (hi) and, for bf16, its residual (lo)
            pa[0] = Mma<T>::pack(xa[0], xa[1]);
            pa[1] = Mma<T>::pack(xb[0], xb[1]);
            pa[2] = Mma<T>::pack(xa[2], xa[3]);
            pa[3] = Mma<T>::pack(xb[2], xb[3]);
            if constexpr (Mma<T>::kSplitP) {
                pl[0] = Mma<T>::residual(xa[0], xa[1], pa[0]);
                pl[1] = Mma<T>::residual(xb[0], xb[1], pa[1]);
                pl[2] = Mma<T>::residual(xa[2], xa[3], pa[2]);
                pl[3] = Mma<T>::residual(xb[2], xb[3], pa[3]);
            }
            if (__any_sync(0xffffffffu, alpha_a != 1.0f || alpha_b != 1.0f)) {
#pragma unroll
                for (int n = 0; n < C::kNTiles; ++n) {
                    o[n][0] *= alpha_a;
                    o[n][1] *= alpha_a;
                    o[n][2] *= alpha_b;
                    o[n][3] *= alpha_b;
                }
            }

            // ---- O += P V over the head dimension (pairs of 8-wide tiles)
            // V rows of tokens at or past the sequence length are zeroed: whatever
            // the unused slots hold (even NaN) must not reach the result.
            uint32_t keep_lo = 0xffffffffu, keep_hi = 0xffffffffu;  // V rows qd, qd+1 / qd+8, qd+9
            if (pos0 + kTile > ctx) {
                keep_lo = (tp[0] < ctx ? 0x0000ffffu : 0u) | (tp[1] < ctx ? 0xffff0000u : 0u);
                keep_hi = (tp[2] < ctx ? 0x0000ffffu : 0u) | (tp[3] < ctx ? 0xffff0000u : 0u);
            }
#pragma unroll
            for (int j = 0; j < C::kNTiles / 2; ++j) {
                uint32_t b[4];
                const uint32_t addr =
                    vbase + (j / 4) * kTcBoxBytes + v_row_off + (((uint32_t)(2 * (j % 4)) << 4) ^ v_x);
                ldsm_x4_trans(b, addr);
                b[0] &= keep_lo;
                b[1] &= keep_hi;
                b[2] &= keep_lo;
                b[3] &= keep_hi;
                Mma<T>::run(o[2 * j], pa, b[0], b[1]);
                Mma<T>::run(o[2 * j + 1], pa, b[2], b[3]);
                if constexpr (Mma<T>::kSplitP) {
                    Mma<T>::run(o[2 * j], pl, b[0], b[1]);
                    Mma<T>::run(o[2 * j + 1], pl, b[2], b[3]);
                }
            }
        }
        __syncwarp();
        ++consumed;
        if (lane == 0 && k + kStages < nw) {
            int r0, r1;
            tile_rows<B>(s_blk, nbp, warp + (k + kStages) * kWarps, num_kv_heads, h, r0, r1);
            tc_issue<D>(kbase, &bars[st], tm_k, tm_v, r0, r1, B == 8, policy);
        }
    }

    if (stage_new) cp_async_wait_all();  // no staging copy of this thread is still in flight
    if (timed_out) {
        if (lane == 0) pkv::raise_flag(status, PKV_DEV_WAIT_TIMEOUT);
        for (int k = consumed; k < nw && k < consumed + kStages; ++k) {
            pkv::mbar_wait(&bars[k % kStages], (k / kStages) & 1, kWaitLimitNs);
        }
    }

    // ---- merge the warps through shared-memory records
    // records [kWarps][kRows][kRec]: m, l, two unused words (acc starts 16-byte aligned), acc[D]
    constexpr int kRec = D + 4;
    float* mg = reinterpret_cast<float*>(smem);
    static_assert(kWarps * kRows * kRec * 4 <= C::kTilesBytes, "merge area must fit in the tile area");
    if constexpr (!kMQ) {
        // lane (ra, qd) holds O^T[16 j + ra (+ 8)][qd, qd + 1]; its sums cover
        // tokens ra and ra + 8 of every block, so they add up over the 8 lanes
        // that share qd
#pragma unroll
        for (int sh = 4; sh < 32; sh <<= 1) {
            l_a += __shfl_xor_sync(0xffffffffu, l_a, sh);
            l_b += __shfl_xor_sync(0xffffffffu, l_b, sh);
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int row = qd + e;
            if (row < rows) {
                float* rec = mg + (warp * kRows + row) * kRec;
                if (ra == 0) {
                    rec[0] = e ? m_b : m_a;
                    rec[1] = e ? l_b : l_a;
                }
#pragma unroll
                for (int j = 0; j < C::kNTiles / 2; ++j) {
                    rec[4 + 16 * j + ra] = ot[j][e];
                    rec[4 + 16 * j + ra + 8] = ot[j][2 + e];
                }
            }
        }
    } else {
        // lane (ra, qd) holds O[ra][8 n + qd .. +1] and O[rb][...]
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 1);
        l_a += __shfl_xor_sync(0xffffffffu, l_a, 2);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 1);
        l_b += __shfl_xor_sync(0xffffffffu, l_b, 2);
        __syncthreads();
        if (live_a) {
            float* rec = mg + (warp * kRows + ra) * kRec;
            if ((lane & 3) == 0) {
                rec[0] = m_a;
                rec[1] = l_a;
            }
#pragma unroll
            for (int n = 0; n < C::kNTiles; ++n)
                *reinterpret_cast<float2*>(rec + 4 + 8 * n + qd) = make_float2(o[n][0], o[n][1]);
        }
        if (live_b) {
            float* rec = mg + (warp * kRows + rb) * kRec;
            if ((lane & 3) == 0) {
                rec[0] = m_b;
                rec[1] = l_b;
            }
#pragma unroll
            for (int n = 0; n < C::kNTiles; ++n)
                *reinterpret_cast<float2*>(rec + 4 + 8 * n + qd) = make_float2(o[n][2], o[n][3]);
        }
    }
    __syncthreads();

    // One warp per query row, each lane owning head_dim / 32 consecutive
    // outputs; the weights of the warps' records are computed once per row.
    constexpr int kPer = D / 32;
    using Vec = typename std::conditional<kPer == 4, float4, float2>::type;
    if constexpr (kPlan == kPlanOwn) {
        slot = (x_own + part_tokens - 1) / part_tokens + p;
        nparts = split_parts(x_own, ctx, part_tokens);
    }
    uint32_t mismatch = 0u;  // group pass: members whose tables differ from the leader's
    if constexpr (kPlan == kPlanGroup) {
        mismatch = reinterpret_cast<volatile uint32_t*>(new_bar)[1];
        if (threadIdx.x == 0 && mismatch != 0u) pkv::raise_flag(status, PKV_DEV_BAD_PLAN);
    }
    for (int r = warp; r < rows; r += kWarps) {
        if (kPlan == kPlanGroup && !((cover >> (r / G)) & 1u)) continue;  // a member computed elsewhere
        if (kPlan == kPlanGroup && ((mismatch >> (r / G)) & 1u)) {
            // poison record (m = +inf, which no score produces): the reduce
            // leaves this member's output row unwritten
            if (lane == 0) {
                const int64_t orow = ((int64_t)row0 + r / G) * num_q_heads + h * G + r % G;
                ws_ml[(orow * max_parts + slot) * 2] = INFINITY;
                ws_ml[(orow * max_parts + slot) * 2 + 1] = 0.0f;
            }
            continue;
        }
        float mw[kWarps];
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            mw[w] = mg[(w * kRows + r) * kRec];
            M = fmaxf(M, mw[w]);
        }
        const float Mu = M == -INFINITY ? 0.0f : M;  // a row that saw no token here: all weights 0
        float L = 0.0f, O[kPer];
#pragma unroll
        for (int e = 0; e < kPer; ++e) O[e] = 0.0f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float* rec = mg + (w * kRows + r) * kRec;
            const float wgt = pkv::fast_exp2(mw[w] - Mu);
            L = fmaf(rec[1], wgt, L);
            const Vec v = *reinterpret_cast<const Vec*>(rec + 4 + lane * kPer);
            const float* vf = reinterpret_cast<const float*>(&v);
#pragma unroll
            for (int e = 0; e < kPer; ++e) O[e] = fmaf(vf[e], wgt, O[e]);
        }
        const int64_t orow = ((int64_t)row0 + r / G) * num_q_heads + h * G + r % G;
        if (nparts == 1) {
#pragma unroll
            for (int e = 0; e < kPer; ++e) pkv::store_out(out + orow * D + lane * kPer + e, O[e] / L);
        } else {
            // the reduce reads these right after this kernel: keep them in L2
            const uint64_t keep = pkv::policy_evict_last();
            Vec ov;
            float* of = reinterpret_cast<float*>(&ov);
#pragma unroll
            for (int e = 0; e < kPer; ++e) of[e] = O[e];
            pkv::st_global_hint(reinterpret_cast<Vec*>(ws_acc + (orow * max_parts + slot) * D) + lane, ov, keep);
            if (lane == 0) {
                pkv::st_global_hint(ws_ml + (orow * max_parts + slot) * 2, M, keep);
                pkv::st_global_hint(ws_ml + (orow * max_parts + slot) * 2 + 1, L, keep);
            }
        }
    }
}

// An ordinary launch: one CTA per (partition, kv head, sequence) of the grid.
template <typename T, int D, int G, bool kMQ, int B, int PT>
__global__ void __launch_bounds__(kWarps * 32)
    decode_partition_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                               T* __restrict__ out, float* __restrict__ ws_acc, float* __restrict__ ws_ml,
                               const T* __restrict__ q, const T* __restrict__ k_new, const T* __restrict__ v_new,
                               T* __restrict__ k_cache_w, T* __restrict__ v_cache_w,
                               const int32_t* __restrict__ block_tables, int32_t mb,
                               const int32_t* __restrict__ context_lens, int32_t max_ctx, int32_t q_len,
                               int32_t num_q_heads, int32_t num_kv_heads, int32_t num_blocks, float scale_log2,
                               int32_t max_parts, int* status)
{
    partition_tc<T, D, G, kMQ, B, PT, kPlanNone>(&tm_k, &tm_v, out, ws_acc, ws_ml, q, k_new, v_new, k_cache_w,
                                                  v_cache_w, block_tables, mb, context_lens, max_ctx, q_len,
                                                  num_q_heads, num_kv_heads, num_blocks, scale_log2, max_parts,
                                                  status, nullptr, nullptr, 0, blockIdx.x, blockIdx.y, blockIdx.z);
}

// paged_attention_decode_shared: both passes in one launch, one CTA per (work
// item, kv head), kv head fastest.  A work item (int32 pair) is (~g, p): the
// group pass over partition p of group g's shared positions, or (s, p):
// partition p of sequence s's own positions (with its new token's slot
// write).  The host lists the items longest first, so the long group
// partitions start early and the short ones fill the tail.  3 CTAs per SM
// for both forms: the register budget is capped at 168.
template <typename T, int D, int G, int B, int PT>
__global__ void __launch_bounds__(kWarps * 32, 3)
    decode_shared_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                            T* __restrict__ out, float* __restrict__ ws_acc, float* __restrict__ ws_ml,
                            const T* __restrict__ q, const T* __restrict__ k_new, const T* __restrict__ v_new,
                            T* __restrict__ k_cache_w, T* __restrict__ v_cache_w,
                            const int32_t* __restrict__ block_tables, int32_t mb,
                            const int32_t* __restrict__ context_lens, int32_t max_ctx, int32_t num_q_heads,
                            int32_t num_kv_heads, int32_t num_blocks, float scale_log2, int32_t max_parts,
                            int* status, const int32_t* __restrict__ plan_groups, int32_t num_groups,
                            const int32_t* __restrict__ shared_lens, int32_t num_seqs,
                            const int2* __restrict__ work)
{
    pkv::grid_dependency_wait();  // the work list may come from the previous kernel
    const int item = (int)(blockIdx.x / (unsigned)num_kv_heads), h = (int)(blockIdx.x % (unsigned)num_kv_heads);
    int2 w;
    asm volatile("ld.global.nc.v2.s32 {%0, %1}, [%2];" : "=r"(w.x), "=r"(w.y) : "l"(work + item));
    // a partition index past ceil(max_ctx / PT) fits no sequence (and keeps p * PT in range)
    if (w.y < 0 || w.y >= (max_ctx + PT - 1) / PT || (w.x < 0 ? ~w.x >= num_groups : w.x >= num_seqs)) {
        if (threadIdx.x == 0) pkv::raise_flag(status, PKV_DEV_BAD_PLAN);
        return;
    }
    if (w.x < 0) {
        // a group of at most 8 rows (members x G) runs the transposed 8-column
        // form, a larger one the 16-row form (either checks the group again)
        const int n = pkv::ld_early(plan_groups + 2 * (int64_t)(~w.x) + 1);
        if (n * G <= 8)
            partition_tc<T, D, G, false, B, PT, kPlanGroup>(&tm_k, &tm_v, out, ws_acc, ws_ml, q, nullptr, nullptr,
                                                             k_cache_w, v_cache_w, block_tables, mb, context_lens,
                                                             max_ctx, 1, num_q_heads, num_kv_heads, num_blocks,
                                                             scale_log2, max_parts, status, plan_groups, shared_lens,
                                                             num_seqs, w.y, h, ~w.x);
        else
            partition_tc<T, D, G, true, B, PT, kPlanGroup>(&tm_k, &tm_v, out, ws_acc, ws_ml, q, nullptr, nullptr,
                                                            k_cache_w, v_cache_w, block_tables, mb, context_lens,
                                                            max_ctx, 1, num_q_heads, num_kv_heads, num_blocks,
                                                            scale_log2, max_parts, status, plan_groups, shared_lens,
                                                            num_seqs, w.y, h, ~w.x);
    } else {
        partition_tc<T, D, G, false, B, PT, kPlanOwn>(&tm_k, &tm_v, out, ws_acc, ws_ml, q, k_new, v_new, k_cache_w,
                                                       v_cache_w, block_tables, mb, context_lens, max_ctx, 1,
                                                       num_q_heads, num_kv_heads, num_blocks, scale_log2, max_parts,
                                                       status, plan_groups, shared_lens, num_seqs, w.y, h, w.x);
    }
}

}  // namespace
