/*
 * paged_kv.h -- C ABI of the paged KV cache decode path for NVIDIA B200
 * (sm_100a).
 *
 * The KV cache of every sequence is stored in fixed-size physical blocks of
 * 16 tokens.  A per-sequence block table maps logical block j (tokens
 * 16j .. 16j+15) to a physical block anywhere in one shared pool.  Blocks are
 * handed out when a sequence needs them and returned when it finishes.
 * Sequences that share a prompt share its physical blocks, and a shared
 * block is copied before a sequence writes into it.
 *   Sources: "PagedAttention: How vLLM Serves AI Like an Operating System",
 *   sections "How It Works", "PagedAttention Memory Layout", "The Magic: No
 *   Pre-allocation" and "Copy-on-Write: Sharing KV Cache"; "vLLM
 *   Architecture and PagedAttention", "Page Table Visualization".
 *
 * Conventions shared by every call:
 *  - Memory.  The caller owns all memory.  Device buffers are raw device
 *    pointers, for example from torch.  No device call here allocates device
 *    memory; paged_attention_decode takes a caller-supplied workspace whose
 *    size paged_attention_workspace_bytes reports.  Pointers marked HOST are
 *    host memory, read before the call returns.
 *  - Streams.  `stream` is a cudaStream_t passed as void*; NULL means the
 *    legacy default stream.  Device calls only enqueue work and return
 *    without synchronising.  The decode kernels are launched with
 *    programmatic stream serialisation and release the next kernel on the
 *    stream before they finish.  An ordinary launch after them still waits
 *    for all of them; a kernel that the caller launches with programmatic
 *    serialisation itself must call cudaGridDependencySynchronize() (PTX
 *    griddepcontrol.wait) before it reads what the decode call wrote, as
 *    any such kernel must.
 *  - Cache layout.  k_cache and v_cache are each
 *    [num_blocks][num_kv_heads][block_size][head_dim], row-major, in the
 *    element type `dtype`.  Every (block, kv head) tile is therefore one
 *    contiguous block_size * head_dim run.
 *  - Slots.  Token position t of a sequence lives in physical block
 *    table[t / block_size], at offset t % block_size.  Its slot number is
 *    physical_block * block_size + offset.
 *  - Errors.  Every call returns a status code: PKV_OK or a negative
 *    PKV_ERR_*.  No exception crosses the ABI.  Arguments that the host can
 *    check are checked before anything is enqueued.  Values that only the
 *    device sees (block ids in tables, slots, context lengths) are checked by
 *    the kernels.  A kernel never reads or writes outside the buffers
 *    described here: it skips the bad item and sets a flag in a sticky
 *    per-device status word, which pkv_device_status reads.
 *  - Supported decode shapes: block_size 8, 16 or 32 (16 is the pages'
 *    choice), head_dim 64 or 128, num_q_heads / num_kv_heads in
 *    {1, 2, 4, 8}.  Element type fp32, fp16 or bf16, with fp32
 *    accumulation.  Other shapes return PKV_ERR_UNSUPPORTED.  The slot
 *    write, block copy, swap and allocator take any block size.
 */
#ifndef PAGED_KV_H
#define PAGED_KV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ------------------------------------------------------ */
#define PKV_OK 0
#define PKV_ERR_INVALID_ARG (-1)   /* bad pointer, size, shape or id         */
#define PKV_ERR_UNSUPPORTED (-2)   /* valid but not built (dtype/shape)      */
#define PKV_ERR_CUDA (-3)          /* a CUDA call failed: pkv_last_cuda_error */
#define PKV_ERR_OUT_OF_BLOCKS (-4) /* the free list cannot cover the request */
#define PKV_ERR_BAD_BLOCK (-5)     /* block id outside the pool / not held   */
#define PKV_ERR_DEVICE (-6)        /* a device-side check failed (flags set) */
#define PKV_ERR_SCRATCH_LIMIT (-7) /* the batch needs more scratch than the
                                      fixed array of the no-alloc variant   */
#define PKV_ERR_HOST_MEMORY (-8)   /* host memory for the allocator's or the
                                      plan's own bookkeeping could not be
                                      allocated; see pkv_alloc_create      */

/* ---- element types ----------------------------------------------------- */
#define PKV_F32 0
#define PKV_F16 1
#define PKV_BF16 2

/* ---- device status flags (pkv_device_status) --------------------------- */
#define PKV_DEV_BAD_BLOCK_ID 1   /* a block table entry outside [0, num_blocks) */
#define PKV_DEV_BAD_SLOT 2       /* a slot >= num_blocks * block_size           */
#define PKV_DEV_BAD_CONTEXT 4    /* context_len < 1, beyond the table row, or
                                    above the max_context_len of the launch   */
#define PKV_DEV_WAIT_TIMEOUT 8   /* an on-chip copy wait gave up (bounded spin) */
#define PKV_DEV_BAD_PLAN 16      /* a shared-prefix plan that does not fit the
                                    lengths or the launch (decode_shared)     */

/*
 * paged_kv_write -- store the new tokens' key and value rows in their slots.
 * (The cache is filled block by block as tokens arrive: "How It Works",
 *  "The Magic: No Pre-allocation".)
 *
 *  k_new, v_new   device, [num_tokens][num_kv_heads][head_dim], dtype
 *  k_cache,
 *  v_cache        device, cache layout above; rows of written slots change
 *  slot_mapping   device, int64 [num_tokens]; slot of each token.  A negative
 *                 slot skips that token (padding).  A slot at or beyond
 *                 num_blocks * block_size is skipped and raises
 *                 PKV_DEV_BAD_SLOT.  Slots must be distinct; if two tokens
 *                 name one slot, which row lands there is unspecified.
 *  head_dim * element size must be a multiple of 16 bytes, and all four
 *  data pointers must be 16-byte aligned.
 * The copy is bit-exact.  num_tokens == 0 is a no-op.
 */
int paged_kv_write(const void* k_new, const void* v_new, void* k_cache, void* v_cache,
                   const int64_t* slot_mapping, int32_t num_tokens, int32_t num_kv_heads,
                   int32_t head_dim, int32_t block_size, int32_t num_blocks, int32_t dtype,
                   void* stream);

/*
 * Split-K partitions.  Decode splits each sequence into partitions of
 * PKV_PARTITION_TOKENS tokens, one thread block each, and merges them.  A
 * launch of fp16 / bf16 with num_seqs * num_kv_heads >=
 * PKV_LONG_MIN_PAIRS_PER_SM x the device's multiprocessor count (a "large
 * batch": its (sequence, kv head) pairs alone fill the GPU) and
 * max_context_len >= PKV_LONG_MIN_CONTEXT uses PKV_PARTITION_TOKENS_WIDE
 * instead: fewer thread blocks, and fewer of them past a shorter sequence's
 * end, save more fixed per-block cost than the longer blocks add to the
 * tail.  A multi-query launch of more than 8 query rows per kv head
 * (q_len * num_q_heads / num_kv_heads > 8, the 16-row form) uses
 * PKV_PARTITION_TOKENS_WIDE on a large batch of any context length and
 * PKV_PARTITION_TOKENS_LONG otherwise: every partition ends with 16 rows of
 * output or split-K records, so fewer, longer partitions write and merge
 * less.  Shared-prefix decode follows the one-query rule.  The choice
 * depends only on these launch values, so calls with the same shape always
 * split the same way.
 */
#define PKV_PARTITION_TOKENS 512
#define PKV_PARTITION_TOKENS_LONG 1024
#define PKV_PARTITION_TOKENS_WIDE 2048
#define PKV_LONG_MIN_CONTEXT 4096
#define PKV_LONG_MIN_PAIRS_PER_SM 12

/*
 * paged_attention_partition_tokens -- the partition size, in tokens, that
 * paged_attention_decode and paged_attention_decode_mq use for this launch
 * shape on the current device (rule above).  Returns PKV_PARTITION_TOKENS,
 * PKV_PARTITION_TOKENS_WIDE, or a negative PKV_ERR_* code (no CUDA device:
 * PKV_ERR_CUDA).
 */
int32_t paged_attention_partition_tokens(int32_t num_seqs, int32_t num_kv_heads, int32_t max_context_len,
                                         int32_t dtype);

/*
 * paged_attention_mq_partition_tokens -- the same for a
 * paged_attention_decode_mq launch of q_len new tokens per sequence (rule
 * above; q_len 1 gives paged_attention_partition_tokens).  Returns
 * PKV_PARTITION_TOKENS, PKV_PARTITION_TOKENS_LONG, PKV_PARTITION_TOKENS_WIDE,
 * or a negative PKV_ERR_*
 * code: PKV_ERR_INVALID_ARG for a bad shape (num_q_heads not a multiple of
 * num_kv_heads included), PKV_ERR_CUDA with no CUDA device where the rule
 * needs the multiprocessor count.
 */
int32_t paged_attention_mq_partition_tokens(int32_t num_seqs, int32_t q_len, int32_t num_q_heads,
                                            int32_t num_kv_heads, int32_t max_context_len, int32_t dtype);

/*
 * paged_attention_workspace_bytes -- size of the workspace that
 * paged_attention_decode needs for this batch shape.  The value is 0 when
 * max_context_len fits in one partition (PKV_PARTITION_TOKENS tokens).
 * Otherwise the workspace holds, per (sequence, query head, partition), an
 * fp32 running max, an fp32 sum and head_dim fp32 partial outputs.  It is
 * sized for PKV_PARTITION_TOKENS partitions, which covers the long ones too.
 */
size_t paged_attention_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                       int32_t max_context_len);

/*
 * paged_attention_decode -- one decode step of attention over the paged
 * cache.  The result equals ordinary softmax attention over the sequence's
 * tokens laid out contiguously: the paging changes where the tokens are
 * stored, not what is computed ("Throughput Impact: The Numbers": no
 * approximations).
 *
 *   out[s][i][:] = sum_t softmax_t(scale * q[s][i] . K_s[t]) * V_s[t]
 *
 * Here t runs over the first context_lens[s] token positions of sequence s,
 * K_s[t] / V_s[t] are read for kv head i / (num_q_heads / num_kv_heads)
 * through block_tables[s], and each query head group reads each K/V block
 * once.
 *
 *  out            device, [num_seqs][num_q_heads][head_dim], dtype
 *  q              device, [num_seqs][num_q_heads][head_dim], dtype
 *  k_cache,
 *  v_cache        device, cache layout above (read only)
 *  block_tables   device, int32 [num_seqs][max_blocks_per_seq]; only the
 *                 first ceil(context_lens[s] / block_size) entries of row s
 *                 are read, the rest may hold anything.  An entry outside
 *                 [0, num_blocks) raises PKV_DEV_BAD_BLOCK_ID and block 0 is
 *                 read in its place.
 *  context_lens   device, int32 [num_seqs]: tokens to attend to, counting
 *                 the step's new token, which the caller must already have
 *                 written with paged_kv_write.  A value < 1, above
 *                 max_blocks_per_seq * block_size or above max_context_len
 *                 raises PKV_DEV_BAD_CONTEXT.  For < 1 the output row is
 *                 zero; for the other two the length is clamped.
 *  max_context_len  host int, >= every context_lens[s]; it sizes the grid,
 *                 so the host never reads device data.
 *  scale          softmax scale, usually 1/sqrt(head_dim)
 *  workspace      device, >= paged_attention_workspace_bytes(...) bytes,
 *                 256-byte aligned; may be NULL when that size is 0.  It is
 *                 scratch for the call and is overwritten.
 * Accumulation is fp32.  The result is rounded once to dtype.  It depends
 * only on the values, never on where the blocks sit in the pool: permuting
 * the physical placement gives bit-identical output.
 */
int paged_attention_decode(void* out, const void* q, const void* k_cache, const void* v_cache,
                           const int32_t* block_tables, int32_t max_blocks_per_seq,
                           const int32_t* context_lens, int32_t num_seqs, int32_t max_context_len,
                           int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                           int32_t block_size, int32_t num_blocks, float scale, int32_t dtype,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * paged_attention_decode_mq -- decode attention for q_len >= 1 new tokens per
 * sequence, optionally fused with their slot write.  Typical uses are
 * checking a draft model's proposed tokens in one pass (speculative
 * decoding: "PagedAttention & Continuous Batching: How vLLM Achieves 24x
 * Serving Throughput", item 7), and the single-token decode step with its
 * cache write in the same launch.
 *
 * context_lens[s] counts the new tokens.  New token j (0-based) sits at
 * position ctx - q_len + j and attends causally to positions
 * 0 .. ctx - q_len + j, so
 *
 *   out[s][j][i][:] = sum_{t <= ctx-q_len+j} softmax_t(scale * q[s][j][i] . K_s[t]) * V_s[t]
 *
 *  out, q         device, [num_seqs][q_len][num_q_heads][head_dim], dtype
 *  k_new, v_new   device, [num_seqs][q_len][num_kv_heads][head_dim], or
 *                 both NULL.  When given, the call first stores the new
 *                 tokens' rows in their slots, reached through block_tables
 *                 (the same bytes paged_kv_write would store), and attends
 *                 to them in the same launch.  When NULL, the caller must
 *                 already have written them.  The written blocks must not be
 *                 shared (the allocator's copy-on-write guarantees this).
 *  k_cache, v_cache  device, cache layout above; written only when k_new is
 *                 given.
 *  workspace      >= paged_attention_mq_workspace_bytes(...) bytes, 256-byte
 *                 aligned, or NULL when that size is 0.
 *  A context length below q_len raises PKV_DEV_BAD_CONTEXT and zeroes that
 *  sequence's output rows.  All other arguments and checks are as in
 *  paged_attention_decode.
 *  Limits: q_len * (num_q_heads / num_kv_heads) <= 16, because the query
 *  rows of one kv head fill one 16-row tensor-core operand.  fp32 supports
 *  only q_len == 1 without a fused write (PKV_ERR_UNSUPPORTED otherwise).
 * With q_len == 1 and no fused write, the result equals
 * paged_attention_decode bit for bit.
 */
size_t paged_attention_mq_workspace_bytes(int32_t num_seqs, int32_t q_len, int32_t num_q_heads,
                                          int32_t head_dim, int32_t max_context_len);
int paged_attention_decode_mq(void* out, const void* q, const void* k_new, const void* v_new,
                              void* k_cache, void* v_cache, const int32_t* block_tables,
                              int32_t max_blocks_per_seq, const int32_t* context_lens,
                              int32_t num_seqs, int32_t q_len, int32_t max_context_len,
                              int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                              int32_t block_size, int32_t num_blocks, float scale, int32_t dtype,
                              void* workspace, size_t workspace_bytes, void* stream);

/*
 * Shared-prefix decode.  Samples forked from one prompt (and requests that
 * found the same cached prefix) hold the same physical blocks for their
 * common positions ("Copy-on-Write: Sharing KV Cache", "Parallel Sampling"
 * and "Prefix Caching").  The pages share those blocks to save memory;
 * these two calls also read them once per step instead of once per sample.
 * The result is the same attention as paged_attention_decode, within its
 * rounding.
 *
 * pkv_shared_prefix_plan -- host only.  From the host copies of a batch's
 * block tables and context lengths, find groups: runs of consecutive
 * sequences (in batch order) whose tables start with the same physical
 * blocks.  For each group it picks x, the shared length: a multiple of
 * block_size, below every member's length, and covered by the blocks the
 * members have in common.
 *
 *  block_tables   host, int32 [num_seqs][max_blocks_per_seq]
 *  context_lens   host, int32 [num_seqs]; each in [1, max_blocks_per_seq *
 *                 block_size], else PKV_ERR_INVALID_ARG
 *  max_group      members per group, at most; for decode:
 *                 PKV_SHARED_MAX_ROWS / (num_q_heads / num_kv_heads).  A
 *                 longer run splits into several groups.
 *  min_shared_tokens  a group forms only where x >= this (and x >= one block)
 *  part_tokens    the decode launch's partition size:
 *                 paged_attention_partition_tokens(num_seqs, num_kv_heads,
 *                 max_context_len, dtype)
 *  groups_out     host, int32 [num_seqs][2]: (first sequence, members) of each
 *                 group, in batch order; *num_groups_out of them are set
 *  shared_lens_out  host, int32 [num_seqs]: the group's x for each member,
 *                 0 for a sequence in no group
 *  work_out       host, int32 [work_cap][2]: the decode launch's work items,
 *                 *num_work_out of them.  (~g, p) is partition p (of
 *                 part_tokens positions) of group g's shared positions
 *                 [0, x); (s, p) is partition p of sequence s's own positions
 *                 [x, ctx).  Longest first.  work_out NULL: only
 *                 *num_work_out is set (a size query).  A work_cap below the
 *                 count returns PKV_ERR_INVALID_ARG with *num_work_out set.
 *  max_shared_len_out  max of shared_lens_out (0 if no group)
 *  max_own_len_out  max over sequences of context_lens[s] - shared_lens_out[s]
 * Groups have at least 2 members and never overlap.  The result depends only
 * on the arguments.  PKV_ERR_HOST_MEMORY if the work list's host scratch
 * cannot be allocated.
 */
#define PKV_SHARED_MAX_ROWS 16
int pkv_shared_prefix_plan(const int32_t* block_tables, int32_t max_blocks_per_seq,
                           const int32_t* context_lens, int32_t num_seqs, int32_t block_size,
                           int32_t max_group, int32_t min_shared_tokens, int32_t part_tokens,
                           int32_t* groups_out, int32_t* num_groups_out, int32_t* shared_lens_out,
                           int32_t* work_out, int32_t work_cap, int32_t* num_work_out,
                           int32_t* max_shared_len_out, int32_t* max_own_len_out);

/*
 * pkv_shared_prefix_order -- host only.  A batch order in which sequences
 * whose tables start with the same physical blocks are adjacent, for a
 * serving loop whose batch interleaves requests that share a cached prefix
 * ("Prefix Caching") or samples of several prompts: pkv_shared_prefix_plan
 * groups only runs of consecutive sequences.  The order sorts the sequences
 * by the ids of their shareable blocks (those wholly below their last
 * position, up to the first negative entry) lexicographically, and is
 * stable: sequences with equal rows keep their batch order.
 *
 *  block_tables, context_lens  as pkv_shared_prefix_plan (host int32)
 *  order_out      host, int64 [num_seqs]: position i of the reordered batch
 *                 holds sequence order_out[i] (a permutation of 0..num_seqs-1)
 * Returns PKV_OK, PKV_ERR_INVALID_ARG (a length outside [1,
 * max_blocks_per_seq * block_size], bad sizes, null pointers) or
 * PKV_ERR_HOST_MEMORY.
 */
int pkv_shared_prefix_order(const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                            int32_t num_seqs, int32_t block_size, int64_t* order_out);

/*
 * paged_attention_decode_shared -- one decode step (one new token per
 * sequence, optionally fused with its slot write) with a plan from
 * pkv_shared_prefix_plan.  Computes the attention paged_attention_decode_mq
 * with q_len 1 computes, within its tolerance (the bits equal it where no
 * group forms; a group's shared partitions round differently):
 *
 *   out[s][i][:] = sum_{t < ctx_s} softmax_t(scale * q[s][i] . K_s[t]) * V_s[t]
 *
 * but in two passes, run by one launch over the plan's work list.  The group
 * pass reads the blocks of positions [0, x) of a group once, through the
 * first member's table, and attends all members' query heads to them
 * together (members x (num_q_heads / num_kv_heads) rows: at most 8 in the
 * 8-column tensor-core form, up to 16 in the 16-row form).  Each sequence's
 * own pass reads its positions [x, ctx), and the split-K reduce merges both.
 *
 *  groups         device, int32 [num_groups][2], as groups_out; may be NULL
 *                 when num_groups is 0
 *  shared_lens    device, int32 [num_seqs], as shared_lens_out
 *  work           device, int32 [num_work][2], as work_out, 8-byte aligned;
 *                 num_work (>= 1) sizes the grid, so the host never reads
 *                 device data
 *  work_part_tokens  the part_tokens the list was made for; it must equal
 *                 this launch's partition size, else PKV_ERR_INVALID_ARG
 *  workspace      >= paged_attention_shared_workspace_bytes(...) bytes,
 *                 256-byte aligned (never NULL)
 *  All other arguments are those of paged_attention_decode_mq with q_len 1.
 * The plan is a promise about the tables: the members of a group hold the
 * same blocks for positions [0, x).  A plan made before a table changed (a
 * copy-on-write repoint, an eviction) breaks it.  The group pass checks it
 * on the device: each covered member's table entries over the partition's
 * blocks are compared with the first member's.  A member that differs
 * raises PKV_DEV_BAD_PLAN and gets no result: the reduce leaves its output
 * rows unwritten, and the other members' rows are still computed.  The call
 * also checks: a work item naming a group or sequence outside the batch or a
 * partition past max_context_len, a group with more than
 * PKV_SHARED_MAX_ROWS rows, or one whose x does not fit the cache or
 * max_context_len raises PKV_DEV_BAD_PLAN and is skipped; a member whose own
 * x differs from its group's, or is not below its length, raises
 * PKV_DEV_BAD_PLAN.  Outputs of sequences named in such
 * a plan are then unspecified (never out-of-bounds accesses).  A sequence in
 * no group with x = 0 is computed whole by its own pass.  fp32 caches return
 * PKV_ERR_UNSUPPORTED.
 */
size_t paged_attention_shared_workspace_bytes(int32_t num_seqs, int32_t num_q_heads, int32_t head_dim,
                                              int32_t max_context_len);
int paged_attention_decode_shared(void* out, const void* q, const void* k_new, const void* v_new,
                                  void* k_cache, void* v_cache, const int32_t* block_tables,
                                  int32_t max_blocks_per_seq, const int32_t* context_lens, int32_t num_seqs,
                                  int32_t max_context_len, const int32_t* groups, int32_t num_groups,
                                  const int32_t* shared_lens, const int32_t* work, int32_t num_work,
                                  int32_t work_part_tokens, int32_t num_q_heads, int32_t num_kv_heads,
                                  int32_t head_dim, int32_t block_size, int32_t num_blocks, float scale, int32_t dtype,
                                  void* workspace, size_t workspace_bytes, void* stream);

/*
 * pkv_debug_shared_occupancy -- test hook: resident thread blocks per SM of
 * paged_attention_decode_shared's kernel for this instantiation (fp16 /
 * bf16), as the CUDA occupancy calculator reports it with the kernel's
 * shared memory; long_partitions != 0 selects the PKV_PARTITION_TOKENS_WIDE
 * variant, 0 the PKV_PARTITION_TOKENS one.  Launches nothing.  Returns
 * PKV_ERR_UNSUPPORTED for shapes the call does not build.
 */
int pkv_debug_shared_occupancy(int32_t dtype, int32_t head_dim, int32_t group, int32_t block_size,
                               int32_t long_partitions, int32_t* ctas_per_sm);

/*
 * paged_attention_decode_noalloc -- paged_attention_decode without a
 * caller-supplied workspace, for callers that cannot allocate device memory
 * when they decode: runtimes whose device memory is one fixed arena handed
 * out at start-up (nothing is left to allocate from), and embedders that
 * must never call the CUDA allocator (cudaMalloc and cudaFree can
 * synchronise the device and take a process-wide lock, which a latency-
 * bound decode loop cannot afford).  It has no counterpart in the pages; it
 * is an interface convenience of this library.
 *
 * The arguments and the result are those of paged_attention_decode.  The
 * split-K scratch comes from one fixed array of PKV_NOALLOC_SCRATCH_BYTES
 * (64 MiB) in the library's own device memory.  Every GPU that loads the
 * library's decode module holds that array until the process exits.  The
 * call allocates nothing: no cudaMalloc, no cudaFree, no allocating library
 * routine.
 *
 *  - Errors: a call that paged_attention_decode would reject for any
 *    workspace gets the same code here.  A valid call whose
 *    paged_attention_workspace_bytes(num_seqs, num_q_heads, head_dim,
 *    max_context_len) exceeds PKV_NOALLOC_SCRATCH_BYTES returns
 *    PKV_ERR_SCRATCH_LIMIT and enqueues nothing.  Example that fits: 128
 *    sequences x 32 query heads x 8192 tokens at head_dim 128 need 34 MB.
 *  - Set-up: the first call on a device resolves the array's device address
 *    (cudaGetSymbolAddress, with that device current) and keeps it.  Like
 *    every decode entry point, the first call of each launch shape (dtype,
 *    head_dim, query heads per kv head, block size and partition size) also
 *    sets that kernel's shared-memory limit.  Make those first calls before
 *    any stream capture.
 *  - Lifetime: the address is kept for the life of the process, like the
 *    status word's.  Do not use the library across a cudaDeviceReset (or any
 *    other destruction of the device's primary context).
 *  - Sharing: all calls on one device share the one array, which keeps the
 *    last call's contents.  Nothing in it needs to start at zero: each call
 *    writes every scratch entry before reading it.  Calls that overlap on
 *    the GPU (for example on two streams without ordering between them)
 *    race on the array; order them on one stream or by events.
 */
#define PKV_NOALLOC_SCRATCH_BYTES 67108864
int paged_attention_decode_noalloc(void* out, const void* q, const void* k_cache,
                                   const void* v_cache, const int32_t* block_tables,
                                   int32_t max_blocks_per_seq, const int32_t* context_lens,
                                   int32_t num_seqs, int32_t max_context_len, int32_t num_q_heads,
                                   int32_t num_kv_heads, int32_t head_dim, int32_t block_size,
                                   int32_t num_blocks, float scale, int32_t dtype, void* stream);

/*
 * block_copy -- copy-on-write copies: for each pair (src, dst), physical
 * block dst becomes a copy of block src, in the keys and the values of
 * every kv head.  ("Copy-on-Write: Sharing KV Cache": a request that must
 * modify a shared block copies it first.)
 *
 *  pairs          HOST, int64 [num_pairs][2] as (src, dst).  The whole list
 *                 is checked before any copy is enqueued:
 *                   - ids must lie in [0, num_blocks);
 *                   - src != dst;
 *                   - no dst may appear twice;
 *                   - no dst may also be a src in the same call.
 *                 A list that breaks any rule, whose result would depend on
 *                 copy order, returns PKV_ERR_INVALID_ARG.
 *  The copy is bit-exact.  num_pairs == 0 is a no-op.  Both cache pointers
 *  must be 16-byte aligned.
 */
int block_copy(void* k_cache, void* v_cache, const int64_t* pairs, int32_t num_pairs,
               int32_t num_kv_heads, int32_t head_dim, int32_t block_size, int32_t num_blocks,
               int32_t dtype, void* stream);

/*
 * swap_blocks_out / swap_blocks_in -- move whole blocks (keys and values of
 * every kv head) between the device cache and host memory, so a preempted
 * sequence can give its device blocks back and later resume where it stopped.
 * ("vLLM Architecture": the scheduler preempts low-priority requests by
 * swapping their blocks to CPU memory.)
 *
 *  block_ids      HOST, int64 [n], each in [0, num_blocks).  For swap-in,
 *                 no id may appear twice (PKV_ERR_INVALID_ARG).
 *  host_k, host_v HOST memory, pinned (page-locked) and mapped into the
 *                 device's address space (cudaHostAlloc / cudaMallocHost, or
 *                 torch pin_memory()); each [n][num_kv_heads][block_size]
 *                 [head_dim] of dtype.  Slot i holds block block_ids[i].
 *                 Pageable memory returns PKV_ERR_INVALID_ARG.
 *  swap_blocks_out copies device -> host; swap_blocks_in host -> device.
 *  One kernel launch per 1024 blocks moves the data over the host link.
 *  The call is asynchronous on `stream`; the host buffers must stay alive
 *  and untouched until the stream reaches this point.  The copy is bit-exact.
 */
int swap_blocks_out(const void* k_cache, const void* v_cache, const int64_t* block_ids, int32_t n,
                    void* host_k, void* host_v, int32_t num_kv_heads, int32_t head_dim,
                    int32_t block_size, int32_t num_blocks, int32_t dtype, void* stream);
int swap_blocks_in(void* k_cache, void* v_cache, const int64_t* block_ids, int32_t n,
                   const void* host_k, const void* host_v, int32_t num_kv_heads, int32_t head_dim,
                   int32_t block_size, int32_t num_blocks, int32_t dtype, void* stream);

/*
 * pkv_slot_mapping -- HOST helper: slots_out[s] = slot of token position
 * positions[s] of sequence s, given its block-table row (host int32
 * [num_seqs][max_blocks_per_seq]).  Returns PKV_ERR_INVALID_ARG for a
 * position whose logical block lies beyond the row, and PKV_ERR_BAD_BLOCK
 * for a negative table entry.  A negative position yields slot -1.
 */
int pkv_slot_mapping(const int32_t* block_tables, int32_t max_blocks_per_seq,
                     const int32_t* positions, int32_t num_seqs, int32_t block_size,
                     int64_t* slots_out);

/*
 * pkv_device_status -- read, and if `clear` is nonzero reset, the sticky
 * status word of `device`.  This synchronises that device.  *flags_out
 * receives an OR of PKV_DEV_* flags, or 0.
 */
int pkv_device_status(int32_t device, int32_t* flags_out, int32_t clear);

/*
 * pkv_debug_wait_timeout -- test hook for failure detection.  It launches
 * one warp that waits, through the same bounded wait the decode kernels
 * use, on an mbarrier that nothing arrives on.  After limit_ns nanoseconds
 * (at most 1 s) the wait gives up and sets PKV_DEV_WAIT_TIMEOUT in the
 * status word.  The kernel then exits normally and the context stays
 * usable.  It never hangs and never faults.
 */
int pkv_debug_wait_timeout(int64_t limit_ns, void* stream);

/* The last cudaError_t seen by any call in this thread, as an int. */
int pkv_last_cuda_error(void);

/*
 * pkv_debug_decode_occupancy -- test hook: thread blocks per SM that the
 * decode partition kernel of this configuration keeps resident on the
 * current device (cudaOccupancyMaxActiveBlocksPerMultiprocessor, with the
 * kernel's own shared memory).  group = num_q_heads / num_kv_heads; q_len > 1
 * selects the multi-query kernel; long_partitions != 0 the
 * PKV_PARTITION_TOKENS_WIDE variant (fp16 / bf16), 0 the other one
 * (PKV_PARTITION_TOKENS, or PKV_PARTITION_TOKENS_LONG for more than 8 rows
 * per kv head).  Enqueues nothing.  A
 * tensor-core kernel is built for 3 per SM (its shared memory and 168
 * registers); fewer means a build lost a third of the bytes in flight.
 */
int pkv_debug_decode_occupancy(int32_t dtype, int32_t head_dim, int32_t group, int32_t q_len,
                               int32_t block_size, int32_t long_partitions, int32_t* ctas_per_sm);

/* A static, human-readable name for a PKV_* status code. */
const char* pkv_status_string(int status);

/* ======================================================================== *
 * Host block allocator: pool of physical blocks, free list, reference
 * counts, per-sequence block tables, and copy-on-write decisions.
 * ("How It Works"; "The Magic: No Pre-allocation"; "Copy-on-Write: Sharing
 *  KV Cache", "Parallel Sampling" and "Prefix Caching"; "vLLM
 *  Architecture": the KV cache manager that allocates and frees blocks.)
 *
 * Policy:
 *  - The free list is a stack.  initial_order gives the order in which blocks
 *    are first handed out (NULL = 0, 1, 2, ...).  A freed block goes on top.
 *  - A sequence gets a new block exactly when its token count crosses a
 *    multiple of block_size, so n tokens hold ceil(n / block_size) blocks.
 *  - Freeing a sequence releases its blocks from the last logical block to
 *    the first; a block returns to the free list when its count reaches 0.
 *  - Before a sequence writes into a partially filled block that others
 *    also hold (count > 1), it moves to a fresh private block and reports the
 *    (src, dst) copy pair.  The last holder (count == 1) writes in place.
 *  - A call that cannot get every block it needs returns
 *    PKV_ERR_OUT_OF_BLOCKS and changes nothing.
 *  - No C++ exception leaves a call.  If the allocator cannot get host
 *    memory for its own bookkeeping the call returns PKV_ERR_HOST_MEMORY.
 *    Creation, adding a sequence, appends, forks, prefix sharing, prompt
 *    admission and swap-in allocate before they change anything, so such a
 *    failure leaves the allocator as it was (prompt admission may then cache
 *    fewer of the prompt's blocks, which only costs later lookups).  After a
 *    failing free or swap-out, destroy the allocator.
 * Sequence ids are arbitrary int64 values chosen by the caller.
 * One allocator is not thread-safe; use one per thread or lock around it.
 * ======================================================================== */
typedef struct pkv_allocator pkv_allocator;

typedef struct pkv_alloc_stats {
    int32_t num_blocks;
    int32_t free_blocks;
    int32_t used_blocks;          /* num_blocks - free_blocks                 */
    int32_t shared_blocks;        /* blocks with reference count > 1          */
    int64_t num_seqs;
    int64_t num_tokens;           /* sum of the sequences' token counts       */
    int64_t fragmentation_tokens; /* sum over sequences of unused slots in
                                     their blocks (at most block_size - 1 each) */
} pkv_alloc_stats;

/* num_blocks >= 0, block_size >= 1; initial_order: HOST int32 [num_blocks]
 * permutation of 0..num_blocks-1, or NULL.  *out receives the handle. */
int pkv_alloc_create(int32_t num_blocks, int32_t block_size, const int32_t* initial_order,
                     pkv_allocator** out);
void pkv_alloc_destroy(pkv_allocator* a);

/* Register an empty sequence.  An id already in use -> PKV_ERR_INVALID_ARG. */
int pkv_seq_add(pkv_allocator* a, int64_t seq);

/* Reserve slots for n >= 0 new tokens of `seq`.  slots_out (HOST int64 [n],
 * may be NULL) receives their slots in order.  If the first write lands in
 * a shared partial block, the sequence moves to a fresh block first:
 * *cow_out = 1 and cow_pair_out (HOST int64 [2], may be NULL) = (src, dst).
 * Otherwise *cow_out = 0.  cow_out may be NULL. */
int pkv_seq_append_tokens(pkv_allocator* a, int64_t seq, int32_t n, int64_t* slots_out,
                          int64_t* cow_pair_out, int32_t* cow_out);

/* One new token for each of n_seqs distinct sequences, in order (one
 * decode step).  slots_out: HOST int64 [n_seqs].  cow_pairs_out: HOST int64
 * [n_seqs][2], may be NULL.  The first *n_cow_out rows receive the copy
 * pairs.  All-or-nothing: if the free list cannot cover every sequence,
 * nothing changes. */
int pkv_batch_append_one(pkv_allocator* a, const int64_t* seqs, int32_t n_seqs,
                         int64_t* slots_out, int64_t* cow_pairs_out, int32_t* n_cow_out);

/* Release a finished sequence ("its pages are immediately freed"). */
int pkv_seq_free(pkv_allocator* a, int64_t seq);

/* New sequence `child` sharing every block of `parent` (parallel sampling). */
int pkv_seq_fork(pkv_allocator* a, int64_t parent, int64_t child);

/* Point an empty sequence at existing allocated blocks (a shared system
 * prompt).  blocks: HOST int32 [n_blocks], each with count >= 1.  n_tokens
 * must satisfy ceil(n_tokens / block_size) == n_blocks. */
int pkv_seq_share_prefix(pkv_allocator* a, int64_t seq, const int32_t* blocks, int32_t n_blocks,
                         int32_t n_tokens);

/* Copy the block table of `seq` into out (HOST int32 [cap]).  *n_out receives
 * its length.  If the table is longer than cap, the call returns
 * PKV_ERR_INVALID_ARG and writes nothing. */
int pkv_seq_block_table(const pkv_allocator* a, int64_t seq, int32_t* out, int32_t cap,
                        int32_t* n_out);
int pkv_seq_num_tokens(const pkv_allocator* a, int64_t seq, int32_t* out);

/* Block tables and context lengths of n_seqs sequences, ready for
 * paged_attention_decode.  tables_out: HOST int32
 * [n_seqs][max_blocks_per_seq]; entries past a table's end are set to pad,
 * or left as they are when pad is PKV_TABLE_KEEP_TAIL (decode never reads
 * them).  A serving loop that refills the same buffer every step passes
 * PKV_TABLE_KEEP_TAIL and writes only the live entries.
 * context_lens_out: HOST int32 [n_seqs], may be NULL. */
#define PKV_TABLE_KEEP_TAIL (-2147483647 - 1)
int pkv_batch_tables(const pkv_allocator* a, const int64_t* seqs, int32_t n_seqs,
                     int32_t* tables_out, int32_t max_blocks_per_seq, int32_t pad,
                     int32_t* context_lens_out);

/* Prefix cache ("Prefix Caching": a system prompt identical across
 * requests is stored once; "PagedAttention & Continuous Batching…",
 * item 5).  pkv_seq_append_prompt gives an empty sequence its prompt
 * (token_ids: HOST int32 [n]).  It walks the prompt's full blocks in order
 * and reuses every leading block whose content is already cached.  A
 * block's identity is the block before it, that block's generation and its
 * own block_size token ids, compared exactly.  From the first miss on it
 * takes fresh blocks and makes each new full block findable.  slots_out
 * (HOST int64 [n], may be NULL) receives -1 for the cached tokens (their
 * K/V is already in place) and the slot of every other token.
 * *n_cached_out receives the number of cached tokens, a multiple of
 * block_size.  A cached block that no sequence uses any more stays
 * findable.  It is handed out again (evicted, least recently released
 * first) only when no never-cached block is free; pkv_num_free and
 * pkv_free_list count it as free.  All-or-nothing:
 * PKV_ERR_OUT_OF_BLOCKS changes nothing. */
typedef struct pkv_prefix_stats {
    int32_t cached_blocks;      /* blocks findable by content                 */
    int32_t evictable_blocks;   /* of those, used by no sequence              */
    int64_t prompts;            /* pkv_seq_append_prompt calls with a full block */
    int64_t prompts_with_hits;  /* of those, calls that reused >= 1 block     */
    int64_t hit_tokens;         /* prompt tokens served from the cache        */
    int64_t evictions;          /* cached blocks reclaimed for new content    */
} pkv_prefix_stats;
int pkv_seq_append_prompt(pkv_allocator* a, int64_t seq, const int32_t* token_ids, int32_t n,
                          int64_t* slots_out, int32_t* n_cached_out);
int pkv_prefix_cache_stats(const pkv_allocator* a, pkv_prefix_stats* out);

/* Preemption.  pkv_seq_swap_out lists the sequence's blocks in logical
 * order in blocks_out (HOST int32 [cap]; *n_out = count), for
 * swap_blocks_out.  It then releases them like pkv_seq_free, but the
 * sequence stays registered, swapped out, with its token count.
 * pkv_seq_swap_in takes fresh blocks for a swapped-out sequence in one
 * all-or-nothing step (PKV_ERR_OUT_OF_BLOCKS changes nothing) and lists
 * them in logical order, the destinations for swap_blocks_in.  While a
 * sequence is swapped out, append, fork, share_prefix and
 * pkv_batch_tables refuse it (PKV_ERR_INVALID_ARG); pkv_seq_free drops it. */
int pkv_seq_swap_out(pkv_allocator* a, int64_t seq, int32_t* blocks_out, int32_t cap, int32_t* n_out);
int pkv_seq_swap_in(pkv_allocator* a, int64_t seq, int32_t* blocks_out, int32_t cap, int32_t* n_out);
int pkv_seq_is_swapped(const pkv_allocator* a, int64_t seq, int32_t* out);

int32_t pkv_num_free(const pkv_allocator* a);
/* The free blocks in the order they will be handed out (HOST int32 [cap]). */
int pkv_free_list(const pkv_allocator* a, int32_t* out, int32_t cap, int32_t* n_out);
/* Reference count of a block (0 = free); -1 for an id outside the pool. */
int32_t pkv_refcount(const pkv_allocator* a, int32_t block);
int pkv_alloc_get_stats(const pkv_allocator* a, pkv_alloc_stats* out);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_KV_H */
