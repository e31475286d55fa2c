/*
 * A plain C99 program that uses the library only through include/paged_kv.h.
 * It shows that the boundary compiles as C, links, and works without Python.
 *
 *   abi_consumer host  host-side calls only: the allocator on the pages'
 *                      copy-on-write example, slot mapping, workspace sizes,
 *                      argument checks that happen before any device work.
 *   abi_consumer gpu   (built with -DWITH_CUDA) one decode step on device 0
 *                      through the C ABI on cudaMalloc'd buffers: block copy,
 *                      slot write, split-K decode; then shared-prefix decode
 *                      of the same step with the forked sample beside its
 *                      parent.  The results are checked against the fp64
 *                      oracle library (test infrastructure): the cache bit
 *                      for bit, attention within 2e-3 + 1e-2 |ref| per
 *                      element.
 *
 * Exit code 0 when every check passes; otherwise the first failing check is
 * printed and the exit code is 1.
 */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "paged_kv.h"

#define CHECK(cond)                                                                   \
    do {                                                                              \
        if (!(cond)) {                                                                \
            fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
            return 1;                                                                 \
        }                                                                             \
    } while (0)

/* ---- host-side calls ---------------------------------------------------- */
static int host_checks(void)
{
    /* 12 blocks of 16 tokens, handed out in a scattered order */
    const int32_t order[12] = {7, 1, 10, 4, 0, 9, 3, 11, 6, 2, 8, 5};
    pkv_allocator* a = NULL;
    int64_t slots[64];
    int64_t pair[2];
    int32_t cow = -1;
    int32_t table[8];
    int32_t n = 0;
    int32_t t;

    CHECK(pkv_alloc_create(12, 16, order, &a) == PKV_OK && a != NULL);
    CHECK(pkv_seq_add(a, 0) == PKV_OK);
    /* 40 tokens fill two blocks and part of a third: the 17th and 33rd
       tokens open new blocks */
    CHECK(pkv_seq_append_tokens(a, 0, 40, slots, pair, &cow) == PKV_OK && cow == 0);
    CHECK(pkv_seq_block_table(a, 0, table, 8, &n) == PKV_OK && n == 3);
    for (t = 0; t < 40; ++t) CHECK(slots[t] == (int64_t)table[t / 16] * 16 + t % 16);
    CHECK(pkv_num_free(a) == 9);

    /* a forked sample shares every block of its parent */
    CHECK(pkv_seq_fork(a, 0, 1) == PKV_OK);
    CHECK(pkv_refcount(a, table[0]) == 2 && pkv_refcount(a, table[2]) == 2);
    {
        /* the sample's next token goes into the shared, partly filled block:
           it gets a private copy first, and the parent keeps the original */
        const int64_t seqs[1] = {1};
        int64_t s1 = -1;
        int64_t pairs[2] = {-1, -1};
        int32_t ncow = 0;
        int32_t child[8];
        int32_t nc = 0;
        CHECK(pkv_batch_append_one(a, seqs, 1, &s1, pairs, &ncow) == PKV_OK && ncow == 1);
        CHECK(pairs[0] == table[2] && pairs[1] != table[2]);
        CHECK(pkv_refcount(a, table[2]) == 1 && pkv_refcount(a, (int32_t)pairs[1]) == 1);
        CHECK(pkv_seq_block_table(a, 1, child, 8, &nc) == PKV_OK && nc == 3);
        CHECK(child[0] == table[0] && child[1] == table[1] && child[2] == (int32_t)pairs[1]);
        CHECK(s1 == pairs[1] * 16 + 40 % 16);
    }
    {
        const int32_t pos[2] = {39, -1};
        int64_t sm[2] = {0, 0};
        int32_t two[6];
        memcpy(two, table, 3 * sizeof(int32_t));
        memcpy(two + 3, table, 3 * sizeof(int32_t));
        CHECK(pkv_slot_mapping(two, 3, pos, 2, 16, sm) == PKV_OK);
        CHECK(sm[0] == (int64_t)table[2] * 16 + 7 && sm[1] == -1);
    }
    /* freeing both sequences returns every block */
    CHECK(pkv_seq_free(a, 0) == PKV_OK && pkv_seq_free(a, 1) == PKV_OK);
    CHECK(pkv_num_free(a) == 12);
    pkv_alloc_destroy(a);

    /* one partition needs no workspace; two need (max, sum, partial) records */
    CHECK(paged_attention_workspace_bytes(4, 32, 128, PKV_PARTITION_TOKENS) == 0);
    CHECK(paged_attention_workspace_bytes(2, 32, 128, 1000) == (size_t)2 * 32 * 2 * 130 * 4);

    /* rejected on the host before anything is enqueued */
    CHECK(paged_kv_write(NULL, NULL, NULL, NULL, NULL, 4, 8, 128, 16, 10, 7, NULL) == PKV_ERR_UNSUPPORTED);
    CHECK(paged_kv_write(NULL, NULL, NULL, NULL, NULL, 4, 8, 128, 16, 10, PKV_BF16, NULL) ==
          PKV_ERR_INVALID_ARG);
    CHECK(paged_attention_decode(NULL, NULL, NULL, NULL, NULL, 4, NULL, 2, 100, 32, 8, 96, 16, 10, 0.1f, PKV_BF16,
                                 NULL, 0, NULL) == PKV_ERR_UNSUPPORTED);
    {
        const int64_t bad[2] = {3, 3};  /* a block copied onto itself */
        CHECK(block_copy(NULL, NULL, bad, 1, 2, 128, 16, 8, PKV_BF16, NULL) == PKV_ERR_INVALID_ARG);
    }
    {
        /* shared-prefix plan on the pages' parallel-sampling example: four
           outputs share prompt blocks 0-5 and own two blocks each */
        int32_t tabs[4 * 8], lens4[4], groups[8], shared[4], work[2 * 16];
        int32_t ng = 0, nw = 0, mxs = 0, mxo = 0, j, k;
        for (j = 0; j < 4; ++j) {
            for (k = 0; k < 6; ++k) tabs[j * 8 + k] = k;
            tabs[j * 8 + 6] = 6 + 2 * j;
            tabs[j * 8 + 7] = 7 + 2 * j;
            lens4[j] = 6 * 16 + 20;
        }
        CHECK(pkv_shared_prefix_plan(tabs, 8, lens4, 4, 16, 4, 16, 512, groups, &ng, shared, work, 16, &nw, &mxs,
                                     &mxo) == PKV_OK);
        CHECK(ng == 1 && groups[0] == 0 && groups[1] == 4 && mxs == 96 && mxo == 20);
        for (j = 0; j < 4; ++j) CHECK(shared[j] == 96);
        CHECK(nw == 5);                 /* the group's shared partition, then one own partition each */
        CHECK(work[0] == ~0 && work[1] == 0);
        CHECK(paged_attention_shared_workspace_bytes(2, 32, 128, 1000) == (size_t)2 * 32 * 3 * 130 * 4);
    }
    /* a multi-query launch of more than 8 rows per kv head takes the long or the wide partitions, by
       the device's SM count (no device: PKV_ERR_CUDA); up to 8 rows and short contexts need no device */
    {
        const int32_t mq = paged_attention_mq_partition_tokens(64, 16, 40, 40, 600, PKV_F16);
        CHECK(mq == PKV_PARTITION_TOKENS_LONG || mq == PKV_PARTITION_TOKENS_WIDE || mq == PKV_ERR_CUDA);
    }
    CHECK(paged_attention_mq_partition_tokens(8, 2, 16, 4, 100, PKV_BF16) == PKV_PARTITION_TOKENS);
    CHECK(paged_attention_mq_partition_tokens(8, 16, 40, 7, 100, PKV_F16) == PKV_ERR_INVALID_ARG);
    CHECK(strcmp(pkv_status_string(PKV_OK), "ok") == 0);
    CHECK(strcmp(pkv_status_string(PKV_ERR_OUT_OF_BLOCKS), "unknown status") != 0);
    return 0;
}

#ifdef WITH_CUDA
#include <cuda_runtime.h>

/* The fp64 oracle (liboracle.so, test infrastructure).  Element codes there:
   0 fp32, 1 fp16, 2 bf16. */
int oracle_paged_decode(double* out, const void* q, const void* k_cache, const void* v_cache,
                        const int32_t* block_tables, int32_t max_blocks_per_seq, const int32_t* context_lens,
                        int32_t num_seqs, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                        int32_t block_size, int32_t num_blocks, double scale, int dtype);
int oracle_kv_write(void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                    const int64_t* slot_mapping, int32_t num_tokens, int32_t num_kv_heads, int32_t head_dim,
                    int32_t block_size, int32_t num_blocks, int dtype);
int oracle_block_copy(void* k_cache, void* v_cache, const int64_t* pairs, int32_t n, int32_t num_kv_heads,
                      int32_t head_dim, int32_t block_size, int32_t num_blocks, int dtype);

/* inputs: a 64-bit linear congruential generator, bf16 by truncation */
static uint64_t g_rng = 398u;

static uint16_t rand_bf16(void)
{
    float f;
    uint32_t u;
    g_rng = g_rng * 6364136223846793005ull + 1442695040888963407ull;
    f = (float)((int32_t)(g_rng >> 33) % 20001 - 10000) / 5000.0f; /* in [-2, 2] */
    memcpy(&u, &f, 4);
    return (uint16_t)(u >> 16);
}

static double bf16_value(uint16_t b)
{
    const uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

#define CUDA_CHECK(call) CHECK((call) == cudaSuccess)

static int gpu_checks(void)
{
    enum { S = 4, HQ = 8, HKV = 2, D = 128, B = 16, NB = 256, MB = 128 };
    const int32_t prompt[S - 1] = {699, 32, 1499}; /* sequence 3 is a fork of sequence 0 */
    const size_t blk_elems = (size_t)HKV * B * D;
    const size_t cache_bytes = NB * blk_elems * 2;
    int32_t order[NB];
    pkv_allocator* a = NULL;
    int64_t seqs[S] = {0, 1, 2, 3};
    int64_t slots[S];
    int64_t pairs[2 * S];
    int32_t ncow = 0;
    int32_t tables[S * MB];
    int32_t lens[S];
    uint16_t *hk, *hv, *hq, *hkn, *hvn, *hout, *gk, *gv;
    double* ref;
    void *dk, *dv, *dq, *dkn, *dvn, *dout, *dws = NULL, *dtab, *dlen, *dslots;
    size_t ws_bytes;
    int32_t max_ctx = 0, flags = -1;
    int i, s;
    size_t e;

    /* allocator: a scattered pool, three prompts, one fork, then one new
       token for every sequence (the fork's first token copies a block) */
    for (i = 0; i < NB; ++i) order[i] = (i * 97 + 13) % NB;
    CHECK(pkv_alloc_create(NB, B, order, &a) == PKV_OK);
    for (s = 0; s < S - 1; ++s) {
        CHECK(pkv_seq_add(a, s) == PKV_OK);
        CHECK(pkv_seq_append_tokens(a, s, prompt[s], NULL, NULL, NULL) == PKV_OK);
    }
    CHECK(pkv_seq_fork(a, 0, 3) == PKV_OK);
    CHECK(pkv_batch_append_one(a, seqs, S, slots, pairs, &ncow) == PKV_OK && ncow == 1);
    CHECK(pkv_batch_tables(a, seqs, S, tables, MB, -1, lens) == PKV_OK);
    for (s = 0; s < S; ++s) max_ctx = lens[s] > max_ctx ? lens[s] : max_ctx;

    /* host data */
    hk = malloc(cache_bytes);
    hv = malloc(cache_bytes);
    gk = malloc(cache_bytes);
    gv = malloc(cache_bytes);
    hq = malloc((size_t)S * HQ * D * 2);
    hout = malloc((size_t)S * HQ * D * 2);
    hkn = malloc((size_t)S * HKV * D * 2);
    hvn = malloc((size_t)S * HKV * D * 2);
    ref = malloc((size_t)S * HQ * D * sizeof(double));
    CHECK(hk && hv && gk && gv && hq && hout && hkn && hvn && ref);
    for (e = 0; e < NB * blk_elems; ++e) hk[e] = rand_bf16();
    for (e = 0; e < NB * blk_elems; ++e) hv[e] = rand_bf16();
    for (e = 0; e < (size_t)S * HQ * D; ++e) hq[e] = rand_bf16();
    for (e = 0; e < (size_t)S * HKV * D; ++e) hkn[e] = rand_bf16();
    for (e = 0; e < (size_t)S * HKV * D; ++e) hvn[e] = rand_bf16();

    /* device: copy-on-write copy, slot write, decode */
    CUDA_CHECK(cudaSetDevice(0));
    CUDA_CHECK(cudaMalloc(&dk, cache_bytes));
    CUDA_CHECK(cudaMalloc(&dv, cache_bytes));
    CUDA_CHECK(cudaMalloc(&dq, (size_t)S * HQ * D * 2));
    CUDA_CHECK(cudaMalloc(&dout, (size_t)S * HQ * D * 2));
    CUDA_CHECK(cudaMalloc(&dkn, (size_t)S * HKV * D * 2));
    CUDA_CHECK(cudaMalloc(&dvn, (size_t)S * HKV * D * 2));
    CUDA_CHECK(cudaMalloc(&dtab, sizeof(tables)));
    CUDA_CHECK(cudaMalloc(&dlen, sizeof(lens)));
    CUDA_CHECK(cudaMalloc(&dslots, sizeof(slots)));
    ws_bytes = paged_attention_workspace_bytes(S, HQ, D, max_ctx);
    CHECK(ws_bytes > 0);
    CUDA_CHECK(cudaMalloc(&dws, ws_bytes));
    CUDA_CHECK(cudaMemcpy(dk, hk, cache_bytes, cudaMemcpyHostToDevice));
    CUDA_CHECK(cudaMemcpy(dv, hv, cache_bytes, cudaMemcpyHostToDevice));
    CUDA_CHECK(cudaMemcpy(dq, hq, (size_t)S * HQ * D * 2, cudaMemcpyHostToDevice));
    CUDA_CHECK(cudaMemcpy(dkn, hkn, (size_t)S * HKV * D * 2, cudaMemcpyHostToDevice));
    CUDA_CHECK(cudaMemcpy(dvn, hvn, (size_t)S * HKV * D * 2, cudaMemcpyHostToDevice));
    CUDA_CHECK(cudaMemcpy(dtab, tables, sizeof(tables), cudaMemcpyHostToDevice));
    CUDA_CHECK(cudaMemcpy(dlen, lens, sizeof(lens), cudaMemcpyHostToDevice));
    CUDA_CHECK(cudaMemcpy(dslots, slots, sizeof(slots), cudaMemcpyHostToDevice));

    CHECK(block_copy(dk, dv, pairs, ncow, HKV, D, B, NB, PKV_BF16, NULL) == PKV_OK);
    CHECK(paged_kv_write(dkn, dvn, dk, dv, dslots, S, HKV, D, B, NB, PKV_BF16, NULL) == PKV_OK);
    CHECK(paged_attention_decode(dout, dq, dk, dv, dtab, MB, dlen, S, max_ctx, HQ, HKV, D, B, NB,
                                 (float)(1.0 / sqrt((double)D)), PKV_BF16, dws, ws_bytes, NULL) == PKV_OK);
    CUDA_CHECK(cudaDeviceSynchronize());
    CUDA_CHECK(cudaMemcpy(gk, dk, cache_bytes, cudaMemcpyDeviceToHost));
    CUDA_CHECK(cudaMemcpy(gv, dv, cache_bytes, cudaMemcpyDeviceToHost));
    CUDA_CHECK(cudaMemcpy(hout, dout, (size_t)S * HQ * D * 2, cudaMemcpyDeviceToHost));
    CHECK(pkv_device_status(0, &flags, 1) == PKV_OK && flags == 0);

    /* oracle: the same step on the host copy */
    CHECK(oracle_block_copy(hk, hv, pairs, ncow, HKV, D, B, NB, 2) == 0);
    CHECK(oracle_kv_write(hk, hv, hkn, hvn, slots, S, HKV, D, B, NB, 2) == 0);
    CHECK(memcmp(gk, hk, cache_bytes) == 0 && memcmp(gv, hv, cache_bytes) == 0);
    CHECK(oracle_paged_decode(ref, hq, hk, hv, tables, MB, lens, S, HQ, HKV, D, B, NB,
                              (double)(float)(1.0 / sqrt((double)D)), 2) == 0);
    for (e = 0; e < (size_t)S * HQ * D; ++e) {
        const double got = bf16_value(hout[e]);
        CHECK(fabs(got - ref[e]) <= 2e-3 + 1e-2 * fabs(ref[e]));
    }

    {
        /* shared-prefix decode of the same step (the new tokens are written),
           with the fork beside its parent: batch order 0, 3, 1, 2 */
        const int64_t order2[S] = {0, 3, 1, 2};
        int32_t tab2[S * MB], len2[S], groups[2 * S], shared[S], work[2 * S * (MB * B / 512 + 1)];
        int32_t ng = 0, nw = 0, mxs = 0, mxo = 0, part, r;
        uint16_t* q2 = malloc((size_t)S * HQ * D * 2);
        void *dq2, *dout2, *dtab2, *dlen2, *dgroups, *dshared, *dwork, *dws2;
        size_t ws2;
        CHECK(q2 != NULL);
        CHECK(pkv_batch_tables(a, order2, S, tab2, MB, -1, len2) == PKV_OK);
        part = paged_attention_partition_tokens(S, HKV, max_ctx, PKV_BF16);
        CHECK(part == PKV_PARTITION_TOKENS);
        CHECK(pkv_shared_prefix_plan(tab2, MB, len2, S, B, PKV_SHARED_MAX_ROWS / (HQ / HKV), 128, part, groups, &ng,
                                     shared, work, (int32_t)(sizeof(work) / sizeof(work[0]) / 2), &nw, &mxs,
                                     &mxo) == PKV_OK);
        CHECK(ng == 1 && groups[0] == 0 && groups[1] == 2 && shared[0] == 688 && shared[2] == 0);
        for (r = 0; r < S; ++r) memcpy(q2 + (size_t)r * HQ * D, hq + (size_t)order2[r] * HQ * D, (size_t)HQ * D * 2);
        ws2 = paged_attention_shared_workspace_bytes(S, HQ, D, max_ctx);
        CUDA_CHECK(cudaMalloc(&dq2, (size_t)S * HQ * D * 2));
        CUDA_CHECK(cudaMalloc(&dout2, (size_t)S * HQ * D * 2));
        CUDA_CHECK(cudaMalloc(&dtab2, sizeof(tab2)));
        CUDA_CHECK(cudaMalloc(&dlen2, sizeof(len2)));
        CUDA_CHECK(cudaMalloc(&dgroups, sizeof(groups)));
        CUDA_CHECK(cudaMalloc(&dshared, sizeof(shared)));
        CUDA_CHECK(cudaMalloc(&dwork, sizeof(work)));
        CUDA_CHECK(cudaMalloc(&dws2, ws2));
        CUDA_CHECK(cudaMemcpy(dq2, q2, (size_t)S * HQ * D * 2, cudaMemcpyHostToDevice));
        CUDA_CHECK(cudaMemcpy(dtab2, tab2, sizeof(tab2), cudaMemcpyHostToDevice));
        CUDA_CHECK(cudaMemcpy(dlen2, len2, sizeof(len2), cudaMemcpyHostToDevice));
        CUDA_CHECK(cudaMemcpy(dgroups, groups, sizeof(groups), cudaMemcpyHostToDevice));
        CUDA_CHECK(cudaMemcpy(dshared, shared, sizeof(shared), cudaMemcpyHostToDevice));
        CUDA_CHECK(cudaMemcpy(dwork, work, sizeof(work), cudaMemcpyHostToDevice));
        CHECK(paged_attention_decode_shared(dout2, dq2, NULL, NULL, dk, dv, dtab2, MB, dlen2, S, max_ctx, dgroups, ng,
                                            dshared, dwork, nw, part, HQ, HKV, D, B, NB,
                                            (float)(1.0 / sqrt((double)D)), PKV_BF16, dws2, ws2, NULL) == PKV_OK);
        CUDA_CHECK(cudaDeviceSynchronize());
        CUDA_CHECK(cudaMemcpy(hout, dout2, (size_t)S * HQ * D * 2, cudaMemcpyDeviceToHost));
        CHECK(pkv_device_status(0, &flags, 1) == PKV_OK && flags == 0);
        for (r = 0; r < S; ++r)
            for (e = 0; e < (size_t)HQ * D; ++e) {
                const double want = ref[(size_t)order2[r] * HQ * D + e];
                CHECK(fabs(bf16_value(hout[(size_t)r * HQ * D + e]) - want) <= 2e-3 + 1e-2 * fabs(want));
            }
        cudaFree(dq2);
        cudaFree(dout2);
        cudaFree(dtab2);
        cudaFree(dlen2);
        cudaFree(dgroups);
        cudaFree(dshared);
        cudaFree(dwork);
        cudaFree(dws2);
        free(q2);
    }

    cudaFree(dk);
    cudaFree(dv);
    cudaFree(dq);
    cudaFree(dout);
    cudaFree(dkn);
    cudaFree(dvn);
    cudaFree(dtab);
    cudaFree(dlen);
    cudaFree(dslots);
    cudaFree(dws);
    free(hk);
    free(hv);
    free(gk);
    free(gv);
    free(hq);
    free(hout);
    free(hkn);
    free(hvn);
    free(ref);
    pkv_alloc_destroy(a);
    return 0;
}
#endif

int main(int argc, char** argv)
{
    const char* mode = argc > 1 ? argv[1] : "host";
    if (strcmp(mode, "host") == 0) return host_checks();
#ifdef WITH_CUDA
    if (strcmp(mode, "gpu") == 0) return host_checks() || gpu_checks();
#endif
    fprintf(stderr, "usage: %s host|gpu\n", argv[0]);
    return 2;
}
