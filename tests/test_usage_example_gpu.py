"""The library's usage example, as a GPU test: one decode step of three
requests through the host allocator (copy-on-write pairs, then the slot
write fused into the decode launch), and then parallel sampling with
shared-prefix decode.  The project's README quotes this code."""

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_usage_example(cuda_device):
    import paged_kv_cache_398_b200 as pkv

    NB, Hkv, B, D, Hq = 4096, 8, 16, 128, 32
    k_cache = torch.zeros(NB, Hkv, B, D, dtype=torch.bfloat16, device="cuda")
    v_cache = torch.zeros_like(k_cache)
    alloc = pkv.BlockAllocator(NB, B)

    for s, prompt_len in enumerate((700, 33, 2100)):    # admit three requests
        alloc.add(s)
        slots, _ = alloc.append_tokens(s, prompt_len)    # their prompts' K/V go to these slots

    seqs = [0, 1, 2]
    slots, cow_pairs = alloc.append_one_batch(seqs)     # one new token each (+ copy-on-write pairs)
    tables, lens = alloc.batch_tables(seqs, max_blocks_per_seq=256)
    if cow_pairs.numel():
        pkv.block_copy(k_cache, v_cache, cow_pairs)
    q = torch.randn(3, 1, Hq, D, dtype=torch.bfloat16, device="cuda")       # this step's queries
    k_new = torch.randn(3, 1, Hkv, D, dtype=torch.bfloat16, device="cuda")  # and new keys / values
    v_new = torch.randn_like(k_new)
    out = torch.empty_like(q)
    pkv.paged_attention_decode_mq(out, q, k_cache, v_cache, tables.cuda(), lens.cuda(), D ** -0.5,
                                  int(lens.max()), k_new=k_new, v_new=v_new)   # slot write + attention
    assert pkv.pkv_device_status(0) == 0                # no bad ids, slots or lengths were seen

    # parallel sampling: one prompt forked into four samples that share its
    # blocks, which shared-prefix decode reads once for all four
    alloc.add(10)
    alloc.append_tokens(10, 1500)                       # the prompt
    for child in (11, 12, 13):
        alloc.fork(10, child)                           # the samples share its blocks (reference counts)
    family = [10, 11, 12, 13]
    slots, cow_pairs = alloc.append_one_batch(family)   # the shared partial block is copied on write
    tables, lens = alloc.batch_tables(family, max_blocks_per_seq=256)
    if cow_pairs.numel():
        pkv.block_copy(k_cache, v_cache, cow_pairs)
    part = pkv.paged_attention_partition_tokens(4, Hkv, int(lens.max()), torch.bfloat16)
    plan = pkv.pkv_shared_prefix_plan(tables, lens, B, pkv.SHARED_MAX_ROWS // (Hq // Hkv), part).to("cuda")
    q4 = torch.randn(4, Hq, D, dtype=torch.bfloat16, device="cuda")
    k4 = torch.randn(4, Hkv, D, dtype=torch.bfloat16, device="cuda")
    v4 = torch.randn_like(k4)
    out4 = torch.empty_like(q4)
    pkv.paged_attention_decode_shared(out4, q4, k_cache, v_cache, tables.cuda(), lens.cuda(), D ** -0.5,
                                      int(lens.max()), plan.groups, plan.shared_lens, plan.work, plan.part_tokens,
                                      k_new=k4, v_new=v4)     # the 93 shared prompt blocks cross HBM once
    assert plan.groups.tolist() == [[0, 4]] and pkv.pkv_device_status(0) == 0

    torch.cuda.synchronize()
    assert out.shape == (3, 1, 32, 128) and torch.isfinite(out.float()).all()
    assert out4.shape == (4, 32, 128) and torch.isfinite(out4.float()).all()
