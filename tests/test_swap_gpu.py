"""Preemption by swapping blocks to host memory (needs a B200).

swap_blocks_out / swap_blocks_in must move whole blocks bit-exactly between
the device cache and pinned host memory.  A sequence swapped out, with its
blocks overwritten by another request and swapped back into different
blocks, must decode to the same bits as before (the output does not depend
on where the blocks sit).
"""

import pytest
import torch

import paged_kv_cache_398_b200 as pkv
from paged_kv_cache_398_b200.workloads import make_custom

pytestmark = pytest.mark.gpu
B = 16


@pytest.fixture(autouse=True)
def _clean_status(cuda_device):
    pkv.pkv_device_status(0, clear=True)
    yield
    torch.cuda.synchronize()


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
def test_swap_round_trip_is_bit_exact(dtype):
    w = make_custom([100, 250, 37], 8, 4, 64, dtype, seed=12, spare_blocks=40).to("cuda")
    ids = [int(b) for b in w.block_tables[1, :16].tolist()] + [int(w.block_tables[0, 0])]
    n = len(ids)
    hk = torch.empty(n, 4, B, 64, dtype=dtype).pin_memory()
    hv = torch.empty(n, 4, B, 64, dtype=dtype).pin_memory()
    pkv.swap_blocks_out(w.k_cache, w.v_cache, ids, hk, hv)
    torch.cuda.synchronize()
    idx = torch.tensor(ids, device="cuda")
    assert torch.equal(hk, w.k_cache[idx].cpu()) and torch.equal(hv, w.v_cache[idx].cpu())
    # back into other (free) blocks: those become copies, nothing else changes
    used = set(w.block_tables[w.block_tables >= 0].tolist())
    dst = [b for b in range(w.num_blocks) if b not in used][:n]
    k0, v0 = w.k_cache.clone(), w.v_cache.clone()
    pkv.swap_blocks_in(w.k_cache, w.v_cache, dst, hk, hv)
    torch.cuda.synchronize()
    k0[torch.tensor(dst, device="cuda")] = k0[idx]
    v0[torch.tensor(dst, device="cuda")] = v0[idx]
    assert torch.equal(w.k_cache, k0) and torch.equal(w.v_cache, v0)


def test_preempt_and_resume_decodes_identically():
    Hq, Hkv, D, dtype = 32, 8, 128, torch.bfloat16
    NB = 400
    alloc = pkv.BlockAllocator(NB, B, initial_order=torch.randperm(NB, generator=torch.Generator().manual_seed(2)))
    lens = [700, 1300, 90]
    g = torch.Generator(device="cuda").manual_seed(9)
    k_cache = torch.randn(NB, Hkv, B, D, generator=g, device="cuda").to(dtype)
    v_cache = torch.randn(NB, Hkv, B, D, generator=g, device="cuda").to(dtype)
    q = torch.randn(3, Hq, D, generator=g, device="cuda").to(dtype)
    for s, n in enumerate(lens):
        alloc.add(s)
        alloc.append_tokens(s, n)
    MB = 128

    def decode():
        tables, ctx = alloc.batch_tables(range(3), MB)
        out = torch.empty_like(q)
        pkv.paged_attention_decode(out, q, k_cache, v_cache, tables.cuda(), ctx.cuda(), 0.088, max(lens))
        return out

    before = decode()
    # preempt sequence 1: its blocks go to pinned host memory and back to the pool
    out_ids = alloc.swap_out(1)
    hk = torch.empty(len(out_ids), Hkv, B, D, dtype=dtype).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    pkv.swap_blocks_out(k_cache, v_cache, out_ids, hk, hv)
    # a new request takes the freed blocks and overwrites them
    alloc.add(7)
    slots, _ = alloc.append_tokens(7, 1300)
    junk = torch.randn(len(slots), Hkv, D, generator=g, device="cuda").to(dtype)
    pkv.paged_kv_write(junk, junk, k_cache, v_cache, torch.tensor(slots, device="cuda"))
    alloc.free(7)
    alloc.add(8)
    alloc.append_tokens(8, 48)            # shuffles the free list before the swap-in
    # resume sequence 1 in fresh blocks
    in_ids = alloc.swap_in(1)
    assert in_ids != out_ids
    pkv.swap_blocks_in(k_cache, v_cache, in_ids, hk, hv)
    after = decode()
    torch.cuda.synchronize()
    assert torch.equal(before, after)
    assert pkv.pkv_device_status(0) == 0


def test_pageable_host_memory_is_rejected():
    w = make_custom([40], 4, 4, 64, torch.float16, seed=3).to("cuda")
    hk = torch.empty(1, 4, B, 64, dtype=torch.float16)          # not pinned
    hv = torch.empty_like(hk)
    with pytest.raises(pkv.PagedKVError):
        pkv.swap_blocks_out(w.k_cache, w.v_cache, [0], hk, hv)
