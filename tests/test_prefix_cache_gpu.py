"""Prefix caching end to end (needs a B200).

Requests that begin with the same system prompt find its full blocks in the
allocator's prefix cache (pkv_seq_append_prompt) and only write the K/V of
their own tokens.  Decoding through the shared, found blocks must match the
oracle's decode of each request's complete K/V laid out privately.  The
system prompt's K/V depends only on (position, token), as it would in a
model, so reusing its blocks is valid.
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_398_b200 as pkv

pytestmark = pytest.mark.gpu
B = 16
ATOL, RTOL = 2e-3, 1e-2


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_prefix_cache_decode_matches_private_layout(dtype):
    Hq, Hkv, D = 16, 4, 128
    g = torch.Generator().manual_seed(77)
    system = torch.randint(0, 1000, (40,), generator=g).tolist()     # 2 full blocks + 8 tokens
    sys_k = torch.randn(len(system), Hkv, D, generator=g).to(dtype)
    sys_v = torch.randn(len(system), Hkv, D, generator=g).to(dtype)
    NB = 64
    alloc = pkv.BlockAllocator(NB, B, initial_order=torch.randperm(NB, generator=g))
    k_cache = torch.zeros(NB, Hkv, B, D, dtype=dtype, device="cuda")
    v_cache = torch.zeros_like(k_cache)
    full_k, full_v, cached_counts = [], [], []
    for r, extra in enumerate((37, 5, 90)):
        toks = system + torch.randint(0, 1000, (extra,), generator=g).tolist()
        rk = torch.cat([sys_k, torch.randn(extra, Hkv, D, generator=g).to(dtype)])
        rv = torch.cat([sys_v, torch.randn(extra, Hkv, D, generator=g).to(dtype)])
        alloc.add(r)
        slots, cached = alloc.append_prompt(r, toks)
        cached_counts.append(cached)
        keep = slots >= 0
        pkv.paged_kv_write(rk[keep].cuda(), rv[keep].cuda(), k_cache, v_cache, slots[keep].cuda())
        full_k.append(rk)
        full_v.append(rv)
    assert cached_counts == [0, 32, 32]
    assert alloc.block_table(1)[:2] == alloc.block_table(0)[:2] == alloc.block_table(2)[:2]

    S = 3
    q = torch.randn(S, Hq, D, generator=g).to(dtype)
    tables, lens = alloc.batch_tables(range(S), 16)
    out = torch.empty(S, Hq, D, dtype=dtype, device="cuda")
    pkv.paged_attention_decode(out, q.cuda(), k_cache, v_cache, tables.cuda(), lens.cuda(), D ** -0.5,
                               int(lens.max()))
    torch.cuda.synchronize()
    assert pkv.pkv_device_status(0) == 0

    # oracle: every request's complete K/V in private contiguous blocks
    nbs = [-(-int(n) // B) for n in lens]
    priv_k = torch.zeros(sum(nbs), Hkv, B, D, dtype=dtype)
    priv_v = torch.zeros_like(priv_k)
    ptab = torch.full((S, max(nbs)), -1, dtype=torch.int32)
    first = 0
    for r in range(S):
        n = int(lens[r])
        pad = nbs[r] * B - n
        kk = torch.cat([full_k[r], torch.zeros(pad, Hkv, D, dtype=dtype)]).reshape(nbs[r], B, Hkv, D)
        vv = torch.cat([full_v[r], torch.zeros(pad, Hkv, D, dtype=dtype)]).reshape(nbs[r], B, Hkv, D)
        priv_k[first:first + nbs[r]] = kk.permute(0, 2, 1, 3)
        priv_v[first:first + nbs[r]] = vv.permute(0, 2, 1, 3)
        ptab[r, :nbs[r]] = torch.arange(first, first + nbs[r], dtype=torch.int32)
        first += nbs[r]
    ref = oracle.paged_decode(q, priv_k, priv_v, ptab, lens, D ** -0.5)
    got = out.cpu().double().numpy()
    assert np.all(np.abs(got - ref) <= ATOL + RTOL * np.abs(ref))
