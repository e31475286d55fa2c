"""A serving loop over many steps (needs a B200).

Requests arrive with prompts, fork into parallel samples, generate one token
per step and finish, so blocks are shared, copied on write, released and
handed out again with stale contents.  The native allocator decides the
slots, tables and copy pairs; the product runs block_copy and the fused
write + decode each step, either through the ordinary entry or through
shared-prefix decode, whose plan groups each request's samples (the batch
lists every family's members together, so the plan can find them).  The test keeps every request's token K/V on the
host, drawn from its own generator, and checks each step's output against
the oracle's decode of those tokens laid out privately: the oracle never
sees the product's cache.
"""

import random

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_398_b200 as pkv

pytestmark = pytest.mark.gpu
ATOL, RTOL = 2e-3, 1e-2


def _private_layout(tokens_k, tokens_v, B, dtype):
    """Every request's K/V in its own contiguous blocks: (k, v, tables, lens)."""
    nbs = [-(-len(t) // B) for t in tokens_k]
    Hkv, D = tokens_k[0][0].shape
    k = torch.zeros(sum(nbs), Hkv, B, D, dtype=dtype)
    v = torch.zeros_like(k)
    tables = torch.full((len(nbs), max(nbs)), -1, dtype=torch.int32)
    first = 0
    for r, (tk, tv) in enumerate(zip(tokens_k, tokens_v)):
        n = len(tk)
        kk = torch.stack(tk)  # [n, Hkv, D]
        vv = torch.stack(tv)
        for t in range(n):
            k[first + t // B, :, t % B] = kk[t]
            v[first + t // B, :, t % B] = vv[t]
        tables[r, :nbs[r]] = torch.arange(first, first + nbs[r], dtype=torch.int32)
        first += nbs[r]
    lens = torch.tensor([len(t) for t in tokens_k], dtype=torch.int32)
    return k, v, tables, lens


@pytest.mark.parametrize("path", ["fused", "shared"])
@pytest.mark.parametrize("dtype,B,G", [(torch.bfloat16, 16, 4), (torch.float16, 8, 2)])
def test_serving_loop_matches_oracle_every_step(dtype, B, G, path):
    rng = random.Random(1234 + B)
    gen = torch.Generator().manual_seed(99 + B)
    Hkv, D = 2, 64
    Hq = Hkv * G
    NB, MB = 4096, 160
    alloc = pkv.BlockAllocator(NB, B, initial_order=torch.randperm(NB, generator=gen))
    k_cache = torch.randn(NB, Hkv, B, D, generator=gen).to(dtype).cuda()   # stale contents everywhere
    v_cache = torch.randn(NB, Hkv, B, D, generator=gen).to(dtype).cuda()
    tok_k, tok_v = {}, {}          # request id -> list of [Hkv, D] host tensors
    root = {}                      # request id -> the request its family started from
    next_id = 0

    def new_tokens(n):
        return ([torch.randn(Hkv, D, generator=gen).to(dtype) for _ in range(n)],
                [torch.randn(Hkv, D, generator=gen).to(dtype) for _ in range(n)])

    def admit(n):
        nonlocal next_id
        sid = next_id
        next_id += 1
        alloc.add(sid)
        root[sid] = sid
        slots, _ = alloc.append_tokens(sid, n)
        tk, tv = new_tokens(n)
        idx = torch.tensor(slots, device="cuda")
        k_cache[idx // B, :, idx % B] = torch.stack(tk).cuda()   # prompt K/V written outside the step
        v_cache[idx // B, :, idx % B] = torch.stack(tv).cuda()
        tok_k[sid], tok_v[sid] = tk, tv

    for _ in range(6):
        admit(rng.randint(1, 300))
    copies_seen = groups_seen = 0
    for step in range(40):
        # requests arrive, fork into samples and finish
        if rng.random() < 0.3 and len(tok_k) < 24:
            admit(rng.randint(1, 400))
        if rng.random() < 0.3 and tok_k:
            parent = rng.choice(sorted(tok_k))
            alloc.fork(parent, next_id)
            root[next_id] = root[parent]
            tok_k[next_id], tok_v[next_id] = list(tok_k[parent]), list(tok_v[parent])
            next_id += 1
        if rng.random() < 0.25 and len(tok_k) > 2:
            done = rng.choice(sorted(tok_k))
            alloc.free(done)
            del tok_k[done], tok_v[done]
        live = sorted(tok_k, key=lambda r: (root[r], r))   # families together
        if any(len(tok_k[s]) + 1 > MB * B for s in live):
            break
        # this step: one new token per live request
        slots, pairs = alloc.append_one_batch(live)
        tables, lens = alloc.batch_tables(live, MB)
        copies_seen += pairs.shape[0]
        nk, nv = new_tokens(len(live))
        for i, s in enumerate(live):
            tok_k[s].append(nk[i])
            tok_v[s].append(nv[i])
        q = torch.randn(len(live), 1, Hq, D, generator=gen).to(dtype)
        if pairs.numel():
            pkv.block_copy(k_cache, v_cache, pairs)
        out = torch.empty(len(live), 1, Hq, D, dtype=dtype, device="cuda")
        if path == "shared":
            part = pkv.paged_attention_partition_tokens(len(live), Hkv, int(lens.max()), dtype)
            plan = pkv.pkv_shared_prefix_plan(tables, lens, B, pkv.SHARED_MAX_ROWS // G, part, B)
            groups_seen += plan.groups.shape[0]
            d = plan.to("cuda")
            pkv.paged_attention_decode_shared(out[:, 0], q[:, 0].contiguous().cuda(), k_cache, v_cache,
                                              tables.cuda(), lens.cuda(), D ** -0.5, int(lens.max()), d.groups,
                                              d.shared_lens, d.work, d.part_tokens,
                                              k_new=torch.stack(nk).cuda(), v_new=torch.stack(nv).cuda())
        else:
            pkv.paged_attention_decode_mq(out, q.cuda(), k_cache, v_cache, tables.cuda(), lens.cuda(), D ** -0.5,
                                          int(lens.max()), k_new=torch.stack(nk)[:, None].cuda(),
                                          v_new=torch.stack(nv)[:, None].cuda())
        torch.cuda.synchronize()
        assert pkv.pkv_device_status(0) == 0, f"step {step}"
        pk, pv, ptab, plens = _private_layout([tok_k[s] for s in live], [tok_v[s] for s in live], B, dtype)
        assert torch.equal(plens, lens)
        ref = oracle.paged_decode(q[:, 0].contiguous(), pk, pv, ptab, plens, D ** -0.5)
        got = out[:, 0].double().cpu().numpy()
        bad = np.abs(got - ref) > ATOL + RTOL * np.abs(ref)
        assert not bad.any(), f"step {step}: {int(bad.sum())} elements out of tolerance"
    assert copies_seen > 0          # forks of partly filled blocks were copied on write
    assert step >= 30
    if path == "shared":
        assert groups_seen > 0      # families shared blocks that their group read once
