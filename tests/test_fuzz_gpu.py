"""Seeded random parity cases against the oracle (needs a B200).

Each case draws a shape (dtype, head_dim, query group, block size, batch,
kv heads), random context lengths on both sides of the split-K threshold,
the number of new tokens per sequence, whether the slot write is fused, and
whether unused table entries hold -1 or random ids.  Writes must be bit-exact
and attention within 2e-3 + 1e-2 |ref| of the oracle.
"""

import random

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_398_b200 as pkv
from oracle.allocator_model import slot_for_position
from paged_kv_cache_398_b200.workloads import make_custom

pytestmark = pytest.mark.gpu
ATOL, RTOL = 2e-3, 1e-2


def _case(seed):
    rng = random.Random(seed)
    dtype = rng.choice([torch.float32, torch.float16, torch.bfloat16, torch.bfloat16])
    D = rng.choice([64, 128])
    G = rng.choice([1, 2, 4, 8])
    B = rng.choice([8, 16, 16, 32])
    Hkv = rng.choice([1, 2, 3])
    S = rng.randint(1, 6)
    q_len = 1 if dtype == torch.float32 else rng.choice([1, 1, 2, 3, 4])
    q_len = max(1, min(q_len, 16 // G))
    fused = dtype != torch.float32 and rng.random() < 0.5
    lens = [max(q_len, rng.choice([rng.randint(1, 40), rng.randint(1, 700), rng.randint(500, 2100)]))
            for _ in range(S)]
    return dtype, D, G, B, Hkv, S, q_len, fused, lens, rng.random() < 0.5


def _mq_case(seed):
    """Many new tokens per sequence on one or two query heads per kv head:
    the 16-row form, its long partitions and both write paths."""
    rng = random.Random(20_000 + seed)
    dtype = rng.choice([torch.float16, torch.bfloat16])
    D = rng.choice([64, 128])
    G = rng.choice([1, 1, 2])
    B = rng.choice([8, 16, 16, 32])
    Hkv = rng.choice([1, 2, 3])
    S = rng.randint(1, 5)
    q_len = rng.randint(5, 16 // G)
    fused = rng.random() < 0.5
    lens = [max(q_len, rng.choice([rng.randint(1, 60), rng.randint(500, 1100), rng.randint(1000, 3100)]))
            for _ in range(S)]
    return dtype, D, G, B, Hkv, S, q_len, fused, lens, rng.random() < 0.5


@pytest.mark.parametrize("seed", range(40))
def test_random_case_matches_oracle(seed, cuda_device):
    _check_case(seed, *_case(seed))


@pytest.mark.parametrize("seed", range(12))
def test_random_many_new_tokens_case_matches_oracle(seed, cuda_device):
    _check_case(500 + seed, *_mq_case(seed))


def _check_case(seed, dtype, D, G, B, Hkv, S, q_len, fused, lens, pad_random):
    w = make_custom(lens, Hkv * G, Hkv, D, dtype, seed=1000 + seed, block_size=B, pad_random=pad_random,
                    q_len=q_len if q_len > 1 else None, spare_blocks=5)
    mq = q_len > 1
    q4 = w.q if mq else w.q[:, None]
    kn4 = w.k_new if mq else w.k_new[:, None]
    vn4 = w.v_new if mq else w.v_new[:, None]
    # oracle: slot write of the new tokens, then (multi-query) decode
    slots = torch.tensor([slot_for_position(w.block_tables[s].tolist(), lens[s] - q_len + j, B)
                          for s in range(S) for j in range(q_len)], dtype=torch.int64)
    k_ref, v_ref = w.k_cache.clone(), w.v_cache.clone()
    oracle.kv_write(k_ref, v_ref, kn4.reshape(S * q_len, Hkv, D).contiguous(),
                    vn4.reshape(S * q_len, Hkv, D).contiguous(), slots)
    ref = oracle.paged_decode_mq(q4.contiguous(), k_ref, v_ref, w.block_tables, w.context_lens, w.scale)
    # product
    g = w.to("cuda")
    out = torch.empty(S, q_len, Hkv * G, D, dtype=dtype, device="cuda")
    gq4 = g.q if mq else g.q[:, None]
    if fused:
        pkv.paged_attention_decode_mq(out, gq4.contiguous(), g.k_cache, g.v_cache, g.block_tables, g.context_lens,
                                      g.scale, max(lens), k_new=(g.k_new if mq else g.k_new[:, None]).contiguous(),
                                      v_new=(g.v_new if mq else g.v_new[:, None]).contiguous())
    else:
        prod_slots = torch.cat([pkv.pkv_slot_mapping(w.block_tables, w.context_lens - q_len + j, B)[:, None]
                                for j in range(q_len)], dim=1).reshape(-1)
        assert torch.equal(prod_slots, slots)
        pkv.paged_kv_write(g.k_new.reshape(S * q_len, Hkv, D), g.v_new.reshape(S * q_len, Hkv, D), g.k_cache,
                           g.v_cache, prod_slots.cuda())
        if mq:
            pkv.paged_attention_decode_mq(out, gq4, g.k_cache, g.v_cache, g.block_tables, g.context_lens, g.scale,
                                          max(lens))
        else:
            pkv.paged_attention_decode(out[:, 0], g.q, g.k_cache, g.v_cache, g.block_tables, g.context_lens,
                                       g.scale, max(lens))
    torch.cuda.synchronize()
    assert torch.equal(g.k_cache.cpu(), k_ref) and torch.equal(g.v_cache.cpu(), v_ref)
    got = out.cpu().double().numpy()
    err = np.abs(got - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    assert np.isfinite(got).all()
    assert not bad.any(), f"case {seed}: {int(bad.sum())} out of tolerance, max abs {err.max():.3e}"
    assert pkv.pkv_device_status(0) == 0


def _shared_case(seed):
    rng = random.Random(10_000 + seed)
    dtype = rng.choice([torch.float16, torch.bfloat16])
    D = rng.choice([64, 128])
    G = rng.choice([1, 2, 4, 8])
    B = rng.choice([8, 16, 32])
    Hkv = rng.choice([1, 2, 3])
    samples = rng.randint(1, 16 // G + 1)          # one more than a group holds, at times: the run splits
    prompts = rng.randint(1, 4)
    plo = rng.choice([1, 100, 500])
    prange = (plo, plo + rng.randint(0, 1600))
    orange = (1, rng.choice([5, 40, 700]))
    min_shared = rng.choice([B, 64, 128])
    return dtype, D, G, B, Hkv, samples, prompts, prange, orange, min_shared


@pytest.mark.parametrize("seed", range(24))
def test_random_shared_prefix_case_matches_oracle(seed, cuda_device):
    """Shared-prefix decode on random sampling batches: copy-on-write copies,
    fused slot write, groups that fill or split the 16-row operand, shared
    lengths on and off partition edges, sequences in no group."""
    from paged_kv_cache_398_b200.workloads import make_sampling
    dtype, D, G, B, Hkv, samples, prompts, prange, orange, min_shared = _shared_case(seed)
    w = make_sampling(prompts, samples, prange, orange, Hkv * G, Hkv, D, dtype, seed=2000 + seed, block_size=B)
    S = w.num_seqs
    slots = torch.tensor([slot_for_position(w.block_tables[s].tolist(), int(w.context_lens[s]) - 1, B)
                          for s in range(S)], dtype=torch.int64)
    k_ref, v_ref = w.k_cache.clone(), w.v_cache.clone()
    if w.copy_pairs.numel():
        oracle.block_copy(k_ref, v_ref, w.copy_pairs)
    oracle.kv_write(k_ref, v_ref, w.k_new, w.v_new, slots)
    ref = oracle.paged_decode(w.q, k_ref, v_ref, w.block_tables, w.context_lens, w.scale)
    part = pkv.paged_attention_partition_tokens(S, Hkv, w.max_context_len, dtype)
    plan = pkv.pkv_shared_prefix_plan(w.block_tables, w.context_lens, B, 16 // G, part, min_shared)
    g = w.to("cuda")
    if w.copy_pairs.numel():
        pkv.block_copy(g.k_cache, g.v_cache, w.copy_pairs)
    d = plan.to("cuda")
    out = torch.empty_like(g.q)
    pkv.paged_attention_decode_shared(out, g.q, g.k_cache, g.v_cache, g.block_tables, g.context_lens, g.scale,
                                      w.max_context_len, d.groups, d.shared_lens, d.work, d.part_tokens,
                                      k_new=g.k_new, v_new=g.v_new)
    torch.cuda.synchronize()
    assert pkv.pkv_device_status(0) == 0
    assert torch.equal(g.k_cache.cpu(), k_ref) and torch.equal(g.v_cache.cpu(), v_ref)
    err = np.abs(out.cpu().double().numpy() - ref)
    bad = err > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), (f"seed {seed}: {int(bad.sum())} elements out of tolerance, max abs {err.max():.3e}, "
                           f"groups {plan.groups.tolist()}")
