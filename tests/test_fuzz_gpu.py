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


@pytest.mark.parametrize("seed", range(40))
def test_random_case_matches_oracle(seed, cuda_device):
    dtype, D, G, B, Hkv, S, q_len, fused, lens, pad_random = _case(seed)
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
