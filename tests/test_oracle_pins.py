"""Pins of the CPU oracle to things other than itself (CPU only).

Each check ties one part of the oracle to the pages' worked examples, a closed
form, a library routine on a special case, or an exact invariant, so that a
plausible slip (dropped term, wrong sign, swapped index, transposed operand)
fails at least one of them.  ``test_mutants_are_caught`` plants such slips in
a copy of the oracle's C source and checks that the pins notice.
"""

import math
import os
import re
import subprocess
import tempfile

import numpy as np
import pytest
import torch

import oracle
from oracle.allocator_model import AllocatorModel
from tests.conftest import load_golden

B = 16


# --------------------------------------------------------------------------
# helpers that build inputs (layout [NB, Hkv, B, D]; no oracle arithmetic)
# --------------------------------------------------------------------------
def _contiguous_case(ctx, Hq, Hkv, D, dtype, seed):
    """One sequence stored in blocks 0..n-1 in order, plus the same K/V as
    plain [Hkv, ctx, D] tensors for a library routine."""
    g = torch.Generator().manual_seed(seed)
    nb = -(-ctx // B)
    K = torch.randn(nb * B, Hkv, D, generator=g).to(dtype)
    V = torch.randn(nb * B, Hkv, D, generator=g).to(dtype)
    q = torch.randn(1, Hq, D, generator=g).to(dtype)
    k_cache = K.reshape(nb, B, Hkv, D).permute(0, 2, 1, 3).contiguous()
    v_cache = V.reshape(nb, B, Hkv, D).permute(0, 2, 1, 3).contiguous()
    bt = torch.arange(nb, dtype=torch.int32).reshape(1, nb)
    cl = torch.tensor([ctx], dtype=torch.int32)
    return q, k_cache, v_cache, bt, cl, K[:ctx], V[:ctx]


def _relabel(k_cache, v_cache, bt, perm):
    """Move physical block b to perm[b] and rewrite the tables accordingly."""
    k2 = torch.empty_like(k_cache)
    v2 = torch.empty_like(v_cache)
    k2[perm] = k_cache
    v2[perm] = v_cache
    bt2 = bt.clone()
    m = bt >= 0
    bt2[m] = perm[bt[m].long()].to(torch.int32)
    return k2, v2, bt2


# --------------------------------------------------------------------------
# exact widening of the input types
# --------------------------------------------------------------------------
def check_widen_fp16():
    bits = torch.arange(0, 65536, dtype=torch.int32).to(torch.int16).view(torch.float16)
    got = oracle.widen(bits)
    want = bits.numpy().astype(np.float64)
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    np.testing.assert_array_equal(got[ok], want[ok])


def check_widen_bf16():
    bits = torch.arange(0, 65536, dtype=torch.int32).to(torch.int16).view(torch.bfloat16)
    got = oracle.widen(bits)
    want = bits.to(torch.float64).numpy()
    np.testing.assert_array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    np.testing.assert_array_equal(got[ok], want[ok])


def test_widen_fp16_every_bit_pattern():
    check_widen_fp16()


def test_widen_bf16_every_bit_pattern():
    check_widen_bf16()


# --------------------------------------------------------------------------
# gather through the page's worked block tables
# --------------------------------------------------------------------------
def check_worked_example_gather():
    gold = load_golden("worked_block_tables.json")
    tables = gold["block_tables"]
    # The physical row printed on the page must be exactly what the tables imply.
    row = ["free"] * 12
    for req, phys in tables.items():
        for logical, p in enumerate(phys):
            row[p] = f"{req}:{logical}"
    assert "".join(f"[{c}]" for c in row) == gold["physical_row"]
    assert [i for i, c in enumerate(row) if c == "free"] == gold["free_blocks"]
    # Label every slot of every physical block with (request, logical block,
    # offset) according to the printed row; gathering a request must return
    # its tokens in logical order.
    Hkv, D = 2, 4
    k_cache = torch.full((12, Hkv, B, D), -1.0)
    v_cache = torch.full((12, Hkv, B, D), -1.0)
    code = {"A": 1000, "B": 2000, "C": 3000}
    for p, c in enumerate(row):
        if c == "free":
            continue
        req, logical = c.split(":")
        for off in range(B):
            for h in range(Hkv):
                k_cache[p, h, off, :] = code[req] + int(logical) * B + off + 0.25 * h
                v_cache[p, h, off, :] = -(code[req] + int(logical) * B + off) - 0.25 * h
    for req, phys in tables.items():
        ctx = len(phys) * B - 3
        bt = torch.tensor(phys, dtype=torch.int32)
        for h in range(Hkv):
            kc, vc = oracle.gather(k_cache, v_cache, bt, ctx, h)
            want = code[req] + np.arange(ctx) + 0.25 * h
            np.testing.assert_array_equal(kc[:, 0], want)
            np.testing.assert_array_equal(vc[:, 0], -(code[req] + np.arange(ctx)) - 0.25 * h)


def test_worked_example_gather():
    check_worked_example_gather()


# --------------------------------------------------------------------------
# attention: library routine on the contiguous case, closed forms, invariants
# --------------------------------------------------------------------------
def check_sdpa_contiguous():
    for ctx, Hq, Hkv, D, dtype in [(5, 4, 4, 64, torch.float32), (17, 4, 2, 8, torch.float16),
                                   (33, 8, 2, 16, torch.bfloat16), (64, 2, 1, 64, torch.float32)]:
        q, kc, vc, bt, cl, K, V = _contiguous_case(ctx, Hq, Hkv, D, dtype, seed=ctx)
        scale = 1.0 / math.sqrt(D) * 1.3
        got = oracle.paged_decode(q, kc, vc, bt, cl, scale)[0]
        qq = q.to(torch.float64).reshape(1, Hq, 1, D)
        KK = K.to(torch.float64).permute(1, 0, 2).reshape(1, Hkv, ctx, D)
        VV = V.to(torch.float64).permute(1, 0, 2).reshape(1, Hkv, ctx, D)
        want = torch.nn.functional.scaled_dot_product_attention(
            qq, KK, VV, scale=scale, enable_gqa=True).reshape(Hq, D).numpy()
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_attention_equals_sdpa_on_contiguous_blocks():
    check_sdpa_contiguous()


def check_multi_query_causal_sdpa():
    for ctx, QL, Hq, Hkv, D, dtype in [(20, 3, 4, 2, 16, torch.float32), (33, 4, 8, 2, 8, torch.bfloat16),
                                       (5, 5, 2, 1, 8, torch.float16), (48, 1, 4, 4, 16, torch.float32)]:
        g = torch.Generator().manual_seed(ctx * 7 + QL)
        q, kc, vc, bt, cl, K, V = _contiguous_case(ctx, Hq, Hkv, D, dtype, seed=ctx + QL)
        qm = torch.randn(1, QL, Hq, D, generator=g).to(dtype)
        scale = 0.7 / math.sqrt(D)
        got = oracle.paged_decode_mq(qm, kc, vc, bt, cl, scale)[0]            # [QL, Hq, D]
        # query j sits at position ctx - QL + j and may see keys 0..ctx - QL + j
        allowed = torch.arange(ctx)[None, :] <= (ctx - QL + torch.arange(QL))[:, None]
        qq = qm.to(torch.float64)[0].permute(1, 0, 2).reshape(1, Hq, QL, D)
        KK = K.to(torch.float64).permute(1, 0, 2).reshape(1, Hkv, ctx, D)
        VV = V.to(torch.float64).permute(1, 0, 2).reshape(1, Hkv, ctx, D)
        want = torch.nn.functional.scaled_dot_product_attention(
            qq, KK, VV, attn_mask=allowed, scale=scale, enable_gqa=True)[0].permute(1, 0, 2).numpy()
        np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)
    # a batch of two sequences in one pool: each row must match its own sequence
    QL, Hq, Hkv, D = 3, 4, 2, 8
    g = torch.Generator().manual_seed(5)
    ctxs, starts = (20, 35), (0, 2)
    kc = torch.randn(5, Hkv, B, D, generator=g)
    vc = torch.randn(5, Hkv, B, D, generator=g)
    bt = torch.tensor([[0, 1, -1], [2, 3, 4]], dtype=torch.int32)
    cl = torch.tensor(ctxs, dtype=torch.int32)
    qm = torch.randn(2, QL, Hq, D, generator=g)
    got = oracle.paged_decode_mq(qm, kc, vc, bt, cl, 0.4)
    for sq, (ctx, b0) in enumerate(zip(ctxs, starts)):
        nb = -(-ctx // B)
        K = kc[b0:b0 + nb].permute(1, 0, 2, 3).reshape(1, Hkv, nb * B, D)[:, :, :ctx].double()
        V = vc[b0:b0 + nb].permute(1, 0, 2, 3).reshape(1, Hkv, nb * B, D)[:, :, :ctx].double()
        allowed = torch.arange(ctx)[None, :] <= (ctx - QL + torch.arange(QL))[:, None]
        qq = qm[sq].double().permute(1, 0, 2).reshape(1, Hq, QL, D)
        want = torch.nn.functional.scaled_dot_product_attention(
            qq, K, V, attn_mask=allowed, scale=0.4, enable_gqa=True)[0].permute(1, 0, 2).numpy()
        np.testing.assert_allclose(got[sq], want, rtol=1e-12, atol=1e-12)
    # q_len = 1 is the single-query decode, exactly
    q, kc, vc, bt, cl, K, V = _contiguous_case(30, 4, 2, 16, torch.float32, seed=99)
    a = oracle.paged_decode(q, kc, vc, bt, cl, 0.3)
    b = oracle.paged_decode_mq(q.reshape(1, 1, 4, 16).contiguous(), kc, vc, bt, cl, 0.3)
    np.testing.assert_array_equal(a, b[:, 0])


def test_multi_query_decode_equals_causal_sdpa():
    check_multi_query_causal_sdpa()


def check_single_token_is_its_value():
    q, kc, vc, bt, cl, K, V = _contiguous_case(1, 4, 4, 64, torch.float32, seed=1)
    got = oracle.paged_decode(q, kc, vc, bt, cl, 0.125)[0]
    np.testing.assert_array_equal(got, V[0].to(torch.float64).numpy())


def test_single_token_is_its_value():
    check_single_token_is_its_value()


def check_uniform_scores_give_mean():
    ctx, Hq, Hkv, D = 37, 4, 4, 16
    q, kc, vc, bt, cl, K, V = _contiguous_case(ctx, Hq, Hkv, D, torch.float32, seed=3)
    q.zero_()
    got = oracle.paged_decode(q, kc, vc, bt, cl, 0.25)[0]
    want = V.to(torch.float64).mean(dim=0).numpy()
    np.testing.assert_allclose(got, want, rtol=0, atol=1e-14)
    # equal keys: every score equal, again the mean
    q2, kc2, vc2, bt2, cl2, K2, V2 = _contiguous_case(ctx, Hq, Hkv, D, torch.float32, seed=4)
    kc2[:] = kc2[0, :, 0:1, :]
    got2 = oracle.paged_decode(q2, kc2, vc2, bt2, cl2, 0.25)[0]
    want2 = V2.to(torch.float64).mean(dim=0).numpy()
    np.testing.assert_allclose(got2, want2, rtol=0, atol=1e-14)


def test_uniform_scores_give_mean():
    check_uniform_scores_give_mean()


def check_dominant_key():
    ctx, Hq, Hkv, D = 40, 2, 2, 16
    q, kc, vc, bt, cl, K, V = _contiguous_case(ctx, Hq, Hkv, D, torch.float32, seed=5)
    star = 23
    for h in range(Hkv):
        q[0, h] = K[star, h] * 50.0
    got = oracle.paged_decode(q, kc, vc, bt, cl, 1.0)[0]
    np.testing.assert_allclose(got, V[star].to(torch.float64).numpy(), rtol=0, atol=1e-9)
    assert np.all(np.isfinite(got))


def test_dominant_key_and_large_scores():
    check_dominant_key()


def check_gqa_grouping():
    # kv head h holds the constant value h+1 in every V row: query head i
    # must return (i // G) + 1, which a modular (i % Hkv) grouping would not.
    ctx, Hq, Hkv, D = 21, 8, 2, 8
    q, kc, vc, bt, cl, K, V = _contiguous_case(ctx, Hq, Hkv, D, torch.float32, seed=6)
    for h in range(Hkv):
        vc[:, h] = h + 1.0
    got = oracle.paged_decode(q, kc, vc, bt, cl, 0.3)[0]
    G = Hq // Hkv
    for i in range(Hq):
        np.testing.assert_allclose(got[i], (i // G) + 1.0, rtol=0, atol=1e-14)


def test_gqa_grouping():
    check_gqa_grouping()


def check_placement_invariance():
    from paged_kv_cache_398_b200.workloads import make_workload
    w = make_workload(1)
    ref = oracle.paged_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale)
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(7))
    k2, v2, bt2 = _relabel(w.k_cache, w.v_cache, w.block_tables, perm)
    got = oracle.paged_decode(w.q, k2, v2, bt2, w.context_lens, w.scale)
    np.testing.assert_array_equal(got, ref)
    # scattered placement equals the contiguous identity placement too
    S = w.num_seqs
    for s in range(S):
        ctx = int(w.context_lens[s])
        nb = -(-ctx // B)
        idx = w.block_tables[s, :nb].long()
        kc = w.k_cache[idx].contiguous()
        vc = w.v_cache[idx].contiguous()
        bt = torch.arange(nb, dtype=torch.int32).reshape(1, nb)
        one = oracle.paged_decode(w.q[s:s + 1].contiguous(), kc, vc, bt,
                                  w.context_lens[s:s + 1].contiguous(), w.scale)
        np.testing.assert_array_equal(one[0], ref[s])


def test_placement_invariance():
    check_placement_invariance()


def check_shared_equals_duplicated():
    # Two sequences sharing 3 prefix blocks vs the same data with private copies.
    Hq, Hkv, D = 4, 2, 16
    g = torch.Generator().manual_seed(11)
    NB = 12
    kc = torch.randn(NB, Hkv, B, D, generator=g)
    vc = torch.randn(NB, Hkv, B, D, generator=g)
    q = torch.randn(2, Hq, D, generator=g)
    cl = torch.tensor([60, 55], dtype=torch.int32)
    shared = torch.tensor([[0, 1, 2, 3], [0, 1, 2, 4]], dtype=torch.int32)
    kd, vd = kc.clone(), vc.clone()
    kd[5:8] = kc[0:3]
    vd[5:8] = vc[0:3]
    dup = torch.tensor([[0, 1, 2, 3], [5, 6, 7, 4]], dtype=torch.int32)
    a = oracle.paged_decode(q, kc, vc, shared, cl, 0.2)
    b = oracle.paged_decode(q, kd, vd, dup, cl, 0.2)
    np.testing.assert_array_equal(a, b)


def test_shared_blocks_equal_duplicated_blocks():
    check_shared_equals_duplicated()


def check_unused_table_entries_ignored():
    from paged_kv_cache_398_b200.workloads import make_workload
    a = make_workload(1)
    b = make_workload(1, pad_random=True)
    ra = oracle.paged_decode(a.q, a.k_cache, a.v_cache, a.block_tables, a.context_lens, a.scale)
    rb = oracle.paged_decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale)
    np.testing.assert_array_equal(ra, rb)


def test_unused_table_entries_ignored():
    check_unused_table_entries_ignored()


def test_invalid_inputs_rejected():
    q, kc, vc, bt, cl, K, V = _contiguous_case(20, 2, 2, 8, torch.float32, seed=9)
    with pytest.raises(oracle.OracleError):
        oracle.paged_decode(q, kc, vc, bt, torch.tensor([0], dtype=torch.int32), 1.0)
    bad = bt.clone()
    bad[0, 1] = 99
    with pytest.raises(oracle.OracleError):
        oracle.paged_decode(q, kc, vc, bad, cl, 1.0)
    with pytest.raises(oracle.OracleError):
        oracle.paged_decode(q, kc, vc, bt, torch.tensor([33], dtype=torch.int32), 1.0)


# --------------------------------------------------------------------------
# slot write
# --------------------------------------------------------------------------
def check_write_roundtrip_worked_tables():
    """Write request A's tokens one by one at the slots the allocator model
    hands out for the page's table; gathering A returns them in order."""
    gold = load_golden("worked_block_tables.json")
    order = [0, 2, 6, 4, 7, 1, 3, 9, 5, 8, 10, 11]
    m = AllocatorModel(12, B, initial_order=order)
    Hkv, D = 2, 8
    g = torch.Generator().manual_seed(12)
    kc = torch.zeros(12, Hkv, B, D)
    vc = torch.zeros(12, Hkv, B, D)
    toks_k = torch.randn(45, Hkv, D, generator=g)
    toks_v = torch.randn(45, Hkv, D, generator=g)
    m.add(0)
    for t in range(45):
        slots, cow = m.append_tokens(0, 1)
        oracle.kv_write(kc, vc, toks_k[t:t + 1].contiguous(), toks_v[t:t + 1].contiguous(),
                        torch.tensor(slots, dtype=torch.int64))
    assert m.block_table(0) == gold["block_tables"]["A"]
    bt = torch.tensor(m.block_table(0), dtype=torch.int32)
    for h in range(Hkv):
        k_got, v_got = oracle.gather(kc, vc, bt, 45, h)
        np.testing.assert_array_equal(k_got, toks_k[:, h].double().numpy())
        np.testing.assert_array_equal(v_got, toks_v[:, h].double().numpy())


def test_write_roundtrip_worked_tables():
    check_write_roundtrip_worked_tables()


def check_write_touches_only_its_slot():
    NB, Hkv, D = 6, 3, 8
    g = torch.Generator().manual_seed(13)
    kc = torch.randn(NB, Hkv, B, D, generator=g).to(torch.bfloat16)
    vc = torch.randn(NB, Hkv, B, D, generator=g).to(torch.bfloat16)
    k0, v0 = kc.clone(), vc.clone()
    kn = torch.randn(3, Hkv, D, generator=g).to(torch.bfloat16)
    vn = torch.randn(3, Hkv, D, generator=g).to(torch.bfloat16)
    slots = torch.tensor([4 * B + 9, -1, 1 * B + 0], dtype=torch.int64)
    oracle.kv_write(kc, vc, kn, vn, slots)
    k0[4, :, 9] = kn[0]
    v0[4, :, 9] = vn[0]
    k0[1, :, 0] = kn[2]
    v0[1, :, 0] = vn[2]
    assert torch.equal(kc.view(torch.int16), k0.view(torch.int16))
    assert torch.equal(vc.view(torch.int16), v0.view(torch.int16))
    with pytest.raises(oracle.OracleError):
        oracle.kv_write(kc, vc, kn, vn, torch.tensor([0, 1, NB * B], dtype=torch.int64))
    assert torch.equal(kc.view(torch.int16), k0.view(torch.int16))


def test_write_touches_only_its_slot():
    check_write_touches_only_its_slot()


# --------------------------------------------------------------------------
# copy-on-write block copy
# --------------------------------------------------------------------------
def check_block_copy_semantics():
    NB, Hkv, D = 8, 2, 8
    g = torch.Generator().manual_seed(14)
    kc = torch.randn(NB, Hkv, B, D, generator=g).to(torch.float16)
    vc = torch.randn(NB, Hkv, B, D, generator=g).to(torch.float16)
    k0, v0 = kc.clone(), vc.clone()
    oracle.block_copy(kc, vc, torch.tensor([[2, 5], [3, 7]], dtype=torch.int64))
    want_k, want_v = k0.clone(), v0.clone()
    want_k[5], want_v[5] = k0[2], v0[2]
    want_k[7], want_v[7] = k0[3], v0[3]
    assert torch.equal(kc.view(torch.int16), want_k.view(torch.int16))
    assert torch.equal(vc.view(torch.int16), want_v.view(torch.int16))
    # copy then write to the copy: the source block is untouched
    kn = torch.randn(1, Hkv, D, generator=g).to(torch.float16)
    oracle.kv_write(kc, vc, kn, kn.clone(), torch.tensor([5 * B + 3], dtype=torch.int64))
    assert torch.equal(kc[2].view(torch.int16), k0[2].view(torch.int16))
    assert torch.equal(vc[2].view(torch.int16), v0[2].view(torch.int16))
    assert torch.equal(kc[5, :, 3].view(torch.int16), kn[0].view(torch.int16))


def test_block_copy_semantics():
    check_block_copy_semantics()


def test_block_copy_rejects_order_dependent_lists():
    NB, Hkv, D = 8, 1, 4
    kc = torch.randn(NB, Hkv, B, D)
    vc = torch.randn(NB, Hkv, B, D)
    k0 = kc.clone()
    for pairs in ([[1, 1]], [[1, 2], [3, 2]], [[1, 2], [2, 3]], [[0, 8]], [[-1, 2]]):
        with pytest.raises(oracle.OracleError):
            oracle.block_copy(kc, vc, torch.tensor(pairs, dtype=torch.int64))
    assert torch.equal(kc, k0)


# --------------------------------------------------------------------------
# planted mistakes must be caught
# --------------------------------------------------------------------------
QUICK_CHECKS = [check_worked_example_gather, check_sdpa_contiguous, check_multi_query_causal_sdpa,
                check_single_token_is_its_value,
                check_uniform_scores_give_mean, check_dominant_key, check_gqa_grouping,
                check_placement_invariance, check_shared_equals_duplicated,
                check_write_roundtrip_worked_tables, check_write_touches_only_its_slot,
                check_block_copy_semantics, check_widen_fp16, check_widen_bf16]

MUTANTS = [
    ("int32_t logical = t / block_size;", "int32_t logical = t % block_size;"),
    ("int32_t offset = t % block_size;", "int32_t offset = t / block_size;"),
    ("(((int64_t)phys * num_kv_heads + kv_head) * block_size + offset) * head_dim",
     "(((int64_t)phys * block_size + offset) * num_kv_heads + kv_head) * head_dim"),
    ("scores[t] = scale * dot;", "scores[t] = dot;"),
    ("scores[t] = exp(scores[t] - smax);", "scores[t] = exp(smax - scores[t]);"),
    ("denom += scores[t];", "denom = scores[t];"),
    ("out[d] += p * vc[(int64_t)t * head_dim + d];", "out[d] += p * kc[(int64_t)t * head_dim + d];"),
    ("for (int32_t i = h * group; rc == 0 && i < (h + 1) * group; ++i)",
     "for (int32_t i = h; rc == 0 && i < num_q_heads; i += num_kv_heads)"),
    ("int64_t off = slot % block_size;", "int64_t off = slot / block_size;"),
    ("max_blocks_per_seq, ctx - q_len + j + 1, num_q_heads,", "max_blocks_per_seq, ctx - q_len + j, num_q_heads,"),
    ("int64_t row = (int64_t)s * q_len + j;", "int64_t row = (int64_t)j * num_seqs + s;"),
    ("memcpy((char*)v_cache + (size_t)dst * block_bytes,", "memcpy((char*)v_cache + (size_t)src * block_bytes,"),
    ("v = ldexp((double)(f + 1024), e - 25);", "v = ldexp((double)(f + 1024), e - 24);"),
    ("uint32_t u = (uint32_t)b << 16;", "uint32_t u = (uint32_t)b << 15;"),
]


def _load_mutant(src_text, tmpdir, idx):
    path_c = os.path.join(tmpdir, f"m{idx}.c")
    path_so = os.path.join(tmpdir, f"m{idx}.so")
    with open(path_c, "w") as f:
        f.write(src_text)
    subprocess.check_call(["gcc", "-O1", "-std=c99", "-fPIC", "-shared", "-o", path_so, path_c, "-lm"])
    return path_so


def test_mutants_are_caught(monkeypatch):
    import ctypes
    with open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")) as f:
        src = f.read()
    good = oracle.lib()
    with tempfile.TemporaryDirectory() as td:
        for i, (old, new) in enumerate(MUTANTS):
            assert src.count(old) == 1, f"mutant {i}: pattern not unique in oracle.c: {old}"
            so = _load_mutant(src.replace(old, new), td, i)
            L = ctypes.CDLL(so)
            for name in ("oracle_widen", "oracle_gather", "oracle_paged_decode_seq", "oracle_paged_decode",
                         "oracle_paged_decode_mq", "oracle_kv_write", "oracle_block_copy"):
                fn, ref = getattr(L, name), getattr(good, name)
                fn.argtypes, fn.restype = ref.argtypes, ref.restype
            monkeypatch.setattr(oracle, "_lib", L)
            caught = False
            for chk in QUICK_CHECKS:
                try:
                    chk()
                except (AssertionError, oracle.OracleError):
                    caught = True
                    break
            monkeypatch.setattr(oracle, "_lib", good)
            assert caught, f"mutant {i} ({new}) passed every pin"
