"""Parity of the CUDA path with the CPU oracle (needs a B200).

The product side calls the C ABI through the Python binding; the oracle side
takes the same generator inputs (never the product's outputs) and applies
its own block copy, slot write and attention.  Writes and copies must be
bit-exact; attention must satisfy |gpu - ref| <= 2e-3 + 1e-2 * |ref| per
element against the unrounded fp64 reference.
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_398_b200 as pkv
from oracle.allocator_model import slot_for_position
from paged_kv_cache_398_b200.workloads import make_custom, make_workload

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-3, 1e-2
B = 16


def assert_close(got: torch.Tensor, ref: np.ndarray, what=""):
    g = got.detach().cpu().double().numpy()
    err = np.abs(g - ref)
    bound = ATOL + RTOL * np.abs(ref)
    bad = err > bound
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {bad.size} elements out of tolerance; "
                           f"max abs err {err.max():.3e}")
    return float(err.max())


def oracle_slots(w):
    """Slots of each sequence's new token (its last position), by the oracle."""
    return torch.tensor([slot_for_position(w.block_tables[s].tolist(), int(w.context_lens[s]) - 1, w.block_size)
                         for s in range(w.num_seqs)], dtype=torch.int64)


def product_step(g, slots_dev, out=None):
    """copy-on-write copies, slot write, decode: the product path on device `g`."""
    if g.copy_pairs.numel():
        pkv.block_copy(g.k_cache, g.v_cache, g.copy_pairs.cpu())
    pkv.paged_kv_write(g.k_new, g.v_new, g.k_cache, g.v_cache, slots_dev)
    out = torch.empty_like(g.q) if out is None else out
    pkv.paged_attention_decode(out, g.q, g.k_cache, g.v_cache, g.block_tables, g.context_lens, g.scale,
                               g.max_context_len)
    return out


def oracle_step(w, slots):
    """The same step on CPU copies, entirely by the oracle; returns (out, k, v)."""
    k, v = w.k_cache.clone(), w.v_cache.clone()
    if w.copy_pairs.numel():
        oracle.block_copy(k, v, w.copy_pairs)
    oracle.kv_write(k, v, w.k_new, w.v_new, slots)
    out = oracle.paged_decode(w.q, k, v, w.block_tables, w.context_lens, w.scale)
    return out, k, v


@pytest.fixture(autouse=True)
def _clean_status(cuda_device):
    pkv.pkv_device_status(0, clear=True)
    yield
    torch.cuda.synchronize()


def _run_full_parity(w):
    slots = oracle_slots(w)
    # the product computes its own slot mapping (host helper) and must agree
    prod_slots = pkv.pkv_slot_mapping(w.block_tables, w.context_lens - 1, w.block_size)
    assert torch.equal(prod_slots, slots)
    g = w.to("cuda")
    out = product_step(g, prod_slots.cuda())
    torch.cuda.synchronize()
    ref, k_ref, v_ref = oracle_step(w, slots)
    assert torch.equal(g.k_cache.cpu(), k_ref), "k cache differs after copy + write"
    assert torch.equal(g.v_cache.cpu(), v_ref), "v cache differs after copy + write"
    err = assert_close(out, ref, w.name)
    assert pkv.pkv_device_status(0) == 0
    return err


# ---------------------------------------------------------------------------
# every workload at sizes the oracle finishes in seconds
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("number,kw", [
    (1, {}),
    (2, {"num_seqs": 6}),
    (3, {"num_seqs": 10}),
    (4, {"num_seqs": 10, "max_ctx": 2100}),
    (5, {"num_prompts": 3, "max_prompt": 700, "max_output": 300}),
])
def test_workload_parity_small(number, kw):
    _run_full_parity(make_workload(number, **kw))


def test_tiny_workload_random_table_padding():
    _run_full_parity(make_workload(1, pad_random=True))


# ---------------------------------------------------------------------------
# full-size workloads: bit-exact cache update checked everywhere, attention
# checked on sampled sequences through the oracle
# ---------------------------------------------------------------------------
def _sub_workload(w_dev, seqs):
    """Copy the sampled sequences' blocks (and copy sources) to the CPU,
    relabelled 0..n-1, as a small workload for the oracle."""
    bt = w_dev.block_tables.cpu()
    cl = w_dev.context_lens.cpu()
    pairs = w_dev.copy_pairs.cpu()
    need = []
    for s in seqs:
        need += bt[s, :-(-int(cl[s]) // B)].tolist()
    dsts = set(need)
    sub_pairs = [(int(a), int(b)) for a, b in pairs.tolist() if int(b) in dsts]
    need += [a for a, _ in sub_pairs]
    ids = sorted(set(need))
    remap = {b: i for i, b in enumerate(ids)}
    idx = torch.tensor(ids, dtype=torch.int64, device=w_dev.k_cache.device)
    MB = bt.shape[1]
    sbt = torch.full((len(seqs), MB), -1, dtype=torch.int32)
    for r, s in enumerate(seqs):
        n = -(-int(cl[s]) // B)
        sbt[r, :n] = torch.tensor([remap[b] for b in bt[s, :n].tolist()], dtype=torch.int32)
    sel = torch.tensor(seqs, dtype=torch.int64, device=w_dev.q.device)
    from paged_kv_cache_398_b200.workloads import DecodeWorkload
    return DecodeWorkload(
        name=w_dev.name + "-sample", dtype=w_dev.dtype, num_seqs=len(seqs), num_q_heads=w_dev.num_q_heads,
        num_kv_heads=w_dev.num_kv_heads, head_dim=w_dev.head_dim, block_size=B, num_blocks=len(ids),
        context_lens=cl[seqs].contiguous(), block_tables=sbt,
        copy_pairs=torch.tensor([(remap[a], remap[b]) for a, b in sub_pairs], dtype=torch.int64).reshape(-1, 2),
        q=w_dev.q[sel].cpu(), k_cache=w_dev.k_cache[idx].cpu(), v_cache=w_dev.v_cache[idx].cpu(),
        k_new=w_dev.k_new[sel].cpu(), v_new=w_dev.v_new[sel].cpu(), scale=w_dev.scale, seed=w_dev.seed)


@pytest.mark.parametrize("number", [2, 3, 4, 5])
def test_workload_parity_full_size_sampled(number):
    host = make_workload(number, device="cuda")    # tables on the host, values on the GPU
    w = host.to("cuda")
    S = w.num_seqs
    gen = torch.Generator().manual_seed(number)
    order = torch.argsort(host.context_lens, descending=True).tolist()
    seqs = sorted(set([order[0], order[-1]] + torch.randperm(S, generator=gen)[:6].tolist()))
    sub = _sub_workload(w, seqs)                   # taken before the product step
    slots = oracle_slots(host)
    k_expect = w.k_cache.clone()
    v_expect = w.v_cache.clone()
    for a, b in w.copy_pairs.tolist():            # the definition of the step's cache update
        k_expect[b] = k_expect[a]
        v_expect[b] = v_expect[a]
    sd = slots.cuda()
    k_expect[sd // B, :, sd % B, :] = w.k_new
    v_expect[sd // B, :, sd % B, :] = w.v_new

    out = product_step(w, pkv.pkv_slot_mapping(host.block_tables, host.context_lens - 1).cuda())
    torch.cuda.synchronize()
    assert torch.equal(w.k_cache, k_expect) and torch.equal(w.v_cache, v_expect)
    del k_expect, v_expect

    ref, _, _ = oracle_step(sub, oracle_slots(sub))
    assert_close(out[torch.tensor(seqs, device="cuda")], ref, w.name)
    assert pkv.pkv_device_status(0) == 0


@pytest.mark.parametrize("number", [2, 3])
def test_workload_16_new_tokens_full_size_sampled(number):
    """The 7B and 13B batches at full size with 16 new tokens per sequence
    (the multi-query step of the bench's q_len 16 entries): one fused call
    writes every new token's K/V and attends causally.  The cache update is
    checked everywhere, the attention on sampled sequences (the longest among
    them) against the oracle.  Such launches take the long partitions."""
    import dataclasses
    from paged_kv_cache_398_b200.workloads import _randn
    QL = 16
    base = make_workload(number, device="cuda", min_ctx=QL)
    S, Hq, Hkv, D = base.num_seqs, base.num_q_heads, base.num_kv_heads, base.head_dim
    gd = torch.Generator(device="cuda").manual_seed(70 + number)
    host = dataclasses.replace(base, q=_randn((S, QL, Hq, D), base.dtype, gd, "cuda"),
                               k_new=_randn((S, QL, Hkv, D), base.dtype, gd, "cuda"),
                               v_new=_randn((S, QL, Hkv, D), base.dtype, gd, "cuda"))
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    large = S * Hkv >= pkv._lib.C["PKV_LONG_MIN_PAIRS_PER_SM"] * sms      # the 13B batch; the 7B one is not
    assert pkv.paged_attention_mq_partition_tokens(S, QL, Hq, Hkv, host.max_context_len, host.dtype) == \
        (pkv.PARTITION_TOKENS_WIDE if large else pkv.PARTITION_TOKENS_LONG)
    w = host.to("cuda")
    order = torch.argsort(host.context_lens, descending=True).tolist()
    gen = torch.Generator().manual_seed(number)
    seqs = sorted(set([order[0], order[1], order[-1]] + torch.randperm(S, generator=gen)[:2].tolist()))
    sub = _sub_workload(w, seqs)                   # taken before the product step
    slots = torch.tensor([slot_for_position(host.block_tables[s].tolist(), int(host.context_lens[s]) - QL + j, B)
                          for s in range(S) for j in range(QL)], dtype=torch.int64)
    k_expect, v_expect = w.k_cache.clone(), w.v_cache.clone()
    sd = slots.cuda()
    k_expect[sd // B, :, sd % B, :] = w.k_new.reshape(S * QL, Hkv, D)
    v_expect[sd // B, :, sd % B, :] = w.v_new.reshape(S * QL, Hkv, D)
    out = torch.empty_like(w.q)
    pkv.paged_attention_decode_mq(out, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale,
                                  host.max_context_len, k_new=w.k_new, v_new=w.v_new)
    torch.cuda.synchronize()
    assert torch.equal(w.k_cache, k_expect) and torch.equal(w.v_cache, v_expect)
    del k_expect, v_expect

    n = len(seqs)
    sub_slots = torch.tensor([slot_for_position(sub.block_tables[r].tolist(), int(sub.context_lens[r]) - QL + j, B)
                              for r in range(n) for j in range(QL)], dtype=torch.int64)
    k_ref, v_ref = sub.k_cache.clone(), sub.v_cache.clone()
    oracle.kv_write(k_ref, v_ref, sub.k_new.reshape(n * QL, Hkv, D).contiguous(),
                    sub.v_new.reshape(n * QL, Hkv, D).contiguous(), sub_slots)
    ref = oracle.paged_decode_mq(sub.q, k_ref, v_ref, sub.block_tables, sub.context_lens, sub.scale)
    assert_close(out[torch.tensor(seqs, device="cuda")], ref, f"{w.name}, 16 new tokens")
    assert pkv.pkv_device_status(0) == 0


# ---------------------------------------------------------------------------
# shapes and edges: every dtype, head dim and group size; lengths on and
# around block and partition boundaries; the longest context
# ---------------------------------------------------------------------------
EDGE_LENS = [1, 2, 15, 16, 17, 31, 32, 33, 511, 512, 513, 1024, 1025, 8192]


@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G", [1, 2, 4, 8])
def test_shapes_and_edge_lengths(dtype, D, G):
    Hkv = 2
    w = make_custom(EDGE_LENS, Hkv * G, Hkv, D, dtype, seed=G * 1000 + D)
    _run_full_parity(w)


def test_empty_batch_and_empty_write():
    q = torch.empty(0, 4, 64, device="cuda")
    kc = torch.zeros(2, 4, B, 64, device="cuda")
    out = torch.empty_like(q)
    pkv.paged_attention_decode(out, q, kc, kc.clone(), torch.empty(0, 1, dtype=torch.int32, device="cuda"),
                               torch.empty(0, dtype=torch.int32, device="cuda"), 0.125, 1)
    pkv.paged_kv_write(torch.empty(0, 4, 64, device="cuda"), torch.empty(0, 4, 64, device="cuda"), kc,
                       kc.clone(), torch.empty(0, dtype=torch.int64, device="cuda"))
    pkv.block_copy(kc, kc.clone(), [])
    torch.cuda.synchronize()


# ---------------------------------------------------------------------------
# invariances (bitwise on the GPU)
# ---------------------------------------------------------------------------
def test_placement_permutation_is_bitwise_invariant():
    w = make_workload(4, num_seqs=12, max_ctx=3000).to("cuda")
    out1 = torch.empty_like(w.q)
    pkv.paged_attention_decode(out1, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale,
                               w.max_context_len)
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(3)).cuda()
    k2 = torch.empty_like(w.k_cache)
    v2 = torch.empty_like(w.v_cache)
    k2[perm] = w.k_cache
    v2[perm] = w.v_cache
    bt2 = w.block_tables.clone()
    m = bt2 >= 0
    bt2[m] = perm[bt2[m].long()].int()
    out2 = torch.empty_like(w.q)
    pkv.paged_attention_decode(out2, w.q, k2, v2, bt2, w.context_lens, w.scale, w.max_context_len)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)


def test_shared_prefix_equals_duplicated_blocks():
    w = make_workload(4, num_seqs=8, max_ctx=1500).to("cuda")
    pre = w.meta["prefix_blocks"]
    out1 = torch.empty_like(w.q)
    pkv.paged_attention_decode(out1, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale,
                               w.max_context_len)
    # give every sequence its own copy of the 4 prefix blocks
    S = w.num_seqs
    extra = torch.tensor(pre, device="cuda").repeat(S)
    k2 = torch.cat([w.k_cache, w.k_cache[extra]])
    v2 = torch.cat([w.v_cache, w.v_cache[extra]])
    bt2 = w.block_tables.clone()
    for s in range(S):
        bt2[s, :4] = torch.arange(w.num_blocks + 4 * s, w.num_blocks + 4 * s + 4, device="cuda")
    out2 = torch.empty_like(w.q)
    pkv.paged_attention_decode(out2, w.q, k2, v2, bt2, w.context_lens, w.scale, w.max_context_len)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2)


def test_copy_then_write_leaves_source_untouched():
    w = make_workload(5, num_prompts=2, max_prompt=500, max_output=40).to("cuda")
    src_blocks = sorted({a for a, _ in w.copy_pairs.tolist()})
    before_k = w.k_cache[src_blocks].clone()
    before_v = w.v_cache[src_blocks].clone()
    product_step(w, pkv.pkv_slot_mapping(w.block_tables.cpu(), w.context_lens.cpu() - 1).cuda())
    torch.cuda.synchronize()
    # sample 0 of each prompt may write its new token into the original
    # block (it is the last holder); every other source block is untouched
    slots = pkv.pkv_slot_mapping(w.block_tables.cpu(), w.context_lens.cpu() - 1)
    written = {int(s) // B for s in slots.tolist()}
    for i, blk in enumerate(src_blocks):
        if blk not in written:
            assert torch.equal(w.k_cache[blk], before_k[i])
            assert torch.equal(w.v_cache[blk], before_v[i])


def test_garbage_in_unused_slots_is_ignored():
    w = make_custom([5, 17, 40, 513], 8, 2, 128, torch.bfloat16, seed=9)
    ref_out = None
    for poison in (False, True):
        g = w.to("cuda")
        if poison:
            used = torch.zeros(w.num_blocks, B, dtype=torch.bool)
            for s in range(w.num_seqs):
                for t in range(int(w.context_lens[s])):
                    used[int(w.block_tables[s, t // B]), t % B] = True
            nan_mask = (~used).cuda()[:, None, :, None].expand_as(g.k_cache)
            g.k_cache[nan_mask] = float("nan")
            g.v_cache[nan_mask] = float("inf")
        out = torch.empty_like(g.q)
        pkv.paged_attention_decode(out, g.q, g.k_cache, g.v_cache, g.block_tables, g.context_lens, g.scale,
                                   g.max_context_len)
        torch.cuda.synchronize()
        if ref_out is None:
            ref_out = out
        else:
            assert torch.equal(out, ref_out)


def test_deterministic_repeat():
    w = make_workload(4, num_seqs=16, max_ctx=4000).to("cuda")
    outs = []
    for _ in range(3):
        out = torch.empty_like(w.q)
        pkv.paged_attention_decode(out, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale,
                                   w.max_context_len)
        outs.append(out)
    torch.cuda.synchronize()
    assert torch.equal(outs[0], outs[1]) and torch.equal(outs[0], outs[2])


# ---------------------------------------------------------------------------
# device-side checks raise status flags instead of faulting
# ---------------------------------------------------------------------------
def test_bad_block_id_sets_flag_and_stays_in_bounds():
    w = make_custom([40, 20], 4, 4, 64, torch.float16, seed=4).to("cuda")
    w.block_tables[0, 1] = 10 ** 6
    w.block_tables[1, 0] = -7
    out = torch.empty_like(w.q)
    pkv.paged_attention_decode(out, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale,
                               w.max_context_len)
    flags = pkv.pkv_device_status(0)
    assert flags & pkv._lib.C["PKV_DEV_BAD_BLOCK_ID"]
    assert pkv.pkv_device_status(0) == 0


def test_bad_context_lengths():
    w = make_custom([40, 20, 70], 4, 4, 64, torch.float32, seed=5)
    g = w.to("cuda")
    g.context_lens[1] = 0
    out = torch.full_like(g.q, 7.0)
    pkv.paged_attention_decode(out, g.q, g.k_cache, g.v_cache, g.block_tables, g.context_lens, g.scale, 70)
    flags = pkv.pkv_device_status(0)
    assert flags & pkv._lib.C["PKV_DEV_BAD_CONTEXT"]
    assert torch.equal(out[1].cpu(), torch.zeros_like(out[1].cpu()))
    # the other sequences are unaffected (no write happened in this call)
    ref_nowrite = oracle.paged_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale)
    assert_close(out[[0, 2]], ref_nowrite[[0, 2]])
    # a length above the declared maximum is clamped and flagged
    g.context_lens[1] = 20
    pkv.paged_attention_decode(out, g.q, g.k_cache, g.v_cache, g.block_tables, g.context_lens, g.scale, 40)
    assert pkv.pkv_device_status(0) & pkv._lib.C["PKV_DEV_BAD_CONTEXT"]


def test_bad_slot_sets_flag_and_writes_nothing_else():
    w = make_custom([40, 20], 4, 4, 64, torch.bfloat16, seed=6).to("cuda")
    k0, v0 = w.k_cache.clone(), w.v_cache.clone()
    slots = torch.tensor([w.num_blocks * B + 3, -1], dtype=torch.int64, device="cuda")
    pkv.paged_kv_write(w.k_new, w.v_new, w.k_cache, w.v_cache, slots)
    assert pkv.pkv_device_status(0) & pkv._lib.C["PKV_DEV_BAD_SLOT"]
    assert torch.equal(w.k_cache, k0) and torch.equal(w.v_cache, v0)


def test_block_copy_rejects_order_dependent_lists_on_gpu():
    kc = torch.zeros(8, 2, B, 64, dtype=torch.float16, device="cuda")
    with pytest.raises(pkv.PagedKVError):
        pkv.block_copy(kc, kc.clone(), [[1, 2], [2, 3]])
    with pytest.raises(pkv.PagedKVError):
        pkv.block_copy(kc, kc.clone(), [[1, 9]])


def test_many_copy_pairs_span_launches():
    NB, Hkv, D = 2600, 2, 64
    g = torch.Generator(device="cuda").manual_seed(8)
    kc = torch.randn(NB, Hkv, B, D, device="cuda", generator=g).to(torch.float16)
    vc = torch.randn(NB, Hkv, B, D, device="cuda", generator=g).to(torch.float16)
    pairs = [(i, 1300 + i) for i in range(1300)]
    k0, v0 = kc.clone(), vc.clone()
    pkv.block_copy(kc, vc, pairs)
    torch.cuda.synchronize()
    assert torch.equal(kc[1300:], k0[:1300]) and torch.equal(vc[1300:], v0[:1300])
    assert torch.equal(kc[:1300], k0[:1300])


# ---------------------------------------------------------------------------
# split-K: one workspace serves every batch shape, and the longest contexts
# (hundreds of partitions per sequence) merge correctly
# ---------------------------------------------------------------------------
def test_one_workspace_serves_batches_of_any_shape():
    """One workspace, reused without clearing by batches of other shapes (the
    previous call's records stay in it), gives every batch its own result."""
    shapes = [make_custom([5000, 2000, 700], 32, 8, 128, torch.bfloat16, seed=34),
              make_custom([600, 1100, 40, 3000, 900, 1500, 2600], 8, 2, 64, torch.float16, seed=35),
              make_custom([9000], 16, 2, 128, torch.bfloat16, seed=36)]
    need = max(pkv.paged_attention_workspace_bytes(w.num_seqs, w.num_q_heads, w.head_dim, w.max_context_len)
               for w in shapes)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    for w in shapes + shapes[::-1]:
        ref = oracle.paged_decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale)
        g = w.to("cuda")
        out = torch.full_like(g.q, float("nan"))
        pkv.paged_attention_decode(out, g.q, g.k_cache, g.v_cache, g.block_tables, g.context_lens, g.scale,
                                   g.max_context_len, workspace=ws)
        torch.cuda.synchronize()
        assert_close(out, ref)
        assert pkv.pkv_device_status(0) == 0


@pytest.mark.parametrize("dtype,lens,G,D", [
    (torch.bfloat16, [131072, 70001, 1, 512], 4, 128),   # 256 partitions merged by one CTA
    (torch.float32, [40000, 3], 4, 64),
])
def test_longest_contexts(dtype, lens, G, D):
    w = make_custom(lens, 2 * G, 2, D, dtype, seed=33)
    _run_full_parity(w)


# ---------------------------------------------------------------------------
# long partitions: a batch with enough (sequence, kv head) pairs and a long
# maximum context splits into partitions of PARTITION_TOKENS_WIDE tokens
# ---------------------------------------------------------------------------
def _long_mode_lens(seed, n_short):
    g = torch.Generator().manual_seed(seed)
    short = torch.randint(1, 200, (n_short,), generator=g).tolist()
    return short[:n_short // 2] + [4096, 9000, 1025, 5000, 2048, 2049, 6144] + short[n_short // 2:]


def test_partition_rule_on_this_device():
    C = pkv._lib.C
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    pairs = C["PKV_LONG_MIN_PAIRS_PER_SM"] * sms
    bf16, f32 = torch.bfloat16, torch.float32
    assert pkv.paged_attention_partition_tokens(pairs, 1, 4096, bf16) == pkv.PARTITION_TOKENS_WIDE
    assert pkv.paged_attention_partition_tokens(pairs - 1, 1, 4096, bf16) == pkv.PARTITION_TOKENS
    assert pkv.paged_attention_partition_tokens(pairs, 1, 4095, bf16) == pkv.PARTITION_TOKENS
    assert pkv.paged_attention_partition_tokens(pairs, 1, 9000, f32) == pkv.PARTITION_TOKENS
    # the bench's 8B-GQA batch takes the wide partitions, the 7B and 13B batches do not
    assert pkv.paged_attention_partition_tokens(256, 8, 8130, bf16) == pkv.PARTITION_TOKENS_WIDE
    assert pkv.paged_attention_partition_tokens(64, 40, 3521, torch.float16) == pkv.PARTITION_TOKENS
    assert pkv.paged_attention_partition_tokens(24, 32, 1986, torch.float16) == pkv.PARTITION_TOKENS
    # multi-query: more than 8 rows per kv head take the wide partitions on a large batch of any context length
    # and the long ones otherwise; up to 8 rows keep the rule above
    mq = pkv.paged_attention_mq_partition_tokens
    assert mq(64, 16, 40, 40, 3521, torch.float16) == pkv.PARTITION_TOKENS_WIDE   # the 13B batch: 2560 pairs
    assert mq(24, 16, 32, 32, 2064, torch.float16) == pkv.PARTITION_TOKENS_LONG   # the 7B batch: 768 pairs
    assert mq(2, 4, 32, 8, 300, bf16) == pkv.PARTITION_TOKENS_LONG
    assert mq(pairs - 1, 4, 4, 1, 300, bf16) == pkv.PARTITION_TOKENS_LONG
    assert mq(pairs, 4, 4, 1, 300, bf16) == pkv.PARTITION_TOKENS_WIDE
    assert mq(pairs - 1, 2, 4, 1, 4096, bf16) == pkv.PARTITION_TOKENS
    assert mq(pairs, 2, 4, 1, 4096, bf16) == pkv.PARTITION_TOKENS_WIDE
    assert mq(256, 1, 32, 8, 8130, bf16) == pkv.paged_attention_partition_tokens(256, 8, 8130, bf16)


@pytest.mark.parametrize("block_size,dtype,D,G", [
    (16, torch.bfloat16, 128, 4),
    (8, torch.float16, 64, 8),      # 256 blocks per partition: two table entries per thread
    (32, torch.bfloat16, 128, 1),
])
def test_long_partitions_match_oracle(block_size, dtype, D, G):
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    Hkv = 8
    S = -(-pkv._lib.C["PKV_LONG_MIN_PAIRS_PER_SM"] * sms // Hkv)
    w = make_custom(_long_mode_lens(40 + block_size, S - 7), Hkv * G, Hkv, D, dtype, seed=41 + block_size,
                    block_size=block_size, pad_random=True)
    assert pkv.paged_attention_partition_tokens(S, Hkv, w.max_context_len, dtype) == pkv.PARTITION_TOKENS_WIDE
    _run_full_parity(w)


def test_long_partitions_multi_query_fused():
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    Hkv, G, D, QL, dtype = 8, 4, 128, 3, torch.bfloat16
    S = -(-pkv._lib.C["PKV_LONG_MIN_PAIRS_PER_SM"] * sms // Hkv)
    lens = [max(QL, n) for n in _long_mode_lens(44, S - 7)]
    w = make_custom(lens, Hkv * G, Hkv, D, dtype, seed=45, q_len=QL)
    slots = torch.tensor([slot_for_position(w.block_tables[s].tolist(), lens[s] - QL + j, w.block_size)
                          for s in range(S) for j in range(QL)], dtype=torch.int64)
    k_ref, v_ref = w.k_cache.clone(), w.v_cache.clone()
    oracle.kv_write(k_ref, v_ref, w.k_new.reshape(S * QL, Hkv, D).contiguous(),
                    w.v_new.reshape(S * QL, Hkv, D).contiguous(), slots)
    ref = oracle.paged_decode_mq(w.q, k_ref, v_ref, w.block_tables, w.context_lens, w.scale)
    g = w.to("cuda")
    out = torch.empty_like(g.q)
    pkv.paged_attention_decode_mq(out, g.q, g.k_cache, g.v_cache, g.block_tables, g.context_lens, g.scale,
                                  max(lens), k_new=g.k_new, v_new=g.v_new)
    torch.cuda.synchronize()
    assert torch.equal(g.k_cache.cpu(), k_ref) and torch.equal(g.v_cache.cpu(), v_ref)
    assert_close(out, ref)
    assert pkv.pkv_device_status(0) == 0


def test_bounded_wait_times_out_and_context_survives():
    """A wait on a barrier nothing arrives on gives up after its limit and
    reports PKV_DEV_WAIT_TIMEOUT; the GPU keeps working afterwards."""
    import ctypes
    L = pkv._lib.lib()
    t0 = __import__("time").perf_counter()
    assert L.pkv_debug_wait_timeout(20_000_000, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)) == 0
    flags = pkv.pkv_device_status(0)
    waited = __import__("time").perf_counter() - t0
    assert flags & pkv._lib.C["PKV_DEV_WAIT_TIMEOUT"]
    assert 0.015 < waited < 5.0
    _run_full_parity(make_workload(1))


# ---------------------------------------------------------------------------
# block sizes 8 and 32 (a compute tile is 16 tokens: two blocks or half of one)
# ---------------------------------------------------------------------------
@pytest.mark.parametrize("block_size", [8, 32])
@pytest.mark.parametrize("dtype", [torch.float32, torch.float16, torch.bfloat16])
@pytest.mark.parametrize("D,G", [(64, 1), (128, 4), (128, 8)])
def test_block_sizes_8_and_32(block_size, dtype, D, G):
    lens = [1, 7, 8, 9, 15, 16, 17, 31, 33, 511, 512, 513, 520, 1000, 4100]
    w = make_custom(lens, 2 * G, 2, D, dtype, seed=block_size * 100 + G + D, block_size=block_size)
    _run_full_parity(w)


# ---------------------------------------------------------------------------
# occupancy guard: every tensor-core decode kernel keeps 3 CTAs per SM
# resident (its shared memory allows 3, and 168 registers per thread fit 3);
# a build whose register count crept up would silently lose a third of the
# bytes in flight
# ---------------------------------------------------------------------------
def test_every_decode_kernel_keeps_its_occupancy():
    import ctypes
    L = pkv._lib.lib()
    C = pkv._lib.C
    low = []
    for dtype in (C["PKV_F16"], C["PKV_BF16"]):
        for D in (64, 128):
            for G in (1, 2, 4, 8):
                for q_len in sorted({1, 16 // G} | ({2} if G <= 8 else set())):
                    for B in (8, 16, 32):
                        for long_p in (0, 1):
                            n = ctypes.c_int32(0)
                            rc = L.pkv_debug_decode_occupancy(dtype, D, G, q_len, B, long_p, ctypes.byref(n))
                            assert rc == 0, (dtype, D, G, q_len, B, long_p, rc)
                            if n.value < 3:
                                low.append((dtype, D, G, q_len, B, long_p, n.value))
    assert not low, f"below 3 CTAs per SM: {low}"
    for D in (64, 128):   # the fp32 kernel (fp32 tiles are twice the bytes: 1 CTA per SM at head_dim 128)
        n = ctypes.c_int32(0)
        assert L.pkv_debug_decode_occupancy(C["PKV_F32"], D, 4, 1, 16, 0, ctypes.byref(n)) == 0 and n.value >= 1
    n = ctypes.c_int32(0)
    assert L.pkv_debug_decode_occupancy(C["PKV_F32"], 128, 4, 2, 16, 0, ctypes.byref(n)) == C["PKV_ERR_UNSUPPORTED"]


def test_concurrent_host_threads_on_their_own_streams():
    """Two host threads decode different batches at once, each on its own
    stream with its own workspace (ctypes releases the GIL, so the calls
    overlap on the host, first-call set-up included); each result equals
    the same call made alone, bit for bit."""
    import threading
    batches = [make_custom([700, 33, 2100, 5], 16, 4, 128, torch.bfloat16, seed=60).to("cuda"),
               make_custom([1500, 900, 64], 8, 8, 64, torch.float16, seed=61).to("cuda")]

    def decode(w, stream):
        out = torch.empty_like(w.q)
        with torch.cuda.stream(stream):
            ws = torch.zeros(max(1, pkv.paged_attention_workspace_bytes(w.num_seqs, w.num_q_heads, w.head_dim,
                                                                         w.max_context_len)),
                             dtype=torch.uint8, device="cuda")
            for _ in range(5):
                pkv.paged_attention_decode(out, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens,
                                           w.scale, w.max_context_len, workspace=ws)
        stream.synchronize()
        return out

    alone = [decode(w, torch.cuda.Stream()) for w in batches]
    results = [None, None]
    errors = []

    def worker(i):
        try:
            results[i] = decode(batches[i], torch.cuda.Stream())
        except Exception as e:  # surfaced below
            errors.append(e)

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join(timeout=120)
    assert not errors, errors
    for got, ref in zip(results, alone):
        assert torch.equal(got, ref)
    assert pkv.pkv_device_status(0) == 0
