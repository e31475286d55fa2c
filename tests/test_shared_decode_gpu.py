"""Shared-prefix decode against the oracle (needs a B200).

paged_attention_decode_shared reads the blocks a group of samples shares
once and attends all the group's query heads to them together, then each
sample's own blocks, and merges both.  The oracle knows nothing of groups:
it applies the step's copy-on-write copies and slot writes to a CPU copy of
the cache and decodes every sequence alone through its own block table.
Writes must be bit-exact; attention within |gpu - ref| <= 2e-3 + 1e-2 |ref|.
"""

import pytest
import torch

import oracle
import paged_kv_cache_398_b200 as pkv
from paged_kv_cache_398_b200.workloads import make_sampling, make_workload
from test_parity_gpu import _sub_workload, assert_close, oracle_slots, oracle_step

pytestmark = pytest.mark.gpu
BAD_PLAN = pkv._lib.C["PKV_DEV_BAD_PLAN"]


@pytest.fixture(autouse=True)
def _clean_status(cuda_device):
    pkv.pkv_device_status(0, clear=True)
    yield
    torch.cuda.synchronize()


def make_plan(host, min_shared_tokens=128):
    G = host.num_q_heads // host.num_kv_heads
    pt = pkv.paged_attention_partition_tokens(host.num_seqs, host.num_kv_heads, host.max_context_len, host.dtype)
    return pkv.pkv_shared_prefix_plan(host.block_tables, host.context_lens, host.block_size,
                                      pkv.SHARED_MAX_ROWS // G, pt, min_shared_tokens)


def shared_step(g, host, min_shared_tokens=128, plan=None, out=None):
    """Copy-on-write copies, then the fused write + shared-prefix decode (product)."""
    if plan is None:
        plan = make_plan(host, min_shared_tokens)
    if g.copy_pairs.numel():
        pkv.block_copy(g.k_cache, g.v_cache, g.copy_pairs.cpu())
    d = plan.to("cuda")
    out = torch.empty_like(g.q) if out is None else out
    pkv.paged_attention_decode_shared(out, g.q, g.k_cache, g.v_cache, g.block_tables, g.context_lens, g.scale,
                                      g.max_context_len, d.groups, d.shared_lens, d.work, d.part_tokens,
                                      k_new=g.k_new, v_new=g.v_new)
    return out, plan


def _parity(w, min_shared_tokens=128):
    g = w.to("cuda")
    out, plan = shared_step(g, w, min_shared_tokens)
    torch.cuda.synchronize()
    assert pkv.pkv_device_status(0) == 0
    ref, k_ref, v_ref = oracle_step(w, oracle_slots(w))
    assert torch.equal(g.k_cache.cpu(), k_ref) and torch.equal(g.v_cache.cpu(), v_ref)
    assert_close(out, ref, f"shared decode {w.dtype} B={w.block_size} G={w.num_q_heads // w.num_kv_heads}")
    return plan


@pytest.mark.parametrize("dtype,B,D,Hq,Hkv,samples", [
    (torch.bfloat16, 16, 128, 32, 8, 4),   # the 8B-GQA sampling shape: 16 rows per group
    (torch.float16, 8, 64, 4, 4, 16),      # one query head per kv head: 16 samples per group
    (torch.bfloat16, 32, 128, 16, 2, 2),   # 8 query heads per kv head: groups of 2
    (torch.float16, 16, 128, 8, 4, 8),     # 2 per kv head: 8 samples
    (torch.bfloat16, 8, 128, 8, 2, 3),     # groups smaller than the operand allows
    (torch.bfloat16, 16, 128, 32, 8, 2),   # 2 samples x 4 heads = 8 rows: the transposed 8-column group pass
    (torch.float16, 16, 64, 4, 4, 5),      # 5 samples x 1 head = 5 rows (8-column form)
    (torch.float16, 32, 128, 16, 8, 3),    # 3 samples x 2 heads = 6 rows (8-column form), block size 32
])
def test_shared_decode_matches_oracle(dtype, B, D, Hq, Hkv, samples):
    w = make_sampling(5, samples, (1, 1400), (1, 300), Hq, Hkv, D, dtype, seed=70 + B + samples, block_size=B)
    plan = _parity(w)
    # every prompt with at least 128 shared tokens forms a group of all its samples
    expect = sum(1 for p in w.meta["prompt_lens"] if (p // B) * B >= 128)
    assert plan.groups.shape[0] == expect
    assert all(n == samples for _, n in plan.groups.tolist())


def test_groups_of_both_forms_in_one_launch():
    """A family of 12 samples at 2 query heads per kv head splits into a
    group of 8 (16 rows: the 16-row form) and one of 4 (8 rows: the
    8-column form); both forms run in the same launch."""
    w = make_sampling(3, 12, (600, 1400), (1, 200), 8, 4, 128, torch.bfloat16, seed=91)
    plan = _parity(w)
    sizes = sorted(n for _, n in plan.groups.tolist())
    assert sizes == [4, 4, 4, 8, 8, 8]


def test_interleaved_batch_reordered_for_sharing():
    """A batch whose families are interleaved (as a serving loop may admit
    them): pkv_shared_prefix_order brings each family's samples together, and
    shared-prefix decode of the reordered batch finds every group and
    matches the oracle."""
    import dataclasses
    w = make_sampling(5, 4, (300, 1500), (1, 200), 32, 8, 128, torch.bfloat16, seed=77)
    grouped = make_plan(w).groups.shape[0]
    perm = torch.randperm(w.num_seqs, generator=torch.Generator().manual_seed(8))

    def take(src, idx):
        return dataclasses.replace(src, block_tables=src.block_tables[idx], context_lens=src.context_lens[idx],
                                   q=src.q[idx], k_new=src.k_new[idx], v_new=src.v_new[idx])
    shuffled = take(w, perm)
    assert make_plan(shuffled).groups.shape[0] < grouped
    order = pkv.pkv_shared_prefix_order(shuffled.block_tables, shuffled.context_lens, shuffled.block_size)
    plan = _parity(take(shuffled, order))
    assert plan.groups.shape[0] == grouped


def test_shared_lengths_on_partition_edges():
    # prompts whose shared part ends just before, on and after a partition boundary
    dtype, B = torch.bfloat16, 16
    for i, p in enumerate([511, 512, 513, 1023, 1024, 1040]):
        w = make_sampling(1, 4, (p, p), (1, 40), 32, 8, 128, dtype, seed=90 + i, block_size=B)
        plan = _parity(w, min_shared_tokens=B)
        assert plan.shared_lens.tolist() == [(p // B) * B] * 4


def test_without_groups_equals_multi_query_decode_bitwise():
    # no group forms: every sequence goes through its own pass from position 0,
    # which is the ordinary partitioning of paged_attention_decode_mq
    w = make_sampling(4, 4, (200, 900), (1, 200), 32, 8, 128, torch.bfloat16, seed=5)
    a, b = w.to("cuda"), w.to("cuda")
    out_shared, plan = shared_step(a, w, min_shared_tokens=1 << 20)
    assert plan.groups.numel() == 0
    if b.copy_pairs.numel():
        pkv.block_copy(b.k_cache, b.v_cache, b.copy_pairs.cpu())
    out_mq = torch.empty(w.num_seqs, 1, w.num_q_heads, w.head_dim, dtype=w.dtype, device="cuda")
    pkv.paged_attention_decode_mq(out_mq, b.q[:, None].contiguous(), b.k_cache, b.v_cache, b.block_tables,
                                  b.context_lens, b.scale, b.max_context_len, k_new=b.k_new[:, None].contiguous(),
                                  v_new=b.v_new[:, None].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(out_shared, out_mq[:, 0])
    assert torch.equal(a.k_cache, b.k_cache) and torch.equal(a.v_cache, b.v_cache)


def test_placement_permutation_is_bitwise_invariant():
    w = make_sampling(4, 4, (100, 1500), (1, 300), 32, 8, 128, torch.bfloat16, seed=8)
    perm = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(1))
    inv = torch.argsort(perm)
    w2 = make_sampling(4, 4, (100, 1500), (1, 300), 32, 8, 128, torch.bfloat16, seed=8)
    w2.k_cache, w2.v_cache = w.k_cache[inv].clone(), w.v_cache[inv].clone()   # block b moves to perm[b]
    w2.block_tables = torch.where(w.block_tables >= 0, perm[w.block_tables.clamp(min=0).long()].int(),
                                  w.block_tables)
    w2.copy_pairs = perm[w.copy_pairs]
    o1, _ = shared_step(w.to("cuda"), w)
    o2, _ = shared_step(w2.to("cuda"), w2)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2)


def test_long_partitions_sampling_batch():
    # enough (sequence, kv head) pairs and long enough prompts for the wide partitions
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    prompts = -(-pkv._lib.C["PKV_LONG_MIN_PAIRS_PER_SM"] * sms // 32)   # 4 samples x 8 kv heads each
    w = make_sampling(prompts, 4, (2000, 4096), (1, 1024), 32, 8, 128, torch.bfloat16, seed=11)
    assert pkv.paged_attention_partition_tokens(w.num_seqs, 8, w.max_context_len, w.dtype) == \
        pkv.PARTITION_TOKENS_WIDE
    plan = _parity(w)
    assert plan.groups.shape[0] == prompts


def test_full_size_sampling_workload_sampled():
    host = make_workload(5, device="cuda")
    w = host.to("cuda")
    S = w.num_seqs
    order = torch.argsort(host.context_lens, descending=True).tolist()
    gen = torch.Generator().manual_seed(55)
    seqs = sorted(set([order[0], order[-1]] + torch.randperm(S, generator=gen)[:6].tolist()))
    sub = _sub_workload(w, seqs)                   # taken before the product step
    out, plan = shared_step(w, host)
    torch.cuda.synchronize()
    assert plan.groups.shape[0] == sum(1 for p in host.meta["prompt_lens"] if p >= 128)
    assert pkv.pkv_device_status(0) == 0
    ref, _, _ = oracle_step(sub, oracle_slots(sub))
    assert_close(out[torch.tensor(seqs, device="cuda")], ref, "8b_gqa_sampling shared")


def test_inconsistent_plans_are_flagged_and_stay_in_bounds():
    w = make_sampling(3, 4, (300, 600), (1, 100), 32, 8, 128, torch.bfloat16, seed=21)
    good = make_plan(w)
    assert good.groups.shape[0] == 3
    cases = []
    bad = good.shared_lens.clone()
    bad[1] += w.block_size                       # a member whose x differs from its group's
    cases.append(good._replace(shared_lens=bad))
    g_out = good.groups.clone()
    g_out[2, 0] = w.num_seqs - 2                 # a group that runs past the batch
    cases.append(good._replace(groups=g_out))
    g_big = good.groups.clone()
    g_big[0, 1] = 5                              # 5 members x 4 query heads > 16 rows
    cases.append(good._replace(groups=g_big))
    for item in ([~7, 0], [w.num_seqs, 0], [0, -1], [0, 1 << 20]):
        work = good.work.clone()                 # a group or sequence outside the batch, a bad partition
        work[-1] = torch.tensor(item, dtype=torch.int32)
        cases.append(good._replace(work=work))
    for plan in cases:
        g = w.to("cuda")
        shared_step(g, w, plan=plan)
        torch.cuda.synchronize()
        assert pkv.pkv_device_status(0) & BAD_PLAN
    # the context is intact: a consistent plan still matches the oracle
    _parity(w)


def test_stale_plan_member_table_is_flagged_and_its_row_left_unwritten():
    """A plan made before one member's table changed inside the shared range
    (a copy-on-write repoint after planning): the group pass finds the
    member's block id differing from the leader's, raises PKV_DEV_BAD_PLAN
    and the member's output row is never written; every other row is the
    oracle's attention.  ("Copy-on-Write: Sharing KV Cache": a shared block
    is copied before it diverges, so a table can change under a plan.)"""
    import dataclasses
    w = make_sampling(3, 4, (300, 600), (1, 100), 32, 8, 128, torch.bfloat16, seed=23)
    plan = make_plan(w)
    assert plan.groups.shape[0] == 3
    first, n = plan.groups[1].tolist()
    member = first + 2
    assert n == 4 and int(plan.shared_lens[member]) >= 6 * w.block_size
    used = set(w.block_tables[w.block_tables >= 0].tolist()) | set(w.copy_pairs.flatten().tolist())
    spare = next(b for b in range(w.num_blocks) if b not in used)
    bt = w.block_tables.clone()
    bt[member, 5] = spare                        # block 5 of the shared range, repointed after planning
    moved = dataclasses.replace(w, block_tables=bt)
    g = moved.to("cuda")
    out = torch.full_like(g.q, float("nan"))
    shared_step(g, moved, plan=plan, out=out)
    torch.cuda.synchronize()
    assert pkv.pkv_device_status(0) & BAD_PLAN
    assert torch.isnan(out[member].float()).all()
    ref, _, _ = oracle_step(moved, oracle_slots(moved))
    others = [s for s in range(w.num_seqs) if s != member]
    assert_close(out[torch.tensor(others, device="cuda")], ref[others], "rows of the other sequences")
    # the same batch with a fresh plan: every row, the moved member included
    pkv.pkv_device_status(0, clear=True)
    _parity(moved)


def test_rejected_calls():
    w = make_sampling(2, 4, (300, 400), (1, 50), 32, 8, 128, torch.bfloat16, seed=31).to("cuda")
    host = make_sampling(2, 4, (300, 400), (1, 50), 32, 8, 128, torch.bfloat16, seed=31)
    plan = make_plan(host).to("cuda")
    out = torch.empty_like(w.q)
    args = (out, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, w.max_context_len,
            plan.groups, plan.shared_lens)
    with pytest.raises(pkv.PagedKVError):       # workspace too small
        pkv.paged_attention_decode_shared(*args, plan.work, plan.part_tokens,
                                          workspace=torch.empty(256, dtype=torch.uint8, device="cuda"))
    with pytest.raises(pkv.PagedKVError):       # an empty work list
        pkv.paged_attention_decode_shared(*args, plan.work[:0], plan.part_tokens)
    with pytest.raises(pkv.PagedKVError):       # a list made for another partition size
        pkv.paged_attention_decode_shared(*args, plan.work, plan.part_tokens * 2)
    f = make_sampling(2, 2, (40, 60), (1, 10), 4, 4, 64, torch.float32, seed=3)
    fp = pkv.pkv_shared_prefix_plan(f.block_tables, f.context_lens, 16, 16, pkv.PARTITION_TOKENS, 16).to("cuda")
    f = f.to("cuda")
    with pytest.raises(pkv.PagedKVError) as e:   # fp32: the tensor-core kernel takes 16-bit inputs
        pkv.paged_attention_decode_shared(torch.empty_like(f.q), f.q, f.k_cache, f.v_cache, f.block_tables,
                                          f.context_lens, f.scale, f.max_context_len, fp.groups, fp.shared_lens,
                                          fp.work, fp.part_tokens)
    assert e.value.code == pkv._lib.C["PKV_ERR_UNSUPPORTED"]
    torch.cuda.synchronize()
    assert pkv.pkv_device_status(0) == 0


def test_shared_kernel_keeps_three_ctas_per_sm():
    import ctypes
    L = pkv._lib.lib()
    C = pkv._lib.C
    low = []
    for dtype in (C["PKV_F16"], C["PKV_BF16"]):
        for D in (64, 128):
            for G in (1, 2, 4, 8):
                for B in (8, 16, 32):
                    for long_p in (0, 1):
                        n = ctypes.c_int32(0)
                        assert L.pkv_debug_shared_occupancy(dtype, D, G, B, long_p, ctypes.byref(n)) == 0
                        if n.value < 3:
                            low.append((dtype, D, G, B, long_p, n.value))
    assert not low, f"below 3 CTAs per SM: {low}"
    n = ctypes.c_int32(0)
    assert L.pkv_debug_shared_occupancy(C["PKV_F32"], 128, 4, 16, 0, ctypes.byref(n)) == C["PKV_ERR_UNSUPPORTED"]


def test_shared_decode_replays_from_a_cuda_graph():
    """The shared-prefix step captured once and replayed gives the same bits
    as eager calls, also after the queries change in place (the plan, the
    work list and the workspace are device buffers, so nothing is read back
    or allocated under capture)."""
    host = make_sampling(6, 4, (300, 1500), (1, 200), 32, 8, 128, torch.bfloat16, seed=41)
    w = host.to("cuda")
    plan = make_plan(host).to("cuda")
    ws = torch.empty(pkv.paged_attention_shared_workspace_bytes(w.num_seqs, w.num_q_heads, w.head_dim,
                                                                host.max_context_len),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty_like(w.q)

    def step():
        pkv.paged_attention_decode_shared(out, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale,
                                          host.max_context_len, plan.groups, plan.shared_lens, plan.work,
                                          plan.part_tokens, k_new=w.k_new, v_new=w.v_new, workspace=ws)

    step()                                  # first call on the device: set-up outside capture
    torch.cuda.synchronize()
    eager = out.clone()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()
    out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)
    w.q.copy_(torch.randn(w.q.shape, generator=torch.Generator(device="cuda").manual_seed(3),
                          device="cuda").to(w.q.dtype))
    graph.replay()
    torch.cuda.synchronize()
    replayed = out.clone()
    step()
    torch.cuda.synchronize()
    assert torch.equal(replayed, out) and not torch.equal(replayed, eager)
    assert pkv.pkv_device_status(0) == 0


def test_write_then_shared_decode_equals_fused_bitwise():
    """Without k_new / v_new the call reads new tokens the caller wrote with
    paged_kv_write; the result is the fused call's, bit for bit."""
    host = make_sampling(5, 4, (200, 1800), (1, 300), 32, 8, 128, torch.bfloat16, seed=61)
    plan = make_plan(host)
    fused = host.to("cuda")
    out_fused, _ = shared_step(fused, host, plan=plan)
    sep = host.to("cuda")
    if sep.copy_pairs.numel():
        pkv.block_copy(sep.k_cache, sep.v_cache, sep.copy_pairs.cpu())
    slots = pkv.pkv_slot_mapping(host.block_tables, host.context_lens - 1, host.block_size).cuda()
    pkv.paged_kv_write(sep.k_new, sep.v_new, sep.k_cache, sep.v_cache, slots)
    d = plan.to("cuda")
    out_sep = torch.empty_like(sep.q)
    pkv.paged_attention_decode_shared(out_sep, sep.q, sep.k_cache, sep.v_cache, sep.block_tables, sep.context_lens,
                                      sep.scale, sep.max_context_len, d.groups, d.shared_lens, d.work, d.part_tokens)
    torch.cuda.synchronize()
    assert torch.equal(out_sep, out_fused)
    assert torch.equal(sep.k_cache, fused.k_cache) and torch.equal(sep.v_cache, fused.v_cache)
    assert pkv.pkv_device_status(0) == 0


def test_long_shared_prompt_many_records():
    """One 40,000-token prompt, 16 samples with one query head per kv head:
    the group pass covers about 80 partitions, so each row's reduce merges
    more than 32 records (several passes of its partition loop)."""
    w = make_sampling(1, 16, (40000, 40000), (1, 600), 2, 2, 64, torch.float16, seed=71, block_size=32)
    plan = _parity(w, min_shared_tokens=128)
    assert plan.groups.tolist() == [[0, 16]]
    assert plan.shared_lens[0].item() == (40000 // 32) * 32
    assert -(-plan.shared_lens[0].item() // plan.part_tokens) > 32
