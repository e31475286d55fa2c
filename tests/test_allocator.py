"""The native host block allocator against the oracle's list model (CPU only).

Every operation is applied to both; block tables, slots, copy pairs, free
lists, reference counts and statistics must agree exactly.  The pages'
worked examples run through the native allocator as well.
"""

import random

import pytest
import torch

import paged_kv_cache_398_b200 as pkv
from oracle.allocator_model import AllocatorModel, InvalidArgument, OutOfBlocks
from tests.conftest import load_golden


@pytest.fixture(scope="module", autouse=True)
def _built():
    from paged_kv_cache_398_b200.build import build_library
    build_library()


def _same(a: pkv.BlockAllocator, m: AllocatorModel, seqs):
    assert a.free_list() == m.free_list()
    assert a.num_free() == m.num_free()
    for s in seqs:
        assert a.block_table(s) == m.block_table(s)
        assert a.num_tokens(s) == m.num_tokens(s)
    for b in range(m.num_blocks):
        assert a.refcount(b) == m.refcount(b)
    st, sm = a.stats(), m.stats()
    for k in sm:
        assert st[k] == sm[k], k
    assert a.prefix_stats() == m.prefix_stats()


def test_worked_examples_native():
    gold = load_golden("worked_block_tables.json")
    order = [0, 2, 6, 4, 7, 1, 3, 9, 5, 8, 10, 11]
    a = pkv.BlockAllocator(12, 16, initial_order=order)
    for sid, req, ntok in ((0, "A", 40), (1, "B", 48), (2, "C", 20)):
        a.add(sid)
        a.append_tokens(sid, ntok)
        assert a.block_table(sid) == gold["block_tables"][req]
    assert sorted(a.free_list()) == gold["free_blocks"]

    g = load_golden("on_demand_growth.json")
    a = pkv.BlockAllocator(100, 16)
    a.add(1)
    have = 0
    for tokens, blocks in g["tokens_to_blocks"]:
        a.append_tokens(1, tokens - have)
        have = tokens
        assert len(a.block_table(1)) == blocks
    assert a.stats()["fragmentation_tokens"] <= g["max_waste_tokens"]

    ps = load_golden("parallel_sampling.json")
    a = pkv.BlockAllocator(20, 16)
    a.add(100)
    a.append_tokens(100, 6 * 16)
    for j in range(4):
        a.fork(100, j)
    a.free(100)
    for j in range(4):
        a.append_tokens(j, 32)
        assert a.block_table(j) == ps["prompt_blocks"] + ps["unique_blocks"][j]
    assert a.stats()["used_blocks"] == 14

    pre = load_golden("prefix_sharing.json")
    a = pkv.BlockAllocator(5000, 16)
    a.add(-1)
    a.append_tokens(-1, 64)
    for u in range(pre["users"]):
        a.add(u)
        a.share_prefix(u, pre["prefix_blocks"], 64)
    a.free(-1)
    assert a.stats()["used_blocks"] == pre["blocks_with_sharing"]
    assert a.refcount(0) == pre["users"]

    rel = load_golden("immediate_release.json")
    a = pkv.BlockAllocator(20, 16)
    a.add(0)
    a.append_tokens(0, 6 * 16 - 1)
    before = a.num_free()
    a.free(0)
    assert a.num_free() - before == rel["pages_of_finished_sequence"]


def test_copy_on_write_native():
    a = pkv.BlockAllocator(32, 16)
    a.add(0)
    a.append_tokens(0, 40)
    for j in (1, 2, 3):
        a.fork(0, j)
    pairs = []
    for j in (1, 2, 3, 0):
        slots, cow = a.append_tokens(j, 1)
        if cow:
            pairs.append(cow)
    assert pairs == [(2, 3), (2, 4), (2, 5)]
    assert a.refcount(2) == 1


@pytest.mark.parametrize("seed", [0, 1, 2, 3])
def test_random_operations_match_model(seed):
    rng = random.Random(seed)
    NB = rng.choice([24, 64, 200])
    order = list(range(NB))
    rng.shuffle(order)
    a = pkv.BlockAllocator(NB, 16, initial_order=order)
    m = AllocatorModel(NB, 16, initial_order=order)
    live, next_id = [], 0
    for step in range(400):
        op = rng.random()
        try:
            if op < 0.2 or not live:
                m.add(next_id)
                a.add(next_id)
                live.append(next_id)
                next_id += 1
            elif op < 0.55:
                s = rng.choice(live)
                if m.is_swapped(s):
                    continue
                n = rng.choice([0, 1, 1, 1, 3, 15, 16, 17, 40])
                try:
                    want = m.append_tokens(s, n)
                except OutOfBlocks:
                    with pytest.raises(pkv.OutOfBlocks):
                        a.append_tokens(s, n)
                else:
                    got = a.append_tokens(s, n)
                    assert got == (want[0], want[1])
            elif op < 0.65:
                batch = [q for q in rng.sample(live, k=min(len(live), rng.randint(1, 6))) if not m.is_swapped(q)]
                if not batch:
                    continue
                try:
                    ws, wp = m.append_one_batch(batch)
                except OutOfBlocks:
                    with pytest.raises(pkv.OutOfBlocks):
                        a.append_one_batch(batch)
                else:
                    gs, gp = a.append_one_batch(batch)
                    assert gs.tolist() == ws and [tuple(p) for p in gp.tolist()] == wp
            elif op < 0.8:
                s = rng.choice(live)
                if m.is_swapped(s):
                    continue
                m.fork(s, next_id)
                a.fork(s, next_id)
                live.append(next_id)
                next_id += 1
            elif op < 0.83 and live:
                s = rng.choice(live)
                if m.is_swapped(s):
                    try:
                        want = m.swap_in(s)
                    except OutOfBlocks:
                        with pytest.raises(pkv.OutOfBlocks):
                            a.swap_in(s)
                    else:
                        assert a.swap_in(s) == want
                else:
                    assert a.swap_out(s) == m.swap_out(s)
                assert a.is_swapped(s) == m.is_swapped(s)
            elif op < 0.87 and live:
                s = rng.choice(live)
                if m.num_tokens(s) == 0 and not m.is_swapped(s):
                    src = rng.choice(live)
                    blocks = m.block_table(src)
                    full = len(blocks) * 16
                    if blocks and m.num_tokens(src) == full and not m.is_swapped(src):
                        m.share_prefix(s, blocks, full)
                        a.share_prefix(s, blocks, full)
            else:
                s = rng.choice(live)
                m.free(s)
                a.free(s)
                live.remove(s)
        except InvalidArgument:
            pytest.fail("model rejected a generated operation")
        _same(a, m, live)


def test_invalid_operations_native():
    a = pkv.BlockAllocator(4, 16)
    a.add(0)
    with pytest.raises(pkv.PagedKVError):
        a.add(0)
    with pytest.raises(pkv.PagedKVError):
        a.free(9)
    with pytest.raises(pkv.PagedKVError):
        a.fork(9, 10)
    a.append_tokens(0, 64)
    with pytest.raises(pkv.OutOfBlocks):
        a.append_tokens(0, 1)
    assert a.block_table(0) == [0, 1, 2, 3]
    with pytest.raises(pkv.PagedKVError):
        pkv.BlockAllocator(3, 16, initial_order=[0, 0, 1])
    a.add(1)
    with pytest.raises(pkv.PagedKVError):
        a.share_prefix(1, [0, 1], 40)      # 40 tokens need 3 blocks
    with pytest.raises(pkv.PagedKVError):
        a.append_one_batch([0, 0])


def test_batch_tables_pad():
    a = pkv.BlockAllocator(10, 16)
    for s, n in ((0, 5), (1, 33)):
        a.add(s)
        a.append_tokens(s, n)
    t, lens = a.batch_tables([1, 0], 4, pad=-1)
    assert t.tolist() == [[1, 2, 3, -1], [0, -1, -1, -1]]
    assert lens.tolist() == [33, 5]


def test_serving_loop_buffers_and_keep_tail():
    """A serving loop refills the same host buffers every step: with
    TABLE_KEEP_TAIL only each table's live entries are written, and reused
    output buffers give the same slots and copy pairs as fresh ones."""
    a = pkv.BlockAllocator(64, 16, initial_order=list(reversed(range(64))))
    b = pkv.BlockAllocator(64, 16, initial_order=list(reversed(range(64))))
    for x in (a, b):
        for s, n in enumerate((40, 17, 3)):
            x.add(s)
            x.append_tokens(s, n)
        x.fork(0, 3)
    ids = torch.arange(4, dtype=torch.int64)
    slots_buf = torch.full((8,), -7, dtype=torch.int64)
    pairs_buf = torch.full((8, 2), -7, dtype=torch.int64)
    tables = torch.full((4, 6), 777, dtype=torch.int32)
    lens = torch.zeros(4, dtype=torch.int32)
    for step in range(20):
        s1, p1 = a.append_one_batch(ids, slots_out=slots_buf, pairs_out=pairs_buf)
        s2, p2 = b.append_one_batch(list(range(4)))
        assert torch.equal(s1, s2) and torch.equal(p1, p2)
        t, n = a.batch_tables(ids, 6, pad=pkv.TABLE_KEEP_TAIL, tables_out=tables, lens_out=lens)
        for s in range(4):
            bt = a.block_table(s)
            assert t[s, :len(bt)].tolist() == bt
            assert n[s] == a.num_tokens(s)
    # entries past the longest table each row ever had were never written
    assert tables[2, 4:].tolist() == [777, 777]
    full, _ = a.batch_tables(ids, 6)
    assert (full[2, len(a.block_table(2)):] == -1).all()
    with pytest.raises(ValueError):
        a.batch_tables(ids, 5, tables_out=tables, lens_out=lens)


def test_swap_out_and_in_native():
    """Preemption: a swapped-out sequence gives its blocks back, keeps its
    token count, and resumes in fresh blocks; shared blocks stay with the
    other holders."""
    a = pkv.BlockAllocator(12, 16)
    m = AllocatorModel(12, 16)
    for x in (a, m):
        x.add(0)
        x.append_tokens(0, 40)            # blocks 0, 1, 2
        x.fork(0, 1)                      # 1 shares them
        x.append_tokens(1, 30)            # CoW of block 2 (-> 3), then new blocks 4 and 5
    assert a.block_table(1) == m.block_table(1)
    out_a, out_m = a.swap_out(1), m.swap_out(1)
    assert out_a == out_m == [0, 1, 3, 4, 5]
    assert a.is_swapped(1) and a.num_tokens(1) == 70
    assert a.refcount(0) == 1 and a.refcount(3) == 0       # shared kept, private freed
    for bad in (lambda: a.append_tokens(1, 1), lambda: a.fork(1, 9), lambda: a.batch_tables([1], 8),
                lambda: a.swap_out(1)):
        with pytest.raises(pkv.PagedKVError):
            bad()
    # another request takes the freed blocks; the swapped one comes back elsewhere
    for x in (a, m):
        x.add(2)
        x.append_tokens(2, 32)
    assert a.block_table(2) == m.block_table(2)
    back_a, back_m = a.swap_in(1), m.swap_in(1)
    assert back_a == back_m and len(back_a) == 5
    assert not a.is_swapped(1) and a.block_table(1) == back_a
    assert a.stats() == m.stats()
    with pytest.raises(pkv.PagedKVError):
        a.swap_in(1)


def test_swap_in_is_all_or_nothing():
    a = pkv.BlockAllocator(4, 16)
    a.add(0)
    a.append_tokens(0, 48)                # 3 blocks
    a.swap_out(0)
    a.add(1)
    a.append_tokens(1, 40)                # takes 3 of the 4 blocks
    with pytest.raises(pkv.OutOfBlocks):
        a.swap_in(0)
    assert a.is_swapped(0) and a.num_free() == 1
    a.free(1)
    assert len(a.swap_in(0)) == 3


def test_swap_kernels_reject_bad_lists_on_host():
    from paged_kv_cache_398_b200._lib import C, lib
    import ctypes
    L = lib()
    buf = (ctypes.c_uint8 * 64)()
    p = ctypes.addressof(buf) + (-ctypes.addressof(buf)) % 16
    for ids, fn in (([0, 9], "swap_blocks_out"), ([-1], "swap_blocks_in"), ([2, 2], "swap_blocks_in")):
        t = torch.tensor(ids, dtype=torch.int64)
        rc = getattr(L, fn)(p, p, t.data_ptr(), t.numel(), p, p, 2, 64, 16, 8, C["PKV_F16"], None)
        assert rc == C["PKV_ERR_INVALID_ARG"], (ids, fn)


def test_prefix_cache_golden_native():
    gold = load_golden("prefix_sharing.json")
    B = gold["block_size"]
    system = list(range(1000, 1000 + len(gold["prefix_blocks"]) * B))
    a = pkv.BlockAllocator(5000, B)
    for u in range(gold["users"]):
        a.add(u)
        slots, cached = a.append_prompt(u, system + [7, u % 97, u // 97, 3])
        assert cached == (0 if u == 0 else len(system))
        assert (slots[:cached] == -1).all()
    pre = a.block_table(0)[:len(gold["prefix_blocks"])]
    assert all(a.refcount(b) == gold["users"] for b in pre)
    assert a.stats()["used_blocks"] == gold["blocks_with_sharing"] + gold["users"]


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_prefix_cache_random_prompts_match_model(seed):
    """Prompts drawn from a few shared system prompts, in a pool small
    enough to force evictions; every step compared with the model."""
    rng = random.Random(100 + seed)
    B, NB = 16, 60
    a = pkv.BlockAllocator(NB, B)
    m = AllocatorModel(NB, B)
    systems = [[rng.randrange(50) for _ in range(rng.choice([16, 32, 40, 64]))] for _ in range(3)]
    live, sid = [], 0
    for step in range(300):
        r = rng.random()
        if r < 0.45 or not live:
            toks = list(rng.choice(systems)) + [rng.randrange(50) for _ in range(rng.randrange(0, 40))]
            m.add(sid)
            a.add(sid)
            try:
                want = m.append_prompt(sid, toks)
            except OutOfBlocks:
                with pytest.raises(pkv.OutOfBlocks):
                    a.append_prompt(sid, toks)
                m.free(sid)
                a.free(sid)
            else:
                slots, cached = a.append_prompt(sid, toks)
                assert (slots.tolist(), cached) == want
                live.append(sid)
            sid += 1
        elif r < 0.75:
            s = rng.choice(live)
            m.free(s)
            a.free(s)
            live.remove(s)
        elif r < 0.9:
            s = rng.choice(live)
            n = rng.choice([1, 5, 17])
            try:
                want = m.append_tokens(s, n)
            except OutOfBlocks:
                with pytest.raises(pkv.OutOfBlocks):
                    a.append_tokens(s, n)
            else:
                assert a.append_tokens(s, n) == (want[0], want[1])
        else:
            s = rng.choice(live)
            m.fork(s, sid)
            a.fork(s, sid)
            live.append(sid)
            sid += 1
        _same(a, m, live)
    assert m.prefix_stats()["evictions"] > 0 and m.prefix_stats()["hit_tokens"] > 0
