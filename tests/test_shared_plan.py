"""pkv_shared_prefix_plan: the host half of shared-prefix decode (no GPU).

The plan groups consecutive sequences whose block tables start with the same
physical blocks, and picks for each group the shared length x whose blocks
the group pass reads once.  Checked against the pages' two sharing examples
("Copy-on-Write: Sharing KV Cache": "Parallel Sampling" with prompt blocks
0-5 and two unique blocks per output, and "Prefix Caching" with system
prompt blocks 0-3), against tables that the native allocator builds by
forking, and against a brute-force search over every grouping of small
batches.
"""

import itertools
import random

import pytest
import torch

import paged_kv_cache_398_b200 as pkv

B = 16
PT = 512   # partition size of the work lists


def _tables(rows):
    mb = max(len(r) for r in rows)
    t = torch.full((len(rows), mb), -1, dtype=torch.int32)
    for i, r in enumerate(rows):
        t[i, :len(r)] = torch.tensor(r, dtype=torch.int32)
    return t


def _check_valid(tables, lens, plan, max_group, min_tokens, block_size=B):
    """Every property the decode relies on, checked from the definitions."""
    S = lens.shape[0]
    shared = plan.shared_lens.tolist()
    seen = [False] * S
    prev_end = 0
    for first, n in plan.groups.tolist():
        assert first >= prev_end and 2 <= n <= max_group and first + n <= S
        prev_end = first + n
        x = shared[first]
        assert x % block_size == 0 and x >= max(min_tokens, block_size)
        nb = x // block_size
        for j in range(first, first + n):
            assert not seen[j]
            seen[j] = True
            assert shared[j] == x
            assert x < int(lens[j])                                  # the member keeps its last position
            assert tables[j, :nb].tolist() == tables[first, :nb].tolist()   # same physical blocks
            assert (tables[j, :nb] >= 0).all()
    for j in range(S):
        if not seen[j]:
            assert shared[j] == 0
    assert plan.max_shared_len == max(shared + [0])
    assert plan.max_own_len == max(int(lens[j]) - shared[j] for j in range(S))
    # the work list: every partition of both passes exactly once, longest first
    pt = plan.part_tokens
    expect = {}
    for g, (first, n) in enumerate(plan.groups.tolist()):
        x = shared[first]
        for p in range(-(-x // pt)):
            expect[(~g, p)] = min(pt, x - p * pt)
    for j in range(S):
        own = int(lens[j]) - shared[j]
        for p in range(-(-own // pt)):
            expect[(j, p)] = min(pt, own - p * pt)
    items = [tuple(it) for it in plan.work.tolist()]
    assert len(items) == len(set(items)) and set(items) == set(expect)
    sizes = [expect[it] for it in items]
    assert sizes == sorted(sizes, reverse=True)


def test_parallel_sampling_example():
    # four outputs of one prompt: blocks 0-5 shared, unique blocks [6,7], [8,9], [10,11], [12,13]
    rows = [[0, 1, 2, 3, 4, 5, 6 + 2 * j, 7 + 2 * j] for j in range(4)]
    lens = torch.tensor([6 * B + 20] * 4, dtype=torch.int32)
    plan = pkv.pkv_shared_prefix_plan(_tables(rows), lens, B, max_group=4, part_tokens=PT, min_shared_tokens=B)
    assert plan.groups.tolist() == [[0, 4]]
    assert plan.shared_lens.tolist() == [6 * B] * 4          # the 6 prompt blocks, read once
    assert plan.max_own_len == 20
    # two query rows per sample (G = 8): groups of at most 2
    plan2 = pkv.pkv_shared_prefix_plan(_tables(rows), lens, B, max_group=2, part_tokens=PT, min_shared_tokens=B)
    assert plan2.groups.tolist() == [[0, 2], [2, 2]]


def test_prefix_caching_example():
    # system prompt in blocks 0-3; requests with unique [4,5,6], [7,8,9], [10,11]
    rows = [[0, 1, 2, 3, 4, 5, 6], [0, 1, 2, 3, 7, 8, 9], [0, 1, 2, 3, 10, 11]]
    lens = torch.tensor([7 * B, 7 * B - 3, 6 * B - 1], dtype=torch.int32)
    plan = pkv.pkv_shared_prefix_plan(_tables(rows), lens, B, max_group=16, part_tokens=PT, min_shared_tokens=64)
    assert plan.groups.tolist() == [[0, 3]]
    assert plan.shared_lens.tolist() == [64, 64, 64]
    # a threshold above the system prompt: no group
    none = pkv.pkv_shared_prefix_plan(_tables(rows), lens, B, max_group=16, part_tokens=PT, min_shared_tokens=65)
    assert none.groups.numel() == 0 and none.shared_lens.tolist() == [0, 0, 0]
    assert none.max_own_len == 7 * B


def test_shared_length_stays_below_every_member_length():
    # two sequences hold the same 3 blocks, one of them is exactly 3 blocks long:
    # its last position must stay with its own pass, so x is 2 blocks
    rows = [[5, 6, 7], [5, 6, 7, 8]]
    lens = torch.tensor([3 * B, 3 * B + 4], dtype=torch.int32)
    plan = pkv.pkv_shared_prefix_plan(_tables(rows), lens, B, max_group=4, part_tokens=PT, min_shared_tokens=1)
    assert plan.groups.tolist() == [[0, 2]] and plan.shared_lens.tolist() == [2 * B, 2 * B]
    assert plan.max_own_len == B + 4


def test_a_different_first_block_ends_a_run():
    rows = [[1, 2, 3], [1, 2, 9], [4, 2, 3], [4, 2, 3]]
    lens = torch.tensor([3 * B] * 4, dtype=torch.int32)
    plan = pkv.pkv_shared_prefix_plan(_tables(rows), lens, B, max_group=8, part_tokens=PT, min_shared_tokens=1)
    assert plan.groups.tolist() == [[0, 2], [2, 2]]
    assert plan.shared_lens.tolist() == [2 * B, 2 * B, 2 * B, 2 * B]


def _forked_batch(seed, block_size, n_prompts=6, samples=4):
    """Tables from the native allocator: prompts forked into samples that each
    then append their own tokens (copy-on-write of a partial last block)."""
    rng = random.Random(seed)
    alloc = pkv.BlockAllocator(4096, block_size, initial_order=torch.randperm(4096, generator=torch.Generator().manual_seed(seed)))
    ids = []
    for p in range(n_prompts):
        parent = p * 100
        alloc.add(parent)
        alloc.append_tokens(parent, rng.randint(1, 300))
        kids = [parent] + [parent + j for j in range(1, rng.randint(1, samples))]
        for c in kids[1:]:
            alloc.fork(parent, c)
        for c in kids:
            alloc.append_tokens(c, rng.randint(1, 60))
        ids += kids
        if rng.random() < 0.3:                        # an unrelated request between prompts
            lone = p * 100 + 99
            alloc.add(lone)
            alloc.append_tokens(lone, rng.randint(1, 200))
            ids.append(lone)
    return alloc.batch_tables(ids, 64)


@pytest.mark.parametrize("block_size", [8, 16, 32])
@pytest.mark.parametrize("max_group,min_tokens", [(4, 1), (16, 1), (2, 64), (4, 128)])
def test_plans_of_forked_batches_are_valid(block_size, max_group, min_tokens):
    for seed in range(5):
        tables, lens = _forked_batch(seed * 7 + block_size, block_size)
        for pt in (64, 512):
            plan = pkv.pkv_shared_prefix_plan(tables, lens, block_size, max_group, pt, min_tokens)
            _check_valid(tables, lens, plan, max_group, min_tokens, block_size)


def _best_by_search(tables, lens, max_group, min_tokens):
    """Brute force over every split of the batch into consecutive runs: the
    largest number of block reads saved, sum over groups of (n - 1) * x / B."""
    S = lens.shape[0]
    below = [(int(lens[j]) - 1) // B for j in range(S)]

    def x_of(i, n):
        c = below[i]
        for j in range(i + 1, i + n):
            k = 0
            while k < min(c, below[j]) and tables[i, k] >= 0 and tables[i, k] == tables[j, k]:
                k += 1
            c = k
        return c * B

    best = 0
    for cuts in itertools.product([0, 1], repeat=S - 1):
        i, saved, ok = 0, 0, True
        bounds = [j + 1 for j, c in enumerate(cuts) if c] + [S]
        for end in bounds:
            n = end - i
            if n >= 2:
                x = x_of(i, n)
                if n > max_group or x < max(min_tokens, B):
                    ok = False
                    break
                saved += (n - 1) * x // B
            i = end
        if ok:
            best = max(best, saved)
    return best


def test_greedy_matches_search_on_sampling_batches():
    # runs of samples of one prompt: the greedy plan saves as many block reads
    # as the best split found by exhaustive search
    rng = random.Random(3)
    for trial in range(30):
        rows, lens = [], []
        nxt = 1000
        while len(rows) < rng.randint(4, 9):
            pl = rng.randint(1, 6)
            prompt = list(range(nxt, nxt + pl))
            nxt += pl
            for _ in range(rng.randint(1, 4)):
                own = list(range(nxt, nxt + rng.randint(1, 2)))
                nxt += len(own)
                rows.append(prompt + own)
                lens.append((len(prompt) + len(own) - 1) * B + rng.randint(1, B))
        rows, lens = rows[:9], lens[:9]
        t, cl = _tables(rows), torch.tensor(lens, dtype=torch.int32)
        plan = pkv.pkv_shared_prefix_plan(t, cl, B, max_group=4, part_tokens=PT, min_shared_tokens=1)
        _check_valid(t, cl, plan, 4, 1)
        saved = sum((n - 1) * plan.shared_lens[f].item() // B for f, n in plan.groups.tolist())
        assert saved == _best_by_search(t, cl, 4, 1), trial


def test_invalid_arguments():
    t = _tables([[0, 1], [0, 1]])
    with pytest.raises(pkv.PagedKVError):
        pkv.pkv_shared_prefix_plan(t, torch.tensor([0, 5], dtype=torch.int32), B, 4, PT)        # length 0
    with pytest.raises(pkv.PagedKVError):
        pkv.pkv_shared_prefix_plan(t, torch.tensor([2 * B + 1, 5], dtype=torch.int32), B, 4, PT)  # past the row
    with pytest.raises(pkv.PagedKVError):
        pkv.pkv_shared_prefix_plan(t, torch.tensor([5, 5], dtype=torch.int32), B, 0, PT)        # no room
    with pytest.raises(pkv.PagedKVError):
        pkv.pkv_shared_prefix_plan(t, torch.tensor([5, 5], dtype=torch.int32), B, 4, 0)         # no partition size
    empty = pkv.pkv_shared_prefix_plan(torch.empty(0, 4, dtype=torch.int32), torch.empty(0, dtype=torch.int32),
                                       B, 4, PT)
    assert empty.groups.numel() == 0 and empty.max_shared_len == 0 and empty.max_own_len == 0
    assert empty.work.numel() == 0


def test_work_list_size_query_and_short_buffer():
    import ctypes
    rows = [[0, 1, 2, 3, 4, 5, 6 + 2 * j, 7 + 2 * j] for j in range(4)]
    t, lens = _tables(rows), torch.tensor([6 * B + 20] * 4, dtype=torch.int32)
    L = pkv._lib.lib()
    g, sh = torch.empty(4, 2, dtype=torch.int32), torch.empty(4, dtype=torch.int32)
    ng, nw, a, b = (ctypes.c_int32(0) for _ in range(4))
    args = (t.data_ptr(), t.shape[1], lens.data_ptr(), 4, B, 4, B, 32, g.data_ptr(), ctypes.byref(ng), sh.data_ptr())
    assert L.pkv_shared_prefix_plan(*args, None, 0, ctypes.byref(nw), ctypes.byref(a), ctypes.byref(b)) == 0
    assert nw.value == 3 + 4                  # 96 shared tokens in 32-token partitions, one own item each
    w = torch.empty(6, 2, dtype=torch.int32)
    rc = L.pkv_shared_prefix_plan(*args, w.data_ptr(), 6, ctypes.byref(nw), ctypes.byref(a), ctypes.byref(b))
    assert rc == pkv._lib.C["PKV_ERR_INVALID_ARG"] and nw.value == 7


def test_plans_of_arbitrary_tables_are_valid():
    """Property test: any batch of tables and lengths (runs that share random
    prefixes, invalid ids, lengths anywhere in their rows) gets a plan that
    satisfies every property the decode relies on."""
    from hypothesis import given, settings, strategies as st

    @settings(max_examples=200, deadline=None, derandomize=True)
    @given(st.data())
    def check(data):
        bs = data.draw(st.sampled_from([8, 16, 32]))
        mb = data.draw(st.integers(1, 12))
        S = data.draw(st.integers(1, 10))
        rows, base = [], None
        for _ in range(S):
            if base is None or data.draw(st.booleans()):
                base = data.draw(st.lists(st.integers(-1, 40), min_size=mb, max_size=mb))
            keep = data.draw(st.integers(0, mb))
            tail = data.draw(st.lists(st.integers(-1, 40), min_size=mb - keep, max_size=mb - keep))
            rows.append(base[:keep] + tail)
        t = torch.tensor(rows, dtype=torch.int32)
        lens = torch.tensor([data.draw(st.integers(1, mb * bs)) for _ in range(S)], dtype=torch.int32)
        max_group = data.draw(st.integers(1, 16))
        min_tokens = data.draw(st.sampled_from([0, 1, bs, 64]))
        pt = data.draw(st.sampled_from([bs, 64, 512]))
        plan = pkv.pkv_shared_prefix_plan(t, lens, bs, max_group, pt, min_tokens)
        _check_valid(t, lens, plan, max_group, min_tokens, bs)

    check()


# ---------------------------------------------------------------------------
# pkv_shared_prefix_order: a batch order that makes sharing sequences adjacent
# ---------------------------------------------------------------------------
def test_order_regroups_an_interleaved_batch():
    """Samples of several prompts, shuffled through the batch: the plan of
    the shuffled batch finds (almost) nothing; reordered by
    pkv_shared_prefix_order, it finds every group the unshuffled batch has."""
    from paged_kv_cache_398_b200.workloads import make_sampling
    w = make_sampling(6, 4, (300, 900), (1, 60), 8, 2, 64, torch.float16, seed=17)
    plan = pkv.pkv_shared_prefix_plan(w.block_tables, w.context_lens, B, 4, 512)
    perm = torch.randperm(w.num_seqs, generator=torch.Generator().manual_seed(3))
    bt, cl = w.block_tables[perm], w.context_lens[perm]
    shuffled = pkv.pkv_shared_prefix_plan(bt, cl, B, 4, 512)
    order = pkv.pkv_shared_prefix_order(bt, cl, B)
    assert sorted(order.tolist()) == list(range(w.num_seqs))
    again = pkv.pkv_shared_prefix_plan(bt[order], cl[order], B, 4, 512)
    assert shuffled.groups.shape[0] < plan.groups.shape[0]
    assert again.groups.shape[0] == plan.groups.shape[0]
    assert int(again.shared_lens.sum()) == int(plan.shared_lens.sum())
    _check_valid(bt[order], cl[order], again, 4, 128)


def test_order_makes_every_common_prefix_contiguous():
    """Brute force on random small tables: after the reordering, the
    sequences whose shareable blocks start with any given prefix sit at
    consecutive positions, and sequences with equal rows keep their batch
    order."""
    rng = random.Random(5)
    for _ in range(300):
        S = rng.randint(1, 9)
        lens = [rng.randint(1, 5 * B) for _ in range(S)]
        rows = [[rng.choice([0, 1, 2, rng.randint(3, 40)]) for _ in range(5)] for _ in range(S)]
        for r in rows:                                  # now and then a hole (-1) inside a row
            if rng.random() < 0.2:
                r[rng.randint(0, 4)] = -1
        bt, cl = _tables(rows), torch.tensor(lens, dtype=torch.int32)
        order = pkv.pkv_shared_prefix_order(bt, cl, B).tolist()
        assert sorted(order) == list(range(S))

        def key(s):                                   # shareable blocks: valid ids below the last position
            k = []
            for b in rows[s][:(lens[s] - 1) // B]:
                if b < 0:
                    break
                k.append(b)
            return k
        keys = [key(s) for s in order]
        for L in range(1, 6):
            seen = {}
            for pos, k in enumerate(keys):
                if len(k) >= L:
                    seen.setdefault(tuple(k[:L]), []).append(pos)
            for positions in seen.values():
                # no sequence without the prefix sits between two that hold it
                assert positions == list(range(positions[0], positions[-1] + 1))
        for i in range(S - 1):
            if keys[i] == keys[i + 1]:
                assert order[i] < order[i + 1]


def test_order_rejects_bad_arguments():
    L = pkv._lib.lib()
    C = pkv._lib.C
    bt, cl = _tables([[0, 1], [0, 2]]), torch.tensor([20, 40], dtype=torch.int32)
    assert pkv.pkv_shared_prefix_order(bt[:0], cl[:0], B).numel() == 0
    with pytest.raises(pkv.PagedKVError):
        pkv.pkv_shared_prefix_order(bt, torch.tensor([20, 33], dtype=torch.int32), B)   # past the table
    with pytest.raises(pkv.PagedKVError):
        pkv.pkv_shared_prefix_order(bt, torch.tensor([0, 20], dtype=torch.int32), B)    # empty sequence
    assert L.pkv_shared_prefix_order(None, 2, None, 2, B, None) == C["PKV_ERR_INVALID_ARG"]
