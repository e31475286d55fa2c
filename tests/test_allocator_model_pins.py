"""Pins of the oracle's allocator model to the pages' worked examples (CPU only)."""

import pytest

from oracle.allocator_model import AllocatorModel, InvalidArgument, OutOfBlocks
from tests.conftest import load_golden


def test_on_demand_growth():
    gold = load_golden("on_demand_growth.json")
    B = gold["block_size"]
    m = AllocatorModel(200, B)
    m.add(1)
    have = 0
    for tokens, blocks in gold["tokens_to_blocks"]:
        m.append_tokens(1, tokens - have)
        have = tokens
        assert len(m.block_table(1)) == blocks, (tokens, blocks)
    # the 16th token still fits in the first block; the 17th opens the second
    m2 = AllocatorModel(4, B)
    m2.add(0)
    m2.append_tokens(0, 16)
    assert len(m2.block_table(0)) == 1
    m2.append_tokens(0, 1)
    assert len(m2.block_table(0)) == 2
    # waste: never more than block_size - 1 tokens per sequence
    m3 = AllocatorModel(600, B)
    for n in range(1, 1201, 37):
        m3.add(n)
        m3.append_tokens(n, n)
        waste = len(m3.block_table(n)) * B - n
        assert 0 <= waste <= gold["max_waste_tokens"]
        m3.free(n)


def test_worked_layout_and_free_list():
    gold = load_golden("worked_block_tables.json")
    # hand blocks out in the order that reproduces the page's tables
    order = [0, 2, 6, 4, 7, 1, 3, 9, 5, 8, 10, 11]
    m = AllocatorModel(12, gold["block_size"], initial_order=order)
    for sid, req, ntok in ((0, "A", 40), (1, "B", 48), (2, "C", 20)):
        m.add(sid)
        m.append_tokens(sid, ntok)
        assert m.block_table(sid) == gold["block_tables"][req]
    assert sorted(m.free_list()) == gold["free_blocks"]
    # slot of token t = physical block of its logical block * 16 + offset:
    # request A's token 20 is in logical block 1 (physical 2), offset 4
    m.append_tokens(0, 0)
    slots, _ = m.append_tokens(0, 1)     # token 41 (position 40): logical 2, offset 8
    assert slots == [6 * 16 + 8]


def test_immediate_release():
    gold = load_golden("immediate_release.json")
    B = gold["block_size"]
    m = AllocatorModel(20, B)
    m.add(0)
    m.append_tokens(0, B * gold["pages_of_finished_sequence"] - 5)
    before = m.num_free()
    held = m.block_table(0)
    m.free(0)
    assert m.num_free() == before + gold["pages_of_finished_sequence"]
    # the freed pages are reused first, in logical order
    m.add(1)
    m.append_tokens(1, B * 2)
    assert m.block_table(1) == held[:2]


def test_parallel_sampling():
    gold = load_golden("parallel_sampling.json")
    B, n = gold["block_size"], gold["samples"]
    m = AllocatorModel(20, B)
    m.add(100)
    m.append_tokens(100, len(gold["prompt_blocks"]) * B)   # prompt fills blocks 0-5
    assert m.block_table(100) == gold["prompt_blocks"]
    for j in range(n):
        m.fork(100, j)
    m.free(100)
    for j in range(n):
        slots, cow = m.append_tokens(j, 2 * B)
        assert cow is None                                    # prompt ends on a block edge
        assert m.block_table(j) == gold["prompt_blocks"] + gold["unique_blocks"][j]
    for b in gold["prompt_blocks"]:
        assert m.refcount(b) == n
    used = m.stats()["used_blocks"]
    assert used == gold["prompt_blocks_with_sharing"] + sum(len(u) for u in gold["unique_blocks"])
    assert n * len(gold["prompt_blocks"]) == gold["prompt_blocks_without_sharing"]


def test_prefix_sharing():
    gold = load_golden("prefix_sharing.json")
    B = gold["block_size"]
    m = AllocatorModel(5000, B)
    m.add(-1)
    m.append_tokens(-1, len(gold["prefix_blocks"]) * B)
    assert m.block_table(-1) == gold["prefix_blocks"]
    extra = [3 * B - 2, 3 * B, 2 * B - 7]
    for r, (uniq, ntok) in enumerate(zip(gold["request_unique_blocks"], extra)):
        m.add(r)
        m.share_prefix(r, gold["prefix_blocks"], len(gold["prefix_blocks"]) * B)
        m.append_tokens(r, ntok)
        assert m.block_table(r) == gold["prefix_blocks"] + uniq
    # 1000 users: the system prompt still occupies its 4 blocks only
    m2 = AllocatorModel(5000, B)
    m2.add(-1)
    m2.append_tokens(-1, len(gold["prefix_blocks"]) * B)
    pre = m2.block_table(-1)
    for u in range(gold["users"]):
        m2.add(u)
        m2.share_prefix(u, pre, len(pre) * B)
    m2.free(-1)
    assert m2.stats()["used_blocks"] == gold["blocks_with_sharing"]
    assert all(m2.refcount(b) == gold["users"] for b in pre)
    assert gold["users"] * len(pre) == gold["blocks_without_sharing"]


def test_copy_on_write_rule():
    """Writing into a shared partial block: every holder but the last copies."""
    B = 16
    m = AllocatorModel(32, B)
    m.add(0)
    m.append_tokens(0, 40)          # blocks 0,1,2; block 2 holds 8 tokens
    for j in (1, 2, 3):
        m.fork(0, j)
    assert m.refcount(2) == 4
    pairs = []
    for j in (1, 2, 3, 0):
        slots, cow = m.append_tokens(j, 1)
        if cow:
            pairs.append(cow)
        assert slots[0] % B == 8
    # three writers copied (fresh blocks 3, 4, 5); the last holder wrote in place
    assert pairs == [(2, 3), (2, 4), (2, 5)]
    assert m.block_table(0) == [0, 1, 2]
    assert m.refcount(2) == 1
    assert [m.block_table(j)[-1] for j in (1, 2, 3)] == [3, 4, 5]
    # a full shared block is never copied: the next token opens a new block
    m2 = AllocatorModel(8, B)
    m2.add(0)
    m2.append_tokens(0, 32)
    m2.fork(0, 1)
    _, cow = m2.append_tokens(1, 1)
    assert cow is None


def test_out_of_blocks_changes_nothing():
    m = AllocatorModel(3, 16)
    m.add(0)
    m.append_tokens(0, 40)
    m.fork(0, 1)
    state = (m.free_list(), m.block_table(0), m.block_table(1), m.num_tokens(1))
    with pytest.raises(OutOfBlocks):
        m.append_tokens(1, 30)      # needs a copy block plus one new block; 0 free
    assert state == (m.free_list(), m.block_table(0), m.block_table(1), m.num_tokens(1))
    with pytest.raises(InvalidArgument):
        m.add(0)
    with pytest.raises(InvalidArgument):
        m.free(7)


def test_prefix_cache_found_by_lookup():
    """The page's prefix example, with the sharing found by content: every
    request brings the same 64-token system prompt and its own question."""
    gold = load_golden("prefix_sharing.json")
    B = gold["block_size"]
    system = list(range(1000, 1000 + len(gold["prefix_blocks"]) * B))
    m = AllocatorModel(5000, B)
    for u in range(gold["users"]):
        m.add(u)
        question = [7, u % 97, u // 97, 3]
        slots, cached = m.append_prompt(u, system + question)
        assert cached == (0 if u == 0 else len(system))
        assert slots[:cached] == [-1] * cached
    pre = m.block_table(0)[:len(gold["prefix_blocks"])]
    assert all(m.refcount(b) == gold["users"] for b in pre)
    assert all(m.block_table(u)[:len(pre)] == pre for u in range(gold["users"]))
    # each user: 4 shared system blocks + 1 private block for the question
    assert m.stats()["used_blocks"] == gold["blocks_with_sharing"] + gold["users"]
    assert m.prefix_stats()["hit_tokens"] == (gold["users"] - 1) * len(system)


def test_prefix_cache_keeps_released_blocks_and_evicts_lru():
    B = 16
    m = AllocatorModel(6, B)                   # hands out 0, 1, 2, ...
    p1 = list(range(48))                       # 3 full blocks
    m.add(0)
    m.append_prompt(0, p1)                     # blocks 0, 1, 2, all cached
    m.free(0)                                  # released 2, 1, 0: all stay findable
    assert m.num_free() == 6 and m.prefix_stats()["evictable_blocks"] == 3
    assert m.free_list() == [3, 4, 5, 2, 1, 0]  # never-cached first, then least recently released
    m.add(1)
    _, cached = m.append_prompt(1, p1[:32] + [99] * 16)   # blocks 0, 1 hit; third differs -> block 3
    assert cached == 32 and m.block_table(1) == [0, 1, 3]
    assert m.prefix_stats()["evictable_blocks"] == 1       # block 2 still findable
    m.add(2)
    m.append_tokens(2, 32)                     # blocks 4, 5: the last never-cached ones
    assert m.prefix_stats()["evictions"] == 0
    m.add(3)
    m.append_tokens(3, 1)                      # nothing else free: block 2 is evicted
    assert m.block_table(3) == [2] and m.prefix_stats()["evictions"] == 1
    m.free(2)
    m.add(4)
    _, cached = m.append_prompt(4, p1)
    assert cached == 32                        # the evicted third block no longer matches
    assert m.block_table(4)[:2] == [0, 1]
