"""Host-side pieces of bench.py (CPU only): the relabelled sample of the
batch that the oracle baseline times, and the parity summary the bench
prints for the sampled sequences."""

import types

import numpy as np
import torch

import bench
import oracle
from oracle.allocator_model import slot_for_position
from paged_kv_cache_398_b200.workloads import make_workload


def _full_oracle_step(w):
    slots = torch.tensor([slot_for_position(w.block_tables[s].tolist(), int(w.context_lens[s]) - 1, w.block_size)
                          for s in range(w.num_seqs)], dtype=torch.int64)
    k, v = w.k_cache.clone(), w.v_cache.clone()
    if w.copy_pairs.numel():
        oracle.block_copy(k, v, w.copy_pairs)
    oracle.kv_write(k, v, w.k_new, w.v_new, slots)
    return oracle.paged_decode(w.q, k, v, w.block_tables, w.context_lens, w.scale)


def test_sample_gives_the_same_outputs_as_the_whole_batch():
    """Sampled sequences, their blocks gathered and relabelled (copy-on-write
    sources included), decode to exactly the whole batch's rows."""
    w = make_workload(5, device="cpu", num_prompts=3, max_prompt=400, max_output=200)
    seqs = [1, 4, 6]
    sub = bench.sub_workload(w, w.block_tables, w.context_lens, w.copy_pairs, seqs)
    assert sub.num_blocks < w.num_blocks
    refs = []
    bench.oracle_step_timed(sub, 2, keep=refs)
    whole = _full_oracle_step(w)
    assert np.array_equal(np.stack(refs), whole[seqs])


def test_repeated_step_reference_matches_the_batch_stepped_twice():
    """A sample whose new token lands in the copy-on-write source block makes
    a repeated step differ from the first; the sampled reference of the
    repeated step equals the whole batch's oracle step applied twice."""
    w = make_workload(5, device="cpu", num_prompts=40, max_prompt=300, max_output=6)
    B = w.block_size
    srcs = {int(a) for a, _ in w.copy_pairs.tolist()}
    writers_into_src = [s for s in range(w.num_seqs)
                        if int(w.block_tables[s, (int(w.context_lens[s]) - 1) // B]) in srcs]
    assert writers_into_src                            # the case this covers occurs in this batch
    seqs = sorted({s + 1 for s in writers_into_src if s % 4 == 0} | {2, 5})
    sub = bench.sub_workload(w, w.block_tables, w.context_lens, w.copy_pairs, seqs, repeated=True)
    refs = []
    bench.oracle_step_timed(sub, 2, keep=refs)
    # the whole batch, stepped twice by the oracle
    import oracle
    from oracle.allocator_model import slot_for_position
    slots = torch.tensor([slot_for_position(w.block_tables[s].tolist(), int(w.context_lens[s]) - 1, B)
                          for s in range(w.num_seqs)], dtype=torch.int64)
    k, v = w.k_cache.clone(), w.v_cache.clone()
    for _ in range(2):
        oracle.block_copy(k, v, w.copy_pairs)
        oracle.kv_write(k, v, w.k_new, w.v_new, slots)
    twice = oracle.paged_decode(w.q, k, v, w.block_tables, w.context_lens, w.scale)
    assert np.array_equal(np.stack(refs), twice[seqs])
    once = _full_oracle_step(w)
    assert not np.array_equal(once[seqs], twice[seqs])   # the repetition does change these rows


def test_parity_summary_counts_out_of_tolerance_elements():
    w = make_workload(1, device="cpu")
    seqs = list(range(w.num_seqs))
    sub = bench.sub_workload(w, w.block_tables, w.context_lens, w.copy_pairs, seqs)
    refs = []
    bench.oracle_step_timed(sub, 2, keep=refs)
    st = types.SimpleNamespace(out=torch.tensor(np.stack(refs)).to(w.dtype))
    base = {"seqs": seqs, "refs": refs}
    rep = bench.parity_on_sample(st, base)
    assert rep["out_of_tolerance"] == 0 and rep["max_abs_err"] < 1e-6
    assert rep["elements"] == w.num_seqs * w.num_q_heads * w.head_dim
    st.out[1, 2, 3] += 0.5
    rep = bench.parity_on_sample(st, base)
    assert rep["out_of_tolerance"] == 1 and rep["max_abs_err"] > 0.49


def test_event_brackets_are_few_and_spread():
    for steps in (1, 3, 20, 59, 60, 61, 119, 600, 1500):
        idx = bench.sampled_steps(steps)
        assert idx == sorted(set(idx)) and all(0 <= i < steps for i in idx)
        assert 1 <= len(idx) <= 60
        if steps <= 60:
            assert len(idx) == steps            # short runs bracket every step
    idx = bench.sampled_steps(1500)
    gaps = {b - a for a, b in zip(idx, idx[1:])}
    assert gaps == {25} and len(idx) == 60


def test_multi_query_step_layout():
    """--q-len: every sequence gets q_len new tokens at its last q_len
    positions, after a prompt of ctx - q_len tokens."""
    from oracle.allocator_model import slot_for_position
    QL = 4
    st = bench.build_step(2, torch.device("cpu"), 0, 6, 16, None, QL)
    S = st.w.num_seqs
    assert torch.equal(st.lens_host, st.w.context_lens) and int(st.lens_host.min()) >= QL
    assert tuple(st.q4.shape) == (S, QL, st.w.num_q_heads, st.w.head_dim)
    assert tuple(st.k_rows.shape) == (S * QL, st.w.num_kv_heads, st.w.head_dim)
    for s in range(S):
        for j in range(QL):
            pos = int(st.lens_host[s]) - QL + j
            assert int(st.slots[s * QL + j]) == slot_for_position(st.tables_host[s].tolist(), pos, 16)
    assert st.pairs.shape == (0, 2)


def test_packed_step_inputs_alias_one_buffer():
    """The step's inputs live in one packed buffer at 256-byte offsets (one
    H2D copy per step); a second buffer of the same layout binds the same way
    (the end-to-end loop alternates two)."""
    g = torch.Generator().manual_seed(3)
    S, Hq, Hkv, D, MB = 5, 8, 2, 64, 7
    st = types.SimpleNamespace(q_len=1, inputs=bench.STEP_INPUTS)
    st.q = torch.randn(S, Hq, D, generator=g).to(torch.bfloat16)
    st.k_new = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    st.v_new = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    st.slots = torch.arange(S, dtype=torch.int64) * 3
    st.block_tables = torch.randint(0, 50, (S, MB), generator=g, dtype=torch.int32)
    st.context_lens = torch.randint(1, 100, (S,), generator=g, dtype=torch.int32)
    st.out = torch.empty_like(st.q)
    orig = {n: getattr(st, n).clone() for n in bench.STEP_INPUTS}
    bench.pack_step_inputs(st, "cpu")
    base = st.in_dev.data_ptr()
    for name in bench.STEP_INPUTS:
        t = getattr(st, name)
        assert torch.equal(t, orig[name]) and (t.data_ptr() - base) % 256 == 0
        assert base <= t.data_ptr() < base + st.in_dev.numel()
    assert torch.equal(st.in_host, st.in_dev)
    assert st.q4.shape == (S, 1, Hq, D) and st.k_rows.shape == (S, Hkv, D)
    # a second buffer with the same layout
    other = torch.zeros_like(st.in_dev)
    out2 = torch.empty_like(st.out)
    b = bench.step_bindings(st, bench.input_views(st, other), out2)
    other.copy_(st.in_host)
    for name in bench.STEP_INPUTS:
        assert torch.equal(b[name], orig[name])
        assert b[name].data_ptr() - other.data_ptr() == getattr(st, name).data_ptr() - base
    assert b["out4"].data_ptr() == out2.data_ptr() and b["q4"].data_ptr() == b["q"].data_ptr()


def test_repeated_step_reference_equals_one_step_where_no_source_is_written():
    """On the prefix workload no new token lands in a block another sequence
    reads, so the repeated step's reference is the one-step reference."""
    w = make_workload(4, device="cpu", num_seqs=6, max_ctx=600)
    seqs = [0, 2, 5]
    once = bench.sub_workload(w, w.block_tables, w.context_lens, w.copy_pairs, seqs)
    again = bench.sub_workload(w, w.block_tables, w.context_lens, w.copy_pairs, seqs, repeated=True)
    r1, r2 = [], []
    bench.oracle_step_timed(once, 2, keep=r1)
    bench.oracle_step_timed(again, 2, keep=r2)
    assert np.array_equal(np.stack(r1), np.stack(r2))
    assert len(again.meta["pre_writes"][0]) == len(seqs)   # only the sampled sequences write into these blocks


def test_unique_live_tokens_counts_each_block_once_token_exact():
    """Brute force over (sequence, block) on a small sampling batch: shared
    prompt blocks count once, a partial block counts the most tokens any
    holder uses, and entries past a sequence's blocks are ignored."""
    w = make_workload(5, device="cpu", num_prompts=6, max_prompt=300, max_output=40, pad_random=True)
    B = w.block_size
    live = {}
    for s in range(w.num_seqs):
        n = int(w.context_lens[s])
        for i in range(-(-n // B)):
            b = int(w.block_tables[s, i])
            live[b] = max(live.get(b, 0), min(B, n - i * B))
    assert bench.unique_live_tokens(w.block_tables, w.context_lens, B) == sum(live.values())
    # without sharing it is the plain sum of the lengths
    w2 = make_workload(2, device="cpu", num_seqs=5, max_ctx=200)
    assert bench.unique_live_tokens(w2.block_tables, w2.context_lens, B) == int(w2.context_lens.sum())


def test_multi_query_oracle_sample_equals_the_whole_batch_oracle():
    """The bench's per-sequence oracle step for q_len new tokens (slot write
    of all of them, then causal multi-query decode) equals the oracle run
    on the whole batch at once."""
    QL = 3
    w = make_workload(2, device="cpu", num_seqs=4, max_ctx=120, min_ctx=QL)
    g = torch.Generator().manual_seed(3)
    S, Hq, Hkv, D = w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim
    q = torch.randn(S, QL, Hq, D, generator=g).to(w.dtype)
    kn = torch.randn(S, QL, Hkv, D, generator=g).to(w.dtype)
    vn = torch.randn(S, QL, Hkv, D, generator=g).to(w.dtype)
    seqs = [0, 2, 3]
    sub = bench.sub_workload(w, w.block_tables, w.context_lens, w.copy_pairs, seqs, q=q, k_new=kn, v_new=vn)
    refs = []
    bench.oracle_step_timed(sub, 2, keep=refs)
    k, v = w.k_cache.clone(), w.v_cache.clone()
    slots = torch.tensor([int(w.block_tables[s, p // 16]) * 16 + p % 16
                          for s in range(S) for p in range(int(w.context_lens[s]) - QL, int(w.context_lens[s]))])
    oracle.kv_write(k, v, kn.reshape(-1, Hkv, D), vn.reshape(-1, Hkv, D), slots)
    full = oracle.paged_decode_mq(q, k, v, w.block_tables, w.context_lens, w.scale)
    assert np.array_equal(np.stack(refs), full[seqs])


def test_clock_summary_covers_only_the_timed_windows():
    """The clock record: median SM clock, minimum, peak power and every
    slowdown reason of the samples inside the given windows only."""
    c = bench.ClockSampler.__new__(bench.ClockSampler)
    c.period, c.max_mhz, c.source = 0.002, 1965.0, "nvml"
    c.samples = [(0.0, 900.0, 100.0, 0x8),            # outside: hw_slowdown must not be reported
                 (1.0, 1965.0, 250.0, 0x0), (1.1, 1900.0, 300.0, 0x4), (1.2, 1950.0, 280.0, 0x0),
                 (5.0, 1800.0, 260.0, 0x20)]          # in the second window: sw_thermal_slowdown
    r = c.summary([(0.9, 1.3), (4.9, 5.1)], "test")
    assert r["samples"] == 4 and r["sm_mhz"] == 1925.0 and r["sm_min_mhz"] == 1800.0
    assert r["power_w_max"] == 300.0 and r["sm_max_mhz"] == 1965.0
    assert r["reasons"] == ["sw_power_cap", "sw_thermal_slowdown"]
    empty = c.summary([(2.0, 3.0)], "none")
    assert empty["samples"] == 0 and empty["sm_mhz"] is None
