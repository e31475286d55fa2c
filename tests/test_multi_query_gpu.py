"""Multi-query decode and the fused slot write against the oracle (needs a B200).

q_len new tokens per sequence: token j sits at position ctx - q_len + j and
attends causally.  The product either writes the tokens first
(paged_kv_write) or fuses the write into paged_attention_decode_mq; both must
match the oracle's slot write + multi-query decode, and each other bit for bit.
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


def assert_close(got, ref, what=""):
    g = got.detach().cpu().double().numpy()
    err = np.abs(g - ref)
    assert np.isfinite(g).all(), f"{what}: non-finite output"
    bad = err > ATOL + RTOL * np.abs(ref)
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} out of tolerance, max abs {err.max():.3e}"


def oracle_slots_mq(w, q_len):
    """Slots of the q_len new tokens of every sequence (oracle's own arithmetic)."""
    out = []
    for s in range(w.num_seqs):
        ctx = int(w.context_lens[s])
        row = w.block_tables[s].tolist()
        out += [slot_for_position(row, ctx - q_len + j, w.block_size) for j in range(q_len)]
    return torch.tensor(out, dtype=torch.int64)


def oracle_mq(w, q_len):
    k, v = w.k_cache.clone(), w.v_cache.clone()
    S, Hkv, D = w.num_seqs, w.num_kv_heads, w.head_dim
    oracle.kv_write(k, v, w.k_new.reshape(S * q_len, Hkv, D).contiguous(),
                    w.v_new.reshape(S * q_len, Hkv, D).contiguous(), oracle_slots_mq(w, q_len))
    return oracle.paged_decode_mq(w.q, k, v, w.block_tables, w.context_lens, w.scale), k, v


@pytest.fixture(autouse=True)
def _clean_status(cuda_device):
    pkv.pkv_device_status(0, clear=True)
    yield
    torch.cuda.synchronize()


def _both_paths(w, q_len):
    """(separate write + decode_mq, fused decode_mq) outputs and caches on the GPU."""
    S, Hkv, D = w.num_seqs, w.num_kv_heads, w.head_dim
    Bs = w.block_size
    slots = torch.tensor([slot_for_position(w.block_tables[s].tolist(), int(w.context_lens[s]) - q_len + j, Bs)
                          for s in range(S) for j in range(q_len)], dtype=torch.int64)
    prod_slots = torch.cat([pkv.pkv_slot_mapping(w.block_tables, w.context_lens - q_len + j, Bs)[:, None]
                            for j in range(q_len)], dim=1).reshape(-1)
    assert torch.equal(prod_slots, slots)
    a = w.to("cuda")
    pkv.paged_kv_write(a.k_new.reshape(S * q_len, Hkv, D), a.v_new.reshape(S * q_len, Hkv, D), a.k_cache,
                       a.v_cache, prod_slots.cuda())
    out_a = torch.empty_like(a.q)
    pkv.paged_attention_decode_mq(out_a, a.q, a.k_cache, a.v_cache, a.block_tables, a.context_lens, a.scale,
                                  a.max_context_len)
    b = w.to("cuda")
    out_b = torch.empty_like(b.q)
    pkv.paged_attention_decode_mq(out_b, b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, b.scale,
                                  b.max_context_len, k_new=b.k_new, v_new=b.v_new)
    torch.cuda.synchronize()
    return (out_a, a.k_cache, a.v_cache), (out_b, b.k_cache, b.v_cache)


MQ_LENS = [4, 15, 16, 17, 18, 33, 511, 512, 513, 514, 1024, 1026, 2049, 4099]


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("D", [64, 128])
@pytest.mark.parametrize("G,q_len", [(1, 1), (1, 3), (1, 8), (1, 16), (2, 2), (2, 4), (4, 1), (4, 2), (4, 4),
                                     (8, 2)])
def test_multi_query_and_fused_write_match_oracle(dtype, D, G, q_len):
    # up to 8 rows (q_len * G): the transposed kernel; 9..16 rows: the 16-row kernel
    Hkv = 2
    lens = [max(n, q_len) for n in MQ_LENS]      # every sequence holds its new tokens
    w = make_custom(lens, Hkv * G, Hkv, D, dtype, seed=31 * G + q_len + D, q_len=q_len)
    ref, k_ref, v_ref = oracle_mq(w, q_len)
    (oa, ka, va), (ob, kb, vb) = _both_paths(w, q_len)
    for k_, v_ in ((ka, va), (kb, vb)):
        assert torch.equal(k_.cpu(), k_ref) and torch.equal(v_.cpu(), v_ref), "cache after the new tokens' write"
    assert_close(oa, ref, "write then decode")
    assert_close(ob, ref, "fused")
    assert torch.equal(oa, ob), "fused write must give the same bits as write-then-decode"
    assert pkv.pkv_device_status(0) == 0


def test_single_query_mq_equals_decode_bitwise():
    w = make_workload(4, num_seqs=12, max_ctx=3000).to("cuda")
    out1 = torch.empty_like(w.q)
    pkv.paged_attention_decode(out1, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale,
                               w.max_context_len)
    out2 = torch.empty(w.num_seqs, 1, w.num_q_heads, w.head_dim, dtype=w.dtype, device="cuda")
    pkv.paged_attention_decode_mq(out2, w.q[:, None].contiguous(), w.k_cache, w.v_cache, w.block_tables,
                                  w.context_lens, w.scale, w.max_context_len)
    torch.cuda.synchronize()
    assert torch.equal(out1, out2[:, 0])


def test_fused_single_token_step_equals_write_then_decode():
    host = make_workload(4, num_seqs=24, max_ctx=5000)
    slots = pkv.pkv_slot_mapping(host.block_tables, host.context_lens - 1)
    a, b = host.to("cuda"), host.to("cuda")
    pkv.paged_kv_write(a.k_new, a.v_new, a.k_cache, a.v_cache, slots.cuda())
    out_a = torch.empty_like(a.q)
    pkv.paged_attention_decode(out_a, a.q, a.k_cache, a.v_cache, a.block_tables, a.context_lens, a.scale,
                               a.max_context_len)
    out_b = torch.empty(b.num_seqs, 1, b.num_q_heads, b.head_dim, dtype=b.dtype, device="cuda")
    pkv.paged_attention_decode_mq(out_b, b.q[:, None].contiguous(), b.k_cache, b.v_cache, b.block_tables,
                                  b.context_lens, b.scale, b.max_context_len, k_new=b.k_new[:, None].contiguous(),
                                  v_new=b.v_new[:, None].contiguous())
    torch.cuda.synchronize()
    assert torch.equal(out_a, out_b[:, 0])
    assert torch.equal(a.k_cache, b.k_cache) and torch.equal(a.v_cache, b.v_cache)


def test_context_shorter_than_q_len_is_flagged():
    w = make_custom([5, 2, 40], 4, 2, 64, torch.bfloat16, seed=3, q_len=3).to("cuda")
    out = torch.full_like(w.q, 5.0)
    pkv.paged_attention_decode_mq(out, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale,
                                  w.max_context_len)
    assert pkv.pkv_device_status(0) & pkv._lib.C["PKV_DEV_BAD_CONTEXT"]
    assert torch.equal(out[1].cpu(), torch.zeros_like(out[1].cpu()))


def test_unsupported_combinations_are_rejected():
    w = make_custom([20, 30], 8, 2, 64, torch.float32, seed=4, q_len=2).to("cuda")
    out = torch.empty_like(w.q)
    with pytest.raises(pkv.PagedKVError):
        pkv.paged_attention_decode_mq(out, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale,
                                      w.max_context_len)
    w = make_custom([20, 30], 16, 2, 64, torch.float16, seed=4, q_len=3).to("cuda")   # 3 x 8 rows > 16
    out = torch.empty_like(w.q)
    with pytest.raises(pkv.PagedKVError):
        pkv.paged_attention_decode_mq(out, w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale,
                                      w.max_context_len)


@pytest.mark.parametrize("block_size", [8, 32])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("G,q_len", [(1, 1), (4, 2), (4, 3), (2, 8), (1, 16)])
def test_multi_query_fused_block_sizes_8_and_32(block_size, dtype, G, q_len):
    lens = [max(n, q_len) for n in (5, 8, 9, 17, 33, 510, 514, 1031)]
    w = make_custom(lens, 2 * G, 2, 128, dtype, seed=7 * block_size + G + q_len, q_len=q_len,
                    block_size=block_size)
    ref, k_ref, v_ref = oracle_mq(w, q_len)
    (oa, ka, va), (ob, kb, vb) = _both_paths(w, q_len)
    for k_, v_ in ((ka, va), (kb, vb)):
        assert torch.equal(k_.cpu(), k_ref) and torch.equal(v_.cpu(), v_ref)
    assert_close(oa, ref, "write then decode")
    assert torch.equal(oa, ob)


def test_fused_decode_step_replays_from_a_cuda_graph():
    """The step (fused slot write + decode) captured once and replayed gives
    the same bits as eager calls, also after the inputs change in place."""
    host = make_workload(4, num_seqs=16, max_ctx=3000)
    w = host.to("cuda")
    S, max_ctx = w.num_seqs, host.max_context_len      # a host int: nothing is read back under capture
    q4, kn4, vn4 = w.q[:, None].contiguous(), w.k_new[:, None].contiguous(), w.v_new[:, None].contiguous()
    ws = torch.empty(max(1, pkv.paged_attention_mq_workspace_bytes(S, 1, w.num_q_heads, w.head_dim, max_ctx)),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty_like(q4)

    def step():
        pkv.paged_attention_decode_mq(out, q4, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale,
                                      max_ctx, k_new=kn4, v_new=vn4, workspace=ws)

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
    q4.copy_(torch.randn(q4.shape, generator=torch.Generator(device="cuda").manual_seed(3), device="cuda").to(q4.dtype))
    graph.replay()
    torch.cuda.synchronize()
    replayed = out.clone()
    step()
    torch.cuda.synchronize()
    assert torch.equal(replayed, out) and not torch.equal(replayed, eager)


@pytest.mark.parametrize("G,q_len", [(1, 16), (4, 1)])
def test_back_to_back_fused_calls_when_every_row_fits_one_partition(G, q_len):
    """max_context_len far above every length: the split-K reduce is launched
    but no row needs it, so all of its CTAs but the first leave before they
    wait for the partition kernel.  A second fused call issued right behind
    rewrites the very slots the first one reads (same lengths, other new
    tokens); each call must still attend to its own new tokens only."""
    import dataclasses
    Hkv, D, dtype, max_ctx = 4, 128, torch.float16, 4096
    lens = [max(n, q_len) for n in (1, 17, 200, 333, 480, 500)]   # one partition of 512 or 1024 tokens each
    w1 = make_custom(lens, Hkv * G, Hkv, D, dtype, seed=77 + G, q_len=q_len,
                     max_blocks_per_seq=max_ctx // B)
    g = torch.Generator().manual_seed(5 + G)
    w2 = dataclasses.replace(w1, q=torch.randn(w1.q.shape, generator=g).to(dtype),
                             k_new=torch.randn(w1.k_new.shape, generator=g).to(dtype),
                             v_new=torch.randn(w1.v_new.shape, generator=g).to(dtype))
    ref1, k_ref1, v_ref1 = oracle_mq(w1, q_len)
    ref2, k_ref2, v_ref2 = oracle_mq(dataclasses.replace(w2, k_cache=k_ref1, v_cache=v_ref1), q_len)
    assert pkv.paged_attention_mq_workspace_bytes(w1.num_seqs, q_len, w1.num_q_heads, D, max_ctx) > 0
    a = w1.to("cuda")
    q2, kn2, vn2 = w2.q.cuda(), w2.k_new.cuda(), w2.v_new.cuda()
    out1, out2 = torch.empty_like(a.q), torch.empty_like(a.q)
    for out, q, kn, vn in ((out1, a.q, a.k_new, a.v_new), (out2, q2, kn2, vn2)):
        pkv.paged_attention_decode_mq(out, q, a.k_cache, a.v_cache, a.block_tables, a.context_lens, a.scale,
                                      max_ctx, k_new=kn, v_new=vn)
    torch.cuda.synchronize()
    assert torch.equal(a.k_cache.cpu(), k_ref2) and torch.equal(a.v_cache.cpu(), v_ref2)
    assert_close(out1, ref1, "first call")
    assert_close(out2, ref2, "second call")
    assert pkv.pkv_device_status(0) == 0
