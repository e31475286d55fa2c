"""The C-ABI library loads, exports every declared symbol, and rejects bad
arguments on the host before touching a device (CPU only)."""

import ctypes
import glob
import os
import re

import pytest
import torch

from tests.conftest import ROOT


@pytest.fixture(scope="module")
def L():
    from paged_kv_cache_398_b200.build import build_library
    build_library()
    from paged_kv_cache_398_b200._lib import lib
    return lib()


def _declared_functions():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M):
            names.add(m.group(1))
    names.discard("defined")
    return sorted(names)


def test_header_declares_the_boundary():
    names = _declared_functions()
    for n in ("paged_kv_write", "paged_attention_decode", "block_copy",
              "paged_attention_workspace_bytes", "pkv_alloc_create", "pkv_seq_append_tokens"):
        assert n in names


def test_every_declared_symbol_is_exported(L):
    missing = [n for n in _declared_functions() if not hasattr(L, n)]
    assert not missing, f"not exported: {missing}"


def test_status_strings(L):
    from paged_kv_cache_398_b200._lib import C
    for name, code in C.items():
        if name.startswith("PKV_ERR_") or name == "PKV_OK":
            assert L.pkv_status_string(code) not in (None, b"unknown status")


def test_host_side_rejections(L):
    from paged_kv_cache_398_b200._lib import C
    INV, UNS = C["PKV_ERR_INVALID_ARG"], C["PKV_ERR_UNSUPPORTED"]
    # bad dtype, bad shapes, null pointers: rejected before any CUDA call
    assert L.paged_kv_write(None, None, None, None, None, 4, 8, 128, 16, 10, 7, None) == UNS
    assert L.paged_kv_write(None, None, None, None, None, 4, 8, 128, 16, 10, 2, None) == INV
    assert L.paged_kv_write(None, None, None, None, None, 0, 8, 128, 16, 10, 2, None) == C["PKV_OK"]
    assert L.paged_attention_decode(None, None, None, None, None, 4, None, 2, 100, 32, 8, 96, 16, 10,
                                    ctypes.c_float(0.1), 2, None, 0, None) == UNS
    assert L.paged_attention_decode(None, None, None, None, None, 4, None, 2, 100, 32, 8, 128, 24, 10,
                                    ctypes.c_float(0.1), 2, None, 0, None) == UNS
    assert L.paged_attention_decode(None, None, None, None, None, 4, None, 2, 100, 24, 8, 128, 16, 10,
                                    ctypes.c_float(0.1), 2, None, 0, None) == UNS
    assert L.paged_attention_decode(None, None, None, None, None, 4, None, 2, 100, 30, 8, 128, 16, 10,
                                    ctypes.c_float(0.1), 2, None, 0, None) == INV
    assert L.paged_attention_decode(None, None, None, None, None, 4, None, 2, 100, 32, 8, 128, 16, 10,
                                    ctypes.c_float(0.1), 2, None, 0, None) == INV
    # a workspace that is too small is rejected
    buf = (ctypes.c_uint8 * 4096)()
    p = ctypes.addressof(buf) + (-ctypes.addressof(buf)) % 256
    need = L.paged_attention_workspace_bytes(2, 32, 128, 1000)
    assert need == 2 * 32 * 2 * 130 * 4
    assert L.paged_attention_decode(p, p, p, p, p, 4, p, 2, 1000, 32, 8, 128, 16, 10,
                                    ctypes.c_float(0.1), 2, p, 100, None) == INV
    assert L.paged_attention_workspace_bytes(2, 32, 128, 512) == 0
    # the partition-size query: answers that need no device, and rejections
    assert L.paged_attention_partition_tokens(256, 8, 100, C["PKV_BF16"]) == C["PKV_PARTITION_TOKENS"]
    assert L.paged_attention_partition_tokens(4096, 8, 8192, C["PKV_F32"]) == C["PKV_PARTITION_TOKENS"]
    assert L.paged_attention_partition_tokens(-1, 8, 100, C["PKV_BF16"]) == INV
    assert L.paged_attention_partition_tokens(4, 0, 100, C["PKV_BF16"]) == INV
    assert L.paged_attention_partition_tokens(4, 8, 100, 7) == UNS
    # multi-query: more than 8 query rows per kv head (the 16-row form) always take the long partitions
    MQ = L.paged_attention_mq_partition_tokens
    # more than 8 rows (the 16-row form): the long or wide partitions, by the device's SM count
    # (no device: PKV_ERR_CUDA)
    sixteen = (C["PKV_PARTITION_TOKENS_LONG"], C["PKV_PARTITION_TOKENS_WIDE"]) if torch.cuda.is_available() \
        else (C["PKV_ERR_CUDA"],)
    assert MQ(64, 16, 40, 40, 600, C["PKV_F16"]) in sixteen                               # 16 rows
    assert MQ(8, 3, 16, 4, 100, C["PKV_BF16"]) in sixteen                                 # 3 x 4 = 12 rows
    assert MQ(8, 2, 16, 4, 100, C["PKV_BF16"]) == C["PKV_PARTITION_TOKENS"]             # 8 rows: the short rule
    assert MQ(8, 1, 32, 8, 100, C["PKV_BF16"]) == C["PKV_PARTITION_TOKENS"]
    assert MQ(8, 16, 16, 16, 9000, C["PKV_F32"]) == C["PKV_PARTITION_TOKENS"]           # fp32 keeps the short ones
    assert MQ(8, 16, 40, 7, 100, C["PKV_F16"]) == INV                                  # Hq not a multiple of Hkv
    assert MQ(8, 0, 40, 40, 100, C["PKV_F16"]) == INV
    assert MQ(8, 16, 40, 40, 0, C["PKV_F16"]) == INV
    assert MQ(8, 16, 40, 40, 100, 7) == UNS
    # order-dependent copy lists are rejected on the host
    dummy = ctypes.c_void_p(p)
    for pairs in ([[1, 1]], [[1, 2], [3, 2]], [[1, 2], [2, 3]], [[0, 8]], [[-1, 2]]):
        t = torch.tensor(pairs, dtype=torch.int64)
        assert L.block_copy(dummy, dummy, t.data_ptr(), t.shape[0], 2, 128, 16, 8, 2, None) == INV


def test_slot_mapping_matches_the_allocator_model():
    from oracle.allocator_model import AllocatorModel
    import paged_kv_cache_398_b200 as pkv
    from tests.conftest import load_golden
    gold = load_golden("worked_block_tables.json")
    order = [0, 2, 6, 4, 7, 1, 3, 9, 5, 8, 10, 11]
    m = AllocatorModel(12, 16, initial_order=order)
    for sid, n in ((0, 40), (1, 48), (2, 20)):
        m.add(sid)
        m.append_tokens(sid, n)
    tables = torch.full((3, 3), -1, dtype=torch.int32)
    for sid, req in enumerate("ABC"):
        row = gold["block_tables"][req]
        tables[sid, :len(row)] = torch.tensor(row)
    for pos in range(0, 48):
        positions = torch.tensor([pos, pos, min(pos, 31)], dtype=torch.int32)
        got = pkv.pkv_slot_mapping(tables, positions).tolist()
        for sid in range(3):
            p = int(positions[sid])
            bt = m.block_table(sid)
            if p // 16 < len(bt):
                assert got[sid] == bt[p // 16] * 16 + p % 16
    assert pkv.pkv_slot_mapping(tables, torch.tensor([-1, 0, 0], dtype=torch.int32)).tolist()[0] == -1
    with pytest.raises(pkv.PagedKVError):
        pkv.pkv_slot_mapping(tables, torch.tensor([48, 0, 0], dtype=torch.int32))
    with pytest.raises(pkv.PagedKVError):
        pkv.pkv_slot_mapping(tables, torch.tensor([0, 0, 40], dtype=torch.int32))


def test_shared_decode_host_side_rejections(L):
    """paged_attention_decode_shared's argument checks run before any CUDA call."""
    from paged_kv_cache_398_b200._lib import C
    INV, UNS = C["PKV_ERR_INVALID_ARG"], C["PKV_ERR_UNSUPPORTED"]
    buf = (ctypes.c_uint8 * 8192)()
    p = ctypes.addressof(buf) + (-ctypes.addressof(buf)) % 256
    f = ctypes.c_float(0.1)

    def call(S=2, max_ctx=1000, groups=p, ng=1, work=p, nw=3, D=128, B=16, Hq=32, Hkv=8, dtype=2, kn=p, vn=p,
             ws_bytes=1 << 20):
        return L.paged_attention_decode_shared(p, p, kn, vn, p, p, p, 64, p, S, max_ctx, groups, ng, p, work, nw,
                                               512, Hq, Hkv, D, B, 100, f, dtype, p, ws_bytes, None)

    need = L.paged_attention_shared_workspace_bytes(2, 32, 128, 1000)
    assert need == 2 * 32 * (2 + 1) * 130 * 4      # one record slot per row beyond ceil(1000 / 512)
    assert call(dtype=C["PKV_F32"]) == UNS          # the tensor-core kernel takes 16-bit inputs
    assert call(D=96) == UNS and call(B=24) == UNS and call(Hq=24) == UNS
    assert call(Hq=30) == INV                       # not a multiple of the kv heads
    assert call(kn=None) == INV                     # k_new without v_new
    assert call(nw=0) == INV                        # an empty work list
    assert call(ng=3) == INV                        # more groups than sequences
    assert call(groups=None) == INV                 # groups missing
    assert call(work=p + 4) == INV                  # work items are 8-byte pairs
    assert call(ws_bytes=need - 1) == INV           # workspace too small
    assert call(S=0) == C["PKV_OK"]                 # an empty batch is a no-op
    # the plan, on the host: a query of the work list's size
    t = torch.tensor([[0, 1, 2, 3], [0, 1, 2, 4]], dtype=torch.int32)
    lens = torch.tensor([60, 61], dtype=torch.int32)
    g, sh = torch.empty(2, 2, dtype=torch.int32), torch.empty(2, dtype=torch.int32)
    ng, nw, a, b = (ctypes.c_int32(0) for _ in range(4))
    assert L.pkv_shared_prefix_plan(t.data_ptr(), 4, lens.data_ptr(), 2, 16, 4, 16, 512, g.data_ptr(),
                                    ctypes.byref(ng), sh.data_ptr(), None, 0, ctypes.byref(nw), ctypes.byref(a),
                                    ctypes.byref(b)) == C["PKV_OK"]
    assert (ng.value, nw.value, a.value, b.value) == (1, 3, 48, 13)


def test_copy_and_swap_list_checks_cost_the_list_not_the_pool(L):
    """block_copy and swap_blocks_in check their id lists by sorting them, so
    a check on a pool of 2^20 blocks costs microseconds, not a pool-sized
    scan.  The lists here are rejected (a dst that is also a src; an id
    named twice), which happens on the host before any CUDA call."""
    import time
    from paged_kv_cache_398_b200._lib import C
    INV = C["PKV_ERR_INVALID_ARG"]
    NB = 1 << 20
    fake = ctypes.c_void_p(1 << 20)                     # 16-byte aligned; never dereferenced
    pairs = torch.tensor([[i, NB - 1 - i] for i in range(7)] + [[100, 3]], dtype=torch.int64)  # 3 is a src
    ids = torch.tensor(list(range(0, NB, NB // 15)) + [0], dtype=torch.int64)                   # 0 twice
    args_c = (fake, fake, ctypes.c_void_p(pairs.data_ptr()), pairs.shape[0], 8, 128, 16, NB, 2, None)
    args_s = (fake, fake, ctypes.c_void_p(ids.data_ptr()), ids.shape[0], fake, fake, 8, 128, 16, NB, 2, None)
    assert L.block_copy(*args_c) == INV and L.swap_blocks_in(*args_s) == INV
    for fn, args in ((L.block_copy, args_c), (L.swap_blocks_in, args_s)):
        t0 = time.perf_counter()
        for _ in range(200):
            assert fn(*args) == INV
        per_call = (time.perf_counter() - t0) / 200
        assert per_call < 50e-6, f"{fn.__name__}: {per_call * 1e6:.1f} us a check"
