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
