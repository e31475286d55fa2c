"""paged_attention_decode_noalloc: decode without a caller-supplied workspace.

Some callers cannot allocate device memory at the moment they decode:
runtimes that hand out all device memory as one fixed arena at start-up, and
embedders that must never call the CUDA allocator (it can synchronise the
device and take a process-wide lock).  For them the library offers an entry
point that takes its split-K scratch from a fixed array in the library's own
device memory.

These tests call it through the C ABI (ctypes, raw pointers) and check its
output against the workspace-taking entry point, within the tolerance the
parity tests use, on two calls in a row (the array keeps the previous call's
contents, which must not leak into the next result).  The file is named to
be collected last.
"""

import ctypes

import numpy as np
import pytest
import torch

from paged_kv_cache_398_b200._lib import C, lib
from paged_kv_cache_398_b200.workloads import make_custom, make_workload

pytestmark = pytest.mark.gpu

ATOL, RTOL = 2e-3, 1e-2
_DT = {torch.float32: C["PKV_F32"], torch.float16: C["PKV_F16"], torch.bfloat16: C["PKV_BF16"]}


def _abi_decode(L, w, out, ws=None, noalloc=False):
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    args = [out.data_ptr(), w.q.data_ptr(), w.k_cache.data_ptr(), w.v_cache.data_ptr(),
            w.block_tables.data_ptr(), w.block_tables.shape[1], w.context_lens.data_ptr(), w.num_seqs,
            w.max_context_len, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.num_blocks,
            ctypes.c_float(w.scale), _DT[w.dtype]]
    if noalloc:
        return L.paged_attention_decode_noalloc(*args, stream)
    return L.paged_attention_decode(*args, ws.data_ptr() if ws is not None else None,
                                    0 if ws is None else ws.numel(), stream)


def _within_tolerance(got, ref):
    g = got.double().cpu().numpy()
    r = ref.double().cpu().numpy()
    assert np.isfinite(g).all()
    assert np.all(np.abs(g - r) <= ATOL + RTOL * np.abs(r))


@pytest.mark.parametrize("make", [
    lambda: make_workload(4, num_seqs=48, device="cuda"),           # long contexts: split-K scratch used
    lambda: make_custom([1, 17, 513, 2000, 8192], 16, 2, 64, torch.float16, device="cuda", seed=21),
    lambda: make_workload(1, device="cuda"),                         # one partition: no scratch needed
])
def test_noalloc_matches_workspace_entry_point_twice(make):
    L = lib()
    w = make().to("cuda")
    need = L.paged_attention_workspace_bytes(w.num_seqs, w.num_q_heads, w.head_dim, w.max_context_len)
    assert need <= C["PKV_NOALLOC_SCRATCH_BYTES"]
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    ref = torch.empty_like(w.q)
    assert _abi_decode(L, w, ref, ws) == C["PKV_OK"]
    for call in range(2):
        out = torch.full_like(w.q, float("nan"))
        assert _abi_decode(L, w, out, noalloc=True) == C["PKV_OK"], f"call {call}"
        torch.cuda.synchronize()
        _within_tolerance(out, ref)
        # same kernels, same order of arithmetic: the outputs agree exactly too
        assert torch.equal(out, ref)


def test_noalloc_consecutive_different_batches():
    """A second, smaller batch right after a larger one must not see stale scratch."""
    L = lib()
    big = make_workload(4, num_seqs=32, device="cuda").to("cuda")
    small = make_custom([600, 1100, 40], 8, 2, 128, torch.bfloat16, device="cuda", seed=5).to("cuda")
    for w in (big, small, big):
        need = L.paged_attention_workspace_bytes(w.num_seqs, w.num_q_heads, w.head_dim, w.max_context_len)
        ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
        ref = torch.empty_like(w.q)
        out = torch.empty_like(w.q)
        assert _abi_decode(L, w, ref, ws) == C["PKV_OK"]
        assert _abi_decode(L, w, out, noalloc=True) == C["PKV_OK"]
        torch.cuda.synchronize()
        _within_tolerance(out, ref)


def test_noalloc_rejects_batches_beyond_the_limit():
    L = lib()
    # 1024 sequences x 64 heads x 8192 tokens at head_dim 128 need far more than the array
    S, Hq, D, ctx = 1024, 64, 128, 8192
    need = L.paged_attention_workspace_bytes(S, Hq, D, ctx)
    assert need > C["PKV_NOALLOC_SCRATCH_BYTES"]
    dummy = torch.zeros(16, dtype=torch.uint8, device="cuda")
    p = dummy.data_ptr()
    rc = L.paged_attention_decode_noalloc(p, p, p, p, p, 512, p, S, ctx, Hq, 8, D, 16, 10,
                                          ctypes.c_float(0.1), C["PKV_BF16"], None)
    assert rc == C["PKV_ERR_SCRATCH_LIMIT"]
    assert b"scratch" in L.pkv_status_string(rc)


def test_noalloc_call_allocates_no_device_memory():
    """After a first call of the same shape (which resolves the array's
    address and sets the kernel's attributes), a call leaves the device's
    free memory and torch's allocated bytes unchanged."""
    L = lib()
    w = make_workload(4, num_seqs=24, device="cuda").to("cuda")
    need = L.paged_attention_workspace_bytes(w.num_seqs, w.num_q_heads, w.head_dim, w.max_context_len)
    assert need > 0                                     # the call does use the scratch array
    out = torch.empty_like(w.q)
    assert _abi_decode(L, w, out, noalloc=True) == C["PKV_OK"]
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    torch0 = torch.cuda.memory_allocated()
    for _ in range(3):
        assert _abi_decode(L, w, out, noalloc=True) == C["PKV_OK"]
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0
    assert torch.cuda.memory_allocated() == torch0


def test_noalloc_invalid_arguments_get_the_workspace_entry_points_code():
    """A call that is invalid for any workspace returns the same code from
    both entry points, even when its shape would also exceed the array."""
    L = lib()
    dummy = torch.zeros(16, dtype=torch.uint8, device="cuda")
    p = dummy.data_ptr()
    S, Hq, ctx = 1024, 64, 8192                         # far beyond the array
    for D, Hkv, expect in ((96, 8, "PKV_ERR_UNSUPPORTED"),       # unsupported head_dim
                           (128, 7, "PKV_ERR_INVALID_ARG")):     # Hq not a multiple of Hkv
        common = [p, p, p, p, p, 512, p, S, ctx, Hq, Hkv, D, 16, 10, ctypes.c_float(0.1), C["PKV_BF16"]]
        assert L.paged_attention_decode_noalloc(*common, None) == C[expect]
        assert L.paged_attention_decode(*common, None, 0, None) == C[expect]
