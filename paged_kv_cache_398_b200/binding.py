"""Python binding of the C ABI in include/paged_kv.h (argument marshalling only).

Each function has the name of the C entry point it calls.  It reads sizes
from tensor shapes, checks that the tensors are contiguous, on the GPU and
of one element type, and passes raw pointers and torch's current CUDA stream.
Every step of the computation runs in the library's CUDA kernels.  Failures
raise ``PagedKVError``, carrying the library's status code.
"""

from __future__ import annotations

import ctypes
from typing import NamedTuple, Optional

import torch

from ._lib import C, PagedKVError, check, lib

_DTYPE = {torch.float32: C["PKV_F32"], torch.float16: C["PKV_F16"], torch.bfloat16: C["PKV_BF16"]}
BLOCK_SIZE = 16
PARTITION_TOKENS = C["PKV_PARTITION_TOKENS"]
PARTITION_TOKENS_LONG = C["PKV_PARTITION_TOKENS_LONG"]
PARTITION_TOKENS_WIDE = C["PKV_PARTITION_TOKENS_WIDE"]


def _dtype_code(t: torch.Tensor) -> int:
    try:
        return _DTYPE[t.dtype]
    except KeyError:
        raise PagedKVError("dtype", C["PKV_ERR_UNSUPPORTED"]) from None


def _cuda(name: str, t: torch.Tensor, dtype=None, ndim=None) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions, got {tuple(t.shape)}")
    return t


# torch's current stream as a raw handle, without building a Stream object
# (about 3 us a call otherwise); the public call where torch lacks it.
_raw_current_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(device: torch.device, stream) -> int:
    if stream is not None:
        return stream.cuda_stream
    if _raw_current_stream is not None:
        return _raw_current_stream(device.index if device.index is not None else torch.cuda.current_device())
    return torch.cuda.current_stream(device).cuda_stream


def _cache_shape(k_cache, v_cache):
    _cuda("k_cache", k_cache, ndim=4)
    _cuda("v_cache", v_cache, k_cache.dtype, 4)
    if k_cache.shape != v_cache.shape or k_cache.device != v_cache.device:
        raise ValueError("k_cache and v_cache must have one shape and device")
    NB, Hkv, B, D = k_cache.shape
    return NB, Hkv, B, D


def paged_kv_write(k_new, v_new, k_cache, v_cache, slot_mapping, stream=None) -> None:
    """Store k_new/v_new [T, Hkv, D] in the slots slot_mapping [T] (int64)."""
    NB, Hkv, B, D = _cache_shape(k_cache, v_cache)
    _cuda("k_new", k_new, k_cache.dtype, 3)
    _cuda("v_new", v_new, k_cache.dtype, 3)
    _cuda("slot_mapping", slot_mapping, torch.int64, 1)
    T = slot_mapping.shape[0]
    if tuple(k_new.shape) != (T, Hkv, D) or tuple(v_new.shape) != (T, Hkv, D):
        raise ValueError("k_new/v_new must be [T, Hkv, D] matching slot_mapping and the cache")
    rc = lib().paged_kv_write(k_new.data_ptr(), v_new.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                              slot_mapping.data_ptr(), T, Hkv, D, B, NB, _dtype_code(k_cache),
                              _stream(k_cache.device, stream))
    check("paged_kv_write", rc)


def paged_attention_workspace_bytes(num_seqs: int, num_q_heads: int, head_dim: int,
                                    max_context_len: int) -> int:
    return int(lib().paged_attention_workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len))


def paged_attention_partition_tokens(num_seqs: int, num_kv_heads: int, max_context_len: int,
                                     dtype: torch.dtype) -> int:
    """Split-K partition size (tokens) a decode launch of this shape uses on
    the current CUDA device: PARTITION_TOKENS or PARTITION_TOKENS_WIDE."""
    if dtype not in _DTYPE:
        raise PagedKVError("dtype", C["PKV_ERR_UNSUPPORTED"])
    rc = int(lib().paged_attention_partition_tokens(num_seqs, num_kv_heads, max_context_len, _DTYPE[dtype]))
    check("paged_attention_partition_tokens", min(rc, 0))
    return rc


def paged_attention_mq_partition_tokens(num_seqs: int, q_len: int, num_q_heads: int, num_kv_heads: int,
                                        max_context_len: int, dtype: torch.dtype) -> int:
    """Split-K partition size (tokens) of a paged_attention_decode_mq launch
    of q_len new tokens per sequence: PARTITION_TOKENS, PARTITION_TOKENS_LONG or
    PARTITION_TOKENS_WIDE."""
    if dtype not in _DTYPE:
        raise PagedKVError("dtype", C["PKV_ERR_UNSUPPORTED"])
    rc = int(lib().paged_attention_mq_partition_tokens(num_seqs, q_len, num_q_heads, num_kv_heads,
                                                       max_context_len, _DTYPE[dtype]))
    check("paged_attention_mq_partition_tokens", min(rc, 0))
    return rc


def paged_attention_decode(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                           max_context_len: int, workspace: Optional[torch.Tensor] = None,
                           stream=None) -> torch.Tensor:
    """Decode attention through the block tables; writes and returns `out` [S, Hq, D].

    context_lens counts the step's new token (write it first with
    paged_kv_write).  max_context_len (a host int >= every length) sizes the
    grid.  workspace: a CUDA tensor of at least
    paged_attention_workspace_bytes(...) bytes, or None to let torch
    allocate one for this call.
    """
    NB, Hkv, B, D = _cache_shape(k_cache, v_cache)
    _cuda("q", q, k_cache.dtype, 3)
    _cuda("out", out, k_cache.dtype, 3)
    _cuda("block_tables", block_tables, torch.int32, 2)
    _cuda("context_lens", context_lens, torch.int32, 1)
    S, Hq, Dq = q.shape
    if Dq != D or tuple(out.shape) != (S, Hq, D):
        raise ValueError("q/out must be [S, Hq, D] with the cache's head_dim")
    if block_tables.shape[0] != S or context_lens.shape[0] != S:
        raise ValueError("block_tables/context_lens must have one row per sequence")
    if workspace is None:   # a given workspace's size is checked by the library
        need = paged_attention_workspace_bytes(S, Hq, D, max_context_len)
        if need:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr, ws_bytes = 0, 0
    if workspace is not None:
        _cuda("workspace", workspace)
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    rc = lib().paged_attention_decode(out.data_ptr(), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                      block_tables.data_ptr(), block_tables.shape[1],
                                      context_lens.data_ptr(), S, int(max_context_len), Hq, Hkv, D, B, NB,
                                      float(scale), _dtype_code(k_cache), ws_ptr or None, ws_bytes,
                                      _stream(q.device, stream))
    check("paged_attention_decode", rc)
    return out


def paged_attention_mq_workspace_bytes(num_seqs: int, q_len: int, num_q_heads: int, head_dim: int,
                                       max_context_len: int) -> int:
    return int(lib().paged_attention_mq_workspace_bytes(num_seqs, q_len, num_q_heads, head_dim, max_context_len))


def paged_attention_decode_mq(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                              max_context_len: int, k_new=None, v_new=None,
                              workspace: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Decode for q [S, q_len, Hq, D] new tokens per sequence, causal among them.

    With k_new / v_new [S, q_len, Hkv, D] the new tokens are written to their
    slots (through the block tables) in the same launch.  Returns `out`
    [S, q_len, Hq, D].
    """
    NB, Hkv, B, D = _cache_shape(k_cache, v_cache)
    _cuda("q", q, k_cache.dtype, 4)
    _cuda("out", out, k_cache.dtype, 4)
    _cuda("block_tables", block_tables, torch.int32, 2)
    _cuda("context_lens", context_lens, torch.int32, 1)
    S, QL, Hq, Dq = q.shape
    if Dq != D or tuple(out.shape) != (S, QL, Hq, D):
        raise ValueError("q/out must be [S, q_len, Hq, D] with the cache's head_dim")
    if block_tables.shape[0] != S or context_lens.shape[0] != S:
        raise ValueError("block_tables/context_lens must have one row per sequence")
    if (k_new is None) != (v_new is None):
        raise ValueError("give both k_new and v_new, or neither")
    kn = vn = None
    if k_new is not None:
        _cuda("k_new", k_new, k_cache.dtype, 4)
        _cuda("v_new", v_new, k_cache.dtype, 4)
        if tuple(k_new.shape) != (S, QL, Hkv, D) or tuple(v_new.shape) != (S, QL, Hkv, D):
            raise ValueError("k_new/v_new must be [S, q_len, Hkv, D]")
        kn, vn = k_new.data_ptr(), v_new.data_ptr()
    if workspace is None:   # a given workspace's size is checked by the library
        need = paged_attention_mq_workspace_bytes(S, QL, Hq, D, max_context_len)
        if need:
            workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    ws_ptr, ws_bytes = 0, 0
    if workspace is not None:
        _cuda("workspace", workspace)
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    rc = lib().paged_attention_decode_mq(out.data_ptr(), q.data_ptr(), kn, vn, k_cache.data_ptr(),
                                         v_cache.data_ptr(), block_tables.data_ptr(), block_tables.shape[1],
                                         context_lens.data_ptr(), S, QL, int(max_context_len), Hq, Hkv, D, B, NB,
                                         float(scale), _dtype_code(k_cache), ws_ptr or None, ws_bytes,
                                         _stream(q.device, stream))
    check("paged_attention_decode_mq", rc)
    return out


SHARED_MAX_ROWS = C["PKV_SHARED_MAX_ROWS"]


class SharedPrefixPlan(NamedTuple):
    """pkv_shared_prefix_plan's result: groups int32 [num_groups, 2] (first
    sequence, members), shared_lens int32 [S], the decode launch's work list
    int32 [num_work, 2] for partitions of part_tokens, and two bounds."""
    groups: torch.Tensor
    shared_lens: torch.Tensor
    work: torch.Tensor
    part_tokens: int
    max_shared_len: int
    max_own_len: int

    def to(self, device) -> "SharedPrefixPlan":
        return self._replace(groups=self.groups.to(device), shared_lens=self.shared_lens.to(device),
                             work=self.work.to(device))


def pkv_shared_prefix_plan(block_tables, context_lens, block_size: int, max_group: int, part_tokens: int,
                           min_shared_tokens: int = 128) -> SharedPrefixPlan:
    """Groups of consecutive sequences whose tables start with the same
    blocks, and the decode launch's work list, from HOST int32 block_tables
    [S, MB] and context_lens [S].  max_group: members per group, at most
    (SHARED_MAX_ROWS // (Hq // Hkv) for decode); part_tokens: the launch's
    partition size (paged_attention_partition_tokens)."""
    bt = torch.as_tensor(block_tables, dtype=torch.int32).contiguous()
    cl = torch.as_tensor(context_lens, dtype=torch.int32).contiguous()
    if bt.device.type != "cpu" or cl.device.type != "cpu" or bt.dim() != 2 or cl.dim() != 1 or \
            bt.shape[0] != cl.shape[0]:
        raise ValueError("block_tables [S, MB] and context_lens [S] must be host int32 tensors")
    S = cl.shape[0]
    groups = torch.empty(max(S, 1), 2, dtype=torch.int32)
    shared = torch.empty(max(S, 1), dtype=torch.int32)
    # at most one item per partition of each sequence, plus one where a split adds one
    cap = max(1, S * (-(-max(bt.shape[1], 1) * int(block_size) // max(int(part_tokens), 1)) + 1))
    work = torch.empty(cap, 2, dtype=torch.int32)
    ng, nw = ctypes.c_int32(0), ctypes.c_int32(0)
    mx_shared, mx_own = ctypes.c_int32(0), ctypes.c_int32(0)
    check("pkv_shared_prefix_plan", lib().pkv_shared_prefix_plan(
        bt.data_ptr() if S else None, max(bt.shape[1], 1), cl.data_ptr() if S else None, S, int(block_size),
        int(max_group), int(min_shared_tokens), int(part_tokens), groups.data_ptr(), ctypes.byref(ng),
        shared.data_ptr(), work.data_ptr(), cap, ctypes.byref(nw), ctypes.byref(mx_shared), ctypes.byref(mx_own)))
    return SharedPrefixPlan(groups[:ng.value].clone(), shared[:S].clone(), work[:nw.value].clone(),
                            int(part_tokens), int(mx_shared.value), int(mx_own.value))


def pkv_shared_prefix_order(block_tables, context_lens, block_size: int) -> torch.Tensor:
    """A batch order (int64 permutation) that puts sequences whose HOST int32
    block_tables [S, MB] start with the same blocks next to each other, so
    that pkv_shared_prefix_plan on the reordered batch can group them."""
    bt = torch.as_tensor(block_tables, dtype=torch.int32).contiguous()
    cl = torch.as_tensor(context_lens, dtype=torch.int32).contiguous()
    if bt.device.type != "cpu" or cl.device.type != "cpu" or bt.dim() != 2 or cl.dim() != 1 or \
            bt.shape[0] != cl.shape[0]:
        raise ValueError("block_tables [S, MB] and context_lens [S] must be host int32 tensors")
    S = cl.shape[0]
    order = torch.empty(S, dtype=torch.int64)
    check("pkv_shared_prefix_order", lib().pkv_shared_prefix_order(
        bt.data_ptr() if S else None, max(bt.shape[1], 1), cl.data_ptr() if S else None, S, int(block_size),
        order.data_ptr() if S else None))
    return order


def paged_attention_shared_workspace_bytes(num_seqs: int, num_q_heads: int, head_dim: int,
                                           max_context_len: int) -> int:
    return int(lib().paged_attention_shared_workspace_bytes(num_seqs, num_q_heads, head_dim, max_context_len))


def paged_attention_decode_shared(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                                  max_context_len: int, groups, shared_lens, work, work_part_tokens: int,
                                  k_new=None, v_new=None, workspace: Optional[torch.Tensor] = None,
                                  stream=None) -> torch.Tensor:
    """Decode q [S, Hq, D] reading each group's shared blocks once.  groups
    [num_groups, 2], shared_lens [S] and work [num_work, 2] (int32, on the
    GPU) and work_part_tokens come from pkv_shared_prefix_plan.  With k_new /
    v_new [S, Hkv, D] the new tokens are written to their slots in the same
    call.  Returns out [S, Hq, D]."""
    NB, Hkv, B, D = _cache_shape(k_cache, v_cache)
    _cuda("q", q, k_cache.dtype, 3)
    _cuda("out", out, k_cache.dtype, 3)
    _cuda("block_tables", block_tables, torch.int32, 2)
    _cuda("context_lens", context_lens, torch.int32, 1)
    _cuda("shared_lens", shared_lens, torch.int32, 1)
    _cuda("work", work, torch.int32, 2)
    S, Hq, Dq = q.shape
    if Dq != D or tuple(out.shape) != (S, Hq, D):
        raise ValueError("q/out must be [S, Hq, D] with the cache's head_dim")
    if block_tables.shape[0] != S or context_lens.shape[0] != S or shared_lens.shape[0] != S:
        raise ValueError("block_tables/context_lens/shared_lens must have one row per sequence")
    if work.shape[1] != 2:
        raise ValueError("work must be [num_work, 2]")
    ng = 0 if groups is None else int(groups.shape[0])
    if ng:
        _cuda("groups", groups, torch.int32, 2)
        if groups.shape[1] != 2:
            raise ValueError("groups must be [num_groups, 2]")
    if (k_new is None) != (v_new is None):
        raise ValueError("give both k_new and v_new, or neither")
    kn = vn = None
    if k_new is not None:
        _cuda("k_new", k_new, k_cache.dtype, 3)
        _cuda("v_new", v_new, k_cache.dtype, 3)
        if tuple(k_new.shape) != (S, Hkv, D) or tuple(v_new.shape) != (S, Hkv, D):
            raise ValueError("k_new/v_new must be [S, Hkv, D]")
        kn, vn = k_new.data_ptr(), v_new.data_ptr()
    if workspace is None:
        need = paged_attention_shared_workspace_bytes(S, Hq, D, max_context_len)
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _cuda("workspace", workspace)
    rc = lib().paged_attention_decode_shared(
        out.data_ptr(), q.data_ptr(), kn, vn, k_cache.data_ptr(), v_cache.data_ptr(), block_tables.data_ptr(),
        block_tables.shape[1], context_lens.data_ptr(), S, int(max_context_len),
        groups.data_ptr() if ng else None, ng, shared_lens.data_ptr(), work.data_ptr() if work.numel() else None,
        int(work.shape[0]), int(work_part_tokens), Hq, Hkv, D, B, NB, float(scale), _dtype_code(k_cache),
        workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream(q.device, stream))
    check("paged_attention_decode_shared", rc)
    return out


def paged_attention_decode_noalloc(out, q, k_cache, v_cache, block_tables, context_lens, scale: float,
                                   max_context_len: int, stream=None) -> torch.Tensor:
    """paged_attention_decode with the library's fixed scratch array instead
    of a workspace: for callers that cannot allocate device memory when they
    decode.  Batches needing more than PKV_NOALLOC_SCRATCH_BYTES of scratch
    raise PagedKVError (PKV_ERR_SCRATCH_LIMIT).  Calls that overlap on the
    GPU share that array and race."""
    NB, Hkv, B, D = _cache_shape(k_cache, v_cache)
    _cuda("q", q, k_cache.dtype, 3)
    _cuda("out", out, k_cache.dtype, 3)
    _cuda("block_tables", block_tables, torch.int32, 2)
    _cuda("context_lens", context_lens, torch.int32, 1)
    S, Hq, Dq = q.shape
    if Dq != D or tuple(out.shape) != (S, Hq, D):
        raise ValueError("q/out must be [S, Hq, D] with the cache's head_dim")
    if block_tables.shape[0] != S or context_lens.shape[0] != S:
        raise ValueError("block_tables/context_lens must have one row per sequence")
    rc = lib().paged_attention_decode_noalloc(out.data_ptr(), q.data_ptr(), k_cache.data_ptr(),
                                              v_cache.data_ptr(), block_tables.data_ptr(), block_tables.shape[1],
                                              context_lens.data_ptr(), S, int(max_context_len), Hq, Hkv, D, B, NB,
                                              float(scale), _dtype_code(k_cache), _stream(q.device, stream))
    check("paged_attention_decode_noalloc", rc)
    return out


def block_copy(k_cache, v_cache, pairs, stream=None) -> None:
    """Copy-on-write copies; pairs: host int64 [N, 2] (src, dst) tensor or list."""
    NB, Hkv, B, D = _cache_shape(k_cache, v_cache)
    pr = torch.as_tensor(pairs, dtype=torch.int64, device="cpu").reshape(-1, 2).contiguous()
    rc = lib().block_copy(k_cache.data_ptr(), v_cache.data_ptr(), pr.data_ptr(), pr.shape[0], Hkv, D, B,
                          NB, _dtype_code(k_cache), _stream(k_cache.device, stream))
    check("block_copy", rc)


def _swap(name, k_cache, v_cache, block_ids, host_k, host_v, stream):
    NB, Hkv, B, D = _cache_shape(k_cache, v_cache)
    ids = torch.as_tensor(block_ids, dtype=torch.int64, device="cpu").reshape(-1).contiguous()
    n = ids.numel()
    for nm, t in (("host_k", host_k), ("host_v", host_v)):
        if not isinstance(t, torch.Tensor) or t.device.type != "cpu" or not t.is_contiguous():
            raise ValueError(f"{nm} must be a contiguous host tensor")
        if t.dtype != k_cache.dtype or tuple(t.shape) != (n, Hkv, B, D):
            raise ValueError(f"{nm} must be {k_cache.dtype} [n, Hkv, B, D] with n = len(block_ids)")
    rc = getattr(lib(), name)(k_cache.data_ptr(), v_cache.data_ptr(), ids.data_ptr(), n, host_k.data_ptr(),
                              host_v.data_ptr(), Hkv, D, B, NB, _dtype_code(k_cache), _stream(k_cache.device, stream))
    check(name, rc)


def swap_blocks_out(k_cache, v_cache, block_ids, host_k, host_v, stream=None) -> None:
    """Copy device blocks block_ids[i] into slot i of the pinned host buffers
    host_k / host_v [n, Hkv, B, D] (asynchronous on the stream)."""
    _swap("swap_blocks_out", k_cache, v_cache, block_ids, host_k, host_v, stream)


def swap_blocks_in(k_cache, v_cache, block_ids, host_k, host_v, stream=None) -> None:
    """Copy slot i of the pinned host buffers into device block block_ids[i]."""
    _swap("swap_blocks_in", k_cache, v_cache, block_ids, host_k, host_v, stream)


def pkv_slot_mapping(block_tables: torch.Tensor, positions: torch.Tensor, block_size: int = BLOCK_SIZE):
    """Host helper: slot of positions[s] in sequence s given host tables [S, MB]."""
    bt = torch.as_tensor(block_tables, dtype=torch.int32).contiguous()
    pos = torch.as_tensor(positions, dtype=torch.int32).contiguous()
    if bt.device.type != "cpu" or pos.device.type != "cpu":
        raise ValueError("pkv_slot_mapping takes host tensors")
    out = torch.empty(pos.shape[0], dtype=torch.int64)
    rc = lib().pkv_slot_mapping(bt.data_ptr(), bt.shape[1], pos.data_ptr(), pos.shape[0], block_size,
                                out.data_ptr())
    check("pkv_slot_mapping", rc)
    return out


def pkv_device_status(device: int = 0, clear: bool = True) -> int:
    """Sticky device-side flags (PKV_DEV_*) of `device`; synchronises it."""
    flags = ctypes.c_int32(0)
    rc = lib().pkv_device_status(device, ctypes.byref(flags), 1 if clear else 0)
    check("pkv_device_status", rc)
    return int(flags.value)
