"""Plain, slow, fp64 CPU oracle for the paged KV cache decode path.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference leg of ``bench.py`` may import anything from this
package.  The product library (``paged_kv_cache_398_b200``) never imports,
links or calls it, and the two share no code: the oracle's arithmetic lives in
``oracle.c`` (decode attention, slot write, block copy) and in
``allocator_model.py`` (block allocator), both written from the pages.

Pinned by ``tests/test_oracle_pins.py`` against the pages' worked examples,
closed forms, a library routine on the contiguous special case, brute-force
invariants and exact special cases.  See the module docstrings of each
function for the page section it follows.

The wrappers take torch CPU tensors purely as containers for the bytes and
return numpy fp64 arrays.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

# The oracle's own element-type codes (oracle.c): 0 fp32, 1 fp16, 2 bf16.
_DTYPE_CODE = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}


def build_oracle(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so with gcc (IEEE semantics, no fast-math)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-fno-fast-math", "-ffp-contract=off",
             "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            path = build_oracle()
            L = ctypes.CDLL(path)
            P, I32, I64, D = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
            L.oracle_widen.argtypes = [P, I64, ctypes.c_int]
            L.oracle_widen.restype = D
            L.oracle_gather.argtypes = [P, P, P, P, P, I32, I32, I32, I32, I32, I32, ctypes.c_int]
            L.oracle_gather.restype = ctypes.c_int
            L.oracle_paged_decode_seq.argtypes = [P, P, P, P, P, I32, I32, I32, I32, I32, I32, I32,
                                                  D, ctypes.c_int]
            L.oracle_paged_decode_seq.restype = ctypes.c_int
            L.oracle_paged_decode.argtypes = [P, P, P, P, P, I32, P, I32, I32, I32, I32, I32, I32,
                                              D, ctypes.c_int]
            L.oracle_paged_decode.restype = ctypes.c_int
            L.oracle_paged_decode_mq.argtypes = [P, P, P, P, P, I32, P, I32, I32, I32, I32, I32, I32, I32,
                                                 D, ctypes.c_int]
            L.oracle_paged_decode_mq.restype = ctypes.c_int
            L.oracle_kv_write.argtypes = [P, P, P, P, P, I32, I32, I32, I32, I32, ctypes.c_int]
            L.oracle_kv_write.restype = ctypes.c_int
            L.oracle_block_copy.argtypes = [P, P, P, I32, I32, I32, I32, I32, ctypes.c_int]
            L.oracle_block_copy.restype = ctypes.c_int
            _lib = L
    return _lib


class OracleError(RuntimeError):
    pass


def _cpu(t: torch.Tensor, dtype=None) -> torch.Tensor:
    if t.device.type != "cpu":
        raise OracleError("the oracle takes CPU tensors only")
    if dtype is not None and t.dtype != dtype:
        raise OracleError(f"expected {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise OracleError("the oracle takes contiguous tensors only")
    return t


def _code(t: torch.Tensor) -> int:
    try:
        return _DTYPE_CODE[t.dtype]
    except KeyError:
        raise OracleError(f"unsupported dtype {t.dtype}") from None


def widen(t: torch.Tensor) -> np.ndarray:
    """Every element of a CPU tensor widened to fp64 by the oracle's own decoder."""
    t = _cpu(t).reshape(-1)
    L, code = lib(), _code(t)
    return np.array([L.oracle_widen(t.data_ptr(), i, code) for i in range(t.numel())],
                    dtype=np.float64)


def gather(k_cache, v_cache, block_table_row, ctx: int, kv_head: int):
    """One sequence's K and V for one kv head as contiguous fp64 [ctx, D]."""
    _cpu(k_cache), _cpu(v_cache)
    bt = _cpu(block_table_row, torch.int32)
    NB, Hkv, B, D = k_cache.shape
    kc = np.empty((ctx, D), np.float64)
    vc = np.empty((ctx, D), np.float64)
    rc = lib().oracle_gather(kc.ctypes.data, vc.ctypes.data, k_cache.data_ptr(), v_cache.data_ptr(),
                             bt.data_ptr(), ctx, kv_head, Hkv, D, B, NB, _code(k_cache))
    if rc != 0:
        raise OracleError("gather: block id outside the pool")
    return kc, vc


def paged_decode_seq(s: int, q, k_cache, v_cache, block_tables, context_lens, scale: float):
    """fp64 decode-attention output of sequence s, all query heads: [Hq, D]."""
    _cpu(q), _cpu(k_cache), _cpu(v_cache)
    bt = _cpu(block_tables, torch.int32)
    cl = _cpu(context_lens, torch.int32)
    S, Hq, D = q.shape
    NB, Hkv, B, D2 = k_cache.shape
    MB = bt.shape[1]
    out = np.empty((Hq, D), np.float64)
    q_seq = q.data_ptr() + s * Hq * D * q.element_size()
    rc = lib().oracle_paged_decode_seq(out.ctypes.data, q_seq, k_cache.data_ptr(), v_cache.data_ptr(),
                                       bt.data_ptr() + s * MB * 4, MB, int(cl[s]), Hq, Hkv, D, B, NB,
                                       float(scale), _code(q))
    if rc != 0:
        raise OracleError(f"paged_decode_seq: invalid input for sequence {s}")
    return out


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, scale: float) -> np.ndarray:
    """fp64 decode attention for every sequence and query head: [S, Hq, D].

    q [S, Hq, D]; k_cache, v_cache [NB, Hkv, B, D]; block_tables [S, MB] int32;
    context_lens [S] int32; all CPU, same element dtype for q and the caches.
    """
    _cpu(q), _cpu(k_cache), _cpu(v_cache)
    if not (q.dtype == k_cache.dtype == v_cache.dtype):
        raise OracleError("q and the caches must share one dtype")
    bt = _cpu(block_tables, torch.int32)
    cl = _cpu(context_lens, torch.int32)
    S, Hq, D = q.shape
    NB, Hkv, B, D2 = k_cache.shape
    if D2 != D:
        raise OracleError("head_dim mismatch")
    out = np.empty((S, Hq, D), np.float64)
    rc = lib().oracle_paged_decode(out.ctypes.data, q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                   bt.data_ptr(), bt.shape[1], cl.data_ptr(), S, Hq, Hkv, D, B, NB,
                                   float(scale), _code(q))
    if rc != 0:
        raise OracleError("paged_decode: invalid input")
    return out


def paged_decode_mq(q, k_cache, v_cache, block_tables, context_lens, scale: float) -> np.ndarray:
    """fp64 multi-query decode: q [S, q_len, Hq, D] -> [S, q_len, Hq, D].

    New token j of sequence s is at position ctx_s - q_len + j and attends
    to positions 0 .. ctx_s - q_len + j (causal among the new tokens).
    """
    _cpu(q), _cpu(k_cache), _cpu(v_cache)
    if not (q.dtype == k_cache.dtype == v_cache.dtype):
        raise OracleError("q and the caches must share one dtype")
    bt = _cpu(block_tables, torch.int32)
    cl = _cpu(context_lens, torch.int32)
    S, QL, Hq, D = q.shape
    NB, Hkv, B, D2 = k_cache.shape
    if D2 != D:
        raise OracleError("head_dim mismatch")
    out = np.empty((S, QL, Hq, D), np.float64)
    rc = lib().oracle_paged_decode_mq(out.ctypes.data, q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                      bt.data_ptr(), bt.shape[1], cl.data_ptr(), S, QL, Hq, Hkv, D, B, NB,
                                      float(scale), _code(q))
    if rc != 0:
        raise OracleError("paged_decode_mq: invalid input")
    return out


def kv_write(k_cache, v_cache, k_new, v_new, slot_mapping) -> None:
    """In-place slot write of k_new/v_new [T, Hkv, D] through slot_mapping [T] int64."""
    _cpu(k_cache), _cpu(v_cache), _cpu(k_new), _cpu(v_new)
    sm = _cpu(slot_mapping, torch.int64)
    NB, Hkv, B, D = k_cache.shape
    rc = lib().oracle_kv_write(k_cache.data_ptr(), v_cache.data_ptr(), k_new.data_ptr(), v_new.data_ptr(),
                               sm.data_ptr(), sm.numel(), Hkv, D, B, NB, _code(k_cache))
    if rc != 0:
        raise OracleError("kv_write: slot beyond the pool")


def block_copy(k_cache, v_cache, pairs) -> None:
    """In-place copy-on-write block copy for pairs [N, 2] int64 (src, dst)."""
    _cpu(k_cache), _cpu(v_cache)
    pr = _cpu(pairs, torch.int64)
    NB, Hkv, B, D = k_cache.shape
    rc = lib().oracle_block_copy(k_cache.data_ptr(), v_cache.data_ptr(), pr.data_ptr(), pr.shape[0],
                                 Hkv, D, B, NB, _code(k_cache))
    if rc != 0:
        raise OracleError("block_copy: invalid pair list")
