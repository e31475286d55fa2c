"""ctypes loader for the in-tree CUDA library (libpaged_kv.so).

The library must have been built (``python -m paged_kv_cache_398_b200.build``
or ``__graft_entry__.build()``).  There is no fallback: if it is missing,
every call raises ``LibraryMissing``.
"""

from __future__ import annotations

import ctypes
import os
import re
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libpaged_kv.so")
HEADER = os.path.join(os.path.dirname(HERE), "include", "paged_kv.h")

_lock = threading.Lock()
_lib = None


class LibraryMissing(RuntimeError):
    pass


def _constants() -> dict:
    """#define PKV_* integer constants, read from the public header."""
    out = {}
    with open(HEADER) as f:
        for line in f:
            # an integer, or (a - b) as in the INT32_MIN spelling (-2147483647 - 1)
            m = re.match(r"#define\s+(PKV_\w+)\s+\(?(-?\d+)(?:\s*-\s*(\d+))?\)?", line)
            if m:
                out[m.group(1)] = int(m.group(2)) - int(m.group(3) or 0)
    return out


C = _constants()

P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_SIGS = {
    "paged_kv_write": ([P, P, P, P, P, I32, I32, I32, I32, I32, I32, P], ctypes.c_int),
    "paged_attention_workspace_bytes": ([I32, I32, I32, I32], SZ),
    "paged_attention_partition_tokens": ([I32, I32, I32, I32], I32),
    "paged_attention_mq_partition_tokens": ([I32, I32, I32, I32, I32, I32], I32),
    "pkv_debug_decode_occupancy": ([I32, I32, I32, I32, I32, I32, P], I32),
    "pkv_debug_shared_occupancy": ([I32, I32, I32, I32, I32, P], I32),
    "paged_attention_decode": ([P, P, P, P, P, I32, P, I32, I32, I32, I32, I32, I32, I32,
                                ctypes.c_float, I32, P, SZ, P], ctypes.c_int),
    "paged_attention_mq_workspace_bytes": ([I32, I32, I32, I32, I32], SZ),
    "paged_attention_decode_mq": ([P, P, P, P, P, P, P, I32, P, I32, I32, I32, I32, I32, I32, I32, I32,
                                   ctypes.c_float, I32, P, SZ, P], ctypes.c_int),
    "paged_attention_shared_workspace_bytes": ([I32, I32, I32, I32], SZ),
    "paged_attention_decode_shared": ([P, P, P, P, P, P, P, I32, P, I32, I32, P, I32, P, P, I32, I32, I32, I32, I32,
                                       I32, I32, ctypes.c_float, I32, P, SZ, P], ctypes.c_int),
    "pkv_shared_prefix_plan": ([P, I32, P, I32, I32, I32, I32, I32, P, P, P, P, I32, P, P, P], ctypes.c_int),
    "pkv_shared_prefix_order": ([P, I32, P, I32, I32, P], ctypes.c_int),
    "paged_attention_decode_noalloc": ([P, P, P, P, P, I32, P, I32, I32, I32, I32, I32, I32, I32,
                                        ctypes.c_float, I32, P], ctypes.c_int),
    "block_copy": ([P, P, P, I32, I32, I32, I32, I32, I32, P], ctypes.c_int),
    "swap_blocks_out": ([P, P, P, I32, P, P, I32, I32, I32, I32, I32, P], ctypes.c_int),
    "swap_blocks_in": ([P, P, P, I32, P, P, I32, I32, I32, I32, I32, P], ctypes.c_int),
    "pkv_seq_append_prompt": ([P, I64, P, I32, P, P], ctypes.c_int),
    "pkv_prefix_cache_stats": ([P, P], ctypes.c_int),
    "pkv_seq_swap_out": ([P, I64, P, I32, P], ctypes.c_int),
    "pkv_seq_swap_in": ([P, I64, P, I32, P], ctypes.c_int),
    "pkv_seq_is_swapped": ([P, I64, P], ctypes.c_int),
    "pkv_slot_mapping": ([P, I32, P, I32, I32, P], ctypes.c_int),
    "pkv_device_status": ([I32, P, I32], ctypes.c_int),
    "pkv_last_cuda_error": ([], ctypes.c_int),
    "pkv_debug_wait_timeout": ([I64, P], ctypes.c_int),
    "pkv_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "pkv_alloc_create": ([I32, I32, P, P], ctypes.c_int),
    "pkv_alloc_destroy": ([P], None),
    "pkv_seq_add": ([P, I64], ctypes.c_int),
    "pkv_seq_append_tokens": ([P, I64, I32, P, P, P], ctypes.c_int),
    "pkv_batch_append_one": ([P, P, I32, P, P, P], ctypes.c_int),
    "pkv_seq_free": ([P, I64], ctypes.c_int),
    "pkv_seq_fork": ([P, I64, I64], ctypes.c_int),
    "pkv_seq_share_prefix": ([P, I64, P, I32, I32], ctypes.c_int),
    "pkv_seq_block_table": ([P, I64, P, I32, P], ctypes.c_int),
    "pkv_seq_num_tokens": ([P, I64, P], ctypes.c_int),
    "pkv_batch_tables": ([P, P, I32, P, I32, I32, P], ctypes.c_int),
    "pkv_num_free": ([P], I32),
    "pkv_free_list": ([P, P, I32, P], ctypes.c_int),
    "pkv_refcount": ([P, I32], I32),
    "pkv_alloc_get_stats": ([P, P], ctypes.c_int),
}


def lib():
    """The loaded library, with argument types set.  Raises LibraryMissing."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise LibraryMissing(
                    f"{LIB_PATH} is not built; run `python -m paged_kv_cache_398_b200.build` "
                    "(there is no CPU fallback)")
            L = ctypes.CDLL(LIB_PATH)
            for name, (args, res) in _SIGS.items():
                fn = getattr(L, name)
                fn.argtypes = args
                fn.restype = res
            _lib = L
    return _lib


class PagedKVError(RuntimeError):
    def __init__(self, fn: str, code: int):
        L = lib()
        msg = L.pkv_status_string(code).decode()
        extra = ""
        if code == C["PKV_ERR_CUDA"]:
            extra = f" (cudaError {L.pkv_last_cuda_error()})"
        super().__init__(f"{fn} failed: {msg}{extra} [status {code}]")
        self.code = code


def check(fn: str, code: int) -> None:
    if code != C["PKV_OK"]:
        raise PagedKVError(fn, code)
