"""Paged KV cache decode path for NVIDIA B200 (sm_100a).

The KV cache lives in fixed-size, non-contiguous 16-token physical blocks
reached through per-sequence block tables ("PagedAttention: How vLLM Serves
AI Like an Operating System").  The package is a thin Python binding over the
C ABI of ``include/paged_kv.h``:

* ``paged_kv_write``          -- slot write of the new tokens' K/V
* ``paged_attention_decode``  -- decode attention through the block tables
* ``paged_attention_decode_shared`` -- decode reading a group's shared blocks once
  (plan from ``pkv_shared_prefix_plan``)
* ``block_copy``              -- copy-on-write block copy
* ``swap_blocks_out`` / ``swap_blocks_in`` -- preemption: blocks to / from host memory
* ``BlockAllocator``          -- host block allocator (free list, refcounts, CoW)

The native library ``libpaged_kv.so`` is built in-tree by
``paged_kv_cache_398_b200.build``.  There is no CPU fallback.
"""

from ._lib import LibraryMissing, PagedKVError
from .allocator import TABLE_KEEP_TAIL, BlockAllocator, OutOfBlocks
from .binding import (BLOCK_SIZE, PARTITION_TOKENS, PARTITION_TOKENS_LONG, PARTITION_TOKENS_WIDE, SHARED_MAX_ROWS,
                      SharedPrefixPlan, block_copy, paged_attention_decode, paged_attention_decode_mq, paged_attention_decode_noalloc,
                      paged_attention_decode_shared, paged_attention_mq_workspace_bytes,
                      paged_attention_mq_partition_tokens, paged_attention_partition_tokens,
                      paged_attention_shared_workspace_bytes,
                      paged_attention_workspace_bytes, paged_kv_write, pkv_device_status, pkv_shared_prefix_order,
                      pkv_shared_prefix_plan,
                      pkv_slot_mapping, swap_blocks_in, swap_blocks_out)

__all__ = [
    "BLOCK_SIZE", "PARTITION_TOKENS", "PARTITION_TOKENS_LONG", "PARTITION_TOKENS_WIDE", "TABLE_KEEP_TAIL",
    "BlockAllocator", "LibraryMissing", "OutOfBlocks",
    "PagedKVError", "block_copy", "paged_attention_decode", "paged_attention_decode_mq",
    "paged_attention_decode_noalloc", "paged_attention_decode_shared", "paged_attention_mq_workspace_bytes",
    "paged_attention_mq_partition_tokens", "paged_attention_partition_tokens",
    "paged_attention_shared_workspace_bytes", "paged_attention_workspace_bytes",
    "SHARED_MAX_ROWS", "SharedPrefixPlan", "pkv_shared_prefix_order", "pkv_shared_prefix_plan",
    "paged_kv_write", "pkv_device_status", "pkv_slot_mapping", "swap_blocks_in", "swap_blocks_out",
]
