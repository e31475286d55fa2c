"""Python handle on the native host block allocator (pkv_alloc_* / pkv_seq_*).

Marshalling only: the bookkeeping (free list, reference counts, block
tables, copy-on-write decisions) runs in the C++ allocator of the library.
"""

from __future__ import annotations

import ctypes

import torch

from ._lib import C, PagedKVError, check, lib


TABLE_KEEP_TAIL = C["PKV_TABLE_KEEP_TAIL"]  # batch_tables pad: leave entries past each table's end alone


class AllocStats(ctypes.Structure):
    _fields_ = [("num_blocks", ctypes.c_int32), ("free_blocks", ctypes.c_int32),
                ("used_blocks", ctypes.c_int32), ("shared_blocks", ctypes.c_int32),
                ("num_seqs", ctypes.c_int64), ("num_tokens", ctypes.c_int64),
                ("fragmentation_tokens", ctypes.c_int64)]


class PrefixStats(ctypes.Structure):
    _fields_ = [("cached_blocks", ctypes.c_int32), ("evictable_blocks", ctypes.c_int32),
                ("prompts", ctypes.c_int64), ("prompts_with_hits", ctypes.c_int64),
                ("hit_tokens", ctypes.c_int64), ("evictions", ctypes.c_int64)]


class OutOfBlocks(PagedKVError):
    pass


def _check(fn, rc):
    if rc == C["PKV_ERR_OUT_OF_BLOCKS"]:
        raise OutOfBlocks(fn, rc)
    check(fn, rc)


class BlockAllocator:
    """Pool of `num_blocks` blocks of `block_size` tokens.

    initial_order: optional permutation of the block ids giving the order in
    which blocks are first handed out (the default is 0, 1, 2, ...).
    """

    def __init__(self, num_blocks: int, block_size: int = 16, initial_order=None):
        self._L = lib()
        h = ctypes.c_void_p()
        order = None
        if initial_order is not None:
            order = torch.as_tensor(initial_order, dtype=torch.int32).contiguous()
            if order.numel() != num_blocks:
                raise ValueError("initial_order must list every block once")
        _check("pkv_alloc_create", self._L.pkv_alloc_create(num_blocks, block_size,
                                                            order.data_ptr() if order is not None else None,
                                                            ctypes.byref(h)))
        self._h = h
        self.num_blocks = num_blocks
        self.block_size = block_size

    def close(self):
        if self._h:
            self._L.pkv_alloc_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def add(self, seq: int) -> None:
        _check("pkv_seq_add", self._L.pkv_seq_add(self._h, seq))

    def append_tokens(self, seq: int, n: int):
        """Slots for n new tokens; returns (slots list, (src, dst) or None)."""
        slots = torch.empty(max(n, 1), dtype=torch.int64)
        pair = torch.empty(2, dtype=torch.int64)
        cow = ctypes.c_int32(0)
        _check("pkv_seq_append_tokens", self._L.pkv_seq_append_tokens(
            self._h, seq, n, slots.data_ptr(), pair.data_ptr(), ctypes.byref(cow)))
        return slots[:n].tolist(), (tuple(pair.tolist()) if cow.value else None)

    @staticmethod
    def _ids(seqs) -> torch.Tensor:
        if isinstance(seqs, torch.Tensor) and seqs.dtype == torch.int64 and seqs.device.type == "cpu":
            return seqs.contiguous()
        return torch.as_tensor(list(seqs), dtype=torch.int64).contiguous()

    def append_one_batch(self, seqs, slots_out=None, pairs_out=None):
        """One token for each sequence: (slots int64 tensor, copy pairs int64 [N, 2]).
        seqs: ids (a CPU int64 tensor avoids a conversion); slots_out /
        pairs_out: optional CPU int64 buffers of at least [n] / [n, 2], reused
        by a serving loop."""
        ids = self._ids(seqs)
        n = ids.numel()
        slots = slots_out if slots_out is not None else torch.empty(max(n, 1), dtype=torch.int64)
        pairs = pairs_out if pairs_out is not None else torch.empty(max(n, 1), 2, dtype=torch.int64)
        if slots.dtype != torch.int64 or slots.numel() < n or pairs.dtype != torch.int64 or pairs.numel() < 2 * n:
            raise ValueError("slots_out / pairs_out: CPU int64 buffers of at least [n] and [n, 2]")
        ncow = ctypes.c_int32(0)
        _check("pkv_batch_append_one", self._L.pkv_batch_append_one(
            self._h, ids.data_ptr(), n, slots.data_ptr(), pairs.data_ptr(), ctypes.byref(ncow)))
        return slots[:n], pairs[:ncow.value]

    def free(self, seq: int) -> None:
        _check("pkv_seq_free", self._L.pkv_seq_free(self._h, seq))

    def fork(self, parent: int, child: int) -> None:
        _check("pkv_seq_fork", self._L.pkv_seq_fork(self._h, parent, child))

    def share_prefix(self, seq: int, blocks, num_tokens: int) -> None:
        b = torch.as_tensor(list(blocks), dtype=torch.int32).contiguous()
        _check("pkv_seq_share_prefix", self._L.pkv_seq_share_prefix(
            self._h, seq, b.data_ptr() if b.numel() else None, b.numel(), num_tokens))

    def block_table(self, seq: int) -> list:
        n = ctypes.c_int32(0)
        self._L.pkv_seq_block_table(self._h, seq, None, 0, ctypes.byref(n))
        out = torch.empty(max(n.value, 1), dtype=torch.int32)
        _check("pkv_seq_block_table", self._L.pkv_seq_block_table(
            self._h, seq, out.data_ptr(), out.numel(), ctypes.byref(n)))
        return out[:n.value].tolist()

    def num_tokens(self, seq: int) -> int:
        v = ctypes.c_int32(0)
        _check("pkv_seq_num_tokens", self._L.pkv_seq_num_tokens(self._h, seq, ctypes.byref(v)))
        return int(v.value)

    def batch_tables(self, seqs, max_blocks_per_seq: int, pad: int = -1, tables_out=None, lens_out=None):
        """(block_tables int32 [S, MB], context_lens int32 [S]) as host tensors.
        pad=TABLE_KEEP_TAIL leaves entries past each table's end as they are;
        with tables_out / lens_out (CPU int32, [S, MB] / [S]) a serving loop
        refills the same buffers every step."""
        ids = self._ids(seqs)
        S = ids.numel()
        tables = tables_out if tables_out is not None else torch.empty(max(S, 1), max_blocks_per_seq, dtype=torch.int32)
        lens = lens_out if lens_out is not None else torch.empty(max(S, 1), dtype=torch.int32)
        if (tables.dtype != torch.int32 or not tables.is_contiguous() or tables.dim() != 2
                or tables.shape[0] < S or tables.shape[1] != max_blocks_per_seq
                or lens.dtype != torch.int32 or lens.numel() < S):
            raise ValueError("tables_out / lens_out: CPU int32 buffers [>= S, max_blocks_per_seq] and [>= S]")
        _check("pkv_batch_tables", self._L.pkv_batch_tables(
            self._h, ids.data_ptr(), S, tables.data_ptr(), max_blocks_per_seq, pad, lens.data_ptr()))
        return tables[:S], lens[:S]

    def append_prompt(self, seq: int, tokens):
        """Prompt of a new (empty) sequence, reusing cached prefix blocks.
        Returns (slots int64 tensor with -1 for cached tokens, n_cached)."""
        t = torch.as_tensor(tokens, dtype=torch.int32).reshape(-1).contiguous()
        n = t.numel()
        slots = torch.empty(max(n, 1), dtype=torch.int64)
        cached = ctypes.c_int32(0)
        _check("pkv_seq_append_prompt", self._L.pkv_seq_append_prompt(
            self._h, seq, t.data_ptr() if n else None, n, slots.data_ptr(), ctypes.byref(cached)))
        return slots[:n], int(cached.value)

    def prefix_stats(self) -> dict:
        st = PrefixStats()
        _check("pkv_prefix_cache_stats", self._L.pkv_prefix_cache_stats(self._h, ctypes.byref(st)))
        return {name: int(getattr(st, name)) for name, _ in PrefixStats._fields_}

    def swap_out(self, seq: int) -> list:
        """Release a sequence's blocks for preemption; returns them (logical
        order) so their contents can be copied out with swap_blocks_out."""
        n = ctypes.c_int32(0)
        cap = len(self.block_table(seq))
        out = torch.empty(max(cap, 1), dtype=torch.int32)
        _check("pkv_seq_swap_out", self._L.pkv_seq_swap_out(self._h, seq, out.data_ptr(), out.numel(),
                                                            ctypes.byref(n)))
        return out[:n.value].tolist()

    def swap_in(self, seq: int) -> list:
        """Fresh blocks for a swapped-out sequence (logical order), the
        destinations for swap_blocks_in."""
        n = ctypes.c_int32(0)
        out = torch.empty(max(self.num_blocks, 1), dtype=torch.int32)
        _check("pkv_seq_swap_in", self._L.pkv_seq_swap_in(self._h, seq, out.data_ptr(), out.numel(),
                                                          ctypes.byref(n)))
        return out[:n.value].tolist()

    def is_swapped(self, seq: int) -> bool:
        v = ctypes.c_int32(0)
        _check("pkv_seq_is_swapped", self._L.pkv_seq_is_swapped(self._h, seq, ctypes.byref(v)))
        return bool(v.value)

    def num_free(self) -> int:
        return int(self._L.pkv_num_free(self._h))

    def free_list(self) -> list:
        n = ctypes.c_int32(0)
        out = torch.empty(max(self.num_blocks, 1), dtype=torch.int32)
        _check("pkv_free_list", self._L.pkv_free_list(self._h, out.data_ptr(), out.numel(), ctypes.byref(n)))
        return out[:n.value].tolist()

    def refcount(self, block: int) -> int:
        return int(self._L.pkv_refcount(self._h, block))

    def stats(self) -> dict:
        st = AllocStats()
        _check("pkv_alloc_get_stats", self._L.pkv_alloc_get_stats(self._h, ctypes.byref(st)))
        return {name: int(getattr(st, name)) for name, _ in AllocStats._fields_}
