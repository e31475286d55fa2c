"""List-based model of the host block allocator (test infrastructure).

TEST INFRASTRUCTURE: only ``tests/`` may use this module.  It restates, with
plain Python lists and dicts, the bookkeeping the pages describe, so the
product's C++ allocator can be compared with it operation by operation:

* Pool of fixed-size physical blocks and a free list of unused ones
  ("PagedAttention: How vLLM Serves AI Like an Operating System",
  "How It Works" and the "PagedAttention Memory Layout" example, whose free
  list is [5, 8, 10, 11]).
* On-demand allocation: a sequence gets one block when its first token
  arrives and another when token 17, 33, ... arrives, so n tokens hold
  ceil(n / 16) blocks and waste at most 15 slots ("The Magic: No
  Pre-allocation").
* Immediate release of a finished sequence's blocks ("vLLM Architecture and
  PagedAttention", page table visualisation: "its 6 pages are immediately
  freed").
* Sharing with reference counts: parallel samples share the prompt's blocks,
  a shared system prompt is shared by every request ("Copy-on-Write: Sharing
  KV Cache", "Parallel Sampling" and "Prefix Caching").
* Copy-on-write: a sequence about to write into a block that another
  sequence also holds first moves to a private copy ("Copy-on-Write").

Policy choices the pages leave open (the product follows the same ones):

* The free list is a stack.  ``initial_order`` is the order in which blocks
  are first handed out; a released block goes on top and is reused first.
* Releasing a sequence pushes its blocks from the last logical block to the
  first, so the next allocations get them back in logical order.  Only blocks
  whose reference count drops to zero are pushed.
* The writer whose target block is shared (reference count > 1) copies; the
  last holder (count == 1) writes in place.
* An operation that cannot get every block it needs fails with
  ``OutOfBlocks`` and changes nothing.
* Prefix cache ("Prefix Caching": a system prompt shared by many requests
  is stored once; "PagedAttention & Continuous Batching...", item 5).
  ``append_prompt`` walks a new request's full prompt blocks in order and
  reuses every leading block whose identity -- (block before it, that
  block's generation, its own token ids) -- is cached; from the first miss
  on it takes fresh blocks and caches each new full block.  A cached block
  whose count drops to zero stays findable; it is handed out again, least
  recently released first, only when no never-cached block is free.  The
  generation of a block grows each time it is handed out.
* Swapping a sequence out ("vLLM Architecture": the scheduler preempts
  low-priority requests by swapping their blocks to CPU memory) reports its
  blocks in logical order, then releases them like ``free``.  The sequence
  keeps its token count.  Swapping it back in takes fresh blocks in one
  all-or-nothing step.  A swapped-out sequence accepts no other operation
  except ``free``.
"""

from __future__ import annotations

from collections import OrderedDict


def slot_for_position(block_table, position: int, block_size: int) -> int:
    """Slot of token `position` of a sequence with this block table: its
    physical block times the block size plus its offset in the block."""
    return int(block_table[position // block_size]) * block_size + position % block_size


class OutOfBlocks(Exception):
    pass


class InvalidArgument(Exception):
    pass


class AllocatorModel:
    def __init__(self, num_blocks: int, block_size: int, initial_order=None):
        if num_blocks < 0 or block_size < 1:
            raise InvalidArgument("bad pool shape")
        order = list(range(num_blocks)) if initial_order is None else [int(b) for b in initial_order]
        if sorted(order) != list(range(num_blocks)):
            raise InvalidArgument("initial_order must be a permutation of the block ids")
        self.num_blocks = num_blocks
        self.block_size = block_size
        # The top of the stack is the end of the list.
        self._free = list(reversed(order))
        self._ref = [0] * num_blocks
        self._seqs: dict[int, dict] = {}
        self._cache: dict = {}          # (parent, parent_gen, tokens) -> block
        self._key_of: dict = {}         # block -> its key
        self._gen = [0] * num_blocks
        self._lru: OrderedDict = OrderedDict()   # cached, unused blocks; first = evicted first
        self._counts = {"prompts": 0, "prompts_with_hits": 0, "hit_tokens": 0, "evictions": 0}

    # --- queries -------------------------------------------------------
    def num_free(self) -> int:
        return len(self._free) + len(self._lru)

    def free_list(self) -> list[int]:
        """Free blocks in the order they will be handed out (never-cached
        blocks first, then cached unused blocks, least recently released first)."""
        return list(reversed(self._free)) + list(self._lru)

    def prefix_stats(self) -> dict:
        return {"cached_blocks": len(self._cache), "evictable_blocks": len(self._lru), **self._counts}

    def refcount(self, block: int) -> int:
        return self._ref[block]

    def block_table(self, seq: int) -> list[int]:
        return list(self._seq(seq)["blocks"])

    def num_tokens(self, seq: int) -> int:
        return self._seq(seq)["ntok"]

    def stats(self) -> dict:
        frag = sum(len(s["blocks"]) * self.block_size - s["ntok"] for s in self._seqs.values() if not s["swapped"])
        return {
            "num_blocks": self.num_blocks,
            "free_blocks": self.num_free(),
            "used_blocks": self.num_blocks - self.num_free(),
            "shared_blocks": sum(1 for r in self._ref if r > 1),
            "num_seqs": len(self._seqs),
            "num_tokens": sum(s["ntok"] for s in self._seqs.values()),
            "fragmentation_tokens": frag,
        }

    # --- helpers -------------------------------------------------------
    def _seq(self, seq: int) -> dict:
        if seq not in self._seqs:
            raise InvalidArgument(f"unknown sequence {seq}")
        return self._seqs[seq]

    def _pop(self) -> int:
        if self._free:
            b = self._free.pop()
        else:                                   # evict the least recently released cached block
            b, _ = self._lru.popitem(last=False)
            del self._cache[self._key_of.pop(b)]
            self._counts["evictions"] += 1
        self._gen[b] += 1
        self._ref[b] = 1
        return b

    def _decref(self, b: int) -> None:
        self._ref[b] -= 1
        if self._ref[b] == 0:
            if b in self._key_of:
                self._lru[b] = None             # keep its contents findable
            else:
                self._free.append(b)

    def _needs(self, seq: dict, n: int) -> int:
        """Blocks an append of n tokens takes from the free list."""
        if n == 0:
            return 0
        ntok, blocks = seq["ntok"], seq["blocks"]
        cow = 1 if (ntok % self.block_size != 0 and self._ref[blocks[-1]] > 1) else 0
        total_blocks = -(-(ntok + n) // self.block_size)
        return cow + total_blocks - len(blocks)

    def _append(self, seq: dict, n: int):
        B = self.block_size
        ntok, blocks = seq["ntok"], seq["blocks"]
        cow = None
        if n > 0 and ntok % B != 0 and self._ref[blocks[-1]] > 1:
            src = blocks[-1]
            dst = self._pop()
            self._decref(src)
            blocks[-1] = dst
            cow = (src, dst)
        slots = []
        for p in range(ntok, ntok + n):
            if p % B == 0:
                blocks.append(self._pop())
            slots.append(slot_for_position(blocks, p, B))
        seq["ntok"] = ntok + n
        return slots, cow

    # --- operations ----------------------------------------------------
    def add(self, seq: int) -> None:
        if seq in self._seqs:
            raise InvalidArgument(f"sequence {seq} exists")
        self._seqs[seq] = {"blocks": [], "ntok": 0, "swapped": False, "nswap": 0}

    def _live(self, seq: int) -> dict:
        s = self._seq(seq)
        if s["swapped"]:
            raise InvalidArgument(f"sequence {seq} is swapped out")
        return s

    def is_swapped(self, seq: int) -> bool:
        return self._seq(seq)["swapped"]

    def swap_out(self, seq: int) -> list[int]:
        """Blocks to copy to host memory (logical order); they are released."""
        s = self._live(seq)
        blocks = list(s["blocks"])
        for b in reversed(blocks):
            self._decref(b)
        s["blocks"] = []
        s["swapped"] = True
        s["nswap"] = len(blocks)
        return blocks

    def swap_in(self, seq: int) -> list[int]:
        """Fresh blocks for a swapped-out sequence, in logical order."""
        s = self._seq(seq)
        if not s["swapped"]:
            raise InvalidArgument(f"sequence {seq} is not swapped out")
        n = s["nswap"]
        if n > self.num_free():
            raise OutOfBlocks()
        s["blocks"] = [self._pop() for _ in range(n)]
        s["swapped"] = False
        s["nswap"] = 0
        return list(s["blocks"])

    def append_tokens(self, seq: int, n: int):
        """Reserve slots for n new tokens; returns (slots, cow_pair_or_None)."""
        if n < 0:
            raise InvalidArgument("negative token count")
        s = self._live(seq)
        if self._needs(s, n) > self.num_free():
            raise OutOfBlocks()
        return self._append(s, n)

    def append_prompt(self, seq: int, tokens):
        """Prompt of a new request: (slots with -1 for cached tokens, n_cached)."""
        tokens = [int(t) for t in tokens]
        s = self._live(seq)
        if s["blocks"] or s["ntok"]:
            raise InvalidArgument("append_prompt needs an empty sequence")
        B, n = self.block_size, len(tokens)
        nfull = n // B
        hit, parent, pgen = [], -1, 0
        for k in range(nfull):
            key = (parent, pgen, tuple(tokens[k * B:(k + 1) * B]))
            if key not in self._cache:
                break
            b = self._cache[key]
            hit.append(b)
            parent, pgen = b, self._gen[b]
        revived = sum(1 for b in hit if self._ref[b] == 0)
        if -(-n // B) - len(hit) > self.num_free() - revived:
            raise OutOfBlocks()
        if nfull:
            self._counts["prompts"] += 1
            self._counts["prompts_with_hits"] += 1 if hit else 0
        for b in hit:
            if self._ref[b] == 0:
                del self._lru[b]
            self._ref[b] += 1
        s["blocks"] = list(hit)
        cached = len(hit) * B
        self._counts["hit_tokens"] += cached
        s["ntok"] = cached
        slots, _ = self._append(s, n - cached)
        for k in range(len(hit), nfull):
            b = s["blocks"][k]
            par = s["blocks"][k - 1] if k else -1
            key = (par, self._gen[par] if par >= 0 else 0, tuple(tokens[k * B:(k + 1) * B]))
            self._cache[key] = b
            self._key_of[b] = key
        return [-1] * cached + slots, cached

    def append_one_batch(self, seqs):
        """One new token for each sequence, in order: (slots, cow_pairs)."""
        if len(set(seqs)) != len(seqs):
            raise InvalidArgument("a sequence is named twice")
        recs = [self._live(q) for q in seqs]
        if sum(self._needs(r, 1) for r in recs) > self.num_free():
            raise OutOfBlocks()
        slots, pairs = [], []
        for r in recs:
            sl, cow = self._append(r, 1)
            slots.extend(sl)
            if cow is not None:
                pairs.append(cow)
        return slots, pairs

    def free(self, seq: int) -> None:
        s = self._seq(seq)
        for b in reversed(s["blocks"]):
            self._decref(b)
        del self._seqs[seq]

    def fork(self, parent: int, child: int) -> None:
        p = self._live(parent)
        if child in self._seqs:
            raise InvalidArgument(f"sequence {child} exists")
        for b in p["blocks"]:
            self._ref[b] += 1
        self._seqs[child] = {"blocks": list(p["blocks"]), "ntok": p["ntok"], "swapped": False, "nswap": 0}

    def share_prefix(self, seq: int, blocks, num_tokens: int) -> None:
        """Point an empty sequence at existing (allocated) blocks holding num_tokens tokens."""
        s = self._live(seq)
        blocks = [int(b) for b in blocks]
        B = self.block_size
        if s["blocks"] or s["ntok"]:
            raise InvalidArgument("sequence is not empty")
        if -(-num_tokens // B) != len(blocks) or num_tokens < 0:
            raise InvalidArgument("token count does not fill the given blocks")
        for b in blocks:
            if not (0 <= b < self.num_blocks) or self._ref[b] < 1:
                raise InvalidArgument(f"block {b} is not allocated")
        for b in blocks:
            self._ref[b] += 1
        s["blocks"] = blocks
        s["ntok"] = num_tokens
