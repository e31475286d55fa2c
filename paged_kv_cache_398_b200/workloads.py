"""Seeded synthetic decode-step workloads, shared by the tests and the benchmark.

This module draws random numbers and lays out the structure of each workload
(which physical block each logical block of each sequence uses).  It holds
none of the attention, slot-write or block-copy arithmetic, and it imports
neither the CUDA library nor the oracle, so both sides can take their inputs
from it.

Workload shapes follow the serving scenarios of the pages:

* "tiny": 4 sequences of 5, 17, 33 and 64 tokens; fp32; head_dim 64; a pool of
  32 blocks handed out by a seeded permutation.
* "7b": 24 sequences, 32 heads, head_dim 128, fp16, lengths uniform in
  [1, 2048] (the 7B / 2048-token serving scenario of "vLLM Architecture and
  PagedAttention", "Throughput Comparison").
* "13b": 64 sequences, 40 heads, head_dim 128, fp16, chat-like lengths:
  prompt and output lengths lognormal with means 300 and 250 tokens (sigma
  1.0, our choice), summed and clipped to [1, 4096].  It stands in for the
  ShareGPT serving trace of "PagedAttention: How vLLM Serves AI Like an
  Operating System", "Throughput Impact: The Numbers".
* "8b_gqa_prefix": 256 sequences, 32 query heads over 8 kv heads, head_dim
  128, bf16; every sequence starts with the same 4 physical blocks (a 64-token
  system prompt, "Prefix Caching"), total lengths uniform in [65, 8192].
* "8b_gqa_sampling": 128 prompts x 4 samples, same heads, bf16; prompts
  uniform in [256, 4096] tokens whose full blocks the 4 samples share
  ("Parallel Sampling"); a prompt's partial last block stays with sample 0,
  and samples 1..3 get fresh blocks to be filled by a copy-on-write copy
  of it (the copy pairs are part of the step); each sample then has
  [1, 1024] output tokens of its own.

All values are N(0, 1), drawn in fp32 and rounded to the workload's dtype.
Seed = 398000 + workload number (1..5).  Draw order: lengths, then the pool
permutation, then Q, then the cache contents, then the new token's K/V, then
(only on request) random ids for the unused block-table entries.
The pool holds the blocks the batch needs plus 12.5% spare, handed out in a
seeded random order so that every sequence's blocks are scattered.
Unused block-table entries hold -1 (or random ids, on request).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch

BLOCK_SIZE = 16

WORKLOADS = {
    1: "tiny",
    2: "7b",
    3: "13b",
    4: "8b_gqa_prefix",
    5: "8b_gqa_sampling",
}


@dataclass
class DecodeWorkload:
    name: str
    dtype: torch.dtype
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    num_blocks: int
    context_lens: torch.Tensor        # [S] int32, CPU; includes the step's new token
    block_tables: torch.Tensor        # [S, MB] int32, CPU
    copy_pairs: torch.Tensor          # [N, 2] int64, CPU; (src, dst); may be empty
    q: torch.Tensor                   # [S, Hq, D]
    k_cache: torch.Tensor             # [NB, Hkv, B, D]
    v_cache: torch.Tensor             # [NB, Hkv, B, D]
    k_new: torch.Tensor               # [S, Hkv, D]
    v_new: torch.Tensor               # [S, Hkv, D]
    scale: float
    seed: int
    meta: dict = field(default_factory=dict)

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_tables.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max())

    def to(self, device) -> "DecodeWorkload":
        """Copy of the workload whose tensors live on `device`."""
        kw = {}
        for name in ("context_lens", "block_tables", "copy_pairs", "q", "k_cache", "v_cache",
                     "k_new", "v_new"):
            kw[name] = getattr(self, name).to(device)
        return DecodeWorkload(name=self.name, dtype=self.dtype, num_seqs=self.num_seqs,
                              num_q_heads=self.num_q_heads, num_kv_heads=self.num_kv_heads,
                              head_dim=self.head_dim, block_size=self.block_size,
                              num_blocks=self.num_blocks, scale=self.scale, seed=self.seed,
                              meta=dict(self.meta), **kw)


def _nblk(n: int, bs: int) -> int:
    return -(-n // bs)


def _randn(shape, dtype, gen, device, chunk_rows: int = 4096) -> torch.Tensor:
    """N(0,1) in fp32, rounded to dtype, generated in chunks along dim 0."""
    out = torch.empty(shape, dtype=dtype, device=device)
    for i in range(0, shape[0], chunk_rows):
        j = min(i + chunk_rows, shape[0])
        out[i:j] = torch.randn((j - i,) + tuple(shape[1:]), generator=gen, device=device,
                               dtype=torch.float32).to(dtype)
    return out


def _lognormal(n: int, mean: float, sigma: float, gen) -> torch.Tensor:
    mu = math.log(mean) - sigma * sigma / 2.0
    z = torch.randn(n, generator=gen, dtype=torch.float64)
    return torch.round(torch.exp(mu + sigma * z))


def make_workload(number: int, device="cpu", *, num_seqs=None, max_ctx=None, min_ctx=None,
                  num_prompts=None, max_prompt=None, max_output=None, seed=None,
                  pad_random: bool = False, block_size: int = BLOCK_SIZE) -> DecodeWorkload:
    """Build workload `number` (1..5).  Keyword overrides shrink it for tests.

    Lengths, the pool permutation and the block tables are always drawn on the
    CPU generator; Q, the cache contents and the new K/V are drawn on `device`
    (a CUDA generator when device is a GPU), so a full-size workload never
    passes through host memory.
    """
    name = WORKLOADS[number]
    seed = 398000 + number if seed is None else seed
    g = torch.Generator().manual_seed(seed)
    B = block_size
    copy_pairs = []
    meta = {"workload": name}

    if number == 1:
        S, Hq, Hkv, D, dtype = 4, 4, 4, 64, torch.float32
        ctx = [5, 17, 33, 64]
        NB = 32
        perm = torch.randperm(NB, generator=g).tolist()
        tables, k = [], 0
        for c in ctx:
            n = _nblk(c, B)
            tables.append(perm[k:k + n])
            k += n
    elif number in (2, 3, 4):
        if number == 2:
            S, Hq, Hkv, D, dtype = 24, 32, 32, 128, torch.float16
            lo, hi = 1, 2048
        elif number == 3:
            S, Hq, Hkv, D, dtype = 64, 40, 40, 128, torch.float16
            lo, hi = 1, 4096
        else:
            S, Hq, Hkv, D, dtype = 256, 32, 8, 128, torch.bfloat16
            lo, hi = 65, 8192
        S = num_seqs or S
        hi = max_ctx or hi
        lo = min_ctx or lo
        if number == 3:
            p = _lognormal(S, 300.0, 1.0, g)
            o = _lognormal(S, 250.0, 1.0, g)
            ctx = torch.clamp(p + o, lo, hi).to(torch.int64).tolist()
        else:
            ctx = torch.randint(lo, hi + 1, (S,), generator=g).tolist()
        prefix = 64 // B if number == 4 else 0      # the 64-token system prompt
        need = prefix + sum(_nblk(c, B) - prefix for c in ctx)
        NB = need + _nblk(need, 8)
        perm = torch.randperm(NB, generator=g).tolist()
        shared = perm[:prefix]
        k = prefix
        tables = []
        for c in ctx:
            n = _nblk(c, B) - prefix
            tables.append(shared + perm[k:k + n])
            k += n
        if prefix:
            meta["prefix_blocks"] = shared
    elif number == 5:
        P_ = num_prompts or 128
        n_samp = 4
        Hq, Hkv, D, dtype = 32, 8, 128, torch.bfloat16
        S = P_ * n_samp
        pmax = max_prompt or 4096
        omax = max_output or 1024
        plen = torch.randint(min(256, pmax), pmax + 1, (P_,), generator=g).tolist()
        olen = torch.randint(1, omax + 1, (S,), generator=g).tolist()
        ctx = [plen[i // n_samp] + olen[i] for i in range(S)]
        need = 0
        for i in range(P_):
            need += plen[i] // B + (n_samp if plen[i] % B else 0)
            for j in range(n_samp):
                c = ctx[i * n_samp + j]
                need += _nblk(c, B) - _nblk(plen[i], B)
        NB = need + _nblk(need, 8)
        perm = torch.randperm(NB, generator=g).tolist()
        k = 0
        tables = []
        for i in range(P_):
            nfull = plen[i] // B
            full = perm[k:k + nfull]
            k += nfull
            part = []
            if plen[i] % B:
                part = perm[k:k + n_samp]       # [original, fresh_1, fresh_2, fresh_3]
                k += n_samp
                for j in range(1, n_samp):
                    copy_pairs.append((part[0], part[j]))
            for j in range(n_samp):
                c = ctx[i * n_samp + j]
                nout = _nblk(c, B) - _nblk(plen[i], B)
                tail = perm[k:k + nout]
                k += nout
                tables.append(full + ([part[j]] if part else []) + tail)
        meta["prompt_lens"] = plen
        meta["samples"] = n_samp
    else:
        raise ValueError(f"unknown workload {number}")

    MB = max(len(t) for t in tables)
    if number == 4:
        MB = max(MB, _nblk(hi, B))
    elif number == 5:
        MB = max(MB, _nblk(pmax + omax, B))
    else:
        MB = max(MB, _nblk(max(ctx), B))
    bt = torch.full((len(tables), MB), -1, dtype=torch.int32)
    for s, row in enumerate(tables):
        bt[s, :len(row)] = torch.tensor(row, dtype=torch.int32)

    dev = torch.device(device)
    gd = g if dev.type == "cpu" else torch.Generator(device=dev).manual_seed(seed)
    q = _randn((S, Hq, D), dtype, gd, dev)
    k_cache = _randn((NB, Hkv, B, D), dtype, gd, dev)
    v_cache = _randn((NB, Hkv, B, D), dtype, gd, dev)
    k_new = _randn((S, Hkv, D), dtype, gd, dev)
    v_new = _randn((S, Hkv, D), dtype, gd, dev)
    if pad_random:
        # drawn last, so the values are the same with or without it
        junk = torch.randint(0, NB, bt.shape, generator=g, dtype=torch.int32)
        bt = torch.where(bt < 0, junk, bt)
    pairs = torch.tensor(copy_pairs, dtype=torch.int64).reshape(-1, 2)
    return DecodeWorkload(name=name, dtype=dtype, num_seqs=S, num_q_heads=Hq, num_kv_heads=Hkv,
                          head_dim=D, block_size=B, num_blocks=NB,
                          context_lens=torch.tensor(ctx, dtype=torch.int32), block_tables=bt,
                          copy_pairs=pairs, q=q, k_cache=k_cache, v_cache=v_cache, k_new=k_new,
                          v_new=v_new, scale=1.0 / math.sqrt(D), seed=seed, meta=meta)


def make_custom(context_lens, num_q_heads: int, num_kv_heads: int, head_dim: int, dtype,
                device="cpu", *, seed: int = 1234, spare_blocks: int = 3,
                max_blocks_per_seq=None, pad_random: bool = False, q_len=None,
                block_size: int = BLOCK_SIZE) -> DecodeWorkload:
    """A batch with the given context lengths and head shape, blocks dealt
    from a seeded permutation of a pool with `spare_blocks` unused blocks.
    With q_len given, q is [S, q_len, Hq, D] and k_new / v_new are
    [S, q_len, Hkv, D] (several new tokens per sequence)."""
    g = torch.Generator().manual_seed(seed)
    B = block_size
    ctx = [int(c) for c in context_lens]
    need = sum(_nblk(max(c, 1), B) for c in ctx)
    NB = need + spare_blocks
    perm = torch.randperm(NB, generator=g).tolist()
    tables, k = [], 0
    for c in ctx:
        n = _nblk(max(c, 1), B)
        tables.append(perm[k:k + n])
        k += n
    MB = max_blocks_per_seq or max(len(t) for t in tables)
    bt = torch.full((len(ctx), MB), -1, dtype=torch.int32)
    for s, row in enumerate(tables):
        bt[s, :len(row)] = torch.tensor(row, dtype=torch.int32)
    S, Hq, Hkv, D = len(ctx), num_q_heads, num_kv_heads, head_dim
    dev = torch.device(device)
    gd = g if dev.type == "cpu" else torch.Generator(device=dev).manual_seed(seed)
    lead = (S,) if q_len is None else (S, q_len)
    q = _randn(lead + (Hq, D), dtype, gd, dev)
    k_cache = _randn((NB, Hkv, B, D), dtype, gd, dev)
    v_cache = _randn((NB, Hkv, B, D), dtype, gd, dev)
    k_new = _randn(lead + (Hkv, D), dtype, gd, dev)
    v_new = _randn(lead + (Hkv, D), dtype, gd, dev)
    if pad_random:
        junk = torch.randint(0, NB, bt.shape, generator=g, dtype=torch.int32)
        bt = torch.where(bt < 0, junk, bt)
    return DecodeWorkload(name="custom", dtype=dtype, num_seqs=S, num_q_heads=Hq, num_kv_heads=Hkv,
                          head_dim=D, block_size=B, num_blocks=NB,
                          context_lens=torch.tensor(ctx, dtype=torch.int32), block_tables=bt,
                          copy_pairs=torch.empty(0, 2, dtype=torch.int64), q=q, k_cache=k_cache,
                          v_cache=v_cache, k_new=k_new, v_new=v_new, scale=1.0 / math.sqrt(D),
                          seed=seed, meta={"workload": "custom"})


def make_sampling(num_prompts: int, samples: int, prompt_range, output_range, num_q_heads: int,
                  num_kv_heads: int, head_dim: int, dtype, device="cpu", *, seed: int = 1234,
                  block_size: int = BLOCK_SIZE) -> DecodeWorkload:
    """Parallel sampling with any head shape: `samples` consecutive sequences
    per prompt share the prompt's full blocks; the prompt's partial last
    block stays with sample 0 and the other samples get fresh blocks filled by
    copy-on-write copies (the step's copy pairs); each sample then has its own
    output blocks.  Prompt and output lengths are uniform in the given
    inclusive ranges.  The layout of workload "8b_gqa_sampling", with the
    same draw order (lengths, pool permutation, Q, cache, new K/V)."""
    g = torch.Generator().manual_seed(seed)
    B = block_size
    plen = torch.randint(prompt_range[0], prompt_range[1] + 1, (num_prompts,), generator=g).tolist()
    olen = torch.randint(output_range[0], output_range[1] + 1, (num_prompts * samples,), generator=g).tolist()
    ctx = [plen[i // samples] + olen[i] for i in range(num_prompts * samples)]
    need = 0
    for i in range(num_prompts):
        need += plen[i] // B + (samples if plen[i] % B else 0)
        for j in range(samples):
            need += _nblk(ctx[i * samples + j], B) - _nblk(plen[i], B)
    NB = need + _nblk(need, 8)
    perm = torch.randperm(NB, generator=g).tolist()
    k, tables, pairs = 0, [], []
    for i in range(num_prompts):
        full = perm[k:k + plen[i] // B]
        k += plen[i] // B
        part = []
        if plen[i] % B:
            part = perm[k:k + samples]
            k += samples
            pairs += [(part[0], part[j]) for j in range(1, samples)]
        for j in range(samples):
            nout = _nblk(ctx[i * samples + j], B) - _nblk(plen[i], B)
            tables.append(full + ([part[j]] if part else []) + perm[k:k + nout])
            k += nout
    MB = max(len(t) for t in tables)
    bt = torch.full((len(tables), MB), -1, dtype=torch.int32)
    for s, row in enumerate(tables):
        bt[s, :len(row)] = torch.tensor(row, dtype=torch.int32)
    S, Hq, Hkv, D = len(ctx), num_q_heads, num_kv_heads, head_dim
    dev = torch.device(device)
    gd = g if dev.type == "cpu" else torch.Generator(device=dev).manual_seed(seed)
    q = _randn((S, Hq, D), dtype, gd, dev)
    k_cache = _randn((NB, Hkv, B, D), dtype, gd, dev)
    v_cache = _randn((NB, Hkv, B, D), dtype, gd, dev)
    k_new = _randn((S, Hkv, D), dtype, gd, dev)
    v_new = _randn((S, Hkv, D), dtype, gd, dev)
    return DecodeWorkload(name="sampling", dtype=dtype, num_seqs=S, num_q_heads=Hq, num_kv_heads=Hkv,
                          head_dim=D, block_size=B, num_blocks=NB,
                          context_lens=torch.tensor(ctx, dtype=torch.int32), block_tables=bt,
                          copy_pairs=torch.tensor(pairs, dtype=torch.int64).reshape(-1, 2), q=q,
                          k_cache=k_cache, v_cache=v_cache, k_new=k_new, v_new=v_new,
                          scale=1.0 / math.sqrt(D), seed=seed,
                          meta={"workload": "sampling", "prompt_lens": plen, "samples": samples})
