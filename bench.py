#!/usr/bin/env python
"""Decode-step benchmark of the paged KV cache path on one B200 (or N replicas).

Workload (default): the 8B-GQA shared-prefix batch -- 256 sequences, 32 query
heads over 8 kv heads, head_dim 128, bf16, 16-token blocks; every sequence
shares 4 physical prefix blocks (64 tokens) and has total context uniform in
[65, 8192].  The native host allocator lays the batch out (shared prefix,
on-demand blocks from a shuffled free list) and hands out this step's slots.

One timed step = the whole device path of a decode step:
  block_copy (copy-on-write pairs, if any) -> paged_kv_write -> paged_attention_decode
on inputs already resident in HBM.  The K/V stream (4.3 GB) is far larger
than L2 (126 MB), so no L2 flush is needed between steps.

value  = effective KV GB/s = sum_s ctx_s * Hkv * D * 2 (K and V) * elem / step time
e2e    = the same metric with, per step, pinned host -> device copies of the
         step's inputs and a device -> host copy of the output in the timed region
roofline = decode kernel(s) only: algorithmic bytes (K/V + Q + out + tables)
           per launch / mean launch time (CUDA events on the launching stream)

`--impl reference` times the plain CPU oracle on a bounded sample of the same
workload on the host cores (the slow baseline), and prints the same line.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import torch  # noqa: E402

METRIC = "paged decode attention: effective KV GB/s (% of HBM peak), seq-steps/s"
WORKLOAD_NAMES = {1: "tiny", 2: "7b", 3: "13b", 4: "8b_gqa_prefix", 5: "8b_gqa_sampling"}
FALLBACK_HBM_GBS = 6650.0


DECODE_SOURCES = ("paged_kv_cache_398_b200/csrc/decode.cu", "paged_kv_cache_398_b200/csrc/decode_tc.cuh",
                  "paged_kv_cache_398_b200/csrc/decode_common.cuh", "paged_kv_cache_398_b200/csrc/common.cuh")
TRAFFIC_RECORD = os.path.join(ROOT, "profiles", "decode_traffic.json")
NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e, nominal (the measured copy peak is the roofline denominator)


def decode_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for rel in DECODE_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def recorded_traffic(workload: str, num_seqs: int, path: str, block_size: int, q_len: int):
    """DRAM bytes per decode call from the committed ncu record, or None if
    there is none for this step or the decode sources changed since.  The
    record is captured on a smaller cut of the same recipe that takes the
    same kernel instantiation, and scaled to the full batch by its
    algorithmic bytes (its "scaling" key says how)."""
    try:
        with open(TRAFFIC_RECORD) as f:
            rec = json.load(f)
    except (OSError, ValueError):
        return None
    if rec.get("source_sha256") != decode_source_hash():
        return None
    if (rec.get("workload"), rec.get("applies_to_num_seqs"), rec.get("path"), rec.get("block_size"),
            rec.get("q_len", 1)) != (workload, num_seqs, path, block_size, q_len):
        return None
    return rec.get("dram_bytes_per_call")


def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ----------------------------------------------------------------------------
# workload state
# ----------------------------------------------------------------------------
class Step:
    """Everything one decode step needs, resident on the GPU."""


def build_step(number: int, device, rank: int = 0, num_seqs=None, block_size: int = 16, max_ctx=None,
               q_len: int = 1, path: str = "fused"):
    """The decode step of workload `number`.  q_len > 1: every sequence
    brings q_len new tokens (draft tokens to verify, causal among them) after
    a prompt of ctx - q_len tokens; the recipe's shortest context is raised
    to leave room for them.  path 'shared': the host also plans which
    sequences share leading blocks (pkv_shared_prefix_plan), and the plan's
    two arrays travel with the step's inputs."""
    import paged_kv_cache_398_b200 as pkv
    from paged_kv_cache_398_b200.workloads import make_workload

    seed = rank_seed(number, rank)
    kw = {}
    if num_seqs:
        kw = {"num_prompts": max(1, num_seqs // 4)} if number == 5 else {"num_seqs": num_seqs}
    if max_ctx and number in (2, 3, 4):
        kw["max_ctx"] = max_ctx
    if q_len > 1:
        if number not in (2, 3, 4):
            raise SystemExit("--q-len > 1 is measured on workloads 2-4")
        kw["min_ctx"] = q_len + (64 if number == 4 else 0)   # room for the prompt and the new tokens
    w = make_workload(number, device=device, seed=seed, block_size=block_size, **kw)   # lengths on host, values on the GPU
    S = w.num_seqs
    st = Step()
    st.w = w
    st.host_alloc_us = None
    st.host_step_us = None
    st.prefix = None
    st.admit_us_per_request = None
    if number == 5:
        # parallel sampling: the generator's tables already hold the shared
        # prompt blocks; the step's copy-on-write pairs come with them
        tables, lens, pairs = w.block_tables, w.context_lens, w.copy_pairs
        slots = pkv.pkv_slot_mapping(tables, lens - 1)
    else:
        gen = torch.Generator().manual_seed(seed + 7)
        perm = torch.randperm(w.num_blocks, generator=gen)
        alloc = pkv.BlockAllocator(w.num_blocks, w.block_size, initial_order=perm)
        if number == 4:
            # every request starts with the same 64-token system prompt; the
            # prefix cache finds its 4 blocks instead of being told about them
            system = torch.randint(0, 128000, (64,), generator=gen)
            t0 = time.perf_counter()
            for s in range(S):
                own = torch.randint(0, 128000, (int(w.context_lens[s]) - q_len - 64,), generator=gen)
                alloc.add(s)
                alloc.append_prompt(s, torch.cat([system, own]))
            st.admit_us_per_request = (time.perf_counter() - t0) * 1e6 / S
            st.prefix = alloc.prefix_stats()
            assert st.prefix["hit_tokens"] == 64 * (S - 1)     # every request found the system prompt
        else:
            for s in range(S):
                alloc.add(s)
                alloc.append_tokens(s, int(w.context_lens[s]) - q_len)
        seqs = list(range(S))
        t0 = time.perf_counter()
        if q_len == 1:
            slots, pairs = alloc.append_one_batch(seqs)      # this step's slots (+ CoW pairs)
        else:
            per_seq = [alloc.append_tokens(s, q_len) for s in seqs]
            slots = torch.cat([torch.as_tensor(sl, dtype=torch.int64) for sl, _ in per_seq])
            pairs = torch.tensor([c for _, c in per_seq if c is not None], dtype=torch.int64).reshape(-1, 2)
        tables, lens = alloc.batch_tables(seqs, w.max_blocks_per_seq)
        st.host_alloc_us = (time.perf_counter() - t0) * 1e6
        assert torch.equal(lens, w.context_lens)
        st.alloc = alloc
        st.host_step_us = host_step_cost(alloc, S, w.max_blocks_per_seq + 2)
    st.tables_host, st.lens_host, st.slots_host, st.pairs = tables, lens, slots, pairs
    st.inputs = STEP_INPUTS
    st.plan, st.host_plan_us = None, None
    if path == "shared":
        if q_len != 1:
            raise SystemExit("--path shared decodes one new token per sequence")
        pt = pkv.paged_attention_partition_tokens(S, w.num_kv_heads, int(lens.max()), w.dtype)
        t0 = time.perf_counter()
        st.plan = pkv.pkv_shared_prefix_plan(tables, lens, w.block_size,
                                             pkv.SHARED_MAX_ROWS // (w.num_q_heads // w.num_kv_heads), pt)
        st.host_plan_us = (time.perf_counter() - t0) * 1e6
        times = []                               # as a serving loop pays it, step after step
        for _ in range(20):
            t0 = time.perf_counter()
            pkv.pkv_shared_prefix_plan(tables, lens, w.block_size,
                                       pkv.SHARED_MAX_ROWS // (w.num_q_heads // w.num_kv_heads), pt)
            times.append(time.perf_counter() - t0)
        st.host_plan_us_steady = statistics.median(times) * 1e6
        st.groups, st.shared_lens, st.work = st.plan.groups, st.plan.shared_lens, st.plan.work
        st.inputs = STEP_INPUTS + ("groups", "shared_lens", "work")
    st.block_tables = tables.to(device)
    st.context_lens = lens.to(device)
    st.slots = slots.to(device)
    st.q_len = q_len
    st.k_cache, st.v_cache = w.k_cache, w.v_cache
    if q_len == 1:
        st.q, st.k_new, st.v_new = w.q, w.k_new, w.v_new
    else:
        from paged_kv_cache_398_b200.workloads import _randn
        gd = torch.Generator(device=device).manual_seed(seed + 11)
        st.q = _randn((S, q_len, w.num_q_heads, w.head_dim), w.dtype, gd, device)
        st.k_new = _randn((S, q_len, w.num_kv_heads, w.head_dim), w.dtype, gd, device)
        st.v_new = _randn((S, q_len, w.num_kv_heads, w.head_dim), w.dtype, gd, device)
    st.out = torch.empty_like(st.q)
    pack_step_inputs(st, device)
    st.path = "separate"
    st.max_ctx = int(lens.max())
    ws_bytes = (pkv.paged_attention_shared_workspace_bytes(S, w.num_q_heads, w.head_dim, st.max_ctx)
                if path == "shared" else
                pkv.paged_attention_mq_workspace_bytes(S, q_len, w.num_q_heads, w.head_dim, st.max_ctx))
    st.workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=device)
    e = w.q.element_size()
    ctx = lens.to(torch.int64)
    nblk = (ctx + w.block_size - 1) // w.block_size
    per_token = w.num_kv_heads * w.head_dim * 2 * e            # K and V of one position, all kv heads
    st.kv_bytes = int(ctx.sum()) * per_token                    # logical: every sequence's own context
    st.kv_unique_bytes = unique_live_tokens(tables, lens, w.block_size) * per_token
    other = 2 * S * q_len * w.num_q_heads * w.head_dim * e + 4 * int(nblk.sum()) + 4 * S   # Q, out, tables, lens
    st.decode_bytes = st.kv_bytes + other
    st.write_bytes = 2 * 2 * S * q_len * w.num_kv_heads * w.head_dim * e + 8 * S * q_len
    st.copy_bytes = 2 * 2 * pairs.shape[0] * w.num_kv_heads * w.block_size * w.head_dim * e
    st.part_tokens = pkv.paged_attention_mq_partition_tokens(S, q_len, w.num_q_heads, w.num_kv_heads, st.max_ctx,
                                                             w.dtype)
    st.max_parts = (st.max_ctx + st.part_tokens - 1) // st.part_tokens
    st.launches_separate = (1 if pairs.shape[0] else 0) + 1 + 1 + (1 if st.max_parts > 1 else 0)
    st.launches_fused = st.launches_separate - 1
    st.shared_bytes = None
    if st.plan is not None:
        # block copies, both passes (one launch), reduce
        st.launches_shared = (1 if pairs.shape[0] else 0) + 2
        # K/V the two passes must read under the plan: each group's shared
        # positions once, every sequence's own positions once
        x = st.plan.shared_lens.to(torch.int64)
        first = st.plan.groups[:, 0].to(torch.int64)
        tokens = int(x[first].sum()) + int((ctx - x).sum())
        st.plan_bytes = 4 * S + 8 * first.numel() + 8 * st.plan.work.shape[0]   # shared_lens, groups, work list
        st.shared_bytes = tokens * per_token + other + st.plan_bytes + st.write_bytes
    # the decode call's bytes (roofline): the K/V it must read counted once per
    # physical block's live tokens (unique), or once per sequence (logical)
    extra = {"fused": st.write_bytes, "shared": st.write_bytes + getattr(st, "plan_bytes", 0), "separate": 0}[path]
    st.call_bytes_unique = st.kv_unique_bytes + other + extra
    st.call_bytes_logical = st.kv_bytes + other + extra
    return st


def unique_live_tokens(tables, lens, block_size: int) -> int:
    """Token-exact count of the K/V positions a step must read at least once:
    each physical block the batch's tables reach counts its live tokens once
    (the most any sequence holding it uses), however many sequences share it."""
    lens = lens.to(torch.int64)
    nblk = (lens + block_size - 1) // block_size
    mb = tables.shape[1]
    idx = torch.arange(mb, dtype=torch.int64)
    live = idx[None, :] < nblk[:, None]                                  # [S, MB] entries in use
    used = (lens[:, None] - idx[None, :] * block_size).clamp(0, block_size)
    ids = tables.to(torch.int64)[live]
    used = used[live]
    keep = ids >= 0                       # an invalid id reads nothing the call counts
    ids, used = ids[keep], used[keep]
    if ids.numel() == 0:
        return 0
    per_block = torch.zeros(int(ids.max()) + 1, dtype=torch.int64)
    per_block.scatter_reduce_(0, ids, used, reduce="amax")
    return int(per_block.sum())


STEP_INPUTS = ("q", "k_new", "v_new", "slots", "block_tables", "context_lens")


def pack_step_inputs(st, device):
    """Place a step's inputs (q, new K/V, slots, tables, lengths) in one
    device buffer, each at a 256-byte aligned offset, with a pinned host
    mirror, so the end-to-end loop moves them with one host-to-device copy
    instead of six.  The tensors are rebound to views of the buffer."""
    st.in_layout, total = [], 0
    for name in st.inputs:
        t = getattr(st, name)
        st.in_layout.append((name, total, t.numel() * t.element_size(), t.dtype, tuple(t.shape)))
        total += -(-t.numel() * t.element_size() // 256) * 256
    st.in_dev = torch.empty(max(total, 256), dtype=torch.uint8, device=device)
    views = input_views(st, st.in_dev)
    for name, view in views.items():
        view.copy_(getattr(st, name).contiguous())
    st.in_host = st.in_dev.cpu().pin_memory() if st.in_dev.is_cuda else st.in_dev.clone()
    bind_step_inputs(st, views, st.out)


def input_views(st, buf):
    """The step's input tensors as views of a packed buffer laid out as st.in_layout."""
    return {name: buf[off:off + n].view(dtype).view(shape) for name, off, n, dtype, shape in st.in_layout}


def step_bindings(st, views, out):
    """Every tensor attribute a step reads, for one set of input views and
    one output: the inputs, and their [S, q_len, ...] views (for
    paged_attention_decode_mq) and flat [S * q_len, ...] rows (for
    paged_kv_write)."""
    b = dict(views)
    b["out"] = out
    S, q_len = b["q"].shape[0], st.q_len
    lead = (S, q_len)
    b["q4"], b["out4"] = b["q"].reshape(lead + b["q"].shape[-2:]), out.reshape(lead + out.shape[-2:])
    b["k_new4"], b["v_new4"] = (b[n].reshape(lead + b[n].shape[-2:]) for n in ("k_new", "v_new"))
    b["k_rows"], b["v_rows"] = (b[n].reshape(S * q_len, *b[n].shape[-2:]) for n in ("k_new", "v_new"))
    return b


def bind_step_inputs(st, views, out):
    """Point the step at one set of input views and one output tensor."""
    for name, t in step_bindings(st, views, out).items():
        setattr(st, name, t)


def e2e_steps_pipelined(st, n: int, dev, h_out):
    """n steps end to end, as a serving loop runs them: every step's inputs
    go from pinned host memory to the device and its output comes back to
    pinned host memory.  Two packed input buffers and two outputs let step
    i+1's inputs cross on an H2D stream, and step i-1's output on a D2H
    stream, while step i's kernels run on the current stream.  Returns the
    CUDA events that bracket all of it on the current stream."""
    comp = torch.cuda.current_stream(dev)
    if not hasattr(st, "e2e_bufs"):
        st.e2e_bufs = [st.in_dev, torch.empty_like(st.in_dev)]
        st.e2e_outs = [st.out, torch.empty_like(st.out)]
        # all of a step's tensor attributes per buffer, made once: rebinding
        # is then a few attribute stores, so the host keeps ahead of short steps
        st.e2e_bind = [list(step_bindings(st, input_views(st, b), o).items())
                       for b, o in zip(st.e2e_bufs, st.e2e_outs)]
        st.e2e_streams = (torch.cuda.Stream(dev), torch.cuda.Stream(dev))
    h2d, d2h = st.e2e_streams
    bufs, outs = st.e2e_bufs, st.e2e_outs
    in_ready, in_free, out_ready, out_free = ([torch.cuda.Event(), torch.cuda.Event()] for _ in range(4))
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(comp)
    h2d.wait_event(start)
    d2h.wait_event(start)
    with torch.cuda.stream(h2d):
        bufs[0].copy_(st.in_host, non_blocking=True)
    in_ready[0].record(h2d)
    for i in range(n):
        b, nb = i % 2, (i + 1) % 2
        if i + 1 < n:
            if i >= 1:
                h2d.wait_event(in_free[nb])          # step i-1 has finished with buffer nb
            with torch.cuda.stream(h2d):
                bufs[nb].copy_(st.in_host, non_blocking=True)
            in_ready[nb].record(h2d)
        comp.wait_event(in_ready[b])
        if i >= 2:
            comp.wait_event(out_free[b])             # step i-2's output has left outs[b]
        for name, t in st.e2e_bind[b]:
            setattr(st, name, t)
        run_step(st)
        in_free[b].record(comp)
        out_ready[b].record(comp)
        d2h.wait_event(out_ready[b])
        with torch.cuda.stream(d2h):
            h_out[b].copy_(outs[b], non_blocking=True)
        out_free[b].record(d2h)
    comp.wait_stream(d2h)
    comp.wait_stream(h2d)
    stop.record(comp)
    return start, stop


def host_step_cost(alloc, S: int, mb: int, steps: int = 20) -> float:
    """Median host time of one more decode step's allocation, as a serving
    loop pays it: slots (and copy-on-write pairs) for one token per sequence,
    then the block tables refilled in place (live entries only) into reused
    buffers.  Runs after the timed step's inputs were taken, so it changes
    nothing the GPU sees."""
    import paged_kv_cache_398_b200 as pkv
    ids = torch.arange(S, dtype=torch.int64)
    slots, pairs = torch.empty(S, dtype=torch.int64), torch.empty(S, 2, dtype=torch.int64)
    tables, lens = torch.full((S, mb), -1, dtype=torch.int32), torch.empty(S, dtype=torch.int32)
    alloc.batch_tables(ids, mb, tables_out=tables, lens_out=lens)
    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        alloc.append_one_batch(ids, slots_out=slots, pairs_out=pairs)
        alloc.batch_tables(ids, mb, pad=pkv.TABLE_KEEP_TAIL, tables_out=tables, lens_out=lens)
        times.append(time.perf_counter() - t0)
    return statistics.median(times) * 1e6


def run_step(st, ev=None):
    """One decode step on the device.  path 'separate': paged_kv_write, then
    paged_attention_decode.  path 'fused': paged_attention_decode_mq with the
    new tokens' K/V, which writes them to their slots in the same launch.
    With `ev` (four CUDA events) the step records them before the block copy,
    after it, after the slot write and after the decode call."""
    import paged_kv_cache_398_b200 as pkv
    if ev is not None:
        ev[0].record()
    if st.pairs.shape[0]:
        pkv.block_copy(st.k_cache, st.v_cache, st.pairs)
    if ev is not None:
        ev[1].record()
    if st.path == "separate":
        pkv.paged_kv_write(st.k_rows, st.v_rows, st.k_cache, st.v_cache, st.slots)
    if ev is not None:
        ev[2].record()
    run_decode(st)
    if ev is not None:
        ev[3].record()


def run_decode(st):
    """The step's decode call alone (the call run_step makes after its copies and write)."""
    import paged_kv_cache_398_b200 as pkv
    if st.path == "separate" and st.q_len == 1:
        pkv.paged_attention_decode(st.out, st.q, st.k_cache, st.v_cache, st.block_tables, st.context_lens,
                                   st.w.scale, st.max_ctx, workspace=st.workspace)
    elif st.path == "separate":
        pkv.paged_attention_decode_mq(st.out4, st.q4, st.k_cache, st.v_cache, st.block_tables, st.context_lens,
                                      st.w.scale, st.max_ctx, workspace=st.workspace)
    elif st.path == "shared":
        pl = st.plan
        pkv.paged_attention_decode_shared(st.out, st.q, st.k_cache, st.v_cache, st.block_tables, st.context_lens,
                                          st.w.scale, st.max_ctx, st.groups, st.shared_lens, st.work, pl.part_tokens,
                                          k_new=st.k_new, v_new=st.v_new, workspace=st.workspace)
    else:
        pkv.paged_attention_decode_mq(st.out4, st.q4, st.k_cache, st.v_cache, st.block_tables, st.context_lens,
                                      st.w.scale, st.max_ctx, k_new=st.k_new4, v_new=st.v_new4,
                                      workspace=st.workspace)


def sampled_steps(steps: int, samples: int = 60):
    """Indices of the timed steps whose kernels are bracketed by CUDA events.
    An event between two launches costs the second one its programmatic
    early launch (on the small batches about 7 us a step), so only about
    `samples` steps, spread evenly, carry them; the rest run as a user's
    loop would."""
    every = max(1, -(-steps // samples))
    return sorted(i for i in range(steps) if i % every == every - 1)


# ----------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------
class ClockSampler:
    """SM clock, power and clock-event reasons of this GPU, sampled every
    `period_s` on a host thread through NVML (or, without the Python NVML
    binding, from `nvidia-smi -lms`, at its coarser period).  summary()
    covers the samples that fall inside the given wall-clock windows."""

    REASONS = (("sw_power_cap", 0x4), ("hw_slowdown", 0x8), ("sw_thermal_slowdown", 0x20),
               ("hw_thermal_slowdown", 0x40), ("hw_power_brake_slowdown", 0x80))
    SMI_FIELDS = ("pci.bus_id,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active")

    def __init__(self, device_index: int, period_s: float = 0.002):
        p = torch.cuda.get_device_properties(device_index)
        self.bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
        self.period = period_s
        self.samples = []          # (monotonic time, sm MHz, power W, reasons bit mask)
        self.max_mhz = None
        self.source = None
        self.nvml = None
        self._stop = threading.Event()
        self.thread = self.proc = None

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            h = pynvml.nvmlDeviceGetHandleByPciBusId(self.bus)
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(h, pynvml.NVML_CLOCK_SM))
            reasons = getattr(pynvml, "nvmlDeviceGetCurrentClocksEventReasons",
                              getattr(pynvml, "nvmlDeviceGetCurrentClocksThrottleReasons", None))
            self.source = "nvml"
            self.nvml = pynvml
            self.thread = threading.Thread(target=self._poll_nvml, args=(pynvml, h, reasons), daemon=True)
        except Exception:
            try:
                self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.SMI_FIELDS}",
                                              "--format=csv,noheader,nounits", "-lms", "20"],
                                             stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            except Exception:
                return
            self.source = "nvidia-smi"
            self.thread = threading.Thread(target=self._read_smi, daemon=True)
        self.thread.start()

    def _poll_nvml(self, nvml, h, reasons):
        while not self._stop.is_set():
            try:
                t = time.monotonic()
                sm = float(nvml.nvmlDeviceGetClockInfo(h, nvml.NVML_CLOCK_SM))
                pw = nvml.nvmlDeviceGetPowerUsage(h) / 1000.0
                rs = int(reasons(h)) if reasons else 0
                self.samples.append((t, sm, pw, rs))
            except Exception:
                return
            self._stop.wait(self.period)

    def _read_smi(self):
        for line in self.proc.stdout:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 5 or not parts[0].upper().endswith(self.bus[-7:]):   # "BB:DD.F" of this GPU
                continue
            try:
                self.max_mhz = float(parts[2])
                self.samples.append((time.monotonic(), float(parts[1]), float(parts[3]), int(parts[4], 16)))
            except ValueError:
                continue

    def stop(self):
        self._stop.set()
        if self.proc:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        if self.thread:
            self.thread.join(timeout=5)
            self.thread = None
        if self.nvml is not None:
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
            self.nvml = None

    def summary(self, windows, label: str):
        """Median SM clock, peak power and every slowdown reason seen in the samples inside `windows`."""
        win = [x for x in self.samples if any(a <= x[0] <= b for a, b in windows)]
        if not win:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "window": label, "source": self.source or "unavailable"}
        mask = 0
        for x in win:
            mask |= x[3]
        return {"sm_mhz": statistics.median(x[1] for x in win), "sm_min_mhz": min(x[1] for x in win),
                "sm_max_mhz": self.max_mhz, "power_w_max": max(x[2] for x in win),
                "reasons": [n for n, bit in self.REASONS if mask & bit], "samples": len(win),
                "period_ms": self.period * 1e3 if self.source == "nvml" else 20.0,
                "window": label, "source": self.source}


# ----------------------------------------------------------------------------
# the oracle on the host cores
# ----------------------------------------------------------------------------
def sub_workload(w, tables, lens, pairs, seqs, repeated: bool = False, q=None, k_new=None, v_new=None):
    """The listed sequences' blocks (plus copy sources) copied to the host and
    relabelled 0..n-1, with their tables, as an oracle input.

    repeated: the input of the step as the timed loop runs it, after it has
    already run once.  A step is not idempotent when a sequence's new token
    lands in a copy-on-write source block (a sample whose own output still
    fits in the prompt's partial block): the next repetition copies that
    token into its siblings' blocks.  meta["pre_writes"] then holds the new
    token of every sequence of the batch, sampled or not, whose slot lies in
    these blocks, for oracle_step_timed to apply once (copies + those writes)
    before the step it times.

    q / k_new / v_new: the step's own tensors when they are not the
    workload's (multi-query steps: [S, q_len, heads, D])."""
    from paged_kv_cache_398_b200.workloads import DecodeWorkload
    B = w.block_size
    q = w.q if q is None else q
    k_new = w.k_new if k_new is None else k_new
    v_new = w.v_new if v_new is None else v_new
    need = []
    for s in seqs:
        need += tables[s, :-(-int(lens[s]) // B)].tolist()
    dsts = set(need)
    sub_pairs = [(int(a), int(b)) for a, b in pairs.tolist() if int(b) in dsts]
    need += [a for a, _ in sub_pairs]
    ids = sorted(set(need))
    remap = {b: i for i, b in enumerate(ids)}
    idx = torch.tensor(ids, dtype=torch.int64, device=w.k_cache.device)
    sbt = torch.full((len(seqs), tables.shape[1]), -1, dtype=torch.int32)
    for r, s in enumerate(seqs):
        n = -(-int(lens[s]) // B)
        sbt[r, :n] = torch.tensor([remap[b] for b in tables[s, :n].tolist()], dtype=torch.int32)
    sel = torch.tensor(seqs, dtype=torch.int64, device=q.device)
    meta = {}
    if repeated:
        writers, slots = [], []
        for s in range(lens.shape[0]):
            pos = int(lens[s]) - 1
            b = int(tables[s, pos // B])
            if b in remap:
                writers.append(s)
                slots.append(remap[b] * B + pos % B)
        wsel = torch.tensor(writers, dtype=torch.int64, device=q.device)
        meta["pre_writes"] = (torch.tensor(slots, dtype=torch.int64), k_new[wsel].cpu(), v_new[wsel].cpu())
    return DecodeWorkload(
        name=w.name + "-sample", dtype=w.dtype, num_seqs=len(seqs), num_q_heads=w.num_q_heads,
        num_kv_heads=w.num_kv_heads, head_dim=w.head_dim, block_size=B, num_blocks=len(ids),
        context_lens=lens[seqs].contiguous(), block_tables=sbt,
        copy_pairs=torch.tensor([(remap[a], remap[b]) for a, b in sub_pairs], dtype=torch.int64).reshape(-1, 2),
        q=q[sel].cpu(), k_cache=w.k_cache[idx].cpu(), v_cache=w.v_cache[idx].cpu(),
        k_new=k_new[sel].cpu(), v_new=v_new[sel].cpu(), scale=w.scale, seed=w.seed, meta=meta)


def oracle_step_timed(sub, threads: int, keep=None):
    """Run the oracle's copy + write + decode on `sub`; returns wall seconds.
    With `keep` (a list), the fp64 outputs of the sequences ([Hq, D], or
    [q_len, Hq, D] for a multi-query step) are appended to it."""
    import concurrent.futures as cf

    import oracle
    from oracle.allocator_model import slot_for_position
    B = sub.block_size
    mq = sub.q.dim() == 4                      # [n, q_len, Hq, D]: q_len new tokens per sequence
    ql = sub.q.shape[1] if mq else 1
    slots = torch.tensor([slot_for_position(sub.block_tables[s].tolist(), int(sub.context_lens[s]) - ql + j, B)
                          for s in range(sub.num_seqs) for j in range(ql)], dtype=torch.int64)
    k_rows = sub.k_new.reshape(-1, *sub.k_new.shape[-2:])
    v_rows = sub.v_new.reshape(-1, *sub.v_new.shape[-2:])
    k, v = sub.k_cache.clone(), sub.v_cache.clone()
    if "pre_writes" in sub.meta:                 # the step's earlier repetition (untimed)
        pre_slots, pre_k, pre_v = sub.meta["pre_writes"]
        if sub.copy_pairs.numel():
            oracle.block_copy(k, v, sub.copy_pairs)
        oracle.kv_write(k, v, pre_k, pre_v, pre_slots)

    def one(s):
        if mq:
            return oracle.paged_decode_mq(sub.q[s:s + 1], k, v, sub.block_tables[s:s + 1],
                                          sub.context_lens[s:s + 1], sub.scale)[0]
        return oracle.paged_decode_seq(s, sub.q, k, v, sub.block_tables, sub.context_lens, sub.scale)

    t0 = time.perf_counter()
    if sub.copy_pairs.numel():
        oracle.block_copy(k, v, sub.copy_pairs)
    oracle.kv_write(k, v, k_rows, v_rows, slots)
    with cf.ThreadPoolExecutor(max_workers=threads) as ex:
        outs = list(ex.map(one, range(sub.num_seqs)))
    t = time.perf_counter() - t0
    if keep is not None:
        keep.extend(outs)
    return t


def sample_kv_bytes(sub) -> int:
    return int(sub.context_lens.to(torch.int64).sum()) * sub.num_kv_heads * sub.head_dim * 2 * sub.q.element_size()


def cpu_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def pick_sample(lens, work_seconds_target: float, per_token_s: float):
    """Leading sequences whose oracle work adds up to about the target."""
    seqs, acc = [], 0.0
    for s in range(len(lens)):
        seqs.append(s)
        acc += int(lens[s]) * per_token_s
        if acc >= work_seconds_target:
            break
    return seqs


def step_sub_workload(st, seqs, repeated: bool = False):
    """The oracle input for the listed sequences of a built step (its own Q
    and new K/V, which may be multi-query)."""
    return sub_workload(st.w, st.tables_host, st.lens_host, st.pairs, seqs, repeated=repeated,
                        q=st.q, k_new=st.k_new, v_new=st.v_new)


def cpu_baseline(st, threads: int, target_s: float = 30.0):
    """The oracle on the host cores, on the leading sequences of the step
    whose single-thread work adds up to about target_s seconds.  Returns its
    throughput and, under "refs", its fp64 outputs for the parity check."""
    lens = st.lens_host
    probe = step_sub_workload(st, [0])
    t1 = oracle_step_timed(probe, 1)
    per_tok = t1 / max(1, int(lens[0]))
    seqs = pick_sample(lens, target_s, per_tok)
    sub = step_sub_workload(st, seqs, repeated=True)
    refs = []
    t = oracle_step_timed(sub, threads, keep=refs)
    return {"value": sample_kv_bytes(sub) / t / 1e9, "unit": "GB/s", "cores": threads, "kind": "oracle",
            "sample": (f"{len(seqs)} of {len(lens)} sequences (all {sub.num_q_heads} query heads"
                       f"{f', {st.q_len} new tokens each' if st.q_len > 1 else ''}): "
                       f"copy + slot write + decode by the fp64 C oracle, {t:.2f} s wall on {threads} threads"),
            "seconds": t, "seqs": seqs, "refs": refs}


def parity_on_sample(st, base, atol: float = 2e-3, rtol: float = 1e-2):
    """The timed steps' output of the sampled sequences against the oracle's
    fp64 output of the same step as the loop repeats it (from its second
    repetition on, every repetition leaves the cache as the one before, so
    the last step's output is the one to compare)."""
    import numpy as np
    got = st.out[torch.tensor(base["seqs"], device=st.out.device)].double().cpu().numpy()
    ref = np.stack(base["refs"])
    err = np.abs(got - ref)
    big = np.abs(ref) > 1e-3
    shape = " x ".join(str(n) for n in ref.shape[1:])
    return {"max_abs_err": float(err.max()), "max_rel_err": float((err[big] / np.abs(ref[big])).max()),
            "out_of_tolerance": int((err > atol + rtol * np.abs(ref)).sum()), "elements": int(err.size),
            "tolerance": f"|gpu - oracle| <= {atol:g} + {rtol:g} |oracle| per element",
            "sample": f"{len(base['seqs'])} of {st.out.shape[0]} sequences, each {shape} "
                      f"({'new tokens x ' if ref.ndim == 4 else ''}query heads x head_dim)"}


# ----------------------------------------------------------------------------
# arms
# ----------------------------------------------------------------------------
def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    from paged_kv_cache_398_b200.workloads import make_workload
    threads = cpu_threads()
    # a bounded sample of the workload's recipe, built on the host only
    n = args.reference_seqs
    w = make_workload(args.workload, device="cpu", **({"num_prompts": max(1, n // 4)} if args.workload == 5
                                                       else {"num_seqs": n}))
    lens, tables, pairs = w.context_lens, w.block_tables, w.copy_pairs
    sub = sub_workload(w, tables, lens, pairs, list(range(w.num_seqs)))
    for _ in range(args.warmup):
        oracle_step_timed(sub, threads)
    times = [oracle_step_timed(sub, threads) for _ in range(args.steps)]
    total = sum(times)
    kvb = sample_kv_bytes(sub)
    value = kvb * args.steps / total / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total / args.steps * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": str(w.dtype).replace("torch.", ""), "data": "synthetic",
        "config": {"workload": WORKLOAD_NAMES[args.workload], "sample_seqs": w.num_seqs,
                   "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim,
                   "block_size": w.block_size},
        "seq_steps_per_s": w.num_seqs * args.steps / total,
        "cpu_baseline": {"kind": "oracle", "cores": threads, "value": value, "unit": "GB/s",
                         "sample": f"{w.num_seqs} sequences of the workload recipe per step, fp64 C oracle "
                                   f"(copy + slot write + decode) on {threads} host threads"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def fragmentation_report(lens, max_len: int = 8192):
    """Internal fragmentation of the batch's contexts under paged allocation
    with block sizes 8, 16 and 32 (the native allocator's own count: empty
    slots in each sequence's last block), against one contiguous
    reservation of max_len tokens per request."""
    import paged_kv_cache_398_b200 as pkv
    lens = [int(n) for n in lens]
    total = sum(lens)
    rep = {}
    for bs in (8, 16, 32):
        need = sum(-(-n // bs) for n in lens)
        a = pkv.BlockAllocator(need, bs)
        for i, n in enumerate(lens):
            a.add(i)
            a.append_tokens(i, n)
        st = a.stats()
        held = st["used_blocks"] * bs
        rep[f"block_{bs}"] = {"waste_tokens": st["fragmentation_tokens"],
                              "waste_pct": 100.0 * st["fragmentation_tokens"] / held,
                              "max_waste_per_seq": bs - 1}
    rep["contiguous_max_len"] = {"max_len": max_len, "waste_pct": 100.0 * (1 - total / (max_len * len(lens)))}
    return rep


def measure_swap(st, dev, nblocks: int = 2048, iters: int = 10):
    """Preemption traffic: swap_blocks_out / swap_blocks_in of nblocks blocks
    of this workload's cache (then back into the same blocks, so the cache
    is unchanged), against a plain pinned copy of the same bytes over the
    host link.  GB/s counts K and V."""
    import paged_kv_cache_398_b200 as pkv
    w = st.w
    n = min(nblocks, w.num_blocks)
    ids = torch.randperm(w.num_blocks, generator=torch.Generator().manual_seed(5))[:n]
    shape = (n, w.num_kv_heads, w.block_size, w.head_dim)
    hk = torch.empty(shape, dtype=w.dtype).pin_memory()
    hv = torch.empty(shape, dtype=w.dtype).pin_memory()
    dk = torch.empty(shape, dtype=w.dtype, device=dev)
    nbytes = 2 * hk.numel() * hk.element_size()

    def timed(fn):
        for _ in range(3):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        a.record()
        for _ in range(iters):
            fn()
        b.record()
        torch.cuda.synchronize(dev)
        return nbytes * iters / (a.elapsed_time(b) / 1e3) / 1e9

    out_gbps = timed(lambda: pkv.swap_blocks_out(st.k_cache, st.v_cache, ids, hk, hv))
    in_gbps = timed(lambda: pkv.swap_blocks_in(st.k_cache, st.v_cache, ids, hk, hv))
    d2h = timed(lambda: (hk.copy_(dk, non_blocking=True), hv.copy_(dk, non_blocking=True)))
    h2d = timed(lambda: (dk.copy_(hk, non_blocking=True), dk.copy_(hv, non_blocking=True)))
    return {"blocks": n, "bytes_per_call": nbytes, "out_gbps": out_gbps, "in_gbps": in_gbps,
            "link_d2h_gbps": d2h, "link_h2d_gbps": h2d,
            "note": "one gather/scatter kernel over pinned host memory vs a contiguous pinned copy of the same size"}


def reduce_over_ranks(dist, device, times_ms, amounts):
    """Max over ranks of each time, sum over ranks of each amount (timing and
    byte counts only; the decode path itself exchanges nothing)."""
    t = torch.tensor(list(times_ms), dtype=torch.float64, device=device)
    a = torch.tensor(list(amounts), dtype=torch.float64, device=device)
    if dist is not None:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(a, op=dist.ReduceOp.SUM)
    return t.tolist() + a.tolist()


def rank_seed(number: int, rank: int) -> int:
    """Each replica decodes its own batch of the same shape."""
    return 398000 + number + 1000 * rank


def time_step(st, steps: int, warmup: int, dev, barrier):
    """`warmup` untimed steps, then `steps` timed ones between a barrier and a
    device synchronise on both sides (CUDA events around all of them), then
    the same steps again with events around each call of the evenly spread
    sampled steps (the per-call breakdown), then the end-to-end loop (host
    inputs in, host output out, every step) for the same number of steps.
    Returns the times and the wall-clock windows of the timed and the
    end-to-end loops (for the clock record)."""
    for _ in range(warmup):
        run_step(st)
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    w0 = time.monotonic()
    start.record()
    for _ in range(steps):
        run_step(st)
    end.record()
    barrier()
    w1 = time.monotonic()
    # the per-call breakdown (kernel_ms) from a loop of its own: an event
    # between two launches costs the second its early launch, so the timed
    # loop above carries none
    sampled = sampled_steps(steps)
    evs = {i: tuple(torch.cuda.Event(enable_timing=True) for _ in range(4)) for i in sampled}
    for i in range(steps):
        run_step(st, evs.get(i))
    barrier()
    r = {"ms": start.elapsed_time(end),
         "dec_ms": [ev[2].elapsed_time(ev[3]) for ev in evs.values()],
         "copy_ms": [ev[0].elapsed_time(ev[1]) for ev in evs.values()] if st.pairs.shape[0] else None,
         "write_ms": [ev[1].elapsed_time(ev[2]) for ev in evs.values()] if st.path == "separate" else None,
         "decode_loop_ms": None}
    if not decode_only_step(st):
        # the roofline's duration: the decode call alone, timed over a loop of
        # its own (repeating it reads what the step reads; the cache is as the
        # timed steps left it)
        for _ in range(warmup):
            run_decode(st)
        barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        for _ in range(steps):
            run_decode(st)
        b.record()
        barrier()
        r["decode_loop_ms"] = a.elapsed_time(b)

    # ---- end to end: host inputs in, host output out, every step ------------
    # the step's inputs (q, new K/V, slots, tables, lengths) sit packed in one
    # pinned host buffer and go over in one copy; the output comes back in one.
    # The copies of neighbouring steps overlap the kernels (e2e_steps_pipelined).
    h_out = [torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory() for _ in range(2)]
    r["h2d"] = st.in_host.numel()
    r["d2h"] = h_out[0].numel() * h_out[0].element_size()
    e2e_steps_pipelined(st, max(1, warmup), dev, h_out)
    barrier()
    w2 = time.monotonic()
    e0, e1 = e2e_steps_pipelined(st, steps, dev, h_out)
    barrier()
    w3 = time.monotonic()
    r["e2e_ms"] = e0.elapsed_time(e1)
    r["windows"] = [(w0, w1), (w2, w3)]
    return r


E2E_HOW = ("every step: packed inputs from pinned host memory in one H2D copy, output to pinned host memory in "
           "one D2H copy; two input and output buffers, copies on their own streams overlapping the "
           "neighbouring steps' kernels")

ROOFLINE_KERNEL = {"fused": "paged_attention_decode_mq with fused slot write (partition kernel + split-K reduce)",
                   "shared": "paged_attention_decode_shared with fused slot write "
                             "(group and own passes in one launch + split-K reduce)",
                   "separate": "paged_attention_decode (partition kernel + split-K reduce)"}


def launches_per_step(st) -> int:
    return {"fused": st.launches_fused, "separate": st.launches_separate,
            "shared": getattr(st, "launches_shared", None)}[st.path]


def decode_only_step(st) -> bool:
    """Whether a step is the decode call alone (no copy-on-write pairs, write fused)."""
    return st.path in ("fused", "shared") and st.pairs.shape[0] == 0


def decode_call_ms(st, r, steps: int):
    """Mean duration of the step's decode call, and how it was measured: the
    timed loop's CUDA-event time / steps when the step is the call alone, else
    the same over a loop of the decode call alone run right after it."""
    if decode_only_step(st):
        return r["ms"] / steps, "CUDA events around the timed loop / steps (the step is the decode call alone)"
    return (r["decode_loop_ms"] / steps,
            "CUDA events around a loop of the decode call alone (same steps), after the timed loop")


def roofline_of(st, dec_mean_ms: float, peak: float, peak_kind: str, how: str = "") -> dict:
    """The decode call against the HBM roofline.  achieved = the bytes the
    call must move (each physical block's live K/V tokens once, Q, out,
    tables, lengths, and the fused new K/V in and out) / its mean duration."""
    achieved = st.call_bytes_unique / (dec_mean_ms / 1e3) / 1e9
    logical = st.call_bytes_logical / (dec_mean_ms / 1e3) / 1e9
    return {"kernel": ROOFLINE_KERNEL[st.path], "bound": "hbm", "achieved": achieved, "peak": peak,
            "peak_kind": peak_kind, "unit": "GB/s", "frac": achieved / peak,
            "algorithmic_bytes_per_launch": st.call_bytes_unique,
            "logical_bytes_per_launch": st.call_bytes_logical, "frac_logical": logical / peak,
            "decode_ms_mean": dec_mean_ms, "duration": how}


# The benchmark spec's other configurations, measured after the headline in the
# same run: (key, workload, new tokens per sequence, path, timed steps).
# q_len 16 on the MHA batches is the multi-query (draft verification) shape.
# The headline batch also runs through shared-prefix decode, whose host-built
# work list launches only live (sequence, partition) items, longest first.
ENTRIES = (
    ("8b_gqa_prefix_shared", 4, 1, "shared", 300),
    ("tiny", 1, 1, "separate", 2000),
    ("7b", 2, 1, "fused", 2000),
    ("7b_q16", 2, 16, "fused", 1000),
    ("13b", 3, 1, "fused", 1000),
    ("13b_q16", 3, 16, "fused", 600),
    ("8b_gqa_sampling", 5, 1, "shared", 300),
    ("8b_gqa_sampling_ordinary", 5, 1, "fused", 200),
)


def measure_entry(spec, dev, threads: int, clocks, peak: float, peak_kind: str, barrier, warmup: int = 20,
                  oracle_s: float = 6.0):
    key, number, q_len, path, steps = spec
    st = build_step(number, dev, 0, None, 16, None, q_len, path)
    st.path = path
    torch.cuda.synchronize(dev)
    base = cpu_baseline(st, threads, target_s=oracle_s)   # the oracle's input is taken before any product step
    r = time_step(st, steps, warmup, dev, barrier)
    S = st.w.num_seqs
    dec_mean, how = decode_call_ms(st, r, steps)
    entry = {
        "workload": WORKLOAD_NAMES[number], "num_seqs": S, "num_q_heads": st.w.num_q_heads,
        "num_kv_heads": st.w.num_kv_heads, "head_dim": st.w.head_dim, "q_len": q_len, "path": path,
        "dtype": str(st.w.dtype).replace("torch.", ""), "context_tokens": int(st.lens_host.sum()),
        "partition_tokens": st.part_tokens, "steps": steps, "warmup": warmup,
        "value": st.kv_bytes * steps / (r["ms"] / 1e3) / 1e9, "unit": "GB/s",
        "ms_per_step": r["ms"] / steps,
        "seq_steps_per_s": S * steps / (r["ms"] / 1e3),
        "new_tokens_per_s": S * q_len * steps / (r["ms"] / 1e3),
        "kv_bytes_logical": st.kv_bytes, "kv_bytes_unique": st.kv_unique_bytes,
        "e2e": {"value": st.kv_bytes * steps / (r["e2e_ms"] / 1e3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"], "ms_per_step": r["e2e_ms"] / steps},
        "roofline": roofline_of(st, dec_mean, peak, peak_kind, how),
        "parity": parity_on_sample(st, base),
        "clocks": clocks.summary(r["windows"], "this entry's timed and end-to-end loops"),
        "gpu_launches": launches_per_step(st) * steps,
        "l2": f"{st.kv_unique_bytes / 1e6:.0f} MB of unique K/V per step vs 126 MB of L2, no flush",
    }
    if st.plan is not None:
        entry["shared_prefix"] = {"groups": int(st.plan.groups.shape[0]), "work_items": int(st.plan.work.shape[0]),
                                  "host_plan_us_steady": st.host_plan_us_steady,
                                  "plan": "built on the host from the step's tables and lengths, outside the timed "
                                          "region like the tables themselves"}
    del st
    torch.cuda.empty_cache()
    return entry


def run_ours(args):
    import paged_kv_cache_398_b200 as pkv  # noqa: F401  (loads the library before any timing)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=dev)

    def barrier():
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize(dev)

    st = build_step(args.workload, dev, rank, args.num_seqs, args.block_size, args.max_ctx, args.q_len, args.path)
    st.path = args.path
    torch.cuda.synchronize(dev)
    threads = cpu_threads()
    # the oracle sample is copied off the device before the first product step
    base = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        base = cpu_baseline(st, threads)

    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.05)
    r = time_step(st, args.steps, args.warmup, dev, barrier)
    ms, e2e_ms = r["ms"], r["e2e_ms"]
    swap = measure_swap(st, dev) if not args.no_swap else None

    ms_max, e2e_max, kv_total, uniq_total = reduce_over_ranks(
        dist, dev, [ms, e2e_ms], [float(st.kv_bytes), float(st.kv_unique_bytes)])
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        clocks.stop()
        return 0

    peak, peak_kind = hbm_peak()
    entries = None
    if world == 1 and not args.no_workloads:
        entries = {spec[0]: measure_entry(spec, dev, threads, clocks, peak, peak_kind, barrier)
                   for spec in ENTRIES}
    clocks.stop()

    S = st.w.num_seqs
    value = kv_total * args.steps / (ms_max / 1e3) / 1e9
    dec_mean, how = decode_call_ms(st, r, args.steps)
    roof = roofline_of(st, dec_mean, peak, peak_kind, how)
    roof["traffic"] = recorded_traffic(WORKLOAD_NAMES[args.workload], S, st.path, st.w.block_size, st.q_len)
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": str(st.w.dtype).replace("torch.", ""),
        "data": "synthetic",
        "config": {"workload": WORKLOAD_NAMES[args.workload], "num_seqs": S,
                   "num_q_heads": st.w.num_q_heads, "num_kv_heads": st.w.num_kv_heads,
                   "head_dim": st.w.head_dim, "block_size": st.w.block_size,
                   "context_tokens": int(st.lens_host.sum()), "max_context_len": st.max_ctx,
                   "partition_tokens": st.part_tokens, "q_len": st.q_len,
                   "l2": f"inputs larger than L2 ({st.kv_bytes / 1e9:.2f} GB of K/V per step), no flush",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "pct_of_hbm_peak": 100.0 * value / peak,
        "pct_of_nominal_hbm": 100.0 * value / NOMINAL_HBM_GBS,
        "seq_steps_per_s": S * world * args.steps / (ms_max / 1e3),
        "new_tokens_per_s": S * st.q_len * world * args.steps / (ms_max / 1e3),
        "unique_kv_gbps": uniq_total * args.steps / (ms_max / 1e3) / 1e9,
        "kernel_ms": {"decode_mean": statistics.mean(r["dec_ms"]), "decode_min": min(r["dec_ms"]),
                      "kv_write_mean": statistics.mean(r["write_ms"]) if r["write_ms"] else None,
                      "block_copy_mean": statistics.mean(r["copy_ms"]) if r["copy_ms"] else None,
                      "sampled_steps": len(r["dec_ms"]),
                      "how": "CUDA events around each call on its stream, in evenly spread steps of a loop "
                             "run after the timed one"},
        "roofline": roof,
        "cpu_baseline": ({k: v for k, v in base.items() if k in ("value", "unit", "cores", "kind", "sample")}
                         if base else None),
        "parity": parity_on_sample(st, base) if base else None,
        "e2e": {"value": kv_total * args.steps / (e2e_max / 1e3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": r["h2d"], "d2h_bytes_per_step": r["d2h"],
                "ms_per_step": e2e_max / args.steps, "how": E2E_HOW},
        "gpu_launches": launches_per_step(st) * args.steps,
        "path": st.path,
        "host_alloc_us_per_step": st.host_alloc_us,
        "host_alloc_us_per_step_steady": st.host_step_us,
        "shared_prefix": (None if st.plan is None else
                          {"groups": int(st.plan.groups.shape[0]), "work_items": int(st.plan.work.shape[0]),
                           "max_shared_len": st.plan.max_shared_len,
                           "max_own_len": st.plan.max_own_len, "host_plan_us": st.host_plan_us,
                           "host_plan_us_steady": st.host_plan_us_steady}),
        "prefix_cache": (None if st.prefix is None else
                         {"admit_us_per_request": st.admit_us_per_request, "hit_tokens": st.prefix["hit_tokens"],
                          "blocks_shared": st.prefix["hit_tokens"] // st.w.block_size,
                          "cached_blocks": st.prefix["cached_blocks"]}),
        "clocks": clocks.summary(r["windows"], "the timed loop and the end-to-end loop"),
        "swap": swap,
        "fragmentation": fragmentation_report(st.lens_host),
        "workloads": entries,
        "wall_s_timed": r["windows"][0][1] - r["windows"][0][0],
    }
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=4, choices=sorted(WORKLOAD_NAMES))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-swap", action="store_true", help="skip the swap-out / swap-in measurement")
    ap.add_argument("--no-workloads", action="store_true",
                    help="skip the other configurations (the line's workloads object)")
    ap.add_argument("--block-size", type=int, default=16, choices=[8, 16, 32],
                    help="tokens per block (the pages use 16)")
    ap.add_argument("--path", choices=["fused", "separate", "shared"], default="fused",
                    help="fused: slot write inside the decode launch; separate: paged_kv_write then decode; "
                         "shared: fused, reading the blocks a group of samples shares once per step")
    ap.add_argument("--reference-seqs", type=int, default=16)
    ap.add_argument("--num-seqs", type=int, default=None,
                    help="smaller batch of the same recipe (profiling); the default is the full workload")
    ap.add_argument("--q-len", type=int, default=1,
                    help="new tokens per sequence (multi-query decode, e.g. draft tokens to verify; workloads 2-4)")
    ap.add_argument("--max-ctx", type=int, default=None,
                    help="shorter contexts of the same recipe (profiling; workloads 2-4)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
