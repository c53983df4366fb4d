"""Synthetic continuous-batching traces driven through the host runtime.

Each builder returns a ``Trace``: a scheduler in its start state plus the
per-step workload actions, seeded and deterministic.  ``Trace.plans(n)``
runs the scheduler for n steps (host only) and returns the StepPlans the
kernels execute; the caller runs them in order.

* ``batch64_2k``: 64 running sequences, lengths uniform in [1, 2048], 32/8
  heads, head_dim 128, bf16; each sequence stops after Geometric(1/256) decode
  steps and is replaced from a queue whose prompt lengths are uniform in
  [1, 2048] (their K/V are written in the step they are admitted; prefill
  attention is not part of this workload).  Pool = ceil(1.1 x blocks needed at
  step 0), handed out from a seeded permutation.
* ``prefix_share_fp8``: 256 running sequences that share one 2048-token
  prefix (the same physical blocks) plus suffixes uniform in [16, 512], 64/8
  heads, fp8 cache; every step retires 32 random sequences and forks 32 from
  random survivors, so shared partly-filled blocks are copied on the first
  divergent write.
* ``long_context``: 16 sequences of 32768 tokens, 32/8 heads, bf16, blocks
  scattered over a 40960-block pool; every step decodes one more token of
  each (split-K over many partitions).
* ``mixed``: chunked prefill interleaved with decode under token budget
  8192.  Step 0 is 192 decode sequences with lognormal lengths (median 1024,
  sigma 1, capped at 8192) plus 8 prompts in prefill whose next 512-token
  chunk attends a cached prefix uniform in [0, 4096]; 32/8 heads, head_dim
  128, bf16.  Decode sequences stop after Geometric(1/256) steps; a prompt
  that finishes its prefill joins the decode batch; new prompts (U[512, 4608]
  tokens) arrive so that 8 prompts are always in prefill, each advancing by
  one chunk of at most 512 tokens per step.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

from . import inputs as I
from .runtime import BlockAllocator, Scheduler, SchedulerConfig, Sequence, blocks_for


@dataclass
class Trace:
    name: str
    sched: Scheduler
    Hq: int
    Hkv: int
    D: int
    fp8: bool
    rng: np.random.Generator
    before_step: object = None  # callable(trace) run before each scheduler step
    next_id: int = 0
    info: dict = field(default_factory=dict)

    def plans(self, n):
        out = []
        for _ in range(n):
            if self.before_step is not None:
                self.before_step(self)
            plan = self.sched.step()
            out.append(plan)
            self.sched.complete(plan)
        return out

    def new_id(self):
        self.next_id += 1
        return self.next_id - 1


def _refill_queue(tr: Trace, depth=16, lo=1, hi=2048, p=1.0 / 256):
    while len(tr.sched.waiting) < depth:
        L = int(tr.rng.integers(lo, hi + 1))
        tr.sched.add_request(Sequence(tr.new_id(), L, int(tr.rng.geometric(p))))


def batch64_2k(seed=0, max_steps=10_000) -> Trace:
    rng = np.random.default_rng(40_000 + seed)
    n, p = 64, 1.0 / 256
    lens = rng.integers(1, 2049, n)  # decode-step lengths (incl. the step's own token)
    need = int(sum(blocks_for(int(L)) for L in lens))
    pool = int(math.ceil(1.1 * need))
    alloc = BlockAllocator(pool, order=rng.permutation(pool))
    # tables wide enough for the longest possible sequence over the trace
    cfg = SchedulerConfig(max_num_seqs=n, max_num_batched_tokens=8192, max_chunk=8192,
                          max_blocks_per_seq=blocks_for(2048 + max_steps))
    sched = Scheduler(alloc, cfg)
    tr = Trace("64 seqs x U[1,2048], 32/8 heads, d128, bf16", sched, 32, 8, 128, False, rng,
               before_step=lambda t: _refill_queue(t, 16, 1, 2048, p))
    for L in lens:
        sched.restore(tr.new_id(), int(L) - 1, int(rng.geometric(p)))
    tr.info["pool_blocks"] = pool
    return tr


def prefix_share_fp8(seed=0, n=256, forks=32, prefix=2048) -> Trace:
    rng = np.random.default_rng(50_000 + seed)
    suf = rng.integers(16, 513, n)
    need = blocks_for(prefix) + int(sum(blocks_for(prefix + int(s)) - blocks_for(prefix) for s in suf))
    pool = int(math.ceil(1.25 * need)) + 4 * forks
    alloc = BlockAllocator(pool, order=rng.permutation(pool))
    cfg = SchedulerConfig(max_num_seqs=n + forks, max_num_batched_tokens=8192,
                          max_blocks_per_seq=blocks_for(prefix + 512 + 4096))
    sched = Scheduler(alloc, cfg)
    tr = Trace("256 seqs sharing a 2048-token prefix, 64/8 heads, d128, fp8", sched, 64, 8, 128, True, rng)
    root = sched.restore(tr.new_id(), prefix, 10 ** 9)
    # every sequence shares the prefix blocks, then owns its suffix blocks
    for s in suf:
        child = sched.fork(root, tr.new_id(), 10 ** 9)
        for k in range(int(s) - 1):
            sched.kv.slot_for(child, child.num_cached)
            child.num_cached += 1
            child.prefill_end = child.num_cached
            child.num_tokens = child.num_cached + 1
    sched.kv.take_copies()  # set-up copies (none: the prefix is block-aligned)
    sched.retire(root)

    def churn(t: Trace):
        running = list(t.sched.running)
        for s in t.rng.choice(len(running), forks, replace=False):
            t.sched.retire(running[int(s)])
        parents = [t.sched.running[int(i)] for i in t.rng.choice(len(t.sched.running), forks, replace=False)]
        for par in parents:
            t.sched.fork(par, t.new_id(), 10 ** 9)

    tr.before_step = churn
    tr.info["pool_blocks"] = pool
    tr.info["shared_prefix_blocks"] = blocks_for(prefix)
    return tr


def _keep_prompts_in_prefill(tr: Trace, n_prompts, chunk, p):
    """New prompts arrive so that n_prompts are in prefill (running or
    waiting): U[chunk, 4096 + chunk] tokens each, then Geometric(p) decode
    steps."""
    busy = sum(1 for s in tr.sched.running if s.in_prefill) + len(tr.sched.waiting)
    for _ in range(n_prompts - busy):
        L = int(tr.rng.integers(chunk, 4096 + chunk + 1))
        tr.sched.add_request(Sequence(tr.new_id(), L, int(tr.rng.geometric(p))))


def mixed(seed=0, n_decode=192, chunk=512, n_prompts=8, headroom_steps=48, p=1.0 / 256) -> Trace:
    rng = np.random.default_rng(60_000 + seed)
    lens = I.lognormal_lengths(rng, n_decode)        # decode-step lengths (incl. the step's own token)
    prefixes = rng.integers(0, 4097, n_prompts)      # cached part of each prompt in prefill
    togo = chunk * rng.integers(1, 5, n_prompts)     # its chunks still to run (1..4 of 512)
    need = int(sum(blocks_for(int(L)) for L in lens)) + int(sum(blocks_for(int(a + b))
                                                                 for a, b in zip(prefixes, togo)))
    # room for the prompts of headroom_steps steps (about n_prompts*chunk tokens a step) on top of 1.1x
    pool = int(math.ceil(1.1 * need)) + blocks_for(headroom_steps * n_prompts * chunk)
    alloc = BlockAllocator(pool, order=rng.permutation(pool))
    cfg = SchedulerConfig(max_num_seqs=n_decode + 8 * n_prompts, max_num_batched_tokens=8192, max_chunk=chunk,
                          max_blocks_per_seq=blocks_for(8192 + 4096 + chunk))
    sched = Scheduler(alloc, cfg)
    tr = Trace(f"{n_decode} decode seqs (lognormal, median 1024, cap 8192) + {n_prompts} prefill chunks x "
               f"{chunk} over U[0,4096] prefixes, budget 8192, 32/8 heads, d128, bf16", sched, 32, 8, 128, False, rng,
               before_step=lambda t: _keep_prompts_in_prefill(t, n_prompts, chunk, p))
    for L in lens:
        sched.restore(tr.new_id(), int(L) - 1, int(rng.geometric(p)))
    for a, b in zip(prefixes, togo):
        # a prompt part-way through its prefill: a cached prefix, chunks to go
        s = Sequence(tr.new_id(), int(a + b), int(rng.geometric(p)), num_cached=int(a), prefill_end=int(a + b))
        for _ in range(blocks_for(int(a))):
            s.block_table.append(alloc.alloc())
        sched.add_running(s)
    tr.info["pool_blocks"] = pool
    return tr


def long_context(seed=0, n=16, seq_len=32768, pool=40960) -> Trace:
    rng = np.random.default_rng(70_000 + seed)
    alloc = BlockAllocator(pool, order=rng.permutation(pool))
    cfg = SchedulerConfig(max_num_seqs=n, max_num_batched_tokens=8192,
                          max_blocks_per_seq=blocks_for(seq_len + 1024))
    sched = Scheduler(alloc, cfg)
    tr = Trace(f"{n} seqs x {seq_len}, 32/8 heads, d128, bf16", sched, 32, 8, 128, False, rng)
    for _ in range(n):
        sched.restore(tr.new_id(), seq_len - 1, 10 ** 9)
    tr.info["pool_blocks"] = pool
    return tr
