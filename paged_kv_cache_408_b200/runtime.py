"""Host runtime: refcounted block allocator and iteration-level scheduler.

Sources (by page and section):

* "Production Serving: Continuous Batching and PagedAttention", The Build,
  Step 4 "Implement the paged KV cache" -- one pool of fixed 16-token pages,
  a LIFO free list, a page table per sequence, a new page exactly when the
  stored length is a multiple of 16, every page returned when the sequence
  ends, an error when the free list is empty.
* same page, Step 2 "Build the continuous batcher" and "Continuous batching,
  the thing you actually want" -- every step retires finished requests and
  admits waiting ones; the batch membership changes at every step.
* same page, "The two ideas together" -- admission control (admit only when
  pages are available) and preemption (evict someone when memory runs out).
* "Continuous batching and PagedAttention", How the scheduler works -- each
  step schedules the decoding conversations first and fills the remaining
  token budget with prefill chunks; PagedAttention: KV cache memory -- blocks
  are shared copy-on-write; running out mid-generation preempts a
  conversation whose cache is later recomputed.
* same page, What it means in production -- max_num_seqs and
  max_num_batched_tokens bound the batch.
* "Production Serving: Continuous Batching and PagedAttention", The Build,
  Step 8 "Prefix caching" -- a cache from full-page token prefixes to the
  pages that hold them; a new prompt looks up its longest cached full-page
  prefix, shares those pages (refcount + 1) and only computes the rest.

Readings where the pages are silent: the preempted sequence is the most
recently admitted running one; admission needs the blocks of the request's
whole prompt plus a watermark of 1% of the pool; a fork shares every block of
its parent, including a partly filled last block, and the first write into a
block with refcount > 1 copies it (the copy is emitted as a (src, dst) pair
for ``pa_copy_blocks``, which must run before the step's writes).

Everything here is integer bookkeeping on the host; the step it produces is a
``StepPlan`` of numpy arrays that the caller uploads and hands to the
kernels.
"""
from __future__ import annotations

import math
from collections import OrderedDict, deque
from dataclasses import dataclass, field

import numpy as np

BLOCK_SIZE = 16


class OutOfBlocksError(RuntimeError):
    """The free list is empty (the pages' OutOfPagesError)."""


# --------------------------------------------------------------- allocator
class BlockAllocator:
    """Pool of ``num_blocks`` physical blocks with a LIFO free list and
    reference counts.  ``order`` is the initial free list (bottom first); the
    pages use ``range(num_blocks)``, so ``alloc`` pops the highest id first."""

    def __init__(self, num_blocks: int, order=None):
        self.num_blocks = int(num_blocks)
        self.free_list = list(range(self.num_blocks)) if order is None else [int(b) for b in order]
        if sorted(self.free_list) != list(range(self.num_blocks)):
            raise ValueError("order must be a permutation of the pool")
        self.ref = np.zeros(self.num_blocks, np.int32)
        self.copies_emitted = 0
        self.cache: PrefixCache | None = None  # attached by PrefixCache

    @property
    def num_free(self) -> int:
        """Blocks an allocation can take: the free list plus cached blocks
        that no sequence holds (evicted on demand)."""
        return len(self.free_list) + (self.cache.num_evictable if self.cache else 0)

    def alloc(self) -> int:
        if self.free_list:
            b = self.free_list.pop()
        elif self.cache is not None and self.cache.num_evictable:
            b = self.cache.evict()
        else:
            raise OutOfBlocksError()
        self.ref[b] = 1
        return b

    def incref(self, b: int) -> None:
        if self.ref[b] <= 0:
            raise RuntimeError(f"incref of free block {b}")
        self.ref[b] += 1

    def decref(self, b: int) -> None:
        if self.ref[b] <= 0:
            raise RuntimeError(f"decref of free block {b}")
        self.ref[b] -= 1
        if self.ref[b] == 0:
            if self.cache is not None and self.cache.holds(b):
                self.cache.park(b)  # stays cached until a lookup revives it or space is needed
            else:
                self.free_list.append(b)


# ------------------------------------------------------------ prefix cache
class PrefixCache:
    """Full-block token prefixes -> physical blocks ("Production Serving:
    Continuous Batching and PagedAttention", Step 8 "Prefix caching").

    The pages key a dict by the token tuple of every full-page prefix.  Here
    the key of block i of a prompt is (block holding tokens [0, 16 i) -- or
    -1 for i = 0 --, the 16 token ids of block i): the same identity, since
    the parent block stands for its whole prefix, without keys that grow with
    the prefix.  A lookup walks the prompt block by block from the start and
    returns the longest cached full-block prefix; its blocks are shared
    (refcount + 1).

    A cached block that no sequence holds any more is not freed: it waits in
    LRU order (least recently released first) for a lookup to revive it, and
    is evicted -- key removed, together with every cached block below it,
    whose key names it -- only when an allocation finds the free list empty.
    Sequences release their blocks last-to-first, so a prefix's deepest
    blocks are evicted first.
    """

    def __init__(self, allocator: BlockAllocator):
        self.alloc = allocator
        allocator.cache = self
        self.block_of: dict[tuple, int] = {}   # key -> block
        self.key_of: dict[int, tuple] = {}     # block -> key
        self.children: dict[int, set] = {}    # block -> cached blocks keyed under it
        self.lru: OrderedDict[int, None] = OrderedDict()  # cached, refcount 0
        self.hits = 0      # blocks shared by lookups
        self.evictions = 0

    @property
    def num_evictable(self) -> int:
        return len(self.lru)

    def holds(self, b: int) -> bool:
        return b in self.key_of

    def park(self, b: int) -> None:
        self.lru[b] = None

    def _keys(self, tokens):
        tokens = np.asarray(tokens)
        for i in range(len(tokens) // BLOCK_SIZE):
            yield tuple(int(t) for t in tokens[i * BLOCK_SIZE:(i + 1) * BLOCK_SIZE])

    def peek(self, tokens) -> int:
        """Blocks a lookup of ``tokens`` would share (no side effects)."""
        parent, n = -1, 0
        for blk in self._keys(tokens):
            b = self.block_of.get((parent, blk))
            if b is None:
                break
            parent, n = b, n + 1
        return n

    def match(self, tokens) -> tuple[int, list]:
        """Longest cached full-block prefix of ``tokens``: (tokens covered,
        blocks), each block's refcount incremented (revived if parked)."""
        blocks, parent = [], -1
        for blk in self._keys(tokens):
            b = self.block_of.get((parent, blk))
            if b is None:
                break
            blocks.append(b)
            parent = b
        for b in blocks:
            if self.alloc.ref[b] == 0:
                del self.lru[b]
                self.alloc.ref[b] = 1
            else:
                self.alloc.incref(b)
        self.hits += len(blocks)
        return BLOCK_SIZE * len(blocks), blocks

    def insert(self, tokens, block_table) -> None:
        """Register the full blocks of a computed prompt: ``tokens`` are the
        positions whose K/V are in ``block_table``'s blocks."""
        parent = -1
        for i, blk in enumerate(self._keys(tokens)):
            key = (parent, blk)
            b = self.block_of.get(key)
            if b is None:
                b = int(block_table[i])
                if b in self.key_of:  # this block already caches another prefix
                    return
                self.block_of[key] = b
                self.key_of[b] = key
                if parent >= 0:
                    self.children.setdefault(parent, set()).add(b)
            parent = b

    def _forget(self, b: int) -> None:
        """Drop b's key and, recursively, the keys of the blocks under it;
        those of them that no sequence holds go back to the free list."""
        for c in self.children.pop(b, ()):
            self._forget(c)
            if c in self.lru:
                del self.lru[c]
                self.alloc.free_list.append(c)
        key = self.key_of.pop(b)
        del self.block_of[key]
        if key[0] >= 0 and key[0] in self.children:
            self.children[key[0]].discard(b)

    def evict(self) -> int:
        """Take the least recently released cached block for a new use."""
        b, _ = self.lru.popitem(last=False)
        self._forget(b)
        self.evictions += 1
        return b


# ---------------------------------------------------------------- sequences
WAITING, RUNNING, FINISHED = "waiting", "running", "finished"


@dataclass
class Sequence:
    """A request as the scheduler sees it (the pages' Request record, with
    token ids replaced by counts).

    num_tokens   tokens known so far (prompt + sampled);
    num_cached   positions whose K/V are in the cache;
    prefill_end  positions that must be cached before decoding resumes;
    decode_left  decode steps still to run (a synthetic stop length);
    """
    seq_id: int
    num_tokens: int
    decode_left: int
    num_cached: int = 0
    prefill_end: int = 0
    fresh: bool = True  # prefill of a new prompt (samples a token when done)
    block_table: list = field(default_factory=list)
    status: str = WAITING
    admitted_at: int = -1
    preemptions: int = 0
    tokens: np.ndarray | None = None  # prompt token ids (needed only for prefix caching)

    @property
    def in_prefill(self) -> bool:
        return self.num_cached < self.prefill_end


def blocks_for(n_tokens: int) -> int:
    return (n_tokens + BLOCK_SIZE - 1) // BLOCK_SIZE


class KVManager:
    """Per-sequence block tables on top of a BlockAllocator: slot assignment
    with copy-on-write, forks and release."""

    def __init__(self, allocator: BlockAllocator):
        self.alloc = allocator
        self.pending_copies: list[tuple[int, int]] = []

    def slot_for(self, seq: Sequence, pos: int) -> int:
        """Slot of position ``pos`` (must be seq.num_cached + k for the
        positions being written this step, in order); allocates a block when
        ``pos`` starts one and copies a shared block before writing into it."""
        j, off = divmod(pos, BLOCK_SIZE)
        if j == len(seq.block_table):
            if off != 0:
                raise RuntimeError("positions must be written in order")
            seq.block_table.append(self.alloc.alloc())
        elif j > len(seq.block_table):
            raise RuntimeError("positions must be written in order")
        b = seq.block_table[j]
        if self.alloc.ref[b] > 1:  # shared: copy before the first divergent write
            d = self.alloc.alloc()
            self.pending_copies.append((b, d))
            self.alloc.copies_emitted += 1
            self.alloc.decref(b)
            seq.block_table[j] = d
            b = d
        return b * BLOCK_SIZE + off

    def fork(self, parent: Sequence, seq_id: int, decode_left: int) -> Sequence:
        child = Sequence(seq_id, parent.num_tokens, decode_left, parent.num_cached, parent.prefill_end,
                         parent.fresh, list(parent.block_table), parent.status)
        for b in child.block_table:
            self.alloc.incref(b)
        return child

    def release(self, seq: Sequence) -> None:
        # table order, as the pages return pages; with a prefix cache, deepest
        # first, so that its LRU evicts a prefix's leaves before its root
        order = seq.block_table if self.alloc.cache is None else reversed(seq.block_table)
        for b in order:
            self.alloc.decref(b)
        seq.block_table = []

    def take_copies(self) -> np.ndarray:
        c = np.array(self.pending_copies, np.int32).reshape(-1, 2)
        self.pending_copies = []
        return c


# ----------------------------------------------------------------- the step
@dataclass
class StepPlan:
    """Metadata of one step, ready for upload.  New tokens are ordered
    decode tokens first, then prefill chunks in order."""
    step: int
    copies: np.ndarray            # int32 [n, 2] (src, dst): run before the writes
    slots: np.ndarray             # int64 [T] slot of every new token
    decode_ids: np.ndarray        # int64 [nd]
    decode_tables: np.ndarray     # int32 [nd, max_blocks] (-1 padded)
    decode_lens: np.ndarray       # int32 [nd] (including this step's token)
    prefill_ids: np.ndarray       # int64 [nc]
    prefill_cu: np.ndarray        # int32 [nc+1]
    prefill_prefix: np.ndarray    # int32 [nc]
    prefill_tables: np.ndarray    # int32 [nc, max_blocks]
    preempted: list = field(default_factory=list)
    admitted: list = field(default_factory=list)
    retired: list = field(default_factory=list)

    @property
    def num_decode(self) -> int:
        return len(self.decode_ids)

    @property
    def num_prefill_tokens(self) -> int:
        return int(self.prefill_cu[-1]) if len(self.prefill_cu) else 0

    @property
    def max_chunk(self) -> int:
        return int(np.diff(self.prefill_cu).max(initial=0))

    @property
    def shared_decode_blocks(self) -> int:
        """Leading block-table entries that every decode sequence shares (the
        same physical blocks, e.g. a forked prompt) and fills completely:
        the prefix a cascade decode attends once for the whole batch."""
        t = self.decode_tables
        if len(t) == 0:
            return 0
        same = (t == t[0]).all(axis=0)
        n = int(np.argmin(same)) if not same.all() else t.shape[1]
        return min(n, int(self.decode_lens.min()) // BLOCK_SIZE)


@dataclass
class SchedulerConfig:
    max_num_seqs: int = 256
    max_num_batched_tokens: int = 8192
    max_chunk: int = 8192          # longest prefill chunk
    max_blocks_per_seq: int = 512  # width of the uploaded block tables
    watermark: float = 0.01        # fraction of the pool kept free at admission
    prefix_cache: bool = False     # share cached full-block prompt prefixes


class Scheduler:
    """Iteration-level scheduler.  ``step()`` plans one step; the caller runs
    the kernels and then calls ``complete(plan)``."""

    def __init__(self, allocator: BlockAllocator, cfg: SchedulerConfig | None = None):
        self.cfg = cfg or SchedulerConfig()
        self.kv = KVManager(allocator)
        self.alloc = allocator
        self.waiting: deque[Sequence] = deque()
        self.running: list[Sequence] = []
        self.finished: list[Sequence] = []
        self.step_no = 0
        self.admit_counter = 0
        self.num_preemptions = 0
        self.watermark_blocks = int(math.ceil(self.cfg.watermark * allocator.num_blocks))
        self.cache = PrefixCache(allocator) if self.cfg.prefix_cache else None

    # -- requests
    def add_request(self, seq: Sequence) -> None:
        if blocks_for(seq.num_tokens) > self.cfg.max_blocks_per_seq:
            raise ValueError(f"request {seq.seq_id}: {seq.num_tokens} tokens exceed the "
                             f"{self.cfg.max_blocks_per_seq}-block table")
        seq.status = WAITING
        if seq.prefill_end == 0 and seq.fresh:
            seq.prefill_end = seq.num_tokens
        self.waiting.append(seq)

    def restore(self, seq_id: int, cached_tokens: int, decode_left: int) -> Sequence:
        """Register a sequence that is mid-generation: ``cached_tokens``
        positions already in the cache (blocks allocated here), its next
        decode step writes position ``cached_tokens``."""
        s = Sequence(seq_id, cached_tokens + 1, decode_left, cached_tokens, cached_tokens, False)
        for _ in range(blocks_for(cached_tokens)):
            s.block_table.append(self.alloc.alloc())
        self.add_running(s)
        return s

    def add_running(self, seq: Sequence) -> None:
        """Register a sequence whose blocks are already allocated (a fork, or
        a sequence restored at start-up)."""
        seq.status = RUNNING
        seq.admitted_at = self.admit_counter
        self.admit_counter += 1
        self.running.append(seq)

    def fork(self, parent: Sequence, seq_id: int, decode_left: int) -> Sequence:
        child = self.kv.fork(parent, seq_id, decode_left)
        self.add_running(child)
        return child

    def retire(self, seq: Sequence) -> None:
        if seq.status == RUNNING:
            self.running.remove(seq)
        elif seq.status == WAITING:
            self.waiting.remove(seq)
        self.kv.release(seq)
        seq.status = FINISHED
        self.finished.append(seq)

    # -- policy pieces
    def _preempt_one(self, plan: StepPlan) -> Sequence | None:
        """Evict the most recently admitted running sequence (recompute)."""
        if not self.running:
            return None
        victim = max(self.running, key=lambda s: s.admitted_at)
        self.running.remove(victim)
        self.kv.release(victim)
        victim.prefill_end = victim.num_cached if not victim.in_prefill else victim.prefill_end
        victim.num_cached = 0
        victim.status = WAITING
        victim.preemptions += 1
        self.num_preemptions += 1
        self.waiting.appendleft(victim)
        plan.preempted.append(victim.seq_id)
        return victim

    def _lookup_tokens(self, seq: Sequence):
        """Prompt positions a prefix-cache lookup may cover: all but the last
        one, which must be computed to continue the sequence."""
        if self.cache is None or seq.tokens is None or seq.num_cached or seq.block_table:
            return None
        return np.asarray(seq.tokens)[:max(0, seq.prefill_end - 1)]

    def _can_admit(self, seq: Sequence) -> bool:
        need = blocks_for(seq.prefill_end)
        toks = self._lookup_tokens(seq)
        if toks is not None:
            need -= self.cache.peek(toks)  # shared blocks are not allocated
        return self.alloc.num_free >= need + self.watermark_blocks

    def _table(self, seqs) -> np.ndarray:
        mb = self.cfg.max_blocks_per_seq
        t = np.full((len(seqs), mb), -1, np.int32)
        for i, s in enumerate(seqs):
            if len(s.block_table) > mb:
                raise RuntimeError(f"sequence {s.seq_id} needs {len(s.block_table)} blocks > {mb}")
            t[i, :len(s.block_table)] = s.block_table
        return t

    # -- one step
    def step(self) -> StepPlan:
        plan = StepPlan(self.step_no, None, None, None, None, None, None, None, None, None)
        # 1. retire finished sequences
        for s in [s for s in self.running if s.decode_left <= 0 and not s.in_prefill]:
            self.retire(s)
            plan.retired.append(s.seq_id)
        # 2. decode first: one new token per decoding sequence
        decode: list[Sequence] = []
        slots: list[int] = []
        for s in sorted([s for s in self.running if not s.in_prefill], key=lambda s: s.admitted_at):
            if s.status != RUNNING:
                continue  # preempted while making room for an earlier one
            while True:
                try:
                    slot = self.kv.slot_for(s, s.num_cached)
                    break
                except OutOfBlocksError:
                    victim = self._preempt_one(plan)
                    if victim is None or victim is s:
                        slot = None
                        break
            if slot is None:
                continue
            decode.append(s)
            slots.append(slot)
        budget = self.cfg.max_num_batched_tokens - len(decode)
        # 3. fill the rest of the budget with prefill chunks: running first, then admissions
        chunks: list[tuple[Sequence, int, int]] = []
        for s in sorted([s for s in self.running if s.in_prefill], key=lambda s: s.admitted_at):
            if budget <= 0:
                break
            n = min(budget, s.prefill_end - s.num_cached, self.cfg.max_chunk)
            got = self._chunk_slots(s, n, slots, plan)
            if got:
                chunks.append((s, s.num_cached, got))
                budget -= got
        while budget > 0 and self.waiting and len(self.running) < self.cfg.max_num_seqs:
            s = self.waiting[0]
            if s.seq_id in plan.preempted or not self._can_admit(s):
                break  # a sequence evicted in this step waits at least one step
            self.waiting.popleft()
            toks = self._lookup_tokens(s)
            if toks is not None:
                s.num_cached, s.block_table = self.cache.match(toks)
            self.add_running(s)
            plan.admitted.append(s.seq_id)
            n = min(budget, s.prefill_end - s.num_cached, self.cfg.max_chunk)
            got = self._chunk_slots(s, n, slots, plan)
            if got:
                chunks.append((s, s.num_cached, got))
                budget -= got
        # 4. metadata
        plan.copies = self.kv.take_copies()
        plan.slots = np.array(slots, np.int64)
        plan.decode_ids = np.array([s.seq_id for s in decode], np.int64)
        plan.decode_tables = self._table(decode)
        plan.decode_lens = np.array([s.num_cached + 1 for s in decode], np.int32)
        plan.prefill_ids = np.array([s.seq_id for s, _, _ in chunks], np.int64)
        cu = np.zeros(len(chunks) + 1, np.int32)
        cu[1:] = np.cumsum([n for _, _, n in chunks]) if chunks else []
        plan.prefill_cu = cu
        plan.prefill_prefix = np.array([p for _, p, _ in chunks], np.int32)
        plan.prefill_tables = self._table([s for s, _, _ in chunks])
        self._inflight = (decode, chunks)
        return plan

    def _chunk_slots(self, s: Sequence, n: int, slots: list, plan: StepPlan) -> int:
        """Slots for positions num_cached .. num_cached+n-1 of s.  Prefill
        never preempts: when the pool runs dry the chunk is cut short and
        resumes next step (decodes keep priority)."""
        got = 0
        for k in range(n):
            try:
                slots.append(self.kv.slot_for(s, s.num_cached + k))
            except OutOfBlocksError:
                break
            got += 1
        return got

    def complete(self, plan: StepPlan) -> None:
        """Advance the sequences of the step the caller has just run."""
        decode, chunks = self._inflight
        cap = BLOCK_SIZE * self.cfg.max_blocks_per_seq
        for s in decode:
            if s.status != RUNNING:
                continue
            s.num_cached += 1
            s.prefill_end = s.num_cached
            s.num_tokens = s.num_cached + 1
            s.decode_left -= 1
            if s.num_cached >= cap:  # the block table is full: the sequence ends here
                s.decode_left = 0
        for s, start, n in chunks:
            if s.status != RUNNING:
                continue
            s.num_cached = start + n
            if s.num_cached >= s.prefill_end and s.fresh:
                s.fresh = False
                s.num_tokens = s.num_cached + 1  # the prompt's last position samples a token
                if self.cache is not None and s.tokens is not None:
                    self.cache.insert(np.asarray(s.tokens)[:s.num_cached], s.block_table)
        self.step_no += 1

    # -- accounting
    def kv_accounting(self) -> dict:
        """Cached tokens of the running sequences (each sequence counted in
        full) against the distinct blocks they hold: below 1 by the paging
        waste (under one block per sequence), above 1 where blocks are shared
        (forks, cached prefixes)."""
        held = set()
        stored = 0
        for s in self.running:
            held.update(s.block_table)
            stored += s.num_cached
        return {"sequences": len(self.running), "cached_tokens": int(stored), "held_blocks": len(held),
                "tokens_per_block_capacity": float(stored / (BLOCK_SIZE * len(held))) if held else 1.0}

    def kv_utilisation(self) -> float:
        """Stored tokens / capacity of the blocks held by running sequences
        (shared blocks counted once)."""
        return self.kv_accounting()["tokens_per_block_capacity"]


# ------------------------------------------------------------ invariants
def check_invariants(sched: Scheduler) -> None:
    """refcount[p] == number of block tables referencing p; the free list,
    the parked cached blocks and the referenced blocks partition the pool;
    every cached key names a block that is referenced or parked, and its
    parent is cached too."""
    a = sched.alloc
    count = np.zeros(a.num_blocks, np.int64)
    for s in sched.running:
        for b in s.block_table:
            count[b] += 1
    for s in sched.waiting:
        for b in s.block_table:
            count[b] += 1
    if not np.array_equal(count, a.ref):
        bad = np.nonzero(count != a.ref)[0][:5]
        raise AssertionError(f"refcount mismatch at blocks {bad.tolist()}")
    free = np.zeros(a.num_blocks, bool)
    free[a.free_list] = True
    if len(a.free_list) != int(free.sum()):
        raise AssertionError("duplicate entries in the free list")
    parked = np.zeros(a.num_blocks, bool)
    if a.cache is not None:
        parked[list(a.cache.lru)] = True
        for b, key in a.cache.key_of.items():
            if free[b] or (a.ref[b] == 0 and not parked[b]):
                raise AssertionError(f"cached block {b} is free")
            if a.cache.block_of.get(key) != b or (key[0] >= 0 and key[0] not in a.cache.key_of):
                raise AssertionError(f"cache maps of block {b} disagree")
        if any(b not in a.cache.key_of for b in a.cache.lru):
            raise AssertionError("a parked block has no key")
    if np.any(free & parked) or np.any((free | parked) & (a.ref > 0)) or np.any(~(free | parked) & (a.ref == 0)):
        raise AssertionError("free list, parked cached blocks and referenced blocks do not partition the pool")
