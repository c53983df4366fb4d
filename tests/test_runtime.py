"""Host runtime: block allocator, copy-on-write and the iteration-level
scheduler, checked against an independent model of the pages' page pool,
the pages' own arithmetic, and invariants on seeded traces."""
import numpy as np
import pytest

from paged_kv_cache_408_b200 import runtime as R
from paged_kv_cache_408_b200 import traces as T


# ---------------------------------------------------------------- a model
class PagePoolModel:
    """Independent restatement of the pages' page pool ("Production Serving:
    Continuous Batching and PagedAttention", Step 4): a free list that starts
    as range(N), pop() to allocate, append() to free, a page appended to the
    table exactly when the stored length is a multiple of 16, every page
    returned at the end; plus copy-on-write for pages shared by forks."""

    def __init__(self, n, order=None):
        self.free = list(range(n)) if order is None else list(order)
        self.count = {}

    def take(self):
        if not self.free:
            raise MemoryError
        p = self.free.pop()
        self.count[p] = 1
        return p

    def drop(self, p):
        self.count[p] -= 1
        if self.count[p] == 0:
            del self.count[p]
            self.free.append(p)


def model_append(pool, table, length, copies):
    if length % 16 == 0:
        table.append(pool.take())
    elif pool.count[table[-1]] > 1:  # shared last page: copy before writing
        new = pool.take()
        copies.append((table[-1], new))
        pool.drop(table[-1])
        table[-1] = new
    return table[-1] * 16 + length % 16


def test_allocator_matches_the_page_pool_model_on_a_seeded_trace():
    rng = np.random.default_rng(0)
    n = 300
    order = rng.permutation(n)
    alloc = R.BlockAllocator(n, order=order)
    kv = R.KVManager(alloc)
    pool = PagePoolModel(n, order)
    seqs, model = {}, {}
    next_id = 0
    for step in range(3000):
        op = rng.random()
        if op < 0.05 or not seqs:  # new sequence
            s = R.Sequence(next_id, 1, 1)
            seqs[next_id] = s
            model[next_id] = ([], [0])
            next_id += 1
        elif op < 0.08:  # fork
            pid = int(rng.choice(list(seqs)))
            child = kv.fork(seqs[pid], next_id, 1)
            seqs[next_id] = child
            for p in model[pid][0]:
                pool.count[p] += 1
            model[next_id] = (list(model[pid][0]), [model[pid][1][0]])
            next_id += 1
        elif op < 0.12:  # finish
            sid = int(rng.choice(list(seqs)))
            kv.release(seqs.pop(sid))
            for p in model.pop(sid)[0]:
                pool.drop(p)
        else:  # append one token
            sid = int(rng.choice(list(seqs)))
            s = seqs[sid]
            try:
                slot = kv.slot_for(s, s.num_cached)
            except R.OutOfBlocksError:
                with pytest.raises(MemoryError):
                    model_append(pool, model[sid][0], model[sid][1][0], [])
                continue
            copies = []
            mslot = model_append(pool, model[sid][0], model[sid][1][0], copies)
            s.num_cached += 1
            model[sid][1][0] += 1
            assert slot == mslot
            assert kv.take_copies().tolist() == [list(c) for c in copies]
        for sid, s in seqs.items():
            assert s.block_table == model[sid][0]
        assert alloc.free_list == pool.free


def test_free_list_is_lifo_from_range_and_empty_pool_raises():
    a = R.BlockAllocator(4)
    assert [a.alloc() for _ in range(4)] == [3, 2, 1, 0]
    with pytest.raises(R.OutOfBlocksError):
        a.alloc()
    a.decref(2)
    a.decref(0)
    assert a.alloc() == 0 and a.alloc() == 2


def test_a_block_is_allocated_exactly_when_length_is_a_multiple_of_16():
    a = R.BlockAllocator(10)
    kv = R.KVManager(a)
    s = R.Sequence(0, 1, 1)
    grew = []
    for pos in range(50):
        before = len(s.block_table)
        kv.slot_for(s, pos)
        s.num_cached += 1
        grew.append(len(s.block_table) > before)
    assert [i for i, g in enumerate(grew) if g] == [0, 16, 32, 48]


def test_fork_copies_the_shared_partial_block_once_and_balances_refcounts():
    a = R.BlockAllocator(20)
    kv = R.KVManager(a)
    parent = R.Sequence(0, 1, 1)
    for pos in range(20):  # two blocks, the second partly filled (4 of 16)
        kv.slot_for(parent, pos)
        parent.num_cached += 1
    child = kv.fork(parent, 1, 1)
    assert child.block_table == parent.block_table
    assert a.ref[parent.block_table[0]] == 2 and a.ref[parent.block_table[1]] == 2
    shared_last = parent.block_table[1]
    kv.slot_for(child, child.num_cached)  # first divergent write: copy
    (src, dst), = kv.take_copies().tolist()
    assert src == shared_last and dst == child.block_table[1] and dst != shared_last
    assert a.ref[shared_last] == 1
    kv.slot_for(parent, parent.num_cached)  # the parent now owns the block alone: no copy
    assert kv.take_copies().shape == (0, 2)
    kv.release(child)
    kv.release(parent)
    assert a.num_free == 20 and not a.ref.any()


def test_fork_at_a_block_boundary_needs_no_copy():
    a = R.BlockAllocator(20)
    kv = R.KVManager(a)
    parent = R.Sequence(0, 1, 1)
    for pos in range(32):
        kv.slot_for(parent, pos)
        parent.num_cached += 1
    child = kv.fork(parent, 1, 1)
    kv.slot_for(child, 32)
    kv.slot_for(parent, 32)
    assert kv.take_copies().shape == (0, 2)
    assert child.block_table[:2] == parent.block_table[:2] and child.block_table[2] != parent.block_table[2]


# -------------------------------------------------------- the pages' arithmetic
def test_contiguous_reservation_arithmetic():
    # 4096-token reservations, 200-token average answers: ~5% used;
    # 100 requests reserve 409,600 tokens (the page says "400,000") for 20,000 stored
    assert abs(200 / 4096 - 0.05) < 0.002
    assert 100 * 4096 == 409_600 and 100 * 200 == 20_000


def test_paged_waste_per_sequence_is_below_one_block():
    rng = np.random.default_rng(3)
    for n in rng.integers(1, 5000, 500):
        waste = 16 * R.blocks_for(int(n)) - int(n)
        assert 0 <= waste <= 15


def test_reservation_of_8_blocks_in_a_32_block_pool_admits_4_conversations():
    # "32 blocks, 8 blocks max per conversation": reserving the maximum up front
    pool, per_conv = 32, 8
    admitted = 0
    free = pool
    while free >= per_conv:
        free -= per_conv
        admitted += 1
    assert admitted == 4


# ------------------------------------------------------------- scheduler
def make_sched(n_blocks, **cfg):
    return R.Scheduler(R.BlockAllocator(n_blocks), R.SchedulerConfig(**cfg))


def test_decode_first_then_prefill_chunks_fill_the_token_budget():
    s = make_sched(400, max_num_batched_tokens=100, max_chunk=64, max_blocks_per_seq=64)
    for i in range(3):
        s.restore(i, 10 + i, 50)
    s.add_request(R.Sequence(10, 200, 5))
    plan = s.step()
    assert plan.num_decode == 3
    assert plan.decode_lens.tolist() == [11, 12, 13]
    assert plan.prefill_cu.tolist() == [0, 64]  # min(budget 97, chunk cap 64)
    assert len(plan.slots) == 3 + 64
    s.complete(plan)
    plan = s.step()
    assert plan.prefill_prefix.tolist() == [64] and plan.prefill_cu.tolist() == [0, 64]


def test_admission_control_keeps_a_watermark():
    s = make_sched(100, watermark=0.1, max_blocks_per_seq=128)  # watermark 10 blocks
    s.add_request(R.Sequence(0, 16 * 85, 5))   # 85 blocks: 85 + 10 <= 100 -> admitted
    s.add_request(R.Sequence(1, 16 * 10, 5))   # 10 more: 10 + 10 > 15 free -> waits
    plan = s.step()
    assert plan.admitted == [0]
    assert [r.seq_id for r in s.waiting] == [1]


def test_preemption_evicts_the_youngest_and_recompute_resumes():
    s = make_sched(6, watermark=0.0, max_blocks_per_seq=16)
    old = s.restore(0, 32, 100)   # 2 blocks, next token opens block 3
    young = s.restore(1, 48, 100)  # 3 blocks, next token opens block 4
    plan = s.step()                # 6 blocks needed, 5 + 1 free: the youngest goes
    assert plan.preempted == [1] and plan.decode_ids.tolist() == [0]
    assert young.status == R.WAITING and young.num_cached == 0 and young.prefill_end == 48
    s.complete(plan)
    R.check_invariants(s)
    s.retire(old)
    for _ in range(3):
        plan = s.step()
        s.complete(plan)
        R.check_invariants(s)
    assert young.status == R.RUNNING and young.num_cached >= 48 and not young.in_prefill


def test_requests_longer_than_the_table_are_refused_and_growth_stops_at_it():
    s = make_sched(100, max_blocks_per_seq=4)
    with pytest.raises(ValueError):
        s.add_request(R.Sequence(0, 16 * 4 + 1, 5))
    seq = s.restore(1, 16 * 4 - 2, 10)  # room for 2 more tokens in its table
    for _ in range(5):
        plan = s.step()
        s.complete(plan)
    assert seq.status == R.FINISHED and seq.num_cached <= 16 * 4


def test_retired_sequences_return_every_block():
    s = make_sched(50, max_blocks_per_seq=16)
    a = s.restore(0, 40, 1)
    b = s.restore(1, 17, 1)
    plan = s.step()
    s.complete(plan)
    plan = s.step()  # both ran out of decode steps: retired
    assert sorted(plan.retired) == [0, 1]
    assert s.alloc.num_free == 50


# -------------------------------------------------------------- traces
@pytest.mark.parametrize("builder,steps", [(T.batch64_2k, 200), (T.prefix_share_fp8, 40), (T.long_context, 20)])
def test_trace_invariants_every_step(builder, steps):
    tr = builder(0)
    total_copies = 0
    for _ in range(steps):
        plan = tr.plans(1)[0]
        R.check_invariants(tr.sched)
        assert len(set(plan.slots.tolist())) == len(plan.slots)       # distinct slots
        if plan.copies.size:
            dsts = plan.copies[:, 1].tolist()
            assert len(set(dsts)) == len(dsts)                         # distinct destinations
            assert not set(dsts) & set(plan.copies[:, 0].tolist())     # no dst is a src
        total_copies += len(plan.copies)
        for row, n in zip(plan.decode_tables, plan.decode_lens):
            assert (row[:R.blocks_for(int(n))] >= 0).all()
    if builder is T.prefix_share_fp8:
        assert total_copies > 0


def test_batch64_trace_keeps_64_sequences_and_utilisation_high():
    tr = T.batch64_2k(0)
    plans = tr.plans(200)
    nd = np.array([p.num_decode for p in plans])
    # replacements spend their admission step writing their prompt, then decode
    assert nd.max() <= 64 and nd.min() >= 56 and nd.mean() >= 62
    assert tr.sched.kv_utilisation() > 0.96  # paging wastes less than one block per sequence


def test_shared_decode_blocks_is_the_common_fully_covered_table_prefix():
    rng = np.random.default_rng(11)
    for _ in range(200):
        B, W = int(rng.integers(1, 6)), int(rng.integers(1, 9))
        t = rng.integers(0, 3, (B, W)).astype(np.int32)
        lens = rng.integers(1, 16 * W + 1, B).astype(np.int32)
        plan = R.StepPlan(0, np.zeros((0, 2), np.int32), np.zeros(0, np.int64), np.arange(B), t, lens,
                          np.zeros(0, np.int64), np.zeros(1, np.int32), np.zeros(0, np.int32),
                          np.zeros((0, W), np.int32))
        want = 0
        while (want < W and all(t[b, want] == t[0, want] for b in range(B))
               and all(lens[b] >= 16 * (want + 1) for b in range(B))):
            want += 1
        assert plan.shared_decode_blocks == want


def test_forked_trace_shares_its_prompt_blocks_every_step():
    from paged_kv_cache_408_b200 import traces
    tr = traces.prefix_share_fp8(0, n=24, forks=4, prefix=256)
    for plan in tr.plans(6):
        assert plan.num_decode == 24 and plan.shared_decode_blocks >= 16


def test_kv_accounting_shows_paging_waste_and_sharing():
    from paged_kv_cache_408_b200 import traces
    tr = traces.batch64_2k(0)
    tr.plans(5)
    acc = tr.sched.kv_accounting()
    assert acc["sequences"] == 64 and 0.9 < acc["tokens_per_block_capacity"] <= 1.0
    # the waste is below one block per sequence
    assert acc["held_blocks"] * 16 - acc["cached_tokens"] < 16 * acc["sequences"]
    tr = traces.prefix_share_fp8(0)
    tr.plans(2)
    acc = tr.sched.kv_accounting()
    # 256 sequences over one 2048-token prefix: each stored token far more often than once
    assert acc["sequences"] == 256 and acc["tokens_per_block_capacity"] > 5
    import json
    json.dumps(acc)  # bench.py prints it in its JSON line


def test_mixed_trace_plans_carry_prefill_chunks():
    """The mixed trace drives chunked prefill through the scheduler: step 0 is
    192 decode rows plus 8 chunks of 512 tokens over cached prefixes in
    [0, 4096]; every later step keeps 8 prompts in prefill, each advancing by
    a chunk of at most 512 tokens within the 8192-token budget, decode rows
    first; the invariants of the pool hold after every step."""
    from paged_kv_cache_408_b200 import traces
    tr = traces.mixed(0)
    plans = []
    for _ in range(12):
        plans += tr.plans(1)
        R.check_invariants(tr.sched)
    p0 = plans[0]
    assert p0.num_decode == 192 and len(p0.prefill_ids) == 8 and p0.num_prefill_tokens == 8 * 512
    assert (np.diff(p0.prefill_cu) == 512).all()
    assert ((p0.prefill_prefix >= 0) & (p0.prefill_prefix <= 4096)).all()
    for p in plans:
        chunks = np.diff(p.prefill_cu)
        assert len(chunks) == 8 and (chunks > 0).all() and (chunks <= 512).all()
        assert p.num_decode + p.num_prefill_tokens <= 8192
        # slots: decode tokens first (one per row), then each chunk's tokens in order
        assert len(p.slots) == p.num_decode + p.num_prefill_tokens
        # a chunk's tables cover its prefix and the chunk itself
        for c in range(len(chunks)):
            need = (int(p.prefill_prefix[c]) + int(chunks[c]) + 15) // 16
            assert (p.prefill_tables[c, :need] >= 0).all()
    # prompts finish and join the decode batch; new prompts start from an empty prefix
    assert max(p.num_decode for p in plans) > 192
    assert any((p.prefill_prefix == 0).any() for p in plans[1:])
