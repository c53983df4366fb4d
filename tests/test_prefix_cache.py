"""Prefix cache of the host runtime ("Production Serving: Continuous Batching
and PagedAttention", Step 8 "Prefix caching"): full-block token prefixes map
to the physical blocks that hold their K/V; a new prompt shares its longest
cached full-block prefix and only computes the rest.

Checked against the pages' own formulation (a dict keyed by the token tuple of
every full-page prefix, searched from the longest prefix down), on seeded
traces, and end to end with the fp64 oracle: a decode through shared cached
blocks gives bitwise the same output as one through freshly written blocks."""
import numpy as np

import oracle
from paged_kv_cache_408_b200 import runtime as R

BS = R.BLOCK_SIZE


def cache_with(n_blocks=64):
    a = R.BlockAllocator(n_blocks)
    return a, R.PrefixCache(a)


def alloc_table(a, n):
    return [a.alloc() for _ in range(n)]


def test_lookup_returns_the_longest_full_block_prefix_and_shares_its_blocks():
    a, c = cache_with()
    p = np.arange(40)                      # 2 full blocks + 8 tokens
    t = alloc_table(a, 3)
    c.insert(p, t)
    assert c.match(np.arange(5)) == (0, [])                     # shorter than a block
    n, blocks = c.match(np.concatenate([np.arange(20), [999] * 30]))
    assert (n, blocks) == (16, t[:1])                            # diverges inside block 1
    n, blocks = c.match(np.arange(100))
    assert (n, blocks) == (32, t[:2])                            # the partial third block is not cached
    assert a.ref[t[0]] == 3 and a.ref[t[1]] == 2 and a.ref[t[2]] == 1
    assert c.match(np.concatenate([[7], np.arange(1, 40)])) == (0, [])  # the first token differs


def test_a_parked_block_is_revived_and_an_evicted_one_is_forgotten():
    a, c = cache_with(8)
    t = alloc_table(a, 3)
    c.insert(np.arange(48), t)
    for b in reversed(t):
        a.decref(b)                      # the sequence ends: blocks parked, not freed
    assert a.num_free == 8 and len(a.free_list) == 5 and c.num_evictable == 3
    n, blocks = c.match(np.arange(48))   # revived without allocating
    assert (n, blocks) == (48, t) and list(a.ref[t]) == [1, 1, 1] and c.num_evictable == 0
    for b in reversed(t):
        a.decref(b)
    # drain the free list: the next allocations evict the least recently
    # released block (the deepest one) and drop its key
    got = [a.alloc() for _ in range(6)]
    assert got[5] == t[2] and c.evictions == 1
    assert c.match(np.arange(48)) == (32, t[:2])
    for b in reversed(t[:2]):
        a.decref(b)
    assert a.alloc() == t[1] and c.evictions == 2   # the deepest block was released first
    assert c.match(np.arange(48)) == (16, t[:1])


def test_evicting_a_block_drops_the_keys_below_it():
    a, c = cache_with(8)
    t = alloc_table(a, 3)
    c.insert(np.arange(48), t)
    # release root first, so the root is the least recently released
    for b in t:
        a.decref(b)
    for _ in range(5):
        a.alloc()
    b = a.alloc()                        # evicts t[0]; t[1], t[2] lose their keys and are freed
    assert b == t[0] and not c.holds(t[1]) and not c.holds(t[2]) and c.num_evictable == 0
    assert sorted(a.free_list) == sorted(t[1:])
    assert c.match(np.arange(48)) == (0, [])


class PagesPrefixCache:
    """The pages' formulation: a dict from the token tuple of every cached
    full-page prefix to its pages; lookup from the longest full-page prefix
    of the query down."""

    def __init__(self):
        self.cache = {}

    def insert(self, tokens, pages):
        for n in range(BS, len(tokens) // BS * BS + 1, BS):
            key = tuple(int(x) for x in tokens[:n])
            if key not in self.cache:
                self.cache[key] = list(pages[:n // BS])
            pages = self.cache[key] + list(pages[n // BS:])  # later blocks chain below the cached ones

    def find(self, tokens):
        for n in range(len(tokens) // BS * BS, 0, -BS):
            key = tuple(int(x) for x in tokens[:n])
            if key in self.cache:
                return n, self.cache[key]
        return 0, []

    def evict(self, b):
        self.cache = {k: v for k, v in self.cache.items() if b not in v}


def test_matches_the_pages_prefix_cache_on_a_seeded_trace():
    rng = np.random.default_rng(5)
    a = R.BlockAllocator(120, order=rng.permutation(120))
    c = R.PrefixCache(a)
    ref = PagesPrefixCache()
    evict = c.evict

    def tracked_evict():
        b = evict()
        ref.evict(b)
        return b
    c.evict = tracked_evict
    # prompts over a small vocabulary built from a few shared "system prompts"
    systems = [rng.integers(0, 4, rng.integers(8, 70)) for _ in range(5)]
    live = []
    for step in range(400):
        if live and rng.random() < 0.45:
            table = live.pop(int(rng.integers(len(live))))
            for b in reversed(table):
                a.decref(b)
            continue
        prompt = np.concatenate([systems[rng.integers(5)], rng.integers(0, 4, rng.integers(0, 40))])
        look = prompt[:max(0, len(prompt) - 1)]
        want_n, want_blocks = ref.find(look)
        n, blocks = c.match(look)
        assert n == want_n and blocks == want_blocks, step
        try:
            table = blocks + [a.alloc() for _ in range(R.blocks_for(len(prompt)) - len(blocks))]
        except R.OutOfBlocksError:
            for b in reversed(blocks):
                a.decref(b)
            continue
        c.insert(prompt, table)
        ref.insert(prompt, table)
        live.append(table)
    assert c.hits > 0 and c.evictions > 0


def shared_prompt_trace(prefix_cache):
    rng = np.random.default_rng(7)
    system = rng.integers(0, 1000, 200)
    s = R.Scheduler(R.BlockAllocator(300), R.SchedulerConfig(max_num_batched_tokens=256, max_blocks_per_seq=32,
                                                             prefix_cache=prefix_cache))
    for i in range(12):
        p = np.concatenate([system, rng.integers(0, 1000, int(rng.integers(1, 60)))])
        seq = R.Sequence(i, len(p), int(rng.integers(1, 6)))
        seq.tokens = p
        s.add_request(seq)
    return s


def test_scheduler_shares_cached_prompt_blocks_and_computes_less():
    computed = {}
    for pc in (False, True):
        s = shared_prompt_trace(pc)
        n_prefill = 0
        for _ in range(60):
            plan = s.step()
            R.check_invariants(s)
            n_prefill += plan.num_prefill_tokens
            s.complete(plan)
        assert len(s.finished) == 12
        computed[pc] = n_prefill
    # the 200-token system prompt's 12 full blocks are computed once, not 12 times
    assert computed[False] - computed[True] >= 10 * 12 * BS


def kv_of(token, pos, Hkv, D, salt):
    """K or V row of a token at a position: a fixed function of both, so that
    blocks holding the same full-block prefix hold the same bytes."""
    r = np.random.default_rng([int(token), int(pos), salt])
    x = r.standard_normal((Hkv, D)).astype(np.float32)
    return (x.view(np.uint32) >> 16).astype(np.uint16)  # bf16 truncation of a fixed draw


def test_decode_through_shared_cached_blocks_is_bitwise_identical():
    """Run the same requests with and without the prefix cache, writing each
    computed position's K/V (a fixed function of token and position) with the
    oracle, then decode every sequence with the oracle: outputs are equal."""
    Hkv, Hq, D = 2, 4, 64
    outs = {}
    for pc in (False, True):
        s = shared_prompt_trace(pc)
        kc = np.zeros((300, Hkv, BS, D), np.uint16)
        vc = np.zeros_like(kc)
        written = 0
        res = {}
        for _ in range(60):
            plan = s.step()
            # the positions this step writes, in slot order: decodes, then chunks
            pos_tok = []
            for sid in plan.decode_ids:
                q = next(x for x in s.running if x.seq_id == sid)
                pos_tok.append((q.num_cached, int(q.tokens[q.num_cached]) if q.num_cached < len(q.tokens) else 7))
            for sid, start, n in zip(plan.prefill_ids, plan.prefill_prefix, np.diff(plan.prefill_cu)):
                q = next(x for x in s.running if x.seq_id == sid)
                pos_tok += [(p, int(q.tokens[p])) for p in range(start, start + n)]
            if pos_tok:
                k = np.stack([kv_of(t, p, Hkv, D, 1) for p, t in pos_tok])
                v = np.stack([kv_of(t, p, Hkv, D, 2) for p, t in pos_tok])
                oracle.write_kv(k, v, plan.slots, kc, vc)
                written += len(pos_tok)
            if plan.num_decode:
                qv = np.stack([(np.random.default_rng([int(sid), int(n)]).standard_normal((Hq, D)).astype(np.float32)
                                .view(np.uint32) >> 16).astype(np.uint16)
                               for sid, n in zip(plan.decode_ids, plan.decode_lens)])
                o = oracle.decode(qv, kc, vc, plan.decode_tables, plan.decode_lens, 0.125)
                for i, sid in enumerate(plan.decode_ids):
                    res[(int(sid), int(plan.decode_lens[i]))] = o[i]
            s.complete(plan)
        outs[pc] = (res, written)
    (r0, w0), (r1, w1) = outs[False], outs[True]
    assert w1 < w0 and r0.keys() == r1.keys() and len(r0) > 0
    for key in r0:
        np.testing.assert_array_equal(r0[key], r1[key])
