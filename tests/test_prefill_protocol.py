"""The prefill kernel's synchronisation protocol, restated as a discrete model
and explored over random schedules on the CPU (no race checker runs on the
GPU here).

Actors, as in `prefill_kernel` (csrc/prefill.cu): the TMA warp fills K and V
ring slots (waiting on the slot's "empty" barrier before a refill); the MMA
warp issues, per key tile j, P_t(j).V_j for each query tile t as soon as that
tile's softmax has written P_t(j), then S_t(j+1) = Q_t.K_{j+1}^T once that
P.V has completed (S_t(j+1) overwrites P_t(j) in TMEM); one softmax actor per
query tile waits for S_t(j), writes P_t(j) and signals it.  MMA completions
(tcgen05.commit) and copy completions arrive later, in issue order.

Checked for every schedule: no deadlock; no waiter sees its barrier two or
more phases past the one it waits for (a parity wait would pass on a stale
phase); S_t(j+1) is never issued before P_t(j).V_j has completed.  Two planted
protocol mistakes (an O-done wait skipped on odd tiles, S issued without the
O-done wait) must each be caught.

With a bf16 cache the kernel keeps P in shared memory instead (`psmem`
below): the loader fills K_{j+1} before V_j into a K ring and a V ring;
the MMA warp issues S_t(j+1) as soon as softmax t has loaded S_t(j) into
registers ("S free") and then P_t(j).V_j once P_t(j) is in shared memory;
softmax t writes P_t(j) only after P_t(j-1).V_{j-1} has
completed (O done), which also makes its O rescale safe.  Checked: the
softmax always reads the scores of the tile it waits for, every MMA reads
the K or V tile it expects, P_t(j) is still in its buffer when its P.V
completes, a slot is never refilled before the MMAs reading it completed.
Planted: the S-free wait skipped, the O-done wait before the P write skipped."""
import random

import pytest


class Barrier:
    def __init__(self, name, count=1):
        self.name, self.count, self.pending, self.phase = name, count, count, 0

    def arrive(self):
        self.pending -= 1
        if self.pending == 0:
            self.phase += 1
            self.pending = self.count


def explore(ntl, nslot, seeds, skip_odd_odone=False, no_odone_wait=False, fp8=False, early_refill=False):
    """Run random schedules; return None or a description of the first violation.

    fp8: the loader of an E4M3 cache -- one warp issues the TMA of each
    tile's codes into the slot's staging area ("kload"/"vload" complete when
    they land), both loader warps widen them into the slot and arrive on
    full (count 2 here, one per warp); the slot of tile j-1 is refilled with
    tile j-1+nslot once its empty barrier completes.  early_refill (a planted
    mistake): refill the slot of tile j with tile j+nslot before its MMAs
    are done."""
    nq, ntiles = len(ntl), max(ntl)
    for seed in range(seeds):
        rnd = random.Random(seed)
        ring = {k: [Barrier(f"{k}{i}", 2 if fp8 and k in ("kfull", "vfull") else 1) for i in range(nslot)]
                for k in ("kfull", "kempty", "vfull", "vempty", "kload", "vload")}
        consumed = {"k": [-1] * nslot, "v": [-1] * nslot}  # last tile whose MMAs read the slot, per slot
        loaded = {"k": [-1] * nslot, "v": [-1] * nslot}    # tile whose codes sit in the slot
        tile = {k: [Barrier(f"{k}{t}") for t in range(nq)] for k in ("sfull", "pfull", "odone", "ofinal")}
        pending = []       # asynchronous completions, delivered in issue order
        pv_done = [-1] * nq  # last tile j whose P.V has completed, per query tile

        class Commit:      # a P.V completion: marks the data, then arrives
            def __init__(self, t, j):
                self.t, self.j = t, j

            def arrive(self):
                pv_done[self.t] = max(pv_done[self.t], self.j)
                tile["odone"][self.t].arrive()

        def loader():
            for j in range(ntiles):
                s, use = j % nslot, j // nslot
                for kind in ("k", "v"):
                    if use:
                        yield ring[kind + "empty"][s], use - 1
                    pending.append(ring[kind + "full"][s])

        class Landed:  # the TMA of tile j's codes lands in slot s
            def __init__(self, kind, s, j):
                self.kind, self.s, self.j = kind, s, j

            def arrive(self):
                loaded[self.kind][self.s] = self.j
                ring[self.kind + "load"][self.s].arrive()

        def issue(kind, j):
            s = j % nslot
            if j >= nslot and consumed[kind][s] < j - nslot:
                violation.append(f"{kind} codes of tile {j} issued over tile {j - nslot} still in use")
            pending.append(Landed(kind, s, j))

        violation = []

        def fp8_issuer():
            for j in range(min(nslot, ntiles)):
                issue("k", j)
                issue("v", j)
            for j in range(ntiles):
                for kind in ("k", "v"):
                    yield ring[kind + "load"][j % nslot], j // nslot
                    if loaded[kind][j % nslot] != j:
                        yield None, f"{kind} tile {j} widened from the codes of tile {loaded[kind][j % nslot]}"
                    ring[kind + "full"][j % nslot].arrive()
                jr, jd = (j + nslot, j) if early_refill else (j - 1 + nslot, j - 1)
                if jd >= 0 and jr < ntiles:
                    for kind in ("k", "v"):
                        if not early_refill:
                            yield ring[kind + "empty"][jd % nslot], jd // nslot
                        issue(kind, jr)
                if violation:
                    yield None, violation[0]

        def fp8_widener():  # the second loader warp: widens the same tiles
            for j in range(ntiles):
                for kind in ("k", "v"):
                    yield ring[kind + "load"][j % nslot], j // nslot
                    ring[kind + "full"][j % nslot].arrive()

        class Consumed:  # the MMAs reading a slot's tile have completed
            def __init__(self, kind, s, j, bar):
                self.kind, self.s, self.j, self.bar = kind, s, j, bar

            def arrive(self):
                consumed[self.kind][self.s] = max(consumed[self.kind][self.s], self.j)
                self.bar.arrive()

        def mma():
            violation = []
            if ntiles:
                yield ring["kfull"][0], 0
                for t in range(nq):
                    if ntl[t]:
                        pending.append(tile["sfull"][t])
                pending.append(Consumed("k", 0, 0, ring["kempty"][0]))
            for j in range(ntiles):
                s, jn = j % nslot, j + 1
                yield ring["vfull"][s], j // nslot
                kready = False
                for t in range(nq):
                    if j < ntl[t]:
                        yield tile["pfull"][t], j
                        pending.append(Commit(t, j))
                        if j == ntl[t] - 1:
                            pending.append(tile["ofinal"][t])
                    if jn < ntl[t]:
                        if not kready:
                            yield ring["kfull"][jn % nslot], jn // nslot
                            kready = True
                        if not no_odone_wait and not (skip_odd_odone and j % 2):
                            yield tile["odone"][t], j
                        if pv_done[t] < j:
                            violation.append(f"S_{t}({jn}) issued before P_{t}({j}).V completed")
                            yield None, violation[-1]
                        pending.append(tile["sfull"][t])
                pending.append(Consumed("v", s, j, ring["vempty"][s]))
                if jn < ntiles:
                    if not kready:
                        yield ring["kfull"][jn % nslot], jn // nslot
                    pending.append(Consumed("k", jn % nslot, jn, ring["kempty"][jn % nslot]))

        def softmax(t):
            for j in range(ntl[t]):
                yield tile["sfull"][t], j
                tile["pfull"][t].arrive()
            if ntl[t]:
                yield tile["ofinal"][t], 0

        loaders = {"issue": fp8_issuer(), "widen": fp8_widener()} if fp8 else {"load": loader()}
        actors = {**loaders, "mma": mma(), **{f"softmax{t}": softmax(t) for t in range(nq)}}
        waiting = {k: None for k in actors}
        done = set()
        while len(done) < len(actors):
            progress = False
            if pending and rnd.random() < 0.5:
                pending.pop(0).arrive()
                progress = True
            order = list(actors)
            rnd.shuffle(order)
            for k in order:
                if k in done:
                    continue
                if waiting[k] is not None:
                    bar, phase = waiting[k]
                    if bar is None:
                        return f"seed {seed}: {phase}"
                    if bar.phase > phase + 1:
                        return f"seed {seed}: {k} waits for phase {phase} of {bar.name}, already at {bar.phase}"
                    if bar.phase <= phase:
                        continue
                    waiting[k] = None
                try:
                    waiting[k] = next(actors[k])
                except StopIteration:
                    done.add(k)
                progress = True
            if not progress:
                if pending:
                    pending.pop(0).arrive()
                    continue
                stuck = {k: (w[0].name, w[1]) for k, w in waiting.items() if w and k not in done}
                return f"seed {seed}: deadlock {stuck}"
    return None


def explore_psmem(ntl, nsk, nsv, seeds, skip_sfree=False, skip_odone=False, skip_qwait=False):
    """Random schedules of the P-in-shared-memory protocol (a K ring of nsk
    slots, a V ring of nsv slots, a P buffer per query tile, the query tiles
    copied once by the loader thread); None or the first violation."""
    nq, ntiles = len(ntl), max(ntl)
    for seed in range(seeds):
        rnd = random.Random(7000 + seed)
        ns = {"k": nsk, "v": nsv}
        ring = {k + e: [Barrier(f"{k}{e}{i}") for i in range(ns[k])] for k in ("k", "v") for e in ("full", "empty")}
        tile = {k: [Barrier(f"{k}{t}") for t in range(nq)] for k in ("sfull", "sfree", "pfull", "odone", "ofinal")}
        consumed = {"k": [-1] * nsk, "v": [-1] * nsv}  # last tile whose MMAs completed, per slot
        held = {"k": [-1] * nsk, "v": [-1] * nsv}      # the tile whose data sits in each slot
        s_data = [-1] * nq   # the key tile whose scores sit in S_t's TMEM columns
        p_data = [-1] * nq   # the key tile whose P sits in P_t's buffer
        pv_done = [-1] * nq
        qbar, q_landed = Barrier("qfull"), [False]
        pending, side, violation = [], [], []

        class Done:  # an asynchronous completion: apply its effect, then arrive
            def __init__(self, bar, effect=None):
                self.bar, self.effect = bar, effect

            def arrive(self):
                if self.effect:
                    self.effect()
                self.bar.arrive()

        def landed(kind, j):
            def f():
                held[kind][j % ns[kind]] = j
            return f

        def fill(kind, j):
            sl, use = j % ns[kind], j // ns[kind]
            if use:
                yield ring[kind + "empty"][sl], use - 1
                if consumed[kind][sl] < j - ns[kind]:
                    yield None, f"{kind} tile {j} copied over tile {j - ns[kind]} still in use"
            pending.append(Done(ring[kind + "full"][sl], landed(kind, j)))

        def loader():
            # the query tiles' copy completes on its own, in no order with
            # the K/V copies and the MMAs (the side queue)
            side.append(Done(qbar, lambda: q_landed.__setitem__(0, True)))
            if ntiles:
                yield from fill("k", 0)
            for j in range(ntiles):
                if j + 1 < ntiles:
                    yield from fill("k", j + 1)
                yield from fill("v", j)
            yield qbar, 0  # the copy has landed before the CTA may exit

        def consumed_by(kind, sl, j):
            def f():
                consumed[kind][sl] = max(consumed[kind][sl], j)
            return f

        def scores(t, j):
            def f():
                if not q_landed[0]:
                    violation.append(f"S_{t}({j}) computed before the query tiles landed")
                if held["k"][j % nsk] != j:
                    violation.append(f"S_{t}({j}) computed from K tile {held['k'][j % nsk]}")
                s_data[t] = j
            return f

        def pv(t, j):
            def f():
                if p_data[t] != j:
                    violation.append(f"P_{t}({j}).V completed with P_{t}({p_data[t]}) in the buffer")
                if held["v"][j % nsv] != j:
                    violation.append(f"P_{t}({j}).V read V tile {held['v'][j % nsv]}")
                pv_done[t] = j
            return f

        def mma():
            if ntiles:
                if not skip_qwait:
                    yield qbar, 0
                yield ring["kfull"][0], 0
                for t in range(nq):
                    if ntl[t]:
                        pending.append(Done(tile["sfull"][t], scores(t, 0)))
                pending.append(Done(ring["kempty"][0], consumed_by("k", 0, 0)))
            for j in range(ntiles):
                jn = j + 1
                if jn < ntiles:
                    sn = jn % nsk
                    yield ring["kfull"][sn], jn // nsk
                    for t in range(nq):
                        if jn < ntl[t]:
                            if not skip_sfree:
                                yield tile["sfree"][t], j
                            pending.append(Done(tile["sfull"][t], scores(t, jn)))
                    pending.append(Done(ring["kempty"][sn], consumed_by("k", sn, jn)))
                sv = j % nsv
                yield ring["vfull"][sv], j // nsv
                for t in range(nq):
                    if j < ntl[t]:
                        yield tile["pfull"][t], j
                        pending.append(Done(tile["odone"][t], pv(t, j)))
                        if j == ntl[t] - 1:
                            pending.append(Done(tile["ofinal"][t]))
                pending.append(Done(ring["vempty"][sv], consumed_by("v", sv, j)))
                if violation:
                    yield None, violation[0]

        def softmax(t):
            for j in range(ntl[t]):
                yield tile["sfull"][t], j
                if s_data[t] != j:
                    yield None, f"softmax {t} read the scores of tile {s_data[t]} for tile {j}"
                tile["sfree"][t].arrive()
                if j > 0:
                    if not skip_odone:
                        yield tile["odone"][t], j - 1
                    if pv_done[t] < j - 1:
                        yield None, f"P_{t}({j}) written (and O_{t} rescaled) before P_{t}({j - 1}).V completed"
                p_data[t] = j
                tile["pfull"][t].arrive()
            if ntl[t]:
                yield tile["ofinal"][t], 0
                if pv_done[t] != ntl[t] - 1:
                    yield None, f"epilogue of tile {t} before its last P.V"

        actors = {"load": loader(), "mma": mma(), **{f"softmax{t}": softmax(t) for t in range(nq)}}
        err = run_schedule(actors, pending, rnd, side)
        if err or violation:
            return f"seed {seed}: {err or violation[0]}"
    return None


def run_schedule(actors, pending, rnd, side=None):
    """Drive generator actors that yield (barrier, phase) waits, or (None,
    message) for a violation; completions in `pending` arrive in order at
    random times, and an actor that could run is delayed now and then (so a
    completion may overtake a thread between its wait and its next step).
    Completions in `side` arrive one at a time in any order and at any time
    (another engine's).  Returns None or the first violation / deadlock."""
    side = [] if side is None else side
    waiting = {k: None for k in actors}
    done = set()
    while len(done) < len(actors):
        progress = False
        if pending and rnd.random() < 0.5:
            pending.pop(0).arrive()
            progress = True
        if side and rnd.random() < 0.1:
            side.pop(rnd.randrange(len(side))).arrive()
            progress = True
        order = list(actors)
        rnd.shuffle(order)
        for k in order:
            if k in done:
                continue
            if waiting[k] is not None:
                bar, phase = waiting[k]
                if bar is None:
                    return phase
                if bar.phase > phase + 1:
                    return f"{k} waits for phase {phase} of {bar.name}, already at {bar.phase}"
                if bar.phase <= phase:
                    continue
            if rnd.random() < 0.3:  # runnable, but slow this round
                progress = True
                continue
            waiting[k] = None
            try:
                waiting[k] = next(actors[k])
                if waiting[k][0] is None:
                    return waiting[k][1]
            except StopIteration:
                done.add(k)
            progress = True
        if not progress:
            if pending or side:
                (pending if pending and (not side or rnd.random() < 0.5) else side).pop(0).arrive()
                continue
            stuck = {k: (w[0].name, w[1]) for k, w in waiting.items() if w and k not in done}
            return f"deadlock {stuck}"
    return None


# (K/V tiles of query tile 0, of query tile 1): a causal chunk's second tile
# needs one more key tile; a tile past the chunk end needs none
SHAPES = [(1, 0), (3, 0), (2, 3), (5, 6), (9, 10), (1, 1), (4, 4), (8, 8)]


@pytest.mark.parametrize("ntl", SHAPES)
@pytest.mark.parametrize("nslot", [2, 4])
def test_protocol_has_no_deadlock_aliasing_or_overwrite(ntl, nslot):
    assert explore(list(ntl), nslot, seeds=120) is None


@pytest.mark.parametrize("ntl", SHAPES)
@pytest.mark.parametrize("nsk,nsv", [(2, 1), (3, 3), (1, 1)])
def test_psmem_protocol_has_no_deadlock_stale_data_or_overwrite(ntl, nsk, nsv):
    """P in shared memory (bf16 cache): 2 K slots and 1 V slot at head_dim
    128, 3 and 3 at head_dim 64, a P buffer per query tile."""
    assert explore_psmem(list(ntl), nsk, nsv, seeds=120) is None


def test_psmem_skipped_s_free_wait_is_caught():
    found = [explore_psmem([6, 7], 2, 1, seeds=200, skip_sfree=True),
             explore_psmem([9, 10], 3, 3, seeds=200, skip_sfree=True)]
    assert all(found), found


def test_psmem_scores_issued_before_the_query_tiles_landed_is_caught():
    found = [explore_psmem([3, 4], 2, 1, seeds=200, skip_qwait=True),
             explore_psmem([1, 0], 3, 3, seeds=200, skip_qwait=True)]
    assert all(found), found


def test_psmem_p_written_before_its_buffer_is_free_is_caught():
    found = [explore_psmem([6, 7], 2, 1, seeds=200, skip_odone=True),
             explore_psmem([9, 10], 3, 3, seeds=200, skip_odone=True)]
    assert all(found), found


@pytest.mark.parametrize("ntl", SHAPES)
@pytest.mark.parametrize("nslot", [2])
def test_fp8_loader_protocol(ntl, nslot):
    """The E4M3 loader (TMA of codes into staging, widening by two warps,
    refill of a slot once its previous tile's MMAs are done): no deadlock, no
    stale phase, no tile widened from another tile's codes, no codes issued
    over a tile still being read."""
    assert explore(list(ntl), nslot, seeds=120, fp8=True) is None


def test_fp8_refill_before_the_slot_is_free_is_caught():
    found = [explore([6, 7], 2, seeds=200, fp8=True, early_refill=True),
             explore([9, 10], 2, seeds=200, fp8=True, early_refill=True)]
    assert any(found), "refilling a slot before its MMAs completed went unnoticed"


def test_a_skipped_o_done_wait_is_caught():
    found = [explore([6, 7], 2, seeds=200, skip_odd_odone=True), explore([6, 7], 4, seeds=200, skip_odd_odone=True)]
    assert any(found), "skipping the O-done wait on odd tiles went unnoticed"


def test_issuing_s_without_the_o_done_wait_is_caught():
    assert explore([5, 6], 2, seeds=200, no_odone_wait=True) is not None


# ------------------------------------------------------------------------
# Giving up after a lost transaction.  Every wait of a launch shares one
# deadline; in the kernel a role evaluates `ok && mbar_wait(...)`, so after
# its first failed wait it issues no further wait of the protocol.  The
# loader and the MMA warp then stop issuing and drain what they have in
# flight (a short fresh budget); the two softmax warps that share a row
# keep meeting at their named barrier (which has no deadline) and keep
# arriving on P full, so neither is left waiting on the other.
#
# The model below drops one asynchronous completion at random (a copy or an
# MMA commit that never arrives).  When no actor can progress, the clock
# passes the deadline and every blocked wait fails; before that, a blocked
# wait may also fail on its own now and then (its thread's deadline passed
# just before a slow completion arrived), so partners can fail at different
# points of the protocol.  Checked: every actor
# finishes (no thread stranded at a named barrier), and no actor issues a
# protocol wait after its first failed one.

def explore_give_up(ntl, nslot, seeds, break_softmax_loop=False, wait_after_failure=False, psmem=None):
    """psmem = (nsk, nsv): the P-in-shared-memory protocol of a bf16 cache."""
    nq, ntiles = len(ntl), max(ntl)
    nsk, nsv = psmem if psmem else (nslot, nslot)
    for seed in range(seeds):
        rnd = random.Random(1000 + seed)
        ring = {k: [Barrier(f"{k}{i}") for i in range(nsk if k[0] == "k" else nsv)]
                for k in ("kfull", "kempty", "vfull", "vempty")}
        tile = {k: [Barrier(f"{k}{t}", 2 if k in ("pfull", "sfree") else 1) for t in range(nq)]
                for k in ("sfull", "sfree", "pfull", "odone", "ofinal")}
        mma_done = Barrier("mma_done")
        qbar = Barrier("qfull")
        pending = []
        drop_at = rnd.randrange(1, 4 * ntiles * (nq + 2) + 2)
        sent = [0]

        def post(bar):
            sent[0] += 1
            if sent[0] != drop_at:  # the dropped completion never arrives
                pending.append(bar)

        def wait(bar, phase, ok):
            """Protocol wait as the kernel issues it: skipped once ok is false."""
            if ok or wait_after_failure:
                r = yield ("wait", bar, phase)
                return ok and r
            return False

        def loader():
            ok, issued = True, {"k": 0, "v": 0}
            for j in range(ntiles):
                if not ok:
                    break
                s, use = j % nslot, j // nslot
                for kind in ("k", "v"):
                    if use:
                        ok = yield from wait(ring[kind + "empty"][s], use - 1, ok)
                        if not ok:
                            break
                    issued[kind] = j + 1
                    post(ring[kind + "full"][s])
            if not ok:
                for kind in ("k", "v"):
                    for sl in range(nslot):
                        if issued[kind] > sl:
                            yield ("drain", ring[kind + "full"][sl], (issued[kind] - 1 - sl) // nslot)

        def mma():
            ok = True
            if ntiles:
                ok = yield from wait(ring["kfull"][0], 0, ok)
                if ok:
                    for t in range(nq):
                        if ntl[t]:
                            post(tile["sfull"][t])
                    post(ring["kempty"][0])
            for j in range(ntiles):
                if not ok:
                    break
                s, jn = j % nslot, j + 1
                ok = yield from wait(ring["vfull"][s], j // nslot, ok)
                if not ok:
                    break
                kready = False
                for t in range(nq):
                    if j < ntl[t]:
                        ok = yield from wait(tile["pfull"][t], j, ok)
                        if not ok:
                            break
                        post(tile["odone"][t])
                        if j == ntl[t] - 1:
                            post(tile["ofinal"][t])
                    if jn < ntl[t]:
                        if not kready:
                            ok = yield from wait(ring["kfull"][jn % nslot], jn // nslot, ok)
                            if not ok:
                                break
                            kready = True
                        ok = yield from wait(tile["odone"][t], j, ok)
                        if not ok:
                            break
                        post(tile["sfull"][t])
                if not ok:
                    break
                post(ring["vempty"][s])
                if jn < ntiles:
                    if not kready:
                        ok = yield from wait(ring["kfull"][jn % nslot], jn // nslot, ok)
                        if not ok:
                            break
                    post(ring["kempty"][jn % nslot])
            post(mma_done)
            yield ("wait" if ok else "drain", mma_done, 0)

        def softmax(t, half):
            ok = True
            for j in range(ntl[t]):
                ok = yield from wait(tile["sfull"][t], j, ok)
                if not ok and break_softmax_loop:
                    break
                yield ("named", t)
                tile["pfull"][t].arrive()
            if ntl[t]:
                yield ("named", t)
                ok = yield from wait(tile["ofinal"][t], 0, ok)

        def loader_ps():
            ok, issued = True, {"k": 0, "v": 0}
            ns = {"k": nsk, "v": nsv}

            def fill(kind, j, ok):
                sl, use = j % ns[kind], j // ns[kind]
                if use:
                    ok = yield from wait(ring[kind + "empty"][sl], use - 1, ok)
                    if not ok:
                        return False
                issued[kind] = j + 1
                post(ring[kind + "full"][sl])
                return True

            post(qbar)  # the query tiles (may be the completion that is lost)
            if ntiles:
                ok = yield from fill("k", 0, ok)
            for j in range(ntiles):
                if not ok:
                    break
                if j + 1 < ntiles:
                    ok = yield from fill("k", j + 1, ok)
                    if not ok:
                        break
                ok = yield from fill("v", j, ok)
            if not ok:
                for kind in ("k", "v"):
                    for sl in range(ns[kind]):
                        if issued[kind] > sl:
                            yield ("drain", ring[kind + "full"][sl], (issued[kind] - 1 - sl) // ns[kind])
            # the query copy has landed before exit: on the launch's deadline,
            # or after a failure on the short drain budget
            r = yield ("wait" if ok else "drain", qbar, 0)
            ok = ok and r

        def mma_ps():
            ok = True
            if ntiles:
                ok = yield from wait(qbar, 0, ok)
                ok = yield from wait(ring["kfull"][0], 0, ok)
                if ok:
                    for t in range(nq):
                        if ntl[t]:
                            post(tile["sfull"][t])
                    post(ring["kempty"][0])
            for j in range(ntiles):
                if not ok:
                    break
                jn = j + 1
                if jn < ntiles:
                    ok = yield from wait(ring["kfull"][jn % nsk], jn // nsk, ok)
                    for t in range(nq):
                        if ok and jn < ntl[t]:
                            ok = yield from wait(tile["sfree"][t], j, ok)
                            if ok:
                                post(tile["sfull"][t])
                    if not ok:
                        break
                    post(ring["kempty"][jn % nsk])
                ok = yield from wait(ring["vfull"][j % nsv], j // nsv, ok)
                for t in range(nq):
                    if ok and j < ntl[t]:
                        ok = yield from wait(tile["pfull"][t], j, ok)
                        if ok:
                            post(tile["odone"][t])
                            if j == ntl[t] - 1:
                                post(tile["ofinal"][t])
                if not ok:
                    break
                post(ring["vempty"][j % nsv])
            post(mma_done)
            yield ("wait" if ok else "drain", mma_done, 0)

        def softmax_ps(t, half):
            ok = True
            for j in range(ntl[t]):
                ok = yield from wait(tile["sfull"][t], j, ok)
                if not ok and break_softmax_loop:
                    break
                tile["sfree"][t].arrive()
                yield ("named", t)
                if not ok:
                    tile["pfull"][t].arrive()
                    continue
                if j > 0:
                    ok = yield from wait(tile["odone"][t], j - 1, ok)
                tile["pfull"][t].arrive()
            if ntl[t]:
                ok = yield from wait(tile["ofinal"][t], 0, ok)
                yield ("named", t)

        if psmem:
            actors = {"load": loader_ps(), "mma": mma_ps(),
                      **{f"softmax{t}.{h}": softmax_ps(t, h) for t in range(nq) for h in range(2)}}
        else:
            actors = {"load": loader(), "mma": mma(),
                      **{f"softmax{t}.{h}": softmax(t, h) for t in range(nq) for h in range(2)}}
        state = {k: None for k in actors}   # the event the actor is blocked on
        reply = {k: None for k in actors}
        failed = set()
        named = {}  # t -> actors arrived at the current named barrier
        expired = False
        done = set()
        while len(done) < len(actors):
            progress = False
            if pending and rnd.random() < 0.5:
                pending.pop(0).arrive()
                progress = True
            order = list(actors)
            rnd.shuffle(order)
            for k in order:
                if k in done:
                    continue
                ev = state[k]
                if ev is not None:
                    if ev[0] in ("wait", "drain"):
                        bar, phase = ev[1], ev[2]
                        if bar.phase > phase:
                            reply[k] = True
                        elif expired or (ev[0] == "wait" and rnd.random() < 0.01):
                            # past the deadline; or this thread's deadline passed
                            # just before a slow completion (threads take their
                            # deadlines at slightly different times)
                            reply[k] = False
                            if ev[0] == "wait":
                                failed.add(k)
                        else:
                            continue
                    elif ev[0] == "named":
                        if k not in named.get(ev[1], set()):
                            named.setdefault(ev[1], set()).add(k)
                        if len(named[ev[1]]) < 2:
                            continue
                        reply[k] = None
                        # the second arriver releases both
                        other = [a for a in named[ev[1]] if a != k][0]
                        if state[other] == ev and other != k:
                            state[other] = ("released",)
                        named[ev[1]] = set()
                    elif ev[0] == "released":
                        reply[k] = None
                    state[k] = None
                try:
                    nxt = actors[k].send(reply[k]) if reply[k] is not None or ev is not None else next(actors[k])
                except StopIteration:
                    done.add(k)
                    progress = True
                    continue
                reply[k] = None
                if nxt[0] == "wait" and k in failed:
                    return f"seed {seed}: {k} issued a wait after a failed one"
                state[k] = nxt
                progress = True
            if not progress:
                if pending:
                    pending.pop(0).arrive()
                elif not expired:
                    expired = True  # the clock passes the launch deadline
                else:
                    stuck = {k: state[k][:2] if state[k] else None for k in actors if k not in done}
                    return f"seed {seed}: stranded {stuck}"
    return None


@pytest.mark.parametrize("ntl", [(1, 0), (3, 3), (5, 6), (9, 10)])
@pytest.mark.parametrize("nslot", [2, 4])
def test_a_lost_transaction_ends_every_role_without_further_waits(ntl, nslot):
    assert explore_give_up(list(ntl), nslot, seeds=150) is None


@pytest.mark.parametrize("ntl", [(1, 0), (3, 3), (5, 6), (9, 10)])
@pytest.mark.parametrize("psmem", [(2, 1), (3, 3)])
def test_psmem_lost_transaction_ends_every_role_without_further_waits(ntl, psmem):
    assert explore_give_up(list(ntl), 0, seeds=150, psmem=psmem) is None


def test_psmem_softmax_leaving_its_loop_after_a_failure_is_caught():
    found = [explore_give_up([5, 6], 0, seeds=300, break_softmax_loop=True, psmem=ps) for ps in ((2, 1), (3, 3))]
    assert any(f and "stranded" in f for f in found), found


def test_psmem_waiting_again_after_a_failure_is_caught():
    found = [explore_give_up([5, 6], 0, seeds=300, wait_after_failure=True, psmem=ps) for ps in ((2, 1), (3, 3))]
    assert any(f and "after a failed one" in f for f in found), found


def test_softmax_leaving_its_loop_after_a_failure_is_caught():
    """A softmax warp that stopped at its first failed wait would strand its
    partner at the named barrier: the model must report it."""
    found = [explore_give_up([5, 6], ns, seeds=300, break_softmax_loop=True) for ns in (2, 4)]
    assert any(f and "stranded" in f for f in found), found


def test_waiting_again_after_a_failure_is_caught():
    """Evaluating the wait before the ok flag (waits issued after a failure)
    must be reported."""
    found = [explore_give_up([5, 6], ns, seeds=300, wait_after_failure=True) for ns in (2, 4)]
    assert any(f and "after a failed one" in f for f in found), found
