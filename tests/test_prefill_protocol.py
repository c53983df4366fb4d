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
O-done wait) must each be caught."""
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


# (K/V tiles of query tile 0, of query tile 1): a causal chunk's second tile
# needs one more key tile; a tile past the chunk end needs none
SHAPES = [(1, 0), (3, 0), (2, 3), (5, 6), (9, 10), (1, 1), (4, 4), (8, 8)]


@pytest.mark.parametrize("ntl", SHAPES)
@pytest.mark.parametrize("nslot", [2, 4])
def test_protocol_has_no_deadlock_aliasing_or_overwrite(ntl, nslot):
    assert explore(list(ntl), nslot, seeds=120) is None


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

def explore_give_up(ntl, nslot, seeds, break_softmax_loop=False, wait_after_failure=False):
    nq, ntiles = len(ntl), max(ntl)
    for seed in range(seeds):
        rnd = random.Random(1000 + seed)
        ring = {k: [Barrier(f"{k}{i}") for i in range(nslot)] for k in ("kfull", "kempty", "vfull", "vempty")}
        tile = {k: [Barrier(f"{k}{t}", 2 if k == "pfull" else 1) for t in range(nq)]
                for k in ("sfull", "pfull", "odone", "ofinal")}
        mma_done = Barrier("mma_done")
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
