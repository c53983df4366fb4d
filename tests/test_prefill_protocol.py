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


def explore(ntl, nslot, seeds, skip_odd_odone=False, no_odone_wait=False):
    """Run random schedules; return None or a description of the first violation."""
    nq, ntiles = len(ntl), max(ntl)
    for seed in range(seeds):
        rnd = random.Random(seed)
        ring = {k: [Barrier(f"{k}{i}") for i in range(nslot)] for k in ("kfull", "kempty", "vfull", "vempty")}
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

        def mma():
            violation = []
            if ntiles:
                yield ring["kfull"][0], 0
                for t in range(nq):
                    if ntl[t]:
                        pending.append(tile["sfull"][t])
                pending.append(ring["kempty"][0])
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
                pending.append(ring["vempty"][s])
                if jn < ntiles:
                    if not kready:
                        yield ring["kfull"][jn % nslot], jn // nslot
                    pending.append(ring["kempty"][jn % nslot])

        def softmax(t):
            for j in range(ntl[t]):
                yield tile["sfull"][t], j
                tile["pfull"][t].arrive()
            if ntl[t]:
                yield tile["ofinal"][t], 0

        actors = {"load": loader(), "mma": mma(), **{f"softmax{t}": softmax(t) for t in range(nq)}}
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


def test_a_skipped_o_done_wait_is_caught():
    found = [explore([6, 7], 2, seeds=200, skip_odd_odone=True), explore([6, 7], 4, seeds=200, skip_odd_odone=True)]
    assert any(found), "skipping the O-done wait on odd tiles went unnoticed"


def test_issuing_s_without_the_o_done_wait_is_caught():
    assert explore([5, 6], 2, seeds=200, no_odone_wait=True) is not None
