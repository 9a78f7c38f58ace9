"""Host-side model of the pipelined refine kernel's hand-off protocol (CPU).

k_refine_pipe (route_refine.cu) runs three warp groups and one UMMA warp per
CTA that hand buffers to each other through mbarriers.  This model replays
each role's sequence of arrivals and parity waits exactly as the kernel
orders them, under many random schedules and random tile counts per query
(including empty candidate lists), for one and two TMEM score buffers.  It
checks that every wait is eventually satisfied (no deadlock) and that no
buffer is rewritten while its previous user still reads it:

* stage s (tile rows) is reloaded only after the UMMAs of the tile that last
  used it completed;
* accumulator a is overwritten only after the epilogue read it;
* score buffer b is written only after the top-k of the query that last used
  it finished;
* candidate list row r is rebuilt only after every reader of the query that
  last used it is done (gather warps, UMMA warp, top-k);
* the head tile is reloaded only after the previous query's UMMAs completed.

An mbarrier is modelled as in PTX: a phase completes when its expected
arrival count is reached; a wait on parity P succeeds once the phase with
parity P has completed, i.e. while the current phase's parity differs from P.
Asynchronous completions (TMA copies landing, UMMA commits) fire at random
later points.
"""
import random

import pytest


class Bar:
    def __init__(self, count):
        self.count, self.pending, self.phase = count, 0, 0

    def arrive(self):
        self.pending += 1
        assert self.pending <= self.count
        if self.pending == self.count:
            self.pending, self.phase = 0, self.phase + 1

    def done(self, parity):
        return (self.phase & 1) != parity


class Model:
    def __init__(self, nts, nsb, rng):
        self.nts, self.nsb, self.rng = nts, nsb, rng
        self.nq = len(nts)
        self.full = [Bar(1), Bar(1)]      # the four gathering warps modelled as one arrival
        self.tfull = [Bar(1), Bar(1)]
        self.tempty = [Bar(1), Bar(1)]
        self.qfull, self.qempty = Bar(1), Bar(1)
        self.cready = [Bar(1), Bar(1)]
        self.sready = [Bar(1), Bar(1)]
        self.sfree = [Bar(1), Bar(1)]
        self.mread = [Bar(1), Bar(1)]
        self.tma_events = []              # copies in flight (complete in any order)
        self.mma_events = []              # UMMA commits (complete in issue order)
        # buffer ownership for hazard checks
        self.stage_mma_pending = [None, None]   # tile whose UMMA may still read stage s
        self.acc_unread = [None, None]          # tile whose accumulator is not yet read
        self.score_in_use = [None, None]        # query whose top-k may still read buffer b
        self.row_users = [set(), set()]         # (role, query) still reading list row r
        self.qtile_mma_pending = None           # query whose UMMAs may still read the head tile
        self.topk_done = set()

    # ---------------------------------------------------------------- roles
    def wait(self, bar, parity):
        while not bar.done(parity):
            yield

    def build_group(self):
        def build(q):
            r = q & 1
            if q >= 2:
                yield from self.wait(self.mread[r], ((q - 2) >> 1) & 1)
            assert not self.row_users[r], f"row {r} rebuilt for query {q} while read by {self.row_users[r]}"
            self.row_users[r] = {("gather", q), ("mma", q), ("topk", q)}
            self.cready[r].arrive()
        if self.nq:
            yield from build(0)
        for q in range(self.nq):
            if q + 1 < self.nq:
                yield from build(q + 1)
            yield from self.wait(self.sready[q & 1], (q >> 1) & 1)
            sb = q % self.nsb
            if self.nts[q]:  # a query without tiles reads no score columns
                assert self.score_in_use[sb] == q, "top-k reads a buffer holding another query"
            yield                             # the top-k runs
            self.row_users[q & 1].discard(("topk", q))
            self.score_in_use[sb] = None
            self.topk_done.add(q)
            self.sfree[sb].arrive()

    def gather_group(self):
        g = 0
        for q in range(self.nq):
            yield from self.wait(self.cready[q & 1], (q >> 1) & 1)
            nt, sb = self.nts[q], q % self.nsb
            for j in range(nt + 2):
                gj = g + j
                if j >= 2:
                    yield from self.wait(self.tfull[gj & 1], ((gj - 2) >> 1) & 1)
                if j < nt:
                    s = gj & 1
                    assert self.stage_mma_pending[s] is None, f"stage {s} reloaded under tile {self.stage_mma_pending[s]}"
                    self.tma_events.append(("land", s))
                if j == 2 and q >= self.nsb:
                    yield from self.wait(self.sfree[sb], ((q - self.nsb) // self.nsb) & 1)
                if j >= 2:
                    a = gj & 1
                    assert self.acc_unread[a] == gj - 2
                    self.acc_unread[a] = None
                    self.tempty[a].arrive()
                    if j == 2:
                        assert self.score_in_use[sb] is None and (q < self.nsb or q - self.nsb in self.topk_done), \
                            f"score buffer {sb} written for query {q} before the top-k of query {q - self.nsb}"
                        self.score_in_use[sb] = q
                yield
            self.row_users[q & 1].discard(("gather", q))
            self.sready[q & 1].arrive()
            g += nt

    def mma_warp(self):
        g = commits = 0
        for q in range(self.nq):
            yield from self.wait(self.cready[q & 1], (q >> 1) & 1)
            nt = self.nts[q]  # the list length: all this warp reads of the list's slot
            self.row_users[q & 1].discard(("mma", q))
            self.mread[q & 1].arrive()
            if q > 0:
                yield from self.wait(self.qempty, (commits - 1) & 1)
            assert self.qtile_mma_pending is None, "head tile reloaded under running UMMAs"
            self.tma_events.append(("qland", None))
            yield from self.wait(self.qfull, q & 1)
            for j in range(nt):
                gj = g + j
                s = gj & 1
                yield from self.wait(self.full[s], (gj >> 1) & 1)
                if gj >= 2:
                    yield from self.wait(self.tempty[s], ((gj >> 1) & 1) ^ 1)
                assert self.acc_unread[s] is None, "accumulator overwritten before it was read"
                self.stage_mma_pending[s] = gj
                self.qtile_mma_pending = q
                self.mma_events.append(("commit", gj))
                yield
            self.mma_events.append(("qcommit", q))
            commits += 1
            g += nt

    # ------------------------------------------------------- async events
    def fire(self, ev):
        kind, x = ev
        if kind == "land":
            self.full[x].arrive()
        elif kind == "qland":
            self.qfull.arrive()
        elif kind == "commit":
            s = x & 1
            self.stage_mma_pending[s] = None
            self.acc_unread[s] = x
            self.tfull[s].arrive()
        elif kind == "qcommit":
            # every UMMA issued before it has completed
            self.qtile_mma_pending = None
            self.qempty.arrive()

    def run(self):
        roles = [self.build_group(), self.gather_group(), self.mma_warp()]
        live = list(roles)
        steps = 0
        while live or self.tma_events or self.mma_events:
            steps += 1
            assert steps < 200000, "no progress"
            choices = [("role", r) for r in live]
            if self.tma_events:
                choices.append(("tma", None))
            if self.mma_events:
                choices.append(("mma", None))
            kind, r = self.rng.choice(choices)
            if kind == "tma":
                self.fire(self.tma_events.pop(self.rng.randrange(len(self.tma_events))))
                continue
            if kind == "mma":
                self.fire(self.mma_events.pop(0))
                continue
            try:
                next(r)
            except StopIteration:
                live.remove(r)
        assert all(b.pending == 0 for b in self.cready + self.sready + self.sfree)
        assert len(self.topk_done) == self.nq


@pytest.mark.parametrize("nsb", [1, 2])
def test_pipe_protocol_random_schedules(nsb):
    rng = random.Random(1234 + nsb)
    for trial in range(1500):
        nq = rng.randint(0, 7)
        nts = [rng.choice([0, 1, 1, 2, 3, 4, 5]) for _ in range(nq)]
        Model(nts, nsb, random.Random(rng.random())).run()


def test_pipe_protocol_model_catches_a_missing_wait():
    """Planted mistake: the gathering warps skip the score-buffer wait.  The
    model must report the reuse on some schedule."""
    class Broken(Model):
        def wait(self, bar, parity):
            if any(bar is b for b in self.sfree):
                return iter(())
            return Model.wait(self, bar, parity)
    rng = random.Random(7)
    caught = False
    for _ in range(500):
        try:
            Broken([3, 3, 3, 3], 1, random.Random(rng.random())).run()
        except AssertionError:
            caught = True
            break
    assert caught


def test_pipe_protocol_needs_the_length_read_barrier():
    """Without the wait on the UMMA warp's length read, a query with no tiles
    lets its list slot be rebuilt before that warp read the old length: the
    model finds the reuse on some schedule."""
    class NoLengthWait(Model):
        def wait(self, bar, parity):
            if any(bar is b for b in self.mread):
                return iter(())
            return Model.wait(self, bar, parity)
    rng = random.Random(11)
    caught = False
    for _ in range(3000):
        try:
            NoLengthWait([3, 0, 0, 0, 2, 0], 2, random.Random(rng.random())).run()
        except AssertionError:
            caught = True
            break
    assert caught
