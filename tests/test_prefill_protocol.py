"""Model check of the prefill kernel's mbarrier protocol on the CPU.

A prefill attention CTA is persistent: it walks a list of units (a block of
16 query tokens for one KV head), with its tiles counted across units.  Four
kinds of actors meet only at mbarriers whose waits test the PARITY of a
phase (mbarrier.try_wait.parity):
  * the TMA producer: per unit the Q tile (once q_empty says the previous
    unit's S MMAs are done with the buffer), then the unit's K tiles through
    a 3-stage ring and V tiles through a 2-stage ring (full / empty barrier
    per stage, phases counted across units);
  * the MMA thread: per unit S of the first two tiles (after q_full), then
    per tile PV_j once P_j is written (the unit's first PV overwrites O: the
    softmax warps read the previous unit's O out before writing that P) and
    S two tiles ahead within the unit; the next unit's first S come after
    this unit's last PV.  S_j goes into S buffer j mod 2; the unit's last S also
    commits q_empty.  Its tcgen05.commit arrivals fire when every earlier MMA
    has completed (the model's tensor pipe completes operations in issue
    order);
  * two softmax warpgroups: per tile wait for S_j, exchange the half-row
    maxima through a shared-memory slot pair (red_full[j mod 2]), wait for
    PV_{j-1} before writing P_j over the single P buffer (and, inside a unit,
    rescaling O); at the unit's end wait for its last PV, exchange the row
    sums through their own slots (l_full, a phase per unit) and read O.

This test replays the protocol with the kernel's stage counts under many
random interleavings, random TMA landing delays and random tensor-pipe
delays, for units of 1 to 14 tiles and lists of 1 to 5 units, and asserts
that every run finishes (no deadlock), that no barrier ever runs two phases
past a waiter (which a parity wait cannot tell apart), and that every buffer
(Q, the K / V stages, the S buffers, P, O, the exchange slots) is read only
while it holds the value its reader expects and overwritten only after its
last reader is done.  Variants that drop one of the waits are caught."""
import random

import pytest

KS, VS = 3, 2


class Bar:
    def __init__(self, name, count):
        self.name, self.count, self.pending, self.tx, self.done = name, count, count, 0, 0

    def arrive(self, n=1, tx=0):
        self.tx += tx
        self.pending -= n
        assert self.pending >= 0, f"{self.name}: too many arrivals"
        self._check()

    def complete_tx(self, tx):
        self.tx -= tx
        self._check()

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.done += 1
            self.pending = self.count

    def ready(self, phase):
        """The parity wait for `phase` (0-based) succeeds."""
        assert self.done <= phase + 1, f"{self.name}: ran {self.done - phase - 1} phase(s) past a waiter of phase {phase}"
        return self.done >= phase + 1


class Model:
    """units: tile counts of the CTA's units.  Flags drop one wait each (the
    mutants the tests must catch)."""

    def __init__(self, units, rng, skip_pv_wait=False, late_o_read=False, skip_q_empty=False):
        self.units, self.rng = list(units), rng
        self.skip_pv_wait, self.late_o_read, self.skip_q_empty = skip_pv_wait, late_o_read, skip_q_empty
        self.base = [sum(self.units[:i]) for i in range(len(self.units))]  # first tile of each unit
        self.unit_of_tile = [i for i, n in enumerate(self.units) for _ in range(n)]
        self.n_tiles = sum(self.units)
        self.q_full = Bar("q_full", 1)
        self.q_empty = Bar("q_empty", 1)
        self.k_full = [Bar(f"k_full{i}", 1) for i in range(KS)]
        self.k_empty = [Bar(f"k_empty{i}", 1) for i in range(KS)]
        self.v_full = [Bar(f"v_full{i}", 1) for i in range(VS)]
        self.v_empty = [Bar(f"v_empty{i}", 1) for i in range(VS)]
        self.s_full = [Bar("s_full0", 1), Bar("s_full1", 1)]
        self.p_full = Bar("p_full", 8)
        self.pv_done = Bar("pv_done", 1)
        self.red_full = [Bar("red_full0", 2), Bar("red_full1", 2)]   # one arrival per warpgroup here
        self.l_full = Bar("l_full", 2)
        # buffer contents (tags) and progress records
        self.q_buf = None                     # unit whose Q is in the buffer
        self.k_stage = [None] * KS
        self.v_stage = [None] * VS
        self.s_buf = [None, None]
        self.s_done = set()                   # tiles whose S has been computed
        self.s_reads = {}                     # tile -> warpgroups that read S
        self.p_half = [None, None]            # tile whose P half each warpgroup wrote
        self.o = None                         # (unit, last tile folded into O)
        self.o_reads = set()                  # (unit, wg) that read O out
        self.pv_completed = -1                # last PV completed (in order)
        self.slot = {}                        # (parity, wg) -> tag
        self.slot_reads = {}                  # (tile, wg) -> read done
        self.lslot = [None, None]             # per warpgroup: unit whose row sums it holds
        self.l_reads = set()                  # (unit, wg) that read the other half's l
        self.landing = []                     # (kind, stage, tag, bytes)
        self.pipe = []                        # issued tensor ops in order

    # ---- actors (generators that yield wait predicates) ----
    def tma(self):
        for i, n in enumerate(self.units):
            if i > 0 and not self.skip_q_empty:
                yield lambda: self.q_empty.ready(i - 1)
            self.q_full.arrive(tx=2)
            self.landing.append(("q", 0, i, 2))
            for jj in range(n):
                j = self.base[i] + jj
                sk, sv = j % KS, j % VS
                if j >= KS:
                    yield lambda: self.k_empty[sk].ready(j // KS - 1)
                self.k_full[sk].arrive(tx=2)
                self.landing.append(("k", sk, j, 2))
                if j >= VS:
                    yield lambda: self.v_empty[sv].ready(j // VS - 1)
                self.v_full[sv].arrive(tx=2)
                self.landing.append(("v", sv, j, 2))

    def issue_s(self, j, last):
        yield lambda: self.k_full[j % KS].ready(j // KS)
        self.pipe.append(("S", j, last))

    def mma(self):
        for i, n in enumerate(self.units):
            t0 = self.base[i]
            if i == 0:
                yield lambda: self.q_full.ready(0)
                yield from self.issue_s(t0, n == 1)
                if n > 1:
                    yield from self.issue_s(t0 + 1, n == 2)
            for jj in range(n):
                j = t0 + jj
                yield lambda: self.p_full.ready(j)
                yield lambda: self.v_full[j % VS].ready(j // VS)
                self.pipe.append(("PV", j, jj == 0))
                if jj + 2 < n:
                    yield from self.issue_s(j + 2, jj + 2 == n - 1)
            if i + 1 < len(self.units):
                nn, t1 = self.units[i + 1], self.base[i + 1]
                yield lambda: self.q_full.ready(i + 1)
                yield from self.issue_s(t1, nn == 1)
                if nn > 1:
                    yield from self.issue_s(t1 + 1, nn == 2)

    def read_o(self, wg, i, last):
        assert self.o == (i, last), f"wg{wg} read O holding {self.o} at the end of unit {i}"
        self.o_reads.add((i, wg))

    def softmax(self, wg):
        pending_o = None  # late_o_read: the previous unit's O, read after this unit's first P
        for i, n in enumerate(self.units):
            for jj in range(n):
                j = self.base[i] + jj
                yield lambda: self.s_full[j & 1].ready(j >> 1)
                assert self.s_buf[j & 1] == j, f"wg{wg} read S buffer {j & 1} holding {self.s_buf[j & 1]}, wanted {j}"
                self.s_reads.setdefault(j, set()).add(wg)
                # exchange half-row maxima
                self.slot[(j & 1, wg)] = ("max", j)
                self.red_full[j & 1].arrive()
                yield lambda: self.red_full[j & 1].ready(j >> 1)
                assert self.slot[(j & 1, 1 - wg)] == ("max", j), f"wg{wg} read a stale or overwritten max slot at tile {j}"
                self.slot_reads[(j, wg)] = True
                if j > 0 and not self.skip_pv_wait:
                    yield lambda: self.pv_done.ready(j - 1)
                if jj > 0:
                    # O may be rescaled now: it holds this unit's PVs through j - 1
                    assert self.o == (i, j - 1), f"wg{wg} rescaled O holding {self.o} at tile {j} of unit {i}"
                # P is overwritten only once the PV that read it has completed
                assert j == 0 or self.pv_completed >= j - 1, "P overwritten under a pending PV"
                self.p_half[wg] = j
                self.p_full.arrive(4)
                if pending_o is not None:
                    yield None
                    self.read_o(wg, *pending_o)
                    pending_o = None
            last = self.base[i] + n - 1
            yield lambda: self.pv_done.ready(last)
            # row sums through their own slots
            if i > 0:
                assert (i - 1, 1 - wg) in self.l_reads, "l written over a slot the other warpgroup still reads"
            self.lslot[wg] = ("l", i)
            self.l_full.arrive()
            yield lambda: self.l_full.ready(i)
            assert self.lslot[1 - wg] == ("l", i), f"wg{wg} read row sums {self.lslot[1 - wg]} in unit {i}"
            self.l_reads.add((i, wg))
            if self.late_o_read and i + 1 < len(self.units):
                pending_o = (i, last)
            else:
                self.read_o(wg, i, last)

    # ---- asynchronous hardware ----
    def land_one(self):
        i = self.rng.randrange(len(self.landing))
        kind, stage, tag, tx = self.landing.pop(i)
        if kind == "q":
            if tag > 0:
                prev = self.base[tag - 1]
                assert all(t in self.s_done for t in range(prev, prev + self.units[tag - 1])), \
                    f"Q of unit {tag} landed over unit {tag - 1}'s Q while its S MMAs were pending"
            self.q_buf = tag
            self.q_full.complete_tx(tx)
        elif kind == "k":
            j = tag
            assert j < KS or (self.k_stage[stage] == j - KS and j - KS in self.s_done), \
                "K stage overwritten before its S was done"
            self.k_stage[stage] = j
            self.k_full[stage].complete_tx(tx)
        else:
            j = tag
            assert j < VS or (self.v_stage[stage] == j - VS and self.pv_completed >= j - VS), \
                "V stage overwritten before its PV was done"
            self.v_stage[stage] = j
            self.v_full[stage].complete_tx(tx)

    def run_pipe(self):
        op = self.pipe.pop(0)
        if op[0] == "S":
            _, j, last = op
            unit = self.unit_of_tile[j]
            assert self.q_buf == unit, f"S_{j} of unit {unit} read the Q of unit {self.q_buf}"
            assert self.k_stage[j % KS] == j, f"S_{j} read the wrong K stage"
            if j >= 2:
                assert self.s_reads.get(j - 2) == {0, 1}, f"S_{j} overwrote S_{j - 2} before both warpgroups read it"
            self.s_buf[j & 1] = j
            self.s_done.add(j)
            self.k_empty[j % KS].arrive()
            self.s_full[j & 1].arrive()
            if last:
                self.q_empty.arrive()
        else:
            _, j, first = op
            unit = self.unit_of_tile[j]
            assert self.p_half == [j, j], f"PV_{j} read P halves of tiles {self.p_half}"
            assert self.v_stage[j % VS] == j, f"PV_{j} read the wrong V stage"
            if first:
                assert unit == 0 or {(unit - 1, 0), (unit - 1, 1)} <= self.o_reads, \
                    f"PV_{j} overwrote O before unit {unit - 1}'s O was read out"
            else:
                assert self.o == (unit, j - 1), f"PV_{j} accumulated onto O holding {self.o}"
            self.o = (unit, j)
            self.pv_completed = j
            self.v_empty[j % VS].arrive()
            self.pv_done.arrive()


def run(units, seed, **flags):
    rng = random.Random(seed)
    m = Model(units, rng, **flags)
    actors = {"tma": m.tma(), "mma": m.mma(), "sm0": m.softmax(0), "sm1": m.softmax(1)}
    waits = {name: None for name in actors}
    done = set()
    for _ in range(400_000):
        if len(done) == len(actors) and not m.pipe and not m.landing:
            return
        choices = [name for name in actors if name not in done and (waits[name] is None or waits[name]())]
        if m.landing:
            choices.append("land")
        if m.pipe:
            choices.append("pipe")
        assert choices, f"deadlock at units={units}: waiting {[k for k in actors if k not in done]}"
        pick = rng.choice(choices)
        if pick == "land":
            m.land_one()
        elif pick == "pipe":
            m.run_pipe()
        else:
            try:
                waits[pick] = next(actors[pick])
            except StopIteration:
                done.add(pick)
    raise AssertionError("did not finish")


@pytest.mark.parametrize("n", list(range(1, 15)))
def test_prefill_protocol_random_interleavings(n):
    """One unit of n tiles (a CTA with a single unit)."""
    for seed in range(150):
        run([n], 1000 * n + seed)


@pytest.mark.parametrize("seed0", range(6))
def test_prefill_protocol_across_units(seed0):
    """A persistent CTA's list of units, long and short mixed (1 to 9 tiles,
    1 to 5 units): Q is reloaded and O handed over at every boundary."""
    rng = random.Random(seed0)
    for trial in range(60):
        units = [rng.randint(1, 9) for _ in range(rng.randint(1, 5))]
        run(units, 100_000 * seed0 + trial)


def caught(units, n_seeds, **flags):
    failures = 0
    for seed in range(n_seeds):
        try:
            run(units, seed, **flags)
        except AssertionError:
            failures += 1
    return failures


def test_the_model_catches_a_softmax_that_does_not_wait_for_the_previous_pv():
    """P would be overwritten under a pending PV."""
    assert caught([6], 300, skip_pv_wait=True) > 0


def test_the_model_catches_o_read_after_the_next_units_first_p():
    """The kernel needs no barrier of its own for O: each softmax warp reads O
    out before it writes its half of the next unit's first P, and that PV,
    which overwrites O, waits for all of P.  A softmax that read O only after
    writing that P would lose it."""
    assert caught([3, 2, 4], 300, late_o_read=True) > 0


def test_the_model_catches_a_producer_that_does_not_wait_for_q_empty():
    """The next unit's Q would land while the previous unit's S MMAs still read Q."""
    assert caught([4, 3, 5], 300, skip_q_empty=True) > 0
