"""Model check of the prefill kernel's mbarrier protocol on the CPU.

The prefill attention CTA runs four kinds of actors that meet only at
mbarriers whose waits test the PARITY of a phase (mbarrier.try_wait.parity):
  * the TMA producer: Q once, then K tiles through a 3-stage ring and V tiles
    through a 2-stage ring (full / empty barrier per stage);
  * the MMA thread: S_j = Q K_j^T into S buffer j mod 2 (S_0 and S_1 up front,
    S_{j+2} right after PV_j), and PV_j once P_j is written; its
    tcgen05.commit arrivals fire when every earlier MMA has completed (the
    model's tensor pipe completes operations in issue order);
  * two softmax warpgroups: wait for S_j, exchange their half-row maxima
    through a shared-memory slot pair (red_full[j mod 2]), wait for PV_{j-1}
    before writing P_j over the single P buffer (and rescaling O), and
    at the end exchange their row sums (l_full) and read O after the last PV.

This test replays the protocol with the kernel's stage counts under many
random interleavings, random TMA landing delays and random tensor-pipe
delays, for 1 to 14 tiles, and asserts that every run finishes (no
deadlock), that no barrier ever runs two phases past a waiter (which a
parity wait cannot tell apart), and that every buffer (K / V stages, the S
buffers, P, O, the exchange slots) is read only while it holds the value its
reader expects and overwritten only after its last reader is done."""
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
    def __init__(self, n, rng):
        self.n, self.rng = n, rng
        self.q_full = Bar("q_full", 1)
        self.k_full = [Bar(f"k_full{i}", 1) for i in range(KS)]
        self.k_empty = [Bar(f"k_empty{i}", 1) for i in range(KS)]
        self.v_full = [Bar(f"v_full{i}", 1) for i in range(VS)]
        self.v_empty = [Bar(f"v_empty{i}", 1) for i in range(VS)]
        self.s_full = [Bar("s_full0", 1), Bar("s_full1", 1)]
        self.p_full = Bar("p_full", 8)       # 8 softmax warps
        self.pv_done = Bar("pv_done", 1)
        self.red_full = [Bar("red_full0", 2), Bar("red_full1", 2)]   # one arrival per warpgroup here
        self.l_full = Bar("l_full", 2)
        # buffer contents (tile tags) and progress records
        self.k_stage = [None] * KS
        self.v_stage = [None] * VS
        self.q_loaded = False
        self.s_buf = [None, None]
        self.s_done = set()                   # tiles whose S has been computed
        self.s_reads = {}                     # tile -> warpgroups that read S
        self.p_half = [None, None]            # tile whose P half each warpgroup wrote
        self.pv_completed = -1                # last PV completed (in order)
        self.pv_started = -1
        self.slot = {}                        # (parity, wg) -> tag
        self.slot_reads = {}                  # (tile, wg) -> read done
        self.landing = []                     # (kind, stage, tile, bytes)
        self.pipe = []                        # issued tensor ops in order

    # ---- actors (generators that yield wait predicates) ----
    def tma(self):
        self.landing.append(("q", 0, None, 2))
        self.q_full.arrive(tx=2)
        for j in range(self.n):
            sk, sv = j % KS, j % VS
            if j >= KS:
                yield lambda: self.k_empty[sk].ready(j // KS - 1)
            self.k_full[sk].arrive(tx=2)
            self.landing.append(("k", sk, j, 2))
            if j >= VS:
                yield lambda: self.v_empty[sv].ready(j // VS - 1)
            self.v_full[sv].arrive(tx=2)
            self.landing.append(("v", sv, j, 2))

    def issue_s(self, j):
        yield lambda: self.k_full[j % KS].ready(j // KS)
        self.pipe.append(("S", j))

    def mma(self):
        yield lambda: self.q_full.ready(0)
        yield from self.issue_s(0)
        if self.n > 1:
            yield from self.issue_s(1)
        for j in range(self.n):
            yield lambda: self.p_full.ready(j)
            yield lambda: self.v_full[j % VS].ready(j // VS)
            self.pipe.append(("PV", j))
            if j + 2 < self.n:
                yield from self.issue_s(j + 2)

    def softmax(self, wg):
        for j in range(self.n):
            yield lambda: self.s_full[j & 1].ready(j >> 1)
            assert self.s_buf[j & 1] == j, f"wg{wg} read S buffer {j & 1} holding {self.s_buf[j & 1]}, wanted {j}"
            self.s_reads.setdefault(j, set()).add(wg)
            # exchange half-row maxima
            self.slot[(j & 1, wg)] = ("max", j)
            self.red_full[j & 1].arrive()
            yield lambda: self.red_full[j & 1].ready(j >> 1)
            assert self.slot[(j & 1, 1 - wg)] == ("max", j), f"wg{wg} read a stale or overwritten max slot at tile {j}"
            self.slot_reads[(j, wg)] = True
            if j > 0:
                yield lambda: self.pv_done.ready(j - 1)
                # O may be rescaled now: PV_{j-1} has completed and PV_j cannot start
                assert self.pv_completed >= j - 1 and self.pv_started < j
            # P is overwritten only once the PV that read it has completed
            assert j == 0 or self.pv_completed >= j - 1, "P overwritten under a pending PV"
            self.p_half[wg] = j
            self.p_full.arrive(4)
        last = self.n - 1
        yield lambda: self.pv_done.ready(last)
        # row sums through the slot pair the last tile did not use
        if self.n >= 2:
            assert self.slot_reads.get((self.n - 2, 1 - wg)), "l written over a slot the other warpgroup still reads"
        self.slot[(self.n & 1, wg)] = ("l", wg)
        self.l_full.arrive()
        yield lambda: self.l_full.ready(0)
        assert self.slot[(self.n & 1, 1 - wg)] == ("l", 1 - wg)
        assert self.pv_completed == last

    # ---- asynchronous hardware ----
    def land_one(self):
        i = self.rng.randrange(len(self.landing))
        kind, stage, j, tx = self.landing.pop(i)
        if kind == "q":
            self.q_loaded = True
            self.q_full.complete_tx(tx)
        elif kind == "k":
            assert j < KS or (self.k_stage[stage] == j - KS and j - KS in self.s_done), \
                "K stage overwritten before its S was done"
            self.k_stage[stage] = j
            self.k_full[stage].complete_tx(tx)
        else:
            assert j < VS or (self.v_stage[stage] == j - VS and self.pv_completed >= j - VS), \
                "V stage overwritten before its PV was done"
            self.v_stage[stage] = j
            self.v_full[stage].complete_tx(tx)

    def run_pipe(self):
        kind, j = self.pipe.pop(0)
        if kind == "S":
            assert self.q_loaded and self.k_stage[j % KS] == j, f"S_{j} read the wrong K stage"
            if j >= 2:
                assert self.s_reads.get(j - 2) == {0, 1}, f"S_{j} overwrote S_{j - 2} before both warpgroups read it"
            self.s_buf[j & 1] = j
            self.s_done.add(j)
            self.k_empty[j % KS].arrive()
            self.s_full[j & 1].arrive()
        else:
            assert self.p_half == [j, j], f"PV_{j} read P halves of tiles {self.p_half}"
            assert self.v_stage[j % VS] == j, f"PV_{j} read the wrong V stage"
            self.pv_started = j
            self.pv_completed = j
            self.v_empty[j % VS].arrive()
            self.pv_done.arrive()


def run(n, seed):
    rng = random.Random(seed)
    m = Model(n, rng)
    actors = {"tma": m.tma(), "mma": m.mma(), "sm0": m.softmax(0), "sm1": m.softmax(1)}
    waits = {name: None for name in actors}
    done = set()
    for _ in range(200_000):
        if len(done) == len(actors) and not m.pipe and not m.landing:
            return
        choices = [name for name in actors if name not in done and (waits[name] is None or waits[name]())]
        if m.landing:
            choices.append("land")
        if m.pipe:
            choices.append("pipe")
        assert choices, f"deadlock at n={n}: waiting {[k for k in actors if k not in done]}"
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
    for seed in range(150):
        run(n, 1000 * n + seed)


def test_the_model_catches_a_broken_protocol():
    """With the softmax not waiting for the previous PV before writing P, the
    model must find P overwritten under a pending PV."""
    class Broken(Model):
        def softmax(self, wg):
            for j in range(self.n):
                yield lambda: self.s_full[j & 1].ready(j >> 1)
                self.s_reads.setdefault(j, set()).add(wg)
                self.slot[(j & 1, wg)] = ("max", j)
                self.red_full[j & 1].arrive()
                yield lambda: self.red_full[j & 1].ready(j >> 1)
                self.slot_reads[(j, wg)] = True
                self.p_half[wg] = j          # no wait for PV_{j-1}
                self.p_full.arrive(4)
            yield lambda: self.pv_done.ready(self.n - 1)
            self.l_full.arrive()
            yield lambda: self.l_full.ready(0)

    failures = 0
    for seed in range(300):
        rng = random.Random(seed)
        m = Broken(6, rng)
        actors = {"tma": m.tma(), "mma": m.mma(), "sm0": m.softmax(0), "sm1": m.softmax(1)}
        waits = {k: None for k in actors}
        done = set()
        try:
            for _ in range(100_000):
                if len(done) == len(actors) and not m.pipe and not m.landing:
                    break
                choices = [k for k in actors if k not in done and (waits[k] is None or waits[k]())]
                if m.landing:
                    choices.append("land")
                if m.pipe:
                    choices.append("pipe")
                if not choices:
                    raise AssertionError("deadlock")
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
        except AssertionError:
            failures += 1
    assert failures > 0
