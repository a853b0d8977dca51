"""Model check, on the CPU, of what the decode and prefill kernels do when a
bounded wait runs out (FLINT_ERR_TIMEOUT).

Every mbarrier wait in both kernels gives up after a time limit, or at once
once the CTA's abort flag is up (after one failed test of the barrier).  A
CTA that gives up must still leave nothing in flight when it exits: a TMA or
bulk copy that lands after the CTA is gone would write into shared memory
that the next CTA on the SM owns, and a tensor-core MMA still running when
the TMEM columns are freed would write into another CTA's accumulators.  So
each kernel ends with a drain: the decode kernel's producer waits (bounded)
for the phases of the last item inputs and of the last kStages tiles it
issued; the persistent prefill kernel's producer waits for the last Q, K
and V phases it issued (a Q tile per unit), and its MMA thread waits for a
commit that fires once every MMA it issued has completed, before TMEM is
freed; the prefill norm/RoPE kernel's producer waits for the slots of the
last tokens it handed out.

The models below replay each kernel's protocol with random interleavings,
random landing times of the copies and of the tensor pipe, and random
time-outs (any blocked wait may give up; the first one raises the abort
flag), plus runs where the producer never arms one chosen stage (the GPU
test hook).  They assert that every run ends, that the status is TIMEOUT
exactly when a wait gave up, that no consumer reads a stage before the tile
it expects has landed, and that when the CTA exits no copy is in flight and
no MMA is pending.  A drain keyed on the tile count instead of the tiles
actually issued is shown to exit with a copy in flight.
"""
import random

import pytest


class Bar:
    """An mbarrier: `count` arrivals plus a transaction byte count per phase;
    waits test the parity of a phase."""

    def __init__(self, count):
        self.count, self.pending, self.tx, self.done = count, count, 0, 0

    def arrive(self, tx=0):
        self.tx += tx
        self.pending -= 1
        assert self.pending >= 0, "too many arrivals in a phase"
        self._check()

    def complete_tx(self, tx):
        self.tx -= tx
        self._check()

    def _check(self):
        if self.pending == 0 and self.tx == 0:
            self.done += 1
            self.pending = self.count

    def parity_ok(self, parity):
        # try_wait.parity(P) succeeds once the phase of parity P has completed,
        # i.e. while the current (incomplete) phase has the other parity
        return (self.done & 1) != parity


class Cta:
    """Shared state of one CTA: the abort flag, the status, in-flight copies."""

    def __init__(self, rng, p_timeout):
        self.rng = rng
        self.p_timeout = p_timeout
        self.abort = False
        self.status = 0
        self.gave_up = 0
        self.landing = []  # (barrier, tx, tag)

    def wait(self, bar, parity):
        """Generator of one bounded wait: yields until the phase completed
        (returns True) or the wait gives up (returns False).  A waiter that
        finds the phase incomplete gives up at once if the abort flag is up,
        or at a random moment (its time limit)."""
        while True:
            if bar.parity_ok(parity):
                return True
            if self.abort:
                return False
            if self.rng.random() < self.p_timeout:
                self.gave_up += 1
                return False
            yield

    def raise_abort(self):
        if not self.abort:
            self.status = 5  # FLINT_ERR_TIMEOUT
        self.abort = True

    def land_one(self):
        i = self.rng.randrange(len(self.landing))
        bar, tx, tag = self.landing.pop(i)
        tag["landed"] = True
        bar.complete_tx(tx)


def run_actors(cta, actors, pipe=None, limit=400_000):
    """Round-robin at random over the actors' generators, the landing of
    copies and the tensor pipe, until every actor has returned."""
    live = dict(actors)
    for _ in range(limit):
        if not live:
            return
        choices = list(live)
        if cta.landing:
            choices.append("land")
        if pipe is not None and pipe.ops:
            choices.append("pipe")
        pick = cta.rng.choice(choices)
        if pick == "land":
            cta.land_one()
        elif pick == "pipe":
            pipe.run_one()
        else:
            try:
                next(live[pick])
            except StopIteration:
                del live[pick]
    raise AssertionError("the model did not finish")


# ---------------------------------------------------------------------------
# decode_kernel: one producer warp, consumer warps that all take part in
# every stage, items with staged inputs (in_full / in_empty).

def decode_run(items, stages, warps, rng, p_timeout, stall_at=None, drain="issued", sticky=True):
    """items: tiles per item.  stall_at: tile sequence number whose stage the
    producer never arms (the test hook).  sticky: the kernel's abort rule
    (consumers stop waiting, reading and releasing stages once the flag is
    up; the producer arms nothing more once it sees the flag after a wait);
    sticky=False keeps every warp walking its waits after an abort.  Returns
    the Cta after the exit checks."""
    cta = Cta(rng, p_timeout)
    full = [Bar(1) for _ in range(stages)]
    empty = [Bar(warps) for _ in range(stages)]
    in_full, in_empty = Bar(1), Bar(warps)
    stage_tile = [None] * stages
    res = {}
    item_slot = {"k": None}

    def producer():
        seq = 0
        for k in range(len(items) + 1):
            ok = yield from cta.wait(in_empty, (k & 1) ^ 1)
            if not ok:
                cta.raise_abort()
                res["pc"] = (seq, k)
                return
            item_slot["k"] = k if k < len(items) else -1
            if k < len(items):
                tag = {"landed": False}
                in_full.arrive(tx=1)
                cta.landing.append((in_full, 1, tag))
            else:
                in_full.arrive()
                res["pc"] = (seq, k + 1)
                return
            for _ in range(items[k]):
                s = seq % stages
                ok = yield from cta.wait(empty[s], ((seq // stages) & 1) ^ 1)
                if not ok or (sticky and cta.abort):
                    cta.raise_abort()
                    res["pc"] = (seq, k + 1)
                    return
                if seq != stall_at:
                    old = stage_tile[s]
                    assert old is None or old["landed"], f"stage {s} re-armed while tile {old['seq']} is landing"
                    tag = {"landed": False, "seq": seq}
                    stage_tile[s] = tag
                    full[s].arrive(tx=1)
                    cta.landing.append((full[s], 1, tag))
                seq += 1

    consumed = []

    def consumer(w):
        seq = 0
        k = 0
        while True:
            ok = yield from cta.wait(in_full, k & 1)
            if not ok:
                cta.raise_abort()
                return
            it = item_slot["k"]
            if it is None or it < 0:
                return
            in_empty.arrive()
            for _ in range(items[it]):
                s = seq % stages
                if sticky and cta.abort:
                    seq += 1  # walk on to the item-end barriers without waiting
                    continue
                ok = yield from cta.wait(full[s], (seq // stages) & 1)
                if ok:
                    tag = stage_tile[s]
                    if not cta.abort:
                        assert tag is not None and tag["seq"] == seq and tag["landed"], \
                            f"warp {w} read stage {s} for tile {seq} before it landed"
                    consumed.append(seq)
                    empty[s].arrive()
                else:
                    cta.raise_abort()
                seq += 1
            k += 1
            yield

    # the consumer warps meet at named barriers; the model lets them run free,
    # which only adds interleavings (the item hand-over is checked elsewhere)
    actors = {"producer": producer()}
    for w in range(warps):
        actors[f"c{w}"] = consumer(w)
    run_actors(cta, actors)

    # the drain after __syncthreads (producer lane 0), bounded waits that here
    # may also give up at any time, but copies can land while they wait
    issued, staged = res["pc"]

    def bounded(bar, parity):
        # a copy lands within microseconds, far inside the drain's limit; the
        # wait runs out only on a phase that nothing will complete
        while not bar.parity_ok(parity):
            if not any(b is bar for b, _, _ in cta.landing):
                return
            cta.land_one()

    if staged > 0:
        bounded(in_full, (staged - 1) & 1)
    n_tiles = sum(items)
    last = issued if drain == "issued" else n_tiles
    for s in range(max(0, last - stages), last):
        bounded(full[s % stages], (s // stages) & 1)
    cta.in_flight_at_exit = len(cta.landing)
    return cta


@pytest.mark.parametrize("stages,warps", [(3, 8), (3, 4), (6, 8)])
def test_decode_abort_leaves_nothing_in_flight(stages, warps):
    rng = random.Random(100 * stages + warps)
    for trial in range(400):
        items = [rng.randint(1, 9) for _ in range(rng.randint(1, 5))]
        p = rng.choice([0.0, 0.001, 0.01, 0.05, 0.3])
        cta = decode_run(items, stages, warps, rng, p)
        assert cta.in_flight_at_exit == 0, f"trial {trial}: a copy is in flight at exit ({items}, p={p})"
        assert (cta.status == 5) == (cta.gave_up > 0), f"trial {trial}: status {cta.status}, gave up {cta.gave_up}"


def test_decode_stalled_stage_times_out_and_drains():
    """The GPU test hook: the producer never arms one stage.  The consumers
    give up on it (no other time-outs), the status is TIMEOUT and nothing is
    in flight at exit."""
    rng = random.Random(5)
    for trial in range(300):
        items = [rng.randint(1, 9) for _ in range(rng.randint(1, 4))]
        stall = rng.randrange(sum(items))
        cta = decode_run(items, 3, 8, rng, p_timeout=0.0005, stall_at=stall)
        assert cta.status == 5 and cta.in_flight_at_exit == 0, f"trial {trial}"


def test_decode_abort_without_the_sticky_rule_is_caught():
    """If warps keep walking their waits after an abort, a warp that gave up
    on tile s passes the parity wait of tile s + stages on the phase of tile
    s - stages, releases the stage, and the producer re-arms it while tile
    s is still landing (or the drain misses a copy)."""
    rng = random.Random(21)
    caught = 0
    for trial in range(600):
        items = [rng.randint(4, 12) for _ in range(3)]
        try:
            cta = decode_run(items, 3, 8, rng, 0.05, sticky=False)
            caught += cta.in_flight_at_exit > 0
        except AssertionError:
            caught += 1
    assert caught > 0


def test_decode_drain_keyed_on_the_plan_is_caught():
    """Waiting on the last phases of the whole plan instead of the tiles
    issued lets a parity wait pass on an older phase while the copy of the
    newest one is still landing."""
    rng = random.Random(9)
    caught = 0
    for trial in range(600):
        items = [rng.randint(4, 12) for _ in range(3)]
        cta = decode_run(items, 3, 8, rng, 0.05, drain="plan")
        caught += cta.in_flight_at_exit > 0
    assert caught > 0


# ---------------------------------------------------------------------------
# prefill_kernel: TMA producer (Q, then K / V tiles through 3- and 2-stage
# rings), one MMA-issuing thread (S into two TMEM buffers, P V), two softmax
# warpgroups; the tensor pipe runs issued MMAs in order.

KS, VS = 3, 2


class Pipe:
    def __init__(self, rng):
        self.rng = rng
        self.ops = []  # (on_done callbacks) in issue order

    def issue(self, *callbacks):
        self.ops.append(callbacks)

    def run_one(self):
        for cb in self.ops.pop(0):
            cb()


def prefill_run(units, rng, p_timeout, stall_k=None, drain="issued"):
    """units: tile counts of the persistent CTA's units (an int: one unit).
    stall_k: the CTA's K tile (counted across units) the producer never arms.
    drain: "issued" (the kernel: the last Q, K and V phases the producer
    issued) or "count" (as if every tile of every unit had been issued)."""
    if isinstance(units, int):
        units = [units]
    n_tiles = sum(units)
    cta = Cta(rng, p_timeout)
    pipe = Pipe(rng)
    q_full, q_empty = Bar(1), Bar(1)
    k_full, k_empty = [Bar(1) for _ in range(KS)], [Bar(1) for _ in range(KS)]
    v_full, v_empty = [Bar(1) for _ in range(VS)], [Bar(1) for _ in range(VS)]
    s_full = [Bar(1), Bar(1)]
    p_full, pv_done, mma_done = Bar(2), Bar(1), Bar(1)
    red_full = [Bar(2), Bar(2)]
    l_full = Bar(2)
    k_tag, v_tag = [None] * KS, [None] * VS
    q_tag = [None]
    res = {}

    def load(bar, tags, slot, tile):
        tag = {"landed": False, "tile": tile}
        if tags is not None:
            tags[slot] = tag
        bar.arrive(tx=1)
        cta.landing.append((bar, 1, tag))

    def tma():
        nk = nv = nq = 0
        j = 0
        for i, n in enumerate(units):
            if i > 0:
                ok = yield from cta.wait(q_empty, (i - 1) & 1)
                if not ok:
                    cta.raise_abort()
                    res["tma"] = (nk, nv, nq)
                    return
            if cta.abort:
                res["tma"] = (nk, nv, nq)
                return
            old = q_tag[0]
            assert old is None or old["landed"], f"Q of unit {i} issued while unit {i - 1}'s Q is landing"
            load(q_full, q_tag, 0, i)
            nq += 1
            for _ in range(n):
                sk, sv = j % KS, j % VS
                if j >= KS:
                    ok = yield from cta.wait(k_empty[sk], (j // KS - 1) & 1)
                    if not ok:
                        cta.raise_abort()
                        res["tma"] = (nk, nv, nq)
                        return
                if j != stall_k:
                    load(k_full[sk], k_tag, sk, j)
                nk += 1
                if j >= VS:
                    ok = yield from cta.wait(v_empty[sv], (j // VS - 1) & 1)
                    if not ok:
                        cta.raise_abort()
                        res["tma"] = (nk, nv, nq)
                        return
                load(v_full[sv], v_tag, sv, j)
                nv += 1
                j += 1
        res["tma"] = (nk, nv, nq)

    def issue_s(j, last):
        ok = yield from cta.wait(k_full[j % KS], (j // KS) & 1)
        if not ok:
            return False
        tag = k_tag[j % KS]
        assert tag["tile"] == j and tag["landed"], f"S_{j} issued on a K stage that does not hold tile {j}"
        cbs = [lambda: k_empty[j % KS].arrive(), lambda: s_full[j & 1].arrive()]
        if last:
            cbs.append(lambda: q_empty.arrive())
        pipe.issue(*cbs)
        return True

    def mma():
        base = 0
        ok = yield from cta.wait(q_full, 0)
        if ok:
            ok = yield from issue_s(0, units[0] == 1)
        if ok and units[0] > 1:
            ok = yield from issue_s(1, units[0] == 2)
        for i, n in enumerate(units):
            if not ok:
                break
            for jj in range(n):
                j = base + jj
                ok = yield from cta.wait(p_full, j & 1)
                if ok:
                    ok = yield from cta.wait(v_full[j % VS], (j // VS) & 1)
                if not ok:
                    break
                pipe.issue(lambda j=j: v_empty[j % VS].arrive(), lambda: pv_done.arrive())
                if jj + 2 < n:
                    ok = yield from issue_s(j + 2, jj + 2 == n - 1)
                    if not ok:
                        break
            if not ok:
                break
            base += n
            if i + 1 < len(units):
                nn = units[i + 1]
                ok = yield from cta.wait(q_full, (i + 1) & 1)
                if ok:
                    ok = yield from issue_s(base, nn == 1)
                if ok and nn > 1:
                    ok = yield from issue_s(base + 1, nn == 2)
        if not ok:
            cta.raise_abort()
        # commit: fires once every MMA issued so far has completed
        pipe.issue(lambda: mma_done.arrive())
        while not mma_done.parity_ok(0):
            yield  # the wait is bounded in the kernel; the pipe always drains here
        res["mma_idle"] = not pipe.ops

    def softmax(wg):
        ok = True
        j = 0
        for i, n in enumerate(units):
            for _ in range(n):
                ok = yield from cta.wait(s_full[j & 1], (j >> 1) & 1)
                if not ok:
                    break
                red_full[j & 1].arrive()
                ok = yield from cta.wait(red_full[j & 1], (j >> 1) & 1)
                if not ok:
                    break
                if j > 0:
                    ok = yield from cta.wait(pv_done, (j - 1) & 1)
                    if not ok:
                        break
                p_full.arrive()
                j += 1
            if ok:
                ok = yield from cta.wait(pv_done, (j - 1) & 1)
            l_full.arrive()
            if ok:
                ok = yield from cta.wait(l_full, i & 1)
            if not ok:
                cta.raise_abort()
                return

    run_actors(cta, {"tma": tma(), "mma": mma(), "sm0": softmax(0), "sm1": softmax(1)}, pipe)
    # after __syncthreads: the producer drains if the CTA aborted, then TMEM
    # is freed (the MMA thread waited for its commit above)
    assert res.get("mma_idle", True), "TMEM freed while an MMA is pending"

    def bounded(bar, parity):
        # a copy lands within microseconds, far inside the drain's limit; the
        # wait runs out only on a phase that nothing will complete
        while not bar.parity_ok(parity):
            if not any(b is bar for b, _, _ in cta.landing):
                return
            cta.land_one()

    if cta.abort:
        nk, nv, nq = res["tma"] if drain == "issued" else (n_tiles, n_tiles, len(units))
        if nq > 0:
            bounded(q_full, (nq - 1) & 1)
        for j in range(max(0, nk - KS), nk):
            bounded(k_full[j % KS], (j // KS) & 1)
        for j in range(max(0, nv - VS), nv):
            bounded(v_full[j % VS], (j // VS) & 1)
    cta.in_flight_at_exit = len(cta.landing)
    return cta


@pytest.mark.parametrize("n", [1, 2, 3, 5, 8, 13])
def test_prefill_abort_leaves_nothing_in_flight(n):
    rng = random.Random(n)
    for trial in range(300):
        p = rng.choice([0.0, 0.001, 0.01, 0.05, 0.3])
        cta = prefill_run(n, rng, p)
        assert cta.in_flight_at_exit == 0, f"trial {trial}: a copy is in flight at exit (n={n}, p={p})"
        assert (cta.status == 5) == (cta.gave_up > 0)


def test_prefill_abort_across_units_leaves_nothing_in_flight():
    """A persistent CTA's units (Q reloaded per unit): the drain also waits
    for the last Q it issued."""
    rng = random.Random(31)
    for trial in range(400):
        units = [rng.randint(1, 7) for _ in range(rng.randint(2, 5))]
        p = rng.choice([0.0, 0.001, 0.01, 0.05, 0.3])
        cta = prefill_run(units, rng, p)
        assert cta.in_flight_at_exit == 0, f"trial {trial}: a copy is in flight at exit ({units}, p={p})"
        assert (cta.status == 5) == (cta.gave_up > 0)


def test_prefill_stalled_k_stage_times_out_and_drains():
    rng = random.Random(11)
    for trial in range(300):
        units = [rng.randint(1, 8) for _ in range(rng.randint(1, 3))]
        cta = prefill_run(units, rng, 0.0005, stall_k=rng.randrange(sum(units)))
        assert cta.status == 5 and cta.in_flight_at_exit == 0, f"trial {trial}"


def test_prefill_drain_keyed_on_the_tile_count_is_caught():
    """A drain over the last phases of all tiles, as if every tile had been
    issued, passes parity waits on older phases while an issued copy is still
    landing when the producer gave up early."""
    rng = random.Random(12)
    caught = 0
    for trial in range(600):
        units = [rng.randint(3, 8) for _ in range(rng.randint(1, 3))]
        cta = prefill_run(units, rng, 0.05, drain="count")
        caught += cta.in_flight_at_exit > 0
    assert caught > 0


# ---------------------------------------------------------------------------
# prefill_prep_kernel: one producer warp fills a ring of token slots (the
# expected bytes raised first, the copies issued, then the warp's arrivals);
# every consumer warp reads every token's slot and releases it.

def prep_run(n, slots, warps, rng, p_timeout, stall_k=None, drain="handed_out"):
    """n: tokens of the CTA's range.  stall_k: token whose slot the producer
    never arms (the test hook).  drain: "handed_out" (the kernel: the last
    `slots` tokens the producer got to) or "range" (the last `slots` tokens
    of the whole range, a mistake the tests below catch)."""
    cta = Cta(rng, p_timeout)
    full = [Bar(1) for _ in range(slots)]
    empty = [Bar(warps) for _ in range(slots)]
    slot_tok = [None] * slots
    res = {}

    def producer():
        k = 0
        while k < n:
            s = k % slots
            if k >= slots:
                ok = yield from cta.wait(empty[s], (k // slots - 1) & 1)
                if not ok:
                    cta.raise_abort()
                    break
            if cta.abort:
                break
            if k != stall_k:
                old = slot_tok[s]
                assert old is None or old["landed"], f"slot {s} re-armed while token {old['k']} is landing"
                tag = {"landed": False, "k": k}
                slot_tok[s] = tag
                full[s].tx += 1                        # expect_tx, no arrival
                cta.landing.append((full[s], 1, tag))  # the bulk copies
                yield
                full[s].arrive()                       # after the angles and the row
            k += 1
        res["handed_out"] = k

    def consumer(w):
        for k in range(n):
            s = k % slots
            ok = yield from cta.wait(full[s], (k // slots) & 1)
            if not ok:
                cta.raise_abort()
                return
            tag = slot_tok[s]
            assert tag is not None and tag["k"] == k and tag["landed"], \
                f"warp {w} read slot {s} for token {k} before it landed"
            empty[s].arrive()
            yield

    actors = {"producer": producer()}
    for w in range(warps):
        actors[f"c{w}"] = consumer(w)
    run_actors(cta, actors)

    # __syncthreads, then the drain (producer lane 0) after an abort
    if cta.abort:
        last = res["handed_out"] if drain == "handed_out" else n
        for k in range(max(0, last - slots), last):
            if k == stall_k:
                continue
            bar, parity = full[k % slots], (k // slots) & 1
            while not bar.parity_ok(parity):
                if not any(b is bar for b, _, _ in cta.landing):
                    break
                cta.land_one()
    cta.in_flight_at_exit = len(cta.landing)
    return cta


@pytest.mark.parametrize("slots", [2, 6, 8])
def test_prefill_prep_abort_leaves_nothing_in_flight(slots):
    rng = random.Random(700 + slots)
    for trial in range(400):
        n = rng.randint(1, 30)
        p = rng.choice([0.0, 0.001, 0.01, 0.05, 0.3])
        cta = prep_run(n, slots, 8, rng, p)
        assert cta.in_flight_at_exit == 0, f"trial {trial}: a copy is in flight at exit (n={n}, p={p})"
        assert (cta.status == 5) == (cta.gave_up > 0), f"trial {trial}: status {cta.status}, gave up {cta.gave_up}"


def test_prefill_prep_stalled_slot_times_out_and_drains():
    """The GPU test hook: the producer never arms one token's slot; the
    consumers give up on it, the producer (waiting for that slot to come
    free) sees the abort, the status is TIMEOUT and nothing is in flight."""
    rng = random.Random(77)
    for trial in range(300):
        n = rng.randint(2, 30)
        stall = rng.randrange(n)
        cta = prep_run(n, 6, 8, rng, p_timeout=0.0005, stall_k=stall)
        assert cta.status == 5 and cta.in_flight_at_exit == 0, f"trial {trial}"


def test_prefill_prep_drain_keyed_on_the_range_is_caught():
    """Waiting on the last slots of the token range instead of the tokens the
    producer handed out: after an early abort those phases were never armed,
    and a parity wait on one passes on an older phase while a copy lands."""
    rng = random.Random(78)
    caught = 0
    for trial in range(600):
        n = rng.randint(12, 30)
        cta = prep_run(n, 6, 8, rng, 0.05, drain="range")
        caught += cta.in_flight_at_exit > 0
    assert caught > 0
