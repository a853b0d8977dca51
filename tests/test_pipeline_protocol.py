"""Model check of the decode kernel's TMA/mbarrier pipeline protocol on the CPU.

The kernel streams tiles through kStages shared-memory stages.  Each stage
has a "full" barrier (one producer arrival + the TMA byte count) and an
"empty" barrier (one arrival per consumer warp); waits test only the PARITY
of a barrier's phase, as mbarrier.try_wait.parity does.  A parity wait
cannot tell phase k from phase k - 2, so the protocol must guarantee that no
waiter can fall two phases behind or run two phases ahead.

This test replays the protocol under many random interleavings and random
TMA landing times, and asserts that (a) a consumer only reads a stage after
the exact tile it expects has landed, (b) the producer never re-arms a
stage whose previous load is still in flight.  The kernel's scheme (every
consumer warp takes a slice of every tile, so every warp waits on every
stage in order) passes for 4 or 8 consumer warps and 3 or 6 stages, as do
groups that take alternate tiles when the group count divides the stage
count; the earlier round-robin scheme (tile i to warp i mod 4 with 6 stages)
is shown to fail.
"""
import random

import pytest

STAGES = 6
WARPS = 4     # warps per consumer group in the model


class Barrier:
    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.completed = 0  # phases completed so far

    def parity_done(self, parity):
        # try_wait.parity(P) succeeds when the current phase's parity differs from P
        return (self.completed & 1) != parity

    def arrive(self, tx=0):
        self.tx += tx
        self.pending -= 1
        assert self.pending >= 0, "arrival count went negative"
        self._maybe_complete()

    def complete_tx(self, tx):
        self.tx -= tx
        self._maybe_complete()

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.completed += 1
            self.pending = self.count


def simulate(n_tiles, scheme, rng, groups=1, warps=None, stages=None):
    """scheme "all_warps": `groups` groups of WARPS warps; group q takes the
    tiles i with i % groups == q and all its warps take part in each of them.
    scheme "round_robin": whole tiles to single warps, i % WARPS."""
    global STAGES, WARPS
    saved = STAGES, WARPS
    STAGES = stages or STAGES
    WARPS = warps or WARPS
    try:
        return _simulate(n_tiles, scheme, rng, groups)
    finally:
        STAGES, WARPS = saved


def _simulate(n_tiles, scheme, rng, groups):
    full = [Barrier(1) for _ in range(STAGES)]
    empty = [Barrier(WARPS if scheme == "all_warps" else 1) for _ in range(STAGES)]
    in_flight = []          # (stage, tile) loads not landed yet
    landed_tile = [None] * STAGES
    prod = 0
    if scheme == "all_warps":
        work = [[i for i in range(n_tiles) if i % groups == w // WARPS] for w in range(WARPS * groups)]
    else:
        work = [[i for i in range(n_tiles) if i % WARPS == w] for w in range(WARPS)]
    nw = len(work)
    pos = [0] * nw
    while True:
        actions = []
        if prod < n_tiles:
            s = prod % STAGES
            if empty[s].parity_done(((prod // STAGES) & 1) ^ 1):
                actions.append("produce")
        if in_flight:
            actions.append("land")
        for w in range(nw):
            if pos[w] < len(work[w]):
                i = work[w][pos[w]]
                if full[i % STAGES].parity_done((i // STAGES) & 1):
                    actions.append(("consume", w))
        if not actions:
            break
        a = rng.choice(actions)
        if a == "produce":
            s = prod % STAGES
            if full[s].pending != 1 or full[s].tx != 0:
                return f"stage {s} re-armed while tile {landed_tile[s]} is still in flight"
            full[s].arrive(tx=32768)
            in_flight.append((s, prod))
            prod += 1
        elif a == "land":
            s, i = in_flight.pop(rng.randrange(len(in_flight)))
            landed_tile[s] = i
            full[s].complete_tx(32768)
        else:
            w = a[1]
            i = work[w][pos[w]]
            s = i % STAGES
            if landed_tile[s] != i or full[s].completed != i // STAGES + 1:
                return f"warp {w} read stage {s} for tile {i} but it holds tile {landed_tile[s]}"
            empty[s].arrive()
            pos[w] += 1
    if prod != n_tiles or any(pos[w] != len(work[w]) for w in range(nw)):
        return "deadlock"
    return None


@pytest.mark.parametrize("warps,stages", [(4, 6), (8, 3), (8, 6)])
def test_every_warp_on_every_stage_is_safe(warps, stages):
    rng = random.Random(warps * 10 + stages)
    for trial in range(300):
        err = simulate(rng.randint(1, 200), "all_warps", rng, warps=warps, stages=stages)
        assert err is None, f"trial {trial}: {err}"


@pytest.mark.parametrize("groups", [1, 2, 3])
def test_kernel_scheme_is_safe_under_random_interleavings(groups):
    # the kernel needs STAGES % groups == 0 so that a stage always belongs to
    # the same group
    assert STAGES % groups == 0
    rng = random.Random(groups)
    for trial in range(300):
        err = simulate(rng.randint(1, 200), "all_warps", rng, groups=groups)
        assert err is None, f"trial {trial}: {err}"


def test_groups_that_do_not_divide_the_stages_are_unsafe():
    rng = random.Random(4)
    errors = [simulate(200, "all_warps", rng, groups=4) for _ in range(100)]
    assert any(e is not None for e in errors)


def test_round_robin_scheme_is_unsafe():
    rng = random.Random(2)
    errors = [simulate(200, "round_robin", rng) for _ in range(200)]
    assert any(e is not None for e in errors)


# ---------------------------------------------------------------------------
# The item hand-over: the producer picks each item (its static list, then
# claims on the run-time queue), writes its index to a shared slot, and arms
# the staged-input barrier; consumer warp 0 copies the slot to a second shared
# word once its wait succeeds, all consumer warps meet at a named barrier and
# read that word, and -1 tells them to stop.  In the kernel two things keep
# warp 0 from rewriting that word while a warp still has to read it: every
# warp reads it before it releases the inputs (arrive on in_empty), so the
# next phase cannot be armed before, and an item's end includes another named
# barrier.  The model checks, under random interleavings and random landing
# times of the staged copies, that every warp reads the item the producer
# chose for that phase, that the producer never rewrites the slot before warp
# 0 copied it and that nobody deadlocks: with either protection alone, and
# that with neither a warp can read the wrong item.

def simulate_handover(items, rng, warps=8, item_end_barrier=True, release_after_read=True):
    in_full, in_empty = Barrier(1), Barrier(warps)
    slot, cur = None, None
    landing = []              # staged copies in flight (phase k)
    # producer state
    pk, p_done, p_waiting_arm = 0, False, False
    # consumer state per warp: phase k, step
    ck = [0] * warps
    step = ["wait"] * warps   # wait -> bar1 -> read -> (item) -> bar2 -> wait
    seen = [[] for _ in range(warps)]
    bar_count = {"b1": 0, "b2": 0}
    bar_gen = {"b1": 0, "b2": 0}
    at_bar = [None] * warps   # (name, gen) a warp is blocked at
    plan = list(items) + [-1]
    for _ in range(100000):
        acts = []
        if not p_done and in_empty.parity_done((pk & 1) ^ 1):
            acts.append("produce")
        if landing:
            acts.append("land")
        for w in range(warps):
            st = step[w]
            if st == "wait" and in_full.parity_done(ck[w] & 1):
                acts.append(("wait", w))
            elif st in ("bar1", "bar2"):
                name, gen = at_bar[w]
                if bar_gen[name] > gen:
                    acts.append((st, w))
            elif st in ("read", "item"):
                acts.append((st, w))
        if not acts:
            break
        a = rng.choice(acts)
        if a == "produce":
            it = plan[pk]
            if slot is not None and cur != slot and pk > 0:
                return f"slot rewritten at phase {pk} before warp 0 copied it"
            slot = it
            if it >= 0:
                in_full.arrive(tx=1)
                landing.append(pk)
            else:
                in_full.arrive()
                p_done = True
            pk += 1
        elif a == "land":
            landing.pop(rng.randrange(len(landing)))
            in_full.complete_tx(1)
        else:
            kind, w = a
            if kind == "wait":
                if w == 0:
                    cur = slot
                if not release_after_read and plan[ck[w]] >= 0:
                    in_empty.arrive()
                step[w] = "bar1"
                at_bar[w] = ("b1", bar_gen["b1"])
                bar_count["b1"] += 1
                if bar_count["b1"] == warps:
                    bar_count["b1"] = 0
                    bar_gen["b1"] += 1
            elif kind == "bar1":
                step[w] = "read"
            elif kind == "read":
                it = cur
                seen[w].append(it)
                if it != plan[ck[w]]:
                    return f"warp {w} read item {it} for phase {ck[w]}, expected {plan[ck[w]]}"
                if it < 0:
                    step[w] = "done"
                else:
                    if release_after_read:
                        in_empty.arrive()
                    step[w] = "item"
            elif kind == "item":
                ck[w] += 1
                if item_end_barrier:
                    step[w] = "bar2"
                    at_bar[w] = ("b2", bar_gen["b2"])
                    bar_count["b2"] += 1
                    if bar_count["b2"] == warps:
                        bar_count["b2"] = 0
                        bar_gen["b2"] += 1
                else:
                    step[w] = "wait"
            elif kind == "bar2":
                step[w] = "wait"
    if not p_done or any(s != "done" for s in step):
        return "deadlock"
    if any(s != plan for s in seen):
        return "a warp missed an item"
    return None


@pytest.mark.parametrize("item_end_barrier,release_after_read", [(True, True), (True, False), (False, True)])
def test_item_handover_is_safe_under_random_interleavings(item_end_barrier, release_after_read):
    rng = random.Random(7)
    for trial in range(300):
        items = [rng.randrange(600) for _ in range(rng.randint(0, 30))]
        err = simulate_handover(items, rng, item_end_barrier=item_end_barrier,
                                release_after_read=release_after_read)
        assert err is None, f"trial {trial}: {err}"


def test_item_handover_with_neither_protection_is_unsafe():
    rng = random.Random(8)
    errors = [simulate_handover([rng.randrange(600) for _ in range(20)], rng, item_end_barrier=False,
                                release_after_read=False)
              for _ in range(300)]
    assert any(e is not None for e in errors)
