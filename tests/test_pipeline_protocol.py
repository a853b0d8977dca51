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
