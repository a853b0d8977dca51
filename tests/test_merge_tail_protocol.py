"""Model check of the decode kernel's merge at the launch's end, on the CPU.

A problem split over many CTAs is merged, at the end of the launch, by the
CTAs that finish streaming first.  Its items raise ready flags in the
workspace as their partials land, and every CTA takes one merge ticket once
its streaming is over.
  * Ticket word (32 bits): block 0 adds 2^12 - (G - 1), the others add 1.
    The low 12 bits return to zero after the G tickets of a launch, and the
    carry out of them counts launches (the epoch E, bits 12..31).  A CTA's
    rank is the number of tickets taken before its own.
  * A raised flag holds E + 1.  At the item's end the publishing thread
    reads E from the ticket word and then raises the flag, both before its
    own CTA takes a ticket.
  * A CTA that aborted (a wait ran out) stops taking items and stores E + 1
    into the abort word with its ticket; the merging CTAs stop waiting when
    they see it.
  * The CTA of rank G - 1 resets the queue head and zeroes every flag that
    the launch did not raise.

The model replays launches of random plans under random interleavings of
the CTAs' steps.  It checks that the ranks of a launch are 0..G-1 and the
epoch is the same in every CTA; that the word ends each launch with its low
bits at zero and the epoch one higher; that a merging CTA never sees a flag
as raised before this launch raised it, even when the epoch wraps; that no
CTA claims from the queue after the reset; and that every launch ends, an
aborted one too.  Mutants are caught: no flag clearing (with a narrow epoch,
where stale flags come back), the reset by a CTA other than rank G - 1, a
ticket taken before the CTA's last publication, and an abort that leaves the
abort word unset.
"""
import itertools
import random

import pytest

SHIFT = 12
LOW = (1 << SHIFT) - 1
MASK32 = 0xFFFFFFFF


def take_ticket(word, block, G):
    """The ticket atomic: returns (new word, rank, ready value E + 1)."""
    add = ((1 << SHIFT) - (G - 1)) if block == 0 else 1
    old = word
    new = (word + add) & MASK32
    lo = old & LOW
    if block == 0 or lo < (1 << (SHIFT - 1)):
        rank = lo
    else:
        rank = lo + G - (1 << SHIFT)
    return new, rank, (old >> SHIFT) + 1


@pytest.mark.parametrize("G", [1, 2, 3, 4, 5])
def test_ticket_ranks_every_arrival_order(G):
    for start_epoch in (0, 1, (1 << 20) - 1):
        for order in itertools.permutations(range(G)):
            word = start_epoch << SHIFT
            ranks, readies = {}, set()
            for b in order:
                word, rank, ready = take_ticket(word, b, G)
                ranks[b] = rank
                readies.add(ready)
            assert sorted(ranks.values()) == list(range(G))
            assert [ranks[b] for b in order] == list(range(G))  # rank = tickets taken before
            assert readies == {start_epoch + 1}
            assert word & LOW == 0
            assert word >> SHIFT == (start_epoch + 1) % (1 << 20)


@pytest.mark.parametrize("G", [148, 296, 7])
def test_ticket_ranks_random_orders(G):
    rng = random.Random(G)
    word = 0
    for launch in range(200):
        order = list(range(G))
        rng.shuffle(order)
        e0 = word >> SHIFT
        for i, b in enumerate(order):
            word, rank, ready = take_ticket(word, b, G)
            assert rank == i and ready == e0 + 1
        assert word & LOW == 0 and word >> SHIFT == e0 + 1


def launch(ws, rng, G, n_items, deferred, epoch_bits=20, clear=True, reset_rank=None,
           ticket_early=False, queue_items=0, abort_cta=None, abort_word=True):
    """One launch of the model.  ws: dict with 'ticket', 'flags', 'queue',
    'abort'.  deferred[i]: item i belongs to a deferred problem (it raises a
    flag and is merged).  Items [0, n_static) are dealt round robin to the
    CTAs; the last `queue_items` items are claimed from the queue.  CTA
    `abort_cta` aborts after its first item.  Returns (violations, whether a
    merge gave up on an abort)."""
    errors = []
    gave_up = []
    emask = (1 << epoch_bits) - 1
    reset_rank = G - 1 if reset_rank is None else reset_rank
    n_static = n_items - queue_items
    published = set()
    owner = {i: i % G for i in range(n_static)}

    def cta(b):
        mine = [i for i in range(n_static) if owner[i] == b]
        rank = ready = None
        aborted = False
        if ticket_early:
            ws["ticket"], rank, ready = take_ticket(ws["ticket"], b, G)
            yield
        # stream the static items, then claim queued ones until the queue is dry
        done = 0
        while True:
            if b == abort_cta and done == 1:
                aborted = True  # a wait ran out: no further item is taken
                break
            if mine:
                i = mine.pop(0)
            else:
                q = ws["queue"]
                ws["queue"] += 1
                yield
                if q >= queue_items:
                    break
                i = n_static + q
                if ws.get("reset_done"):
                    errors.append(f"claim of queue slot {q} after the queue reset")
            yield  # streaming the item
            if deferred[i]:
                e = (ws["ticket"] >> SHIFT) & emask
                yield
                ws["flags"][i] = e + 1
                published.add(i)
                yield
            done += 1
        if not ticket_early:
            ws["ticket"], rank, ready = take_ticket(ws["ticket"], b, G)
        ready = ((ready - 1) & emask) + 1  # E + 1 for an epoch of epoch_bits bits
        if aborted and abort_word:
            ws["abort"] = ready
        yield
        if rank == reset_rank:
            ws["queue"] = 0
            ws["reset_done"] = True
            if clear:
                for i in range(len(ws["flags"])):
                    if i >= n_items or not deferred[i]:
                        ws["flags"][i] = 0
            yield
        # merge: ranks 0..2 each fold every deferred item in order
        if rank < 3:
            for i in range(n_items):
                if not deferred[i]:
                    continue
                spins = 0
                while ws["flags"][i] != ready:
                    if ws["abort"] == ready:
                        gave_up.append(i)
                        return
                    spins += 1
                    if spins > 10_000:
                        errors.append(f"wait on item {i} never ended")
                        return
                    yield
                if i not in published:
                    errors.append(f"item {i} seen ready before this launch raised its flag")
                yield

    actors = {b: cta(b) for b in range(G)}
    steps = 0
    while actors:
        b = rng.choice(list(actors))
        try:
            next(actors[b])
        except StopIteration:
            del actors[b]
        steps += 1
        if steps > 2_000_000:
            errors.append("launch did not end")
            break
    ws["reset_done"] = False
    if ws["queue"] != 0 and abort_cta is None:
        errors.append("queue head not reset")
    if ws["ticket"] & LOW:
        errors.append("ticket low bits not back at zero")
    return errors, bool(gave_up)


def fresh_ws(max_items, word=0):
    return {"ticket": word, "flags": [0] * max_items, "queue": 0, "abort": 0}


def run_launches(seed, n_launches, max_items=24, **kw):
    rng = random.Random(seed)
    ws = fresh_ws(max_items, kw.pop("start_word", 0))
    errors = []
    for _ in range(n_launches):
        G = rng.randint(1, 6)
        n_items = rng.randint(1, max_items)
        queue_items = rng.randint(0, n_items // 2)
        deferred = [rng.random() < 0.6 for _ in range(n_items)]
        errors += launch(ws, rng, G, n_items, deferred, queue_items=queue_items, **kw)[0]
        if errors:
            break
    return errors


def test_merge_tail_protocol_under_random_plans():
    assert run_launches(1, 600) == []


def test_merge_tail_protocol_across_the_epoch_wrap():
    # start just before the 20-bit epoch wraps to zero
    assert run_launches(2, 80, start_word=((1 << 20) - 3) << SHIFT) == []


def test_clearing_makes_even_a_one_bit_epoch_safe():
    assert run_launches(3, 600, epoch_bits=1) == []


def test_no_clearing_with_a_narrow_epoch_is_caught():
    # without the clearing a flag from two launches back matches again
    errors = run_launches(4, 600, epoch_bits=1, clear=False)
    assert any("before this launch raised" in e for e in errors), errors


def test_reset_by_another_rank_is_caught():
    errors = []
    for seed in range(40):
        errors = run_launches(10 + seed, 60, reset_rank=0)
        if errors:
            break
    assert any("after the queue reset" in e for e in errors), errors


def test_ticket_before_the_last_publication_is_caught():
    # a ticket taken at the CTA's start lets the epoch carry before the
    # publishers read it: a flag then carries the next launch's value
    errors = []
    for seed in range(40):
        errors = run_launches(100 + seed, 60, ticket_early=True)
        if errors:
            break
    assert errors, "an early ticket should break the protocol"


def aborted_launches(seed, n_launches, abort_word=True):
    """Launches in which one CTA aborts after its first item; the workspace is
    zeroed after each, as the library asks after a device error."""
    rng = random.Random(seed)
    errors, gave_up = [], 0
    for _ in range(n_launches):
        ws = fresh_ws(24, rng.randrange(1 << 20) << SHIFT)
        G = rng.randint(2, 6)
        n_items = rng.randint(2 * G, 24)
        deferred = [True] * n_items  # every item merged: the aborted CTA's are awaited
        e, g = launch(ws, rng, G, n_items, deferred, abort_cta=rng.randrange(G), abort_word=abort_word)
        errors += e
        gave_up += g
        if errors:
            break
    return errors, gave_up


def test_an_abort_ends_every_wait():
    errors, gave_up = aborted_launches(7, 150)
    assert errors == []
    assert gave_up > 0  # the merging CTAs did wait on the aborted CTA's items


def test_abort_without_the_abort_word_is_caught():
    errors, _ = aborted_launches(8, 150, abort_word=False)
    assert any("never ended" in e for e in errors), errors
