"""The schedule of the resident tensor-stop launch, replayed on the CPU.

The launch runs the iterations in rounds of C (10 for 32-element lanes, 4
below), starts round r only once the stop decision of round r-2 is published,
leaves the loop when that decision reports a first rise f (the kept iterate is
then f - 1: the stop rule of techreport.ngo, "Weight-only quantization
without the calibration tax", section "Outlier-aware optimization without
gradients", keeps the iterate before the tensor error stops falling), and
keeps the zero-point of every iteration it runs in a ring of 2C + 2 slots,
slot = iteration mod (2C + 2), from which the outputs are written.  This
replays that schedule for every iteration count up to 120 and every position
of the first rise, and checks what the kernel relies on: the kept iterate's
zero-point is still in the ring when the outputs are written; no round past
the decision that stops the run is started; and, over random interleavings
of the warps, the four-entry rings of published decisions and of partial
rows are never overwritten while a reader may still need them and no warp
waits forever.
"""
import pytest


def replay(iters, C, rise):
    """Rounds run, ring contents and kept iterate for a first rise at `rise`
    (None: the error falls to the end)."""
    slots = 2 * C + 2
    nrounds = -(-iters // C)
    ring = {}
    ran = []
    for r in range(nrounds):
        if r >= 2:
            # round r-2 is published: it reports the first rise among iterations < (r-1) C
            if rise is not None and rise < (r - 1) * C:
                return max(rise - 1, 0), ring, ran
        for c in range(min(C, iters - r * C)):
            m = r * C + c
            ring[m % slots] = m  # z of iteration m, stored before it is evaluated
        ran.append(r)
    # every round ran: the rule over all of them
    kept = max(rise - 1, 0) if rise is not None else iters - 1
    return kept, ring, ran


@pytest.mark.parametrize("C", [4, 10])
def test_kept_zero_point_is_in_the_ring(C):
    slots = 2 * C + 2
    for iters in range(1, 121):
        for rise in [None] + list(range(1, iters)):
            kept, ring, ran = replay(iters, C, rise)
            assert ring.get(kept % slots) == kept, (iters, rise, kept, ran)
            if rise is not None:
                # the run stops at the start of the round after the one that published the rise
                last = (rise // C) + 1
                assert max(ran) <= min(last, -(-iters // C) - 1), (iters, rise, ran)


def simulate(nw, nrounds, seed, look=2, ring=4):
    """Warps interleaved at random under the launch's rules (a warp starts round
    r once round r - look is published; rings of `ring` entries); asserts on
    every read and overwrite of the two rings.  Returns the number of steps."""
    import random
    rng = random.Random(seed)
    nxt = [0] * nw            # the round each warp runs next
    started = [False] * nw    # has it passed that round's start (its wait)?
    finished = [False] * nw
    posted = [0] * nrounds
    published = [False] * nrounds
    pending = []              # rounds every warp posted, not yet published
    dec = {}                  # decision ring entry -> round it holds
    rows = {}                 # partial row -> round it holds
    steps = 0
    while not all(finished):
        acts = []
        for w in range(nw):
            if finished[w]:
                continue
            r = nxt[w]
            if r == nrounds:  # the final wait for the last round's decision
                if published[nrounds - 1]:
                    acts.append(("final", w))
            elif not started[w]:
                if r < look or published[r - look]:
                    acts.append(("start", w))
            else:
                acts.append(("post", w))
        acts += [("publish", r) for r in pending if r == 0 or published[r - 1]]
        assert acts, "no warp can move: the protocol would wait forever"
        kind, x = rng.choice(acts)
        steps += 1
        if kind == "start":
            r = nxt[x]
            if r >= look:
                assert dec.get((r - look) % ring) == r - look, "decision overwritten before it was read"
            started[x] = True
        elif kind == "post":
            r = nxt[x]
            if r >= ring:
                assert published[r - ring], "partial row overwritten before its round was summed"
            rows[r % ring] = r
            posted[r] += 1
            if posted[r] == nw:
                pending.append(r)
            nxt[x] += 1
            started[x] = False
        elif kind == "publish":
            r = x
            pending.remove(r)
            assert rows[r % ring] == r, "partial row of this round overwritten"
            if r >= 1:
                assert dec.get((r - 1) % ring) == r - 1, "decision of round r-1 overwritten before its successor read it"
            if r >= ring:
                # the entry's previous round is read at the start of round (r - ring) + look by every warp
                q = r - ring + look
                assert all(nxt[w] > q or (nxt[w] == q and started[w]) for w in range(nw)), "overwritten too early"
            dec[r % ring] = r
            published[r] = True
        else:
            assert dec.get((nrounds - 1) % ring) == nrounds - 1
            finished[x] = True
    return steps


@pytest.mark.parametrize("nw", [1, 2, 3, 7])
def test_rings_under_random_interleavings(nw):
    for seed in range(60):
        for nrounds in (1, 2, 3, 5, 9, 23):
            assert simulate(nw, nrounds, seed) > 0


@pytest.mark.parametrize("look,ring", [(3, 2), (2, 1)])
def test_the_simulation_sees_a_broken_protocol(look, ring):
    """Negative controls: rings with fewer entries than the lookahead (a
    decision is read `look` rounds after it is published, and the ring's
    entry is reused `ring` rounds later) overwrite a decision that is still
    needed, and the simulation must say so.  The launch waits two rounds and
    keeps four entries."""
    failures = 0
    for seed in range(40):
        for nrounds in (5, 9, 23):
            try:
                simulate(3, nrounds, seed, look, ring)
            except AssertionError:
                failures += 1
    assert failures > 0
