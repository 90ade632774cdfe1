"""Model check of the clusters' softmax exchange (host-side simulation).

The prototype-split cluster pass (more than 128 prototypes; section 2.2 of
the SequenceO1 reading notes puts the final layers at about a thousand)
combines each row's softmax over C CTAs.  Every softmax warp writes its
rows' slice totals of tile u into its own slot [group][u & 1][self] and
sends that run to every other CTA as one bulk copy: the copy engine reads
the sender's slot when it delivers (not when the copy is issued), the data
lands in the receiver's slot [group][u & 1][sender] and adds its bytes to
the receiver's barrier [group][u & 1]; the receiver arms that barrier once
per tile (one arrival plus the expected bytes), waits for the phase to
complete, then reads the slots.  No acknowledgement travels back: the
argument is that a CTA can only send tile u + 2 of a group after it
received every CTA's tile u + 1, which each CTA sends only after reading its
own tile u slots, and after its tile u copy from this CTA had landed.

This test runs that protocol on a model of the mbarrier (pending arrivals,
transaction bytes that may arrive before or after the arming, phase parity)
with arbitrary interleavings and arbitrary delivery delays, and checks that
  * every read sees the values of its own tile from every sender;
  * no value lands in a slot that still holds an unread value;
  * no copy reads a source slot that its sender has already rewritten for a
    later tile;
  * no barrier phase completes on bytes of another tile;
  * no wait finds its barrier two phases ahead (the hardware waits on the
    phase parity);
  * nothing deadlocks (every CTA finishes every tile).
A variant with one buffer per group in place of two (single-buffered slots)
must fail, which shows the check can catch the hazard the double buffering
avoids.  `simulate_abort` checks the drain the kernels run on the abort
path."""

import random

import pytest


class Barrier:
    """mbarrier: a phase completes when its pending arrivals reach 0 and its
    transaction count is back to 0."""

    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.phase = 0          # completed phases
        self.tiles = set()      # tiles whose bytes were counted in this phase

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count
            done = self.tiles
            self.tiles = set()
            return done
        return None

    def arrive_expect(self, nbytes, tile):
        self.tx += nbytes
        self.pending -= 1
        self.tiles.add(tile)
        return self._maybe_complete()

    def complete_tx(self, nbytes, tile):
        self.tx -= nbytes
        self.tiles.add(tile)
        return self._maybe_complete()


def simulate(C, tiles, seed, buffers=2, warps=4):
    """C CTAs x 2 softmax groups x `warps` warps.  Every warp sends its rows
    of each tile to the other CTAs (one unit per warp and receiver); warp 0
    of a group arms the group's barrier for the tile with the units of all
    warps of all senders; every warp waits on the barrier, then reads the
    slots of its own rows."""
    rng = random.Random(seed)
    groups = 2
    bars = [[[Barrier(1) for _ in range(buffers)] for _ in range(groups)] for _ in range(C)]
    # slots[CTA][group][buf][sender][warp] = (tile, read?)
    slots = [[[[[None] * warps for _ in range(C)] for _ in range(buffers)] for _ in range(groups)]
             for _ in range(C)]
    # each (CTA, group, warp) walks its tiles u = g, g + 2, ... (local v = u // 2)
    # own[CTA][group][buf][warp] = the tile whose values the warp last wrote
    # into its own slot (the source of its copies)
    own = [[[[None] * warps for _ in range(buffers)] for _ in range(groups)] for _ in range(C)]
    step = {(h, g, w): ("send", g) for h in range(C) for g in range(groups) for w in range(warps)}
    in_flight = []  # (receiver, group, buf, sender, warp, tile)
    errors = []

    def on_complete(done, h, g, b, u_expected):
        if done is not None and done != {u_expected}:
            errors.append(f"CTA {h} group {g} buf {b}: phase completed on tiles {done}")

    guard = 0
    while True:
        guard += 1
        if guard > 400000:
            errors.append("no progress (deadlock)")
            break
        actors = [key for key, (st, u) in step.items() if u < tiles]
        if not actors and not in_flight:
            break
        choices = [("cta", a) for a in actors] + [("deliver", i) for i in range(len(in_flight))]
        kind, what = rng.choice(choices)
        if kind == "deliver":
            recv, g, b, sender, w, tile = in_flight.pop(what)
            if own[sender][g][b][w] != tile:
                errors.append(f"CTA {sender} warp {w}: copy of tile {tile} read its source "
                              f"after it was rewritten for tile {own[sender][g][b][w]}")
            cell = slots[recv][g][b][sender][w]
            if cell is not None and not cell[1]:
                errors.append(f"CTA {recv}: slot [{g}][{b}][{sender}][{w}] overwritten by tile "
                              f"{tile} before tile {cell[0]} was read")
            slots[recv][g][b][sender][w] = (tile, False)
            on_complete(bars[recv][g][b].complete_tx(1, tile), recv, g, b, tile)
            continue
        h, g, w = what
        st, u = step[what]
        v = u // 2
        par = v % buffers
        if st == "send":
            if w == 0:
                on_complete(bars[h][g][par].arrive_expect((C - 1) * warps, u), h, g, par, u)
            own[h][g][par][w] = u
            for p in range(C):
                if p != h:
                    in_flight.append((p, g, par, h, w, u))
            step[what] = ("wait", u)
        elif st == "wait":
            # the phase for local tile v is phase number v // buffers of the
            # barrier; the hardware waits on its parity, so the barrier must
            # never be two phases past it when the wait runs
            want = v // buffers
            if bars[h][g][par].phase > want + 1:
                errors.append(f"CTA {h} group {g} warp {w} tile {u}: barrier two phases ahead")
            if bars[h][g][par].phase > want:
                for p in range(C):
                    if p == h:
                        continue
                    cell = slots[h][g][par][p][w]
                    if cell is None or cell[0] != u:
                        errors.append(f"CTA {h} group {g} warp {w} tile {u}: slot from {p} "
                                      f"holds {cell}")
                    else:
                        slots[h][g][par][p][w] = (u, True)
                step[what] = ("send", u + 2)
        if errors:
            break
    return errors


@pytest.mark.parametrize("C", [2, 3, 4, 8])
def test_double_buffered_exchange_is_safe(C):
    for seed in range(40 if C < 8 else 15):
        errs = simulate(C, tiles=14, seed=seed)
        assert not errs, f"C={C} seed={seed}: {errs[:3]}"


def test_single_buffered_exchange_is_caught():
    # With one slot set and one barrier per group, a fast CTA's next tile
    # can land before a slow CTA has read the current one.
    found = False
    for seed in range(200):
        if simulate(4, tiles=12, seed=seed, buffers=1):
            found = True
            break
    assert found


def test_source_rewrite_is_caught():
    # Single-buffered, a warp can also rewrite its own slot for its next
    # tile while a copy of the current tile still has to read it.
    assert any(any("read its source" in e for e in simulate(4, tiles=12, seed=seed, buffers=1))
               for seed in range(400))


def simulate_abort(C, tiles, seed, warps=4, settle=True):
    """The same exchange, but one CTA stops at a random moment (a wait ran
    out), and every other CTA stops when it would wait for data that the
    stopped CTA never sends (its own bounded wait runs out).  Then the drain
    at the end of the cluster passes (sa_fused.cu with CLU, and
    sa_fused_pair.cu with C = 2 and one group), step for step:
      * every softmax warp has counted the tiles of its group it sent
        (xch_sent), saw complete (xch_waited) and, warp 0, armed
        (xch_armed); the counts are published and all pass a cluster
        barrier;
      * per group, waited = the largest xch_waited of its warps, armed =
        warp 0's xch_armed, top = the largest count any other CTA's warp
        sent; for the local tiles v in [waited, min(top, waited + 2)) the
        drain arms the phase if v >= armed and settles with complete_tx the
        share of every (sender, warp) whose count is <= v; then it waits
        for those phases.
    Checks that top never exceeds waited + 2 (so the cap drops nothing and
    the open tiles sit on the two barriers of the double buffer), that when
    a CTA's phases have all completed no value to it is still in flight (so
    it may pass the final barrier), and that the phases do complete once the
    values in flight have landed (no stuck wait)."""
    rng = random.Random(seed)
    groups = 2
    bars = [[[Barrier(1) for _ in range(2)] for _ in range(groups)] for _ in range(C)]
    armed = [[0] * groups for _ in range(C)]          # xch_armed of warp 0, per group
    sent = {}                                         # xch_sent, (CTA, group, warp)
    waited = {}                                       # xch_waited, (CTA, group, warp)
    step = {(h, g, w): ("send", g) for h in range(C) for g in range(groups) for w in range(warps)}
    stopped = [False] * C
    in_flight = []
    victim = rng.randrange(C)
    stop_after = rng.randrange(1, 40)
    moves = 0
    errors = []
    # run until every actor is done or stuck
    while True:
        moves += 1
        if moves == stop_after:
            stopped[victim] = True
        live = [key for key, (st, u) in step.items() if u < tiles and not stopped[key[0]]]
        runnable = []
        for key in live:
            h, g, w = key
            st, u = step[key]
            v = u // 2
            if st == "send" or bars[h][g][v % 2].phase > v // 2:
                runnable.append(("cta", key))
        choices = runnable + [("deliver", i) for i in range(len(in_flight))]
        if not choices:
            break  # every remaining actor waits for something that never comes
        kind, what = rng.choice(choices)
        if kind == "deliver":
            recv, g, b, sender, w, tile = in_flight.pop(what)
            bars[recv][g][b].complete_tx(1, tile)
            continue
        h, g, w = what
        st, u = step[what]
        v = u // 2
        if st == "send":
            if w == 0:
                bars[h][g][v % 2].arrive_expect((C - 1) * warps, u)
                armed[h][g] = v + 1
            for p in range(C):
                if p != h:
                    in_flight.append((p, g, v % 2, h, w, u))
            sent[(h, g, w)] = v + 1
            step[what] = ("wait", u)
        else:
            waited[(h, g, w)] = v + 1
            step[what] = ("send", u + 2)
    # every CTA has stopped: the drain
    open_tiles = {}
    for h in range(C):
        for g in range(groups):
            wt = max(waited.get((h, g, w), 0) for w in range(warps))
            top = max([sent.get((p, g, w), 0) for p in range(C) if p != h for w in range(warps)]
                      + [armed[h][g]])
            if top > wt + 2:
                errors.append(f"CTA {h} group {g}: top {top} > waited {wt} + 2")
            hi = min(top, wt + 2)
            for v in range(wt, hi):
                if v >= armed[h][g]:
                    bars[h][g][v % 2].arrive_expect((C - 1) * warps, 2 * v + g)
                for p in range(C):
                    if p == h:
                        continue
                    for w in range(warps):
                        if sent.get((p, g, w), 0) <= v and settle:
                            bars[h][g][v % 2].complete_tx(1, 2 * v + g)
            open_tiles[(h, g)] = (wt, hi)

    def drained(h):
        # the drain's bounded waits: phase v // 2 of barrier v % 2 complete
        return all(bars[h][g][v % 2].phase > v // 2
                   for g in range(groups) for v in range(*open_tiles[(h, g)]))

    while True:
        for h in range(C):
            if drained(h) and any(m[0] == h for m in in_flight):
                errors.append(f"CTA {h} drained with values still in flight")
        if errors or not in_flight:
            break
        recv, g, b, sender, w, tile = in_flight.pop(rng.randrange(len(in_flight)))
        bars[recv][g][b].complete_tx(1, tile)
    for h in range(C):
        if not drained(h):
            errors.append(f"CTA {h}: a drain phase never completes")
    return errors


@pytest.mark.parametrize("C", [2, 4, 8])
def test_abort_drain(C):
    for seed in range(40):
        errs = simulate_abort(C, tiles=10, seed=seed)
        assert not errs, f"C={C} seed={seed}: {errs[:3]}"


def test_abort_without_settling_gets_stuck():
    # Without settling the shares that were never sent, some drain phase
    # never completes (the bounded wait would run out): the settle step is
    # what makes the drain finish.
    assert any(simulate_abort(4, tiles=10, seed=s, settle=False) for s in range(40))
