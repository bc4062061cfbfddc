"""Models of the one-launch rings' hop hand-offs, run under random schedules
(CPU only).

RING_CLUSTER (ranks are CTAs of a cluster) passes hop h from rank r to rank
r+1 through slot h mod N of rank r+1, with one mbarrier per slot and no credit
flowing back.  It relies on three claims:

* a sender never overwrites a slot before the receiving thread has read the
  hop it held (the ring's own dependencies keep a sender within N-1 hops);
* every wait sees the barrier at most one phase ahead of the phase it waits
  for, so the parity test is exact (no stale read, no missed phase);
* an arrival (or transaction count) always lands in the phase of its own hop.

That model runs every thread (lane) of every rank as its own process, with
the per-tile program of the kernel (send, then receive/send alternating,
ending on a receive: 2N-2 of each per tile), and two barrier mechanisms:

* "tx" (RING_CLUSTER): barrier count 1; the receiver's lane 0 arms the slot
  (its arrival plus the expected bytes) for hops 0..N-1 at the start and for
  hop h+N right after reading hop h; each sender lane's store completes its
  bytes, possibly before the slot is armed;
* "arrive": barrier count = lanes; each sender lane arrives once per hop
  (the hand-off an earlier form of the CTA ring used; kept as a second
  mechanism the protocol argument covers).

RING_CTA (ranks are warps of one CTA) uses no mbarrier: at hop h every warp
stores into the next warp's slot of buffer h mod 2, the CTA passes one
barrier, and every warp reads its own slot.  Its model lets the warps run
freely between barriers and checks that every read sees its own hop and that
no store lands on a hop not yet read; with one buffer instead of two, some
schedule breaks that.

RING_CTA also stages each thread's own inputs in shared-memory cells with
asynchronous copies, one commit group per cell: a deterministic model of one
thread's program checks that the wait before every read leaves that cell's
copy complete (n - 1 newer groups may still be in flight, never n), and that
a refill never follows a read of the same cell without a barrier between.

A random scheduler picks any enabled step; a receive is enabled when the
hardware's test passes.  The checks are the claims above, and that every
schedule finishes (no deadlock).
"""
import random

import pytest


class Barrier:
    def __init__(self, count, armed_tx=0):
        self.count = count
        self.pending = count
        self.tx = 0
        self.done = 0  # completed phases
        if armed_tx:  # armed before anyone can store (initial expect_tx)
            self.pending -= 1
            self.tx += armed_tx

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.done += 1
            self.pending = self.count
            self.tx = 0

    def arrive(self, expect_tx=0):
        assert self.pending > 0
        self.pending -= 1
        self.tx += expect_tx
        self._maybe_complete()

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        self._maybe_complete()

    def parity_passes(self, phase):
        """try_wait.parity: true when the current phase's parity differs
        from the awaited phase's parity"""
        return (self.done & 1) != (phase & 1)


def simulate(n, lanes, tiles, mode, seed):
    rng = random.Random(seed)
    H = tiles * (2 * n - 2)  # hops sent (and received) by every rank
    program = []
    for _ in range(tiles):
        program += ["S"] + ["R", "S"] * (2 * n - 3) + ["R"]
    assert program.count("S") == program.count("R") == H

    if mode == "arrive":
        bars = [[Barrier(lanes) for _ in range(n)] for _ in range(n)]  # [receiver][slot]
    else:  # slots of hops that never come stay unarmed
        bars = [[Barrier(1, armed_tx=lanes if j < H else 0) for j in range(n)] for _ in range(n)]
    slot = [[[None] * lanes for _ in range(n)] for _ in range(n)]  # hop id held, [receiver][slot][lane]
    read = [[[True] * lanes for _ in range(n)] for _ in range(n)]  # has the receiver lane read it
    pc = {(r, t): 0 for r in range(n) for t in range(lanes)}
    sent = {(r, t): 0 for r in range(n) for t in range(lanes)}
    recv = {(r, t): 0 for r in range(n) for t in range(lanes)}

    def enabled(p):
        r, t = p
        if pc[p] == len(program):
            return False
        if program[pc[p]] == "S":
            return True
        h = recv[p]
        b = bars[r][h % n]
        if not b.parity_passes(h // n):
            return False
        # the claim behind the parity test: the barrier is exactly one phase past the awaited one
        assert b.done == h // n + 1, (mode, n, lanes, seed, "stale or missed phase", r, t, h, b.done)
        return True

    steps = 0
    while True:
        ready = [p for p in pc if enabled(p)]
        if not ready:
            assert all(pc[p] == len(program) for p in pc), (mode, n, lanes, tiles, seed, "deadlock")
            break
        p = rng.choice(ready)
        r, t = p
        steps += 1
        if program[pc[p]] == "S":
            h = sent[p]
            q = (r + 1) % n
            j = h % n
            # the slot piece must be free: empty, or holding hop h - n already read by lane t of q
            assert slot[q][j][t] is None or (slot[q][j][t] == h - n and read[q][j][t]), \
                (mode, n, lanes, seed, "overwrite before read", r, t, h)
            slot[q][j][t] = h
            read[q][j][t] = False
            b = bars[q][j]
            # the arrival / bytes belong to the phase of this hop
            assert b.done == h // n, (mode, n, lanes, seed, "landed in another phase", r, t, h, b.done)
            if mode == "arrive":
                b.arrive()
            else:
                b.complete_tx(1)
            sent[p] += 1
        else:
            h = recv[p]
            j = h % n
            assert slot[r][j][t] == h and not read[r][j][t], (mode, n, lanes, seed, "stale data", r, t, h)
            read[r][j][t] = True
            if mode == "tx" and t == 0 and h + n < H:
                b = bars[r][j]
                assert b.done == (h + n) // n, (mode, n, lanes, seed, "armed in another phase", r, h, b.done)
                b.arrive(expect_tx=lanes)
            recv[p] += 1
        pc[p] += 1
    assert all(sent[p] == H and recv[p] == H for p in pc)
    return steps


@pytest.mark.parametrize("mode", ["arrive", "tx"])
@pytest.mark.parametrize("n", [2, 3, 4, 5, 8])
@pytest.mark.parametrize("lanes", [1, 2, 3])
def test_handoff_protocol_under_random_schedules(mode, n, lanes):
    for seed in range(40):
        simulate(n, lanes, tiles=1 + seed % 3, mode=mode, seed=seed * 7919 + n * 31 + lanes)


def test_model_catches_too_few_slots():
    """The model is not vacuous: with N-1 slots per receiver (a sender may
    then reach a slot whose previous hop is still unread) some schedule
    breaks one of the claims."""
    def simulate_fewer_slots(n, seed):
        rng = random.Random(seed)
        s = n - 1
        H = 2 * (2 * n - 2)
        program = (["S"] + ["R", "S"] * (2 * n - 3) + ["R"]) * 2
        bars = [[Barrier(1) for _ in range(s)] for _ in range(n)]
        slot = [[None] * s for _ in range(n)]
        read = [[True] * s for _ in range(n)]
        pc = [0] * n
        sent = [0] * n
        recv = [0] * n
        while True:
            ready = []
            for r in range(n):
                if pc[r] == len(program):
                    continue
                if program[pc[r]] == "S":
                    ready.append(r)
                else:
                    h = recv[r]
                    if bars[r][h % s].parity_passes(h // s):
                        ready.append(r)
            if not ready:
                return all(pc[r] == len(program) for r in range(n))
            r = rng.choice(ready)
            if program[pc[r]] == "S":
                h, q = sent[r], (r + 1) % n
                if not (slot[q][h % s] is None or (slot[q][h % s] == h - s and read[q][h % s])):
                    return False
                if bars[q][h % s].done != h // s:
                    return False
                slot[q][h % s] = h
                read[q][h % s] = False
                bars[q][h % s].arrive()
                sent[r] += 1
            else:
                h = recv[r]
                if slot[r][h % s] != h:
                    return False
                read[r][h % s] = True
                recv[r] += 1
            pc[r] += 1

    assert not all(simulate_fewer_slots(4, seed) for seed in range(200))


def simulate_lockstep(n, tiles, buffers, seed):
    """RING_CTA's hand-off: per hop, store into the next warp's slot of buffer
    h mod ``buffers``, one CTA-wide barrier, read the own slot.  Returns
    False at the first violation (overwrite of an unread hop, or a read of
    the wrong hop); True when every schedule step was clean."""
    rng = random.Random(seed)
    H = tiles * (2 * n - 2)
    program = ["S", "B", "R"] * H
    slot = [[None] * n for _ in range(buffers)]  # hop held, [buffer][receiving warp]
    read = [[True] * n for _ in range(buffers)]
    pc = [0] * n
    while True:
        ready = []
        for w in range(n):
            if pc[w] == len(program):
                continue
            if program[pc[w]] == "B":
                # every warp must have arrived at this barrier (the same index in every program)
                if all(pc[v] >= pc[w] for v in range(n)):
                    ready.append(w)
            else:
                ready.append(w)
        if not ready:
            assert all(pc[w] == len(program) for w in range(n)), ("deadlock", n, seed)
            return True
        w = rng.choice(ready)
        h = pc[w] // 3
        op = program[pc[w]]
        b = h % buffers
        if op == "S":
            q = (w + 1) % n
            if not (slot[b][q] is None or (slot[b][q] == h - buffers and read[b][q])):
                return False
            slot[b][q] = h
            read[b][q] = False
        elif op == "R":
            if slot[b][w] != h or read[b][w]:
                return False
            read[b][w] = True
        pc[w] += 1


@pytest.mark.parametrize("n", [2, 3, 4, 5, 8])
def test_cta_ring_double_buffer_under_random_schedules(n):
    for seed in range(200):
        assert simulate_lockstep(n, tiles=1 + seed % 3, buffers=2, seed=seed * 131 + n)


def test_cta_ring_model_catches_a_single_buffer():
    assert not all(simulate_lockstep(4, tiles=2, buffers=1, seed=seed) for seed in range(200))


def simulate_cells(n, tiles, pending_allowed):
    """RING_CTA's own-input cells, one thread's program over `tiles` tiles.

    Each thread copies every reduce-scatter step's input into its own cell
    (cp.async, one commit group per cell) and reads cell k at step k.  The
    prologue fills cells 0..n-1 for the first tile; in each tile, after the
    barrier of hop k (k = 1..n-1) the thread refills cell k-1 for the next
    tile, and after the first all-gather barrier cell n-1; before every read
    it waits until at most `pending_allowed` groups are in flight.  Copies
    complete in commit order, as late as the wait allows.  Returns False if a
    read could see a cell whose copy for that (tile, step) has not completed,
    or a refill could land before the cell's last read; True otherwise."""
    groups = []          # (tile, cell) per committed group, in order
    completed = 0        # groups known complete (the wait's guarantee)
    cell_tile = {}       # cell -> tile whose data a completed group put there
    last_read = {}       # cell -> event index of its last read
    barrier_at = []      # event indices of barriers
    ev = 0

    def commit(tile, cell):
        nonlocal ev
        groups.append((tile, cell))
        ev += 1

    def wait(allowed):
        nonlocal completed, ev
        completed = max(completed, len(groups) - allowed)
        for g in groups[:completed]:
            cell_tile[g[1]] = g[0]
        ev += 1

    def read(tile, cell):
        nonlocal ev
        if cell_tile.get(cell) != tile:
            return False
        last_read[cell] = ev
        ev += 1
        return True

    def barrier():
        nonlocal ev
        barrier_at.append(ev)
        ev += 1

    def refill(tile, cell):
        # the refill must follow the cell's last read with a barrier in between
        lr = last_read.get(cell)
        if lr is not None and not any(lr < b for b in barrier_at):
            return False
        commit(tile, cell)
        return True

    for k in range(n):
        commit(0, k)
    for tile in range(tiles):
        nxt = tile + 1  # a refill for a tile past the end is an empty group
        wait(pending_allowed)
        if not read(tile, 0):
            return False
        for k in range(1, n):
            barrier()
            if not refill(nxt, k - 1):
                return False
            wait(pending_allowed)
            if not read(tile, k):
                return False
        for j in range(1, n):
            barrier()
            if j == 1 and not refill(nxt, n - 1):
                return False
    return True


@pytest.mark.parametrize("n", [2, 3, 4, 5, 6, 7, 8])
def test_cta_ring_cells_are_ready_when_read(n):
    assert simulate_cells(n, tiles=4, pending_allowed=n - 1)


def test_cta_ring_cell_model_catches_a_loose_wait():
    # allowing n groups in flight lets a read see the previous tile's data
    assert not simulate_cells(4, tiles=3, pending_allowed=4)
