"""Event model of the wide tcgen05 kernel's barrier protocol (head dims
129..256), run on the CPU.

The kernel's three roles are restated as generators that wait on mbarrier
phases and arrive on them in the order `run_producer_wide`, `run_mma_wide`
and the wide mode of `run_softmax` do:
  producer: per tile, Q after q_empty; K of blocks lo and lo+1; then for each
            block j: V_j, and K_{j+2} if it exists (each K two 32 KB halves,
            each V one or two halves) into a ring of 5 slots;
  MMA:      per tile, Q; S of lo and lo+1 into the two S buffers; per block
            j: V_j, P_j, P·V (one pv_done commit), release V, o_full on the
            last block, S_{j+2} into the buffer P_j came from, q_empty after
            the tile's last S;
  softmax:  per block: S, optionally a rescale of O that first waits for the
            previous block's P·V (pv_done), P; o_full after a tile.
Waits follow mbarrier parity semantics (a wait for parity x passes while the
current phase's parity differs from x).  Random interleavings must finish
without a deadlock, no wait may pass before the phase it stands for has
completed, and every ring slot must hold what the MMA role expects."""
import random

import pytest

SLOTS = 5


class Bar:
    def __init__(self, count=1):
        self.count, self.pending, self.phases = count, 0, 0

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.phases += 1


def run(tiles, v_halves, seed):
    bars = {}

    def b(name):
        if name not in bars:
            bars[name] = Bar()
        return bars[name]

    for name in ["q_full", "q_empty", "o_full", "pv_done", "s_full0", "s_full1", "p_full0", "p_full1"] + \
            [f"full{i}" for i in range(SLOTS)] + [f"empty{i}" for i in range(SLOTS)]:
        b(name)
    ring = {}
    log = []

    def producer():
        fill = q_fill = 0
        for lo, hi in tiles:
            if hi < lo:
                continue
            yield ("wait", "q_empty", (q_fill & 1) ^ 1, q_fill - 1)
            b("q_full").arrive()
            q_fill += 1

            def load(tag):
                nonlocal fill
                s = fill % SLOTS
                yield ("wait", f"empty{s}", ((fill // SLOTS) & 1) ^ 1, fill // SLOTS - 1)
                assert s not in ring, ("slot overwritten before release", s, ring[s], tag)
                ring[s] = tag
                b(f"full{s}").arrive()
                fill += 1

            for blk in [lo, lo + 1] if lo + 1 <= hi else [lo]:
                for h in range(2):
                    yield from load(("K", blk, h))
            for j in range(lo, hi + 1):
                for h in range(v_halves):
                    yield from load(("V", j, h))
                if j + 2 <= hi:
                    for h in range(2):
                        yield from load(("K", j + 2, h))

    def mma():
        use = q_use = g = 0
        p_cnt = [0, 0]

        def take(expect):
            nonlocal use
            s = use % SLOTS
            yield ("wait", f"full{s}", (use // SLOTS) & 1, use // SLOTS)
            assert ring.get(s) == expect, ("ring holds", s, ring.get(s), "expected", expect)
            use += 1
            return s

        def qk(buf, j):
            k0 = yield from take(("K", j, 0))
            k1 = yield from take(("K", j, 1))
            log.append(("S", j, buf))
            b(f"s_full{buf}").arrive()
            for s in (k0, k1):
                del ring[s]
                b(f"empty{s}").arrive()

        for lo, hi in tiles:
            if hi < lo:
                continue
            yield ("wait", "q_full", q_use & 1, q_use)
            q_use += 1
            yield from qk(g & 1, lo)
            if lo == hi:
                b("q_empty").arrive()
            if lo + 1 <= hi:
                yield from qk((g + 1) & 1, lo + 1)
                if lo + 1 == hi:
                    b("q_empty").arrive()
            for j in range(lo, hi + 1):
                buf = g & 1
                vs = []
                for h in range(v_halves):
                    vs.append((yield from take(("V", j, h))))
                yield ("wait", f"p_full{buf}", p_cnt[buf] & 1, p_cnt[buf])
                p_cnt[buf] += 1
                for h, s in enumerate(vs):
                    assert ring.get(s) == ("V", j, h), ("P·V reads a slot that no longer holds V", j, h)
                log.append(("PV", j, buf))
                b("pv_done").arrive()
                for s in vs:
                    del ring[s]
                    b(f"empty{s}").arrive()
                if j == hi:
                    b("o_full").arrive()
                if j + 2 <= hi:
                    yield from qk(buf, j + 2)
                    if j + 2 == hi:
                        b("q_empty").arrive()
                g += 1

    def softmax(rescale_prob, rng):
        s_cnt = [0, 0]
        g = o = 0
        for lo, hi in tiles:
            for j in range(lo, hi + 1):
                buf = g & 1
                yield ("wait", f"s_full{buf}", s_cnt[buf] & 1, s_cnt[buf])
                s_cnt[buf] += 1
                assert ("S", j, buf) in log
                if j > lo and rng.random() < rescale_prob:
                    yield ("wait", "pv_done", (g - 1) & 1, g - 1)
                    assert ("PV", j - 1, (g - 1) & 1) in log  # O holds every earlier block
                b(f"p_full{buf}").arrive()
                g += 1
            if hi >= lo:
                yield ("wait", "o_full", o & 1, o)
                o += 1

    rng = random.Random(seed)
    agents = [producer(), mma(), softmax(0.5, random.Random(seed + 1))]
    pending = [None] * 3
    done = [False] * 3
    while not all(done):
        progressed = False
        order = [0, 1, 2]
        rng.shuffle(order)
        for a in order:
            if done[a]:
                continue
            if pending[a] is not None:
                _, name, parity, phase = pending[a]
                bar = bars[name]
                if (bar.phases & 1) == (parity & 1):
                    continue  # the awaited phase has not completed (or the barrier is two ahead)
                assert bar.phases >= phase + 1, ("wait passed before its phase completed", name, bar.phases, phase)
                assert bar.phases <= phase + 2, ("barrier two phases ahead of its waiter", name)
                pending[a] = None
            try:
                pending[a] = next(agents[a])
            except StopIteration:
                done[a] = True
            progressed = True
        if not progressed:
            raise AssertionError(f"deadlock, waiting on {pending}")


@pytest.mark.parametrize("tiles", [
    [(0, 0), (0, 0)], [(0, 1), (0, 1)], [(0, 2)], [(0, 5), (0, 6)], [(3, 9), (0, -1)],
    [(0, -1), (2, 2)], [(0, 12), (0, 13)], [(5, 5), (4, 6)], [(0, 3), (0, 3), (1, 4), (0, 0)],
])
@pytest.mark.parametrize("v_halves", [1, 2])
def test_wide_protocol_finishes_in_order(tiles, v_halves):
    for seed in range(25):
        run(tiles, v_halves, seed)
