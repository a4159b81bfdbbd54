"""Event model of the two-tile tcgen05 kernel's barrier protocol, run on the
CPU (the same approach as test_wide_protocol_model.py).

Roles, in the order `run_producer`, `run_mma` and `run_softmax` use them:
  producer: per item, Q of tile 0 (after q_empty[0]); then for each key block
            j of the union of the tiles' ranges: K_j (with rope also its
            keyRope chunk, after kr_empty), Q of tile 1 once (at the first
            block), V_j; one ring of `stages` slots for K and V;
  MMA:      per item, Q of the active tiles; K_lo and S = Q·K^T for the tiles
            that have block lo; then per block j: V_j and K_{j+1}; for each
            tile that has j: P(t, j), P·V, o_full[t] on its last block; for
            each tile that has j+1: S(t, j+1) (after that tile's P·V, since P
            aliases S in TMEM), q_empty[t] after its last S;
  softmax t: per item, for each block of its range: S, then (after any O
            rescale) the first half of P (p_half), then the rest (p_full);
            o_full[t] before the epilogue when it had blocks.
Checks: random interleavings finish; no wait passes before its phase; ring
slots hold what the MMA expects; every S reads the Q tile of its own item;
S(t, j+1) is issued after P·V(t, j); a tile's first P·V of an item (which
overwrites O) comes after its previous epilogue."""
import random

import pytest


class Bar:
    def __init__(self):
        self.phases = 0

    def arrive(self):
        self.phases += 1


def tile_range(lo, hi):
    return {"valid": True, "lo": lo, "hi": hi, "active": hi >= lo}


INVALID = {"valid": False, "lo": 0, "hi": -1, "active": False}


def has(tr, j):
    return tr["valid"] and tr["lo"] <= j <= tr["hi"]


def run(items, stages, rope, seed):
    bars = {}

    def b(name):
        if name not in bars:
            bars[name] = Bar()
        return bars[name]

    ring, kr_ring, log = {}, {}, []
    q_buf = [None, None]        # which item's Q each tile's buffer holds
    epilogues = [0, 0]          # epilogues done per tile
    items_started = [0, 0]      # items whose first P·V was issued, per tile

    def union(tr):
        act = [x for x in tr if x["active"]]
        return (min(x["lo"] for x in act), max(x["hi"] for x in act)) if act else None

    def producer():
        fill = kr_fill = 0
        q_fill = [0, 0]
        for n_item, tr in enumerate(items):
            u = union(tr)
            if u is None:
                continue
            lo, hi = u

            def load_q(t):
                yield ("wait", f"q_empty{t}", (q_fill[t] & 1) ^ 1, q_fill[t] - 1)
                q_buf[t] = n_item
                b(f"q_full{t}").arrive()
                q_fill[t] += 1

            def load_kv(tag, with_rope):
                nonlocal fill, kr_fill
                s = fill % stages
                yield ("wait", f"kv_empty{s}", ((fill // stages) & 1) ^ 1, fill // stages - 1)
                if rope and with_rope:
                    r = kr_fill % 2
                    yield ("wait", f"kr_empty{r}", ((kr_fill // 2) & 1) ^ 1, kr_fill // 2 - 1)
                    assert r not in kr_ring, ("keyRope slot overwritten", r)
                    kr_ring[r] = tag
                    kr_fill += 1
                assert s not in ring, ("ring slot overwritten before release", s, ring[s], tag)
                ring[s] = tag
                b(f"kv_full{s}").arrive()
                fill += 1

            if tr[0]["active"]:
                yield from load_q(0)
            for j in range(lo, hi + 1):
                yield from load_kv(("K", j), True)
                if j == lo and tr[1]["active"]:
                    yield from load_q(1)
                yield from load_kv(("V", j), False)

    def mma():
        use = kr_use = 0
        q_use, p_cnt = [0, 0], [0, 0]

        def take(expect):
            nonlocal use
            s = use % stages
            yield ("wait", f"kv_full{s}", (use // stages) & 1, use // stages)
            assert ring.get(s) == expect, ("ring holds", s, ring.get(s), "expected", expect)
            use += 1
            return s

        def release(s):
            del ring[s]
            b(f"kv_empty{s}").arrive()

        def release_rope():
            nonlocal kr_use
            r = kr_use % 2
            del kr_ring[r]
            b(f"kr_empty{r}").arrive()
            kr_use += 1

        def qk(t, j, k_slot):
            assert ring.get(k_slot) == ("K", j), ("S reads a K slot that no longer holds K", j)
            assert q_buf[t] == n_item, ("Q buffer overwritten before the tile's last S", t, q_buf[t], n_item)
            if rope:
                assert kr_ring.get(kr_use % 2) == ("K", j), ("keyRope slot", kr_ring, j)
            if j > tr[t]["lo"]:
                assert ("PV", t, j - 1) in log, ("S overwrote P before its P·V", t, j)
            log.append(("S", t, j))
            b(f"s_full{t}").arrive()
            if j == tr[t]["hi"]:
                b(f"q_empty{t}").arrive()

        for n_item, tr in enumerate(items):
            u = union(tr)
            if u is None:
                continue
            lo, hi = u
            for t in range(2):
                if tr[t]["active"]:
                    yield ("wait", f"q_full{t}", q_use[t] & 1, q_use[t])
            sk = yield from take(("K", lo))
            for t in range(2):
                if has(tr[t], lo):
                    qk(t, lo, sk)
            release(sk)
            if rope:
                release_rope()
            for j in range(lo, hi + 1):
                nxt = j < hi
                sv = yield from take(("V", j))
                sk2 = (yield from take(("K", j + 1))) if nxt else None
                for t in range(2):
                    if has(tr[t], j):
                        # P·V in two halves: keys 0..63 once the softmax has
                        # stored that half of P, keys 64..127 after the rest
                        yield ("wait", f"p_half{t}", p_cnt[t] & 1, p_cnt[t])
                        assert ("Phalf", t, j) in log, ("P·V over a half of P not yet stored", t, j)
                        if j == tr[t]["lo"]:
                            assert epilogues[t] == items_started[t], ("O overwritten before the epilogue", t)
                            items_started[t] += 1
                        assert ring.get(sv) == ("V", j), ("P·V reads a slot that no longer holds V", j)
                        log.append(("PVlo", t, j))
                        yield ("wait", f"p_full{t}", p_cnt[t] & 1, p_cnt[t])
                        p_cnt[t] += 1
                        assert ("P", t, j) in log, ("P·V over P not yet stored", t, j)
                        assert ring.get(sv) == ("V", j), ("P·V reads a slot that no longer holds V", j)
                        log.append(("PV", t, j))
                        if j == tr[t]["hi"]:
                            b(f"o_full{t}").arrive()
                    if nxt and has(tr[t], j + 1):
                        qk(t, j + 1, sk2)
                release(sv)
                if nxt:
                    release(sk2)
                    if rope:
                        release_rope()
            for t in range(2):
                if tr[t]["active"]:
                    q_use[t] += 1

    def softmax(t):
        s_cnt = o_cnt = 0
        for tr in items:
            r = tr[t]
            if not r["valid"]:
                continue
            for j in range(r["lo"], r["hi"] + 1):
                yield ("wait", f"s_full{t}", s_cnt & 1, s_cnt)
                s_cnt += 1
                assert ("S", t, j) in log, ("S read before it was computed", t, j)
                if j > r["lo"]:
                    # an O rescale happens here, before the first half's arrival
                    assert ("PV", t, j - 1) in log, ("O rescaled before the last P·V into it", t, j)
                log.append(("Phalf", t, j))
                b(f"p_half{t}").arrive()
                yield None  # the second half of the exponentials
                log.append(("P", t, j))
                b(f"p_full{t}").arrive()
            if r["active"]:
                yield ("wait", f"o_full{t}", o_cnt & 1, o_cnt)
                o_cnt += 1
                epilogues[t] += 1

    rng = random.Random(seed)
    # qk() is nested in mma() and reads that role's current item `tr`
    agents = [producer(), mma(), softmax(0), softmax(1)]
    pending = [None] * 4
    done = [False] * 4
    stalled = 0
    while not all(done):
        progressed = False
        order = list(range(4))
        rng.shuffle(order)
        # odd seeds: a random subset of the roles moves in each round, so one
        # role can run many steps ahead of another (races show up); even
        # seeds: every role in turn, and a round where none moves is a deadlock
        subset = seed % 2 == 1
        for a in order:
            if done[a] or (subset and rng.random() < 0.5):
                continue
            if pending[a] is not None:
                _, name, parity, phase = pending[a]
                bar = b(name)
                if (bar.phases & 1) == (parity & 1):
                    continue
                assert bar.phases >= phase + 1, ("wait passed before its phase completed", name)
                assert bar.phases <= phase + 2, ("barrier two phases ahead of its waiter", name)
                pending[a] = None
            try:
                pending[a] = next(agents[a])
            except StopIteration:
                done[a] = True
            progressed = True
        stalled = 0 if progressed else stalled + 1
        if (not progressed and not subset) or stalled > 1000:
            raise AssertionError(f"deadlock, waiting on {pending}")


def causal_items(n_items, levels):
    """Items of a causal band: 256-row query block q covers key blocks 0..2q
    (tile 0) and 0..2q+1 (tile 1)."""
    return [(tile_range(0, 2 * (i % levels)), tile_range(0, 2 * (i % levels) + 1)) for i in range(n_items)]


ITEM_SETS = {
    "dense": [(tile_range(0, 5), tile_range(0, 5))] * 4,
    "causal": causal_items(6, 3),
    "band": [(tile_range(2, 6), tile_range(3, 7)), (tile_range(0, 1), tile_range(1, 2))],
    "ragged_tail": [(tile_range(0, 4), INVALID), (tile_range(0, 0), tile_range(0, 0)), (tile_range(0, 3), INVALID)],
    "empty_tiles": [(tile_range(0, -1), tile_range(0, -1)), (tile_range(0, 2), tile_range(0, -1)),
                    (tile_range(0, -1), tile_range(1, 1)), (tile_range(0, 2), tile_range(0, 2))],
    "split_pieces": [(tile_range(0, 4), tile_range(0, 4)), (tile_range(5, 9), tile_range(5, 9)),
                     (tile_range(0, -1), tile_range(10, 10))],
}


@pytest.mark.parametrize("name", list(ITEM_SETS))
@pytest.mark.parametrize("stages,rope", [(4, False), (8, False), (3, True)])
def test_two_tile_protocol_finishes_in_order(name, stages, rope):
    for seed in range(25):
        run(ITEM_SETS[name], stages, rope, seed)

