"""Discrete-event model of the persistent forward's hand-offs (host-side check).

The persistent forward (csrc/fwd_persist.cu, csrc/chain_body.cuh) runs chain
CTAs and worker CTAs in one cooperative grid that hand records and state images
to one another through rings and flags.  This model replays those rules with
random timing and worker counts and checks that
  * every run finishes (the fixed item order cannot deadlock), and
  * no ring slot is overwritten before its last reader is done:
    prep(c) reuses record slot c % RING only after the chain has consumed record
    c - RING and output(c - RING) has read it; the chain exports state image e
    into slot e % RING only after output(e - RING) has read it.
It also checks that the model does catch a deadlock (an order whose output lag
equals the ring depth).  The constants are those of launch.h and chain_body.cuh.
"""
import random

import pytest

RING, LAG, PUBLISH_EVERY = 24, 16, 2


def item(n, P, bh, lag):
    """Item n of the workers' order: (kind, chunk, head), kind 0 = prep, 1 = outputs."""
    if n < 0:
        return None
    lag = min(lag, P)
    head = lag * bh
    if n < head:
        return (0, n // bh, n % bh)
    n -= head
    mid = 2 * bh * (P - lag)
    if n < mid:
        g, k = lag + n // (2 * bh), n % (2 * bh)
        return (0, g, k) if k < bh else (1, g - lag, k - bh)
    n -= mid
    if n < head:
        return (1, P - lag + n // bh, n % bh)
    return None


def simulate(bh, NT, P, W, NS, seed, ring=RING, lag=LAG, max_ticks=200000):
    rnd = random.Random(seed)
    rec_gen = [[0] * ring for _ in range(bh)]
    out_gen = [[0] * ring for _ in range(bh)]
    done_out = set()
    chains = [[dict(seen=0, loaded=0, upd=0, exported=0, prog=0) for _ in range(NT)] for _ in range(bh)]
    workers = [None] * W
    nxt = done = 0
    for tick in range(max_ticks):
        for r in range(bh):
            for ch in chains[r]:
                # producer: record flag first (records seen), then the stage
                c = ch["seen"]
                if c < P and c == ch["loaded"] and rec_gen[r][c % ring] >= c // ring + 1 and rnd.random() < 0.7:
                    ch["seen"] += 1
                c = ch["loaded"]
                if c < ch["seen"] and c < ch["upd"] + NS and rnd.random() < 0.7:
                    ch["loaded"] += 1
                # state update of chunk upd (its stage loaded)
                if ch["upd"] < ch["loaded"] and rnd.random() < 0.7:
                    ch["upd"] += 1
                # export of state image e (computed, record e seen): its slot must be free
                e = ch["exported"]
                if e < P and e <= ch["upd"] and ch["seen"] >= e + 1 and rnd.random() < 0.7:
                    assert e < ring or (r, e - ring) in done_out, "state-image slot overwritten"
                    ch["exported"] += 1
                # publisher: progress every PUBLISH_EVERY exports, and at the end
                n = min(ch["prog"] + PUBLISH_EVERY, P)
                if ch["prog"] < P and ch["exported"] >= n and rnd.random() < 0.5:
                    ch["prog"] = n
        for w in range(W):
            if workers[w] is None:
                it = item(nxt, P, bh, lag)
                if it is None:
                    continue
                nxt += 1
                workers[w] = [it, rnd.randint(1, 6), False]
            it, _, started = workers[w]
            kind, c, r = it
            if not started:
                if kind == 0:
                    ready = c < ring or (out_gen[r][c % ring] >= c // ring
                                         and all(ch["prog"] >= c - ring + 2 for ch in chains[r]))
                    if ready and c >= ring:
                        assert all(ch["upd"] >= c - ring + 1 for ch in chains[r]), "record slot in use by the chain"
                        assert (r, c - ring) in done_out, "record slot in use by an output"
                else:
                    ready = rec_gen[r][c % ring] >= c // ring + 1 and all(ch["prog"] >= c + 1 for ch in chains[r])
                workers[w][2] = ready
                continue
            workers[w][1] -= 1
            if workers[w][1] <= 0:
                if kind == 0:
                    rec_gen[r][c % ring] = c // ring + 1
                else:
                    out_gen[r][c % ring] = c // ring + 1
                    done_out.add((r, c))
                workers[w] = None
                done += 1
        if done == 2 * bh * P and all(ch["prog"] == P and ch["upd"] == P for cs in chains for ch in cs):
            return tick
    return None


@pytest.mark.parametrize("trial", range(40))
def test_persistent_order_finishes_and_keeps_slots(trial):
    rnd = random.Random(trial)
    bh = rnd.choice([1, 2, 3])
    NT = rnd.choice([1, 2])
    P = rnd.choice([1, 2, 7, 16, 17, 24, 25, 40, 60])
    W = rnd.choice([1, 2, 3, 7, 24])
    NS = rnd.choice([2, 3])
    assert simulate(bh, NT, P, W, NS, seed=trial) is not None


def test_item_order_covers_every_item_once():
    for P in (1, 2, 15, 16, 17, 64, 1024):
        for bh in (1, 3, 16):
            items = [item(n, P, bh, LAG) for n in range(2 * P * bh)]
            assert None not in items and len(set(items)) == 2 * P * bh
            pos = {it: n for n, it in enumerate(items)}
            assert all(pos[(0, c, r)] < pos[(1, c, r)] for c in range(P) for r in range(bh))
            assert item(-1, P, bh, LAG) is None and item(2 * P * bh, P, bh, LAG) is None


def test_model_detects_a_deadlocking_order():
    """With the output lag equal to the ring depth and one worker, prep(c) waits
    for output(c - ring), which comes after it in the order."""
    assert simulate(2, 2, 40, 1, 3, seed=0, ring=8, lag=8, max_ticks=20000) is None
    assert simulate(2, 2, 40, 1, 3, seed=0, ring=8, lag=7, max_ticks=200000) is not None
