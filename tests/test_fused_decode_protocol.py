"""Host model of the fused decode kernel's work protocol (decode_fused.cu):
every CTA's producer, consumer warps and bookkeeper warp as coroutines over
the same shared counters, queues and flags, run under random schedules.

The GPU parity tests check the results of real runs; this checks the property
they can only sample: under any interleaving the protocol finishes, runs every
sequence's top-k exactly once and every attention item exactly once.  Each
role follows the kernel's rules step for step; a role waiting on a condition
yields until it holds.  If every live role is waiting, that schedule would
have deadlocked (the kernel's bounded waits would give up): the test fails.

A second test removes one rule on purpose (the producer's wait for its own
bookkeeper before it ends) and checks that the model then finds a schedule
that gets stuck, so the model is able to see the failure it guards against.
"""
import collections
import random

import pytest

K_QUEUE, K_RED_Q, K_FIFO = 4, 4, 16


class World:
    def __init__(self, nb, H, n_cta):
        self.nb, self.H = nb, H
        self.units = [(b, j) for b, n in enumerate(nb) for j in range(n)]
        self.total_attn = H * len(nb)
        self.c_unit = self.c_alloc = self.c_claim = self.c_pub = 0
        self.aq_item = [None] * self.total_attn
        self.aq_flag = [0] * self.total_attn
        self.seq_done = [0] * len(nb)
        self.topk_runs = collections.Counter()
        self.attn_runs = collections.Counter()
        self.n_cta = n_cta


class Cta:
    def __init__(self):
        self.wq = collections.deque()        # producer -> consumers (capacity K_QUEUE)
        self.red = collections.deque()       # consumers -> bookkeeper (capacity K_RED_Q)
        self.fifo = collections.deque()      # bookkeeper -> producer (capacity K_FIFO)
        self.book_done = 0


def producer(W, C, wait_for_bookkeeper=True):
    def push(entry):
        while len(C.wq) >= K_QUEUE:
            yield "wait"
        C.wq.append(entry)

    def drain():
        while C.fifo:
            b = C.fifo[0]
            yield from push(("topk", b))
            C.fifo.popleft()

    pending, pending_flag = -1, 0
    seen_claim = seen_pub = 0
    index_left, attn_left = True, W.total_attn > 0
    units_pushed = 0
    u_next = W.c_unit                      # claimed one unit ahead
    W.c_unit += 1
    yield "step"
    while True:
        yield from drain()
        if pending < 0 and attn_left:
            if not index_left:
                seen_claim = W.c_claim
            if seen_claim >= W.total_attn:
                attn_left = False
            elif not index_left or seen_claim < seen_pub:
                h = W.c_claim
                W.c_claim += 1
                if h >= W.total_attn:
                    attn_left = False
                else:
                    pending, pending_flag = h, 0
                seen_claim = h + 1
            yield "step"
        if pending >= 0 and (not index_left or pending_flag):
            item, pending = pending, -1
            while not W.aq_flag[item]:
                # queue this CTA's own top-k requests while waiting
                yield from drain()
                if not W.aq_flag[item]:
                    yield "wait"
            yield from push(("attn", W.aq_item[item]))
            continue
        if index_left:
            u = u_next
            if u >= len(W.units):
                index_left = False
                continue
            u_next = W.c_unit
            W.c_unit += 1
            if pending >= 0:
                pending_flag = W.aq_flag[pending]
            elif attn_left:
                seen_claim, seen_pub = W.c_claim, W.c_pub
            yield from push(("index",) + W.units[u])
            units_pushed += 1
            continue
        if not attn_left:
            break
    if wait_for_bookkeeper:
        while C.book_done < units_pushed:
            yield from drain()
            if C.book_done < units_pushed:
                yield "wait"
    yield from drain()
    yield from push(("end",))


def consumers(W, C):
    while True:
        while not C.wq:
            yield "wait"
        entry = C.wq.popleft()
        kind = entry[0]
        if kind == "end":
            break
        if kind == "index":
            while len(C.red) >= K_RED_Q:
                yield "wait"
            C.red.append(entry[1:])
        elif kind == "topk":
            b = entry[1]
            W.topk_runs[b] += 1
            base = W.c_alloc                 # publish one item per group
            W.c_alloc += W.H
            yield "step"
            for g in range(W.H):
                W.aq_item[base + g] = (b, g)
            yield "step"
            for g in range(W.H):
                W.aq_flag[base + g] = 1
            yield "step"
            W.c_pub += W.H
        else:
            W.attn_runs[entry[1]] += 1
        yield "step"
    while len(C.red) >= K_RED_Q:
        yield "wait"
    C.red.append(None)                       # end of the bookkeeper's stream


def bookkeeper(W, C):
    while True:
        while not C.red:
            yield "wait"
        unit = C.red.popleft()
        if unit is None:
            return
        b, _ = unit
        W.seq_done[b] += W.H
        if W.seq_done[b] == W.H * W.nb[b]:
            while len(C.fifo) >= K_FIFO:
                yield "wait"
            C.fifo.append(b)
        C.book_done += 1
        yield "step"


def run(nb, H, n_cta, seed, wait_for_bookkeeper=True, max_steps=200000):
    """Random schedule; returns the world, or None if every live role waits."""
    W = World(nb, H, n_cta)
    rng = random.Random(seed)
    procs = []
    for _ in range(n_cta):
        C = Cta()
        procs += [producer(W, C, wait_for_bookkeeper), consumers(W, C), bookkeeper(W, C)]
    live = list(range(len(procs)))
    waiting = set()
    for _ in range(max_steps):
        if not live:
            return W
        runnable = [i for i in live if i not in waiting] or live
        i = rng.choice(runnable)
        try:
            r = next(procs[i])
        except StopIteration:
            live.remove(i)
            waiting.clear()
            continue
        if r == "wait":
            waiting.add(i)
            if waiting >= set(live):
                # every live role retried and still waits: re-check all once
                progressed = False
                for j in list(live):
                    try:
                        if next(procs[j]) != "wait":
                            progressed = True
                    except StopIteration:
                        live.remove(j)
                        progressed = True
                if not progressed:
                    return None
                waiting.clear()
        else:
            waiting.clear()
    raise AssertionError("schedule did not finish within the step bound")


CASES = [
    # (blocks per sequence, groups, CTAs)
    ([3, 1, 5], 2, 4),
    ([8] * 8, 8, 6),
    ([1], 1, 3),
    ([2, 40, 1, 7, 3], 4, 5),
    ([16, 16], 16, 16),
]


@pytest.mark.parametrize("nb,H,n_cta", CASES)
def test_every_schedule_finishes_and_runs_each_step_once(nb, H, n_cta):
    for seed in range(60):
        W = run(nb, H, n_cta, seed)
        assert W is not None, f"stuck under schedule {seed}"
        assert W.c_pub == W.total_attn
        assert all(W.topk_runs[b] == 1 for b in range(len(nb)))
        assert sorted(W.attn_runs) == [(b, g) for b in range(len(nb)) for g in range(H)]
        assert all(v == 1 for v in W.attn_runs.values())


def test_model_sees_a_producer_that_ends_before_its_bookkeeper():
    """Without the end-of-work wait, a CTA can end with a top-k request still
    unqueued; the other CTAs then wait for an item nobody publishes."""
    stuck = sum(run([2, 3, 1], 2, 3, seed, wait_for_bookkeeper=False) is None
                for seed in range(300))
    assert stuck > 0
