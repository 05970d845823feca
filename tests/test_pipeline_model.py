"""Host-side model of the fused kernel's barrier protocol.

The kernel's roles hand shared-memory slots and TMEM accumulators to one
another through mbarriers and waits on phase parity.  A parity wait is exact
only when the phase before the awaited one has completed (and the awaited one
is the latest possible); otherwise it returns early or blocks for good.  This
model runs the roles as interleaved agents under random schedules, with TMA
copies, stores and MMA commits completing after random delays (copies also out
of order), and checks every successful wait and that every schedule finishes.

Roles and rules modelled (`x1cb_conv.cu`):
  * I/O producer: stage n into slot n % r after the slot's previous stage was
    stored (io_empty, phase parity trick), then the copy lands (io_full).
  * Store warp: stages in order; waits out_ready, then the store's read of
    the slot completes (io_empty).
  * MMA warp: accumulator slot J % n_slots after its previous use was drained
    (acc_empty), then the commit lands (acc_full).
  * Epilogue: 4 lane quarters x `turns` warps; turn g takes stages g, g+turns,
    ...: acc_full, then the slot-order guard (deep ring: io_empty of the
    slot's previous stage; shallow ring: the ticket), then io_full, then
    out_ready and acc_empty arrivals.
"""
import random

import pytest


class Early(Exception):
    pass


class Barrier:
    def __init__(self, count):
        self.count = count
        self.pending = 0
        self.completed = 0  # phases completed

    def arrive(self):
        self.pending += 1
        if self.pending == self.count:
            self.pending = 0
            self.completed += 1

    def try_wait(self, phase):
        """Hardware semantics: true iff the current phase's parity differs from
        the awaited phase's parity.  The model also knows which phase was
        meant and flags a true result for a phase that has not completed."""
        ok = (self.completed & 1) != (phase & 1)
        if ok and self.completed < phase + 1:
            raise Early(f"wait for phase {phase} returned with {self.completed} completed")
        if ok and self.completed > phase + 1:
            raise Early(f"wait for phase {phase} aliased with {self.completed} completed")
        return ok


def run(seed, stages_per_tile, tiles, r, n_slots, stages_per_sub, turns, guard=True,
        in_order_copies=False):
    rng = random.Random(seed)
    total = tiles * stages_per_tile
    io_full = [Barrier(1) for _ in range(r)]
    io_empty = [Barrier(1) for _ in range(r)]
    out_ready = [Barrier(4) for _ in range(r)]
    acc_full = [Barrier(1) for _ in range(n_slots)]
    acc_empty = [Barrier(4 * stages_per_sub) for _ in range(n_slots)]
    ticket = [0]
    # asynchronous completions [delay, seq, barrier, in_order]: TMA copies may
    # land in any order; a store's read (the store warp waits for each one)
    # and an MMA commit (it covers every earlier MMA) land in issue order
    events = []
    seq = [0]

    def later(bar, lo, hi, in_order):
        seq[0] += 1
        events.append([rng.randint(lo, hi), seq[0], bar, in_order])

    def producer():
        for n in range(total):
            s, k = n % r, n // r
            while not io_empty[s].try_wait(k - 1 if k else -1):
                yield
            later(io_full[s], 1, 60, in_order_copies)
            yield

    def store():
        for n in range(total):
            s, k = n % r, n // r
            while not out_ready[s].try_wait(k):
                yield
            later(io_empty[s], 1, 20, True)
            yield

    def mma():
        subs = total // stages_per_sub
        for J in range(subs):
            a, k = J % n_slots, J // n_slots
            while not acc_empty[a].try_wait(k - 1 if k else -1):
                yield
            later(acc_full[a], 5, 30, True)
            yield

    def epilogue(turn):
        deep = r >= turns
        for n in range(turn, total, turns):
            s, k = n % r, n // r
            J = n // stages_per_sub
            a, ka = J % n_slots, J // n_slots
            while not acc_full[a].try_wait(ka):
                yield
            if guard and deep:
                while not io_empty[s].try_wait(k - 1 if k else -1):
                    yield
            elif guard:
                while ticket[0] < n:
                    yield
            while not io_full[s].try_wait(k):
                yield
            if guard and not deep:
                ticket[0] = max(ticket[0], n + 1)
            for _ in range(rng.randint(0, 6)):  # the arithmetic
                yield
            out_ready[s].arrive()
            acc_empty[a].arrive()

    agents = [producer(), store(), mma()] + [epilogue(t) for t in range(turns) for _ in range(4)]
    live = list(agents)
    steps = 0
    while live:
        steps += 1
        if steps > 200000:
            raise AssertionError("no progress: a wait can never be satisfied")
        # land due asynchronous completions (ordered kinds wait for their
        # predecessors)
        for e in events:
            e[0] -= 1
        due = [e for e in events if e[0] <= 0]
        rng.shuffle(due)
        for e in due:
            if e[3] and any(o[3] and o[1] < e[1] for o in events):
                continue
            events.remove(e)
            e[2].arrive()
        ag = rng.choice(live)
        try:
            next(ag)
        except StopIteration:
            live.remove(ag)


def test_parity_trick_on_fresh_barrier():
    """A wait for "phase -1" (parity 1) passes on a fresh barrier: the first
    use of an empty slot needs no arrival."""
    assert Barrier(1).try_wait(-1)
    assert not Barrier(1).try_wait(0)


# Res3.2 Conv3: 4 stages per tile, N=256 accumulators (2 slots x 2 stages),
# 7-stage ring; conv1: 1 stage per tile, 4 slots, 3-stage ring; 3x3: 2 stages.
CASES = [
    dict(stages_per_tile=4, r=7, n_slots=2, stages_per_sub=2),
    dict(stages_per_tile=4, r=4, n_slots=2, stages_per_sub=2),
    dict(stages_per_tile=1, r=3, n_slots=4, stages_per_sub=1),
    dict(stages_per_tile=1, r=2, n_slots=4, stages_per_sub=1),
    dict(stages_per_tile=2, r=12, n_slots=4, stages_per_sub=1),
    # shallow I/O rings beside large resident weights or deeper activation rings
    dict(stages_per_tile=4, r=6, n_slots=2, stages_per_sub=2),
    dict(stages_per_tile=4, r=5, n_slots=2, stages_per_sub=2),
    dict(stages_per_tile=2, r=2, n_slots=2, stages_per_sub=2),
    dict(stages_per_tile=2, r=3, n_slots=2, stages_per_sub=2),
    # 8 KB stages: two 32-channel chunks, four stages per N = 256 accumulator
    dict(stages_per_tile=4, r=4, n_slots=2, stages_per_sub=4),
    dict(stages_per_tile=4, r=3, n_slots=2, stages_per_sub=4),
]


@pytest.mark.parametrize("case", CASES, ids=[f"r{c['r']}-slots{c['n_slots']}" for c in CASES])
def test_protocol_waits_are_exact(case):
    for seed in range(40):
        run(seed, tiles=12, turns=4, **case)


@pytest.mark.parametrize("r", [2, 3])
def test_model_catches_a_missing_slot_order_guard(r):
    """Without the guard, a turn can await a stage while the slot's previous
    stage (another turn's) has not landed, and the parity wait returns early.
    The shallow rings of the 3x3 (2 stages) and of conv1 (3) show it in most
    schedules; deep rings need copies landing three or more stages out of
    order, which the guard covers as well."""
    failures = 0
    for seed in range(60):
        try:
            run(seed, tiles=12, turns=4, guard=False, stages_per_tile=1, r=r, n_slots=4,
                stages_per_sub=1)
        except Early:
            failures += 1
    assert failures > 10


def test_model_catches_more_turns_than_tmem_stages():
    """Five turns span three accumulator uses of two slots: aliasing."""
    with pytest.raises((Early, AssertionError)):
        for seed in range(200):
            run(seed, tiles=12, turns=5, stages_per_tile=4, r=8, n_slots=2, stages_per_sub=2)


# ---- the activation ring with several issuing lanes --------------------------------
# The producer warp issues activation boxes in rounds: in round j lane l takes
# box n = j*lanes + l; the lanes wait for their slots' a_empty parity together
# (a warp-wide vote), then their copies go out together.  The MMA warp takes
# the boxes in order (a_full) and commits each slot back (a_empty) after a
# delay.  Copies land in any order; commits, each covering every earlier MMA
# of the issuing thread, land in issue order.  Round j's waits follow round
# j-1's, which saw box j*lanes - 1 - S consumed; a box n of round j needs box
# n - 2S consumed for its parity to name the right phase, i.e. lanes <= S.

def run_a_ring(seed, S, lanes, boxes=60):
    rng = random.Random(seed)
    a_full = [Barrier(1) for _ in range(S)]
    a_empty = [Barrier(1) for _ in range(S)]
    events = []
    last_commit = [0]

    def later(bar, in_order=False):
        d = rng.randint(1, 8)
        if in_order:  # not before the previous commit
            d = max(d, last_commit[0])
            last_commit[0] = d
        events.append([d, bar])

    def producer():
        for base in range(0, boxes, lanes):
            mine = [n for n in range(base, min(base + lanes, boxes))]
            # every lane polls its slot; the round proceeds when all are ready
            while not all(a_empty[n % S].try_wait(n // S - 1 if n >= S else -1) for n in mine):
                yield
            for n in mine:
                later(a_full[n % S])  # expect_tx + copy; lands later
            yield

    def mma():
        for n in range(boxes):
            s, k = n % S, n // S
            while not a_full[s].try_wait(k):
                yield
            later(a_empty[s], in_order=True)  # commit lands after the MMAs
            yield

    live = [producer(), mma()]
    steps = 0
    while live or events:
        steps += 1
        assert steps < 200000, "schedule did not finish"
        for e in events:
            e[0] -= 1
        last_commit[0] = max(0, last_commit[0] - 1)
        for e in [e for e in events if e[0] <= 0]:
            events.remove(e)
            e[1].arrive()
        if live:
            ag = rng.choice(live)
            try:
                next(ag)
            except StopIteration:
                live.remove(ag)


@pytest.mark.parametrize("S,lanes", [(2, 1), (3, 1), (4, 2), (5, 2), (6, 3), (7, 3), (8, 4), (14, 4),
                                     (28, 4)])
def test_issuing_rounds_within_half_the_ring_are_exact(S, lanes):
    """The kernels' choice: lanes = min(4, S // 2)."""
    for seed in range(60):
        run_a_ring(seed, S, lanes)


@pytest.mark.parametrize("S,lanes", [(3, 3), (4, 4)])
def test_issuing_rounds_up_to_the_ring_depth_are_exact(S, lanes):
    for seed in range(60):
        run_a_ring(seed, S, lanes)


@pytest.mark.parametrize("S", [2, 3])
def test_model_catches_more_issuing_lanes_than_slots(S):
    """Four lanes on a 2- or 3-slot ring: one round holds two boxes of the same
    slot, and the second one's wait can never be met (or passes early)."""
    failures = 0
    for seed in range(20):
        try:
            run_a_ring(seed, S, 4)
        except (Early, AssertionError):
            failures += 1
    assert failures == 20



# ---- two MMA warps on one activation ring -------------------------------------------
# Without a shortcut, the convolution kernel's warp 2 issues MMAs too: warp 1
# takes the CTA's even tiles, warp 2 the odd ones, each box by box.  With both
# consuming one ring, a warp can wait on a slot whose previous box (the other
# warp's) has not landed, and its parity wait passes on the box before.  Each
# warp therefore owns half of the ring (even tiles' boxes in slots 0..S/2-1,
# odd tiles' in S/2..S-1), taken in order; the producer still issues boxes in
# tile order, in rounds.

def ring_pos(n, S, bpt, split):
    if not split:
        return n % S, n // S
    half = S // 2
    t, b = divmod(n, bpt)
    li = (t // 2) * bpt + b
    return (t % 2) * half + li % half, li // half


def run_two_mma_warps(seed, S, lanes, bpt, split, tiles=16):
    rng = random.Random(seed)
    a_full = [Barrier(1) for _ in range(S)]
    a_empty = [Barrier(1) for _ in range(S)]
    events = []
    last_commit = [0, 0]
    boxes = tiles * bpt

    def later(bar, who=None):
        d = rng.randint(1, 8)
        if who is not None:  # a warp's commits land in its issue order
            d = max(d, last_commit[who])
            last_commit[who] = d
        events.append([d, bar])

    def producer():
        for base in range(0, boxes, lanes):
            mine = list(range(base, min(base + lanes, boxes)))
            pos = [ring_pos(n, S, bpt, split) for n in mine]
            while not all(a_empty[s].try_wait(k - 1 if k else -1) for s, k in pos):
                yield
            for s, _ in pos:
                later(a_full[s])
            yield

    def mma(w):
        for t in range(w, tiles, 2):
            for b in range(bpt):
                s, k = ring_pos(t * bpt + b, S, bpt, split)
                while not a_full[s].try_wait(k):
                    yield
                later(a_empty[s], who=w)
                yield

    live = [producer(), mma(0), mma(1)]
    steps = 0
    while live or events:
        steps += 1
        assert steps < 100000, "schedule did not finish"
        for e in events:
            e[0] -= 1
        last_commit[0] = max(0, last_commit[0] - 1)
        last_commit[1] = max(0, last_commit[1] - 1)
        for e in [e for e in events if e[0] <= 0]:
            events.remove(e)
            e[1].arrive()
        if live:
            ag = rng.choice(live)
            try:
                next(ag)
            except StopIteration:
                live.remove(ag)


# (S, lanes, bpt): conv1 and the 3x3 (6, 3, 4), the folded stem (12, 4, 1),
# the 3x3 on CTA pairs (14, 4, 4), small even rings
SPLIT_CASES = [(6, 3, 4), (12, 4, 1), (14, 4, 4), (16, 4, 4), (4, 2, 1), (4, 2, 3), (8, 4, 2)]


@pytest.mark.parametrize("S,lanes,bpt", SPLIT_CASES, ids=[str(c) for c in SPLIT_CASES])
def test_two_mma_warps_on_split_ring_are_exact(S, lanes, bpt):
    for seed in range(40):
        run_two_mma_warps(seed, S, lanes, bpt, split=True)


def test_model_catches_two_mma_warps_sharing_the_ring():
    """The shared ring: a warp's wait passes on the other warp's older box."""
    failures = 0
    for seed in range(40):
        try:
            run_two_mma_warps(seed, 6, 3, 4, split=False)
        except (Early, AssertionError):
            failures += 1
    assert failures > 0
