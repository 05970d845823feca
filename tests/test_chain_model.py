"""Host-side model of the fused conv2 -> conv3 kernel's barrier protocol
(x1cb_chain.cu): two CTAs sharing each MMA, one ring of four accumulator
slots filled in issue order with Conv2 tiles and Conv3 chunks, two Conv3 A
buffers, a shortcut ring per CTA.

Roles run as interleaved agents under random schedules; TMA copies land after
random delays and out of order, MMA commits in issue order.  Every parity
wait is checked to be exact (the awaited phase complete, the barrier not a
whole phase ahead) and every schedule must finish.  Planted mistakes (no
stage-order ticket, more epilogue turns than slots) must be caught.
"""
import random

import pytest

from tests.test_pipeline_model import Barrier, Early


def run(seed, tiles, n_chunks, r, a_stages, turns=4, ticket_guard=True, c1=4):
    rng = random.Random(seed)
    SLOTS = 4
    # rank 0's barriers fed from both CTAs
    a_full = [Barrier(3) for _ in range(a_stages)]   # leader's expect + both CTAs' copies
    acc_empty = [Barrier(8) for _ in range(SLOTS)]   # 4 quarter-warps x 2 CTAs
    a3_full = [Barrier(8) for _ in range(2)]
    # per-CTA barriers (commits multicast to both)
    a_empty = [[Barrier(1) for _ in range(a_stages)] for _ in range(2)]
    acc_full = [[Barrier(1) for _ in range(SLOTS)] for _ in range(2)]
    a3_empty = [[Barrier(1) for _ in range(2)] for _ in range(2)]
    io_full = [[Barrier(1) for _ in range(r)] for _ in range(2)]
    io_empty = [[Barrier(1) for _ in range(r)] for _ in range(2)]
    out_ready = [[Barrier(4) for _ in range(r)] for _ in range(2)]
    ticket = [0, 0]
    events, seq = [], [0]

    def later(bars, lo, hi, in_order):
        seq[0] += 1
        events.append([rng.randint(lo, hi), seq[0], bars, in_order])

    def producer(cta):
        n = 0
        for _ in range(tiles):
            for _ in range(c1):
                s, k = n % a_stages, n // a_stages
                while not a_empty[cta][s].try_wait(k - 1 if k else -1):
                    yield
                if cta == 0:
                    a_full[s].arrive()  # arrive.expect_tx
                later([a_full[s]], 1, 50, False)
                n += 1
                yield

    def io_producer(cta):
        for n in range(tiles * n_chunks):
            s, k = n % r, n // r
            while not io_empty[cta][s].try_wait(k - 1 if k else -1):
                yield
            later([io_full[cta][s]], 1, 60, False)
            yield

    def store(cta):
        for n in range(tiles * n_chunks):
            s, k = n % r, n // r
            while not out_ready[cta][s].try_wait(k):
                yield
            later([io_empty[cta][s]], 1, 20, True)
            yield

    def mma():
        slot_use = 0
        n = 0
        for i in range(tiles + 1):
            if i < tiles:
                sl, k = slot_use % SLOTS, slot_use // SLOTS
                while not acc_empty[sl].try_wait(k - 1 if k else -1):
                    yield
                for _ in range(c1):
                    s, ka = n % a_stages, n // a_stages
                    while not a_full[s].try_wait(ka):
                        yield
                    later([a_empty[0][s], a_empty[1][s]], 3, 15, True)
                    n += 1
                    yield
                later([acc_full[0][sl], acc_full[1][sl]], 3, 15, True)
                slot_use += 1
            if i >= 1:
                j = i - 1
                b = j & 1
                while not a3_full[b].try_wait(j >> 1):
                    yield
                for _ in range(n_chunks):
                    sl, k = slot_use % SLOTS, slot_use // SLOTS
                    while not acc_empty[sl].try_wait(k - 1 if k else -1):
                        yield
                    later([acc_full[0][sl], acc_full[1][sl]], 3, 15, True)
                    slot_use += 1
                    yield
                later([a3_empty[0][b], a3_empty[1][b]], 3, 15, True)

    def epilogue(cta, turn):
        k = 0
        uses = 0
        for i in range(tiles + 1):
            if i < tiles:
                if k % turns == turn:
                    sl = k % SLOTS
                    while not acc_full[cta][sl].try_wait(uses):
                        yield
                    b = i & 1
                    while not a3_empty[cta][b].try_wait((i >> 1) - 1 if i >= 2 else -1):
                        yield
                    for _ in range(rng.randint(0, 4)):
                        yield
                    acc_empty[sl].arrive()
                    a3_full[b].arrive()
                    uses += 1
                k += 1
            if i >= 1:
                j = i - 1
                for c in range(n_chunks):
                    if k % turns == turn:
                        sl = k % SLOTS
                        n = j * n_chunks + c
                        s, ks = n % r, n // r
                        while not acc_full[cta][sl].try_wait(uses):
                            yield
                        if ticket_guard:
                            while ticket[cta] < n:
                                yield
                        while not io_full[cta][s].try_wait(ks):
                            yield
                        if ticket_guard:
                            ticket[cta] = max(ticket[cta], n + 1)
                        for _ in range(rng.randint(0, 6)):
                            yield
                        out_ready[cta][s].arrive()
                        acc_empty[sl].arrive()
                        uses += 1
                    k += 1

    agents = [mma()]
    for cta in range(2):
        agents += [producer(cta), io_producer(cta), store(cta)]
        agents += [epilogue(cta, t) for t in range(turns) for _ in range(4)]
    live = list(agents)
    steps = 0
    while live:
        steps += 1
        if steps > 400000:
            raise AssertionError("no progress: a wait can never be satisfied")
        for e in events:
            e[0] -= 1
        due = [e for e in events if e[0] <= 0]
        rng.shuffle(due)
        for e in due:
            if e[3] and any(o[3] and o[1] < e[1] for o in events):
                continue
            events.remove(e)
            for bar in e[2]:
                bar.arrive()
        ag = rng.choice(live)
        try:
            next(ag)
        except StopIteration:
            live.remove(ag)


CASES = [
    dict(n_chunks=4, r=3, a_stages=4),    # Res3.2 block: 512 outputs, 3 shortcut stages
    dict(n_chunks=4, r=2, a_stages=2),
    dict(n_chunks=1, r=2, a_stages=4),    # 128 outputs: one chunk per tile
    dict(n_chunks=8, r=5, a_stages=3),    # 1024 outputs
    dict(n_chunks=3, r=7, a_stages=4),
]


@pytest.mark.parametrize("case", CASES, ids=[f"ch{c['n_chunks']}-r{c['r']}" for c in CASES])
def test_chain_protocol_waits_are_exact(case):
    for seed in range(25):
        run(seed, tiles=7, **case)


def test_model_catches_a_missing_stage_order_ticket():
    """Conv3 chunks reach the turns in an irregular pattern (Conv2 items sit
    between them), so without the ticket a turn can await a stage whose
    previous phase (another turn's) has not landed."""
    failures = 0
    for seed in range(60):
        try:
            run(seed, tiles=7, n_chunks=4, r=2, a_stages=4, ticket_guard=False)
        except Early:
            failures += 1
    assert failures > 5


def test_model_catches_more_turns_than_slots():
    with pytest.raises((Early, AssertionError)):
        for seed in range(100):
            run(seed, tiles=7, n_chunks=4, r=3, a_stages=4, turns=5)
