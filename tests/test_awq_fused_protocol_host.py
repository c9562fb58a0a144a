"""CPU model of the fused AWQ loss kernel's mbarrier protocol
(awq_loss_fused_kernel in csrc/wq_awq.cu).

The kernel's roles run as coroutines over modelled mbarriers (arrival count,
transaction bytes, phase parity as try_wait.parity sees it):

* W producer: 32 lanes; per quantization group g it waits w_empty (phase of
  g - 1), lane 0 arms w_full with the stage's bytes and issues the TMA, every
  lane writes its share of the group's s slot (g mod 2) and arrives (w_full
  counts 33);
* X producer: per 64-channel step kt it waits x_empty (phase of kt - 2) and
  arms x_full (two stages);
* error rows (128 threads): wait w_full, copy the row, arrive w_empty, then
  per half h wait e_empty of slot (2g + h) mod 4 (phase of that slot's previous
  use), write E, arrive e_full;
* MMA: per kt wait e_full and x_full, then an asynchronous commit to x_empty
  and e_empty; a final commit to accum.

TMA landings and MMA completions are delivered at random later points. The
checks: every schedule terminates (no deadlock), every stage, slot and s entry
holds the group or step its reader expects (so no wait passes on a phase of
another use), and nothing is overwritten while a reader still needs it. Two
planted protocol mistakes are run to show the model catches them.
"""
import random

import pytest

XS, ES, SS = 2, 4, 2          # X stages, E slots, s slots
ERR_THREADS, LANES = 128, 32


class Bar:
    """An mbarrier: a phase completes when every arrival and byte is in."""

    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.phase = 0  # completed phases

    def arrive(self):
        self.pending -= 1
        assert self.pending >= 0, "more arrivals than the barrier counts"
        self._maybe_complete()

    def expect_tx(self, nbytes):
        self.tx += nbytes

    def complete_tx(self, nbytes):
        self.tx -= nbytes
        assert self.tx >= 0
        self._maybe_complete()

    def _maybe_complete(self):
        if self.pending == 0 and self.tx == 0:
            self.phase += 1
            self.pending = self.count

    def passed(self, parity):
        # try_wait.parity P succeeds once the phase of parity P has completed
        return (self.phase & 1) != parity


def run_protocol(G, seed, early_w_release=False, wrong_e_parity=False):
    rnd = random.Random(seed)
    KT = 2 * G
    x_full = [Bar(1) for _ in range(XS)]
    x_empty = [Bar(1) for _ in range(XS)]
    w_full, w_empty = Bar(1 + LANES), Bar(ERR_THREADS)
    e_full = [Bar(ERR_THREADS) for _ in range(ES)]
    e_empty = [Bar(1) for _ in range(ES)]
    accum = Bar(1)
    events = []                               # asynchronous completions
    state = {"W": None, "W_readers": 0, "s": [None] * SS, "E": [None] * ES, "X": [None] * XS,
             "mma_E": [False] * ES, "mma_X": [False] * XS, "e_written": [set() for _ in range(ES)],
             "reading_s": {}, "lane0_w_ok": set()}

    def wait(bar, parity):
        while not bar.passed(parity):
            yield

    def w_producer(lane):
        for g in range(G):
            if g > 0:
                if lane == 0:
                    yield from wait(w_empty, (g - 1) & 1)
                    state["lane0_w_ok"].add(g)
                else:
                    while g not in state["lane0_w_ok"]:
                        yield
            if lane == 0:
                assert state["W_readers"] == 0, ("W stage refilled while read", g)
                w_full.expect_tx(32768)
                w_full.arrive()

                def land(g=g):
                    state["W"], state["W_readers"] = g, ERR_THREADS
                    w_full.complete_tx(32768)
                events.append(land)
                slot = g % SS
                for t, grp in state["reading_s"].items():
                    assert grp is None or grp % SS != slot or grp >= g, ("s slot rewritten while read", g, t)
                state["s"][slot] = g
            yield
            w_full.arrive()

    def x_producer():
        for kt in range(KT):
            xs = kt % XS
            if kt >= XS:
                yield from wait(x_empty[xs], ((kt // XS) - 1) & 1)
            assert not state["mma_X"][xs], "X stage refilled while the MMA reads it"
            x_full[xs].expect_tx(65536)
            x_full[xs].arrive()

            def land(xs=xs, kt=kt):
                state["X"][xs] = kt
                x_full[xs].complete_tx(65536)
            events.append(land)
            yield

    def mma():
        for kt in range(KT):
            es, xs = kt % ES, kt % XS
            yield from wait(e_full[es], (kt // ES) & 1)
            yield from wait(x_full[xs], (kt // XS) & 1)
            assert state["E"][es] == kt, ("E slot holds", state["E"][es], "expected", kt)
            assert state["X"][xs] == kt, ("X stage holds", state["X"][xs], "expected", kt)
            state["mma_E"][es] = state["mma_X"][xs] = True

            def done(es=es, xs=xs):
                state["mma_E"][es] = state["mma_X"][xs] = False
                x_empty[xs].arrive()
                e_empty[es].arrive()
            events.append(done)
            yield
        events.append(accum.arrive)

    def error_row(t):
        for g in range(G):
            yield from wait(w_full, g & 1)
            if early_w_release:            # planted: release the stage before copying it
                w_empty.arrive()
                yield
            assert state["W"] == g, ("W stage holds", state["W"], "expected", g)
            assert state["s"][g % SS] == g, ("s slot holds", state["s"][g % SS], "expected", g)
            state["W_readers"] -= 1
            state["reading_s"][t] = g
            if not early_w_release:
                w_empty.arrive()
            yield
            for h in range(2):
                kt = 2 * g + h
                es = kt % ES
                if kt >= ES:
                    parity = (kt // ES) & 1 if wrong_e_parity else ((kt // ES) - 1) & 1
                    yield from wait(e_empty[es], parity)
                assert not state["mma_E"][es], "E slot rewritten while the MMA reads it"
                assert state["s"][g % SS] == g, ("s slot changed under its reader", g)
                yield
                state["e_written"][es].add(t)
                if len(state["e_written"][es]) == ERR_THREADS:
                    state["E"][es] = kt
                    state["e_written"][es].clear()
                e_full[es].arrive()
            state["reading_s"][t] = None
        yield from wait(accum, 0)

    roles = [x_producer(), mma()] + [w_producer(l) for l in range(LANES)] + [error_row(t) for t in range(ERR_THREADS)]
    steps = 0
    while roles or events:
        order = list(range(len(roles)))
        rnd.shuffle(order)
        finished = set()
        for i in order[: max(1, len(order) // 3)]:
            try:
                next(roles[i])
            except StopIteration:
                finished.add(i)
        roles = [r for i, r in enumerate(roles) if i not in finished]
        if events and rnd.random() < 0.5:
            events.pop(rnd.randrange(len(events)))()
        steps += 1
        if steps > 50_000:  # a correct schedule of 8 groups takes a few thousand
            raise RuntimeError("no progress: deadlock")
    assert accum.phase == 1


@pytest.mark.parametrize("G", [1, 2, 3, 5, 8])
def test_fused_loss_protocol_has_no_deadlock_or_aliasing(G):
    for seed in range(4):
        run_protocol(G, seed)


def test_protocol_model_catches_planted_mistakes():
    with pytest.raises(RuntimeError, match="deadlock"):
        run_protocol(4, 0, wrong_e_parity=True)
    caught = 0
    for seed in range(6):
        try:
            run_protocol(4, seed, early_w_release=True)
        except AssertionError:
            caught += 1
    assert caught > 0
