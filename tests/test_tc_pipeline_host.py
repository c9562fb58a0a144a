"""CPU models of the tensor-core W4A16 GEMM's schedule and barrier protocol
(w4a16_gemm_tc_kernel in csrc/wq_gemm_tc.cu). Nothing here needs a GPU.

1. Stream-K schedule. CTA c of P takes the stage units [c U / P, (c + 1) U / P)
   of U = row tiles x stages per tile; a maximal run of one tile's stages is a
   segment. The host enables the schedule only when every CTA has at most one
   tile's worth of units (ceil(U / P) <= stages per tile) and P <= U / 2. The
   checks restate the kernel's index formulas and compare them with brute
   force: every unit is computed exactly once; a CTA has at most two segments;
   a segment that holds a whole tile writes Y itself and every other tile has
   one reducer (the warp that arrives last at the tile's counter), which sums
   the contributors' fp32 slots in CTA order, so the result does not depend on
   arrival order; the counters end at zero.

2. Barrier protocol. The kernel's roles run as coroutines over modelled
   mbarriers (arrivals, transaction bytes, phase parity as try_wait.parity
   sees it):

   * producer (one thread): per stage kt, wait sempty[kt % S] (the phase of
     kt - S), arm full[kt % S] and issue the loads; at the end wait for its
     last S copies to land;
   * dequantizing warps (NH quartets of 4 warps, quartet h taking the stages
     kt = h mod NH): wait full, read the packed tile, publish the quartet's
     previous stage (32 arrivals per warp on afull), wait aempty[kt % NA] (the
     phase of kt - NA), store into tensor-memory buffer kt % NA; the last
     stage is published after the loop; then each segment's epilogue waits
     accum[segment];
   * MMA (one thread): per stage wait afull, issue, commit to aempty and
     sempty; after a segment's last stage commit to accum[segment]. Commits
     arrive when every earlier MMA has completed (in order).

   TMA landings and MMA completions happen at random later points. The checks:
   every schedule ends (no deadlock); each stage, buffer and accumulator holds
   what its reader expects (no wait passes on the phase of another use);
   nothing is overwritten while a reader still needs it. Planted mistakes
   (a ring no deeper than the quartet count, an off-by-one parity, a refill
   without waiting for the MMA) are run to show that the model catches them.
"""
import random
from collections import deque

import pytest


# ---------------------------------------------------------------------------
# 1. Stream-K schedule
# ---------------------------------------------------------------------------

def host_streamk_ctas(cps, sms, units):
    """tc_streamk_ctas: every resident slot, at most units / 2 CTAs."""
    P = min(cps * sms, units // 2)
    return max(P, 1)


def host_enables_streamk(tiles, KT_all, P):
    """The schedule-related part of the host's stream-K condition."""
    units = tiles * KT_all
    return tiles <= 64 * 1024 // 16 and (units + P - 1) // P <= KT_all


def cta_plan(c, P, tiles, KT_all):
    """The kernel's per-CTA quantities, as it computes them."""
    U = tiles * KT_all
    u0, u1 = c * U // P, (c + 1) * U // P
    KT = u1 - u0
    tile0, kg0 = u0 // KT_all, u0 % KT_all
    nseg = 2 if KT > 0 and (u1 - 1) // KT_all != tile0 else 1
    ke0 = KT_all if nseg == 2 else kg0 + KT
    ke1 = (u1 - 1) % KT_all + 1 if nseg == 2 else 0
    kg1 = (u1 - 1) % KT_all
    two = (u1 - 1) // KT_all != tile0
    whole0 = kg0 == 0 and (two or kg1 == KT_all - 1)
    whole1 = kg1 == KT_all - 1
    segs = [(tile0, kg0, ke0, whole0)]
    if nseg == 2:
        segs.append((tile0 + 1, 0, ke1, whole1))
    return dict(u0=u0, u1=u1, KT=KT, segs=segs, two=two)


def owner(u, P, U):
    return ((u + 1) * P - 1) // U


def first_unit(c, P, U):
    return c * U // P


def check_schedule(tiles, KT_all, P):
    U = tiles * KT_all
    plans = [cta_plan(c, P, tiles, KT_all) for c in range(P)]
    covered = {}
    for c, p in enumerate(plans):
        assert p["KT"] >= 2, "every CTA takes at least two stages"
        assert p["KT"] <= KT_all, "at most one tile's worth of stages"
        assert len(p["segs"]) <= 2
        # the units of [u0, u1) span at most two tiles, so the segments are all of them
        assert (p["u1"] - 1) // KT_all - p["u0"] // KT_all <= 1
        for seg, (t, kb, ke, _) in enumerate(p["segs"]):
            assert 0 <= kb < ke <= KT_all
            for k in range(kb, ke):
                assert (t, k) not in covered, "a unit computed twice"
                covered[(t, k)] = (c, seg)
            for u in range(t * KT_all + kb, t * KT_all + ke):
                assert owner(u, P, U) == c
    assert len(covered) == U, "every unit computed"
    # per tile: contributors, whole-tile writers, reducer slots
    for t in range(tiles):
        contrib = sorted({covered[(t, k)][0] for k in range(KT_all)})
        cfirst, clast = owner(t * KT_all, P, U), owner(t * KT_all + KT_all - 1, P, U)
        assert contrib == list(range(cfirst, clast + 1)), "contributors are consecutive CTAs"
        writers = [(c, seg) for c in contrib for seg, s in enumerate(plans[c]["segs"]) if s[0] == t and s[3]]
        if len(contrib) == 1:
            c = contrib[0]
            assert len(writers) == 1 and writers[0][0] == c, "a tile held whole by one CTA writes Y itself"
        else:
            assert writers == [], "a shared tile is never written whole by a contributor"
            for c in contrib:
                seg = [j for j, s in enumerate(plans[c]["segs"]) if s[0] == t]
                assert len(seg) == 1
                wc = 0 if first_unit(c, P, U) // KT_all == t else 1
                assert wc == seg[0], "the reducer reads the slot the contributor wrote"
                assert 2 * c + wc < 2 * P
    return plans, covered


def gated_configs():
    rnd = random.Random(5)
    out = [(224, 64, 1, 148), (64, 64, 2, 148), (86, 32, 2, 148), (32, 86, 2, 148), (1, 2, 1, 148),
           (3, 2, 4, 148), (7, 5, 2, 16), (224, 128, 2, 148)]
    while len(out) < 300:
        tiles, KT_all, cps, sms = rnd.randint(1, 300), rnd.randint(2, 160), rnd.choice([1, 2, 4]), rnd.randint(1, 160)
        out.append((tiles, KT_all, cps, sms))
    return out


def test_streamk_schedule_covers_every_unit_once_with_one_reducer_per_shared_tile():
    checked = 0
    for tiles, KT_all, cps, sms in gated_configs():
        U = tiles * KT_all
        if U < 2:
            continue
        P = host_streamk_ctas(cps, sms, U)
        if not host_enables_streamk(tiles, KT_all, P):
            continue
        check_schedule(tiles, KT_all, P)
        checked += 1
    assert checked > 150


def test_streamk_gate_is_what_bounds_the_segments():
    # Without the host's ceil(U / P) <= stages-per-tile condition a CTA can
    # span three tiles, which the kernel's two segments cannot express.
    tiles, KT_all, P = 10, 2, 3           # 20 units over 3 CTAs: 6 or 7 units each
    assert not host_enables_streamk(tiles, KT_all, P)
    with pytest.raises(AssertionError):
        check_schedule(tiles, KT_all, P)


def test_streamk_reduction_is_independent_of_arrival_order():
    import numpy as np
    tiles, KT_all, P = 37, 24, 52
    assert host_enables_streamk(tiles, KT_all, P)
    plans, covered = check_schedule(tiles, KT_all, P)
    U = tiles * KT_all
    rng = np.random.default_rng(0)
    partial = rng.standard_normal((tiles, KT_all)).astype(np.float32)   # one stage's contribution
    # each contributor's fp32 slot for tile t: the sum of its stages of t, in stage order
    slots = {}
    for (t, k), (c, seg) in sorted(covered.items()):
        slots[(c, seg)] = np.float32(slots.get((c, seg), np.float32(0)) + partial[t, k])
    reference = None
    for trial in range(5):
        cnt = {(t, q): 0 for t in range(tiles) for q in range(4)}
        out = {}
        arrivals = [(c, seg, q) for c, p in enumerate(plans) for seg, s in enumerate(p["segs"]) if not s[3]
                    for q in range(4)]
        random.Random(trial).shuffle(arrivals)
        for c, seg, q in arrivals:
            t = plans[c]["segs"][seg][0]
            cfirst, clast = owner(t * KT_all, P, U), owner(t * KT_all + KT_all - 1, P, U)
            arrived = cnt[(t, q)]
            cnt[(t, q)] += 1
            if arrived == clast - cfirst:        # the last arrival reduces and resets
                cnt[(t, q)] = 0
                acc = np.float32(0)
                for cc in range(cfirst, clast + 1):
                    wc = 0 if first_unit(cc, P, U) // KT_all == t else 1
                    acc = np.float32(acc + slots[(cc, wc)])
                assert (t, q) not in out
                out[(t, q)] = acc
        assert all(v == 0 for v in cnt.values()), "every counter ends at zero"
        for c, p in enumerate(plans):
            for seg, s in enumerate(p["segs"]):
                if s[3]:
                    for q in range(4):
                        out[(s[0], q)] = slots[(c, seg)]
        assert len(out) == 4 * tiles, "every tile written, each lane quarter once"
        if reference is None:
            reference = out
        assert out == reference, "bit-identical whatever the arrival order"


# ---------------------------------------------------------------------------
# 2. Barrier protocol
# ---------------------------------------------------------------------------

WARPS = 4          # dequantizing warps per quartet (one per TMEM lane quarter)


class Bar:
    """An mbarrier: a phase completes when every arrival and byte is in."""

    def __init__(self, count):
        self.count = count
        self.pending = count
        self.tx = 0
        self.phase = 0  # completed phases

    def arrive(self, n=1):
        self.pending -= n
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


def run_pipeline(seg_lens, S, NA, NH, seed, wrong_aempty_parity=False, no_sempty_wait=False):
    """seg_lens: stages of each segment (one or two segments)."""
    rnd = random.Random(seed)
    KT = sum(seg_lens)
    seg_of = [j for j, n in enumerate(seg_lens) for _ in range(n)]
    full = [Bar(1) for _ in range(S)]
    sempty = [Bar(1) for _ in range(S)]
    afull = [Bar(32 * WARPS) for _ in range(NA)]
    aempty = [Bar(1) for _ in range(NA)]
    accum = [Bar(1) for _ in range(2)]
    st = {"slot": [None] * S, "landed": [None] * S, "reads": [0] * KT, "mma_done": [False] * KT,
          "tmem": [None] * NA, "tmem_parts": [set() for _ in range(NA)], "acc": [[] for _ in range(2)],
          "issued": [], "epilogues": 0}
    events = []              # TMA landings, at random later points
    mma_queue = deque()      # MMA completions and commits, in issue order

    def wait(bar, parity):
        while not bar.passed(parity):
            yield

    def producer():
        s = u = 0
        for kt in range(KT):
            if u > 0 and not no_sempty_wait:
                yield from wait(sempty[s], (u - 1) & 1)
            full[s].expect_tx(1)
            full[s].arrive()

            def land(s=s, kt=kt):
                prev = kt - S
                if prev >= 0:
                    assert st["reads"][prev] == WARPS, ("packed tile overwritten before it was read", prev)
                    assert st["mma_done"][prev], ("X tile overwritten while the MMA reads it", prev)
                st["slot"][s] = kt
                full[s].complete_tx(1)
            events.append(land)
            st["issued"].append(kt)
            s, u = (0, u + 1) if s + 1 == S else (s + 1, u)
            yield
        issued = len(st["issued"])
        for kt in range(max(0, issued - S), issued):      # drain the last copies
            yield from wait(full[kt % S], (kt // S) & 1)

    def mma():
        s = b = ub = 0
        for kt in range(KT):
            yield from wait(afull[b], ub & 1)
            assert st["tmem"][b] == kt, ("A buffer holds", st["tmem"][b], "expected", kt)
            assert st["slot"][s] == kt, ("X stage holds", st["slot"][s], "expected", kt)
            j = seg_of[kt]
            if kt == 0 or seg_of[kt - 1] != j:          # a segment's first MMA overwrites
                assert st["acc"][j] == [], "accumulator of a new segment already holds stages"

            def done(kt=kt, b=b, s=s, j=j):
                st["acc"][j].append(kt)
                st["mma_done"][kt] = True
                aempty[b].arrive()
                sempty[s].arrive()
            mma_queue.append(done)
            s = 0 if s + 1 == S else s + 1
            b, ub = (0, ub + 1) if b + 1 == NA else (b + 1, ub)
            if kt + 1 == KT or seg_of[kt + 1] != j:
                mma_queue.append(accum[j].arrive)
            yield

    def dequant(h, q):
        kt, s, u, b, ub = h, h, 0, h, 0
        pend = -1
        while kt < KT:
            yield from wait(full[s], u & 1)
            assert st["slot"][s] == kt, ("packed stage holds", st["slot"][s], "expected", kt)
            st["reads"][kt] += 1
            yield
            if pend >= 0:                               # publish the previous stage
                afull[pend].arrive(32)
                pend = -1
            if kt >= NA:
                parity = (kt // NA) & 1 if wrong_aempty_parity else ((kt // NA) - 1) & 1
                yield from wait(aempty[b], parity)
                assert st["mma_done"][kt - NA], ("A buffer rewritten while the MMA reads it", kt - NA)
            parts = st["tmem_parts"][b]
            parts.add(q)
            if len(parts) == WARPS:
                st["tmem"][b] = kt
                parts.clear()
            pend = b
            kt += NH
            s, u = (s + NH - S, u + 1) if s + NH >= S else (s + NH, u)
            b, ub = (b + NH - NA, ub + 1) if b + NH >= NA else (b + NH, ub)
            yield
        if pend >= 0:
            afull[pend].arrive(32)
        for j in range(len(seg_lens)):
            yield from wait(accum[j], 0)
            lo = sum(seg_lens[:j])
            assert sorted(st["acc"][j]) == list(range(lo, lo + seg_lens[j])), ("segment", j, "incomplete")
        st["epilogues"] += 1

    roles = [producer(), mma()] + [dequant(h, q) for h in range(NH) for q in range(WARPS)]
    steps = 0
    while roles or events or mma_queue:
        order = list(range(len(roles)))
        rnd.shuffle(order)
        finished = set()
        for i in order[: max(1, len(order) // 2)]:
            try:
                next(roles[i])
            except StopIteration:
                finished.add(i)
        roles = [r for i, r in enumerate(roles) if i not in finished]
        if events and rnd.random() < 0.4:
            events.pop(rnd.randrange(len(events)))()
        if mma_queue and rnd.random() < 0.4:
            mma_queue.popleft()()
        steps += 1
        if steps > 20_000:
            raise RuntimeError("no progress: deadlock")
    assert st["epilogues"] == NH * WARPS
    for j in range(len(seg_lens)):
        assert accum[j].phase == 1


CASES = [
    # (segments, S, NA, NH): per-tile schedules (one segment), quartet pairs, stream-K (two segments)
    ((1,), 2, 2, 1), ((5,), 2, 2, 1), ((9,), 3, 3, 1), ((16,), 16, 3, 1), ((7,), 4, 2, 1),
    ((6,), 3, 2, 2), ((9,), 3, 3, 2), ((12,), 5, 3, 2), ((8,), 16, 2, 2),
    ((3, 4), 2, 2, 1), ((7, 2), 3, 3, 1), ((1, 1), 2, 2, 1), ((5, 5), 8, 2, 1), ((2, 9), 4, 3, 1),
]


@pytest.mark.parametrize("segs,S,NA,NH", CASES)
def test_pipeline_protocol_has_no_deadlock_or_aliasing(segs, S, NA, NH):
    for seed in range(3):
        run_pipeline(segs, S, NA, NH, seed)


def test_pipeline_model_catches_planted_mistakes():
    # A ring no deeper than the quartet count: a quartet publishes a stage only
    # when it holds its next one, whose slot the unpublished stage still holds
    # (the host keeps two quartets for rings of three or more stages).
    with pytest.raises(RuntimeError, match="deadlock"):
        run_pipeline((6,), 2, 2, 2, 0)
    # Waiting for the phase of the buffer's current use instead of its previous one
    with pytest.raises((RuntimeError, AssertionError)):
        run_pipeline((8,), 3, 2, 1, 0, wrong_aempty_parity=True)
    # Refilling a stage without waiting for the MMA that reads it
    caught = 0
    for seed in range(6):
        try:
            run_pipeline((10,), 2, 2, 1, seed, no_sempty_wait=True)
        except AssertionError:
            caught += 1
    assert caught > 0
