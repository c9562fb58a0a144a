"""CPU model of the row-streaming GEMV's warp reductions (butterfly_reduce and
group_first_reduce in csrc/wq_gemv_rows.cu). Nothing here needs a GPU.

Each of a warp's 32 lanes holds NV = R x M partial sums (one per batch row and
row of X). The kernel combines them with xor-shuffle halvings that also
transpose: after each exchange a lane keeps half of its values, so at the end
a few lanes hold one total each. The group-first variant runs the halvings
over the low lane bits first; once the LPG lanes of one quantization group
(which share a step and a zero point) are combined, it applies the group's
epilogue (step * (T - offsets - zero * sum x)) to each of the lane's remaining
values, then finishes the sum across groups. The model restates both
functions on a simulated warp and checks every writer lane's total against
the direct sum: for the group-first variant, sum over groups of the group's
affine epilogue applied to the group's total, which is only right if no lanes
of different groups are combined before the epilogue. A planted mistake
(the epilogue applied one halving late) is caught.
"""
import random

import pytest

LANES = 32


def shfl_xor(vals, o):
    return [vals[l ^ o] for l in range(LANES)]


def butterfly_reduce(v, NV):
    """v[lane][i] -> (total per lane, index per lane), as the kernel computes it."""
    v = [list(x) for x in v]
    index = [0] * LANES
    o, c = 16, NV
    while c > 1:
        half = c // 2
        for i in range(half):
            send = [v[l][i] if (l & o) else v[l][i + half] for l in range(LANES)]
            keep = [v[l][i + half] if (l & o) else v[l][i] for l in range(LANES)]
            got = shfl_xor(send, o)
            for l in range(LANES):
                v[l][i] = keep[l] + got[l]
        for l in range(LANES):
            if l & o:
                index[l] += half
        o >>= 1
        c >>= 1
    t = [v[l][0] for l in range(LANES)]
    o = 16 // NV
    while o >= 1:
        got = shfl_xor(t, o)
        t = [t[l] + got[l] for l in range(LANES)]
        o >>= 1
    return t, index


def group_first_index(lane, NV, LPG):
    index, c, o = 0, NV, 1
    while o < LPG:
        if c > 1:
            c //= 2
            if lane & o:
                index += c
        o <<= 1
    return index


def group_first_reduce(v, NV, LPG, epi, late_epilogue=False):
    """epi(lane, i, t): the lane's epilogue of its value index + i."""
    v = [list(x) for x in v]
    index = [0] * LANES
    c = NV
    o = 1
    apply_at = LPG * 2 if late_epilogue else LPG
    while o < 32:
        if o == apply_at:
            for l in range(LANES):
                for i in range(min(c, NV)):
                    v[l][i] = epi(l, i, v[l][i])
        if c > 1:
            half = c // 2
            for i in range(half):
                send = [v[l][i] if (l & o) else v[l][i + half] for l in range(LANES)]
                keep = [v[l][i + half] if (l & o) else v[l][i] for l in range(LANES)]
                got = shfl_xor(send, o)
                for l in range(LANES):
                    v[l][i] = keep[l] + got[l]
            for l in range(LANES):
                if l & o:
                    index[l] += half
            c = half
        else:
            got = shfl_xor([v[l][0] for l in range(LANES)], o)
            for l in range(LANES):
                v[l][0] += got[l]
        o <<= 1
    return [v[l][0] for l in range(LANES)], index


def exact_values(rnd, NV):
    # small integers: every sum is exact, so the model compares totals exactly
    return [[rnd.randint(-50, 50) for _ in range(NV)] for _ in range(LANES)]


@pytest.mark.parametrize("NV", [1, 2, 4, 8, 16, 32])
def test_butterfly_reduce_writers_hold_the_totals(NV):
    rnd = random.Random(NV)
    v = exact_values(rnd, NV)
    t, index = butterfly_reduce(v, NV)
    writers = [l for l in range(LANES) if (l & (LANES // NV - 1)) == 0]
    assert sorted(index[l] for l in writers) == list(range(NV)), "each value written once"
    for l in writers:
        assert t[l] == sum(v[k][index[l]] for k in range(LANES))


@pytest.mark.parametrize("NV", [1, 2, 4, 8, 16, 32])
@pytest.mark.parametrize("LPG", [1, 2, 4])
def test_group_first_reduce_applies_each_groups_epilogue_to_its_own_total(NV, LPG):
    rnd = random.Random(100 * NV + LPG)
    v = exact_values(rnd, NV)
    groups = LANES // LPG
    # per (group, value): an affine epilogue step * (T - offset), integers
    a = [[rnd.choice([1, 2, 3, 5]) for _ in range(NV)] for _ in range(groups)]
    b = [[rnd.randint(-20, 20) for _ in range(NV)] for _ in range(groups)]
    gidx = [group_first_index(l, NV, LPG) for l in range(LANES)]

    def epi(lane, i, t):
        val, g = gidx[lane] + i, lane // LPG
        return a[g][val] * (t - b[g][val])

    t, index = group_first_reduce(v, NV, LPG, epi)
    writers = list(range(NV))                         # lanes < NV write
    assert sorted(index[l] for l in writers) == list(range(NV)), "each value written once"
    for l in range(LANES):  # lanes with the same low log2(NV) bits hold the same total
        assert index[l] == index[l % NV] and t[l] == t[l % NV]
    for l in writers:
        val = index[l]
        want = sum(a[g][val] * (sum(v[k][val] for k in range(g * LPG, (g + 1) * LPG)) - b[g][val])
                   for g in range(groups))
        assert t[l] == want, (NV, LPG, l, val)
    # the step and zero a lane loads (rows lrow0 = gidx / M on) cover the
    # values its epilogue sees: gidx + i for i < max(NV / LPG, 1)
    for l in range(LANES):
        assert gidx[l] + max(NV // LPG, 1) <= NV


def test_group_first_model_catches_an_epilogue_after_groups_mix():
    rnd = random.Random(7)
    NV, LPG = 4, 2
    v = exact_values(rnd, NV)
    groups = LANES // LPG
    a = [[rnd.choice([2, 3, 5]) for _ in range(NV)] for _ in range(groups)]
    gidx = [group_first_index(l, NV, LPG) for l in range(LANES)]

    def epi(lane, i, t):
        return a[lane // LPG][gidx[lane] + i] * t

    t, index = group_first_reduce(v, NV, LPG, epi, late_epilogue=True)
    wrong = 0
    for l in range(NV):
        val = index[l]
        want = sum(a[g][val] * sum(v[k][val] for k in range(g * LPG, (g + 1) * LPG)) for g in range(groups))
        wrong += t[l] != want
    assert wrong > 0
