"""Pins for the CPU oracle: values the pages print, closed forms, invariants and
brute force. Each test would fail on a plausible slip in the oracle (a dropped
term, a wrong sign or index, a transposed operand, the wrong rounding)."""
import json
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle as O

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------------------
# "LLM Quantization: 160GB Model on a Laptop" -- Symmetric Quantization example
# ---------------------------------------------------------------------------

def test_worked_example_symmetric_4bit():
    g = _load("p5_symmetric_worked_example.json")
    v = np.array(g["values"], dtype=np.float16)[None, :]
    codes, steps, zeros = O.quantize_groups(v, g["bits"], len(g["values"]), symmetric=True)
    q = codes.astype(int)[0] - int(zeros[0, 0])
    assert q.tolist() == g["quantized"]
    step = float(steps[0, 0])
    assert abs(step - g["scale_approx"]) < 5e-4
    assert step == 0.127197265625  # smallest fp16 >= 0.8901367/7
    deq = O.dequantize(codes, steps, zeros, len(g["values"]))[0]
    assert np.allclose(deq, g["dequantized_printed"], atol=6e-4)
    rel = np.mean(np.abs(deq - v[0].astype(np.float64)) / np.abs(v[0].astype(np.float64)))
    assert abs(rel - g["average_error_printed"]) < 5e-3


# ---------------------------------------------------------------------------
# "CMU 11-868 L19-L20" -- absmax and zero-point (int8)
# ---------------------------------------------------------------------------

def test_int8_absmax_hand_cases():
    for c in _load("p2_int8_hand_cases.json")["absmax"]:
        q, deq = O.absmax_quantize_int8(np.array(c["X"]))
        assert q.tolist() == c["q"], c["note"]
        mult = 127.0 / np.max(np.abs(c["X"]))
        assert np.allclose(deq, np.array(c["q"]) / mult)


def test_int8_zeropoint_hand_cases():
    for c in _load("p2_int8_hand_cases.json")["zeropoint"]:
        q, deq = O.zeropoint_quantize_int8(np.array(c["X"]))
        assert q.tolist() == c["q"], c["note"]
        if "dequant" in c:
            assert np.allclose(deq, c["dequant"])


def test_asym_8bit_equals_int8_zeropoint_when_step_is_exact():
    """With range 255/256 the step 2^-8 is exact in fp16 and the page's
    multiplier is exactly 256: our unsigned 8-bit codes minus 128 must equal
    the page's int8 codes (including ties, which both round to even)."""
    g = np.random.default_rng(11)
    ks = g.integers(-256, 255, size=126)                 # odd/even halves -> ties
    x = np.concatenate([[-0.5, 127 / 256], ks / 512.0]).astype(np.float16)
    codes, steps, zeros = O.quantize_groups(x[None, :], 8, x.size, symmetric=False)
    assert float(steps[0, 0]) == 2.0 ** -8 and float(zeros[0, 0]) == 128
    q_page, _ = O.zeropoint_quantize_int8(x.astype(np.float64))
    assert (codes[0].astype(int) - 128).tolist() == q_page.astype(int).tolist()


# ---------------------------------------------------------------------------
# "Quantising Large Language Models" -- the group-wise symmetric routine
# ---------------------------------------------------------------------------

def test_symmetric_equals_page_routine_when_step_is_exact():
    """Groups whose max |w| is 7 * 2^-7: the step 2^-7 is exact, so the fp16
    round-up is a no-op and the page's float64 routine must agree exactly."""
    g = np.random.default_rng(3)
    N, K, grp = 4, 512, 128
    w = (g.uniform(-0.05, 0.05, size=(N, K))).astype(np.float16)
    for n in range(N):
        for gi in range(K // grp):
            j = gi * grp + int(g.integers(0, grp))
            w[n, j] = np.float16(7 * 2.0 ** -7) * (1 if (n + gi) % 2 else -1)
    codes, steps, zeros = O.quantize_groups(w, 4, grp, symmetric=True)
    assert np.all(steps == np.float16(2.0 ** -7))
    ours = O.dequantize(codes, steps, zeros, grp)
    # the page's routine: scale = max|w|/qmax, clip(round(w/scale), -qmax-1, qmax) * scale
    wr = w.astype(np.float64).reshape(N, K // grp, grp)
    scale = np.abs(wr).max(axis=2, keepdims=True) / 7
    page = (np.clip(np.round(wr / scale), -8, 7) * scale).reshape(N, K)
    assert np.array_equal(ours, page)


def test_group_size_sweep_error_is_monotone():
    """The page's experiment: a N(0, 0.02) row of 4096 with two 0.8 outliers,
    4-bit symmetric; mean abs error must fall as the group shrinks."""
    g = np.random.default_rng(0)
    row = g.normal(0, 0.02, 4096)
    row[[10, 500]] = 0.8
    w = row.astype(np.float16)[None, :]
    errs = []
    for grp in (4096, 128, 32):
        c, s, z = O.quantize_groups(w, 4, grp, symmetric=True)
        errs.append(np.abs(O.dequantize(c, s, z, grp) - w.astype(np.float64)).mean())
    assert errs[0] > errs[1] > errs[2]


# ---------------------------------------------------------------------------
# fp16 round-up and the asymmetric quantizer
# ---------------------------------------------------------------------------

_F16_ALL = np.arange(1 << 16, dtype=np.uint16).view(np.float16)
_F16_SORTED = np.sort(_F16_ALL[np.isfinite(_F16_ALL)].astype(np.float64))


def test_f16_round_up_brute_force():
    g = np.random.default_rng(5)
    v = np.concatenate([
        g.uniform(0, 1, 3000), 10.0 ** g.uniform(-9, 4.8, 3000),
        _F16_SORTED[_F16_SORTED > 0][:2000],            # exact fp16 values map to themselves
    ]).astype(np.float32)
    got = O.f16_round_up(v).astype(np.float64)
    idx = np.searchsorted(_F16_SORTED, v.astype(np.float64), side="left")
    want = _F16_SORTED[idx]
    assert np.array_equal(got, want)


def _rand_groups(seed, N=64, K=512):
    g = np.random.default_rng(seed)
    w = g.normal(0, 0.02, (N, K))
    w[: N // 4] = np.abs(w[: N // 4]) * -1.0 + 0.004           # skewed negative rows
    w[N // 4: N // 2] *= np.where(g.random((N // 4, K)) < 0.01, 30.0, 1.0)  # outliers
    w[-1, :128] = 0.0                                            # an all-zero group
    w[-2, :128] = 0.01                                           # a constant group
    w[-3, :128] = g.uniform(0.01, 0.03, 128)                     # a group that does not straddle 0
    w[-4, 128:256] = -g.uniform(0.01, 0.03, 128)
    return w.astype(np.float16)


@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("symmetric", [False, True])
def test_quantizer_error_bound_and_code_range(bits, symmetric):
    w = _rand_groups(7)
    codes, steps, zeros = O.quantize_groups(w, bits, 128, symmetric)
    assert codes.max() < (1 << bits)
    z = zeros.astype(np.float64)
    assert np.all((z >= 0) & (z <= (1 << bits) - 1) & (z == np.round(z)))
    deq = O.dequantize(codes, steps, zeros, 128)
    stepk = np.repeat(steps.astype(np.float64), 128, axis=1)
    err = np.abs(deq - w.astype(np.float64))
    assert np.all(err <= stepk * (0.5 + 2.0 ** -20))
    assert np.all(deq[-1, :128] == 0)
    # the all-zero group: step 1 (the reading of [CMU]'s range := 1), its
    # codes at the zero point (0 asymmetric, 2^(b-1) symmetric)
    zp = (1 << (bits - 1)) if symmetric else 0
    assert steps[-1, 0] == 1 and zeros[-1, 0] == zp and np.all(codes[-1, :128] == zp)


@pytest.mark.parametrize("symmetric", [False, True])
def test_step_is_smallest_fp16_at_or_above_quotient(symmetric):
    bits = 4
    w = _rand_groups(8)
    codes, steps, zeros = O.quantize_groups(w, bits, 128, symmetric)
    wg = w.astype(np.float32).reshape(w.shape[0], -1, 128)
    for n in range(0, w.shape[0], 5):
        for gi in range(wg.shape[1]):
            grp = wg[n, gi]
            if symmetric:
                num, den = Fraction(float(np.abs(grp).max())), (1 << (bits - 1)) - 1
            else:
                num = Fraction(float(max(grp.max(), 0))) - Fraction(float(min(grp.min(), 0)))
                den = (1 << bits) - 1
            if num == 0:
                assert float(steps[n, gi]) == 1.0
                continue
            quot = num / den
            s = Fraction(float(steps[n, gi]))
            i = np.searchsorted(_F16_SORTED, float(steps[n, gi]))
            below = Fraction(float(_F16_SORTED[i - 1]))
            slack = Fraction(1, 1 << 23)  # the fp32 quotient and range are rounded
            assert s >= quot * (1 - slack)
            assert below < quot * (1 + slack)


@pytest.mark.parametrize("bits", [3, 4])
def test_codes_are_nearest_with_ties_to_even_brute_force(bits):
    """For the chosen (step, zero), every code is the nearest of all 2^b codes
    to the fp32 quotient w/step; equidistant pairs resolve to an even (q - zero)."""
    g = np.random.default_rng(9)
    w = g.normal(0, 1, (6, 8)).astype(np.float16)
    w[0, :4] = [0.5, -0.5, 1.5, 2.5]                             # exact ties at step 1
    w[0, 4:] = [0.0, 0.0, 0.0, 0.0]
    codes, steps, zeros = O.quantize_groups(w, bits, 8, symmetric=False)
    Q = (1 << bits) - 1
    for n in range(w.shape[0]):
        for gi in range(w.shape[1] // 8):
            sf = np.float32(steps[n, gi])
            z = int(zeros[n, gi])
            for j in range(8):
                k = gi * 8 + j
                quot = float(np.float32(w[n, k]) / sf)
                best = None
                for c in range(Q + 1):
                    d = abs(quot - (c - z))
                    key = (d, (c - z) % 2)
                    if best is None or key < best[0]:
                        best = (key, c)
                assert codes[n, k] == best[1], (n, k, quot, z)


def test_asymmetric_beats_symmetric_on_skewed_groups():
    """"LLM Quantization: 160GB Model on a Laptop", Asymmetric Quantization:
    handling min and max separately lowers the error on skewed data."""
    g = np.random.default_rng(10)
    w = (-np.abs(g.normal(0, 0.02, (32, 1024))) + 0.002).astype(np.float16)
    e = {}
    for sym in (False, True):
        c, s, z = O.quantize_groups(w, 4, 128, sym)
        e[sym] = np.abs(O.dequantize(c, s, z, 128) - w.astype(np.float64)).mean()
    assert e[False] < 0.75 * e[True]


# ---------------------------------------------------------------------------
# Packed layouts
# ---------------------------------------------------------------------------

def test_pack4_hand_words():
    codes = np.array([list(range(8)), list(range(8, 16))], dtype=np.uint8)
    words = O.pack_codes(codes, 4)
    # slot order [k0, k2, k4, k6, k1, k3, k5, k7] from nibble 0 upward
    assert words[0, 0] == 0x75316420
    assert words[1, 0] == 0xFDB9ECA8


def test_pack3_hand_words():
    codes = (np.arange(32) % 8).astype(np.uint8)[None, :]
    words = O.pack_codes(codes, 3)
    # word 0: k0..k9 = 0,1,2,3,4,5,6,7,0,1 in pairs (low field, high field);
    # k30 = 6 (bit 0 = 0), k31 = 7 (bit 0 = 1) -> bit 15 clear, bit 31 set.
    w0 = (0 << 0) | (2 << 3) | (4 << 6) | (6 << 9) | (0 << 12) \
        | (1 << 16) | (3 << 19) | (5 << 22) | (7 << 25) | (1 << 28) | (1 << 31)
    assert w0 == 0x9F590D10
    assert words[0, 0] == w0
    # word 2: k20..k29 = 4,5,6,7,0,1,2,3,4,5; bit 2 of k30 (=1) and of k31 (=1)
    w2 = (4 << 0) | (6 << 3) | (0 << 6) | (2 << 9) | (4 << 12) \
        | (5 << 16) | (7 << 19) | (1 << 22) | (3 << 25) | (5 << 28) | (1 << 15) | (1 << 31)
    assert words[0, 2] == w2


@pytest.mark.parametrize("bits", [3, 4])
def test_pack_roundtrip(bits):
    g = np.random.default_rng(12)
    codes = g.integers(0, 1 << bits, size=(17, 256)).astype(np.uint8)
    words = O.pack_codes(codes, bits)
    assert words.shape == (17, O.packed_words_per_row(256, bits))
    assert np.array_equal(O.unpack_codes(words, bits, 256), codes)


# ---------------------------------------------------------------------------
# Matmul reference
# ---------------------------------------------------------------------------

def test_gemm_ref_closed_forms():
    N, K, M = 5, 256, 3
    g = np.random.default_rng(13)
    X = g.normal(0, 1, (M, K)).astype(np.float16)
    steps = g.uniform(0.001, 0.1, (N, K // 128)).astype(np.float16)
    zeros = g.integers(0, 16, (N, K // 128)).astype(np.float16)
    codes = np.repeat(zeros.astype(np.uint8), 128, axis=1)       # every code == zero
    assert np.all(O.gemm_ref(X, codes, steps, zeros, 128) == 0)
    n, k, q = 3, 200, 15
    codes[n, k] = q
    Y = O.gemm_ref(X, codes, steps, zeros, 128)
    expect = X[:, k].astype(np.float64) * (q - float(zeros[n, k // 128])) * float(steps[n, k // 128])
    assert np.allclose(Y[:, n], expect, rtol=1e-15, atol=0)
    assert np.all(np.delete(Y, n, axis=1) == 0)


def test_gemm_ref_brute_force_loops():
    g = np.random.default_rng(14)
    M, N, K, grp = 2, 3, 64, 32
    X = g.normal(0, 1, (M, K)).astype(np.float16)
    codes = g.integers(0, 16, (N, K)).astype(np.uint8)
    steps = g.uniform(0.001, 0.1, (N, K // grp)).astype(np.float16)
    zeros = g.integers(0, 16, (N, K // grp)).astype(np.float16)
    Y = O.gemm_ref(X, codes, steps, zeros, grp)
    for m in range(M):
        for n in range(N):
            acc = Fraction(0)
            for k in range(K):
                acc += Fraction(float(X[m, k])) * (int(codes[n, k]) - Fraction(float(zeros[n, k // grp]))) \
                    * Fraction(float(steps[n, k // grp]))
            assert abs(Y[m, n] - float(acc)) <= 1e-13 * max(1.0, abs(float(acc)))


# ---------------------------------------------------------------------------
# AWQ pieces
# ---------------------------------------------------------------------------

def test_smoothquant_identity_fp64():
    """"Quantising Large Language Models", outlier features: Y = (X diag(s)^-1)(diag(s) W)."""
    g = np.random.default_rng(15)
    X = g.normal(0, 1, (16, 256))
    W = g.normal(0, 0.02, (64, 256))
    s = np.exp(g.normal(0, 1, 256))
    Y = X @ W.T
    Y2 = (X / s[None, :]) @ (W * s[None, :]).T
    assert np.max(np.abs(Y - Y2)) <= 1e-13 * np.max(np.abs(Y))


def test_absmean_exact_and_order_independent():
    g = np.random.default_rng(16)
    X = (g.normal(0, 1, (48, 16)) * np.where(g.random(16) < 0.2, 20, 1)).astype(np.float16)
    mu = O.activation_absmean(X)
    perm = g.permutation(48)
    assert np.array_equal(mu, O.activation_absmean(X[perm]))
    for k in range(16):
        exact = sum(Fraction(abs(float(v))) for v in X[:, k]) / 48
        assert mu[k] == float(exact)


def test_awq_candidates_endpoints():
    mu = np.array([0.0, 1e-9, 0.3, 1.0, 7.25, 300.0])
    S = O.awq_candidates(mu, O.awq_alpha_grid(20))
    assert np.all(S[0] == 1.0)                                    # alpha = 0
    assert O.awq_alpha_grid(20)[10] == 0.5
    assert np.array_equal(S[10], np.sqrt(np.maximum(mu, 2.0 ** -14)).astype(np.float16))
    assert np.all(S > 0)


def test_awq_alpha0_is_plain_rtn():
    g = np.random.default_rng(17)
    W = g.normal(0, 0.02, (32, 256)).astype(np.float16)
    E = O.awq_error_matrix(W, np.ones(256, np.float16), 4, 128, False)
    c, s, z = O.quantize_groups(W, 4, 128, False)
    assert np.array_equal(E, W.astype(np.float64) - O.dequantize(c, s, z, 128))


def test_awq_loss_brute_force_loops():
    g = np.random.default_rng(18)
    T, K, grp = 3, 16, 8
    X = g.normal(0, 1, (T, K)).astype(np.float16)
    Ws = [g.normal(0, 0.1, (2, K)).astype(np.float16), g.normal(0, 0.1, (1, K)).astype(np.float16)]
    s = np.exp(g.normal(0, 0.5, K)).astype(np.float16)
    L = O.awq_loss(X, Ws, s, 4, grp, False)
    total = 0.0
    for W in Ws:
        c, st, z = O.quantize_groups(W, 4, grp, False, s16=s)
        for t in range(T):
            for n in range(W.shape[0]):
                d = 0.0
                for k in range(K):
                    deq = (int(c[n, k]) - float(z[n, k // grp])) * float(st[n, k // grp])
                    d += float(X[t, k]) * (float(W[n, k]) - deq / float(s[k]))
                total += d * d
    assert abs(L - total) <= 1e-12 * total


def test_salient_channel_error_shrinks_with_scale():
    """"MIT 6.5940 Lab 4 + Lab 5", Question 2: scaling one channel by s while the
    group max is unchanged shrinks that channel's error by about s."""
    g = np.random.default_rng(19)
    errs = {1.0: [], 2.0: []}
    for _ in range(400):
        w = g.normal(0, 0.02, 128)
        w[0] = 0.1                                                # keeps the group max fixed
        w = w.astype(np.float16)
        for sc in (1.0, 2.0):
            s = np.ones(128, np.float16)
            s[5] = sc                                             # w[5] * 2 stays below w[0]
            if abs(float(w[5])) * sc >= 0.1:
                continue
            E = O.awq_error_matrix(w[None, :], s, 3, 128, True)
            errs[sc].append(abs(E[0, 5]))
    ratio = np.mean(errs[2.0]) / np.mean(errs[1.0])
    assert 0.35 < ratio < 0.65


def test_awq_search_picks_minimum_and_beats_rtn():
    import synth
    g = synth.rng(20)
    X = synth.activations(g, 64, 256, channel_frac=0.02, channel_mult=20.0)
    Ws = [synth.weight(g, 48, 256, 0.02), synth.weight(g, 16, 256, 0.02)]
    r = O.awq_search(X, Ws, 4, 128, False)
    assert r["best"] == int(np.argmin(r["losses"]))
    assert r["losses"][r["best"]] <= r["losses"][0]
    assert r["losses"][r["best"]] < 0.9 * r["losses"][0]          # outlier channels make AWQ pay
    assert np.array_equal(r["s"], r["candidates"][r["best"]])
    # the loss at the chosen alpha is what awq_loss reports for that scale
    assert r["losses"][r["best"]] == O.awq_loss(X, Ws, r["s"], 4, 128, False)


def test_awq_loss_falls_then_rises_over_alpha():
    """Too large a scale inflates the group maximum, so the loss over alpha
    falls and then rises ("MIT 6.5940 Lab 4 + Lab 5", "How to self-study it":
    the turning point of the scale sweep): with a few outlier input channels
    the best alpha is interior and the largest alpha loses to alpha = 0."""
    g = np.random.default_rng(3)
    K, N, T = 256, 64, 64
    X = g.normal(0, 1, (T, K))
    X[:, g.choice(K, 3, replace=False)] *= 20
    W = g.normal(0, 0.02, (N, K))
    r = O.awq_search(X.astype(np.float16), [W.astype(np.float16)], 4, 128, False)
    L, best = r["losses"], r["best"]
    assert 0 < best < len(L) - 1
    assert L[0] > 1.5 * L[best] and L[-1] > 3.0 * L[best] and L[-1] > L[0]
    assert np.all(np.diff(L[best:]) > 0)      # rises steadily past the turning point


# ---------------------------------------------------------------------------
# AWQ scale folding ("MIT 6.5940 Lab 4 + Lab 5", "Question 2")
# ---------------------------------------------------------------------------


def _block_params(g, D=64, H=96):
    return {"gamma1": 1.0 + 0.1 * g.standard_normal(D), "wq": g.normal(0, 0.1, (D, D)),
            "wk": g.normal(0, 0.1, (D, D)), "wv": g.normal(0, 0.1, (D, D)), "wo": g.normal(0, 0.1, (D, D)),
            "gamma2": 1.0 + 0.1 * g.standard_normal(D), "wg": g.normal(0, 0.1, (H, D)),
            "wu": g.normal(0, 0.1, (H, D)), "wd": g.normal(0, 0.1, (D, H))}


def test_decoder_block_ref_closed_forms():
    """Residual paths only when o and down are zero; one token attends to itself
    (softmax over one key is 1), so its attention output is v."""
    g = np.random.default_rng(31)
    p = _block_params(g)
    x = g.normal(0, 1, (5, 64))
    z = dict(p, wo=np.zeros((64, 64)), wd=np.zeros((64, 96)))
    assert np.array_equal(O.decoder_block_ref(x, z, 4), x)
    x1 = x[:1]
    h = x1 / np.sqrt(np.mean(x1 * x1) + 1e-6) * p["gamma1"]
    y_attn_only = x1 + (h @ p["wv"].T) @ p["wo"].T
    q = dict(p, wd=np.zeros((64, 96)))
    assert np.allclose(O.decoder_block_ref(x1, q, 4), y_attn_only, rtol=1e-13, atol=1e-13)


def test_fold_block_equivalence_fp64():
    """Folding the four places' s^-1 into gamma1, v_proj's rows, gamma2 and
    up_proj's rows while the scaled linears take W diag(s) leaves the block's
    output unchanged (fp64: to rounding)."""
    g = np.random.default_rng(32)
    p = _block_params(g)
    x = g.normal(0, 1, (7, 64))
    s = [np.exp(g.normal(0, 1, n)) for n in (64, 64, 64, 96)]
    y = O.decoder_block_ref(x, p, 4)
    yf = O.decoder_block_ref(x, O.awq_fold_block(p, *s), 4)
    assert np.max(np.abs(yf - y)) <= 1e-12 * np.max(np.abs(y))
    # the check discriminates: the o_proj scale folded into v_proj's input
    # columns instead of its output rows, or a place left unfolded, changes y
    bad = O.awq_fold_block(p, *s)
    bad["wv"] = p["wv"] * s[0][None, :] / s[1][None, :]
    assert np.max(np.abs(O.decoder_block_ref(x, bad, 4) - y)) > 1e-3 * np.max(np.abs(y))
    bad = O.awq_fold_block(p, *s)
    bad["gamma2"] = p["gamma2"]
    assert np.max(np.abs(O.decoder_block_ref(x, bad, 4) - y)) > 1e-3 * np.max(np.abs(y))


def _fp16_half_ulp(v):
    """Half the fp16 spacing at |v| (normal range)."""
    e = np.floor(np.log2(np.abs(v)))
    return 2.0 ** (np.maximum(e, -14) - 10) / 2


def test_fold_fp16_within_half_ulp_of_exact_quotient():
    """Stored fold results lie within fp16 rounding (plus one fp32 rounding) of
    the exact quotient, per element and along the right axis."""
    g = np.random.default_rng(33)
    gam = (1.0 + 0.2 * g.standard_normal(300)).astype(np.float16)
    s = np.exp(g.normal(0, 1.5, 300)).astype(np.float16)
    out = O.awq_fold_into_norm(gam, s)
    for a, b, o in zip(gam.astype(float), s.astype(float), out.astype(float)):
        exact = Fraction(a) / Fraction(b)
        assert abs(Fraction(o) - exact) <= Fraction(_fp16_half_ulp(float(exact))) * (1 + Fraction(1, 2 ** 12))
    W = g.normal(0, 0.05, (5, 7)).astype(np.float16)
    sr = np.exp(g.normal(0, 1, 5)).astype(np.float16)
    b = g.normal(0, 0.05, 5).astype(np.float16)
    Wf, bf = O.awq_fold_into_linear_rows(W, sr, b)
    for n in range(5):
        for k in range(7):
            exact = Fraction(float(W[n, k])) / Fraction(float(sr[n]))
            assert abs(Fraction(float(Wf[n, k])) - exact) <= \
                Fraction(_fp16_half_ulp(float(exact))) * (1 + Fraction(1, 2 ** 12))
        exact = Fraction(float(b[n])) / Fraction(float(sr[n]))
        assert abs(Fraction(float(bf[n])) - exact) <= Fraction(_fp16_half_ulp(float(exact))) * (1 + Fraction(1, 2 ** 12))


def test_fold_fp16_is_the_correctly_rounded_quotient_exhaustive():
    """The stored fold fp16_rn(fp32_rn(gamma / s)) is the correctly rounded
    fp16 quotient for every positive finite fp16 dividend and every fp16
    divisor in [1, 2) (other divisors differ by a power of two). Reference:
    the fp64 quotient rounded to fp16, which is correctly rounded because a
    quotient of two fp16 values lies about 2^-23 (relative) or more from any
    fp16 rounding midpoint, far beyond fp64's rounding error; a sample of
    it is checked against exact fractions."""
    allw = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16)
    s = (np.arange(1024, 2048) / 1024).astype(np.float16)
    for k in range(0, len(allw), 4096):
        w = allw[k:k + 4096]
        Wv, Sv = np.repeat(w, len(s)), np.tile(s, len(w))
        got = O.awq_fold_into_norm(Wv, Sv)
        want = (Wv.astype(np.float64) / Sv.astype(np.float64)).astype(np.float16)
        assert np.array_equal(got.view(np.uint16), want.view(np.uint16))
    rng = np.random.default_rng(5)
    for _ in range(300):
        w, sv = allw[rng.integers(len(allw))], s[rng.integers(len(s))]
        exact = Fraction(float(w)) / Fraction(float(sv))
        r = np.float16(np.float64(w) / np.float64(sv))
        for nb in (np.nextafter(r, np.float16(np.inf)), np.nextafter(r, np.float16(0))):
            assert abs(Fraction(float(r)) - exact) <= abs(Fraction(float(nb)) - exact)


def test_fold_linear_rows_with_bias_restores_the_consumers_input_fp64():
    """A linear y = x W^T + b whose output rows absorb diag(s)^-1 feeds a
    consumer that now reads y' diag(s): y' * s must equal y (fp64, to
    rounding), bias included; leaving the bias unfolded breaks it."""
    g = np.random.default_rng(34)
    W, b = g.normal(0, 0.1, (24, 40)), g.normal(0, 0.5, 24)
    sv = np.exp(g.normal(0, 1, 24))
    x = g.normal(0, 1, (9, 40))
    y = x @ W.T + b
    Wf, bf = O.awq_fold_into_linear_rows(W, sv, b)
    assert np.max(np.abs((x @ Wf.T + bf) * sv[None, :] - y)) <= 1e-13 * np.max(np.abs(y))
    assert np.max(np.abs((x @ Wf.T + b) * sv[None, :] - y)) > 1e-2 * np.max(np.abs(y))


def test_fold_fp16_hand_values():
    """Hand-derived stored values: quotients exact in fp16 stay exact, and
    1/3 and 1/7 round to the nearest fp16 (spacing 2^-12 on [0.25, 0.5),
    2^-13 on [0.125, 0.25)). A quotient of two fp16 values is never itself
    an fp16 rounding midpoint (it would need 12 significant bits while the
    dividend has 11), so only the fp32 step can create a tie."""
    gam = np.array([1.0 + 2.0 ** -10, 1.0 + 3 * 2.0 ** -10, 3.0], dtype=np.float16)
    s = np.array([2.0, 2.0, 2.0], dtype=np.float16)
    out = O.awq_fold_into_norm(gam, s).astype(np.float64)
    # (1 + 2^-10)/2 = 0.5 + 2^-11 is representable (fp16 spacing at 0.5 is 2^-11)
    assert out[0] == 0.5 + 2.0 ** -11 and out[1] == 0.5 + 3 * 2.0 ** -11 and out[2] == 1.5
    gam = np.array([1.0, 1.0], dtype=np.float16)
    s = np.array([3.0, 7.0], dtype=np.float16)
    out = O.awq_fold_into_norm(gam, s).astype(np.float64)
    assert out[0] == 0.333251953125 and out[1] == 0.142822265625


# ---------------------------------------------------------------------------
# GPTQ ("CMU 11-868 L19-L20 Model Quantization", "The algorithm in four
# steps" and "Why it can actually run: from OBS to GPTQ")
# ---------------------------------------------------------------------------

def _obs_sequential(W16, X16, bits, group, sym, damp=0.01):
    """Optimal Brain Surgeon in its original form: quantize the columns in
    order; after each, move the remaining weights by the closed-form optimal
    compensation -err / [H_F^-1]_qq * [H_F^-1]_q,: and remove the quantized
    column from the inverse Hessian by the rank-one downdate. No Cholesky
    factor, no blocks."""
    W = W16.astype(np.float64).copy()
    X = X16.astype(np.float64)
    N, K = W.shape
    H = 2.0 * X.T @ X
    H += damp * np.mean(np.diag(H)) * np.eye(K)
    Hinv = np.linalg.inv(H)
    codes = np.zeros((N, K), np.uint8)
    st = np.zeros((N, K // group), np.float16)
    zr = np.zeros((N, K // group), np.float16)
    for i in range(K):
        if i % group == 0:
            _, s, z = O.quantize_groups_f32(W[:, i:i + group].astype(np.float32), bits, group, sym)
            st[:, i // group], zr[:, i // group] = s[:, 0], z[:, 0]
        sf = st[:, i // group].astype(np.float32)
        if sym:
            qmax = (1 << (bits - 1)) - 1
            q = np.clip(np.rint(W[:, i].astype(np.float32) / sf), -qmax - 1, qmax).astype(np.int32) + (1 << (bits - 1))
        else:
            q = np.clip(np.rint(W[:, i].astype(np.float32) / sf).astype(np.int32) + zr[:, i // group].astype(np.int32),
                        0, (1 << bits) - 1)
        codes[:, i] = q
        deq = (q - zr[:, i // group].astype(np.float64)) * st[:, i // group].astype(np.float64)
        d = Hinv[i, i]
        W[:, i + 1:] -= np.outer((W[:, i] - deq) / d, Hinv[i, i + 1:])
        Hinv = Hinv - np.outer(Hinv[:, i], Hinv[i, :]) / d
    return codes, st, zr


@pytest.mark.parametrize("block", [1, 4, 32, 64])
@pytest.mark.parametrize("sym", [False, True])
def test_gptq_equals_obs_sequential(block, sym):
    """The Cholesky reformulation and the lazy batch updates change the order
    of computation, not the result: codes, steps and zeros equal the
    sequential OBS procedure on small problems (4-bit, groups of 32)."""
    g = np.random.default_rng(61 + block)
    N, K, T = 12, 64, 40
    W = (0.02 * g.standard_normal((N, K))).astype(np.float16)
    base = g.standard_normal((T, 8))
    X = (base @ g.standard_normal((8, K)) + 0.3 * g.standard_normal((T, K))).astype(np.float16)  # correlated
    ref = _obs_sequential(W, X, 4, 32, sym)
    got = O.gptq_quantize(W, X, 4, 32, sym, block=block)
    for a, b in zip(got, ref):
        assert np.array_equal(a.view(np.uint8) if a.dtype == np.uint8 else a.view(np.uint16),
                              b.view(np.uint8) if b.dtype == np.uint8 else b.view(np.uint16))


def test_gptq_with_uncorrelated_inputs_is_rtn():
    """With orthogonal input channels H is diagonal, so is G: no error is
    passed on and GPTQ gives exactly the round-to-nearest codes."""
    g = np.random.default_rng(62)
    K, N = 128, 16
    X = np.zeros((K, K), np.float16)
    X[np.arange(K), np.arange(K)] = (1.0 + g.random(K)).astype(np.float16)  # exactly orthogonal
    W = (0.02 * g.standard_normal((N, K))).astype(np.float16)
    for bits, sym in ((4, False), (3, True)):
        got = O.gptq_quantize(W, X, bits, 128, sym)
        ref = O.quantize_groups(W, bits, 128, sym)
        assert np.array_equal(got[0], ref[0])
        assert np.array_equal(got[1].view(np.uint16), ref[1].view(np.uint16))


def test_gptq_hessian_damping_and_dead_channels():
    """H = 2 X^T X + lambda I, lambda = 1 % of the mean diagonal; a channel
    that is zero on every token gets H_kk = 1 before the damping and its
    weights quantize as zeros."""
    X = np.array([[1.0, 0.0, 2.0], [3.0, 0.0, -1.0]], np.float16)
    H, dead = O.gptq_hessian(X)
    base = np.array([[20.0, 0.0, -2.0], [0.0, 1.0, 0.0], [-2.0, 0.0, 10.0]])
    lam = 0.01 * (20.0 + 1.0 + 10.0) / 3
    assert np.array_equal(dead, [False, True, False])
    assert np.allclose(H, base + lam * np.eye(3), rtol=0, atol=1e-15)
    g = np.random.default_rng(63)
    Xc = (g.standard_normal((20, 128))).astype(np.float16)
    Xc[:, 7] = 0
    W = (0.02 * g.standard_normal((4, 128))).astype(np.float16)
    codes, st, z = O.gptq_quantize(W, Xc, 4, 128, False)
    assert np.all(O.dequantize(codes, st, z, 128)[:, 7] == 0.0)


def test_gptq_beats_rtn_on_correlated_inputs():
    """The layer-wise objective ||W X - W^ X||^2 ("CMU 11-868 L19-L20",
    "Two core moves") is lower after GPTQ than after round to nearest."""
    g = np.random.default_rng(64)
    N, K, T = 64, 256, 128
    W = (0.02 * g.standard_normal((N, K))).astype(np.float16)
    X = (g.standard_normal((T, 16)) @ g.standard_normal((16, K)) + 0.2 * g.standard_normal((T, K))).astype(np.float16)

    def loss(c, s, z):
        E = W.astype(np.float64) - O.dequantize(c, s, z, 128)
        return float(np.sum((X.astype(np.float64) @ E.T) ** 2))

    for bits in (3, 4):
        assert loss(*O.gptq_quantize(W, X, bits, 128, False)) < 0.8 * loss(*O.quantize_groups(W, bits, 128, False))


# ---------------------------------------------------------------------------
# W4A8 ("MIT 6.5940 Lab 4 + Lab 5", W4A8 with group size 32; int8 absmax of
# "CMU 11-868 L19-L20", "absmax and zero-point")
# ---------------------------------------------------------------------------

def test_act_int8_groups_hand_values_and_bounds():
    """The group's largest magnitude maps to +-127; ties round to even; an
    all-zero group keeps multiplier 1; every value is within half a code step
    of its dequantized code."""
    x = np.zeros((1, 64), np.float16)
    x[0, :4] = [2.0, -1.0, 0.5, 1.0 / 127.0 * 2.0]      # mult = 63.5: 127, -63.5 -> -64 (even), 31.75 -> 32
    q, m = O.act_quantize_int8_groups(x, 32)
    assert m[0, 0] == np.float32(63.5) and m[0, 1] == 1.0
    assert list(q[0, :3]) == [127, -64, 32]
    assert np.all(q[0, 32:] == 0)
    g = np.random.default_rng(71)
    X = (g.standard_normal((5, 256)) * np.exp(g.normal(0, 2, 256))).astype(np.float16)
    q, m = O.act_quantize_int8_groups(X, 32)
    back = q.astype(np.float64).reshape(5, 8, 32) / m.astype(np.float64)[:, :, None]
    err = np.abs(back - X.astype(np.float64).reshape(5, 8, 32))
    assert np.all(err <= (0.5 + 1e-6) / m.astype(np.float64)[:, :, None])
    assert np.all(np.abs(q.reshape(5, 8, 32)).max(axis=2) == 127)


def test_w4a8_ref_reduces_to_the_exact_matmul():
    """With activations that are integers of magnitude <= 127 and a group
    maximum of 127 (multiplier 1), quantizing them changes nothing, and the
    W4A8 reference equals the fp64 matmul of the dequantized weight; the
    integer group sums keep every product exact."""
    g = np.random.default_rng(72)
    K, N, M = 128, 20, 3
    X = g.integers(-127, 128, (M, K)).astype(np.float16)
    X[:, ::32] = 127
    codes, st, z = O.quantize_groups((0.02 * g.standard_normal((N, K))).astype(np.float16), 4, 32, False)
    qx, mult = O.act_quantize_int8_groups(X, 32)
    assert np.all(mult == 1.0) and np.array_equal(qx.astype(np.float16), X)
    assert np.allclose(O.w4a8_gemm_ref(qx, mult, codes, st, z, 32), O.gemm_ref(X, codes, st, z, 32),
                       rtol=1e-14, atol=1e-12)


def test_w4a8_ref_brute_force_loops():
    g = np.random.default_rng(73)
    K, N, M = 64, 3, 2
    codes, st, z = O.quantize_groups((0.02 * g.standard_normal((N, K))).astype(np.float16), 4, 32, True)
    qx, mult = O.act_quantize_int8_groups((g.standard_normal((M, K))).astype(np.float16), 32)
    Y = O.w4a8_gemm_ref(qx, mult, codes, st, z, 32)
    for m in range(M):
        for n in range(N):
            t = Fraction(0)
            for gi in range(2):
                dot = sum((int(codes[n, k]) - int(z[n, gi])) * int(qx[m, k]) for k in range(32 * gi, 32 * gi + 32))
                t += Fraction(dot) * Fraction(float(st[n, gi])) / Fraction(float(mult[m, gi]))
            assert abs(float(t) - Y[m, n]) <= 1e-12 * max(1.0, abs(float(t)))
