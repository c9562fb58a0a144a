"""Arithmetic checks (CPU; exact rational numbers where rounding decides) of
the arguments the CUDA path relies on, independent of any CUDA code:

* the quotient w / step is formed without a division as
  q0 = RN(w y), r = w - step q0, q = RN(q0 + r y) (Markstein's correction),
  with y any fp32 number within one ulp of 1/step (the kernel's reciprocal is
  closer than that); for an fp16 step (11 significant bits) and the small
  integer divisors 3, 7, 15, q must equal RN(w / step) exactly, r must be
  representable in fp32, and the cases include exact ties and near-ties;
* rint by adding 1.5 * 2^23 rounds to nearest with ties to even for |x| < 2^22;
* the dequantized value (level - zero) * step is one exact fma of the offset
  level with the step and the constant -(1.5 * 2^23) * step;
* GPTQ's factor Cholesky(H^-1)^T is the inverse of the "UL" factor of H,
  the route the GPU takes without forming H^-1 (fp64).
"""
import random
from fractions import Fraction as F

import numpy as np
import pytest


def rn32(x: F) -> F:
    """Round a rational to the nearest fp32 value, ties to even (normal range)."""
    if x == 0:
        return F(0)
    sign = 1 if x > 0 else -1
    a = abs(x)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    while F(2) ** e > a:
        e -= 1
    while F(2) ** (e + 1) <= a:
        e += 1
    ulp = F(2) ** (max(e, -126) - 23)
    q = a / ulp
    fl = q.numerator // q.denominator
    rem = q - fl
    if rem > F(1, 2) or (rem == F(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * fl * ulp


def neighbours_of(x: F):
    """The fp32 numbers that bracket x (both equal when x is representable)."""
    y = rn32(x)
    f = np.float32(float(y))
    up = F(float(np.nextafter(f, np.float32(np.inf))))
    dn = F(float(np.nextafter(f, np.float32(-np.inf))))
    if y == x:
        return [y]
    return [y, up if y < x else dn]


def corrected_quotient_ok(w: float, b: float) -> bool:
    w, b = F(w), F(b)
    for y in neighbours_of(1 / b):
        q0 = rn32(w * y)
        r = w - b * q0
        if rn32(r) != r:
            return False
        if rn32(q0 + r * y) != rn32(w / b):
            return False
    return True


def _fp16_positive():
    v = np.arange(1, 0x7C00, dtype=np.uint16).view(np.float16).astype(np.float64)
    return v[v > 0]


@pytest.mark.filterwarnings("ignore:overflow encountered")
def test_corrected_quotient_fp16_steps():
    rng = random.Random(11)
    steps = _fp16_positive()
    n = 0
    for i in range(3000):
        b = float(rng.choice(steps))
        kind = i % 3
        if kind == 0:    # an fp16 weight, |w / step| < 16
            w = float(np.float16(rng.uniform(-15.9, 15.9) * b))
        elif kind == 1:  # an AWQ-scaled weight: fp16 x fp16, exact in fp32
            w = float(np.float32(np.float16(rng.uniform(-4, 4) * b)) * np.float32(np.float16(rng.uniform(0.25, 4))))
        else:            # a tie or a near-tie of a half-integer multiple of the step
            k = rng.randint(-15, 14)
            w = float(np.float32((k + 0.5) * b * (1 + rng.choice([0.0, 2.0 ** -23, -2.0 ** -23]))))
        if not np.isfinite(w) or w == 0 or abs(w / b) >= 16:
            continue
        n += 1
        assert corrected_quotient_ok(w, b), (w, b)
    assert n > 2500


@pytest.mark.parametrize("d", [3, 7, 15])
def test_corrected_quotient_small_divisors(d):
    rng = random.Random(d)
    for _ in range(800):
        a = float(np.float32(rng.uniform(0, 1) * 2.0 ** rng.randint(-40, 15)))
        if a == 0:
            continue
        assert corrected_quotient_ok(a, d), a


def test_round_by_magic_addition():
    magic = F(12582912)  # 1.5 * 2^23
    rng = random.Random(3)
    xs = [F(k, 2) for k in range(-64, 65)]  # every half-integer tie in range
    xs += [F(float(np.float32(rng.uniform(-1e4, 1e4)))) for _ in range(2000)]
    for x in xs:
        got = rn32(x + magic) - magic
        fl = x.numerator // x.denominator
        rem = x - fl
        want = fl + (1 if rem > F(1, 2) or (rem == F(1, 2) and fl % 2 == 1) else 0)
        assert got == want, x


def _bits(v: float) -> int:
    return int(np.array([v], dtype=np.float32).view(np.uint32)[0])


@pytest.mark.parametrize("bits", [3, 4])
def test_offset_level_packing_identity(bits):
    """The packer adds the bit patterns of the offset levels 1.5*2^23 + (l - z),
    each shifted to its field, and subtracts one constant per word:
    sum_j (magic_bits << s_j) - z * sum_j (1 << s_j) (mod 2^32). Since the
    levels l in [0, 2^b - 1] fill disjoint fields, the result must be the
    packed word for every zero point z and every level pattern."""
    magic, mbits = 12582912.0, 0x4B400000
    rng = np.random.default_rng(bits)
    if bits == 4:
        shifts = [4 * (4 + (i >> 1) if i & 1 else i >> 1) for i in range(8)]  # slots [0,2,4,6,1,3,5,7]
    else:
        shifts = [3 * (i // 2) + (16 if i & 1 else 0) for i in range(10)]     # pairs at 3j and 16 + 3j
    G = sum((mbits << s) & 0xFFFFFFFF for s in shifts) & 0xFFFFFFFF
    U = sum(1 << s for s in shifts) & 0xFFFFFFFF
    Q = (1 << bits) - 1
    for z in range(Q + 1):
        for _ in range(200):
            lv = rng.integers(0, Q + 1, len(shifts))
            acc = 0
            for l, s in zip(lv, shifts):
                acc = (acc + (_bits(magic + float(l) - float(z)) << s)) & 0xFFFFFFFF
            word = (acc - ((G - z * U) & 0xFFFFFFFF)) & 0xFFFFFFFF
            want = 0
            for l, s in zip(lv, shifts):
                want |= int(l) << s
            assert word == want, (z, lv)


def test_dequant_as_one_fma_is_exact():
    """The AWQ error pass forms deq = (level - zero) * step as one fma,
    fma(1.5 * 2^23 + level - zero, step, -(1.5 * 2^23) * step): for every
    finite fp16 step and every offset level - zero in [-15, 15] the constant
    -(1.5 * 2^23) * step is an fp32 number, and the fma's single rounding of
    the exact value returns exactly (level - zero) * step."""
    magic = 12582912.0
    steps = _fp16_positive()
    offs = np.arange(-15, 16, dtype=np.float64)
    c = -magic * steps                                   # the fp32 constant
    assert np.all(c.astype(np.float32).astype(np.float64) == c)
    lv = magic + offs[:, None]                           # the offset level, an fp32 number
    assert np.all(lv.astype(np.float32).astype(np.float64) == lv)
    # lv * step has at most 24 + 11 significant bits, so the fp64 sum below is
    # the fma's exact value; one rounding to fp32 is the fma's result.
    exact = lv * steps[None, :] + c[None, :]
    fused = exact.astype(np.float32).astype(np.float64)
    want = offs[:, None] * steps[None, :]
    assert np.array_equal(fused, want)
    assert np.array_equal(want.astype(np.float32).astype(np.float64), want)


def _fp16_finite_nonzero():
    v = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16).view(np.float16).astype(np.float64)
    return v[np.isfinite(v) & (v != 0)]


def test_corrected_quotient_fold_operands():
    """AWQ scale folding divides an fp16 weight (norm weight, linear row or
    bias) by an fp16 scale with the same correction: any finite nonzero fp16
    divisor of either sign (subnormals included) and any finite fp16 dividend
    must give RN(w / s) exactly."""
    rng = random.Random(13)
    vals = _fp16_finite_nonzero()
    small = vals[np.abs(vals) < 2.0 ** -14]  # the subnormals
    for i in range(4000):
        s = float(rng.choice(small if i % 5 == 0 else vals))
        w = float(rng.choice(small if i % 7 == 0 else vals))
        assert corrected_quotient_ok(w, s), (w, s)
    # the extreme magnitudes
    for w in (65504.0, -65504.0, 2.0 ** -24, -(2.0 ** -24), 1.0):
        for s in (2.0 ** -24, -(2.0 ** -24), 65504.0, -65504.0, 3.0, 2.0 ** -14):
            assert corrected_quotient_ok(w, s), (w, s)


def test_gptq_factor_from_the_ul_factorization():
    """The GPU's route to GPTQ's factor: the "UL" factorization H = U U^T
    with U upper triangular (computed from the bottom-right corner), then
    G = U^-1. G is upper triangular with a positive diagonal and
    G^T G = U^-T U^-1 = H^-1, so by the uniqueness of the Cholesky factor it
    is the page's Cholesky(H^-1)^T, reached without forming H^-1 (fp64)."""
    g = np.random.default_rng(9)
    K = 48
    X = g.normal(0, 1, (200, K)) @ (np.eye(K) + 0.3 * g.normal(0, 1, (K, K)))
    H = 2.0 * X.T @ X
    H += 0.01 * np.mean(np.diag(H)) * np.eye(K)
    # UL by columns from the last: U[j][j] = sqrt(H[j][j] - sum_{k>j} U[j][k]^2),
    # U[i][j] = (H[i][j] - sum_{k>j} U[i][k] U[j][k]) / U[j][j] for i < j
    U = np.zeros((K, K))
    for j in range(K - 1, -1, -1):
        U[j, j] = np.sqrt(H[j, j] - U[j, j + 1:] @ U[j, j + 1:])
        for i in range(j):
            U[i, j] = (H[i, j] - U[i, j + 1:] @ U[j, j + 1:]) / U[j, j]
    assert np.allclose(np.triu(U), U) and np.all(np.diag(U) > 0)
    assert np.max(np.abs(U @ U.T - H)) <= 1e-12 * np.max(np.abs(H))
    G = np.linalg.solve(U, np.eye(K))               # U^-1, upper triangular
    ref = np.linalg.cholesky(np.linalg.inv(H)).T     # the page's factor
    assert np.allclose(np.triu(G), G, atol=1e-14 * np.max(np.abs(G)))
    assert np.max(np.abs(G - ref)) <= 1e-9 * np.max(np.abs(ref))
    # the ordinary (LU-order) Cholesky factor of H does not give it
    L = np.linalg.cholesky(H)
    assert np.max(np.abs(np.linalg.inv(L).T - ref)) > 1e-3 * np.max(np.abs(ref))
