"""CPU oracle for group-wise weight-only quantization (W4A16 / W3A16) and AWQ.

TEST INFRASTRUCTURE ONLY. This is a plain, slow, obviously-correct numpy
restatement of what the CUDA library computes. Only ``tests/``,
``__graft_entry__.smoke()`` and the ``cpu_baseline`` / ``--impl reference``
legs of ``bench.py`` may import it. It shares no code with the CUDA path:
neither side imports the other; both take their inputs from ``synth``.

Every function cites the web page (by title) and the section it restates.
Pages cited:

* [MIT-Lab4/5] "MIT 6.5940 Lab 4 + Lab 5: Quantizing an LLM with AWQ, Then
  Running LLaMA2-7B on Your Own Laptop"
* [CMU-L19/20] "CMU 11-868 L19-L20 Model Quantization: GPTQ Saves Memory, and
  the Speedup Comes Along for the Ride"
* [Quantising-LLMs] "Quantising Large Language Models for Efficient Inference"
* [TinyChat] "TinyChat (AWQ on-device runtime)"
* [160GB-Laptop] "LLM Quantization: 160GB Model on a Laptop"

Floating-point contract (the pages fix none of it; these are this library's
readings, identical on the GPU):

* fp16 inputs are widened exactly to fp32. With AWQ scaling, w' = w * s_k in
  fp32 (exact: an 11-bit by 11-bit significand product fits in 24 bits).
* Every quantization decision (range, step, zero point, code) is taken in
  IEEE fp32 with round-to-nearest-even: fp32 division, ``rint`` (ties to
  even), integer add, clamp.
* The per-group step is stored in fp16 rounded toward +inf, so the clamped
  range never cuts off the group's extreme values.
* Dequantized weights, matmul references and AWQ losses are computed in fp64.

Pins: every function here is checked in ``tests/test_oracle_pins.py`` against
values the pages print, closed forms, invariants or brute force; none is
"parity unpinned".
"""
from __future__ import annotations


import numpy as np

__all__ = [
    "f16_round_up",
    "quantize_groups",
    "quantize_groups_f32",
    "dequantize",
    "pack_codes",
    "unpack_codes",
    "packed_words_per_row",
    "gemm_ref",
    "absmax_quantize_int8",
    "zeropoint_quantize_int8",
    "activation_absmean",
    "awq_alpha_grid",
    "awq_candidates",
    "awq_error_matrix",
    "awq_loss",
    "awq_search",
    "awq_fold_into_norm",
    "awq_fold_into_linear_rows",
    "decoder_block_ref",
    "awq_fold_block",
    "act_quantize_int8_groups",
    "w4a8_gemm_ref",
    "gptq_hessian",
    "gptq_quantize",
    "GPTQ_DAMP",
    "MU_FLOOR",
]


# ---------------------------------------------------------------------------
# fp16 rounding helper
# ---------------------------------------------------------------------------

def f16_round_up(v32: np.ndarray) -> np.ndarray:
    """Smallest fp16 value >= each fp32 value (round toward +inf).

    numpy's fp32->fp16 cast rounds to nearest-even; where that result lies
    below the input, step to the next fp16 value upward.
    """
    v32 = np.asarray(v32, dtype=np.float32)
    h = v32.astype(np.float16)
    below = h.astype(np.float32) < v32
    if np.any(below):
        h = h.copy()
        h[below] = np.nextafter(h[below], np.float16(np.inf))
    return h


# ---------------------------------------------------------------------------
# Group-wise quantizer
# ---------------------------------------------------------------------------

def quantize_groups(W16: np.ndarray, bits: int, group: int, symmetric: bool,
                    s16: np.ndarray | None = None):
    """Round-to-nearest group-wise quantization of an [N][K] fp16 weight.

    A group is ``group`` consecutive input channels (along K) of one output
    row: [Quantising-LLMs] "Post-training methods for 4-bit weights" puts one
    scale (and zero point) on each group of 64-128 weights within a row, and
    its numpy routine reshapes each row into groups of that many entries.

    Symmetric (absmax) branch -- [160GB-Laptop] "Symmetric Quantization" and
    the [Quantising-LLMs] routine: qmax = 2^(b-1) - 1, step = max|w| / qmax,
    code = clip(round(w / step), -qmax - 1, qmax), value = code * step.
    Stored as unsigned code + 2^(b-1) with zero point 2^(b-1), so both
    branches dequantize as (q - zero) * step.

    Asymmetric branch -- [160GB-Laptop] "Asymmetric Quantization" maps
    [min, max] onto [qmin, qmax] with step = (max - min) / (qmax - qmin);
    [CMU-L19/20] "absmax and zero-point" writes the offset as a rounded
    integer zero point and uses range := 1 when the range is 0. With
    Q = 2^b - 1: mn = min(min w', 0), mx = max(max w', 0), r = mx - mn,
    step = fp16_up(r / Q) (or 1 when r == 0), zero = clamp(rint(-mn/step), 0, Q),
    q = clamp(rint(w'/step) + zero, 0, Q).

    ``s16`` ([K] fp16, optional) applies AWQ's per-input-channel scaling
    W * diag(s) before quantization ([MIT-Lab4/5] "Question 2").

    Returns (codes uint8 [N][K], steps fp16 [N][K/group], zeros fp16 [N][K/group]).
    """
    W16 = np.asarray(W16)
    assert W16.dtype == np.float16 and W16.ndim == 2
    N, K = W16.shape
    assert K % group == 0, "K must be a multiple of the group size"
    assert 2 <= bits <= 8
    w = W16.astype(np.float32)
    if s16 is not None:
        s16 = np.asarray(s16)
        assert s16.dtype == np.float16 and s16.shape == (K,)
        w = w * s16.astype(np.float32)[None, :]
    return quantize_groups_f32(w, bits, group, symmetric)


def quantize_groups_f32(w: np.ndarray, bits: int, group: int, symmetric: bool):
    """The decisions of ``quantize_groups`` on an fp32 [N][K] array that need
    not hold fp16 values (GPTQ quantizes weights it has already updated)."""
    N, K = w.shape
    G = K // group
    wg = w.reshape(N, G, group)

    if symmetric:
        qmax = (1 << (bits - 1)) - 1
        amax = np.abs(wg).max(axis=2)                      # fp32, exact
        step_h = f16_round_up(amax / np.float32(qmax))
        step_h = np.where(amax == 0, np.float16(1.0), step_h)
        if not np.all(np.isfinite(step_h)):
            raise OverflowError("group step does not fit fp16")
        sf = step_h.astype(np.float32)[:, :, None]
        qs = np.clip(np.rint(wg / sf), -qmax - 1, qmax).astype(np.int32)
        codes = (qs + (1 << (bits - 1))).astype(np.uint8)
        zeros = np.full((N, G), float(1 << (bits - 1)), dtype=np.float16)
    else:
        Q = (1 << bits) - 1
        mn = np.minimum(wg.min(axis=2), np.float32(0))
        mx = np.maximum(wg.max(axis=2), np.float32(0))
        r = (mx - mn).astype(np.float32)                    # fp32 subtraction
        step_h = f16_round_up(r / np.float32(Q))
        step_h = np.where(r == 0, np.float16(1.0), step_h)
        if not np.all(np.isfinite(step_h)):
            raise OverflowError("group step does not fit fp16")
        sf32 = step_h.astype(np.float32)
        zero = np.clip(np.rint(-mn / sf32), 0, Q).astype(np.int32)
        q = np.rint(wg / sf32[:, :, None]).astype(np.int32) + zero[:, :, None]
        codes = np.clip(q, 0, Q).astype(np.uint8)
        zeros = zero.astype(np.float16)
    return codes.reshape(N, K), step_h.astype(np.float16), zeros


def dequantize(codes: np.ndarray, steps: np.ndarray, zeros: np.ndarray, group: int) -> np.ndarray:
    """fp64 weight (q - zero) * step for each element ([160GB-Laptop]
    "Symmetric Quantization": dequantize = code * scale; the zero-point form of
    [CMU-L19/20] "absmax and zero-point": (q - zp) / scale with scale a multiplier)."""
    N, K = codes.shape
    G = K // group
    q = codes.astype(np.float64).reshape(N, G, group)
    z = zeros.astype(np.float64)[:, :, None]
    s = steps.astype(np.float64)[:, :, None]
    return ((q - z) * s).reshape(N, K)


# ---------------------------------------------------------------------------
# Packed layouts
# ---------------------------------------------------------------------------
#
# 4-bit: row-major [N][K/8] uint32. Word c of a row holds k = 8c..8c+7.
#   Nibble slot j (bits 4j..4j+3) holds k = 8c + 2j for j < 4 and
#   k = 8c + 2(j-4) + 1 for j >= 4, i.e. slot order [k0,k2,k4,k6,k1,k3,k5,k7].
#   A mask of 0x000F000F over (word >> 4j) therefore yields the consecutive
#   pair (k_2j, k_2j+1) in the two 16-bit halves. This is the same idea as
#   TinyChatEngine's offline reordering ([MIT-Lab4/5] "Background: why the
#   4-bit weights get reordered first"), redone for 16-bit GPU lanes.
#
# 3-bit: row-major [N][3K/32] uint32. Three words (t = 0, 1, 2) per 32 k:
#   word t, pair j (0..4): bits 3j..3j+2 hold k = 32c + 10t + 2j, bits
#   16+3j..18+3j hold k = 32c + 10t + 2j + 1; k = 32c+30 keeps its bit b in
#   bit 15 of word b and k = 32c+31 keeps its bit b in bit 31 of word b.
#   Exactly 3 bits per weight.

def packed_words_per_row(K: int, bits: int) -> int:
    if bits == 4:
        assert K % 8 == 0
        return K // 8
    if bits == 3:
        assert K % 32 == 0
        return 3 * K // 32
    raise ValueError("bits must be 3 or 4")


def _pack4(codes: np.ndarray) -> np.ndarray:
    N, K = codes.shape
    c = codes.astype(np.uint32).reshape(N, K // 8, 8)
    words = np.zeros((N, K // 8), dtype=np.uint32)
    for j in range(4):
        words |= c[:, :, 2 * j] << np.uint32(4 * j)
        words |= c[:, :, 2 * j + 1] << np.uint32(4 * (j + 4))
    return words


def _unpack4(words: np.ndarray, K: int) -> np.ndarray:
    N = words.shape[0]
    w = words.reshape(N, K // 8)
    out = np.zeros((N, K // 8, 8), dtype=np.uint8)
    for j in range(4):
        out[:, :, 2 * j] = (w >> np.uint32(4 * j)) & 0xF
        out[:, :, 2 * j + 1] = (w >> np.uint32(4 * (j + 4))) & 0xF
    return out.reshape(N, K)


def _pack3(codes: np.ndarray) -> np.ndarray:
    N, K = codes.shape
    c = codes.astype(np.uint32).reshape(N, K // 32, 32)
    words = np.zeros((N, K // 32, 3), dtype=np.uint32)
    for t in range(3):
        for j in range(5):
            words[:, :, t] |= c[:, :, 10 * t + 2 * j] << np.uint32(3 * j)
            words[:, :, t] |= c[:, :, 10 * t + 2 * j + 1] << np.uint32(16 + 3 * j)
        words[:, :, t] |= ((c[:, :, 30] >> np.uint32(t)) & 1) << np.uint32(15)
        words[:, :, t] |= ((c[:, :, 31] >> np.uint32(t)) & 1) << np.uint32(31)
    return words.reshape(N, 3 * K // 32)


def _unpack3(words: np.ndarray, K: int) -> np.ndarray:
    N = words.shape[0]
    w = words.reshape(N, K // 32, 3)
    out = np.zeros((N, K // 32, 32), dtype=np.uint8)
    for t in range(3):
        for j in range(5):
            out[:, :, 10 * t + 2 * j] = (w[:, :, t] >> np.uint32(3 * j)) & 7
            out[:, :, 10 * t + 2 * j + 1] = (w[:, :, t] >> np.uint32(16 + 3 * j)) & 7
        out[:, :, 30] |= (((w[:, :, t] >> np.uint32(15)) & 1) << np.uint32(t)).astype(np.uint8)
        out[:, :, 31] |= (((w[:, :, t] >> np.uint32(31)) & 1) << np.uint32(t)).astype(np.uint8)
    return out.reshape(N, K)


def pack_codes(codes: np.ndarray, bits: int) -> np.ndarray:
    """Pack b-bit codes [N][K] into the documented uint32 layout."""
    assert codes.dtype == np.uint8
    assert int(codes.max(initial=0)) < (1 << bits)
    return _pack4(codes) if bits == 4 else _pack3(codes)


def unpack_codes(words: np.ndarray, bits: int, K: int) -> np.ndarray:
    return _unpack4(words, K) if bits == 4 else _unpack3(words, K)


# ---------------------------------------------------------------------------
# W4A16 / W3A16 matmul reference
# ---------------------------------------------------------------------------

def gemm_ref(X16: np.ndarray, codes: np.ndarray, steps: np.ndarray, zeros: np.ndarray,
             group: int) -> np.ndarray:
    """Y[m][n] = sum_k x[m][k] * (q[n][k] - zero) * step, in fp64.

    This is the weight-only matmul of [Quantising-LLMs] "Weight-only vs
    weight-and-activation quantisation" (16-bit activations, weights
    dequantized inside the matmul), written as a plain fp64 matmul of the
    dequantized weight; one library matmul is the only step.
    """
    D = dequantize(codes, steps, zeros, group)
    return np.asarray(X16, dtype=np.float64) @ D.T


# ---------------------------------------------------------------------------
# int8 absmax / zero-point ([CMU-L19/20] "absmax and zero-point")
# ---------------------------------------------------------------------------

def absmax_quantize_int8(X: np.ndarray):
    """Per-tensor int8 absmax: multiplier 127/max|X|, code = round(multiplier*X)
    (round half to even), dequant = code / multiplier."""
    X = np.asarray(X, dtype=np.float64)
    mult = 127.0 / np.max(np.abs(X))
    q = np.rint(mult * X)
    return q.astype(np.int8), q / mult


def zeropoint_quantize_int8(X: np.ndarray):
    """Per-tensor int8 zero-point: range (1 if zero), multiplier 255/range,
    zp = round(-multiplier*min - 128), code = clip(round(X*multiplier + zp), -128, 127),
    dequant = (code - zp) / multiplier."""
    X = np.asarray(X, dtype=np.float64)
    rng_ = float(np.max(X) - np.min(X))
    rng_ = 1.0 if rng_ == 0 else rng_
    mult = 255.0 / rng_
    zp = np.rint(-mult * np.min(X) - 128.0)
    q = np.clip(np.rint(X * mult + zp), -128, 127)
    return q.astype(np.int8), (q - zp) / mult


# ---------------------------------------------------------------------------
# AWQ: activation statistics, candidate scales, reconstruction loss, search
# ---------------------------------------------------------------------------

MU_FLOOR = 2.0 ** -14


def activation_absmean(X16: np.ndarray) -> np.ndarray:
    """mu_k = mean over calibration tokens of |x_tk|, in fp64.

    [MIT-Lab4/5] "Starting point and setup": forward hooks record the mean
    absolute value of each linear layer's input. Each fp16 value is a
    multiple of 2^-24 below 2^16, so the fp64 sum of up to 2^13 of them is
    exact in any order; one fp64 division by T follows.
    """
    X = np.asarray(X16)
    assert X.dtype == np.float16
    T = X.shape[0]
    return np.abs(X.astype(np.float64)).sum(axis=0) / float(T)


def awq_alpha_grid(n_alpha: int = 20) -> np.ndarray:
    """alpha_j = j / n_alpha in fp64 (0, 0.05, ..., 0.95 for 20)."""
    return np.arange(n_alpha, dtype=np.float64) / float(n_alpha)


def awq_candidates(mu: np.ndarray, alphas: np.ndarray) -> np.ndarray:
    """s_alpha,k = fp16_RN(max(mu_k, 2^-14) ** alpha), fp64 pow.

    [MIT-Lab4/5] "Question 2": scale the salient (large-activation) input
    channels up by s, computed from the activation statistic, and search over
    the scale. The floor on mu keeps s > 0 on all-zero channels.
    """
    m = np.maximum(np.asarray(mu, dtype=np.float64), MU_FLOOR)
    out = np.empty((len(alphas), m.shape[0]), dtype=np.float16)
    for j, a in enumerate(alphas):
        out[j] = np.power(m, float(a)).astype(np.float16)
    return out


def awq_error_matrix(W16: np.ndarray, s16: np.ndarray, bits: int, group: int,
                     symmetric: bool) -> np.ndarray:
    """E = W - Q(W diag(s)) diag(s)^-1 in fp64 ("scale up, quantize, scale
    down" of [MIT-Lab4/5] "Question 2"; Q is quantize-then-dequantize, the
    pseudo quantization of "Starting point and setup")."""
    codes, steps, zeros = quantize_groups(W16, bits, group, symmetric, s16=s16)
    Dq = dequantize(codes, steps, zeros, group)
    return W16.astype(np.float64) - Dq / s16.astype(np.float64)[None, :]


def awq_loss(X16: np.ndarray, Ws, s16: np.ndarray, bits: int, group: int,
             symmetric: bool) -> float:
    """L = sum over linears of || X E^T ||_F^2 in fp64.

    The layer-wise reconstruction objective ||WX - W^X||^2 of [CMU-L19/20]
    "Quantizing during training vs. after it", restricted to W^ =
    Q(W diag s) diag(s)^-1; linears fed by the same input are summed.
    """
    X = np.asarray(X16, dtype=np.float64)
    total = 0.0
    for W in Ws:
        E = awq_error_matrix(W, s16, bits, group, symmetric)
        P = X @ E.T
        total += float(np.sum(P * P))
    return total


def awq_search(X16: np.ndarray, Ws, bits: int, group: int, symmetric: bool,
               alphas: np.ndarray | None = None) -> dict:
    """Grid search over alpha; picks the lowest loss (first index on ties).

    Steps, in the order [MIT-Lab4/5] "Question 2" gives them: compute the
    scale from the activation statistic, scale the weight up, quantize,
    scale down, measure the error, keep the best.
    """
    if alphas is None:
        alphas = awq_alpha_grid(20)
    mu = activation_absmean(X16)
    S = awq_candidates(mu, alphas)
    losses = np.array([awq_loss(X16, Ws, S[j], bits, group, symmetric)
                       for j in range(len(alphas))], dtype=np.float64)
    best = int(np.argmin(losses))
    return {"mu": mu, "candidates": S, "losses": losses, "best": best, "s": S[best].copy(),
            "alphas": np.asarray(alphas, dtype=np.float64)}


# ---------------------------------------------------------------------------
# AWQ scale folding ([MIT-Lab4/5] "Question 2": the searched scales are folded
# into the previous LayerNorm or linear layer)
# ---------------------------------------------------------------------------

def awq_fold_into_norm(gamma: np.ndarray, s: np.ndarray) -> np.ndarray:
    """gamma'_k = gamma_k / s_k: a normalisation layer whose output feeds the
    scaled linears absorbs diag(s)^-1 into its per-channel weight
    ([MIT-Lab4/5] "Question 2", scale_ln_fcs).

    fp16 inputs: the library's stored form, fp16_RN(fp32(gamma) / fp32(s))
    (one IEEE fp32 division, then one rounding to fp16). fp64 inputs: the
    quotient in fp64 (used by the block-equivalence check).
    """
    gamma, s = np.asarray(gamma), np.asarray(s)
    assert gamma.shape == s.shape and gamma.ndim == 1
    if gamma.dtype == np.float16:
        assert s.dtype == np.float16
        return (gamma.astype(np.float32) / s.astype(np.float32)).astype(np.float16)
    return gamma.astype(np.float64) / s.astype(np.float64)


def awq_fold_into_linear_rows(W: np.ndarray, s: np.ndarray, b: np.ndarray | None = None):
    """W'[n][k] = W[n][k] / s_n and b'_n = b_n / s_n: a linear whose output
    feeds the scaled linears (v_proj before o_proj, up_proj before down_proj)
    absorbs diag(s)^-1 into its output rows ([MIT-Lab4/5] "Question 2",
    scale_fc_fc). s has one entry per output row of W. fp16 inputs follow
    the stored-form contract of ``awq_fold_into_norm``; fp64 inputs fold in
    fp64. Returns (W', b') (b' is None without a bias)."""
    W, s = np.asarray(W), np.asarray(s)
    assert W.ndim == 2 and s.shape == (W.shape[0],)
    if W.dtype == np.float16:
        assert s.dtype == np.float16
        s32 = s.astype(np.float32)
        Wf = (W.astype(np.float32) / s32[:, None]).astype(np.float16)
        bf = None if b is None else (np.asarray(b).astype(np.float32) / s32).astype(np.float16)
        return Wf, bf
    s64 = s.astype(np.float64)
    Wf = W.astype(np.float64) / s64[:, None]
    bf = None if b is None else np.asarray(b, dtype=np.float64) / s64
    return Wf, bf


def _rmsnorm(x: np.ndarray, gamma: np.ndarray, eps: float) -> np.ndarray:
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * gamma


def decoder_block_ref(x: np.ndarray, p: dict, n_heads: int, eps: float = 1e-6) -> np.ndarray:
    """One LLaMA-shaped decoder block in fp64, the computation the folded
    scales must leave unchanged: pre-norm (RMS) causal multi-head attention
    with q/k/v/o projections, then a pre-norm SwiGLU MLP (gate, up, down),
    each with a residual connection. Linear weights are nn.Linear [out][in]
    (y = x W^T). ``p`` holds gamma1, wq, wk, wv, wo, gamma2, wg, wu, wd."""
    x = np.asarray(x, dtype=np.float64)
    T, D = x.shape
    hd = D // n_heads
    h = _rmsnorm(x, p["gamma1"], eps)
    q, k, v = h @ p["wq"].T, h @ p["wk"].T, h @ p["wv"].T
    att = np.empty_like(q)
    mask = np.triu(np.ones((T, T), dtype=bool), 1)
    for i in range(n_heads):
        sl = slice(i * hd, (i + 1) * hd)
        a = q[:, sl] @ k[:, sl].T / np.sqrt(hd)
        a[mask] = -np.inf
        a = np.exp(a - a.max(axis=1, keepdims=True))
        att[:, sl] = (a / a.sum(axis=1, keepdims=True)) @ v[:, sl]
    y = x + att @ p["wo"].T
    h2 = _rmsnorm(y, p["gamma2"], eps)
    g, u = h2 @ p["wg"].T, h2 @ p["wu"].T
    return y + ((g / (1.0 + np.exp(-g))) * u) @ p["wd"].T


def awq_fold_block(p: dict, s_qkv, s_o, s_gu, s_down) -> dict:
    """The four search places of a LLaMA block with their scales applied
    ([MIT-Lab4/5] "Question 2": scales searched at the attention input, the
    attention output, the MLP input and the down projection's input, then
    folded into the previous norm or linear): each scaled linear's weight
    becomes W diag(s) and the op that produces its input absorbs diag(s)^-1
    (gamma1 for q/k/v, v_proj's rows for o_proj, gamma2 for gate/up,
    up_proj's rows for down_proj). Every parameter is returned in fp64."""
    f = {k: np.asarray(v, dtype=np.float64) for k, v in p.items()}
    s_qkv, s_o, s_gu, s_down = (np.asarray(t, dtype=np.float64) for t in (s_qkv, s_o, s_gu, s_down))
    out = dict(f)
    out["gamma1"] = awq_fold_into_norm(f["gamma1"], s_qkv)
    for name in ("wq", "wk", "wv"):
        out[name] = f[name] * s_qkv[None, :]
    out["wv"], _ = awq_fold_into_linear_rows(out["wv"], s_o)
    out["wo"] = f["wo"] * s_o[None, :]
    out["gamma2"] = awq_fold_into_norm(f["gamma2"], s_gu)
    out["wg"] = f["wg"] * s_gu[None, :]
    out["wu"] = f["wu"] * s_gu[None, :]
    out["wu"], _ = awq_fold_into_linear_rows(out["wu"], s_down)
    out["wd"] = f["wd"] * s_down[None, :]
    return out


# ---------------------------------------------------------------------------
# GPTQ ([CMU-L19/20] "The algorithm in four steps" and "Why it can actually
# run: from OBS to GPTQ"), written into the same group-wise packed format
# ---------------------------------------------------------------------------

GPTQ_DAMP = 0.01


def gptq_hessian(X16: np.ndarray, damp: float = GPTQ_DAMP):
    """H = 2 X^T X + lambda I in fp64 for calibration inputs X [T][K] (the
    pages' 2XX^T with X stored tokens-major), lambda = damp * mean(diag H).

    Readings (the pages write "+ lambda I" without a value): lambda is 1 % of
    the mean diagonal, and an input channel that is zero on every token has
    H_kk := 1 (its weights are set to 0 by ``gptq_quantize``), so H stays
    positive definite. Returns (H, dead) with dead the zero channels."""
    X = np.asarray(X16, dtype=np.float64)
    H = 2.0 * (X.T @ X)
    dead = np.diag(H) == 0
    H[dead, dead] = 1.0
    H += damp * np.mean(np.diag(H)) * np.eye(H.shape[0])
    return H, dead


def gptq_quantize(W16: np.ndarray, X16: np.ndarray, bits: int, group: int, symmetric: bool,
                  block: int = 128, damp: float = GPTQ_DAMP):
    """GPTQ in the page's four steps, in fp64:

    1. G = Cholesky((2 X X^T + lambda I)^-1)^T, the upper triangular factor
       with H^-1 = G^T G (two library calls: inverse, Cholesky).
    2. Within a block of ``block`` columns, quantize one column (all rows at
       once). When a column starts a quantization group, the group's step and
       zero point are chosen from the group's current (already updated)
       weights with the library's round-to-nearest decisions
       (``quantize_groups`` on the fp32 values).
    3. The column's error, divided by G's diagonal entry.
    4. Update the remaining columns of the block with it; when the block is
       done, update every column to its right in one batch (lazy batch
       update).

    Returns (codes uint8 [N][K], steps fp16 [N][K/group], zeros fp16
    [N][K/group]), the format of ``quantize_groups``."""
    W = np.asarray(W16).astype(np.float64).copy()
    N, K = W.shape
    assert K % group == 0 and (block % group == 0 or group % block == 0)
    H, dead = gptq_hessian(X16, damp)
    W[:, dead] = 0.0
    G = np.linalg.cholesky(np.linalg.inv(H)).T
    codes = np.zeros((N, K), dtype=np.uint8)
    steps = np.zeros((N, K // group), dtype=np.float16)
    zeros = np.zeros((N, K // group), dtype=np.float16)
    step_g = zero_g = None
    for b0 in range(0, K, block):
        b1 = min(b0 + block, K)
        Err = np.zeros((N, b1 - b0))
        for i in range(b0, b1):
            if i % group == 0:
                gc, gs, gz = quantize_groups_f32(W[:, i:i + group].astype(np.float32), bits, group, symmetric)
                steps[:, i // group], zeros[:, i // group] = gs[:, 0], gz[:, 0]
                step_g, zero_g = gs[:, 0].astype(np.float64), gz[:, 0].astype(np.float64)
            q = _code_of(W[:, i].astype(np.float32), steps[:, i // group], zeros[:, i // group], bits, symmetric)
            codes[:, i] = q
            deq = (q.astype(np.float64) - zero_g) * step_g
            err = (W[:, i] - deq) / G[i, i]
            W[:, i + 1:b1] -= np.outer(err, G[i, i + 1:b1])
            Err[:, i - b0] = err
        W[:, b1:] -= Err @ G[b0:b1, b1:]
    return codes, steps, zeros


def _code_of(w32: np.ndarray, step_h: np.ndarray, zero_h: np.ndarray, bits: int, symmetric: bool) -> np.ndarray:
    """Code of one fp32 value per row under its group's (step, zero): the
    rounding and clamp of ``quantize_groups`` (fp32 division, ties to even)."""
    sf = step_h.astype(np.float32)
    if symmetric:
        qmax = (1 << (bits - 1)) - 1
        qs = np.clip(np.rint(w32 / sf), -qmax - 1, qmax).astype(np.int32)
        return (qs + (1 << (bits - 1))).astype(np.uint8)
    Q = (1 << bits) - 1
    q = np.rint(w32 / sf).astype(np.int32) + zero_h.astype(np.int32)
    return np.clip(q, 0, Q).astype(np.uint8)


# ---------------------------------------------------------------------------
# W4A8: 4-bit weights and 8-bit activations, both per group of channels
# ([MIT-Lab4/5] "The five implementation files and grading": the Lab 5 linear
# is W4A8 with group size 32; the int8 absmax form of [CMU-L19/20] "absmax
# and zero-point" applied to each group of activations)
# ---------------------------------------------------------------------------

def act_quantize_int8_groups(X16: np.ndarray, group: int = 32):
    """Per row m and group g of ``group`` consecutive channels: multiplier
    mult = 127 / max|x| (1 for an all-zero group), code = round(mult * x)
    (ties to even), clipped to [-127, 127]. fp32 arithmetic on the fp16
    inputs (one IEEE division, one multiply, rint), as on the GPU.
    Returns (codes int8 [M][K], mult fp32 [M][K/group])."""
    X = np.asarray(X16)
    assert X.dtype == np.float16 and X.ndim == 2
    M, K = X.shape
    assert K % group == 0
    x = X.astype(np.float32).reshape(M, K // group, group)
    amax = np.abs(x).max(axis=2)
    mult = np.where(amax == 0, np.float32(1.0), np.float32(127.0) / np.where(amax == 0, np.float32(1.0), amax))
    mult = mult.astype(np.float32)
    q = np.clip(np.rint(x * mult[:, :, None]), -127, 127).astype(np.int8)
    return q.reshape(M, K), mult


def w4a8_gemm_ref(qx: np.ndarray, mult: np.ndarray, codes: np.ndarray, steps: np.ndarray, zeros: np.ndarray,
                  group: int) -> np.ndarray:
    """Y[m][n] = sum_g (step[n][g] / mult[m][g]) * sum_{k in g} (q[n][k] - zero[n][g]) * qx[m][k]:
    the integer dot product of each group, scaled by the weight's step and
    the activation's 1/multiplier, summed over groups in fp64."""
    M, K = qx.shape
    N = codes.shape[0]
    G = K // group
    qw = codes.astype(np.int64).reshape(N, G, group) - zeros.astype(np.int64)[:, :, None]
    qa = qx.astype(np.int64).reshape(M, G, group)
    dots = np.einsum("mgk,ngk->mng", qa, qw)  # exact integers
    scale = steps.astype(np.float64)[None, :, :] / mult.astype(np.float64)[:, None, :]
    return np.sum(dots.astype(np.float64) * scale, axis=2)
