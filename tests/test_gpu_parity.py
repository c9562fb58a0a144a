"""CUDA path vs the CPU oracle, element by element, through the C ABI.

Integer outputs (codes, packed words, steps, zeros) must match bit for bit;
matmul outputs must meet relative L2 error <= 1e-3 and max abs error <=
1e-2 * max|y| against the oracle's fp64 matmul of the dequantized weight.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

REL_L2 = 1e-3
MAX_ABS = 1e-2


@pytest.fixture(scope="module")
def wq():
    from weight_only_quantization_group_b200 import build
    build.build()
    import weight_only_quantization_group_b200 as m
    assert torch.cuda.is_available()
    return m


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def gpu_quantize(wq, W, s, bits, sym, group=128):
    packed, steps, zeros = wq.wq_quantize_pack(dev(W), None if s is None else dev(s), bits=bits, symmetric=sym,
                                               group_size=group)
    assert wq.wq_get_last_device_error() == 0
    return packed, steps, zeros


def assert_quant_parity(wq, W, s, bits, sym, group=128):
    codes, st, z = O.quantize_groups(W, bits, group, sym, s16=s)
    words = O.pack_codes(codes, bits).reshape(-1)
    packed, steps, zeros = gpu_quantize(wq, W, s, bits, sym, group)
    gs, gz = steps.cpu().numpy(), zeros.cpu().numpy()
    assert np.array_equal(gs.view(np.uint16), st.view(np.uint16)), "steps differ"
    assert np.array_equal(gz.view(np.uint16), z.view(np.uint16)), "zeros differ"
    gp = packed.cpu().numpy().view(np.uint32)
    assert gp.size == words.size
    bad = np.flatnonzero(gp != words)
    assert bad.size == 0, f"{bad.size} packed words differ, first at {bad[:5]}"
    return (codes, st, z), (packed, steps, zeros)


def assert_close(y, yref):
    y = np.asarray(y, dtype=np.float64)
    rel = np.linalg.norm(y - yref) / max(np.linalg.norm(yref), 1e-300)
    mab = np.max(np.abs(y - yref)) / max(np.max(np.abs(yref)), 1e-300)
    assert rel <= REL_L2 and mab <= MAX_ABS, (rel, mab)
    return rel, mab


def _awq_scale(K, seed):
    g = np.random.default_rng(seed)
    return np.exp(g.normal(0, 0.7, K)).astype(np.float16)


# ---------------------------------------------------------------------------
# S3 quantize + pack
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("awq", [False, True])
def test_quantize_pack_parity_ragged(wq, bits, sym, awq):
    g = synth.rng(100 + bits)
    W = synth.weight(g, 333, 1152, 0.02, channel_frac=0.01, channel_mult=10.0, heavy_frac=0.01)
    s = _awq_scale(1152, 7) if awq else None
    assert_quant_parity(wq, W, s, bits, sym)


@pytest.mark.parametrize("group", [32, 64])
@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("awq", [False, True])
def test_quantize_pack_small_groups(wq, group, bits, sym, awq):
    """Groups of 32 and 64 channels ("Quantising Large Language Models",
    group-size sweep; the W4A8 linear of "MIT 6.5940 Lab 4 + Lab 5" uses 32):
    codes, words, steps and zeros bit-exact, ragged N, heavy-tailed weights,
    with and without AWQ scales, and an all-zero group."""
    g = synth.rng(110 + bits + group)
    W = synth.weight(g, 333, 1152, 0.02, channel_frac=0.01, channel_mult=10.0, heavy_frac=0.01)
    W[5, :group] = 0
    s = _awq_scale(1152, 8) if awq else None
    assert_quant_parity(wq, W, s, bits, sym, group)


@pytest.mark.parametrize("group", [32, 64])
@pytest.mark.parametrize("bits", [3, 4])
def test_unpack_dequant_small_groups(wq, group, bits):
    g = synth.rng(210 + group)
    W = synth.weight(g, 77, 768, 0.02, channel_frac=0.02, channel_mult=8.0)
    (codes, st, z), (packed, steps, zeros) = assert_quant_parity(wq, W, None, bits, False, group)
    out = wq.wq_unpack_dequant(packed, steps, zeros, 77, 768, bits=bits, group_size=group).cpu().numpy()
    ref = O.dequantize(codes, st, z, group).astype(np.float16)
    assert np.array_equal(out.view(np.uint16), ref.view(np.uint16))


def test_quantize_pack_edge_groups(wq):
    g = np.random.default_rng(1)
    W = g.normal(0, 0.02, (24, 512))
    W[0] = 0.0                                   # all-zero groups -> step 1, zero 0
    W[1, :128] = 0.01                            # constant group
    W[2, :128] = np.abs(W[2, :128]) + 0.001      # group above 0
    W[3, 128:256] = -np.abs(W[3, 128:256]) - 1e-3
    W[4] *= 1e-5                                 # tiny values -> subnormal fp16 steps
    W[5] *= 500.0                                # large values
    W[6, ::2] = 0.0
    W16 = W.astype(np.float16)
    for bits in (3, 4):
        for sym in (False, True):
            assert_quant_parity(wq, W16, None, bits, sym)


def _near_half_case(bits, sym, rows=12, groups=6, seed=5):
    """Weights and AWQ scales whose scaled values w * s sit on, or within
    2^-16 of, half-integer multiples of the group step: ties (rounded to even
    by the contract), values that the sign of w * s - h * step settles, and
    values only the exact fp32 quotient settles (closer than 2^-18).

    Each group's first two channels (s = 1) fix its step at 2^-7; the other
    channels take fp16 (w, s) pairs found by enumerating every fp16 s in
    [1, 2)."""
    step = 2.0 ** -7
    qmax = (1 << (bits - 1)) - 1
    lo_m, hi_m = (-qmax, qmax) if sym else (-(((1 << bits) - 1) // 2), 1 << (bits - 1))
    s_all = np.arange(0x3C00, 0x4000, dtype=np.uint16).view(np.float16)
    pairs = []
    for m in range(lo_m, hi_m):
        h = m + 0.5
        if abs(h) >= (qmax if sym else 99):
            continue
        w0 = (h * step / s_all.astype(np.float64)).astype(np.float16)
        for w in (np.nextafter(w0, np.float16(-1)), w0, np.nextafter(w0, np.float16(1))):
            a = (w.astype(np.float32) * s_all.astype(np.float32)).astype(np.float64) / step
            dist = np.abs(a - h)
            for i in np.nonzero(dist <= 2.0 ** -16)[0]:
                pairs.append((w[i], s_all[i], dist[i]))
    g = np.random.default_rng(seed)
    g.shuffle(pairs)
    K = 128 * groups
    s = np.ones(K, np.float16)
    W = np.zeros((rows, K), np.float16)
    free = [k for k in range(K) if k % 128 >= 2]
    used = []
    for k, (w, sv, dist) in zip(free, pairs):
        s[k] = sv
        W[:, k] = w
        used.append(dist)
    for k in free[len(used):]:
        s[k] = np.float16(1.0 + g.random())
    # every row: a random third of the channels take other values in range
    bound = 0.95 * (qmax if sym else min(-lo_m, hi_m)) * step
    for r in range(rows):
        sel = np.array(free)[g.random(len(free)) < 1 / 3]
        W[r, sel] = (g.uniform(-bound, bound, len(sel)) / s[sel].astype(np.float64)).astype(np.float16)
    W[:, 0::128] = np.float16(lo_m * step)
    W[:, 1::128] = np.float16(hi_m * step)
    used = np.array(used)
    classes = ((used == 0).sum(), ((used > 0) & (used < 2.0 ** -18)).sum(), (used >= 2.0 ** -18).sum())
    return W, s, classes


@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("sym", [False, True])
def test_quantize_pack_near_half_quotients(wq, bits, sym):
    W, s, (ties, by_division, by_sign) = _near_half_case(bits, sym)
    assert ties > 0 and by_division > 0 and by_sign > 0, (ties, by_division, by_sign)
    codes, st, _ = O.quantize_groups(W, bits, 128, sym, s16=s)
    assert np.all(st.astype(np.float64) == 2.0 ** -7)
    assert_quant_parity(wq, W, s, bits, sym)
    # the same values without scaling: fp16 ties only
    assert_quant_parity(wq, (W.astype(np.float32) * s.astype(np.float32)).astype(np.float16), None, bits, sym)


@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("lo,hi", [(-0.0546875, 0.0625), (-0.0713, 0.01831), (-3.1e-3, 2.9e-2)])
def test_quantize_pack_every_fp16_value_in_range(wq, bits, sym, lo, hi):
    """Every finite fp16 value between lo and hi, 126 to a group, each group
    also holding lo and hi so that all groups share one step (whatever the
    rounded-up range over 2^b - 1 gives: here steps with long significands)."""
    lo16, hi16 = np.float16(lo), np.float16(hi)
    allv = np.arange(0, 0x10000, dtype=np.uint32).astype(np.uint16).view(np.float16)
    allv = allv[np.isfinite(allv)]
    vals = np.unique(allv[(allv >= lo16) & (allv <= hi16)])
    per = 126
    groups = -(-vals.size // per)
    vals = np.concatenate([vals, np.zeros(groups * per - vals.size, np.float16)]).reshape(groups, per)
    grp = np.concatenate([np.full((groups, 1), lo16), np.full((groups, 1), hi16), vals], axis=1)
    gpr = 8  # groups per row
    rows = -(-groups // gpr)
    pad = np.zeros((rows * gpr - groups, 128), np.float16)
    W = np.concatenate([grp, pad]).reshape(rows, gpr * 128)
    _, st, _ = O.quantize_groups(W, bits, 128, sym)
    assert np.unique(st[: groups // gpr]).size == 1
    assert_quant_parity(wq, W, None, bits, sym)


@pytest.mark.parametrize("bad", [np.nan, np.inf, -np.inf])
@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("awq", [False, True])
def test_quantize_pack_non_finite_weight(wq, bad, sym, awq):
    """A non-finite weight makes its group's step non-finite and latches
    WQ_ERR_RANGE; every other group is still quantized per the contract."""
    g = synth.rng(300)
    W = synth.weight(g, 8, 512, 0.02)
    s = _awq_scale(512, 9) if awq else None
    W[3, 200] = bad
    packed, steps, zeros = wq.wq_quantize_pack(dev(W), None if s is None else dev(s), bits=4, symmetric=sym)
    assert wq.wq_get_last_device_error() == wq.WQ_ERR_RANGE
    assert wq.wq_get_last_device_error() == 0
    Wc = W.copy()
    Wc[3, 200] = 0
    codes, st, z = O.quantize_groups(Wc, 4, 128, sym, s16=s)
    gs = steps.cpu().numpy()
    keep = np.ones(gs.shape, bool)
    keep[3, 1] = False
    assert not np.isfinite(gs[3, 1])
    assert np.array_equal(gs.view(np.uint16)[keep], st.view(np.uint16)[keep])
    assert np.array_equal(zeros.cpu().numpy().view(np.uint16)[keep], z.view(np.uint16)[keep])
    words = O.pack_codes(codes, 4).reshape(8, 64)
    gp = packed.cpu().numpy().view(np.uint32).reshape(8, 64)
    wkeep = np.ones(gp.shape, bool)
    wkeep[3, 16:32] = False
    assert np.array_equal(gp[wkeep], words[wkeep])


def test_quantize_pack_small_linear(wq):
    c = synth.config_small_linear(0)
    assert_quant_parity(wq, c.W, None, 4, False)


def test_quantize_pack_llama7b_full(wq):
    for c in synth.config_llama7b_decode(1):
        assert_quant_parity(wq, c.W, None, 4, False)


@pytest.mark.parametrize("bits", [3, 4])
def test_quantize_pack_llama65b_full(wq, bits):
    c = synth.config_llama65b_decode(bits)
    assert_quant_parity(wq, c.W, None, bits, False)


@pytest.mark.parametrize("bits", [3, 4])
def test_unpack_dequant_bit_exact(wq, bits):
    g = synth.rng(200)
    W = synth.weight(g, 77, 768, 0.02, channel_frac=0.02, channel_mult=8.0)
    (codes, st, z), (packed, steps, zeros) = assert_quant_parity(wq, W, None, bits, False)
    out = wq.wq_unpack_dequant(packed, steps, zeros, 77, 768, bits=bits).cpu().numpy()
    ref = O.dequantize(codes, st, z, 128).astype(np.float16)
    assert np.array_equal(out.view(np.uint16), ref.view(np.uint16))


# ---------------------------------------------------------------------------
# S5 GEMV (small M)
# ---------------------------------------------------------------------------

def gemm_workspace(wq, M, N, K, bits, group=128):
    n = wq.wq_gemm_workspace_bytes(M, N, K, bits=bits, group_size=group)
    assert n > 0
    return torch.zeros(n, dtype=torch.uint8, device="cuda")  # zero-filled before its first use


def run_gemm(wq, X, quant_gpu, N, bits, sym=False, group=128, workspace=None):
    packed, steps, zeros = quant_gpu
    Y = wq.wq_w4a16_gemm(dev(X), packed, steps, zeros, N, bits=bits, symmetric=sym, group_size=group,
                         workspace=workspace)
    assert wq.wq_get_last_device_error() == 0
    return Y.cpu().numpy()


@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("M", [1, 2, 3, 5, 8, 11])
@pytest.mark.parametrize("NK", [(333, 1152), (64, 128), (1000, 4096), (17, 11008)])
def test_gemv_parity_ragged(wq, gemv_variant, bits, M, NK):
    N, K = NK
    g = synth.rng(300 + M + bits)
    W = synth.weight(g, N, K, 0.02, channel_frac=0.01, channel_mult=10.0)
    X = synth.activations(g, M, K, channel_frac=0.01, channel_mult=20.0)
    (codes, st, z), qg = assert_quant_parity(wq, W, None, bits, False)
    Y = run_gemm(wq, X, qg, N, bits)
    assert_close(Y, O.gemm_ref(X, codes, st, z, 128))


@pytest.mark.parametrize("bits", [3, 4])
def test_gemv_symmetric(wq, gemv_variant, bits):
    g = synth.rng(400)
    W = synth.weight(g, 256, 2048, 0.02)
    X = synth.activations(g, 2, 2048)
    (codes, st, z), qg = assert_quant_parity(wq, W, None, bits, True)
    assert_close(run_gemm(wq, X, qg, 256, bits, sym=True), O.gemm_ref(X, codes, st, z, 128))


def _gemv_error_bound(X, steps):
    """Bound on the GEMV's rounding error per output. The offset formulations
    form sum_k x_k (q_k - z) from fp32 accumulators that carry an offset per
    product (1024 + q in fp16, or 128 + q/16 scaled back by 16 in fp32): at
    most 16 products per accumulator, each partial sum rounded at 2^-24 of a
    magnitude below 2^11 * sum|x| of the chunk, so the error stays below
    2^-8 * step * sum|x| per 32-channel chunk."""
    K = X.shape[1]
    ax = np.abs(X.astype(np.float64)).reshape(X.shape[0], K // 128, 128).sum(axis=2)   # [M][G]
    return (2.0 ** -8) * (ax @ steps.astype(np.float64).T) + 2.0 ** -24


@pytest.fixture(params=["rows_int", "rows_half", "tiled", "tiled_exact"])
def gemv_variant(wq, request):
    """GEMV kernel choice: the row-streaming kernel where it applies, with
    integer digit products or fp32 offset sums (the default); the tiled
    kernel with offset sums; the tiled kernel with exact fp16 (q - zero)
    products."""
    kern = wq.WQ_GEMV_KERNEL_TILED if request.param.startswith("tiled") else wq.WQ_GEMV_KERNEL_AUTO
    var = {"rows_int": wq.WQ_GEMV_INT_DIGITS, "rows_half": wq.WQ_GEMV_OFFSET_SUMS,
           "tiled": wq.WQ_GEMV_OFFSET_SUMS, "tiled_exact": wq.WQ_GEMV_EXACT}[request.param]
    wq.wq_set_option(wq.WQ_OPT_GEMV_KERNEL, kern)
    wq.wq_set_option(wq.WQ_OPT_GEMV_VARIANT, var)
    yield request.param
    wq.wq_set_option(wq.WQ_OPT_GEMV_KERNEL, wq.WQ_GEMV_KERNEL_AUTO)
    wq.wq_set_option(wq.WQ_OPT_GEMV_VARIANT, wq.WQ_GEMV_OFFSET_SUMS)


def test_gemv_closed_forms(wq, gemv_variant):
    """All codes equal to the zero point -> Y == 0 up to the kernel's rounding
    bound; one nonzero code -> Y = x_k (q - zero) step."""
    N, K = 48, 1024
    g = np.random.default_rng(2)
    X = synth.activations(synth.rng(3), 1, K)
    zeros = g.integers(0, 16, (N, K // 128)).astype(np.float16)
    steps = g.uniform(0.001, 0.1, (N, K // 128)).astype(np.float16)
    bound = _gemv_error_bound(X, steps)
    codes = np.repeat(zeros.astype(np.uint8), 128, axis=1)
    packed = dev(O.pack_codes(codes, 4).reshape(-1).view(np.int32))
    Y = run_gemm(wq, X, (packed, dev(steps), dev(zeros)), N, 4)
    assert np.all(np.abs(Y.astype(np.float64)) <= bound)
    n, k = 21, 517
    codes[n, k] = (int(zeros[n, k // 128]) + 5) % 16
    packed = dev(O.pack_codes(codes, 4).reshape(-1).view(np.int32))
    Y = run_gemm(wq, X, (packed, dev(steps), dev(zeros)), N, 4).astype(np.float64)
    ref = O.gemm_ref(X, codes, steps, zeros, 128)
    others = np.delete(np.arange(N), n)
    assert np.all(np.abs(Y[:, others]) <= bound[:, others])
    assert abs(Y[0, n] - ref[0, n]) <= bound[0, n] + 2 ** -11 * abs(ref[0, n])


@pytest.mark.parametrize("bits", [3, 4])
def test_gemv_every_channel_position(wq, gemv_variant, bits):
    """Row n holds one code away from its zero point, at channel
    (n mod 32) + 224 (n div 32): every position of a 32-channel packing unit
    (and several units and groups) must map back to its own activation, so
    Y[n] = x_k (q - zero) step up to the kernel's rounding bound."""
    N, K = 64, 1024
    g = np.random.default_rng(31 + bits)
    Q = (1 << bits) - 1
    X = synth.activations(synth.rng(32), 1, K)
    zeros = g.integers(0, Q + 1, (N, K // 128)).astype(np.float16)
    steps = g.uniform(0.001, 0.1, (N, K // 128)).astype(np.float16)
    codes = np.repeat(zeros.astype(np.uint8), 128, axis=1)
    for n in range(N):
        k = (n % 32) + 224 * (n // 32)
        codes[n, k] = (int(zeros[n, k // 128]) + 1 + n % Q) % (Q + 1)
    packed = dev(O.pack_codes(codes, bits).reshape(-1).view(np.int32))
    Y = run_gemm(wq, X, (packed, dev(steps), dev(zeros)), N, bits).astype(np.float64)
    ref = O.gemm_ref(X, codes, steps, zeros, 128)
    bound = _gemv_error_bound(X, steps)
    assert np.all(np.abs(Y - ref) <= bound + 2 ** -11 * np.abs(ref)), np.max(np.abs(Y - ref) - bound)


def test_gemv_small_linear(wq):
    c = synth.config_small_linear(0)
    (codes, st, z), qg = assert_quant_parity(wq, c.W, None, 4, False)
    assert_close(run_gemm(wq, c.X, qg, 128, 4), O.gemm_ref(c.X, codes, st, z, 128))


def test_gemv_llama7b_block_full(wq):
    for c in synth.config_llama7b_decode(1):
        N = c.W.shape[0]
        (codes, st, z), qg = assert_quant_parity(wq, c.W, None, 4, False)
        assert_close(run_gemm(wq, c.X, qg, N, 4), O.gemm_ref(c.X, codes, st, z, 128))


@pytest.mark.parametrize("bits", [3, 4])
def test_gemv_llama65b_full(wq, gemv_variant, bits):
    c = synth.config_llama65b_decode(bits)
    (codes, st, z), qg = assert_quant_parity(wq, c.W, None, bits, False)
    assert_close(run_gemm(wq, c.X, qg, 8192, bits), O.gemm_ref(c.X, codes, st, z, 128))


def test_smallm_sweep_full_weight(wq):
    """K=8192, N=28672 at every M of the sweep, against the fp64 oracle; M >= 3
    both without a workspace (one CTA per row tile) and with one (the stream-K
    schedule: 224 row tiles for 148 SMs), the latter twice (same result)."""
    c = synth.config_smallm_sweep(1)
    (codes, st, z), qg = assert_quant_parity(wq, c.W, None, 4, False)
    D = O.dequantize(codes, st, z, 128)
    for M in synth.SMALLM_SWEEP:
        X = synth.smallm_activations(M)
        ref = X.astype(np.float64) @ D.T
        Y = run_gemm(wq, X, qg, 28672, 4)
        assert_close(Y, ref)
        if M >= 3:
            ws = gemm_workspace(wq, M, 28672, 8192, 4)
            Y1 = run_gemm(wq, X, qg, 28672, 4, workspace=ws)
            Y2 = run_gemm(wq, X, qg, 28672, 4, workspace=ws)
            assert_close(Y1, ref)
            assert np.array_equal(Y1.view(np.uint16), Y2.view(np.uint16))


# ---------------------------------------------------------------------------
# S6 tensor-core path (tcgen05), forced, 3- and 4-bit
# ---------------------------------------------------------------------------

@pytest.fixture
def tc_path(wq):
    wq.wq_set_option(wq.WQ_OPT_GEMM_PATH, wq.WQ_PATH_TENSOR_CORE)
    yield
    wq.wq_set_option(wq.WQ_OPT_GEMM_PATH, wq.WQ_PATH_AUTO)


@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("M", [1, 3, 16, 17, 48, 64, 100, 128, 200, 256, 300])
@pytest.mark.parametrize("NK", [(333, 1152), (1000, 4096)])
def test_tc_gemm_parity(wq, tc_path, bits, M, NK):
    N, K = NK
    g = synth.rng(500 + M + 10 * bits)
    W = synth.weight(g, N, K, 0.02, channel_frac=0.01, channel_mult=10.0)
    X = synth.activations(g, M, K, channel_frac=0.01, channel_mult=20.0)
    (codes, st, z), qg = assert_quant_parity(wq, W, None, bits, False)
    assert_close(run_gemm(wq, X, qg, N, bits), O.gemm_ref(X, codes, st, z, 128))


@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("S", [2, 3, 5, 16])
@pytest.mark.parametrize("M", [16, 128, 200])
def test_tc_gemm_ring_depths(wq, tc_path, bits, S, M):
    """Forced shared-memory ring depths (two CTAs per SM or one), including a
    ring deeper than the K loop (K = 1152 has 9 stages of 128 channels); a
    depth that one CTA's shared memory cannot hold is refused."""
    N, K = 333, 1152
    g = synth.rng(600 + M + S + bits)
    W = synth.weight(g, N, K, 0.02, channel_frac=0.01, channel_mult=10.0)
    X = synth.activations(g, M, K, channel_frac=0.01, channel_mult=20.0)
    (codes, st, z), qg = assert_quant_parity(wq, W, None, bits, False)
    wq.wq_set_option(wq.WQ_OPT_TC_STAGES, S)
    try:
        BN = (M + 15) // 16 * 16
        BK = 64 if BN >= 96 and bits == 4 else 128
        if S * ((BK // 64) * BN * 128 + 128 * BK * bits // 8) + 2048 > 220 * 1024:
            with pytest.raises(wq.WQError):
                run_gemm(wq, X, qg, N, bits)
            return
        Y = run_gemm(wq, X, qg, N, bits)
    finally:
        wq.wq_set_option(wq.WQ_OPT_TC_STAGES, 0)
    assert_close(Y, O.gemm_ref(X, codes, st, z, 128))


@pytest.mark.parametrize("sym", [False, True])
def test_tc_gemm_3bit_closed_forms_and_symmetric(wq, tc_path, sym):
    """3-bit tiles: all codes at the zero point give exactly 0; one nonzero
    code per row at every channel position of a 32-channel chunk (the three
    classes of the unpack and the two gathered high-bit channels) gives
    x_k (q - z) step; symmetric codes against the oracle."""
    N, K, M = 128, 512, 16
    X = synth.activations(synth.rng(24), M, K)
    zeros = np.full((N, K // 128), 4, np.float16)
    steps = np.random.default_rng(25).uniform(0.001, 0.1, (N, K // 128)).astype(np.float16)
    codes = np.full((N, K), 4, np.uint8)
    packed = dev(O.pack_codes(codes, 3).reshape(-1).view(np.int32))
    assert np.all(run_gemm(wq, X, (packed, dev(steps), dev(zeros)), N, 3) == 0)
    k_of = (np.arange(N) * 37) % K          # row n: one code at channel k_of[n]
    q = (np.arange(N) % 7 + (np.arange(N) % 7 >= 4)).astype(np.uint8)  # values 0..7 except 4
    codes[np.arange(N), k_of] = q
    packed = dev(O.pack_codes(codes, 3).reshape(-1).view(np.int32))
    Y = run_gemm(wq, X, (packed, dev(steps), dev(zeros)), N, 3).astype(np.float64)
    st = steps[np.arange(N), k_of // 128].astype(np.float64)
    ref = X[:, k_of].astype(np.float64) * ((q.astype(np.float64) - 4) * st)[None, :]
    assert np.all(np.abs(Y - ref) <= 2.0 ** -10 * np.abs(ref) + 2.0 ** -24)
    assert set((k_of % 32).tolist()) == set(range(32))
    W = synth.weight(synth.rng(26), 300, K, 0.02)
    Xs = synth.activations(synth.rng(27), 40, K)
    (codes, st, z), qg = assert_quant_parity(wq, W, None, 3, sym)
    assert_close(run_gemm(wq, Xs, qg, 300, 3, sym=sym), O.gemm_ref(Xs, codes, st, z, 128))


def test_smallm_sweep_3bit_full_weight(wq):
    """The LLaMA-65B-shaped 8192 x 8192 weight at 3 bits through the sweep's
    batch sizes (M >= 3 on the tensor cores), against the fp64 oracle."""
    c = synth.config_llama65b_decode(3)
    (codes, st, z), qg = assert_quant_parity(wq, c.W, None, 3, False)
    D = O.dequantize(codes, st, z, 128)
    for M in synth.SMALLM_SWEEP:
        X = synth.smallm_activations(M)
        assert_close(run_gemm(wq, X, qg, 8192, 3), X.astype(np.float64) @ D.T)


@pytest.mark.parametrize("dw", [4, 8])
@pytest.mark.parametrize("bk", [64, 128])
@pytest.mark.parametrize("M", [3, 16, 100, 128, 200, 300])
@pytest.mark.parametrize("NK", [(333, 1152), (1000, 4096)])
def test_tc_gemm_stage_width(wq, tc_path, dw, bk, M, NK):
    """Both stage widths (half a group and a whole group per stage) and both
    dequantizing-warp counts at every tile width, including two M chunks
    (M = 300)."""
    N, K = NK
    g = synth.rng(700 + M + bk)
    W = synth.weight(g, N, K, 0.02, channel_frac=0.01, channel_mult=10.0)
    X = synth.activations(g, M, K, channel_frac=0.01, channel_mult=20.0)
    (codes, st, z), qg = assert_quant_parity(wq, W, None, 4, False)
    wq.wq_set_option(wq.WQ_OPT_TC_BK, bk)
    wq.wq_set_option(wq.WQ_OPT_TC_DEQUANT_WARPS, dw)
    try:
        Y = run_gemm(wq, X, qg, N, 4)
    finally:
        wq.wq_set_option(wq.WQ_OPT_TC_BK, 0)
        wq.wq_set_option(wq.WQ_OPT_TC_DEQUANT_WARPS, 0)
    assert_close(Y, O.gemm_ref(X, codes, st, z, 128))


@pytest.mark.parametrize("dw", [4, 8])
@pytest.mark.parametrize("bits,group", [(3, 128), (3, 32), (4, 32), (4, 64)])
@pytest.mark.parametrize("M", [3, 40, 130])
def test_tc_gemm_dequant_quartets_bits_groups(wq, tc_path, dw, bits, group, M):
    """One and two dequantizing warp quartets (the second takes every other
    stage) for 3-bit tiles and groups smaller than a stage."""
    N, K = 333, 1152
    g = synth.rng(760 + M + bits + group)
    W = synth.weight(g, N, K, 0.02, channel_frac=0.01, channel_mult=10.0)
    X = synth.activations(g, M, K, channel_frac=0.01, channel_mult=20.0)
    codes, st, z = O.quantize_groups(W, bits, group, False)
    qg = (dev(O.pack_codes(codes, bits).reshape(-1).view(np.int32)), dev(st), dev(z))
    wq.wq_set_option(wq.WQ_OPT_TC_DEQUANT_WARPS, dw)
    try:
        Y = wq.wq_w4a16_gemm(dev(X), *qg, N, bits=bits, group_size=group).cpu().numpy()
        assert wq.wq_get_last_device_error() == 0
    finally:
        wq.wq_set_option(wq.WQ_OPT_TC_DEQUANT_WARPS, 0)
    assert_close(Y, O.gemm_ref(X, codes, st, z, group))


@pytest.fixture
def streamk_forced(wq):
    wq.wq_set_option(wq.WQ_OPT_TC_STREAMK, 2)
    yield
    wq.wq_set_option(wq.WQ_OPT_TC_STREAMK, 0)


@pytest.mark.parametrize("bits,group", [(4, 128), (3, 128), (4, 32), (3, 64)])
@pytest.mark.parametrize("M", [3, 16, 100, 200, 300])
@pytest.mark.parametrize("NK", [(333, 1152), (1000, 4096), (2000, 2048)])
def test_tc_gemm_streamk(wq, tc_path, streamk_forced, bits, group, M, NK):
    """The stream-K schedule forced on small weights: CTAs whose stage ranges
    start and end inside row tiles (one, two or three contributors per tile),
    a ragged last tile, two M chunks; the same result on a second call."""
    N, K = NK
    g = synth.rng(800 + M + bits + group + N)
    W = synth.weight(g, N, K, 0.02, channel_frac=0.01, channel_mult=10.0)
    X = synth.activations(g, M, K, channel_frac=0.01, channel_mult=20.0)
    codes, st, z = O.quantize_groups(W, bits, group, False)
    qg = (dev(O.pack_codes(codes, bits).reshape(-1).view(np.int32)), dev(st), dev(z))
    ws = gemm_workspace(wq, M, N, K, bits, group)
    Y1 = run_gemm(wq, X, qg, N, bits, group=group, workspace=ws)
    Y2 = run_gemm(wq, X, qg, N, bits, group=group, workspace=ws)
    assert_close(Y1, O.gemm_ref(X, codes, st, z, group))
    assert np.array_equal(Y1.view(np.uint16), Y2.view(np.uint16))
    assert int(ws[:65536].count_nonzero()) == 0  # the arrival counters are left at zero


def test_tc_gemm_streamk_workspace_shared_across_shapes(wq, tc_path, streamk_forced):
    """One zero-filled workspace serves calls of different shapes in turn: the
    arrival counters live in a fixed region that each call leaves at zero,
    away from the partial tiles of any shape."""
    g = synth.rng(870)
    shapes = [(16, 2000, 4096), (200, 333, 1152), (64, 4096, 2048), (16, 2000, 4096)]
    n = max(wq.wq_gemm_workspace_bytes(M, N, K) for M, N, K in shapes)
    ws = torch.zeros(n, dtype=torch.uint8, device="cuda")
    for M, N, K in shapes:
        W = synth.weight(g, N, K, 0.02)
        X = synth.activations(g, M, K)
        codes, st, z = O.quantize_groups(W, 4, 128, False)
        qg = (dev(O.pack_codes(codes, 4).reshape(-1).view(np.int32)), dev(st), dev(z))
        assert_close(run_gemm(wq, X, qg, N, 4, workspace=ws), O.gemm_ref(X, codes, st, z, 128))
        assert int(ws[:65536].count_nonzero()) == 0


def test_tc_gemm_workspace_rules(wq, tc_path):
    """A workspace smaller than wq_gemm_workspace_bytes is not used (the
    per-tile schedule runs); an unaligned one is refused; M < 3 needs none."""
    N, K, M = 1000, 4096, 16
    g = synth.rng(850)
    W = synth.weight(g, N, K, 0.02)
    X = synth.activations(g, M, K)
    codes, st, z = O.quantize_groups(W, 4, 128, False)
    qg = (dev(O.pack_codes(codes, 4).reshape(-1).view(np.int32)), dev(st), dev(z))
    assert wq.wq_gemm_workspace_bytes(2, N, K) == 0
    need = wq.wq_gemm_workspace_bytes(M, N, K)
    small = torch.zeros(need - 256, dtype=torch.uint8, device="cuda")
    wq.wq_set_option(wq.WQ_OPT_TC_STREAMK, 2)
    try:
        assert_close(run_gemm(wq, X, qg, N, 4, workspace=small), O.gemm_ref(X, codes, st, z, 128))
        big = torch.zeros(need + 512, dtype=torch.uint8, device="cuda")
        with pytest.raises(wq.WQError) as e:
            wq.wq_w4a16_gemm(dev(X), *qg, N, bits=4, workspace=big[1:])
        assert e.value.status == wq.WQ_ERR_ALIGNMENT
    finally:
        wq.wq_set_option(wq.WQ_OPT_TC_STREAMK, 0)


def test_tc_gemm_symmetric_and_closed_form(wq, tc_path):
    N, K, M = 256, 1024, 32
    g = np.random.default_rng(21)
    X = synth.activations(synth.rng(22), M, K)
    zeros = np.full((N, K // 128), 8, np.float16)
    steps = g.uniform(0.001, 0.1, (N, K // 128)).astype(np.float16)
    codes = np.full((N, K), 8, np.uint8)
    packed = dev(O.pack_codes(codes, 4).reshape(-1).view(np.int32))
    assert np.all(run_gemm(wq, X, (packed, dev(steps), dev(zeros)), N, 4, sym=True) == 0)
    W = synth.weight(synth.rng(23), N, K, 0.02)
    (codes, st, z), qg = assert_quant_parity(wq, W, None, 4, True)
    assert_close(run_gemm(wq, X, qg, N, 4, sym=True), O.gemm_ref(X, codes, st, z, 128))


def test_tc_matches_gemv_path(wq):
    """Both kernels on the same inputs agree with each other as well as the oracle."""
    N, K, M = 512, 2048, 24
    g = synth.rng(600)
    W = synth.weight(g, N, K, 0.02)
    X = synth.activations(g, M, K)
    (codes, st, z), qg = assert_quant_parity(wq, W, None, 4, False)
    ref = O.gemm_ref(X, codes, st, z, 128)
    outs = {}
    for path in (wq.WQ_PATH_GEMV, wq.WQ_PATH_TENSOR_CORE):
        wq.wq_set_option(wq.WQ_OPT_GEMM_PATH, path)
        try:
            outs[path] = run_gemm(wq, X, qg, N, 4)
        finally:
            wq.wq_set_option(wq.WQ_OPT_GEMM_PATH, wq.WQ_PATH_AUTO)
        assert_close(outs[path], ref)
    assert_close(outs[wq.WQ_PATH_TENSOR_CORE], outs[wq.WQ_PATH_GEMV].astype(np.float64))


@pytest.fixture
def rows_shape(wq):
    def set_shape(shape, variant):
        wq.wq_set_option(wq.WQ_OPT_GEMV_ROWS_SHAPE, shape)
        wq.wq_set_option(wq.WQ_OPT_GEMV_VARIANT, variant)
    yield set_shape
    wq.wq_set_option(wq.WQ_OPT_GEMV_ROWS_SHAPE, 0)
    wq.wq_set_option(wq.WQ_OPT_GEMV_VARIANT, wq.WQ_GEMV_OFFSET_SUMS)


@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("variant", ["int", "half"])
@pytest.mark.parametrize("shape", [1, 2, 3, 4])
@pytest.mark.parametrize("M", [1, 2])
@pytest.mark.parametrize("NK", [(333, 1152), (1000, 4096), (17, 11008), (130, 16384), (4099, 256)])
def test_gemv_rows_shapes(wq, rows_shape, bits, variant, shape, M, NK):
    """Every (rows per batch, channels per lane, register stages) shape of the
    row-streaming kernel with both ways of forming the lane sums, at 4 and 3
    bits (3-bit rows run shapes 2 and 3 with offset sums); ragged N,
    inactive lanes (K = 256 leaves most lanes of the single warp idle), K up
    to 16384, and CTAs with fewer row batches than stages (N = 17)."""
    N, K = NK
    g = synth.rng(800 + shape + M)
    W = synth.weight(g, N, K, 0.02, channel_frac=0.01, channel_mult=10.0)
    X = synth.activations(g, M, K, channel_frac=0.01, channel_mult=20.0)
    (codes, st, z), qg = assert_quant_parity(wq, W, None, bits, False)
    rows_shape(shape, wq.WQ_GEMV_INT_DIGITS if variant == "int" else wq.WQ_GEMV_OFFSET_SUMS)
    assert_close(run_gemm(wq, X, qg, N, bits), O.gemm_ref(X, codes, st, z, 128))


@pytest.mark.parametrize("shape", [2, 4])
@pytest.mark.parametrize("NK", [(333, 1152), (4096, 4096), (17, 11008), (4099, 256)])
def test_gemv_rows_grid_rule0(wq, rows_shape, shape, NK):
    """Grid rule 0 (one CTA per batch, or equal batches per CTA) against the oracle."""
    N, K = NK
    g = synth.rng(870 + shape)
    W = synth.weight(g, N, K, 0.02, channel_frac=0.01, channel_mult=10.0)
    X = synth.activations(g, 1, K, channel_frac=0.01, channel_mult=20.0)
    (codes, st, z), qg = assert_quant_parity(wq, W, None, 4, False)
    rows_shape(shape, wq.WQ_GEMV_OFFSET_SUMS)
    wq.wq_set_option(wq.WQ_OPT_GEMV_GRID, 0)
    try:
        Y = run_gemm(wq, X, qg, N, 4)
    finally:
        wq.wq_set_option(wq.WQ_OPT_GEMV_GRID, 1)
    assert_close(Y, O.gemm_ref(X, codes, st, z, 128))


@pytest.mark.parametrize("M", [1, 2])
def test_gemv_int_digits_error_bound(wq, rows_shape, M):
    """The integer-digit variant rounds only its fixed-point image of X (exact
    here for all but values below 2^-13 of a lane's largest), the fp32
    combination of each lane's digit sums, the fp32 sums across lanes and
    warps, and the fp16 output. So every output lies within half an fp16 ulp
    of the exact value plus 2^-20 of sum_k |x_k (q_k - zero) step|, far inside
    the offset-sum variant's 2^-8 step sum|x| per chunk."""
    N, K = 777, 4096
    g = synth.rng(900 + M)
    W = synth.weight(g, N, K, 0.02, channel_frac=0.01, channel_mult=10.0)
    X = synth.activations(g, M, K)
    (codes, st, z), qg = assert_quant_parity(wq, W, None, 4, False)
    rows_shape(0, wq.WQ_GEMV_INT_DIGITS)
    Y = run_gemm(wq, X, qg, N, 4).astype(np.float64)
    D = O.dequantize(codes, st, z, 128)
    ref = X.astype(np.float64) @ D.T
    mag = np.abs(X.astype(np.float64)) @ np.abs(D).T
    assert np.all(np.abs(Y - ref) <= 2.0 ** -11 * np.abs(ref) + 2.0 ** -20 * mag + 2.0 ** -24)


def test_gemv_int_digits_extreme_activations(wq, rows_shape):
    """fp16 extremes inside one lane's channels (65504, subnormals, zeros,
    mixed signs) and an all-zero lane: the per-lane exponent keeps every
    image in range, and all-zero X gives exactly zero."""
    N, K = 64, 1024
    g = synth.rng(950)
    W = synth.weight(g, N, K, 0.02)
    (codes, st, z), qg = assert_quant_parity(wq, W, None, 4, False)
    X = synth.activations(g, 2, K)
    X[0, :64] = 0
    X[0, 64] = 65504.0
    X[0, 65] = -65504.0
    X[0, 66:70] = np.float16(6e-8)
    X[0, 70] = np.float16(-2.0 ** -14)
    X[1, 128:192] = np.float16(-3e-5)
    X[1, 192] = 1000.0
    for variant in (wq.WQ_GEMV_INT_DIGITS, wq.WQ_GEMV_OFFSET_SUMS):
        rows_shape(0, variant)
        for M in (1, 2):
            Xm = X[:M] if M == 1 else X
            Y = run_gemm(wq, Xm, qg, N, 4)
            ref = O.gemm_ref(Xm, codes, st, z, 128)
            assert np.all(np.isfinite(Y))
            assert_close(Y, ref)
    rows_shape(0, wq.WQ_GEMV_INT_DIGITS)
    assert np.all(run_gemm(wq, np.zeros((1, K), np.float16), qg, N, 4) == 0)


@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("M", [1, 2, 5])
@pytest.mark.parametrize("NK", [(64, 32768), (333, 16512)])
def test_gemv_beyond_row_kernel_k(wq, bits, M, NK):
    """K above the row-streaming kernel's 16384 channels: the default dispatch
    sends M <= 2 to the tiled kernel (activations in shared memory, cluster
    split-K for few rows); M = 5 with 3 bits also takes the tiled kernel."""
    N, K = NK
    g = synth.rng(950 + M + bits)
    W = synth.weight(g, N, K, 0.02, channel_frac=0.01, channel_mult=10.0)
    X = synth.activations(g, M, K, channel_frac=0.01, channel_mult=20.0)
    (codes, st, z), qg = assert_quant_parity(wq, W, None, bits, False)
    assert_close(run_gemm(wq, X, qg, N, bits), O.gemm_ref(X, codes, st, z, 128))


# ---------------------------------------------------------------------------
# groups of 32 and 64 channels through the matmul (row-streaming GEMV for
# M <= 2 where its lanes hold whole groups, the tensor cores otherwise)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("group", [32, 64])
@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("M", [1, 2, 3, 16, 130])
@pytest.mark.parametrize("NK", [(333, 1152), (1000, 4096), (64, 11008)])
def test_gemm_small_groups(wq, group, bits, M, NK):
    N, K = NK
    g = synth.rng(1200 + M + bits + group)
    W = synth.weight(g, N, K, 0.02, channel_frac=0.01, channel_mult=10.0)
    X = synth.activations(g, M, K, channel_frac=0.01, channel_mult=20.0)
    (codes, st, z), qg = assert_quant_parity(wq, W, None, bits, False, group)
    assert_close(run_gemm(wq, X, qg, N, bits, group=group), O.gemm_ref(X, codes, st, z, group))


@pytest.mark.parametrize("group", [32, 64])
def test_gemm_small_groups_variants(wq, group):
    """Every row-kernel shape and both lane-sum variants at M = 1 and 2, the
    tensor-core kernel forced at M = 1 and with 64-channel stages, symmetric
    codes: all against the oracle."""
    N, K = 300, 2048
    g = synth.rng(1300 + group)
    W = synth.weight(g, N, K, 0.02, channel_frac=0.01, channel_mult=10.0)
    (codes, st, z), qg = assert_quant_parity(wq, W, None, 4, True, group)
    for M in (1, 2):
        X = synth.activations(g, M, K, channel_frac=0.01, channel_mult=20.0)
        ref = O.gemm_ref(X, codes, st, z, group)
        for shape in (1, 2, 3, 4):
            for variant in (wq.WQ_GEMV_OFFSET_SUMS, wq.WQ_GEMV_INT_DIGITS):
                wq.wq_set_option(wq.WQ_OPT_GEMV_ROWS_SHAPE, shape)
                wq.wq_set_option(wq.WQ_OPT_GEMV_VARIANT, variant)
                try:
                    assert_close(run_gemm(wq, X, qg, N, 4, sym=True, group=group), ref)
                finally:
                    wq.wq_set_option(wq.WQ_OPT_GEMV_ROWS_SHAPE, 0)
                    wq.wq_set_option(wq.WQ_OPT_GEMV_VARIANT, wq.WQ_GEMV_OFFSET_SUMS)
        wq.wq_set_option(wq.WQ_OPT_GEMM_PATH, wq.WQ_PATH_TENSOR_CORE)
        try:
            assert_close(run_gemm(wq, X, qg, N, 4, sym=True, group=group), ref)
        finally:
            wq.wq_set_option(wq.WQ_OPT_GEMM_PATH, wq.WQ_PATH_AUTO)
    X = synth.activations(g, 100, K)
    wq.wq_set_option(wq.WQ_OPT_TC_BK, 64)
    try:
        assert_close(run_gemm(wq, X, qg, N, 4, sym=True, group=group), O.gemm_ref(X, codes, st, z, group))
    finally:
        wq.wq_set_option(wq.WQ_OPT_TC_BK, 0)



@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("M,ks", [(3, 2), (3, 4), (3, 8), (16, 2), (16, 4), (16, 8), (64, 2), (100, 2), (128, 2)])
def test_tc_gemm_split_k(wq, tc_path, ks, bits, M):
    """K split over a cluster of 2, 4 or 8 CTAs per row tile (partial tiles
    added in rank order through distributed shared memory): ragged N, ranges
    that do not divide K evenly (K = 4224 has 33 stages of 128 channels), and
    groups of 128 or 32 channels. (Wider tiles with more CTAs do not fit their
    partial tiles in the first CTA's ring and are refused; see below.)"""
    N, K = 333, 4224
    g = synth.rng(1400 + ks + M + bits)
    W = synth.weight(g, N, K, 0.02, channel_frac=0.01, channel_mult=10.0)
    X = synth.activations(g, M, K, channel_frac=0.01, channel_mult=20.0)
    for group in (128, 32):
        (codes, st, z), qg = assert_quant_parity(wq, W, None, bits, False, group)
        wq.wq_set_option(wq.WQ_OPT_TC_KSPLIT, ks)
        try:
            Y = run_gemm(wq, X, qg, N, bits, group=group)
        finally:
            wq.wq_set_option(wq.WQ_OPT_TC_KSPLIT, 0)
        assert_close(Y, O.gemm_ref(X, codes, st, z, group))


def test_tc_gemm_split_k_refused_when_partials_do_not_fit(wq, tc_path):
    """A split whose partial tiles exceed the first CTA's ring is refused
    (WQ_ERR_CUDA), not run: M = 256 with a two-stage ring at 8 CTAs."""
    N, K, M = 256, 4096, 256
    g = synth.rng(1500)
    W = synth.weight(g, N, K, 0.02)
    (_, _, _), qg = assert_quant_parity(wq, W, None, 4, False)
    wq.wq_set_option(wq.WQ_OPT_TC_KSPLIT, 8)
    wq.wq_set_option(wq.WQ_OPT_TC_STAGES, 2)
    try:
        with pytest.raises(wq.WQError) as e:
            run_gemm(wq, synth.activations(g, M, K), qg, N, 4)
        assert e.value.status == wq.WQ_ERR_CUDA
    finally:
        wq.wq_set_option(wq.WQ_OPT_TC_KSPLIT, 0)
        wq.wq_set_option(wq.WQ_OPT_TC_STAGES, 0)


@pytest.mark.parametrize("group", [128, 64, 32])
@pytest.mark.parametrize("M", [3, 4])
@pytest.mark.parametrize("NK", [(333, 1152), (4096, 4096), (100, 8192)])
def test_gemv_rows_m3_m4(wq, group, M, NK):
    """The row-streaming kernel's M = 4 instance (M = 3 with a zero fourth row)
    forced for K <= 8192, against the oracle."""
    N, K = NK
    g = synth.rng(2300 + M + group + N)
    W = synth.weight(g, N, K, 0.02, channel_frac=0.01, channel_mult=10.0)
    X = synth.activations(g, M, K, channel_frac=0.01, channel_mult=20.0)
    (codes, st, z), qg = assert_quant_parity(wq, W, None, 4, False, group)
    wq.wq_set_option(wq.WQ_OPT_GEMM_PATH, wq.WQ_PATH_GEMV)
    try:
        Y = run_gemm(wq, X, qg, N, 4, group=group)
    finally:
        wq.wq_set_option(wq.WQ_OPT_GEMM_PATH, wq.WQ_PATH_AUTO)
    assert_close(Y, O.gemm_ref(X, codes, st, z, group))

