"""AWQ scale search on the GPU vs the CPU oracle, through the C ABI.

mu (activation statistic) and the candidate scales must match bit for bit
(a candidate may differ only where fp64 pow lands within 1e-12 of an fp16
rounding midpoint -- flagged, never seen).

Losses: the loss GEMM multiplies the fp16 error matrix by X on the tensor
cores with fp32 accumulation, and that accumulator rounds toward zero: every
16-channel step of K loses up to an ulp of the running sum, so the GPU
losses come out low by a nearly alpha-independent factor that grows with K
(measured on the LLaMA-2-7B block: -7e-6 to -9e-6 at K = 4096, -2.4e-5 at
K = 11008); the fp16 rounding of E adds a zero-mean part. Bound used:
LOSS_RTOL = 1e-4 (2 * (K / 16) * 2^-24 = 1.3e-4 at K = 11008 if every step
lost a whole ulp of |D|).

alpha: what decides it is the alpha-dependent part of the error, measured
below 3e-6 relative at full size; the chosen alpha must be the oracle's
unless the oracle's two best losses are within ALPHA_TIE = 1e-5 of each
other (then the runner-up is accepted). The output scale is the chosen
candidate bit for bit, and packing with it matches the oracle.
"""
import hashlib
import json
import os

import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")

LOSS_RTOL = 1e-4
ALPHA_TIE = 1e-5
LOSS_TOL = {"two_kernels": (LOSS_RTOL, ALPHA_TIE), "fused": (LOSS_RTOL, ALPHA_TIE)}


@pytest.fixture(scope="module")
def wq():
    from weight_only_quantization_group_b200 import build
    build.build()
    import weight_only_quantization_group_b200 as m
    return m


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _near_f16_midpoint(v):
    h = v.astype(np.float16).astype(np.float64)
    up = np.nextafter(v.astype(np.float16), np.float16(np.inf)).astype(np.float64)
    dn = np.nextafter(v.astype(np.float16), np.float16(-np.inf)).astype(np.float64)
    mids = np.stack([(h + up) / 2, (h + dn) / 2])
    return np.any(np.abs(mids - v[None]) <= 1e-12 * np.abs(v[None]), axis=0)


LOSS_PATHS = ("two_kernels", "fused")


def check_search(wq, X, Ws, bits=4, sym=False, alphas=None):
    """Both ways of forming the losses (the error matrix in global memory, or
    built inside the loss GEMM) against one oracle search."""
    alphas = O.awq_alpha_grid(20) if alphas is None else np.asarray(alphas, np.float64)
    ref = O.awq_search(X, Ws, bits, 128, sym, alphas)
    res = None
    for path in LOSS_PATHS:
        r = _check_one(wq, X, Ws, bits, sym, alphas, ref, path)
        res = res or r
    return res


def _check_one(wq, X, Ws, bits, sym, alphas, ref, path):
    old = wq.wq_get_option(wq.WQ_OPT_AWQ_LOSS)
    wq.wq_set_option(wq.WQ_OPT_AWQ_LOSS,
                     wq.WQ_AWQ_LOSS_FUSED if path == "fused" else wq.WQ_AWQ_LOSS_TWO_KERNELS)
    try:
        out = wq.wq_awq_scale_search(dev(X), [dev(W) for W in Ws], list(alphas), bits=bits, symmetric=sym)
        assert wq.wq_get_last_device_error() == 0, path
    finally:
        wq.wq_set_option(wq.WQ_OPT_AWQ_LOSS, old)
    mu = out["mu"].cpu().numpy()
    assert np.array_equal(mu, ref["mu"]), "activation statistic differs"
    losses = out["losses"].cpu().numpy()
    rtol, tie = LOSS_TOL[path]
    rel = np.abs(losses - ref["losses"]) / ref["losses"]
    assert np.all(rel <= rtol), (path, rel)
    best = int(out["best"].cpu().numpy()[0])
    order = np.argsort(ref["losses"], kind="stable")
    if best != ref["best"]:
        gap = (ref["losses"][order[1]] - ref["losses"][order[0]]) / ref["losses"][order[0]]
        assert gap < tie and best == order[1], ("alpha differs", path, best, ref["best"], gap)
    s = out["s"].cpu().numpy()
    cand = O.awq_candidates(ref["mu"], alphas)[best]
    diff = s.view(np.uint16) != cand.view(np.uint16)
    if np.any(diff):
        m = np.maximum(ref["mu"], O.MU_FLOOR)[diff]
        assert np.all(_near_f16_midpoint(np.power(m, alphas[best]))), "candidate scales differ"
    # then pack with the chosen scale
    for W in Ws:
        packed, steps, zeros = wq.wq_quantize_pack(dev(W), dev(s), bits=bits, symmetric=sym)
        codes, st, z = O.quantize_groups(W, bits, 128, sym, s16=s)
        assert np.array_equal(packed.cpu().numpy().view(np.uint32), O.pack_codes(codes, bits).reshape(-1))
        assert np.array_equal(steps.cpu().numpy().view(np.uint16), st.view(np.uint16))
    return ref, losses, best, rel


@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("sym", [False, True])
def test_awq_search_small(wq, bits, sym):
    g = synth.rng(700 + bits)
    X = synth.activations(g, 72, 384, channel_frac=0.02, channel_mult=20.0)
    Ws = [synth.weight(g, 96, 384, 0.02), synth.weight(g, 200, 384, 0.02)]
    ref, losses, best, rel = check_search(wq, X, Ws, bits, sym)
    assert ref["losses"][ref["best"]] < ref["losses"][0]


def test_awq_search_ragged_and_zero_channel(wq):
    g = synth.rng(701)
    X = synth.activations(g, 131, 640, channel_frac=0.01, channel_mult=20.0)
    X[:, 5] = 0                         # an all-zero calibration channel -> mu floor
    Ws = [synth.weight(g, 1, 640, 0.02), synth.weight(g, 129, 640, 0.02), synth.weight(g, 7, 640, 0.02)]
    check_search(wq, X, Ws, 4, False, alphas=[0.0, 0.1, 0.25, 0.5, 0.8, 1.0])


@pytest.mark.parametrize("path", LOSS_PATHS)
def test_awq_alpha_zero_only_equals_rtn(wq, path):
    g = synth.rng(702)
    X = synth.activations(g, 40, 256)
    W = synth.weight(g, 64, 256, 0.02)
    old = wq.wq_get_option(wq.WQ_OPT_AWQ_LOSS)
    wq.wq_set_option(wq.WQ_OPT_AWQ_LOSS, wq.WQ_AWQ_LOSS_FUSED if path == "fused" else wq.WQ_AWQ_LOSS_TWO_KERNELS)
    try:
        out = wq.wq_awq_scale_search(dev(X), [dev(W)], [0.0])
    finally:
        wq.wq_set_option(wq.WQ_OPT_AWQ_LOSS, old)
    assert wq.wq_get_last_device_error() == 0
    assert np.all(out["s"].cpu().numpy() == 1.0)
    L = float(out["losses"].cpu().numpy()[0])
    ref = O.awq_loss(X, [W], np.ones(256, np.float16), 4, 128, False)
    assert abs(L - ref) <= LOSS_TOL[path][0] * ref


@pytest.mark.parametrize("T", [1, 511, 512, 513, 1100])
def test_awq_fused_token_chunks(wq, T):
    """The fused kernel covers 512 tokens per CTA: one token, a ragged chunk,
    exactly one chunk, and several chunks give the same losses as the oracle
    and as the two-kernel path (rows and tokens past the end read as zeros)."""
    g = synth.rng(703 + T)
    X = synth.activations(g, T, 384, channel_frac=0.02, channel_mult=20.0)
    Ws = [synth.weight(g, 130, 384, 0.02), synth.weight(g, 3, 384, 0.02)]
    check_search(wq, X, Ws, 4, False, alphas=[0.0, 0.3, 0.6])


def test_awq_block_o_and_down_full_both_paths(wq):
    """Two of the four search places of a LLaMA-2-7B block at full size
    (T=512; o: K=4096,N=4096; down: K=11008,N=4096), both loss paths against
    the oracle computed here."""
    groups = synth.config_awq_block(5)
    for name, X, named in groups:
        if name not in ("o", "down"):
            continue
        ref, losses, best, rel = check_search(wq, X, [W for _, W in named])
        print(name, "best", best, "max rel loss err", float(rel.max()))


def _digest(a):
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


@pytest.mark.parametrize("bits", [4, 3])
def test_awq_block_all_places_full_size(wq, bits):
    """All four search places of a LLaMA-2-7B-shaped block at full size (q|k|v
    N=12288, o, gate|up N=22016, down K=11008; T=512; 20 alphas) on the
    default (fused) path, against the oracle's search stored by
    tests/golden/make_awq_block_golden.py: mu and the chosen s bit for bit
    (SHA-256 of their bytes), the losses within LOSS_RTOL, alpha equal
    unless the oracle's two best are within ALPHA_TIE, and the alpha-dependent
    part of the loss error (its spread over the 20 alphas) below ALPHA_TIE / 2.
    Then the weights are packed with s and run through the decode GEMV
    against the oracle."""
    with open(os.path.join(GOLDEN, f"awq_llama7b_block_w{bits}_oracle.json")) as f:
        gold = json.load(f)
    worst = 0.0
    for name, X, named in synth.config_awq_block(5):
        g = gold["places"][name]
        Ws = [W for _, W in named]
        out = wq.wq_awq_scale_search(dev(X), [dev(W) for W in Ws], bits=bits)
        assert wq.wq_get_last_device_error() == 0
        assert _digest(out["mu"].cpu().numpy()) == g["mu_sha256"], name
        ref = np.array([float.fromhex(h) for h in g["losses_hex"]])
        losses = out["losses"].cpu().numpy()
        rel = np.abs(losses - ref) / ref
        worst = max(worst, float(rel.max()))
        assert np.all(rel <= LOSS_RTOL), (name, rel.max())
        signed = (losses - ref) / ref
        assert signed.max() - signed.min() <= ALPHA_TIE / 2, (name, signed.min(), signed.max())
        best = int(out["best"].item())
        if best != g["best"]:
            assert g["gap12"] < ALPHA_TIE, (name, best, g["best"], g["gap12"])
        else:
            assert _digest(out["s"].cpu().numpy().view(np.uint16)) == g["s_sha256"], name
        # the chosen scale drives the packing and the decode matmul: X diag(s)^-1
        # against the oracle's fp64 matmul of the dequantized weight
        s = out["s"].cpu().numpy()
        W = Ws[0]
        codes, st, z = O.quantize_groups(W, bits, 128, False, s16=s)
        packed, steps, zeros = wq.wq_quantize_pack(dev(W), dev(s), bits=bits)
        assert np.array_equal(packed.cpu().numpy().view(np.uint32), O.pack_codes(codes, bits).reshape(-1))
        xs = (X[:1].astype(np.float32) / s.astype(np.float32)).astype(np.float16)
        y = wq.wq_w4a16_gemm(dev(xs), packed, steps, zeros, W.shape[0], bits=bits).cpu().numpy()
        yref = O.gemm_ref(xs, codes, st, z, 128)
        assert np.linalg.norm(y - yref) / np.linalg.norm(yref) <= 1e-3, name
    print(f"{bits}-bit block: worst relative loss error {worst:.3g}")


def test_workspace_errors(wq):
    X = torch.zeros((8, 256), dtype=torch.float16, device="cuda")
    W = torch.zeros((16, 256), dtype=torch.float16, device="cuda")
    need = wq.wq_awq_workspace_bytes(8, 256, [16], 20)
    assert need > 0
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(wq.WQError) as e:
        wq.wq_awq_scale_search(X, [W], workspace=small)
    assert e.value.status == wq.WQ_ERR_WORKSPACE
