"""AWQ scale search on the GPU vs the CPU oracle, through the C ABI.

mu (activation statistic) and the candidate scales must match bit for bit
(a candidate may differ only where fp64 pow lands within 1e-12 of an fp16
rounding midpoint -- flagged, never seen); losses must agree to 1e-4 relative
(the GPU loss GEMM runs on the tensor cores with the error matrix in fp16 and
fp32 accumulation); the chosen alpha must be the oracle's unless the oracle's
two best losses are within that tolerance of each other; the output scale is
the chosen candidate bit for bit, and packing with it matches the oracle.
"""
import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

LOSS_RTOL = 1e-4


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
    rel = np.abs(losses - ref["losses"]) / ref["losses"]
    assert np.all(rel <= LOSS_RTOL), (path, rel)
    best = int(out["best"].cpu().numpy()[0])
    order = np.argsort(ref["losses"], kind="stable")
    if best != ref["best"]:
        gap = (ref["losses"][order[1]] - ref["losses"][order[0]]) / ref["losses"][order[0]]
        assert gap < LOSS_RTOL and best == order[1], ("alpha differs", path, best, ref["best"], gap)
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
    assert abs(L - ref) <= LOSS_RTOL * ref


@pytest.mark.parametrize("T", [1, 511, 512, 513, 1100])
def test_awq_fused_token_chunks(wq, T):
    """The fused kernel covers 512 tokens per CTA: one token, a ragged chunk,
    exactly one chunk, and several chunks give the same losses as the oracle
    and as the two-kernel path (rows and tokens past the end read as zeros)."""
    g = synth.rng(703 + T)
    X = synth.activations(g, T, 384, channel_frac=0.02, channel_mult=20.0)
    Ws = [synth.weight(g, 130, 384, 0.02), synth.weight(g, 3, 384, 0.02)]
    check_search(wq, X, Ws, 4, False, alphas=[0.0, 0.3, 0.6])


def test_awq_block_o_and_down_full(wq):
    """Two of the four search places of a LLaMA-2-7B block at full size
    (T=512; o: K=4096,N=4096; down: K=11008,N=4096)."""
    groups = synth.config_awq_block(5)
    for name, X, named in groups:
        if name not in ("o", "down"):
            continue
        ref, losses, best, rel = check_search(wq, X, [W for _, W in named])
        print(name, "best", best, "max rel loss err", float(rel.max()))


def test_awq_block_qkv_gateup_rows(wq):
    """The other two places with the first 1024 rows of each linear (full K, T)."""
    groups = synth.config_awq_block(5)
    for name, X, named in groups:
        if name not in ("qkv", "gate_up"):
            continue
        check_search(wq, X, [W[:1024] for _, W in named])


def test_workspace_errors(wq):
    X = torch.zeros((8, 256), dtype=torch.float16, device="cuda")
    W = torch.zeros((16, 256), dtype=torch.float16, device="cuda")
    need = wq.wq_awq_workspace_bytes(8, 256, [16], 20)
    assert need > 0
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(wq.WQError) as e:
        wq.wq_awq_scale_search(X, [W], workspace=small)
    assert e.value.status == wq.WQ_ERR_WORKSPACE
