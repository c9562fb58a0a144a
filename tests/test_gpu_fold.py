"""AWQ scale folding on the GPU vs the oracle, bit for bit, through the C ABI
("MIT 6.5940 Lab 4 + Lab 5", "Question 2": the searched scales are folded
into the previous norm or linear layer)."""
import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wq():
    from weight_only_quantization_group_b200 import build
    build.build()
    import weight_only_quantization_group_b200 as m
    assert torch.cuda.is_available()
    return m


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _bits(t):
    return t.cpu().numpy().view(np.uint16)


def _awq_like_scales(n, seed):
    """Candidate scales as the search makes them: fp16(mu^alpha) of outlier-
    heavy activation means, at a spread of alphas."""
    X = synth.activations(synth.rng(seed), 64, n, channel_frac=0.01, channel_mult=20.0)
    mu = O.activation_absmean(X)
    S = O.awq_candidates(mu, O.awq_alpha_grid(20))
    return S[np.arange(n) % 20, np.arange(n)]


@pytest.mark.parametrize("K", [4096, 11008, 4099, 8, 1])
def test_fold_norm_bit_exact(wq, K):
    g = np.random.default_rng(K)
    gam = (1.0 + 0.3 * g.standard_normal(K)).astype(np.float16)
    s = _awq_like_scales(K, K + 1)
    out = wq.wq_awq_fold_norm(dev(gam), dev(s))
    assert wq.wq_get_last_device_error() == 0
    assert np.array_equal(_bits(out), O.awq_fold_into_norm(gam, s).view(np.uint16))


@pytest.mark.parametrize("N,K,bias", [(4096, 4096, False), (11008, 4096, True), (333, 136, True), (17, 100, False),
                                      (5, 3, True)])
def test_fold_linear_rows_bit_exact(wq, N, K, bias):
    g = np.random.default_rng(N * 7 + K)
    W = synth.weight(g, N, K, 0.02)
    b = (0.02 * g.standard_normal(N)).astype(np.float16) if bias else None
    s = _awq_like_scales(N, N + K)
    Wf, bf = wq.wq_awq_fold_linear_rows(dev(W), dev(s), None if b is None else dev(b))
    assert wq.wq_get_last_device_error() == 0
    rW, rb = O.awq_fold_into_linear_rows(W, s, b)
    assert np.array_equal(_bits(Wf), rW.view(np.uint16))
    if bias:
        assert np.array_equal(_bits(bf), rb.view(np.uint16))
    else:
        assert bf is None


def test_fold_in_place_and_unaligned_views(wq):
    """Outputs may be the inputs; a view one element into a buffer takes the
    scalar path and gives the same bits."""
    g = np.random.default_rng(5)
    W = synth.weight(g, 64, 256, 0.02)
    s = _awq_like_scales(64, 6)
    Wd = dev(W)
    wq.wq_awq_fold_linear_rows(Wd, dev(s), out=(Wd, None))
    assert np.array_equal(_bits(Wd), O.awq_fold_into_linear_rows(W, s)[0].view(np.uint16))
    gam = (1.0 + 0.3 * g.standard_normal(513)).astype(np.float16)
    sk = _awq_like_scales(513, 7)
    buf = dev(np.concatenate([[np.float16(0)], gam]))
    sbuf = dev(np.concatenate([[np.float16(1)], sk]))
    view, sview = buf[1:], sbuf[1:]
    wq.wq_awq_fold_norm(view, sview, out=view)
    assert wq.wq_get_last_device_error() == 0
    assert np.array_equal(_bits(view), O.awq_fold_into_norm(gam, sk).view(np.uint16))
    assert _bits(buf)[0] == 0  # the element before the view is untouched


def test_fold_overflow_latches_range(wq):
    """A quotient beyond fp16 (a large weight over a tiny scale) latches
    WQ_ERR_RANGE; the other elements are still exact."""
    gam = np.array([60000.0, 1.0, 2.0, 3.0] * 4, dtype=np.float16)
    s = np.array([2.0 ** -4, 2.0, 4.0, 8.0] * 4, dtype=np.float16)
    out = wq.wq_awq_fold_norm(dev(gam), dev(s))
    assert wq.wq_get_last_device_error() == wq.WQ_ERR_RANGE
    assert wq.wq_get_last_device_error() == 0  # read clears it
    ref = O.awq_fold_into_norm(gam, s)
    fin = np.isfinite(ref.astype(np.float32))
    assert np.array_equal(_bits(out)[fin], ref.view(np.uint16)[fin])


def test_folded_block_matches_unfolded_on_gpu_fold(wq):
    """The four folds of a small LLaMA-shaped block done by the library (fp16
    storage), the scaled weights W diag(s) formed exactly in fp64: the block's
    output stays within the fp16 rounding of the folded parameters."""
    g = np.random.default_rng(41)
    D, H = 128, 256
    p = {"gamma1": (1.0 + 0.1 * g.standard_normal(D)).astype(np.float16),
         "gamma2": (1.0 + 0.1 * g.standard_normal(D)).astype(np.float16)}
    for name, shape in (("wq", (D, D)), ("wk", (D, D)), ("wv", (D, D)), ("wo", (D, D)), ("wg", (H, D)),
                        ("wu", (H, D)), ("wd", (D, H))):
        p[name] = synth.weight(g, *shape, 0.08)
    s = [_awq_like_scales(n, 50 + i) for i, n in enumerate((D, D, D, H))]
    x = synth.activations(g, 6, D).astype(np.float64)
    y = O.decoder_block_ref(x, p, 4)
    f = {k: v.astype(np.float64) for k, v in p.items()}
    s64 = [t.astype(np.float64) for t in s]
    f["gamma1"] = wq.wq_awq_fold_norm(dev(p["gamma1"]), dev(s[0])).cpu().numpy().astype(np.float64)
    f["gamma2"] = wq.wq_awq_fold_norm(dev(p["gamma2"]), dev(s[2])).cpu().numpy().astype(np.float64)
    for n in ("wq", "wk", "wv"):
        f[n] = f[n] * s64[0][None, :]
    # v_proj: scaled by s_qkv on its input, its rows folded by s_o (fp16 storage of W_v / s_o)
    wv_rows = wq.wq_awq_fold_linear_rows(dev(p["wv"]), dev(s[1]))[0].cpu().numpy().astype(np.float64)
    f["wv"] = wv_rows * s64[0][None, :]
    f["wo"] = f["wo"] * s64[1][None, :]
    f["wg"] = f["wg"] * s64[2][None, :]
    wu_rows = wq.wq_awq_fold_linear_rows(dev(p["wu"]), dev(s[3]))[0].cpu().numpy().astype(np.float64)
    f["wu"] = wu_rows * s64[2][None, :]
    f["wd"] = f["wd"] * s64[3][None, :]
    assert wq.wq_get_last_device_error() == 0
    yf = O.decoder_block_ref(x, f, 4)
    rel = np.linalg.norm(yf - y) / np.linalg.norm(y)
    assert rel <= 2e-3, rel  # fp16 storage: 2^-11 relative per folded parameter
