"""GPTQ on the GPU (fp64, through the C ABI) against the fp64 oracle
("CMU 11-868 L19-L20 Model Quantization", "The algorithm in four steps").

Both sides run the same sequence of decisions on fp64 running weights; only
the order of floating-point sums differs (the Hessian, the factorizations,
the batched updates). A code changes only where that difference moves a
running weight across an fp32 rounding boundary of its quotient, and then the
error feedback carries the change along that row. So the checks are: steps
and zeros equal in at least 99 % of the rows that have no changed code,
codes equal in at least 99.9 % of all places, and the layer loss
||X (W - W^)^T||^2 within 1e-4 relative of the oracle's. Where the method
reduces to round to nearest (orthogonal input channels) the result must be
bit-exact.
"""
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
    return m


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _loss(X, W, codes, st, z, group):
    E = W.astype(np.float64) - O.dequantize(codes, st, z, group)
    P = X.astype(np.float64) @ E.T
    return float(np.sum(P * P))


def _gpu_gptq(wq, W, X, bits, group, sym):
    packed, steps, zeros = wq.wq_gptq_quantize_pack(dev(W), dev(X), bits=bits, group_size=group, symmetric=sym)
    assert wq.wq_get_last_device_error() == 0
    codes = O.unpack_codes(packed.cpu().numpy().view(np.uint32).reshape(W.shape[0], -1), bits, W.shape[1])
    return codes, steps.cpu().numpy(), zeros.cpu().numpy()


def _correlated_inputs(g, T, K, rank=32):
    base = g.standard_normal((T, rank)) @ g.standard_normal((rank, K))
    return (base / np.sqrt(rank) + 0.3 * g.standard_normal((T, K))).astype(np.float16)


def check_against_oracle(wq, W, X, bits, group, sym):
    ref = O.gptq_quantize(W, X, bits, group, sym)
    got = _gpu_gptq(wq, W, X, bits, group, sym)
    same_codes = got[0] == ref[0]
    assert same_codes.mean() >= 0.999, same_codes.mean()
    clean = same_codes.all(axis=1)
    assert clean.mean() >= 0.99, clean.mean()
    assert np.array_equal(got[1][clean].view(np.uint16), ref[1][clean].view(np.uint16))
    assert np.array_equal(got[2][clean].view(np.uint16), ref[2][clean].view(np.uint16))
    Lg, Lr = _loss(X, W, *got, group), _loss(X, W, *ref, group)
    assert abs(Lg - Lr) <= 1e-4 * Lr, (Lg, Lr)
    Lrtn = _loss(X, W, *O.quantize_groups(W, bits, group, sym), group)
    return Lg, Lrtn, float(same_codes.mean())


@pytest.mark.parametrize("bits", [3, 4])
@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("group", [128, 64, 32])
def test_gptq_matches_oracle_small(wq, bits, sym, group):
    g = synth.rng(1600 + bits + group)
    N, K, T = 333, 1152, 200
    W = synth.weight(g, N, K, 0.02, channel_frac=0.01, channel_mult=10.0)
    X = _correlated_inputs(g, T, K)
    Lg, Lrtn, same = check_against_oracle(wq, W, X, bits, group, sym)
    assert Lg < Lrtn  # error feedback pays on correlated inputs


def test_gptq_matches_oracle_llama_shape(wq):
    """One 1024-row slice of a LLaMA-2-7B q_proj (K = 4096) with 512
    calibration tokens with outlier channels, 4-bit asymmetric, group 128."""
    g = synth.rng(1700)
    W = synth.weight(g, 1024, 4096, 0.02)
    X = synth.activations(g, 512, 4096, channel_frac=0.01, channel_mult=20.0)
    Lg, Lrtn, same = check_against_oracle(wq, W, X, 4, 128, False)
    print("gptq loss", Lg, "rtn loss", Lrtn, "codes equal", same)


def test_gptq_is_rtn_for_orthogonal_inputs(wq):
    """Orthogonal input channels make H diagonal, so no error is passed on:
    the result equals wq_quantize_pack bit for bit."""
    g = synth.rng(1800)
    K, N = 512, 77
    X = np.zeros((K, K), np.float16)
    X[np.arange(K), np.arange(K)] = (1.0 + g.random(K)).astype(np.float16)
    W = synth.weight(g, N, K, 0.02)
    for bits, sym, group in ((4, False, 128), (3, True, 64), (4, True, 32)):
        p1, s1, z1 = wq.wq_gptq_quantize_pack(dev(W), dev(X), bits=bits, group_size=group, symmetric=sym)
        p2, s2, z2 = wq.wq_quantize_pack(dev(W), bits=bits, group_size=group, symmetric=sym)
        assert wq.wq_get_last_device_error() == 0
        assert torch.equal(p1, p2) and torch.equal(s1.view(torch.int16), s2.view(torch.int16))
        assert torch.equal(z1.view(torch.int16), z2.view(torch.int16))


def test_gptq_dead_channel_and_matmul(wq):
    """An input channel that is zero on every token quantizes to zero weights;
    the GPTQ-packed weight feeds the matmul like any other."""
    g = synth.rng(1900)
    N, K, T = 256, 1024, 128
    W = synth.weight(g, N, K, 0.02)
    X = _correlated_inputs(g, T, K)
    X[:, 300] = 0
    packed, steps, zeros = wq.wq_gptq_quantize_pack(dev(W), dev(X))
    assert wq.wq_get_last_device_error() == 0
    codes = O.unpack_codes(packed.cpu().numpy().view(np.uint32).reshape(N, -1), 4, K)
    D = O.dequantize(codes, steps.cpu().numpy(), zeros.cpu().numpy(), 128)
    assert np.all(D[:, 300] == 0)
    for M in (1, 16):
        Xm = synth.activations(g, M, K)
        Y = wq.wq_w4a16_gemm(dev(Xm), packed, steps, zeros, N).cpu().numpy().astype(np.float64)
        ref = Xm.astype(np.float64) @ D.T
        assert np.linalg.norm(Y - ref) / np.linalg.norm(ref) <= 1e-3


def test_gptq_workspace_errors(wq):
    W = torch.zeros((64, 256), dtype=torch.float16, device="cuda")
    X = torch.zeros((8, 256), dtype=torch.float16, device="cuda")
    need = wq.wq_gptq_workspace_bytes(64, 256)
    assert need >= 2 * 256 * 256 * 8 + 64 * 256 * 8
    with pytest.raises(wq.WQError) as e:
        wq.wq_gptq_quantize_pack(W, X, workspace=torch.empty(need - 256, dtype=torch.uint8, device="cuda"))
    assert e.value.status == wq.WQ_ERR_WORKSPACE
