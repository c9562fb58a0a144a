"""W4A8 on the GPU against the oracle, through the C ABI ("MIT 6.5940 Lab 4 +
Lab 5": the Lab 5 linear, 4-bit weights and 8-bit activations with group size
32; the int8 absmax of "CMU 11-868 L19-L20", "absmax and zero-point").

Activation codes and multipliers are bit-exact (same fp32 operations); the
matmul's group sums are exact integers on both sides, so Y differs from the
oracle's fp64 sum only by fp32 scaling and summation and the fp16 output:
rel L2 <= 1e-3 and max abs <= 1e-2 * max|y| (the W4A16 tolerance), and
within 2^-10 relative plus 2^-20 of the sum of |terms| per output.
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


@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("M", [1, 3, 4, 9])
def test_act_int8_bit_exact(wq, group, M):
    g = synth.rng(2000 + M + group)
    X = synth.activations(g, M, 4096, channel_frac=0.01, channel_mult=20.0)
    X[0, :group] = 0                                   # an all-zero group: multiplier 1
    X[-1, group:2 * group] = np.float16(65504.0)        # the fp16 maximum
    q, mult = wq.wq_quantize_act_int8(dev(X), group_size=group)
    rq, rm = O.act_quantize_int8_groups(X, group)
    assert np.array_equal(q.cpu().numpy(), rq)
    assert np.array_equal(mult.cpu().numpy().view(np.uint32), rm.view(np.uint32))


@pytest.mark.parametrize("group", [32, 64, 128])
@pytest.mark.parametrize("sym", [False, True])
@pytest.mark.parametrize("M", [1, 2, 5])
@pytest.mark.parametrize("NK", [(333, 1152), (1000, 4096), (77, 11008)])
def test_w4a8_gemm_matches_oracle(wq, group, sym, M, NK):
    N, K = NK
    g = synth.rng(2100 + M + group + N)
    W = synth.weight(g, N, K, 0.02, channel_frac=0.01, channel_mult=10.0)
    X = synth.activations(g, M, K, channel_frac=0.01, channel_mult=20.0)
    codes, st, z = O.quantize_groups(W, 4, group, sym)
    packed, steps, zeros = wq.wq_quantize_pack(dev(W), bits=4, group_size=group, symmetric=sym)
    q, mult = wq.wq_quantize_act_int8(dev(X), group_size=group)
    Y = wq.wq_w4a8_gemm(q, mult, packed, steps, zeros, N, group_size=group, symmetric=sym)
    assert wq.wq_get_last_device_error() == 0
    rq, rm = O.act_quantize_int8_groups(X, group)
    ref = O.w4a8_gemm_ref(rq, rm, codes, st, z, group)
    y = Y.cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert rel <= 1e-3 and np.max(np.abs(y - ref)) <= 1e-2 * np.max(np.abs(ref)), rel
    G = K // group
    qw = np.abs(codes.astype(np.float64).reshape(N, G, group) - z.astype(np.float64)[:, :, None])
    qa = np.abs(rq.astype(np.float64).reshape(M, G, group))
    mag = np.einsum("mgk,ngk,ng,mg->mn", qa, qw, st.astype(np.float64), 1.0 / rm.astype(np.float64))
    assert np.all(np.abs(y - ref) <= 2.0 ** -10 * np.abs(ref) + 2.0 ** -20 * mag + 2.0 ** -24)


def test_w4a8_close_to_w4a16(wq):
    """Lab 5's W4A8 is an approximation of the W4A16 matmul: on the 8192 x 8192
    LLaMA-65B shape the int8 activations move Y by about 1 % (relative L2),
    the size of the per-group int8 rounding of X."""
    c = synth.config_llama65b_decode(4)
    packed, steps, zeros = wq.wq_quantize_pack(dev(c.W), bits=4, group_size=32)
    X = dev(c.X)
    y16 = wq.wq_w4a16_gemm(X, packed, steps, zeros, 8192, group_size=32).cpu().numpy().astype(np.float64)
    q, mult = wq.wq_quantize_act_int8(X, group_size=32)
    y8 = wq.wq_w4a8_gemm(q, mult, packed, steps, zeros, 8192, group_size=32).cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(y8 - y16) / np.linalg.norm(y16)
    assert 1e-4 < rel < 3e-2, rel
