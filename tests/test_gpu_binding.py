"""The binding's argument checks with device tensors: a buffer shorter than
the call needs, a wrong dtype, a tensor on another device or a weight whose K
differs from the activations' raises before the C ABI is called, so no
kernel ever reads or writes past a buffer. Each bad call is checked to leave
the device error flag clear, and a good call on the same tensors still gives
the right shape."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wq():
    from weight_only_quantization_group_b200 import build
    build.build()
    import weight_only_quantization_group_b200 as m
    return m


@pytest.fixture(scope="module")
def operands(wq):
    import torch
    g = synth.rng(1200)
    N, K, M = 96, 512, 3
    W = torch.from_numpy(synth.weight(g, N, K, 0.02)).cuda()
    X = torch.from_numpy(synth.activations(g, M, K)).cuda()
    packed, steps, zeros = wq.wq_quantize_pack(W, bits=4)
    assert wq.wq_get_last_device_error() == wq.WQ_OK
    return W, X, packed, steps, zeros, N, K, M


def test_gemm_refuses_short_or_mistyped_operands(wq, operands):
    import torch
    W, X, packed, steps, zeros, N, K, M = operands
    with pytest.raises(ValueError, match="packed holds"):
        wq.wq_w4a16_gemm(X, packed[:-1], steps, zeros, N)
    with pytest.raises(ValueError, match="packed holds"):
        wq.wq_w4a16_gemm(X, packed, steps, zeros, N + 8)        # N beyond the packed weight
    with pytest.raises(TypeError, match="steps must be"):
        wq.wq_w4a16_gemm(X, packed, steps.float(), zeros, N)
    with pytest.raises(ValueError, match="out holds"):
        wq.wq_w4a16_gemm(X, packed, steps, zeros, N, out=torch.empty((M, N - 1), dtype=torch.float16,
                                                                      device="cuda"))
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        wq.wq_w4a16_gemm(X, packed, steps, zeros, N, out=torch.empty((M, N), dtype=torch.float16))
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        wq.wq_w4a16_gemm(X, packed.cpu(), steps, zeros, N)
    assert wq.wq_get_last_device_error() == wq.WQ_OK
    Y = wq.wq_w4a16_gemm(X, packed, steps, zeros, N)
    assert wq.wq_get_last_device_error() == wq.WQ_OK
    assert tuple(Y.shape) == (M, N) and bool(torch.isfinite(Y).all())


def test_quantize_and_unpack_refuse_short_outputs(wq, operands):
    import torch
    W, X, packed, steps, zeros, N, K, M = operands
    with pytest.raises(ValueError, match="packed holds"):
        wq.wq_quantize_pack(W, bits=4, out=(packed[: packed.numel() // 2], steps, zeros))
    with pytest.raises(ValueError, match="s holds"):
        wq.wq_quantize_pack(W, torch.ones(K - 8, dtype=torch.float16, device="cuda"), bits=4)
    with pytest.raises(ValueError, match="out holds"):
        wq.wq_unpack_dequant(packed, steps, zeros, N, K, out=torch.empty((N, K - 128), dtype=torch.float16,
                                                                          device="cuda"))
    with pytest.raises(ValueError, match="zeros holds"):
        wq.wq_unpack_dequant(packed, steps, zeros[:1], N, K)
    assert wq.wq_get_last_device_error() == wq.WQ_OK


def test_awq_refuses_a_weight_of_another_width(wq, operands):
    import torch
    W, X, packed, steps, zeros, N, K, M = operands
    with pytest.raises(ValueError, match=r"W\[1\] must be \[N\]\[512\]"):
        wq.wq_awq_scale_search(X, [W, W[:, :256].contiguous()])
    with pytest.raises(ValueError, match=r"W\[0\] must be \[N\]\[512\]"):
        wq.wq_awq_scale_search_noalloc(X, [W[:, :384].contiguous()])
    out = {"s": torch.empty(K, dtype=torch.float16, device="cuda"),
           "mu": torch.empty(K, dtype=torch.float64, device="cuda"),
           "losses": torch.empty(3, dtype=torch.float64, device="cuda"),   # 20 alphas need 20
           "best": torch.empty(1, dtype=torch.int32, device="cuda")}
    with pytest.raises(ValueError, match="losses"):
        wq.wq_awq_scale_search_noalloc(X, [W], out=out)
    assert wq.wq_get_last_device_error() == wq.WQ_OK
    assert np.isfinite(float(wq.wq_awq_scale_search(X, [W], [0.0, 0.5])["losses"].cpu().numpy().min()))
