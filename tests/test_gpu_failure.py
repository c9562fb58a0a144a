"""Failure handling on the device without a fault: a bounded wait that runs
out is reported through the device flag, the kernel returns, and the GPU
stays usable.

The tensor-core kernel's producer is told to issue no loads (the
WQ_OPT_TEST_STALL hook), so its consumers wait on barriers that nothing
completes. With a 50 ms wait limit they give up, latch WQ_ERR_TIMEOUT, free
their tensor memory and exit; nothing traps and nothing spins unbounded."""
import numpy as np
import pytest

import synth
from oracle import wq_oracle as O

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def wq():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    from weight_only_quantization_group_b200 import build
    build.build()
    import weight_only_quantization_group_b200 as m
    return m


def _gemm(wq, X, q, N):
    import torch
    return wq.wq_w4a16_gemm(torch.from_numpy(X).cuda(), *q, N, bits=4)


def test_timeout_is_reported_and_device_recovers(wq):
    import torch
    N, K, M = 128, 256, 16
    g = synth.rng(990)
    W = synth.weight(g, N, K, 0.02)
    X = synth.activations(g, M, K)
    q = wq.wq_quantize_pack(torch.from_numpy(W).cuda(), bits=4)
    assert wq.wq_get_last_device_error() == wq.WQ_OK
    wq.wq_set_option(wq.WQ_OPT_GEMM_PATH, wq.WQ_PATH_TENSOR_CORE)
    wq.wq_set_option(wq.WQ_OPT_WAIT_LIMIT_MS, 50)
    wq.wq_set_option(wq.WQ_OPT_TEST_STALL, 1)
    try:
        _gemm(wq, X, q, N)  # the launch itself succeeds
        assert wq.wq_get_last_device_error() == wq.WQ_ERR_TIMEOUT
        assert wq.wq_get_last_device_error() == wq.WQ_OK  # read-and-clear
    finally:
        wq.wq_set_option(wq.WQ_OPT_TEST_STALL, 0)
        wq.wq_set_option(wq.WQ_OPT_WAIT_LIMIT_MS, 2000)
    try:
        # the same kernel, same process: correct results and a clean flag
        codes = O.unpack_codes(q[0].cpu().numpy().view(np.uint32).reshape(N, -1), 4, K)
        st, z = q[1].cpu().numpy(), q[2].cpu().numpy()
        Y = _gemm(wq, X, q, N).cpu().numpy().astype(np.float64)
        assert wq.wq_get_last_device_error() == wq.WQ_OK
        ref = O.gemm_ref(X, codes, st, z, 128)
        assert np.linalg.norm(Y - ref) <= 1e-3 * np.linalg.norm(ref)
    finally:
        wq.wq_set_option(wq.WQ_OPT_GEMM_PATH, wq.WQ_PATH_AUTO)
