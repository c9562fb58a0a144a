"""The AWQ scale search entry point that allocates nothing.

Some callers cannot allocate device memory: a host framework may own every
device allocation, or a latency-critical path may not accept the device-wide
synchronization that cudaMalloc can imply. For them the library offers
wq_awq_scale_search_noalloc, which takes the same inputs and outputs as
wq_awq_scale_search but no workspace: its scratch is a fixed array in the
library's own device memory. These tests call it through the C ABI and check
that two calls in a row give what the workspace entry point gives, and that a
problem beyond the array's limits is refused. The file is collected last.
"""
import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu

# the loss tolerance of the AWQ parity tests (both loss paths)
LOSS_RTOL = {"fused": 1e-4, "two_kernels": 1e-4}

# (T, N_i, bits, symmetric): two row chunks that both end on a 128-row
# boundary; and a ragged case -- T not a multiple of 128, a last chunk whose
# rows end inside a 128-row tile, 3-bit symmetric codes
CASES = {"even": (256, (1700, 1500), 4, False), "ragged": (200, (2100, 1101), 3, True)}


@pytest.fixture(scope="module")
def wq():
    from weight_only_quantization_group_b200 import build
    build.build()
    import weight_only_quantization_group_b200 as m
    return m


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("path", ["two_kernels", "fused"])
def test_noalloc_matches_workspace_entry_point_twice(wq, path, case):
    """Both loss paths: the fused one needs no error-matrix chunks at all."""
    old = wq.wq_get_option(wq.WQ_OPT_AWQ_LOSS)
    wq.wq_set_option(wq.WQ_OPT_AWQ_LOSS, wq.WQ_AWQ_LOSS_FUSED if path == "fused" else wq.WQ_AWQ_LOSS_TWO_KERNELS)
    try:
        _noalloc_matches(wq, LOSS_RTOL[path], *CASES[case])
    finally:
        wq.wq_set_option(wq.WQ_OPT_AWQ_LOSS, old)


def _noalloc_matches(wq, rtol, T, Ns, bits, sym):
    g = synth.rng(900 + T)
    K = 4096  # 2048-row error chunks: the stacked rows span two chunks
    X = dev(synth.activations(g, T, K, channel_frac=0.01, channel_mult=20.0))
    Ws = [dev(synth.weight(g, n, K, 0.02)) for n in Ns]
    ref = wq.wq_awq_scale_search(X, Ws, bits=bits, symmetric=sym)
    assert wq.wq_get_last_device_error() == 0
    for _ in range(2):
        out = wq.wq_awq_scale_search_noalloc(X, Ws, bits=bits, symmetric=sym)
        assert wq.wq_get_last_device_error() == 0
        assert torch.equal(out["mu"], ref["mu"])
        rel = (out["losses"] - ref["losses"]).abs() / ref["losses"]
        assert float(rel.max()) <= rtol
        assert int(out["best"].item()) == int(ref["best"].item())
        assert torch.equal(out["s"].view(torch.int16), ref["s"].view(torch.int16))


def test_noalloc_refuses_problems_beyond_its_scratch(wq):
    X = torch.zeros((8, 32768), dtype=torch.float16, device="cuda")
    W = torch.zeros((16, 32768), dtype=torch.float16, device="cuda")
    with pytest.raises(wq.WQError) as e:
        wq.wq_awq_scale_search_noalloc(X, [W])
    assert e.value.status == wq.WQ_ERR_WORKSPACE
