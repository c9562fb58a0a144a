"""Host-side checks of the C-ABI library: it loads without a GPU, exports every
symbol the header declares, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "wq.h")


@pytest.fixture(scope="session")
def wq():
    from weight_only_quantization_group_b200 import build
    build.build()
    import weight_only_quantization_group_b200 as m
    return m


def _declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(wq_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    for required in ("wq_quantize_pack", "wq_w4a16_gemm", "wq_unpack_dequant", "wq_get_last_device_error"):
        assert required in names


def test_library_exports_every_declared_symbol(wq):
    L = ctypes.CDLL(wq.library_path)
    missing = [n for n in _declared_functions() if not hasattr(L, n)]
    assert not missing, missing
    assert set(_declared_functions()) == set(wq.EXPORTED_SYMBOLS)


def test_abi_version_and_status_strings(wq):
    assert wq.wq_abi_version() == 1
    for code in range(8):
        assert wq.wq_status_string(code).startswith("WQ_")
    assert wq.wq_status_string(99) == "unknown wq status"


def test_packed_word_counts(wq):
    assert wq.wq_packed_words(4096, 4096, bits=4) == 4096 * 4096 // 8
    assert wq.wq_packed_words(8192, 8192, bits=3) == 8192 * 8192 * 3 // 32
    assert wq.wq_packed_words(7, 11008, bits=4) == 7 * 11008 // 8
    assert wq.wq_packed_words(128, 200, bits=4) == 0      # K not a multiple of 128
    assert wq.wq_packed_words(128, 256, bits=5) == 0      # unsupported width
    assert wq.wq_packed_words(0, 256, bits=4) == 0


def _cfg(wq, bits=4, group=128, sym=0):
    return wq._Cfg(bits, group, sym)


def _cuda_device_present():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


# The validation tests pass fake device addresses that every call must reject
# before it touches CUDA; on a machine with a GPU they do not run, so that a
# check that wrongly passed could never launch a kernel on them.
fake_pointers = pytest.mark.skipif(_cuda_device_present(), reason="fake device addresses: host-only")


@fake_pointers
def test_argument_validation_without_gpu(wq):
    L = wq.lib()
    good = 0x10000  # a fake, 16-byte aligned address; validation fails before any use
    c = _cfg(wq)
    by = ctypes.byref
    # unsupported / invalid configs
    assert L.wq_quantize_pack(good, None, 8, 256, by(_cfg(wq, bits=5)), good, good, good, None) == wq.WQ_ERR_UNSUPPORTED
    assert L.wq_quantize_pack(good, None, 8, 256, by(_cfg(wq, bits=1)), good, good, good, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_quantize_pack(good, None, 8, 256, by(_cfg(wq, group=48)), good, good, good, None) == wq.WQ_ERR_INVALID_ARG
    n_i = (ctypes.c_int64 * 1)(16)
    assert L.wq_awq_workspace_bytes(8, 256, n_i, 1, 20, by(_cfg(wq, group=64))) == 0  # AWQ: groups of 128 only
    assert L.wq_quantize_pack(good, None, 8, 256, by(_cfg(wq, sym=2)), good, good, good, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_quantize_pack(good, None, 8, 256, None, good, good, good, None) == wq.WQ_ERR_INVALID_ARG
    # shapes
    assert L.wq_quantize_pack(good, None, 0, 256, by(c), good, good, good, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_quantize_pack(good, None, 8, 200, by(c), good, good, good, None) == wq.WQ_ERR_INVALID_ARG
    # null and misaligned pointers
    assert L.wq_quantize_pack(None, None, 8, 256, by(c), good, good, good, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_quantize_pack(good + 8, None, 8, 256, by(c), good, good, good, None) == wq.WQ_ERR_ALIGNMENT
    assert L.wq_quantize_pack(good, good + 2, 8, 256, by(c), good, good, good, None) == wq.WQ_ERR_ALIGNMENT
    # matmul
    assert L.wq_w4a16_gemm(good, good, good, good, 0, 8, 256, by(c), good, None, 0, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_w4a16_gemm(good + 4, good, good, good, 1, 8, 256, by(c), good, None, 0, None) == wq.WQ_ERR_ALIGNMENT
    assert L.wq_w4a16_gemm(good, good, good, good, 1, 8, 256, by(c), None, None, 0, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_unpack_dequant(good, good, good, 8, 256, by(_cfg(wq, bits=6)), good, None) == wq.WQ_ERR_UNSUPPORTED
    assert wq.wq_gemm_workspace_bytes(1, 4096, 4096) == 0
    # an unaligned workspace is refused before anything is launched
    assert L.wq_w4a16_gemm(good, good, good, good, 16, 8, 256, by(c), good, good + 8, 1 << 20, None) == \
        wq.WQ_ERR_ALIGNMENT
    # scale folding
    assert L.wq_awq_fold_norm(None, good, 8, good, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_awq_fold_norm(good, good, 0, good, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_awq_fold_norm(good + 1, good, 8, good, None) == wq.WQ_ERR_ALIGNMENT
    assert L.wq_awq_fold_linear_rows(good, good, good, 4, 8, good, None, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_awq_fold_linear_rows(good, None, good, 0, 8, good, None, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_awq_fold_linear_rows(good, None, good + 1, 4, 8, good, None, None) == wq.WQ_ERR_ALIGNMENT


@fake_pointers
def test_search_gptq_and_w4a8_validation_without_gpu(wq):
    """AWQ search, GPTQ, int8 activations and W4A8: every argument check
    returns its status before anything touches CUDA."""
    L = wq.lib()
    good = 0x10000
    by = ctypes.byref
    c = _cfg(wq)
    VP = ctypes.c_void_p
    # AWQ search: W_dev is a host array of device pointers
    W2 = (VP * 2)(good, good)
    N2 = (ctypes.c_int64 * 2)(128, 256)
    al = (ctypes.c_double * 3)(0.0, 0.05, 0.1)

    def search(X=good, T=64, K=256, W=W2, N=N2, n_lin=2, cfg=c, alpha=al, n_alpha=3, s_out=good,
               mu=None, loss=None, best=None, ws=good, ws_bytes=1 << 30):
        return L.wq_awq_scale_search(X, T, K, W, N, n_lin, by(cfg) if cfg is not None else None, alpha, n_alpha,
                                     s_out, mu, loss, best, ws, ws_bytes, None)

    assert search(cfg=_cfg(wq, group=64)) == wq.WQ_ERR_UNSUPPORTED        # AWQ: groups of 128
    assert search(cfg=None) == wq.WQ_ERR_INVALID_ARG
    assert search(T=0) == wq.WQ_ERR_INVALID_ARG
    assert search(K=200) == wq.WQ_ERR_INVALID_ARG
    assert search(n_lin=0) == wq.WQ_ERR_INVALID_ARG and search(n_lin=9) == wq.WQ_ERR_INVALID_ARG
    assert search(n_alpha=0) == wq.WQ_ERR_INVALID_ARG and search(n_alpha=65) == wq.WQ_ERR_INVALID_ARG
    assert search(N=(ctypes.c_int64 * 2)(128, 0)) == wq.WQ_ERR_INVALID_ARG
    assert search(X=None) == wq.WQ_ERR_INVALID_ARG and search(s_out=None) == wq.WQ_ERR_INVALID_ARG
    assert search(W=(VP * 2)(good, None)) == wq.WQ_ERR_INVALID_ARG
    assert search(W=(VP * 2)(good, good + 8)) == wq.WQ_ERR_ALIGNMENT
    assert search(alpha=(ctypes.c_double * 3)(0.0, float("nan"), 0.1)) == wq.WQ_ERR_INVALID_ARG
    assert search(X=good + 8) == wq.WQ_ERR_ALIGNMENT
    assert search(loss=good + 4) == wq.WQ_ERR_ALIGNMENT and search(best=good + 2) == wq.WQ_ERR_ALIGNMENT
    assert search(ws=None) == wq.WQ_ERR_WORKSPACE
    need = L.wq_awq_workspace_bytes(64, 256, N2, 2, 3, by(c))
    assert need > 0 and search(ws_bytes=need - 1) == wq.WQ_ERR_WORKSPACE
    assert search(ws=good + 128, ws_bytes=need) == wq.WQ_ERR_ALIGNMENT
    assert L.wq_awq_scale_search_noalloc(good, 64, 32768, W2, N2, 2, by(c), al, 3, good, None, None, None,
                                         None) == wq.WQ_ERR_WORKSPACE       # K beyond the fixed scratch

    # GPTQ
    def gptq(X=good, T=64, W=good, N=8, K=256, cfg=c, damp=0.01, packed=good, ws=good, ws_bytes=1 << 30):
        return L.wq_gptq_quantize_pack(X, T, W, N, K, by(cfg), damp, packed, good, good, ws, ws_bytes, None)

    assert gptq(cfg=_cfg(wq, bits=5)) == wq.WQ_ERR_UNSUPPORTED
    assert gptq(T=0) == wq.WQ_ERR_INVALID_ARG and gptq(K=100) == wq.WQ_ERR_INVALID_ARG
    assert gptq(damp=-0.1) == wq.WQ_ERR_INVALID_ARG and gptq(damp=float("nan")) == wq.WQ_ERR_INVALID_ARG
    assert gptq(X=None) == wq.WQ_ERR_INVALID_ARG
    assert gptq(packed=good + 4) == wq.WQ_ERR_ALIGNMENT and gptq(W=good + 1) == wq.WQ_ERR_ALIGNMENT
    need = L.wq_gptq_workspace_bytes(8, 256, by(c))
    assert need > 0 and gptq(ws_bytes=need - 1) == wq.WQ_ERR_WORKSPACE and gptq(ws=None) == wq.WQ_ERR_WORKSPACE
    assert gptq(ws=good + 64, ws_bytes=need) == wq.WQ_ERR_ALIGNMENT

    # int8 activations
    assert L.wq_quantize_act_int8(good, 2, 256, 48, good, good, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_quantize_act_int8(good, 0, 256, 32, good, good, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_quantize_act_int8(good, 2, 80, 32, good, good, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_quantize_act_int8(good, 2, 256, 32, None, good, None) == wq.WQ_ERR_INVALID_ARG
    assert L.wq_quantize_act_int8(good, 2, 256, 32, good + 2, good, None) == wq.WQ_ERR_ALIGNMENT

    # W4A8
    c32 = _cfg(wq, group=32)

    def w4a8(q=good, M=2, N=8, K=256, cfg=c32, Y=good):
        return L.wq_w4a8_gemm(q, good, good, good, good, M, N, K, by(cfg), Y, None)

    assert w4a8(cfg=_cfg(wq, bits=3, group=32)) == wq.WQ_ERR_UNSUPPORTED
    assert w4a8(K=32768) == wq.WQ_ERR_UNSUPPORTED
    assert w4a8(M=0) == wq.WQ_ERR_INVALID_ARG and w4a8(Y=None) == wq.WQ_ERR_INVALID_ARG
    assert w4a8(q=good + 4) == wq.WQ_ERR_ALIGNMENT


def test_option_values_are_validated(wq):
    """wq_set_option accepts exactly the documented values and wq_get_option
    reads them back; unknown options and values are refused."""
    cases = {
        wq.WQ_OPT_GEMM_PATH: ([0, 1, 2], [-1, 3]),
        wq.WQ_OPT_CROSSOVER_M: ([1, 3, 64], [0, -5]),
        wq.WQ_OPT_GEMV_VARIANT: ([0, 1, 2], [3, -1]),
        wq.WQ_OPT_GEMV_KERNEL: ([0, 2], [1, 3]),
        wq.WQ_OPT_GEMV_ROWS_SHAPE: ([0, 1, 2, 3, 4, 0], [5, -1]),
        wq.WQ_OPT_PDL: ([0, 1], [2]),
        wq.WQ_OPT_TC_STAGES: ([0, 2, 5, 16], [1, 17, -1]),
        wq.WQ_OPT_GEMV_GRID: ([1, 0], [2, -1]),
        wq.WQ_OPT_TC_BK: ([64, 128, 0], [32, 1, -1]),
        wq.WQ_OPT_TC_DEQUANT_WARPS: ([4, 8, 0], [2, 6, -1]),
        wq.WQ_OPT_WAIT_LIMIT_MS: ([1, 60000, 2000], [0, 60001]),
        wq.WQ_OPT_TEST_STALL: ([1, 0], [2, -1]),
        wq.WQ_OPT_AWQ_LOSS: ([1, 0], [2, -1]),
        wq.WQ_OPT_TC_KSPLIT: ([0, 1, 2, 4, 8], [3, 16, -1]),
        wq.WQ_OPT_TC_STREAMK: ([1, 2, 0], [3, -1]),
    }
    for opt, (good, bad) in cases.items():
        old = wq.wq_get_option(opt)
        try:
            for v in good:
                wq.wq_set_option(opt, v)
                assert wq.wq_get_option(opt) == v
            for v in bad:
                with pytest.raises(wq.WQError):
                    wq.wq_set_option(opt, v)
                assert wq.wq_get_option(opt) == good[-1]
        finally:
            wq.wq_set_option(opt, old)
    assert wq.wq_get_option(999) == -1
    with pytest.raises(wq.WQError):
        wq.wq_set_option(999, 0)


def test_packed_weight_round_trip_and_header_checks(wq, tmp_path):
    """save_packed / load_packed keep the three tensors bit for bit and refuse
    a file whose layout version or sizes do not match."""
    import torch
    N, K = 5, 256
    g = torch.Generator().manual_seed(3)
    packed = torch.randint(-2**31, 2**31 - 1, (N * K // 8,), dtype=torch.int32, generator=g)
    steps = torch.rand((N, K // 128), generator=g).to(torch.float16)
    zeros = torch.randint(0, 16, (N, K // 128), generator=g).to(torch.float16)
    p = tmp_path / "w.pt"
    wq.save_packed(p, packed, steps, zeros, N, K, bits=4)
    pk, st, zr, h = wq.load_packed(p)
    assert torch.equal(pk, packed) and torch.equal(st, steps) and torch.equal(zr, zeros)
    assert h["layout_version"] == wq.wq_layout_version() == 1 and (h["N"], h["K"], h["bits"]) == (N, K, 4)
    d = torch.load(p, weights_only=True)
    d["header"]["layout_version"] = 2
    torch.save(d, tmp_path / "v2.pt")
    with pytest.raises(ValueError):
        wq.load_packed(tmp_path / "v2.pt")
    d["header"]["layout_version"] = 1
    d["header"]["K"] = 384
    torch.save(d, tmp_path / "bad.pt")
    with pytest.raises(ValueError):
        wq.load_packed(tmp_path / "bad.pt")


def test_binding_checks_tensor_sizes_before_the_abi(wq):
    """The C ABI takes bare pointers, so the binding checks every tensor's
    dtype, contiguity and byte size first: a buffer too short for the call
    (the kernels would read or write past its end) raises instead. CPU tensors
    stand in for device ones; the device checks come after these."""
    import torch
    c = wq._cfg(4, 128, False)
    N, K, M = 64, 512, 3
    X = torch.zeros((M, K), dtype=torch.float16)
    packed = torch.zeros(N * K // 8, dtype=torch.int32)
    steps = torch.zeros((N, K // 128), dtype=torch.float16)
    zeros = torch.zeros((N, K // 128), dtype=torch.float16)
    out = torch.zeros((M, N), dtype=torch.float16)
    wq._gemm_operands(X, packed, steps, zeros, N, c, out)  # exact sizes pass
    wq._gemm_operands(X, packed.view(torch.uint8), steps, zeros, N, c, None)  # any integer view of the words
    with pytest.raises(ValueError, match="packed holds"):
        wq._gemm_operands(X, packed[:-1], steps, zeros, N, c, out)
    with pytest.raises(ValueError, match="packed holds"):
        wq._gemm_operands(X, packed, steps, zeros, N + 1, c, None)   # N larger than the weight
    with pytest.raises(ValueError, match="steps holds"):
        wq._gemm_operands(X, packed, steps[:-1], zeros, N, c, out)
    with pytest.raises(TypeError, match="zeros must be"):
        wq._gemm_operands(X, packed, steps, zeros.float(), N, c, out)
    with pytest.raises(ValueError, match="out holds"):
        wq._gemm_operands(X, packed, steps, zeros, N, c, out[:-1])
    with pytest.raises(ValueError, match="contiguous"):
        wq._gemm_operands(X, packed, steps.t(), zeros, N, c, out)
    with pytest.raises(ValueError, match=r"X must be \[M\]\[K\]"):
        wq._gemm_operands(X[0], packed, steps, zeros, N, c, out)
    with pytest.raises(TypeError, match="must be a torch.Tensor"):
        wq._gemm_operands(X, list(range(8)), steps, zeros, N, c, out)
    # 3-bit: three words per 32 channels
    c3 = wq._cfg(3, 128, False)
    p3 = torch.zeros(N * K * 3 // 32 // 4, dtype=torch.int32)   # a quarter of what is needed
    with pytest.raises(ValueError, match="packed holds"):
        wq._quant_operands(N, K, c3, p3, steps, zeros)
    wq._quant_operands(N, K, c3, torch.zeros(N * K * 3 // 32, dtype=torch.int32), steps, zeros)
    # an invalid shape needs nothing here: the library reports it itself
    wq._quant_operands(N, 200, c, packed[:0], steps[:0], zeros[:0])


def test_binding_checks_awq_shapes(wq):
    import torch
    X = torch.zeros((16, 256), dtype=torch.float16)
    wq._awq_operands(X, [torch.zeros((8, 256), dtype=torch.float16)] * 2)
    with pytest.raises(ValueError, match=r"W\[1\] must be \[N\]\[256\]"):
        wq._awq_operands(X, [torch.zeros((8, 256), dtype=torch.float16), torch.zeros((8, 128), dtype=torch.float16)])
    with pytest.raises(ValueError, match="at least one weight"):
        wq._awq_operands(X, [])
    with pytest.raises(ValueError, match=r"X must be \[T\]\[K\]"):
        wq._awq_operands(X.view(-1), [torch.zeros((8, 256), dtype=torch.float16)])


def test_binding_checks_devices(wq):
    """Every tensor of a call must live on the first operand's device."""
    import torch
    a = torch.zeros(4)
    wq._on_device_of(a, b=torch.zeros(2), c=None)
    with pytest.raises(ValueError, match="must be a CUDA tensor on cpu, got meta"):
        wq._on_device_of(a, b=torch.zeros(2, device="meta"))
    import contextlib
    assert isinstance(wq._device_of(a), contextlib.nullcontext)  # nothing to switch for a host tensor
    N, K = 8, 256  # a host buffer never reaches the ABI as a device pointer
    with pytest.raises(ValueError, match="packed must be a CUDA tensor"):
        wq.wq_unpack_dequant(torch.zeros(N * K // 8, dtype=torch.int32), torch.zeros((N, 2), dtype=torch.float16),
                             torch.zeros((N, 2), dtype=torch.float16), N, K)


def test_awq_workspace_size_is_its_layout(wq):
    """wq_awq_workspace_bytes is the sum of the search's regions, each rounded
    up to 256 bytes: mu (fp64 [K]), the candidates (fp16 [n_alpha][K]), one
    fp64 partial loss per (alpha, tile) -- 128x128 tiles of the two-kernel
    loss or (alpha, 128-row tile of one linear, 512-token chunk) of the fused
    one, whichever count is larger -- and, on the two-kernel loss path only,
    the fp16 error matrices of one batch of alphas (as many as fit 1 GiB, at
    least one). The default fused path keeps no error matrix."""
    def a256(x):
        return (x + 255) // 256 * 256

    for T, K, Ns, n_alpha in [(512, 4096, [4096] * 3, 20), (8, 256, [16], 20), (131, 640, [1, 129, 7], 6),
                              (512, 11008, [4096], 20)]:
        N = sum(Ns)
        tiles = max(-(-T // 128) * -(-N // 128), sum(-(-n // 128) for n in Ns) * -(-T // 512))
        batch = max(1, min(n_alpha, (1 << 30) // (N * K * 2)))
        want = a256(K * 8) + a256(n_alpha * K * 2) + a256(n_alpha * tiles * 8)
        assert wq.wq_awq_workspace_bytes(T, K, Ns, n_alpha) == want, (T, K, Ns)
        old = wq.wq_get_option(wq.WQ_OPT_AWQ_LOSS)
        try:
            wq.wq_set_option(wq.WQ_OPT_AWQ_LOSS, wq.WQ_AWQ_LOSS_TWO_KERNELS)
            assert wq.wq_awq_workspace_bytes(T, K, Ns, n_alpha) == want + a256(batch * N * K * 2), (T, K, Ns)
        finally:
            wq.wq_set_option(wq.WQ_OPT_AWQ_LOSS, old)


def test_binding_constants_match_the_header(wq):
    """Every numeric #define of include/wq.h (status codes, options and their
    values) has the same value in the Python binding; the two version numbers
    are read from the library instead."""
    src = open(HEADER).read()
    defines = dict((n, int(v)) for n, v in re.findall(r"#define (WQ_[A-Z0-9_]+) (-?\d+)\b", src))
    assert defines["WQ_ABI_VERSION"] == wq.wq_abi_version()
    assert defines["WQ_LAYOUT_VERSION"] == wq.wq_layout_version()
    for name, value in defines.items():
        if name in ("WQ_ABI_VERSION", "WQ_LAYOUT_VERSION"):
            continue
        assert getattr(wq, name) == value, name
    assert sum(n.startswith("WQ_OPT_") for n in defines) >= 12


def test_awq_workspace_follows_the_loss_path(wq):
    """The fused loss path keeps no error matrix, so its workspace is smaller
    by the E batch (here every alpha fits one 1 GiB batch: 20 x N x K x 2)."""
    T, K, Ns = 512, 4096, [4096, 4096, 4096]
    old = wq.wq_get_option(wq.WQ_OPT_AWQ_LOSS)
    try:
        wq.wq_set_option(wq.WQ_OPT_AWQ_LOSS, wq.WQ_AWQ_LOSS_TWO_KERNELS)
        two = wq.wq_awq_workspace_bytes(T, K, Ns, 20)
        wq.wq_set_option(wq.WQ_OPT_AWQ_LOSS, wq.WQ_AWQ_LOSS_FUSED)
        fused = wq.wq_awq_workspace_bytes(T, K, Ns, 20)
    finally:
        wq.wq_set_option(wq.WQ_OPT_AWQ_LOSS, old)
    batch = min(20, (1 << 30) // (sum(Ns) * K * 2))
    assert two - fused == batch * sum(Ns) * K * 2
    assert 0 < fused < 8 << 20


def test_gemm_workspace_size_is_its_layout(wq):
    """The tensor-core kernel's stream-K workspace: 64 KB of arrival counters,
    then two fp32 partial tiles (128 rows x M rounded up to 16) per CTA of the
    persistent grid (two CTAs per SM on 148 SMs, at most half the stage
    units); none for M < 3 (the row GEMV)."""
    sms = 148
    for M, N, K, cps in ((16, 28672, 8192, 2), (4, 8192, 8192, 2), (16, 1000, 4096, 2)):
        BN = (M + 15) // 16 * 16
        units = (N + 127) // 128 * (K // 128)
        P = min(cps * sms, units // 2)
        assert wq.wq_gemm_workspace_bytes(M, N, K) == 65536 + P * 2 * 128 * BN * 4
    assert wq.wq_gemm_workspace_bytes(2, 28672, 8192) == 0
    assert wq.wq_gemm_workspace_bytes(16, 28672, 8192, group_size=48) == 0  # invalid configuration
