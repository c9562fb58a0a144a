"""Python binding of libwq.so: group-wise weight-only quantization for B200.

A thin ctypes layer over the C ABI declared in ``include/wq.h``. Each
``wq_*`` function here has the same name and meaning as the C entry point; it
only checks tensor metadata, allocates outputs with torch (device memory is
the one thing torch provides), passes raw pointers and the current CUDA
stream, and raises :class:`WQError` on a non-OK status. Every step of the
computation runs in the library's CUDA kernels; there is no CPU fallback.
"""
from __future__ import annotations

import contextlib
import ctypes
import os

import torch

__all__ = [
    "WQError",
    "save_packed",
    "load_packed",
    "wq_layout_version",
    "lib",
    "library_path",
    "wq_abi_version",
    "wq_status_string",
    "wq_packed_words",
    "wq_quantize_pack",
    "wq_unpack_dequant",
    "wq_gemm_workspace_bytes",
    "wq_w4a16_gemm",
    "wq_get_last_device_error",
    "wq_set_option",
    "wq_get_option",
    "wq_awq_workspace_bytes",
    "wq_awq_scale_search",
    "wq_awq_scale_search_noalloc",
    "wq_awq_fold_norm",
    "wq_awq_fold_linear_rows",
    "wq_gptq_workspace_bytes",
    "wq_gptq_quantize_pack",
    "wq_quantize_act_int8",
    "wq_w4a8_gemm",
    "EXPORTED_SYMBOLS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libwq.so")

# Every symbol include/wq.h declares.
EXPORTED_SYMBOLS = (
    "wq_abi_version",
    "wq_layout_version",
    "wq_status_string",
    "wq_packed_words",
    "wq_quantize_pack",
    "wq_unpack_dequant",
    "wq_gemm_workspace_bytes",
    "wq_w4a16_gemm",
    "wq_get_last_device_error",
    "wq_set_option",
    "wq_get_option",
    "wq_awq_workspace_bytes",
    "wq_awq_scale_search",
    "wq_awq_scale_search_noalloc",
    "wq_awq_fold_norm",
    "wq_awq_fold_linear_rows",
    "wq_gptq_workspace_bytes",
    "wq_gptq_quantize_pack",
    "wq_quantize_act_int8",
    "wq_w4a8_gemm",
)

WQ_OK = 0
WQ_ERR_INVALID_ARG = 1
WQ_ERR_UNSUPPORTED = 2
WQ_ERR_ALIGNMENT = 3
WQ_ERR_CUDA = 4
WQ_ERR_TIMEOUT = 5
WQ_ERR_WORKSPACE = 6
WQ_ERR_RANGE = 7

WQ_OPT_GEMM_PATH = 1
WQ_OPT_CROSSOVER_M = 2
WQ_PATH_AUTO = 0
WQ_PATH_GEMV = 1
WQ_PATH_TENSOR_CORE = 2
WQ_OPT_GEMV_VARIANT = 4
WQ_GEMV_OFFSET_SUMS = 0
WQ_GEMV_EXACT = 1
WQ_GEMV_INT_DIGITS = 2
WQ_OPT_GEMV_KERNEL = 5
WQ_GEMV_KERNEL_AUTO = 0
WQ_GEMV_KERNEL_TILED = 2
WQ_OPT_GEMV_ROWS_SHAPE = 6
WQ_OPT_PDL = 7
WQ_OPT_TC_STAGES = 9
WQ_OPT_GEMV_GRID = 10
WQ_OPT_TC_BK = 11
WQ_OPT_TC_DEQUANT_WARPS = 12
WQ_OPT_WAIT_LIMIT_MS = 13
WQ_OPT_TEST_STALL = 14
WQ_OPT_AWQ_LOSS = 15
WQ_OPT_TC_KSPLIT = 16
WQ_OPT_TC_STREAMK = 17
WQ_AWQ_LOSS_TWO_KERNELS = 0
WQ_AWQ_LOSS_FUSED = 1


class WQError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {lib().wq_status_string(self.status).decode()}")


class _Cfg(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("group_size", ctypes.c_int32), ("symmetric", ctypes.c_int32)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(library_path):
        raise ImportError(
            f"{library_path} is missing: build the CUDA library first "
            "(python -m weight_only_quantization_group_b200.build)")
    L = ctypes.CDLL(library_path)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    cfgp = ctypes.POINTER(_Cfg)
    sig = {
        "wq_abi_version": (i32, []),
        "wq_layout_version": (i32, []),
        "wq_status_string": (ctypes.c_char_p, [i32]),
        "wq_packed_words": (sz, [i64, i64, cfgp]),
        "wq_quantize_pack": (i32, [vp, vp, i64, i64, cfgp, vp, vp, vp, vp]),
        "wq_unpack_dequant": (i32, [vp, vp, vp, i64, i64, cfgp, vp, vp]),
        "wq_gemm_workspace_bytes": (sz, [i64, i64, i64, cfgp]),
        "wq_w4a16_gemm": (i32, [vp, vp, vp, vp, i64, i64, i64, cfgp, vp, vp, sz, vp]),
        "wq_get_last_device_error": (i32, [vp]),
        "wq_set_option": (i32, [i32, i64]),
        "wq_get_option": (i64, [i32]),
        "wq_awq_workspace_bytes": (sz, [i64, i64, ctypes.POINTER(i64), i32, i32, cfgp]),
        "wq_awq_scale_search": (i32, [vp, i64, i64, ctypes.POINTER(vp), ctypes.POINTER(i64), i32, cfgp,
                                      ctypes.POINTER(ctypes.c_double), i32, vp, vp, vp, vp, vp, sz, vp]),
        "wq_awq_scale_search_noalloc": (i32, [vp, i64, i64, ctypes.POINTER(vp), ctypes.POINTER(i64), i32, cfgp,
                                              ctypes.POINTER(ctypes.c_double), i32, vp, vp, vp, vp, vp]),
        "wq_awq_fold_norm": (i32, [vp, vp, i64, vp, vp]),
        "wq_gptq_workspace_bytes": (sz, [i64, i64, cfgp]),
        "wq_quantize_act_int8": (i32, [vp, i64, i64, i32, vp, vp, vp]),
        "wq_w4a8_gemm": (i32, [vp, vp, vp, vp, vp, i64, i64, i64, cfgp, vp, vp]),
        "wq_gptq_quantize_pack": (i32, [vp, i64, vp, i64, i64, cfgp, ctypes.c_double, vp, vp, vp, vp, sz, vp]),
        "wq_awq_fold_linear_rows": (i32, [vp, vp, vp, i64, i64, vp, vp, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L


_lib_handle = None


def lib() -> ctypes.CDLL:
    """The loaded libwq.so (loaded on first use; raises if it is missing)."""
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = _load()
    return _lib_handle


class _LazyLib:
    def __getattr__(self, name):
        return getattr(lib(), name)


_lib = _LazyLib()


_CFG_CACHE: dict = {}


def _cfg(bits: int, group_size: int, symmetric: bool) -> _Cfg:
    """A config struct per (bits, group, symmetric); the library only reads it."""
    key = (int(bits), int(group_size), bool(symmetric))
    c = _CFG_CACHE.get(key)
    if c is None:
        c = _CFG_CACHE[key] = _Cfg(key[0], key[1], 1 if key[2] else 0)
    return c


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(stream, device=None) -> int:
    """The caller's stream, or the current stream of `device` (default: the
    current device) when none is given."""
    if stream is None:
        if _raw_stream is not None:
            return _raw_stream(torch.cuda.current_device() if device is None else device)
        return torch.cuda.current_stream(device).cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _device_of(t: torch.Tensor):
    """A context making t's device the current one for the call: the library
    launches on the current device, and the tensors may live on another."""
    idx = t.device.index
    if idx is None or idx == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(idx)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _check(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _need(t, name: str, dtype, nbytes: int):
    """t: a contiguous tensor (of `dtype`, when given) holding at least
    `nbytes` bytes. The C ABI receives bare pointers, so a short buffer would
    be read or written past its end; these checks run before it is called
    (one combined test on the common path, the precise error otherwise)."""
    try:
        if (dtype is None or t.dtype == dtype) and t.is_contiguous() and t.nbytes >= nbytes:
            return
    except AttributeError:
        raise TypeError(f"{name} must be a torch.Tensor") from None
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    raise ValueError(f"{name} holds {t.nbytes} bytes; this call needs {nbytes}")


def _on_device_of(ref: torch.Tensor, **named):
    """Every named tensor lives on ref's device (ref is a CUDA tensor)."""
    dev = ref.device
    for name, t in named.items():
        if t is not None and t.device != dev:
            raise ValueError(f"{name} must be a CUDA tensor on {dev}, got {t.device}")


_NW_CACHE: dict = {}


def _packed_words_of(N: int, K: int, c: "_Cfg") -> int:
    key = (N, K, c.bits, c.group_size, c.symmetric)
    nw = _NW_CACHE.get(key)
    if nw is None:
        nw = _NW_CACHE[key] = int(_lib.wq_packed_words(N, K, ctypes.byref(c)))
    return nw


def _quant_operands(N: int, K: int, c: "_Cfg", packed, steps, zeros):
    """Sizes of the packed form of an [N][K] weight (0 when the config or the
    shape is invalid: the library reports those itself)."""
    nw = _packed_words_of(N, K, c)
    G = K // c.group_size if nw > 0 else 0
    _need(packed, "packed", None, 4 * nw)
    _need(steps, "steps", torch.float16, 2 * N * G)
    _need(zeros, "zeros", torch.float16, 2 * N * G)


def _gemm_operands(X, packed, steps, zeros, N: int, c: "_Cfg", out):
    """The tensors of wq_w4a16_gemm: X [M][K] fp16, the packed weight of an
    [N][K] matrix, and out (fp16, M*N values) when given."""
    if X.dim() != 2:
        raise ValueError(f"X must be [M][K], got shape {tuple(X.shape)}")
    M, K = X.shape
    _quant_operands(N, K, c, packed, steps, zeros)
    if out is not None:
        _need(out, "out", torch.float16, 2 * M * N)


def _awq_operands(X, Ws):
    """X [T][K] and every W [N_i][K] (the same K)."""
    if X.dim() != 2:
        raise ValueError(f"X must be [T][K], got shape {tuple(X.shape)}")
    K = X.shape[1]
    if len(Ws) == 0:
        raise ValueError("at least one weight is needed")
    for i, W in enumerate(Ws):
        if W.dim() != 2 or W.shape[1] != K:
            raise ValueError(f"W[{i}] must be [N][{K}], got shape {tuple(W.shape)}")


def _raise(st: int, where: str):
    if st != WQ_OK:
        raise WQError(st, where)


def wq_layout_version() -> int:
    """Version of the packed layout (codes, steps, zeros) this library writes and reads."""
    return int(lib().wq_layout_version())


def save_packed(path, packed: torch.Tensor, steps: torch.Tensor, zeros: torch.Tensor, N: int, K: int, *,
                bits: int = 4, group_size: int = 128, symmetric: bool = False) -> None:
    """Store a quantized weight (the three tensors of wq_quantize_pack) with a
    header naming the layout version and the quantization config."""
    header = {"format": "wq-packed", "layout_version": wq_layout_version(), "bits": int(bits),
              "group_size": int(group_size), "symmetric": bool(symmetric), "N": int(N), "K": int(K)}
    torch.save({"header": header, "packed": packed.detach().cpu(), "steps": steps.detach().cpu(),
                "zeros": zeros.detach().cpu()}, path)


def load_packed(path, device=None):
    """Read what save_packed wrote; checks the header against this library's
    layout and the tensor sizes. Returns (packed, steps, zeros, header)."""
    d = torch.load(path, map_location="cpu", weights_only=True)
    h = d.get("header", {})
    if h.get("format") != "wq-packed" or h.get("layout_version") != wq_layout_version():
        raise ValueError(f"{path}: not a wq-packed file of layout version {wq_layout_version()}")
    N, K, bits = h["N"], h["K"], h["bits"]
    words = wq_packed_words(N, K, bits=bits, group_size=h["group_size"], symmetric=h["symmetric"])
    G = K // h["group_size"]
    if (words == 0 or d["packed"].numel() != words or tuple(d["steps"].shape) != (N, G)
            or tuple(d["zeros"].shape) != (N, G)):
        raise ValueError(f"{path}: tensor sizes do not match the header")
    out = [d[k] if device is None else d[k].to(device) for k in ("packed", "steps", "zeros")]
    return out[0], out[1], out[2], h


def wq_abi_version() -> int:
    """ABI version of the loaded libwq.so."""
    return int(_lib.wq_abi_version())


def wq_status_string(status: int) -> str:
    """Name and meaning of a status code."""
    return _lib.wq_status_string(int(status)).decode()


def wq_packed_words(N: int, K: int, bits: int = 4, group_size: int = 128, symmetric: bool = False) -> int:
    """uint32 words of the packed [N][K] weight (N*K/8 at 4 bits, 3*N*K/32 at 3); 0 if invalid."""
    c = _cfg(bits, group_size, symmetric)
    return int(_lib.wq_packed_words(N, K, ctypes.byref(c)))


def wq_quantize_pack(W: torch.Tensor, s: torch.Tensor | None = None, *, bits: int = 4, group_size: int = 128,
                     symmetric: bool = False, out=None, stream=None):
    """Quantize + pack an fp16 [N][K] weight; returns (packed u32 as int32, steps, zeros)."""
    _check(W, torch.float16, "W")
    if W.dim() != 2:
        raise ValueError(f"W must be [N][K], got shape {tuple(W.shape)}")
    N, K = W.shape
    if s is not None:
        _check(s, torch.float16, "s")
        _need(s, "s", torch.float16, 2 * K)
    c = _cfg(bits, group_size, symmetric)
    nw = int(_lib.wq_packed_words(N, K, ctypes.byref(c)))
    if out is None:
        G = K // group_size if group_size > 0 else 0
        packed = torch.empty(max(nw, 1), dtype=torch.int32, device=W.device)
        steps = torch.empty((N, G), dtype=torch.float16, device=W.device)
        zeros = torch.empty((N, G), dtype=torch.float16, device=W.device)
    else:
        packed, steps, zeros = out
        _quant_operands(N, K, c, packed, steps, zeros)
    _on_device_of(W, s=s, packed=packed, steps=steps, zeros=zeros)
    with _device_of(W):
        st = _lib.wq_quantize_pack(_ptr(W), _ptr(s), N, K, ctypes.byref(c), _ptr(packed), _ptr(steps),
                                   _ptr(zeros), _stream(stream, W.device.index))
    _raise(st, "wq_quantize_pack")
    return packed, steps, zeros


def wq_unpack_dequant(packed: torch.Tensor, steps: torch.Tensor, zeros: torch.Tensor, N: int, K: int, *,
                      bits: int = 4, group_size: int = 128, symmetric: bool = False, out=None, stream=None):
    """fp16 [N][K] = fp16((q - zero) * step) from the packed form."""
    c = _cfg(bits, group_size, symmetric)
    _quant_operands(N, K, c, packed, steps, zeros)
    if not packed.is_cuda:
        raise ValueError("packed must be a CUDA tensor")
    if out is None:
        out = torch.empty((N, K), dtype=torch.float16, device=packed.device)
    _need(out, "out", torch.float16, 2 * N * K)
    _on_device_of(packed, steps=steps, zeros=zeros, out=out)
    with _device_of(packed):
        st = _lib.wq_unpack_dequant(_ptr(packed), _ptr(steps), _ptr(zeros), N, K, ctypes.byref(c), _ptr(out),
                                    _stream(stream, packed.device.index))
    _raise(st, "wq_unpack_dequant")
    return out


def wq_gemm_workspace_bytes(M: int, N: int, K: int, *, bits: int = 4, group_size: int = 128,
                            symmetric: bool = False) -> int:
    """Bytes of the optional matmul workspace (the tensor-core kernel's stream-K
    schedule); 0 when M < 3. Allocate it zero-filled once and reuse it."""
    c = _cfg(bits, group_size, symmetric)
    return int(_lib.wq_gemm_workspace_bytes(M, N, K, ctypes.byref(c)))


def wq_w4a16_gemm(X: torch.Tensor, packed: torch.Tensor, steps: torch.Tensor, zeros: torch.Tensor, N: int, *,
                  bits: int = 4, group_size: int = 128, symmetric: bool = False, out=None, workspace=None,
                  stream=None):
    """Y[M][N] = X[M][K] * deq(W)^T with fp32 accumulation; returns Y (fp16).

    `workspace` (optional): a zero-filled uint8 CUDA tensor of at least
    wq_gemm_workspace_bytes(M, N, K, ...) bytes, reusable across calls on one
    stream; with it the tensor-core kernel spreads its stages evenly over the
    SMs (stream-K) for M <= 16."""
    _check(X, torch.float16, "X")
    c = _cfg(bits, group_size, symmetric)
    _gemm_operands(X, packed, steps, zeros, N, c, out)
    M, K = X.shape
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=X.device)
    _on_device_of(X, packed=packed, steps=steps, zeros=zeros, out=out, workspace=workspace)
    ws_ptr, ws_bytes = None, 0
    if workspace is not None:
        ws_ptr, ws_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    with _device_of(X):
        st = lib().wq_w4a16_gemm(X.data_ptr(), packed.data_ptr(), steps.data_ptr(), zeros.data_ptr(), M, N, K,
                                 ctypes.byref(c), out.data_ptr(), ws_ptr, ws_bytes, _stream(stream, X.device.index))
    _raise(st, "wq_w4a16_gemm")
    return out


def wq_get_last_device_error(stream=None) -> int:
    """Synchronize the stream and return (then clear) the device error flag."""
    return int(_lib.wq_get_last_device_error(_stream(stream)))


def wq_set_option(option: int, value: int) -> None:
    """Set a process-wide tuning option (see include/wq.h)."""
    _raise(_lib.wq_set_option(int(option), int(value)), "wq_set_option")


def wq_get_option(option: int) -> int:
    """Current value of a process-wide option (WQ_OPT_*)."""
    return int(_lib.wq_get_option(int(option)))


def wq_awq_workspace_bytes(T: int, K: int, Ns, n_alpha: int = 20, *, bits: int = 4, group_size: int = 128,
                           symmetric: bool = False) -> int:
    """Workspace bytes of wq_awq_scale_search for T calibration rows, K input channels and
    the linears' output sizes Ns (for the loss path WQ_OPT_AWQ_LOSS selects now); 0 if invalid."""
    c = _cfg(bits, group_size, symmetric)
    arr = (ctypes.c_int64 * len(Ns))(*[int(n) for n in Ns])
    return int(_lib.wq_awq_workspace_bytes(T, K, arr, len(Ns), n_alpha, ctypes.byref(c)))


def wq_awq_scale_search(X: torch.Tensor, Ws, alphas=None, *, bits: int = 4, group_size: int = 128,
                        symmetric: bool = False, workspace: torch.Tensor | None = None, stream=None):
    """AWQ scale search over the linears `Ws` (fp16 [N_i][K]) that share the
    calibration input X (fp16 [T][K]). Returns a dict with s (fp16 [K]), mu
    (fp64 [K]), losses (fp64 [n_alpha]) and best (int32 [1]), all on the device."""
    _check(X, torch.float16, "X")
    for i, W in enumerate(Ws):
        _check(W, torch.float16, f"W[{i}]")
    _awq_operands(X, Ws)
    _on_device_of(X, **{f"W[{i}]": W for i, W in enumerate(Ws)}, workspace=workspace)
    T, K = X.shape
    if alphas is None:
        alphas = [j / 20.0 for j in range(20)]
    alphas = [float(a) for a in alphas]
    c = _cfg(bits, group_size, symmetric)
    Ns = [int(W.shape[0]) for W in Ws]
    n_arr = (ctypes.c_int64 * len(Ns))(*Ns)
    a_arr = (ctypes.c_double * len(alphas))(*alphas)
    w_arr = (ctypes.c_void_p * len(Ws))(*[W.data_ptr() for W in Ws])
    need = int(_lib.wq_awq_workspace_bytes(T, K, n_arr, len(Ns), len(alphas), ctypes.byref(c)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=X.device)
    elif not workspace.is_contiguous():
        raise ValueError("workspace must be contiguous")
    s = torch.empty(K, dtype=torch.float16, device=X.device)
    mu = torch.empty(K, dtype=torch.float64, device=X.device)
    losses = torch.empty(len(alphas), dtype=torch.float64, device=X.device)
    best = torch.empty(1, dtype=torch.int32, device=X.device)
    with _device_of(X):
        st = _lib.wq_awq_scale_search(_ptr(X), T, K, w_arr, n_arr, len(Ns), ctypes.byref(c), a_arr, len(alphas),
                                      _ptr(s), _ptr(mu), _ptr(losses), _ptr(best), workspace.data_ptr(),
                                      workspace.numel() * workspace.element_size(), _stream(stream, X.device.index))
    _raise(st, "wq_awq_scale_search")
    return {"s": s, "mu": mu, "losses": losses, "best": best}


def wq_awq_scale_search_noalloc(X: torch.Tensor, Ws, alphas=None, *, bits: int = 4, group_size: int = 128,
                                symmetric: bool = False, out=None, stream=None):
    """wq_awq_scale_search without a workspace: the library's own fixed device
    scratch is used instead (for callers that cannot allocate device memory;
    see include/wq.h for its size, limits and sharing rules). `out`, if given,
    is a dict with preallocated "s", "mu", "losses" and "best" tensors."""
    _check(X, torch.float16, "X")
    for i, W in enumerate(Ws):
        _check(W, torch.float16, f"W[{i}]")
    _awq_operands(X, Ws)
    _on_device_of(X, **{f"W[{i}]": W for i, W in enumerate(Ws)})
    T, K = X.shape
    if alphas is None:
        alphas = [j / 20.0 for j in range(20)]
    alphas = [float(a) for a in alphas]
    c = _cfg(bits, group_size, symmetric)
    Ns = [int(W.shape[0]) for W in Ws]
    n_arr = (ctypes.c_int64 * len(Ns))(*Ns)
    a_arr = (ctypes.c_double * len(alphas))(*alphas)
    w_arr = (ctypes.c_void_p * len(Ws))(*[W.data_ptr() for W in Ws])
    if out is None:
        out = {"s": torch.empty(K, dtype=torch.float16, device=X.device),
               "mu": torch.empty(K, dtype=torch.float64, device=X.device),
               "losses": torch.empty(len(alphas), dtype=torch.float64, device=X.device),
               "best": torch.empty(1, dtype=torch.int32, device=X.device)}
    else:
        _need(out["s"], "out['s']", torch.float16, 2 * K)
        _need(out["mu"], "out['mu']", torch.float64, 8 * K)
        _need(out["losses"], "out['losses']", torch.float64, 8 * len(alphas))
        _need(out["best"], "out['best']", torch.int32, 4)
        _on_device_of(X, **{f"out['{k}']": out[k] for k in ("s", "mu", "losses", "best")})
    with _device_of(X):
        st = _lib.wq_awq_scale_search_noalloc(_ptr(X), T, K, w_arr, n_arr, len(Ns), ctypes.byref(c), a_arr,
                                              len(alphas), _ptr(out["s"]), _ptr(out["mu"]), _ptr(out["losses"]),
                                              _ptr(out["best"]), _stream(stream, X.device.index))
    _raise(st, "wq_awq_scale_search_noalloc")
    return out


def wq_awq_fold_norm(gamma: torch.Tensor, s: torch.Tensor, *, out: torch.Tensor | None = None, stream=None):
    """gamma / s (fp16 [K] each): a normalisation weight absorbing the AWQ
    scales of the linears it feeds. out may be gamma (in place)."""
    _check(gamma, torch.float16, "gamma")
    K = gamma.numel()
    _need(s, "s", torch.float16, 2 * K)
    if out is None:
        out = torch.empty_like(gamma)
    _need(out, "out", torch.float16, 2 * K)
    _on_device_of(gamma, s=s, out=out)
    with _device_of(gamma):
        st = _lib.wq_awq_fold_norm(_ptr(gamma), _ptr(s), K, _ptr(out), _stream(stream, gamma.device.index))
    _raise(st, "wq_awq_fold_norm")
    return out


def wq_awq_fold_linear_rows(W: torch.Tensor, s: torch.Tensor, b: torch.Tensor | None = None, *, out=None,
                            stream=None):
    """W[n][k] / s[n] (and b[n] / s[n]): the linear before a scaled linear
    absorbs its AWQ scales in its output rows. Returns (W', b') (b' None
    without a bias); `out` = (W_out, b_out) may be the inputs (in place)."""
    _check(W, torch.float16, "W")
    if W.dim() != 2:
        raise ValueError(f"W must be [N][K], got shape {tuple(W.shape)}")
    N, K = W.shape
    _need(s, "s", torch.float16, 2 * N)
    if b is not None:
        _need(b, "b", torch.float16, 2 * N)
    if out is None:
        out = (torch.empty_like(W), None if b is None else torch.empty_like(b))
    W_out, b_out = out
    _need(W_out, "out[0]", torch.float16, 2 * N * K)
    if (b is None) != (b_out is None):
        raise ValueError("b and out[1] must both be given or both be None")
    if b_out is not None:
        _need(b_out, "out[1]", torch.float16, 2 * N)
    _on_device_of(W, s=s, b=b, W_out=W_out, b_out=b_out)
    with _device_of(W):
        st = _lib.wq_awq_fold_linear_rows(_ptr(W), _ptr(b), _ptr(s), N, K, _ptr(W_out), _ptr(b_out),
                                          _stream(stream, W.device.index))
    _raise(st, "wq_awq_fold_linear_rows")
    return W_out, b_out


def wq_gptq_workspace_bytes(N: int, K: int, *, bits: int = 4, group_size: int = 128, symmetric: bool = False) -> int:
    """Workspace bytes of wq_gptq_quantize_pack for an [N][K] weight; 0 if invalid."""
    c = _cfg(bits, group_size, symmetric)
    return int(_lib.wq_gptq_workspace_bytes(N, K, ctypes.byref(c)))


def wq_gptq_quantize_pack(W: torch.Tensor, X: torch.Tensor, *, bits: int = 4, group_size: int = 128,
                          symmetric: bool = False, damp: float = 0.01, workspace: torch.Tensor | None = None,
                          out=None, stream=None):
    """GPTQ quantize + pack of an fp16 [N][K] weight with calibration inputs X
    (fp16 [T][K]); returns (packed u32 as int32, steps, zeros) in the layout of
    wq_quantize_pack. `workspace` (uint8, >= wq_gptq_workspace_bytes) is
    allocated when not given."""
    _check(W, torch.float16, "W")
    _check(X, torch.float16, "X")
    if W.dim() != 2 or X.dim() != 2 or X.shape[1] != W.shape[1]:
        raise ValueError(f"W must be [N][K] and X [T][K], got {tuple(W.shape)} and {tuple(X.shape)}")
    N, K = W.shape
    T = X.shape[0]
    c = _cfg(bits, group_size, symmetric)
    nw = _packed_words_of(N, K, c)
    if out is None:
        G = K // group_size if group_size > 0 else 0
        packed = torch.empty(max(nw, 1), dtype=torch.int32, device=W.device)
        steps = torch.empty((N, G), dtype=torch.float16, device=W.device)
        zeros = torch.empty((N, G), dtype=torch.float16, device=W.device)
    else:
        packed, steps, zeros = out
        _quant_operands(N, K, c, packed, steps, zeros)
    need = int(_lib.wq_gptq_workspace_bytes(N, K, ctypes.byref(c)))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=W.device)
    elif not workspace.is_contiguous():
        raise ValueError("workspace must be contiguous")
    _on_device_of(W, X=X, packed=packed, steps=steps, zeros=zeros, workspace=workspace)
    with _device_of(W):
        st = _lib.wq_gptq_quantize_pack(_ptr(X), T, _ptr(W), N, K, ctypes.byref(c), float(damp), _ptr(packed),
                                        _ptr(steps), _ptr(zeros), workspace.data_ptr(),
                                        workspace.numel() * workspace.element_size(), _stream(stream, W.device.index))
    _raise(st, "wq_gptq_quantize_pack")
    return packed, steps, zeros


def wq_quantize_act_int8(X: torch.Tensor, *, group_size: int = 32, out=None, stream=None):
    """int8 codes and fp32 multipliers of fp16 activations X [M][K], one
    multiplier per row and group; returns (q int8 [M][K], mult fp32 [M][K/group])."""
    _check(X, torch.float16, "X")
    if X.dim() != 2:
        raise ValueError(f"X must be [M][K], got shape {tuple(X.shape)}")
    M, K = X.shape
    if out is None:
        q = torch.empty((M, K), dtype=torch.int8, device=X.device)
        mult = torch.empty((M, K // group_size if group_size > 0 else 0), dtype=torch.float32, device=X.device)
    else:
        q, mult = out
        _need(q, "q", torch.int8, M * K)
        _need(mult, "mult", torch.float32, 4 * M * (K // group_size))
    _on_device_of(X, q=q, mult=mult)
    with _device_of(X):
        st = _lib.wq_quantize_act_int8(_ptr(X), M, K, group_size, _ptr(q), _ptr(mult), _stream(stream, X.device.index))
    _raise(st, "wq_quantize_act_int8")
    return q, mult


def wq_w4a8_gemm(q: torch.Tensor, mult: torch.Tensor, packed: torch.Tensor, steps: torch.Tensor,
                 zeros: torch.Tensor, N: int, *, group_size: int = 32, symmetric: bool = False, out=None,
                 stream=None):
    """Y [M][N] fp16 from int8 activation codes (wq_quantize_act_int8) and a
    4-bit packed weight of the same group size."""
    _check(q, torch.int8, "q")
    if q.dim() != 2:
        raise ValueError(f"q must be [M][K], got shape {tuple(q.shape)}")
    M, K = q.shape
    c = _cfg(4, group_size, symmetric)
    _quant_operands(N, K, c, packed, steps, zeros)
    _need(mult, "mult", torch.float32, 4 * M * (K // group_size))
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=q.device)
    _need(out, "out", torch.float16, 2 * M * N)
    _on_device_of(q, mult=mult, packed=packed, steps=steps, zeros=zeros, out=out)
    with _device_of(q):
        st = _lib.wq_w4a8_gemm(_ptr(q), _ptr(mult), _ptr(packed), _ptr(steps), _ptr(zeros), M, N, K,
                               ctypes.byref(c), _ptr(out), _stream(stream, q.device.index))
    _raise(st, "wq_w4a8_gemm")
    return out
