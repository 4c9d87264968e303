"""FlashNorm RMSNorm -> linear on B200: a thin binding of the C ABI in include/flashnorm.h.

Each function here has the name of the C entry point it calls and only marshals arguments: it
checks that the torch tensors are CUDA bf16 / fp32, contiguous and on one device, allocates outputs
the caller did not pass, makes that device current, and hands raw pointers plus its current CUDA
stream to libflashnorm.so. All arithmetic
runs in the library's sm_100a kernels; there is no fallback of any kind. If the library is missing,
importing works but every call raises.

    Wstar = flashnorm_fold_weights(W, g)             # W [d, N] bf16, g [d] bf16 -> W* [N, d]
    y = flashnorm_linear(x, Wstar, eps)              # x [M, d] bf16 -> y [M, N]
    Wgu = flashnorm_fold_weights(W_gu, g, glu=True)  # W_gu [d, 2F]: gate | up
    y = flashnorm_glu(x, Wgu, eps)                   # -> y [M, F]
    y = flashnorm_linear_postnorm(x, Wstar, g2, head_dim, eps2)
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

__all__ = [
    "FlashNormError",
    "library_path",
    "load_library",
    "flashnorm_fold_weights",
    "flashnorm_linear",
    "flashnorm_glu",
    "flashnorm_linear_postnorm",
    "flashnorm_postnorm_workspace_bytes",
    "flashnorm_linear_postnorm_rope",
    "flashnorm_rope_table",
    "flashnorm_fold_layernorm",
    "flashnorm_fold_weights_fp8",
    "flashnorm_linear_fp8",
    "flashnorm_fp8_workspace_bytes",
    "flashnorm_fold_weights_nvfp4",
    "flashnorm_linear_nvfp4",
    "flashnorm_nvfp4_workspace_bytes",
    "flashnorm_layernorm_linear",
    "flashnorm_rmsnorm",
    "flashnorm_linear_unfused",
    "flashnorm_glu_unfused",
    "flashnorm_linear_unfused_noalloc",
    "NOALLOC_MAX_ELEMS",
    "flashnorm_check_device_error",
    "flashnorm_selftest_timeout",
    "flashnorm_version",
    "prepare",
    "PreparedCall",
    "EXPORTED_SYMBOLS",
]

_PKG_DIR = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_PKG_DIR, "libflashnorm.so")

FN_OK, FN_ERR_INVALID_ARG, FN_ERR_UNSUPPORTED, FN_ERR_ALIGN, FN_ERR_CUDA, FN_ERR_TIMEOUT = range(6)
FN_BF16, FN_F32 = 0, 1
NOALLOC_MAX_ELEMS = 1 << 23  # FN_NOALLOC_MAX_ELEMS in include/flashnorm.h
PATHS = {"auto": 0, "tensor": 1, "gemv": 2, "decode": 3, "pair": 4}

_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_F = ctypes.c_float
_INT = ctypes.c_int

# name -> argtypes; restype is fn_status (int) unless listed in _RESTYPES
_SIGNATURES = {
    "flashnorm_fold_weights": [_P, _P, _P, _I64, _I64, _INT, _P],
    "flashnorm_linear": [_P, _P, _P, _I64, _I64, _I64, _F, _INT, _P],
    "flashnorm_linear_ex": [_P, _P, _P, _I64, _I64, _I64, _F, _INT, _INT, _P],
    "flashnorm_glu": [_P, _P, _P, _I64, _I64, _I64, _F, _INT, _P],
    "flashnorm_glu_ex": [_P, _P, _P, _I64, _I64, _I64, _F, _INT, _INT, _P],
    "flashnorm_linear_postnorm": [_P, _P, _P, _P, _I64, _I64, _I64, _I64, _F, _INT, _P],
    "flashnorm_linear_postnorm_ws": [_P, _P, _P, _P, _I64, _I64, _I64, _I64, _F, _INT, _P, _I64, _P],
    "flashnorm_postnorm_workspace_bytes": [_I64, _I64, _I64, _I64, _P],
    "flashnorm_linear_postnorm_rope": [_P, _P, _P, _P, _P, _P, _I64, _I64, _I64, _I64, _I64, _I64, _F, _INT, _P],
    "flashnorm_rope_table": [_P, _I64, _I64, ctypes.c_double, _P],
    "flashnorm_fold_layernorm": [_P, _P, _P, _P, _P, _P, _I64, _I64, _P],
    "flashnorm_fold_weights_fp8": [_P, _P, _P, _P, _I64, _I64, _P],
    "flashnorm_linear_fp8": [_P, _P, _P, _P, _I64, _I64, _I64, _F, _INT, _P],
    "flashnorm_linear_fp8_ex": [_P, _P, _P, _P, _I64, _I64, _I64, _F, _INT, _INT, _P],
    "flashnorm_linear_fp8_ws": [_P, _P, _P, _P, _I64, _I64, _I64, _F, _INT, _INT, _P, _I64, _P],
    "flashnorm_fp8_workspace_bytes": [_I64, _I64, _I64, _P],
    "flashnorm_fold_weights_nvfp4": [_P, _P, _P, _P, _I64, _I64, _P],
    "flashnorm_linear_nvfp4": [_P, _P, _P, _P, _I64, _I64, _I64, _F, _INT, _P, _I64, _P],
    "flashnorm_nvfp4_workspace_bytes": [_I64, _I64, _I64, _P],
    "flashnorm_layernorm_linear": [_P, _P, _P, _P, _P, _I64, _I64, _I64, _F, _INT, _P],
    "flashnorm_rmsnorm": [_P, _P, _P, _I64, _I64, _F, _P],
    "flashnorm_linear_unfused": [_P, _P, _P, _P, _P, _I64, _I64, _I64, _F, _INT, _P],
    "flashnorm_glu_unfused": [_P, _P, _P, _P, _P, _I64, _I64, _I64, _F, _INT, _P],
    "flashnorm_linear_unfused_noalloc": [_P, _P, _P, _P, _I64, _I64, _I64, _F, _INT, _P],
    "flashnorm_check_device_error": [_P],
    "flashnorm_selftest_timeout": [_I64, _P],
    "flashnorm_status_string": [_INT],
    "flashnorm_last_error": [],
    "flashnorm_version": [],
}
_RESTYPES = {"flashnorm_status_string": ctypes.c_char_p, "flashnorm_last_error": ctypes.c_char_p}
EXPORTED_SYMBOLS = tuple(_SIGNATURES)

_lib = None


class FlashNormError(RuntimeError):
    """A library call returned a status other than FN_OK."""

    def __init__(self, fn_name: str, status: int, detail: str):
        self.status = status
        super().__init__(f"{fn_name} failed with status {status}: {detail}")


def library_path() -> str:
    return _LIB_PATH


def load_library() -> ctypes.CDLL:
    """Load libflashnorm.so (once). Raises if it has not been built."""
    global _lib
    if _lib is None:
        if not os.path.exists(_LIB_PATH):
            raise FlashNormError("load_library", -1, f"{_LIB_PATH} is missing; build it with "
                                 "`python -m rmsnorm_linear_projection_fold_b200.build`")
        lib = ctypes.CDLL(_LIB_PATH)
        for name, args in _SIGNATURES.items():
            f = getattr(lib, name)
            f.argtypes = args
            f.restype = _RESTYPES.get(name, ctypes.c_int)
        _lib = lib
    return _lib


def _check(name: str, status: int) -> None:
    if status != FN_OK:
        lib = load_library()
        detail = lib.flashnorm_last_error().decode() or lib.flashnorm_status_string(status).decode()
        raise FlashNormError(name, status, detail)


def _same_device(lead: torch.Tensor, **others) -> None:
    """Every tensor of a call must live on the device of `lead` (the C ABI takes bare pointers)."""
    ld = lead.get_device()  # the CUDA device index, or -1 for any other device (compared in full below)
    for name, t in others.items():
        if t is not None and (ld < 0 or t.get_device() != ld) and t.device != lead.device:
            raise ValueError(f"{name} is on {t.device}, expected {lead.device}")


def _invoke(entry: str, lead: torch.Tensor, *args, report: str | None = None) -> None:
    """Call the library's `entry` with `lead`'s device current: the library launches on, and looks up
    its per-device state for, the current device."""
    _invoke_on(lead.get_device(), entry, *args, report=report)


# While prepare() records, on its own thread: the library calls made (size queries excepted) and every
# tensor whose address was taken, which the prepared call keeps alive. Thread-local, so that calls made by
# other threads meanwhile run as usual.
_rec = threading.local()


def _recording():
    return getattr(_rec, "calls", None)


def _invoke_on(dev: int, entry: str, *args, report: str | None = None) -> None:
    calls = _recording()
    if calls is not None and not entry.endswith("_workspace_bytes"):
        calls.append((dev, entry, args, report or entry))
        return
    lib = load_library()
    if dev == torch.cuda.current_device():
        status = getattr(lib, entry)(*args)
    else:
        with torch.cuda.device(dev):
            status = getattr(lib, entry)(*args)
    _check(report or entry, status)


# The current stream's cudaStream_t as an integer; torch's internal accessor skips building a Stream object
# (about 2 us a call), with the public route where it is absent.
_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream_ptr(t: torch.Tensor):
    if _raw_stream is not None:
        return _raw_stream(t.get_device())
    return torch.cuda.current_stream(t.device).cuda_stream


def _ptr(t):
    """A tensor's device address for a void* argument (None passes NULL)."""
    if t is None:
        return None
    keep = getattr(_rec, "keep", None)
    if keep is not None:
        keep.append(t)
    return t.data_ptr()


class PreparedCall:
    """One library call whose checks and argument marshalling were done once (see prepare). Calling it
    launches the same C-ABI entry point with the same device pointers on the same stream and returns the
    output tensor of the original call; it keeps every tensor whose address it holds alive."""

    __slots__ = ("_fn", "_args", "_dev", "_report", "_keep", "result", "entry")

    def __init__(self, fn, args, dev, report, keep, result, entry):
        self._fn, self._args, self._dev, self._report = fn, args, dev, report
        self._keep, self.result, self.entry = keep, result, entry

    def __call__(self):
        if self._dev == torch.cuda.current_device():
            status = self._fn(*self._args)
        else:
            with torch.cuda.device(self._dev):
                status = self._fn(*self._args)
        _check(self._report, status)
        return self.result


def prepare(func, *args, **kwargs) -> PreparedCall:
    """Plan once, launch many: run func(*args, **kwargs), one of this module's calls that launch work (a
    projection, a fold, the RMSNorm), for its checks and argument marshalling only, and return a
    PreparedCall that launches that call again at the cost of one C call. For loops that repeat one call
    on the same buffers (a serving step, a benchmark). What is fixed at this point: the device addresses
    (rewrite the inputs in place, and read the outputs from .result), the stream (the one current now),
    and any scratch the call chose (a workspace="auto" buffer is allocated here and kept)."""
    if _recording() is not None:
        raise RuntimeError("prepare() does not nest")
    rec, keep = [], []
    _rec.calls, _rec.keep = rec, keep
    try:
        result = func(*args, **kwargs)
    finally:
        _rec.calls, _rec.keep = None, None
    if len(rec) != 1:
        raise ValueError(f"prepare() takes a call that makes one library call; this one made {len(rec)}")
    dev, entry, cargs, report = rec[0]
    f = getattr(load_library(), entry)
    # ctypes skips its per-call conversion for arguments that already have the declared types
    conv = tuple(a if isinstance(a, t) else t(a) for t, a in zip(f.argtypes, cargs))
    return PreparedCall(f, conv, dev, report, keep, result, entry)


def _need(t: torch.Tensor, name: str, dtype=torch.bfloat16, dim=None) -> None:
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dimensions, got shape {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _out_code(out_dtype) -> int:
    if out_dtype == torch.bfloat16:
        return FN_BF16
    if out_dtype == torch.float32:
        return FN_F32
    raise TypeError("out_dtype must be torch.bfloat16 or torch.float32")


def _output(out, shape, dtype, like):
    if out is None:
        return torch.empty(shape, dtype=dtype, device=like.device)
    _need(out, "out", dtype)
    if tuple(out.shape) != tuple(shape):
        raise ValueError(f"out must have shape {tuple(shape)}, got {tuple(out.shape)}")
    _same_device(like, out=out)
    return out


def flashnorm_fold_weights(W: torch.Tensor, g: torch.Tensor, glu: bool = False, out=None) -> torch.Tensor:
    """W* = diag(g) . W rounded once to bf16, stored K-major [N, d] (GLU: gate/up interleaved)."""
    _need(W, "W", dim=2)
    _need(g, "g", dim=1)
    d, N = W.shape
    if g.shape[0] != d:
        raise ValueError("g must have d elements")
    _same_device(W, g=g)
    out = _output(out, (N, d), torch.bfloat16, W)
    _invoke("flashnorm_fold_weights", W, _ptr(W), _ptr(g), _ptr(out), d, N, int(bool(glu)), _stream_ptr(W))
    return out


def flashnorm_linear(x: torch.Tensor, Wstar: torch.Tensor, eps: float, out_dtype=torch.bfloat16, out=None,
                     path: str = "auto") -> torch.Tensor:
    """y = (x . W*) * 1/sqrt(mean(x^2) + eps); x [M, d] bf16, W* [N, d] from fold_weights."""
    _need(x, "x", dim=2)
    _need(Wstar, "Wstar", dim=2)
    M, d = x.shape
    N = Wstar.shape[0]
    if Wstar.shape[1] != d:
        raise ValueError("Wstar must be [N, d] with the d of x")
    _same_device(x, Wstar=Wstar)
    y = _output(out, (M, N), out_dtype, x)
    _invoke("flashnorm_linear_ex", x, _ptr(x), _ptr(Wstar), _ptr(y), M, d, N, float(eps), _out_code(out_dtype),
            PATHS[path], _stream_ptr(x), report="flashnorm_linear")
    return y


def flashnorm_glu(x: torch.Tensor, Wstar_gu: torch.Tensor, eps: float, out_dtype=torch.bfloat16, out=None,
                  path: str = "auto") -> torch.Tensor:
    """y = silu(r * x.W*_gate) * (r * x.W*_up), r = 1/sqrt(mean(x^2)+eps); W*_gu [2F, d] from fold(glu=True)."""
    _need(x, "x", dim=2)
    _need(Wstar_gu, "Wstar_gu", dim=2)
    M, d = x.shape
    if Wstar_gu.shape[1] != d or Wstar_gu.shape[0] % 2:
        raise ValueError("Wstar_gu must be [2F, d] with the d of x")
    F = Wstar_gu.shape[0] // 2
    _same_device(x, Wstar_gu=Wstar_gu)
    y = _output(out, (M, F), out_dtype, x)
    _invoke("flashnorm_glu_ex", x, _ptr(x), _ptr(Wstar_gu), _ptr(y), M, d, F, float(eps), _out_code(out_dtype),
            PATHS[path], _stream_ptr(x), report="flashnorm_glu")
    return y


_ws_bytes_cache = {}


def flashnorm_postnorm_workspace_bytes(M: int, d: int, N: int, head_dim: int, device=None) -> int:
    """Workspace bytes flashnorm_linear_postnorm uses for this shape on `device` (0: no split)."""
    dev = torch.cuda.current_device() if device is None else torch.device(device).index
    if dev is None:
        dev = torch.cuda.current_device()
    key = (dev, int(M), int(d), int(N), int(head_dim))
    hit = _ws_bytes_cache.get(key)
    if hit is not None:
        return hit
    nbytes = ctypes.c_int64(0)
    _invoke_on(dev, "flashnorm_postnorm_workspace_bytes", int(M), int(d), int(N), int(head_dim),
               ctypes.addressof(nbytes))
    _ws_bytes_cache[key] = int(nbytes.value)  # a function of the shape and the device's SM count only
    return int(nbytes.value)


def flashnorm_linear_postnorm(x: torch.Tensor, Wstar: torch.Tensor, g2: torch.Tensor, head_dim: int, eps2: float,
                              out_dtype=torch.bfloat16, out=None, workspace="auto") -> torch.Tensor:
    """Per-head RMSNorm(x . W*; g2, eps2) with the first RMSNorm elided (its gain folded into W*).

    workspace: "auto" allocates the scratch that lets a wide head (256 < head_dim <= 512) with few row
    tiles split its contraction over the whole device (flashnorm_postnorm_workspace_bytes; nothing for
    other shapes); None runs without one (a wide head then stays in one thread-block cluster per row tile);
    or a caller-owned uint8 CUDA tensor of at least that many bytes."""
    _need(x, "x", dim=2)
    _need(Wstar, "Wstar", dim=2)
    _need(g2, "g2", dim=1)
    M, d = x.shape
    N = Wstar.shape[0]
    if Wstar.shape[1] != d:
        raise ValueError("Wstar must be [N, d] with the d of x")
    if g2.shape[0] != head_dim:
        raise ValueError("g2 must have head_dim elements")
    _same_device(x, Wstar=Wstar, g2=g2)
    y = _output(out, (M, N), out_dtype, x)
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError('workspace must be "auto", None or a uint8 CUDA tensor')
        nbytes = flashnorm_postnorm_workspace_bytes(M, d, N, head_dim, x.get_device()) if M > 0 else 0
        ws = torch.empty(nbytes, dtype=torch.uint8, device=x.device) if nbytes > 0 else None
    elif workspace is None:
        ws = None
    else:
        _need(workspace, "workspace", torch.uint8, dim=1)
        _same_device(x, workspace=workspace)
        ws = workspace
    _invoke("flashnorm_linear_postnorm_ws", x, _ptr(x), _ptr(Wstar), _ptr(g2), _ptr(y), M, d, N, int(head_dim),
            float(eps2), _out_code(out_dtype), _ptr(ws), ws.numel() if ws is not None else 0, _stream_ptr(x),
            report="flashnorm_linear_postnorm")
    return y


def flashnorm_fold_weights_fp8(W: torch.Tensor, g: torch.Tensor):
    """(Q uint8 [N, d] E4M3 codes, scales fp32 [N]): the gain fold, then per-channel FP8 quantization."""
    _need(W, "W", dim=2)
    _need(g, "g", dim=1)
    d, N = W.shape
    if g.shape[0] != d:
        raise ValueError("g must have d elements")
    _same_device(W, g=g)
    Q = torch.empty(N, d, dtype=torch.uint8, device=W.device)
    scales = torch.empty(N, dtype=torch.float32, device=W.device)
    _invoke("flashnorm_fold_weights_fp8", W, _ptr(W), _ptr(g), _ptr(Q), _ptr(scales), d, N, _stream_ptr(W))
    return Q, scales


_fp8_ws_bytes_cache = {}
_fp8_ws_cache = {}


def flashnorm_fp8_workspace_bytes(M: int, d: int, N: int, device=None) -> int:
    """Workspace bytes flashnorm_linear_fp8 uses for this shape on `device` (0: no split)."""
    dev = torch.cuda.current_device() if device is None else torch.device(device).index
    if dev is None:
        dev = torch.cuda.current_device()
    key = (dev, int(M), int(d), int(N))
    hit = _fp8_ws_bytes_cache.get(key)
    if hit is not None:
        return hit
    nbytes = ctypes.c_int64(0)
    _invoke_on(dev, "flashnorm_fp8_workspace_bytes", int(M), int(d), int(N), ctypes.addressof(nbytes))
    _fp8_ws_bytes_cache[key] = int(nbytes.value)  # a function of the shape and the device's SM count only
    return int(nbytes.value)


def _fp8_stream_workspace(x: torch.Tensor, nbytes: int) -> torch.Tensor:
    """A zero-initialised workspace of at least `nbytes` kept for x's device and current stream. Calls on
    one stream run in order, and each leaves the workspace's counters at zero, so they can share it."""
    key = (x.get_device(), _stream_ptr(x))
    ws = _fp8_ws_cache.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=x.device)
        _fp8_ws_cache[key] = ws
    return ws


def flashnorm_linear_fp8(x: torch.Tensor, Q: torch.Tensor, scales: torch.Tensor, eps: float,
                         out_dtype=torch.bfloat16, out=None, path: str = "auto", workspace="auto") -> torch.Tensor:
    """Decode (M <= 16) with FP8 weights: y = (x . dec(Q)^T) * scales * 1/sqrt(mean(x^2) + eps).

    path "decode": the tensor-core kernel; "gemv": the CUDA-core GEMV; "auto": the tensor-core kernel,
    except for one token without a workspace (the GEMV).
    workspace: "auto" uses a zero-initialised scratch kept per device and stream, which lets the
    tensor-core kernel split its contraction over independent CTAs (flashnorm_fp8_workspace_bytes; nothing
    for shapes that do not split); None runs without one (the split then stays inside thread-block
    clusters); or a caller-owned uint8 CUDA tensor of at least that many bytes whose first 1024 bytes were
    zero before its first use (every call leaves them zero)."""
    _need(x, "x", dim=2)
    _need(Q, "Q", torch.uint8, dim=2)
    _need(scales, "scales", torch.float32, dim=1)
    M, d = x.shape
    N = Q.shape[0]
    if Q.shape[1] != d or scales.shape[0] != N:
        raise ValueError("Q [N, d] and scales [N] must match x [M, d]")
    _same_device(x, Q=Q, scales=scales)
    y = _output(out, (M, N), out_dtype, x)
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError('workspace must be "auto", None or a uint8 CUDA tensor')
        # the CUDA-core GEMV takes no workspace
        nbytes = flashnorm_fp8_workspace_bytes(M, d, N, x.get_device()) if 0 < M <= 16 and path != "gemv" else 0
        ws = _fp8_stream_workspace(x, nbytes) if nbytes > 0 else None
    elif workspace is None:
        ws = None
    else:
        _need(workspace, "workspace", torch.uint8, dim=1)
        _same_device(x, workspace=workspace)
        ws = workspace
    _invoke("flashnorm_linear_fp8_ws", x, _ptr(x), _ptr(Q), _ptr(scales), _ptr(y), M, d, N, float(eps),
            _out_code(out_dtype), PATHS[path], _ptr(ws), ws.numel() if ws is not None else 0, _stream_ptr(x),
            report="flashnorm_linear_fp8")
    return y


NVFP4_GROUP, NVFP4_GROUP_BYTES = 256, 144  # k per stored group and its bytes (include/flashnorm.h)


def flashnorm_fold_weights_nvfp4(W: torch.Tensor, g: torch.Tensor):
    """(Q4 uint8 [N, ceil(d/256) * 144], s2 fp32 [N]): the gain fold, then NVFP4 quantization (E2M1 codes,
    E4M3 scales per 16 k, a fp32 scale per output channel), in the layout include/flashnorm.h states."""
    _need(W, "W", dim=2)
    _need(g, "g", dim=1)
    d, N = W.shape
    if g.shape[0] != d:
        raise ValueError("g must have d elements")
    _same_device(W, g=g)
    groups = -(-d // NVFP4_GROUP)
    Q4 = torch.empty(N, groups * NVFP4_GROUP_BYTES, dtype=torch.uint8, device=W.device)
    s2 = torch.empty(N, dtype=torch.float32, device=W.device)
    _invoke("flashnorm_fold_weights_nvfp4", W, _ptr(W), _ptr(g), _ptr(Q4), _ptr(s2), d, N, _stream_ptr(W))
    return Q4, s2


_nvfp4_ws_bytes_cache = {}


def flashnorm_nvfp4_workspace_bytes(M: int, d: int, N: int, device=None) -> int:
    """Workspace bytes flashnorm_linear_nvfp4 uses for this shape on `device` (0: no split)."""
    dev = torch.cuda.current_device() if device is None else torch.device(device).index
    if dev is None:
        dev = torch.cuda.current_device()
    key = (dev, int(M), int(d), int(N))
    hit = _nvfp4_ws_bytes_cache.get(key)
    if hit is not None:
        return hit
    nbytes = ctypes.c_int64(0)
    _invoke_on(dev, "flashnorm_nvfp4_workspace_bytes", int(M), int(d), int(N), ctypes.addressof(nbytes))
    _nvfp4_ws_bytes_cache[key] = int(nbytes.value)
    return int(nbytes.value)


def flashnorm_linear_nvfp4(x: torch.Tensor, Q4: torch.Tensor, s2: torch.Tensor, eps: float,
                           out_dtype=torch.bfloat16, out=None, workspace="auto") -> torch.Tensor:
    """Decode (M <= 16) with NVFP4 weights on the tensor cores:
    y = (x . (Q * sb)^T) * s2 * 1/sqrt(mean(x^2) + eps).

    workspace: as for flashnorm_linear_fp8 ("auto": a zero-initialised scratch kept per device and stream;
    None: one CTA per 128-row slab over all of d; or a caller-owned uint8 CUDA tensor)."""
    _need(x, "x", dim=2)
    _need(Q4, "Q4", torch.uint8, dim=2)
    _need(s2, "s2", torch.float32, dim=1)
    M, d = x.shape
    N = Q4.shape[0]
    if Q4.shape[1] != -(-d // NVFP4_GROUP) * NVFP4_GROUP_BYTES or s2.shape[0] != N:
        raise ValueError("Q4 [N, ceil(d/256) * 144] and s2 [N] must match x [M, d]")
    _same_device(x, Q4=Q4, s2=s2)
    y = _output(out, (M, N), out_dtype, x)
    if isinstance(workspace, str):
        if workspace != "auto":
            raise ValueError('workspace must be "auto", None or a uint8 CUDA tensor')
        nbytes = flashnorm_nvfp4_workspace_bytes(M, d, N, x.get_device()) if 0 < M <= 16 else 0
        ws = _fp8_stream_workspace(x, nbytes) if nbytes > 0 else None
    elif workspace is None:
        ws = None
    else:
        _need(workspace, "workspace", torch.uint8, dim=1)
        _same_device(x, workspace=workspace)
        ws = workspace
    _invoke("flashnorm_linear_nvfp4", x, _ptr(x), _ptr(Q4), _ptr(s2), _ptr(y), M, d, N, float(eps),
            _out_code(out_dtype), _ptr(ws), ws.numel() if ws is not None else 0, _stream_ptr(x),
            report="flashnorm_linear_nvfp4")
    return y


def flashnorm_fold_layernorm(W: torch.Tensor, gamma: torch.Tensor, beta=None):
    """LayerNorm fold: (W* [N, d] bf16, colsum [N] fp32, bias [N] fp32) from W [d, N], gamma [d], beta [d] or None."""
    _need(W, "W", dim=2)
    _need(gamma, "gamma", dim=1)
    d, N = W.shape
    if gamma.shape[0] != d:
        raise ValueError("gamma must have d elements")
    if beta is not None:
        _need(beta, "beta", dim=1)
        if beta.shape[0] != d:
            raise ValueError("beta must have d elements")
    _same_device(W, gamma=gamma, beta=beta)
    Ws = torch.empty(N, d, dtype=torch.bfloat16, device=W.device)
    colsum = torch.empty(N, dtype=torch.float32, device=W.device)
    bias = torch.empty(N, dtype=torch.float32, device=W.device)
    _invoke("flashnorm_fold_layernorm", W, _ptr(W), _ptr(gamma), _ptr(beta), _ptr(Ws), _ptr(colsum), _ptr(bias), d,
            N, _stream_ptr(W))
    return Ws, colsum, bias


def flashnorm_layernorm_linear(x: torch.Tensor, Wstar: torch.Tensor, colsum: torch.Tensor, bias: torch.Tensor,
                               eps: float, out_dtype=torch.bfloat16, out=None) -> torch.Tensor:
    """y = LayerNorm(x; gamma, beta) . W from the folded (W*, colsum, bias) of flashnorm_fold_layernorm."""
    _need(x, "x", dim=2)
    _need(Wstar, "Wstar", dim=2)
    _need(colsum, "colsum", torch.float32, dim=1)
    _need(bias, "bias", torch.float32, dim=1)
    M, d = x.shape
    N = Wstar.shape[0]
    if Wstar.shape[1] != d or colsum.shape[0] != N or bias.shape[0] != N:
        raise ValueError("Wstar [N, d], colsum [N] and bias [N] must match x [M, d]")
    _same_device(x, Wstar=Wstar, colsum=colsum, bias=bias)
    y = _output(out, (M, N), out_dtype, x)
    _invoke("flashnorm_layernorm_linear", x, _ptr(x), _ptr(Wstar), _ptr(colsum), _ptr(bias), _ptr(y), M, d, N,
            float(eps), _out_code(out_dtype), _stream_ptr(x))
    return y


def flashnorm_rope_table(max_pos: int, head_dim: int, base: float = 10000.0, device=None, out=None) -> torch.Tensor:
    """(cos, sin) of the rotary angles p * base^(-2i/head_dim), fp32 [max_pos, head_dim/2, 2], on the GPU."""
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
    if out is None:
        out = torch.empty(max_pos, head_dim // 2, 2, dtype=torch.float32, device=dev)
    else:
        _need(out, "out", torch.float32)
        if tuple(out.shape) != (max_pos, head_dim // 2, 2):
            raise ValueError("out must be [max_pos, head_dim / 2, 2]")
    _invoke("flashnorm_rope_table", out, _ptr(out), int(max_pos), int(head_dim), float(base), _stream_ptr(out))
    return out


def flashnorm_linear_postnorm_rope(x: torch.Tensor, Wstar: torch.Tensor, g2: torch.Tensor, rope_cs: torch.Tensor,
                                   positions: torch.Tensor, head_dim: int, n_rope_heads: int, eps2: float,
                                   out_dtype=torch.bfloat16, out=None) -> torch.Tensor:
    """flashnorm_linear_postnorm, then RoPE on the first n_rope_heads heads of every row.

    rope_cs: fp32 [max_pos, head_dim/2, 2] from flashnorm_rope_table; positions: int32 [M] on the GPU.
    """
    _need(x, "x", dim=2)
    _need(Wstar, "Wstar", dim=2)
    _need(g2, "g2", dim=1)
    _need(rope_cs, "rope_cs", torch.float32, dim=3)
    _need(positions, "positions", torch.int32, dim=1)
    M, d = x.shape
    N = Wstar.shape[0]
    if Wstar.shape[1] != d:
        raise ValueError("Wstar must be [N, d] with the d of x")
    if g2.shape[0] != head_dim:
        raise ValueError("g2 must have head_dim elements")
    if positions.shape[0] != M:
        raise ValueError("positions must have one entry per row of x")
    if rope_cs.shape[1:] != (head_dim // 2, 2):
        raise ValueError("rope_cs must be [max_pos, head_dim / 2, 2]")
    _same_device(x, Wstar=Wstar, g2=g2, rope_cs=rope_cs, positions=positions)
    y = _output(out, (M, N), out_dtype, x)
    _invoke("flashnorm_linear_postnorm_rope", x, _ptr(x), _ptr(Wstar), _ptr(g2), _ptr(rope_cs), _ptr(positions),
            _ptr(y), M, d, N, int(head_dim), int(n_rope_heads), int(rope_cs.shape[0]), float(eps2),
            _out_code(out_dtype), _stream_ptr(x))
    return y


def flashnorm_rmsnorm(x: torch.Tensor, g: torch.Tensor, eps: float, out=None) -> torch.Tensor:
    """xn = bf16(x / sqrt(mean(x^2) + eps) * g), the first kernel of the unfused baseline."""
    _need(x, "x", dim=2)
    _need(g, "g", dim=1)
    M, d = x.shape
    _same_device(x, g=g)
    xn = _output(out, (M, d), torch.bfloat16, x)
    _invoke("flashnorm_rmsnorm", x, _ptr(x), _ptr(g), _ptr(xn), M, d, float(eps), _stream_ptr(x))
    return xn


def flashnorm_linear_unfused(x, g, W_kmajor, eps, xn_ws=None, out_dtype=torch.bfloat16, out=None):
    """Unfused baseline: xn = RMSNorm(x; g) in bf16, then y = xn . W (W_kmajor = fold(W, ones))."""
    _need(x, "x", dim=2)
    _need(g, "g", dim=1)
    _need(W_kmajor, "W_kmajor", dim=2)
    M, d = x.shape
    N = W_kmajor.shape[0]
    _same_device(x, g=g, W_kmajor=W_kmajor)
    xn_ws = _output(xn_ws, (M, d), torch.bfloat16, x)
    y = _output(out, (M, N), out_dtype, x)
    _invoke("flashnorm_linear_unfused", x, _ptr(x), _ptr(g), _ptr(W_kmajor), _ptr(xn_ws), _ptr(y), M, d, N,
            float(eps), _out_code(out_dtype), _stream_ptr(x))
    return y


def flashnorm_glu_unfused(x, g, W_kmajor_gu, eps, xn_ws=None, out_dtype=torch.bfloat16, out=None):
    """Unfused GLU baseline: xn = RMSNorm(x; g) in bf16, then silu(xn.W_gate) * (xn.W_up)."""
    _need(x, "x", dim=2)
    _need(g, "g", dim=1)
    _need(W_kmajor_gu, "W_kmajor_gu", dim=2)
    M, d = x.shape
    F = W_kmajor_gu.shape[0] // 2
    _same_device(x, g=g, W_kmajor_gu=W_kmajor_gu)
    xn_ws = _output(xn_ws, (M, d), torch.bfloat16, x)
    y = _output(out, (M, F), out_dtype, x)
    _invoke("flashnorm_glu_unfused", x, _ptr(x), _ptr(g), _ptr(W_kmajor_gu), _ptr(xn_ws), _ptr(y), M, d, F,
            float(eps), _out_code(out_dtype), _stream_ptr(x))
    return y


def flashnorm_linear_unfused_noalloc(x, g, W_kmajor, eps, out_dtype=torch.bfloat16, out=None):
    """flashnorm_linear_unfused with the library's own fixed scratch instead of a workspace argument.

    For callers that cannot allocate device memory on this path (no workspace in their interface, or
    all memory owned by their own pool). M * d must be at most NOALLOC_MAX_ELEMS. Calls share one
    scratch array per device: calls that overlap on the GPU race, so keep them on one stream. Passing
    `out` makes the whole call allocation-free on the Python side too.
    """
    _need(x, "x", dim=2)
    _need(g, "g", dim=1)
    _need(W_kmajor, "W_kmajor", dim=2)
    M, d = x.shape
    N = W_kmajor.shape[0]
    _same_device(x, g=g, W_kmajor=W_kmajor)
    y = _output(out, (M, N), out_dtype, x)
    _invoke("flashnorm_linear_unfused_noalloc", x, _ptr(x), _ptr(g), _ptr(W_kmajor), _ptr(y), M, d, N, float(eps),
            _out_code(out_dtype), _stream_ptr(x))
    return y


def flashnorm_check_device_error(device=None) -> None:
    """Synchronise the current stream and raise if a kernel gave up on a bounded wait."""
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
    lib = load_library()
    s = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    with torch.cuda.device(dev):  # the status word read is the current device's
        status = lib.flashnorm_check_device_error(s)
    _check("flashnorm_check_device_error", status)


def flashnorm_selftest_timeout(limit_us: int = 20000, device=None) -> int:
    """Run the bounded-wait self-test; returns the status the library reported (FN_ERR_TIMEOUT when the
    failure path works). Does not raise for that status."""
    dev = torch.device("cuda", torch.cuda.current_device() if device is None else device)
    lib = load_library()
    s = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    with torch.cuda.device(dev):
        return int(lib.flashnorm_selftest_timeout(int(limit_us), s))


def flashnorm_version() -> int:
    return int(load_library().flashnorm_version())
