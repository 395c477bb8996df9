"""Python binding of libmxq (include/mxq.h): NVFP4 / MXFP8 microscaled linear
layers on B200 (sm_100a).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of ``libmxq.so``.  PyTorch is used for device memory and streams
(tensors are passed as device pointers).  There is no CPU fallback: importing
this package fails loudly when the library has not been built.

Functions keep the C names without the ``mxq_`` prefix and accept torch
tensors (their ``data_ptr()``) or raw integer addresses.  ``stream=None``
means torch's current CUDA stream (or the legacy default stream when torch
has no CUDA).
"""

from __future__ import annotations

import ctypes
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmxq.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python fp8_gemm_diffusion_b200/build.py` "
        "(nvcc, sm_100a). There is no fallback implementation.")

_lib = ctypes.CDLL(LIB_PATH)

# ------------------------------------------------------------------ enums
OK = 0
ERR_INVALID_ARG = 1
ERR_ALIGNMENT = 2
ERR_UNSUPPORTED_SHAPE = 3
ERR_WORKSPACE = 4
ERR_ARCH = 5
ERR_CUDA = 6
ERR_TIMEOUT = 7

NVFP4 = 1
MXFP8 = 2
BF16 = 3
FORMATS = {"nvfp4": NVFP4, "mxfp8": MXFP8, "bf16": BF16}
# mxq_weight_prepare flags (mxq_weight.flags)
WEIGHT_KEEP_BF16 = 1
WEIGHT_NO_TENSOR_SCALE = 2
WEIGHT_MXFP8_RCEIL = 4
SCALE_FLOOR = 0
SCALE_RCEIL = 1

_i64 = ctypes.c_int64
_ptr = ctypes.c_void_p
_sz = ctypes.c_size_t
_int = ctypes.c_int


class mxq_weight(ctypes.Structure):
    _fields_ = [
        ("format", ctypes.c_int32),
        ("flags", ctypes.c_int32),
        ("N", _i64),
        ("K", _i64),
        ("w_bf16", _ptr),
        ("bias_bf16", _ptr),
        ("codes", _ptr),
        ("sf", _ptr),
        ("g_dev", _ptr),
        ("amax_dev", _ptr),
    ]


ACT_NONE = 0
ACT_GELU = 1


class mxq_linear_opts(ctypes.Structure):
    _fields_ = [("min_dim", _i64), ("gemm_event_start", ctypes.c_void_p),
                ("gemm_event_end", ctypes.c_void_p), ("activation", ctypes.c_int32),
                ("reserved", ctypes.c_int32), ("y_amax_dev", ctypes.c_void_p),
                ("x_amax_dev", ctypes.c_void_p)]


def _proto(name, restype, *argtypes):
    fn = getattr(_lib, name)
    fn.restype = restype
    fn.argtypes = list(argtypes)
    return fn


_status_string = _proto("mxq_status_string", ctypes.c_char_p, _int)
_version = _proto("mxq_version", _int)
_last_cuda_error = _proto("mxq_last_cuda_error", _int)
_sf_bytes = _proto("mxq_sf_bytes", _sz, _i64, _i64, _int)
_codes_bytes = _proto("mxq_codes_bytes", _sz, _i64, _i64, _int)
_amax = _proto("mxq_amax", _int, _ptr, _i64, _i64, _i64, _ptr, _ptr)
_quantize_nvfp4 = _proto("mxq_quantize_nvfp4", _int, _ptr, _i64, _i64, _i64, _ptr, _ptr, _ptr,
                         _ptr, _ptr)
_quantize_mxfp8 = _proto("mxq_quantize_mxfp8", _int, _ptr, _i64, _i64, _i64, _ptr, _ptr, _ptr)
_quantize_mxfp8_rule = _proto("mxq_quantize_mxfp8_rule", _int, _ptr, _i64, _i64, _i64, _int, _ptr,
                              _ptr, _ptr)
_gemm_blockscaled = _proto("mxq_gemm_blockscaled", _int, _int, _i64, _i64, _i64, _ptr, _ptr,
                           _ptr, _ptr, _ptr, _ptr, _ptr, _ptr, _i64, _ptr)
_weight_storage_bytes = _proto("mxq_weight_storage_bytes", _sz, _i64, _i64, _int)
_weight_prepare = _proto("mxq_weight_prepare", _int, _int, _ptr, _i64, _i64, _ptr, _int, _ptr,
                         _sz, ctypes.POINTER(mxq_weight), _ptr)
_linear_path = _proto("mxq_linear_path", _int, ctypes.POINTER(mxq_weight), _i64,
                      ctypes.POINTER(mxq_linear_opts))
_linear_workspace_bytes = _proto("mxq_linear_workspace_bytes", _sz, _i64, _i64, _int)
_linear = _proto("mxq_linear", _int, ctypes.POINTER(mxq_weight), _ptr, _i64, _ptr, _ptr, _sz,
                 ctypes.POINTER(mxq_linear_opts), _ptr)
_linear_noalloc = _proto("mxq_linear_noalloc", _int, ctypes.POINTER(mxq_weight), _ptr, _i64,
                         _ptr, ctypes.POINTER(mxq_linear_opts), _ptr)
_linear_kernel_count = _proto("mxq_linear_kernel_count", _int, ctypes.POINTER(mxq_weight), _i64,
                              ctypes.POINTER(mxq_linear_opts))
_get_device_error = _proto("mxq_get_device_error", _int, _ptr)
_attention_workspace_bytes = _proto("mxq_attention_workspace_bytes", _sz, _i64, _i64, _i64)
_attention_mxfp8 = _proto("mxq_attention_mxfp8", _int, _ptr, _ptr, _ptr, _i64, _i64, _i64, ctypes.c_float,
                          _ptr, _ptr, _sz, _ptr)
_convert_f32 = _proto("mxq_convert_f32", _int, _ptr, _i64, _int, _ptr, _ptr)

#: Every symbol include/mxq.h declares (checked by the CPU tests).
EXPORTED = [
    "mxq_status_string", "mxq_version", "mxq_last_cuda_error", "mxq_sf_bytes",
    "mxq_codes_bytes", "mxq_amax", "mxq_quantize_nvfp4", "mxq_quantize_mxfp8",
    "mxq_gemm_blockscaled", "mxq_weight_storage_bytes", "mxq_weight_prepare",
    "mxq_linear_path", "mxq_linear_workspace_bytes", "mxq_linear", "mxq_get_device_error",
    "mxq_convert_f32", "mxq_linear_noalloc", "mxq_linear_kernel_count", "mxq_quantize_mxfp8_rule",
    "mxq_attention_workspace_bytes", "mxq_attention_mxfp8",
]

#: Capacity of the static device scratch of mxq_linear_noalloc (MXQ_NOALLOC_SCRATCH_BYTES).
NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024


class MxqError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = status_string(status)
        if status == ERR_CUDA:
            msg += f" (cuda error {_last_cuda_error()})"
        super().__init__(f"{where}: {msg} [status {status}]")


def _check(st: int, where: str) -> None:
    if st != OK:
        raise MxqError(st, where)


def _addr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        try:
            import torch
            if torch.cuda.is_available():
                return torch.cuda.current_stream().cuda_stream
        except Exception:  # pragma: no cover
            pass
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _fmt(f) -> int:
    return FORMATS[f] if isinstance(f, str) else int(f)


def _shape2(x, rows, k, ld):
    if rows is None:
        rows, k = x.shape
    if ld is None:
        ld = x.stride(0) if hasattr(x, "stride") and x.dim() == 2 and rows > 0 else k
        if ld == 0 or ld < k:
            ld = k
    return int(rows), int(k), int(ld)


# ------------------------------------------------------------- wrappers
def status_string(status: int) -> str:
    return _status_string(int(status)).decode()


def version() -> int:
    return _version()


def last_cuda_error() -> int:
    return _last_cuda_error()


def sf_bytes(rows: int, k: int, fmt) -> int:
    return _sf_bytes(rows, k, _fmt(fmt))


def codes_bytes(rows: int, k: int, fmt) -> int:
    return _codes_bytes(rows, k, _fmt(fmt))


def amax(x, amax_out, rows=None, k=None, ld=None, stream=None) -> None:
    rows, k, ld = _shape2(x, rows, k, ld)
    _check(_amax(_addr(x), rows, k, ld, _addr(amax_out), _stream(stream)), "mxq_amax")


def quantize_nvfp4(x, amax_in, codes, sf, g_out, rows=None, k=None, ld=None, stream=None) -> None:
    """amax_in=None: NVFP4 without a per-tensor scale (g = 1)."""
    rows, k, ld = _shape2(x, rows, k, ld)
    _check(_quantize_nvfp4(_addr(x), rows, k, ld, _addr(amax_in), _addr(codes), _addr(sf),
                           _addr(g_out), _stream(stream)), "mxq_quantize_nvfp4")


def quantize_mxfp8(x, codes, sf, rows=None, k=None, ld=None, stream=None, scale_rule=None) -> None:
    """scale_rule: None / SCALE_FLOOR (the OCP rule) or SCALE_RCEIL."""
    rows, k, ld = _shape2(x, rows, k, ld)
    if scale_rule is None:
        _check(_quantize_mxfp8(_addr(x), rows, k, ld, _addr(codes), _addr(sf), _stream(stream)),
               "mxq_quantize_mxfp8")
    else:
        _check(_quantize_mxfp8_rule(_addr(x), rows, k, ld, int(scale_rule), _addr(codes), _addr(sf),
                                    _stream(stream)), "mxq_quantize_mxfp8_rule")


def gemm_blockscaled(fmt, M, N, K, a, a_sf, a_g, b, b_sf, b_g, bias, y, ldy=None,
                     stream=None) -> None:
    _check(_gemm_blockscaled(_fmt(fmt), M, N, K, _addr(a), _addr(a_sf), _addr(a_g), _addr(b),
                             _addr(b_sf), _addr(b_g), _addr(bias), _addr(y),
                             N if ldy is None else ldy, _stream(stream)),
           "mxq_gemm_blockscaled")


def weight_storage_bytes(N: int, K: int, fmt) -> int:
    return _weight_storage_bytes(N, K, _fmt(fmt))


def weight_prepare(fmt, w, N, K, bias, flags, storage, storage_bytes, stream=None) -> mxq_weight:
    """flags: WEIGHT_KEEP_BF16 | WEIGHT_NO_TENSOR_SCALE bits (0: the defaults)."""
    out = mxq_weight()
    _check(_weight_prepare(_fmt(fmt), _addr(w), N, K, _addr(bias), int(flags),
                           _addr(storage), storage_bytes, ctypes.byref(out), _stream(stream)),
           "mxq_weight_prepare")
    return out


def _opts(min_dim, gemm_events=None, activation=ACT_NONE, y_amax=None, x_amax=None):
    """mxq_linear_opts; gemm_events: (start, end) torch.cuda.Event pair recorded
    around the GEMM launch, or None; activation / y_amax (device float tensor or
    address): the producer epilogue; x_amax: the input's known amax."""
    if (min_dim is None and gemm_events is None and not activation and y_amax is None
            and x_amax is None):
        return None
    o = mxq_linear_opts(int(min_dim or 0))
    if gemm_events is not None:
        o.gemm_event_start, o.gemm_event_end = (ev.cuda_event for ev in gemm_events)
    o.activation = int(activation)
    o.y_amax_dev = _addr(y_amax)
    o.x_amax_dev = _addr(x_amax)
    return ctypes.byref(o)


def linear_path(w: mxq_weight, M: int, min_dim=None) -> int:
    return _linear_path(ctypes.byref(w), M, _opts(min_dim))


def linear_kernel_count(w: mxq_weight, M: int, min_dim=None, x_amax=None) -> int:
    """Kernels one mxq_linear call launches for these arguments (-1: no device)."""
    return _linear_kernel_count(ctypes.byref(w), M, _opts(min_dim, x_amax=x_amax))


def linear_workspace_bytes(M: int, K: int, fmt) -> int:
    return _linear_workspace_bytes(M, K, _fmt(fmt))


def linear(w: mxq_weight, x, M, y, ws, ws_bytes, min_dim=None, stream=None, gemm_events=None,
           activation=ACT_NONE, y_amax=None, x_amax=None) -> None:
    _check(_linear(ctypes.byref(w), _addr(x), M, _addr(y), _addr(ws), ws_bytes,
                   _opts(min_dim, gemm_events, activation, y_amax, x_amax), _stream(stream)),
           "mxq_linear")


def linear_noalloc(w: mxq_weight, x, M, y, min_dim=None, stream=None) -> None:
    """mxq_linear without a workspace argument, for callers that cannot
    allocate device memory (fixed memory budget, or no cudaMalloc allowed in a
    latency-critical loop): the library's static device scratch is used
    instead.  Calls that overlap on the GPU race on that shared scratch."""
    _check(_linear_noalloc(ctypes.byref(w), _addr(x), M, _addr(y), _opts(min_dim),
                           _stream(stream)), "mxq_linear_noalloc")


def attention_workspace_bytes(heads: int, tokens: int, d: int = 128) -> int:
    return _attention_workspace_bytes(heads, tokens, d)


def attention_mxfp8(q, k, v, heads, tokens, out, ws, ws_bytes, d=128, tau=0.0, stream=None) -> None:
    """out = attention(q, k, v) per head through the 8-bit path; q, k, v, out
    [heads][tokens][d] bf16 (tensors or device addresses)."""
    _check(_attention_mxfp8(_addr(q), _addr(k), _addr(v), heads, tokens, d, float(tau), _addr(out),
                            _addr(ws), ws_bytes, _stream(stream)), "mxq_attention_mxfp8")


def attention_forward(q, k, v, tau=0.0, stream=None):
    """Allocates the output and workspace with torch; q, k, v [heads, tokens, d] bf16."""
    import torch
    H, T, d = q.shape
    out = torch.empty_like(q)
    nbytes = attention_workspace_bytes(H, T, d)
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
    attention_mxfp8(q, k, v, H, T, out, ws, nbytes, d=d, tau=tau, stream=stream)
    return out


def get_device_error(stream=None) -> int:
    return _get_device_error(_stream(stream))


def convert_f32(inp, n, code_fmt, out, stream=None) -> None:
    _check(_convert_f32(_addr(inp), n, code_fmt, _addr(out), _stream(stream)), "mxq_convert_f32")


# ------------------------------------------------ torch-owned buffers
class Weight:
    """A prepared layer: the mxq_weight handle plus the torch tensors it points
    into (kept alive here).  Allocation is torch's; quantisation runs in
    mxq_weight_prepare."""

    def __init__(self, w, bias=None, fmt="nvfp4", keep_bf16=False, tensor_scale=True,
                 mxfp8_rceil=False, stream=None):
        """tensor_scale=False: NVFP4 without a per-tensor scale (g = 1 for the
        weight and every activation); mxfp8_rceil=True: MXFP8 with the ceiling
        scale rule."""
        import torch
        N, K = w.shape
        self.w, self.bias, self.fmt = w, bias, _fmt(fmt)
        flags = ((WEIGHT_KEEP_BF16 if keep_bf16 else 0) | (0 if tensor_scale else WEIGHT_NO_TENSOR_SCALE)
                 | (WEIGHT_MXFP8_RCEIL if mxfp8_rceil else 0))
        nbytes = weight_storage_bytes(N, K, self.fmt) if not keep_bf16 else 0
        self.storage = (torch.empty(max(nbytes, 256), dtype=torch.uint8, device=w.device)
                        if nbytes else None)
        self.handle = weight_prepare(self.fmt, w, N, K, bias, flags, self.storage, nbytes,
                                     stream=stream)

    @property
    def N(self):
        return self.handle.N

    @property
    def K(self):
        return self.handle.K


def linear_forward(weight: Weight, x, y=None, ws=None, min_dim=None, stream=None):
    """y = x W^T + bias through mxq_linear; allocates y / workspace with torch
    when not given."""
    import torch
    M, K = x.shape
    path = linear_path(weight.handle, M, min_dim)
    if y is None:
        y = torch.empty(M, weight.N, dtype=torch.bfloat16, device=x.device)
    nbytes = linear_workspace_bytes(M, K, path) if path != BF16 else 0
    if ws is None and nbytes:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
    linear(weight.handle, x, M, y, ws, nbytes if ws is None else ws.numel(), min_dim, stream)
    return y
