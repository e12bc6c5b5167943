"""ctypes binding over libint8mp (see include/int8mp.h).

Argument marshalling only: every step of the forward runs in the library's
CUDA kernels.  Tensors are torch CUDA tensors (torch provides device memory
and the current stream); the functions keep the C names.  The library is
loaded on first use and a missing or unloadable library raises -- there is no
fallback implementation.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "lib", "libint8mp.so")

I8_OK = 0
STATUS_NAMES = {0: "I8_OK", 1: "I8_ERR_INVALID_ARG", 2: "I8_ERR_WORKSPACE", 3: "I8_ERR_CUDA",
                4: "I8_ERR_TIMEOUT", 5: "I8_ERR_UNSUPPORTED"}

PATH_AUTO, PATH_TENSOR_CORE, PATH_DECODE, PATH_TENSOR_CORE_1SM = 0, 1, 2, 3
DECODE_MAX_T = 16
I8_DTYPE_F16, I8_DTYPE_BF16 = 0, 1
_DTYPES = {torch.float16: I8_DTYPE_F16, torch.bfloat16: I8_DTYPE_BF16}

_lib = None
_lock = threading.Lock()


class Int8mpError(RuntimeError):
    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")
        self.status = status


class WsLayout(ctypes.Structure):
    _fields_ = [("status", ctypes.c_uint64), ("mask", ctypes.c_uint64), ("sA", ctypes.c_uint64),
                ("Xq", ctypes.c_uint64), ("Xo", ctypes.c_uint64), ("Wo", ctypes.c_uint64),
                ("total", ctypes.c_uint64), ("ldo", ctypes.c_int64)]


_P, _I64, _F32, _I32, _SZ = ctypes.c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_int, ctypes.c_size_t

SIGNATURES = {
    "int8_status_string": (ctypes.c_char_p, [_I32]),
    "int8_version": (_I32, []),
    "int8_quantize_weight": (_I32, [_P, _I64, _I64, _P, _P, _P]),
    "int8_linear_workspace_bytes": (_SZ, [_I64, _I64, _I64]),
    "int8_linear_forward": (_I32, [_P, _I64, _I64, _P, _P, _P, _I64, _F32, _P, _P, _P, _P, _SZ, _P]),
    "int8_linear_forward_path": (_I32, [_P, _I64, _I64, _P, _P, _P, _I64, _F32, _P, _P, _P, _P, _SZ, _I32, _P]),
    "int8_linear_forward_timed": (_I32, [_P, _I64, _I64, _P, _P, _P, _I64, _F32, _P, _P, _P, _P, _SZ, _I32,
                                         ctypes.POINTER(ctypes.c_void_p), _P]),
    "int8_check_status": (_I32, [_P, ctypes.POINTER(ctypes.c_uint32), _P]),
    "int8_linear_forward_host_workspace_bytes": (_SZ, [_I64, _I64, _I64]),
    "int8_linear_forward_host": (_I32, [_P, _I64, _I64, _P, _P, _P, _I64, _F32, _P, _P, _P, _P, _SZ, _P]),
    "int8_linear_workspace_layout": (_I32, [_I64, _I64, _I64, ctypes.POINTER(WsLayout)]),
    "int8_gemm_i32": (_I32, [_P, _I64, _I64, _P, _I64, _P, _I32, _P, _SZ, _P]),
    "int8_outlier_threshold_bits": (ctypes.c_uint32, [_F32]),
    "int8_selftest_wait_timeout": (_I32, [_P, _SZ, ctypes.c_uint32, _P]),
    "int8_linear_fp16w_workspace_bytes": (_SZ, [_I64, _I64, _I64]),
    "int8_linear_forward_fp16w": (_I32, [_P, _I64, _I64, _P, _P, _I64, _F32, _P, _P, _P, _P, _SZ, _P]),
    "int8_last_cuda_error": (ctypes.c_char_p, []),
    "int8_layer_packed_bytes": (_SZ, [_I64, _I64, _I32]),
    "int8_layer_pack": (_I32, [_P, _P, _P, _I64, _I64, _P, _SZ]),
    "int8_layer_unpack_header": (_I32, [_P, _SZ, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64),
                                        ctypes.POINTER(ctypes.c_int)]),
    "int8_layer_unpack": (_I32, [_P, _SZ, _P, _P, _P]),
    "int8_layer_pack_ex": (_I32, [_P, _P, _P, _I32, _I64, _I64, _P, _SZ]),
    "int8_layer_unpack_header_ex": (_I32, [_P, _SZ, ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int64),
                                           ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]),
    "int8_linear_forward_decode_static": (_I32, [_P, _I64, _I64, _P, _P, _P, _I64, _F32, _P, _P, _P, _P]),
    "int8_quantize_weight_ex": (_I32, [_P, _I32, _I64, _I64, _P, _P, _P]),
    "int8_linear_forward_ex": (_I32, [_P, _I32, _I64, _I64, _P, _P, _P, _I64, _F32, _P, _P, _P, _P, _SZ, _I32,
                                      ctypes.POINTER(ctypes.c_void_p), _P]),
    "int8_linear_forward_fp16w_ex": (_I32, [_P, _I32, _I64, _I64, _P, _P, _I64, _F32, _P, _P, _P, _P, _SZ, _P]),
    "int8_outlier_threshold_bits_ex": (ctypes.c_uint32, [_F32, _I32]),
    "int8_linear_forward_sharded": (_I32, [_P, _I32, _I64, _I64, _P, _P, _P, _I64, _F32,
                                           ctypes.POINTER(ctypes.c_void_p), _I32, _I64, _I64, _P, _P, _P, _SZ,
                                           _I32, _P]),
    "int8_linear_product_kernel": (_I32, [_I64, _I64, _I64, _I32]),
    "int8_linear_forward_host_async": (_I32, [_P, _I32, _I64, _I64, _P, _P, _P, _I64, _F32, _P, _P, _P, _P, _SZ,
                                              _P]),
}
MAX_Y_DST = 8


def lib() -> ctypes.CDLL:
    """Load libint8mp.so (built in-tree by ``build.py``); raise if it is missing."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(
                        f"{LIB_PATH} is missing: build it with `python -m int8_mixed_precision_column_b200.build`")
                h = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in SIGNATURES.items():
                    f = getattr(h, name, None)  # every declared symbol is checked by the ABI tests
                    if f is None:
                        continue
                    f.restype = res
                    f.argtypes = args
                _lib = h
    return _lib


def _check(fn: str, status: int) -> None:
    if status != I8_OK:
        raise Int8mpError(fn, status)


def _ptr(t: torch.Tensor | None) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream: torch.cuda.Stream | None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _require(t: torch.Tensor, dtype: torch.dtype, shape: tuple, name: str) -> None:
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name}: expected contiguous cuda {dtype} {tuple(shape)}, got {t.dtype} "
                         f"{tuple(t.shape)} on {t.device}")


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------

def int8_last_cuda_error() -> str:
    return lib().int8_last_cuda_error().decode()


def int8_status_string(status: int) -> str:
    return lib().int8_status_string(status).decode()


def _dtype_code(t: torch.Tensor, name: str) -> int:
    if t.dtype not in _DTYPES:
        raise ValueError(f"{name}: expected float16 or bfloat16, got {t.dtype}")
    return _DTYPES[t.dtype]


def int8_outlier_threshold_bits(threshold: float, dtype: torch.dtype = torch.float16) -> int:
    if dtype == torch.float16:
        return int(lib().int8_outlier_threshold_bits(threshold))
    return int(lib().int8_outlier_threshold_bits_ex(threshold, _DTYPES[dtype]))


def int8_linear_workspace_bytes(T: int, K: int, N: int) -> int:
    return int(lib().int8_linear_workspace_bytes(T, K, N))


def int8_linear_workspace_layout(T: int, K: int, N: int) -> dict:
    out = WsLayout()
    _check("int8_linear_workspace_layout", lib().int8_linear_workspace_layout(T, K, N, ctypes.byref(out)))
    return {f: getattr(out, f) for f, _ in WsLayout._fields_}


def int8_quantize_weight(W: torch.Tensor, CB: torch.Tensor | None = None, SCB: torch.Tensor | None = None,
                         stream=None):
    """W fp16 or bf16 [N,K] -> (CB int8 [N,K], SCB fp32 [N])."""
    N, K = W.shape
    dt = _dtype_code(W, "W")
    _require(W, W.dtype, (N, K), "W")
    CB = torch.empty((N, K), dtype=torch.int8, device=W.device) if CB is None else CB
    SCB = torch.empty((N,), dtype=torch.float32, device=W.device) if SCB is None else SCB
    _require(CB, torch.int8, (N, K), "CB")
    _require(SCB, torch.float32, (N,), "SCB")
    if dt == I8_DTYPE_F16:
        st = lib().int8_quantize_weight(_ptr(W), N, K, _ptr(CB), _ptr(SCB), _stream(stream))
    else:
        st = lib().int8_quantize_weight_ex(_ptr(W), dt, N, K, _ptr(CB), _ptr(SCB), _stream(stream))
    _check("int8_quantize_weight", st)
    return CB, SCB


def new_workspace(T: int, K: int, N: int, device="cuda") -> torch.Tensor:
    nbytes = int8_linear_workspace_bytes(T, K, N)
    if nbytes == 0:
        raise ValueError(f"unsupported shape T={T} K={K} N={N}")
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def int8_linear_forward(X: torch.Tensor, CB: torch.Tensor, SCB: torch.Tensor, bias: torch.Tensor | None,
                        threshold: float, *, Y=None, idx=None, n_out=None, workspace=None,
                        path: int = PATH_AUTO, stream=None):
    """Returns (Y [T,N], idx int32 [K] (first n_out valid), n_out int32 [1], workspace).
    X, bias and Y share one element type: fp16, or bf16 (the *_ex entry point)."""
    T, K = X.shape
    N = CB.shape[0]
    dt = _dtype_code(X, "X")
    _require(X, X.dtype, (T, K), "X")
    _require(CB, torch.int8, (N, K), "CB")
    _require(SCB, torch.float32, (N,), "SCB")
    if bias is not None:
        _require(bias, X.dtype, (N,), "bias")
    dev = X.device
    Y = torch.empty((T, N), dtype=X.dtype, device=dev) if Y is None else Y
    idx = torch.empty((K,), dtype=torch.int32, device=dev) if idx is None else idx
    n_out = torch.empty((1,), dtype=torch.int32, device=dev) if n_out is None else n_out
    workspace = new_workspace(T, K, N, dev) if workspace is None else workspace
    _require(Y, X.dtype, (T, N), "Y")
    if dt == I8_DTYPE_F16:
        st = lib().int8_linear_forward_path(_ptr(X), T, K, _ptr(CB), _ptr(SCB), _ptr(bias), N, float(threshold),
                                            _ptr(Y), _ptr(idx), _ptr(n_out), _ptr(workspace), workspace.numel(),
                                            int(path), _stream(stream))
    else:
        st = lib().int8_linear_forward_ex(_ptr(X), dt, T, K, _ptr(CB), _ptr(SCB), _ptr(bias), N, float(threshold),
                                          _ptr(Y), _ptr(idx), _ptr(n_out), _ptr(workspace), workspace.numel(),
                                          int(path), None, _stream(stream))
    _check("int8_linear_forward", st)
    return Y, idx, n_out, workspace


def int8_linear_forward_timed(X, CB, SCB, bias, threshold, Y, idx, n_out, workspace, events, *,
                              path: int = PATH_AUTO, stream=None) -> None:
    """Forward that records the four stage events (torch.cuda.Event, already
    materialised by one ``record()``) on the stream: before the first stage,
    after the outlier pass, after row quantisation, after the product kernel."""
    T, K = X.shape
    N = CB.shape[0]
    arr = (ctypes.c_void_p * 4)(*[ctypes.c_void_p(e.cuda_event) for e in events])
    dt = _dtype_code(X, "X")
    if dt == I8_DTYPE_F16:
        st = lib().int8_linear_forward_timed(_ptr(X), T, K, _ptr(CB), _ptr(SCB), _ptr(bias), N, float(threshold),
                                             _ptr(Y), _ptr(idx), _ptr(n_out), _ptr(workspace), workspace.numel(),
                                             int(path), arr, _stream(stream))
    else:
        st = lib().int8_linear_forward_ex(_ptr(X), dt, T, K, _ptr(CB), _ptr(SCB), _ptr(bias), N, float(threshold),
                                          _ptr(Y), _ptr(idx), _ptr(n_out), _ptr(workspace), workspace.numel(),
                                          int(path), arr, _stream(stream))
    _check("int8_linear_forward_timed", st)


def int8_linear_forward_fp16w(X: torch.Tensor, W: torch.Tensor, bias: torch.Tensor | None, threshold: float, *,
                              Y=None, idx=None, n_out=None, workspace=None, stream=None):
    """has_fp16_weights=True forward: W [N,K] (fp16, or bf16 like X) is quantised inside every call.
    Returns (Y, idx, n_out, workspace); CB/SCB of this call sit in the workspace."""
    T, K = X.shape
    N = W.shape[0]
    dt = _dtype_code(X, "X")
    _require(X, X.dtype, (T, K), "X")
    _require(W, X.dtype, (N, K), "W")
    if bias is not None:
        _require(bias, X.dtype, (N,), "bias")
    dev = X.device
    Y = torch.empty((T, N), dtype=X.dtype, device=dev) if Y is None else Y
    idx = torch.empty((K,), dtype=torch.int32, device=dev) if idx is None else idx
    n_out = torch.empty((1,), dtype=torch.int32, device=dev) if n_out is None else n_out
    if workspace is None:
        workspace = torch.empty(int(lib().int8_linear_fp16w_workspace_bytes(T, K, N)), dtype=torch.uint8, device=dev)
    if dt == I8_DTYPE_F16:
        st = lib().int8_linear_forward_fp16w(_ptr(X), T, K, _ptr(W), _ptr(bias), N, float(threshold), _ptr(Y),
                                             _ptr(idx), _ptr(n_out), _ptr(workspace), workspace.numel(),
                                             _stream(stream))
    else:
        st = lib().int8_linear_forward_fp16w_ex(_ptr(X), dt, T, K, _ptr(W), _ptr(bias), N, float(threshold),
                                                _ptr(Y), _ptr(idx), _ptr(n_out), _ptr(workspace), workspace.numel(),
                                                _stream(stream))
    _check("int8_linear_forward_fp16w", st)
    return Y, idx, n_out, workspace


def int8_linear_forward_sharded(X: torch.Tensor, CB: torch.Tensor, SCB: torch.Tensor, bias: torch.Tensor | None,
                                threshold: float, Y_dst: list, ldY: int, col_offset: int, *, idx=None, n_out=None,
                                workspace=None, path: int = PATH_AUTO, stream=None):
    """One output-feature shard of the forward, stored into every buffer of
    ``Y_dst`` (device pointers as ints, or tensors; [T, ldY] of X's dtype) at
    columns [col_offset, col_offset + N).  Returns (idx, n_out, workspace)."""
    T, K = X.shape
    N = CB.shape[0]
    dt = _dtype_code(X, "X")
    _require(X, X.dtype, (T, K), "X")
    _require(CB, torch.int8, (N, K), "CB")
    _require(SCB, torch.float32, (N,), "SCB")
    if bias is not None:
        _require(bias, X.dtype, (N,), "bias")
    if not 1 <= len(Y_dst) <= MAX_Y_DST:
        raise ValueError(f"Y_dst: 1..{MAX_Y_DST} destinations, got {len(Y_dst)}")
    ptrs = []
    for y in Y_dst:
        if isinstance(y, torch.Tensor):
            _require(y, X.dtype, (T, ldY), "Y_dst[i]")
            ptrs.append(y.data_ptr())
        else:
            ptrs.append(int(y))
    dev = X.device
    idx = torch.empty((K,), dtype=torch.int32, device=dev) if idx is None else idx
    n_out = torch.empty((1,), dtype=torch.int32, device=dev) if n_out is None else n_out
    workspace = new_workspace(T, K, N, dev) if workspace is None else workspace
    arr = (ctypes.c_void_p * len(ptrs))(*[ctypes.c_void_p(q) for q in ptrs])
    st = lib().int8_linear_forward_sharded(_ptr(X), dt, T, K, _ptr(CB), _ptr(SCB), _ptr(bias), N, float(threshold),
                                           arr, len(ptrs), int(ldY), int(col_offset), _ptr(idx), _ptr(n_out),
                                           _ptr(workspace), workspace.numel(), int(path), _stream(stream))
    _check("int8_linear_forward_sharded", st)
    return idx, n_out, workspace


def int8_linear_product_kernel(T: int, K: int, N: int, path: int = PATH_AUTO) -> int:
    """The product kernel a forward runs: PATH_TENSOR_CORE (SM pairs), PATH_DECODE or
    PATH_TENSOR_CORE_1SM; -1 if the forward would reject the arguments."""
    return int(lib().int8_linear_product_kernel(T, K, N, int(path)))


def int8_check_status(workspace: torch.Tensor, stream=None) -> tuple[int, int]:
    where = ctypes.c_uint32(0)
    st = lib().int8_check_status(_ptr(workspace), ctypes.byref(where), _stream(stream))
    return int(st), int(where.value)


def int8_gemm_i32(Xq: torch.Tensor, CB: torch.Tensor, path: int = PATH_AUTO, workspace=None, stream=None):
    T, K = Xq.shape
    N = CB.shape[0]
    _require(Xq, torch.int8, (T, K), "Xq")
    _require(CB, torch.int8, (N, K), "CB")
    acc = torch.empty((T, N), dtype=torch.int32, device=Xq.device)
    ws = torch.empty(256, dtype=torch.uint8, device=Xq.device) if workspace is None else workspace
    _check("int8_gemm_i32", lib().int8_gemm_i32(_ptr(Xq), T, K, _ptr(CB), N, _ptr(acc), int(path), _ptr(ws),
                                                ws.numel(), _stream(stream)))
    return acc


def int8_linear_forward_host_workspace_bytes(T: int, K: int, N: int) -> int:
    return int(lib().int8_linear_forward_host_workspace_bytes(T, K, N))


def int8_linear_forward_host(X_host: torch.Tensor, CB: torch.Tensor, SCB: torch.Tensor, bias, threshold: float,
                             Y_host: torch.Tensor, workspace: torch.Tensor, idx_host=None, n_out_host=None,
                             stream=None) -> None:
    """Blocking forward on host X/Y (ideally pinned) with a resident quantised layer."""
    T, K = X_host.shape
    N = CB.shape[0]
    if X_host.is_cuda or Y_host.is_cuda or X_host.dtype != torch.float16 or Y_host.dtype != torch.float16:
        raise ValueError("X_host/Y_host must be fp16 host tensors")
    if not (X_host.is_contiguous() and Y_host.is_contiguous()) or tuple(Y_host.shape) != (T, N):
        raise ValueError("X_host/Y_host must be contiguous with shapes [T,K], [T,N]")
    st = lib().int8_linear_forward_host(_ptr(X_host), T, K, _ptr(CB), _ptr(SCB), _ptr(bias), N, float(threshold),
                                        _ptr(Y_host), _ptr(idx_host), _ptr(n_out_host), _ptr(workspace),
                                        workspace.numel(), _stream(stream))
    _check("int8_linear_forward_host", st)


def int8_linear_forward_host_async(X_host: torch.Tensor, CB: torch.Tensor, SCB: torch.Tensor, bias, threshold: float,
                                   Y_host: torch.Tensor, workspace: torch.Tensor, idx_host=None, n_out_host=None,
                                   stream=None) -> None:
    """Non-blocking forward on pinned host X/Y; synchronise ``stream``, then
    call int8_check_status(workspace) before reading Y_host."""
    T, K = X_host.shape
    N = CB.shape[0]
    dt = _dtype_code(X_host, "X_host")
    if X_host.is_cuda or Y_host.is_cuda or Y_host.dtype != X_host.dtype:
        raise ValueError("X_host/Y_host must be host tensors of one 16-bit dtype")
    if not (X_host.is_pinned() and Y_host.is_pinned()):
        raise ValueError("X_host/Y_host must be pinned (page-locked)")
    if not (X_host.is_contiguous() and Y_host.is_contiguous()) or tuple(Y_host.shape) != (T, N):
        raise ValueError("X_host/Y_host must be contiguous with shapes [T,K], [T,N]")
    st = lib().int8_linear_forward_host_async(_ptr(X_host), dt, T, K, _ptr(CB), _ptr(SCB), _ptr(bias), N,
                                              float(threshold), _ptr(Y_host), _ptr(idx_host), _ptr(n_out_host),
                                              _ptr(workspace), workspace.numel(), _stream(stream))
    _check("int8_linear_forward_host_async", st)


def workspace_views(workspace: torch.Tensor, T: int, K: int, N: int, dtype: torch.dtype = torch.float16) -> dict:
    """Typed views of the forward's intermediate buffers inside ``workspace``
    (``dtype``: the forward's 16-bit element type, that of Xo and Wo)."""
    L = int8_linear_workspace_layout(T, K, N)
    ldo = L["ldo"]
    nw = (K + 31) // 32

    def view(off, nbytes, dtype, shape):
        return workspace[off: off + nbytes].view(dtype).view(shape)

    return {
        "mask": view(L["mask"], nw * 4, torch.int32, (nw,)),
        "sA": view(L["sA"], T * 4, torch.float32, (T,)),
        "Xq": view(L["Xq"], T * K, torch.int8, (T, K)),
        "Xo": view(L["Xo"], T * ldo * 2, dtype, (T, ldo)),
        "Wo": view(L["Wo"], N * ldo * 2, dtype, (N, ldo)),
        "ldo": ldo,
    }


# ---------------------------------------------------------------------------
# persistence of a quantised layer
# ---------------------------------------------------------------------------

def int8_layer_pack(CB: torch.Tensor, SCB: torch.Tensor, bias: torch.Tensor | None = None) -> bytes:
    """Byte image of a quantised layer (CB, SCB, optional fp16 or bf16 bias), any device."""
    N, K = CB.shape
    cb = CB.detach().to("cpu").contiguous()
    scb = SCB.detach().to("cpu", torch.float32).contiguous()
    bdt = torch.bfloat16 if (bias is not None and bias.dtype == torch.bfloat16) else torch.float16
    b = None if bias is None else bias.detach().to("cpu", bdt).contiguous()
    n = int(lib().int8_layer_packed_bytes(N, K, 0 if b is None else 1))
    if n == 0:
        raise ValueError(f"unsupported shape N={N} K={K}")
    out = ctypes.create_string_buffer(n)
    _check("int8_layer_pack", lib().int8_layer_pack_ex(cb.data_ptr(), scb.data_ptr(),
                                                       None if b is None else b.data_ptr(), _DTYPES[bdt], N, K,
                                                       ctypes.addressof(out), n))
    return out.raw


def int8_layer_unpack(image: bytes, device="cuda"):
    """(CB int8 [N,K], SCB fp32 [N], bias fp16/bf16 [N] or None) from a byte image."""
    buf = ctypes.create_string_buffer(bytes(image), len(image))
    N, K, hb, bdt = ctypes.c_int64(0), ctypes.c_int64(0), ctypes.c_int(0), ctypes.c_int(0)
    _check("int8_layer_unpack_header", lib().int8_layer_unpack_header_ex(ctypes.addressof(buf), len(image),
                                                                         ctypes.byref(N), ctypes.byref(K),
                                                                         ctypes.byref(hb), ctypes.byref(bdt)))
    CB = torch.empty((N.value, K.value), dtype=torch.int8)
    SCB = torch.empty((N.value,), dtype=torch.float32)
    b_dtype = torch.bfloat16 if bdt.value == I8_DTYPE_BF16 else torch.float16
    b = torch.empty((N.value,), dtype=b_dtype) if hb.value else None
    _check("int8_layer_unpack", lib().int8_layer_unpack(ctypes.addressof(buf), len(image), CB.data_ptr(), SCB.data_ptr(),
                                                        None if b is None else b.data_ptr()))
    return CB.to(device), SCB.to(device), (None if b is None else b.to(device))


def save_quantized(path: str, CB: torch.Tensor, SCB: torch.Tensor, bias: torch.Tensor | None = None) -> None:
    with open(path, "wb") as f:
        f.write(int8_layer_pack(CB, SCB, bias))


def load_quantized(path: str, device="cuda"):
    with open(path, "rb") as f:
        return int8_layer_unpack(f.read(), device)

