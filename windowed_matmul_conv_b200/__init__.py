"""Python binding of libwbmm.so: WBMM (Windowed Batch Matrix Multiplication)
on B200.

Each ``wbmm_*`` function has the name and meaning of the C entry point in
``include/wbmm.h`` and only marshals arguments: shapes and dtypes come from
the torch tensors, device pointers from ``data_ptr()``, the stream from
``torch.cuda.current_stream()``.  A non-zero status raises ``WbmmError``.
Plain pointers carry no sizes, so before the call the binding checks what
the library cannot: every buffer is on the current device, has the call's
dtype (fp32 for dT) and holds at least the elements the call reads or writes
(``WbmmError`` with ``WBMM_ERR_DTYPE`` or ``WBMM_ERR_INVALID_ARG``).
PyTorch is used for device memory and streams; every step of the operator
runs in the library's CUDA kernels.  Importing this package fails loudly if
the library has not been built (``python windowed_matmul_conv_b200/build.py``).

The convenience functions ``forward``, ``backward``, ``cache_matrices``,
``reparam_merge``, ``forward_cached`` and ``dw3x3`` allocate outputs with
torch and call the entry points above.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libwbmm.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        "libwbmm.so is missing: build it with `python windowed_matmul_conv_b200/build.py` "
        "(nvcc, sm_100a); there is no fallback implementation")

_lib = ctypes.CDLL(LIB_PATH)

WBMM_F32, WBMM_BF16 = 0, 1
# 32-bit arrival counters at the start of a table-gradient workspace
WBMM_DT_COUNTER_WORDS = 65536
STATUS_NAMES = {0: "WBMM_OK", 1: "WBMM_ERR_INVALID_ARG", 2: "WBMM_ERR_SHAPE",
                3: "WBMM_ERR_DTYPE", 4: "WBMM_ERR_ALIGNMENT", 5: "WBMM_ERR_UNSUPPORTED",
                6: "WBMM_ERR_WORKSPACE", 7: "WBMM_ERR_CUDA", 8: "WBMM_ERR_TIMEOUT"}
EXPORTS = ("wbmm_forward", "wbmm_backward_workspace_bytes", "wbmm_backward",
           "wbmm_cache_matrices", "wbmm_reparam_merge", "wbmm_forward_cached", "wbmm_dw3x3",
           "wbmm_get_device_status", "wbmm_status_string", "wbmm_set_wait_budget",
           "wbmm_wait_selftest", "wbmm_launch_count", "wbmm_last_path",
           "wbmm_backward_dt_static", "wbmm_debug_set")

_vp, _i, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
_lib.wbmm_forward.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]
_lib.wbmm_backward_workspace_bytes.argtypes = [_i, _i, _i, _i, _i, _i]
_lib.wbmm_backward_workspace_bytes.restype = _sz
_lib.wbmm_backward.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _sz, _i, _i, _i, _i, _i, _i, _vp]
_lib.wbmm_cache_matrices.argtypes = [_vp, _vp, _i, _i, _i, _vp]
_lib.wbmm_reparam_merge.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _vp]
_lib.wbmm_backward_dt_static.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]
_lib.wbmm_forward_cached.argtypes = [_vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]
_lib.wbmm_dw3x3.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]
_lib.wbmm_get_device_status.argtypes = [_vp]
_lib.wbmm_status_string.argtypes = [_i]
_lib.wbmm_status_string.restype = ctypes.c_char_p
_lib.wbmm_set_wait_budget.argtypes = [ctypes.c_ulonglong]
_lib.wbmm_set_wait_budget.restype = None
_lib.wbmm_wait_selftest.argtypes = [ctypes.c_ulonglong, _vp]
_lib.wbmm_launch_count.argtypes = []
_lib.wbmm_launch_count.restype = ctypes.c_ulonglong
_lib.wbmm_last_path.argtypes = []
_lib.wbmm_debug_set.argtypes = [_i, _i]
for _f in ("wbmm_forward", "wbmm_backward", "wbmm_backward_dt_static", "wbmm_cache_matrices",
           "wbmm_reparam_merge", "wbmm_forward_cached", "wbmm_dw3x3", "wbmm_get_device_status", "wbmm_wait_selftest", "wbmm_last_path",
           "wbmm_debug_set"):
    getattr(_lib, _f).restype = _i


WBMM_ERR_INVALID_ARG, WBMM_ERR_DTYPE = 1, 3


class WbmmError(RuntimeError):
    def __init__(self, status, detail=None):
        self.status = status
        msg = _lib.wbmm_status_string(status).decode()
        super().__init__(msg if detail is None else "%s: %s" % (msg, detail))


def _check(status):
    if status != 0:
        raise WbmmError(status)


def _dt(t):
    if t.dtype == torch.bfloat16:
        return WBMM_BF16
    if t.dtype == torch.float32:
        return WBMM_F32
    raise TypeError("WBMM tensors must be bfloat16 or float32, got %s" % t.dtype)


def _p(t):
    if t is None:
        return None
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("WBMM tensors must be contiguous CUDA tensors")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream, ref=None):
    """Stream handle for a call whose maps live on ``ref``'s device.  The
    library launches on the current device, so ``ref`` and the stream must
    be on it."""
    s = torch.cuda.current_stream() if stream is None else stream
    if ref is not None:
        d, cur = ref.get_device(), torch.cuda.current_device()
        if d != cur or s.device_index != d:
            raise WbmmError(WBMM_ERR_INVALID_ARG,
                            "maps on cuda:%d, stream on cuda:%d, current device cuda:%d"
                            % (d, s.device_index, cur))
    return ctypes.c_void_p(s.cuda_stream)


def _need(name, t, numel, ref, dtype=None):
    """Buffer ``t`` (optional) must sit on ``ref``'s device, have ``ref``'s
    dtype (or ``dtype``) and hold at least ``numel`` elements."""
    want = dtype or ref.dtype
    if t is None or (t.dtype is want and t.numel() >= numel
                     and t.get_device() == ref.get_device()):
        return
    if t.get_device() != ref.get_device():
        raise WbmmError(WBMM_ERR_INVALID_ARG, "%s is on %s, the map on %s"
                        % (name, t.device, ref.device))
    if t.dtype is not want:
        raise WbmmError(WBMM_ERR_DTYPE, "%s is %s, the call needs %s" % (name, t.dtype, want))
    raise WbmmError(WBMM_ERR_INVALID_ARG, "%s holds %d elements, the call needs %d"
                    % (name, t.numel(), numel))


def _tsz(w):
    return (2 * int(w) - 1) ** 2


def _map_shape(x):
    if x.dim() != 4:
        raise ValueError("feature maps must be [B, C, H, W]")
    return tuple(int(v) for v in x.shape)


# --------------------------------------------------------------- entry points

def wbmm_forward(x, T, y, w, stream=None):
    B, C, H, W = _map_shape(x)
    _need("T", T, C * _tsz(w), x)
    _need("y", y, x.numel(), x)
    _check(_lib.wbmm_forward(_p(x), _p(T), _p(y), B, C, H, W, int(w), _dt(x),
                             _stream(stream, x)))


def wbmm_backward_workspace_bytes(B, C, H, W, w, dtype):
    dt = _dt(torch.empty(0, dtype=dtype))
    return int(_lib.wbmm_backward_workspace_bytes(B, C, H, W, int(w), dt))


def wbmm_backward(x, T, dY, dX, dT, workspace, w, stream=None):
    B, C, H, W = _map_shape(dY)
    _need("x", x, dY.numel(), dY)
    _need("T", T, C * _tsz(w), dY)
    _need("dX", dX, dY.numel(), dY)
    _need("dT", dT, C * _tsz(w), dY, torch.float32)
    if workspace is not None and workspace.get_device() != dY.get_device():
        raise WbmmError(WBMM_ERR_INVALID_ARG, "workspace is on %s, the map on %s"
                        % (workspace.device, dY.device))
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.wbmm_backward(_p(x), _p(T), _p(dY), _p(dX), _p(dT), _p(workspace), ws_bytes,
                              B, C, H, W, int(w), _dt(dY), _stream(stream, dY)))


def wbmm_backward_dt_static(x, dY, dT, w, stream=None):
    """dT of wbmm_backward with the library's fixed scratch array (no allocation)."""
    B, C, H, W = _map_shape(dY)
    _need("x", x, dY.numel(), dY)
    _need("dT", dT, C * _tsz(w), dY, torch.float32)
    _check(_lib.wbmm_backward_dt_static(_p(x), _p(dY), _p(dT), B, C, H, W, int(w), _dt(dY),
                                        _stream(stream, dY)))


def wbmm_cache_matrices(T, M, w, stream=None):
    """T: [C, (2w-1)^2]; M: [C, w*w, w*w]."""
    C = int(T.shape[0])
    _need("T", T, C * _tsz(w), T)
    _need("M", M, C * int(w) ** 4, T)
    _check(_lib.wbmm_cache_matrices(_p(T), _p(M), C, int(w), _dt(T), _stream(stream, T)))


def wbmm_forward_cached(x, M, dw3x3, out, w, stream=None):
    B, C, H, W = _map_shape(x)
    _need("M", M, C * int(w) ** 4, x)
    _need("dw3x3", dw3x3, C * 9, x)
    _need("out", out, x.numel(), x)
    _check(_lib.wbmm_forward_cached(_p(x), _p(M), _p(dw3x3), _p(out), B, C, H, W, int(w),
                                    _dt(x), _stream(stream, x)))


def wbmm_dw3x3(y, K, z, stream=None):
    B, C, H, W = _map_shape(y)
    _need("K", K, C * 9, y)
    _need("z", z, y.numel(), y)
    _check(_lib.wbmm_dw3x3(_p(y), _p(K), _p(z), B, C, H, W, _dt(y), _stream(stream, y)))


def wbmm_get_device_status(stream=None):
    """Synchronises the stream; returns the status code (0, or 8 after a timeout)."""
    return int(_lib.wbmm_get_device_status(_stream(stream)))


def wbmm_status_string(status):
    return _lib.wbmm_status_string(int(status)).decode()


def wbmm_set_wait_budget(cycles):
    _lib.wbmm_set_wait_budget(int(cycles))


def wbmm_wait_selftest(cycles, stream=None):
    _check(_lib.wbmm_wait_selftest(int(cycles), _stream(stream)))


def wbmm_launch_count():
    return int(_lib.wbmm_launch_count())


def wbmm_last_path():
    return int(_lib.wbmm_last_path())


# test-only settings of wbmm_debug_set (include/wbmm.h)
WBMM_DEBUG_SKIP_LOAD_WINDOW_MAJOR, WBMM_DEBUG_SKIP_LOAD_TABLE_GRAD, WBMM_DEBUG_RING_CAP = 1, 2, 3


def wbmm_debug_set(what, value):
    _check(_lib.wbmm_debug_set(int(what), int(value)))


# ------------------------------------------------------------ conveniences

def forward(x, T, w, stream=None):
    y = torch.empty_like(x)
    wbmm_forward(x, T, y, w, stream)
    return y


def backward(x, T, dY, w, need_dx=True, need_dt=True, stream=None):
    B, C, H, W = _map_shape(dY)
    dX = torch.empty_like(dY) if need_dx else None
    dT = torch.empty((C, (2 * w - 1) ** 2), dtype=torch.float32, device=dY.device) if need_dt else None
    ws = None
    if need_dt:
        nbytes = wbmm_backward_workspace_bytes(B, C, H, W, w, dY.dtype)
        # zero-filled: the table gradient's arrival counters start at zero
        ws = torch.zeros(max(1, nbytes // 4), dtype=torch.float32, device=dY.device)
    wbmm_backward(x, T, dY, dX, dT, ws, w, stream)
    return dX, dT


def wbmm_reparam_merge(Tw, Tk, M, w, k, stream=None):
    """Tw: [C, (2w-1)^2]; Tk: [C, (2k-1)^2]; M: [C, w*w, w*w]."""
    C = int(Tw.shape[0])
    _need("Tw", Tw, C * _tsz(w), Tw)
    _need("Tk", Tk, C * _tsz(k), Tw)
    _need("M", M, C * int(w) ** 4, Tw)
    _check(_lib.wbmm_reparam_merge(_p(Tw), _p(Tk), _p(M), C, int(w), int(k), _dt(Tw),
                                   _stream(stream, Tw)))


def reparam_merge(Tw, Tk, w, k, stream=None):
    """Inference matrix [C, w*w, w*w] of a w-window branch (table Tw) plus a
    k-window branch (table Tk), k dividing w; feed it to forward_cached."""
    M = torch.empty((Tw.shape[0], w * w, w * w), dtype=Tw.dtype, device=Tw.device)
    wbmm_reparam_merge(Tw, Tk, M, w, k, stream)
    return M


def cache_matrices(T, w, stream=None):
    M = torch.empty((T.shape[0], w * w, w * w), dtype=T.dtype, device=T.device)
    wbmm_cache_matrices(T, M, w, stream)
    return M


def forward_cached(x, M, w, dw=None, stream=None):
    out = torch.empty_like(x)
    wbmm_forward_cached(x, M, dw, out, w, stream)
    return out


def dw3x3(y, K, stream=None):
    z = torch.empty_like(y)
    wbmm_dw3x3(y, K, z, stream)
    return z
