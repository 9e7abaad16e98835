"""WBMM oracle: test infrastructure only.

A plain, slow, fp64 CPU statement of the WBMM operator (Windowed Batch Matrix
Multiplication, arXiv 2607.02097), used to check the CUDA path.  Only tests/,
``__graft_entry__.smoke()`` and the benchmark's CPU-baseline leg may import
this package.  It shares no code with ``windowed_matmul_conv_b200`` and never
imports it.

Every function takes arrays of any real dtype (bf16 / fp32 values convert to
fp64 exactly), returns fp64 numpy arrays, and calls the C loops in
``wbmm_oracle.c``.  Citations for each definition are in that file:
  forward      -- reading notes "Core Idea"; abstract (table-indexed matrix,
                  batched matmul over contiguous windows)
  backward_dx  -- adjoint of the forward map, dX_c = M_c^T dY_c
  backward_dt  -- gradient of the table, dY X^T summed along offset diagonals
  expand       -- reading notes "Method" (inference caching of M)
  dw3x3        -- reading notes "Method", point 3 (inter-block 3x3 mixing)
  forward_cached -- the cached-inference product M_c X_c (numpy matmul)

Parity status: every function here is pinned by tests/test_oracle_pins.py
against library routines (torch conv2d), closed forms and invariants.
"""
import ctypes

import numpy as np

from . import build as _build


def _f64(a):
    """fp64 C-contiguous copy of a numpy array or a CPU torch tensor."""
    if hasattr(a, "detach"):
        a = a.detach().cpu().float().numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _check_map(x, w):
    if x.ndim != 4:
        raise ValueError("feature map must be [B, C, H, W]")
    B, C, H, W = x.shape
    if w < 1 or H % w or W % w:
        raise ValueError("H and W must be multiples of w")
    return B, C, H, W


def table_size(w):
    return (2 * w - 1) ** 2


class Oracle:
    """The oracle's entry points bound to one compiled copy of wbmm_oracle.c."""

    def __init__(self, lib_path):
        lib = ctypes.CDLL(lib_path)
        dp = ctypes.POINTER(ctypes.c_double)
        i = ctypes.c_int
        lib.oracle_forward.argtypes = [dp, dp, dp, i, i, i, i, i]
        lib.oracle_backward_dx.argtypes = [dp, dp, dp, i, i, i, i, i]
        lib.oracle_backward_dt.argtypes = [dp, dp, dp, i, i, i, i, i]
        lib.oracle_expand.argtypes = [dp, dp, i, i]
        lib.oracle_reparam_merge.argtypes = [dp, dp, dp, i, i, i]
        lib.oracle_dw3x3.argtypes = [dp, dp, dp, i, i, i, i]
        lib.oracle_num_threads.restype = ctypes.c_int
        for f in (lib.oracle_forward, lib.oracle_backward_dx, lib.oracle_backward_dt,
                  lib.oracle_expand, lib.oracle_reparam_merge, lib.oracle_dw3x3):
            f.restype = None
        self.lib = lib

    def forward(self, x, T, w):
        """y = WBMM(x; T): per channel, every w x w window times M_c(T_c)."""
        x, T = _f64(x), _f64(T)
        B, C, H, W = _check_map(x, w)
        if T.shape != (C, table_size(w)):
            raise ValueError("T must be [C, (2w-1)^2]")
        y = np.empty_like(x)
        self.lib.oracle_forward(_ptr(x), _ptr(T), _ptr(y), B, C, H, W, w)
        return y

    def backward_dx(self, dy, T, w):
        """dX = M_c^T dY for every window of every channel."""
        dy, T = _f64(dy), _f64(T)
        B, C, H, W = _check_map(dy, w)
        if T.shape != (C, table_size(w)):
            raise ValueError("T must be [C, (2w-1)^2]")
        dx = np.empty_like(dy)
        self.lib.oracle_backward_dx(_ptr(dy), _ptr(T), _ptr(dx), B, C, H, W, w)
        return dx

    def backward_dt(self, x, dy, w):
        """dT[c, idx(dp,dq)] = sum over windows and pairs at offset (dp,dq) of dy*x."""
        x, dy = _f64(x), _f64(dy)
        B, C, H, W = _check_map(x, w)
        if dy.shape != x.shape:
            raise ValueError("dY must have the shape of x")
        dT = np.empty((C, table_size(w)), dtype=np.float64)
        self.lib.oracle_backward_dt(_ptr(x), _ptr(dy), _ptr(dT), B, C, H, W, w)
        return dT

    def expand(self, T, w):
        """M[c] (d x d, u = p*w+q) from the relative table T[c]."""
        T = _f64(T)
        C = T.shape[0]
        if T.shape != (C, table_size(w)):
            raise ValueError("T must be [C, (2w-1)^2]")
        M = np.empty((C, w * w, w * w), dtype=np.float64)
        self.lib.oracle_expand(_ptr(T), _ptr(M), C, w)
        return M

    def reparam_merge(self, Tw, Tk, w, k):
        """Inference matrix of a w-window branch plus a k-window branch (k | w)."""
        Tw, Tk = _f64(Tw), _f64(Tk)
        C = Tw.shape[0]
        if w % k != 0 or Tw.shape != (C, table_size(w)) or Tk.shape != (C, table_size(k)):
            raise ValueError("need k | w, Tw [C, (2w-1)^2] and Tk [C, (2k-1)^2]")
        M = np.empty((C, w * w, w * w), dtype=np.float64)
        self.lib.oracle_reparam_merge(_ptr(Tw), _ptr(Tk), _ptr(M), C, w, k)
        return M

    def dw3x3(self, y, K):
        """Depthwise 3x3 cross-correlation, zero padding 1 at the image border."""
        y, K = _f64(y), _f64(K)
        if y.ndim != 4:
            raise ValueError("feature map must be [B, C, H, W]")
        B, C, H, W = y.shape
        K = np.ascontiguousarray(K.reshape(C, 9))
        z = np.empty_like(y)
        self.lib.oracle_dw3x3(_ptr(y), _ptr(K), _ptr(z), B, C, H, W)
        return z

    def num_threads(self):
        return int(self.lib.oracle_num_threads())

    @staticmethod
    def forward_cached(x, M, w):
        """Forward with an explicit per-channel matrix M[c] (d x d): y = M_c x_window.

        The plain definition of the cached-inference path; it accepts any M,
        not only one expanded from a table.  numpy matmul is the library
        primitive; windows are ordered n = (b*nh + i)*nw + j.
        """
        x, M = _f64(x), _f64(M)
        B, C, H, W = _check_map(x, w)
        d = w * w
        if M.shape != (C, d, d):
            raise ValueError("M must be [C, d, d]")
        nh, nw = H // w, W // w
        # axes (b, c, i, r, j, s) -> (c, r, s, b, i, j) -> [C, d, windows]
        X = x.reshape(B, C, nh, w, nw, w).transpose(1, 3, 5, 0, 2, 4).reshape(C, d, B * nh * nw)
        Y = np.matmul(M, X)
        # axes (c, p, q, b, i, j) -> (b, c, i, p, j, q)
        y = Y.reshape(C, w, w, B, nh, nw).transpose(3, 0, 4, 1, 5, 2).reshape(B, C, H, W)
        return np.ascontiguousarray(y)


_default = None


def default():
    """The oracle built from the committed wbmm_oracle.c."""
    global _default
    if _default is None:
        _default = Oracle(_build.build())
    return _default


def forward(x, T, w):
    return default().forward(x, T, w)


def backward_dx(dy, T, w):
    return default().backward_dx(dy, T, w)


def backward_dt(x, dy, w):
    return default().backward_dt(x, dy, w)


def expand(T, w):
    return default().expand(T, w)


def reparam_merge(Tw, Tk, w, k):
    return default().reparam_merge(Tw, Tk, w, k)


def dw3x3(y, K):
    return default().dw3x3(y, K)


def forward_cached(x, M, w):
    return Oracle.forward_cached(x, M, w)


def num_threads():
    return default().num_threads()
