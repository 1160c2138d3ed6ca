"""fp64 CPU oracle for the ParaGRU / ParaLSTM Newton-scan solve.

TEST INFRASTRUCTURE ONLY: imported by ``tests/``, ``__graft_entry__.smoke()``
and the CPU-baseline leg of ``bench.py``; never by the library.  It shares no
code with the CUDA path.  All functions take and return float64 numpy arrays
in the library's layouts (``u [B,T,G,D]``, ``a, bias [G,D]``, ``h0, c0 [B,D]``,
states ``[B,T,D]``).  See ``pararnn_oracle.c`` for the definitions and the
passages each one follows.

Pins of each function (tests/test_oracle.py):
  gru_seq / lstm_seq       residual of the result is exactly 0; brute force
  gru_step / lstm_step     Jacobians and gate derivatives vs central differences
  gru_bptt / lstm_bptt     vs finite differences of L = sum(g * h)
  gru_newton / lstm_newton prefix exactness, affine one/two-step convergence,
                           convergence to the sequential root; chan_k equal to
                           each channel's update count when solved alone
  linrec                   closed form and tree-order scans
  dense_gru_*              the general cell: ParaGRU when W is diagonal, torch's
                           GRU cell and autograd Jacobian, prefix exactness and
                           convergence of its Newton to the sequential root
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


def _L():
    global _lib
    if _lib is None:
        path = _build.build()
        _lib = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        i, d = ctypes.c_int, ctypes.c_double
        sig = {
            "oracle_set_threads": (None, [i]),
            "oracle_get_threads": (i, []),
            "oracle_gru_step": (None, [i, dp, dp, dp, dp, dp, dp, dp, dp]),
            "oracle_gru_seq": (None, [dp, dp, dp, dp, dp, i, i, i]),
            "oracle_gru_residual": (None, [dp, dp, dp, dp, dp, dp, i, i, i]),
            "oracle_gru_bptt": (None, [dp, dp, dp, dp, dp, dp, dp, dp, dp, dp,
                                       i, i, i]),
            "oracle_gru_newton": (None, [dp, dp, dp, dp, dp, i, i, i, d, i, dp,
                                         ip, ip]),
            "oracle_linrec": (None, [i, dp, dp, d, dp]),
            "oracle_lstm_step": (None, [i, dp, dp, dp, dp, dp, dp, dp, dp, dp,
                                        dp]),
            "oracle_lstm_seq": (None, [dp, dp, dp, dp, dp, dp, dp, i, i, i]),
            "oracle_lstm_residual": (None, [dp, dp, dp, dp, dp, dp, dp, dp, dp,
                                            i, i, i]),
            "oracle_lstm_bptt": (None, [dp, dp, dp, dp, dp, dp, dp, dp, dp, dp,
                                        dp, dp, dp, i, i, i]),
            "oracle_lstm_newton": (None, [dp, dp, dp, dp, dp, dp, dp, i, i, i,
                                          d, i, dp, ip, ip]),
            "oracle_dense_gru_step": (None, [i, i, dp, dp, dp, dp, dp, dp]),
            "oracle_dense_gru_seq": (None, [dp, dp, dp, dp, dp, i, i, i]),
            "oracle_dense_gru_newton": (None, [dp, dp, dp, dp, dp, i, i, i, d, i,
                                               dp, ip]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(_lib, name)
            fn.restype = res
            fn.argtypes = args
    return _lib


def _p(x):
    if x is None:
        return None
    assert x.dtype == np.float64 and x.flags.c_contiguous
    return x.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor (bf16 widens exactly)
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(x, dtype=np.float64)


def set_threads(n: int) -> None:
    _L().oracle_set_threads(int(n))


def get_threads() -> int:
    return int(_L().oracle_get_threads())


# ----------------------------------------------------------------- ParaGRU --
def gru_step(h, u, a, bias=None):
    """Single step over n channels: h [n], u/a/bias [n,3] ->
    (f [n], A [n], dfdu [n,3], dfda [n,3])."""
    h, u, a, bias = _f64(h), _f64(u), _f64(a), _f64(bias)
    n = h.shape[0]
    f, A = np.empty(n), np.empty(n)
    dfdu, dfda = np.empty((n, 3)), np.empty((n, 3))
    _L().oracle_gru_step(n, _p(h), _p(u), _p(a), _p(bias), _p(f), _p(A),
                         _p(dfdu), _p(dfda))
    return f, A, dfdu, dfda


def gru_seq(u, a, bias=None, h0=None):
    u, a, bias, h0 = _f64(u), _f64(a), _f64(bias), _f64(h0)
    B, T, G, D = u.shape
    assert G == 3
    h = np.empty((B, T, D))
    _L().oracle_gru_seq(_p(u), _p(a), _p(bias), _p(h0), _p(h), B, T, D)
    return h


def gru_residual(u, a, bias, h0, h):
    u, a, bias, h0, h = map(_f64, (u, a, bias, h0, h))
    B, T, _, D = u.shape
    res = np.empty((B, T, D))
    _L().oracle_gru_residual(_p(u), _p(a), _p(bias), _p(h0), _p(h), _p(res),
                             B, T, D)
    return res


def gru_bptt(u, a, bias, h0, h, dLdh):
    """-> dict(du [B,T,3,D], da [3,D], dbias [3,D], dh0 [B,D])"""
    u, a, bias, h0, h, g = map(_f64, (u, a, bias, h0, h, dLdh))
    B, T, _, D = u.shape
    du = np.empty((B, T, 3, D))
    da, db = np.empty((3, D)), np.empty((3, D))
    dh0 = np.empty((B, D))
    _L().oracle_gru_bptt(_p(u), _p(a), _p(bias), _p(h0), _p(h), _p(g), _p(du),
                         _p(da), _p(db), _p(dh0), B, T, D)
    return {"du": du, "da": da, "dbias": db, "dh0": dh0}


def gru_newton(u, a, bias=None, h0=None, tol=1e-6, max_iters=None, h_init=None):
    """-> dict(h, iters, trace (max|r| per iterate), chan_k [B,D])"""
    u, a, bias, h0 = _f64(u), _f64(a), _f64(bias), _f64(h0)
    B, T, _, D = u.shape
    if max_iters is None:
        max_iters = T
    h = np.zeros((B, T, D)) if h_init is None else _f64(h_init).copy()
    trace = np.full(max_iters + 1, np.nan)
    it = ctypes.c_int(0)
    ck = np.zeros((B, D), dtype=np.int32)
    _L().oracle_gru_newton(_p(u), _p(a), _p(bias), _p(h0), _p(h), B, T, D,
                           float(tol), int(max_iters), _p(trace),
                           ctypes.byref(it),
                           ck.ctypes.data_as(ctypes.POINTER(ctypes.c_int)))
    n = it.value
    return {"h": h, "iters": n, "trace": trace[: n + 1], "chan_k": ck}


def linrec(A, b, x0=0.0):
    """x_t = A_t x_{t-1} + b_t by forward substitution."""
    A, b = _f64(A), _f64(b)
    x = np.empty_like(b)
    _L().oracle_linrec(b.shape[0], _p(A), _p(b), float(x0), _p(x))
    return x


# ---------------------------------------------------------------- ParaLSTM --
def lstm_step(c, h, u, a, bias=None):
    """c,h [n], u/a/bias [n,4] -> (fc, fh, A [n,2,2], dfdu [n,2,4],
    dfda [n,2,4]); A rows are (c', h'), columns (c, h)."""
    c, h, u, a, bias = map(_f64, (c, h, u, a, bias))
    n = h.shape[0]
    fc, fh = np.empty(n), np.empty(n)
    A = np.empty((n, 2, 2))
    dfdu, dfda = np.empty((n, 2, 4)), np.empty((n, 2, 4))
    _L().oracle_lstm_step(n, _p(c), _p(h), _p(u), _p(a), _p(bias), _p(fc),
                          _p(fh), _p(A), _p(dfdu), _p(dfda))
    return fc, fh, A, dfdu, dfda


def lstm_seq(u, a, bias=None, c0=None, h0=None):
    u, a, bias, c0, h0 = map(_f64, (u, a, bias, c0, h0))
    B, T, G, D = u.shape
    assert G == 4
    c, h = np.empty((B, T, D)), np.empty((B, T, D))
    _L().oracle_lstm_seq(_p(u), _p(a), _p(bias), _p(c0), _p(h0), _p(c), _p(h),
                         B, T, D)
    return c, h


def lstm_residual(u, a, bias, c0, h0, c, h):
    u, a, bias, c0, h0, c, h = map(_f64, (u, a, bias, c0, h0, c, h))
    B, T, _, D = u.shape
    rc, rh = np.empty((B, T, D)), np.empty((B, T, D))
    _L().oracle_lstm_residual(_p(u), _p(a), _p(bias), _p(c0), _p(h0), _p(c),
                              _p(h), _p(rc), _p(rh), B, T, D)
    return rc, rh


def lstm_bptt(u, a, bias, c0, h0, c, h, dLdh):
    """-> dict(du [B,T,4,D], da [4,D], dbias [4,D], dc0 [B,D], dh0 [B,D])"""
    u, a, bias, c0, h0, c, h, g = map(_f64, (u, a, bias, c0, h0, c, h, dLdh))
    B, T, _, D = u.shape
    du = np.empty((B, T, 4, D))
    da, db = np.empty((4, D)), np.empty((4, D))
    dc0, dh0 = np.empty((B, D)), np.empty((B, D))
    _L().oracle_lstm_bptt(_p(u), _p(a), _p(bias), _p(c0), _p(h0), _p(c), _p(h),
                          _p(g), _p(du), _p(da), _p(db), _p(dc0), _p(dh0),
                          B, T, D)
    return {"du": du, "da": da, "dbias": db, "dc0": dc0, "dh0": dh0}


def lstm_newton(u, a, bias=None, c0=None, h0=None, tol=1e-6, max_iters=None,
                c_init=None, h_init=None):
    u, a, bias, c0, h0 = map(_f64, (u, a, bias, c0, h0))
    B, T, _, D = u.shape
    if max_iters is None:
        max_iters = T
    c = np.zeros((B, T, D)) if c_init is None else _f64(c_init).copy()
    h = np.zeros((B, T, D)) if h_init is None else _f64(h_init).copy()
    trace = np.full(max_iters + 1, np.nan)
    it = ctypes.c_int(0)
    ck = np.zeros((B, D), dtype=np.int32)
    _L().oracle_lstm_newton(_p(u), _p(a), _p(bias), _p(c0), _p(h0), _p(c),
                            _p(h), B, T, D, float(tol), int(max_iters),
                            _p(trace), ctypes.byref(it),
                            ck.ctypes.data_as(ctypes.POINTER(ctypes.c_int)))
    n = it.value
    return {"c": c, "h": h, "iters": n, "trace": trace[: n + 1], "chan_k": ck}


# ------------------------------------------- general cell (dense Jacobian) --
def dense_gru_step(h, u, W, bias=None):
    """GRU with full recurrent matrices, one step over n rows: h [n,D],
    u [n,3,D], W [3,D,D], bias [3,D] -> (h' [n,D], J [n,D,D])."""
    h, u, W, bias = map(_f64, (h, u, W, bias))
    n, D = h.shape
    hn, J = np.empty((n, D)), np.empty((n, D, D))
    _L().oracle_dense_gru_step(n, D, _p(h), _p(u), _p(W), _p(bias), _p(hn), _p(J))
    return hn, J


def dense_gru_seq(u, W, bias=None, h0=None):
    u, W, bias, h0 = map(_f64, (u, W, bias, h0))
    B, T, G, D = u.shape
    assert G == 3 and W.shape == (3, D, D)
    h = np.empty((B, T, D))
    _L().oracle_dense_gru_seq(_p(u), _p(W), _p(bias), _p(h0), _p(h), B, T, D)
    return h


def dense_gru_newton(u, W, bias=None, h0=None, tol=1e-6, max_iters=None, h_init=None):
    """-> dict(h, iters, trace (max|r| per iterate))"""
    u, W, bias, h0 = map(_f64, (u, W, bias, h0))
    B, T, _, D = u.shape
    if max_iters is None:
        max_iters = T
    h = np.zeros((B, T, D)) if h_init is None else _f64(h_init).copy()
    trace = np.full(max_iters + 1, np.nan)
    it = ctypes.c_int(0)
    _L().oracle_dense_gru_newton(_p(u), _p(W), _p(bias), _p(h0), _p(h), B, T, D,
                                 float(tol), int(max_iters), _p(trace), ctypes.byref(it))
    n = it.value
    return {"h": h, "iters": n, "trace": trace[: n + 1]}
