"""ParaGRU / ParaLSTM parallel-in-time Newton solve for B200 (sm_100a).

Thin ctypes binding over ``libpararnn.so`` (C ABI: ``include/pararnn.h``).
The functions named ``pararnn_*`` mirror the C entry points one to one and
only marshal arguments: torch tensors are passed as device pointers, the
current torch CUDA stream is used unless one is given, and a negative return
code raises :class:`PararnnError`.  Every step of the solve runs in the CUDA
kernels; there is no CPU fallback.  If the shared library has not been built
(``python -m nonlinear_rnn_paragru_b200.build``) the first call raises.

Convenience wrappers (:func:`gru_solve`, :func:`lstm_solve`, :func:`adjoint`)
allocate outputs, stats and workspace with torch and call the same entry
points.
"""
import ctypes
import os

import torch

__all__ = [
    "PARARNN_F32", "PARARNN_BF16", "PARARNN_GRU", "PARARNN_LSTM",
    "PararnnOpts", "PararnnError", "library_path", "load_library",
    "pararnn_workspace_size", "pararnn_workspace_init", "pararnn_gru_solve",
    "pararnn_lstm_solve", "pararnn_adjoint", "pararnn_adjoint_ex", "pararnn_adjoint_noalloc",
    "pararnn_seq_baseline", "pararnn_gru_step", "pararnn_lstm_step",
    "pararnn_unfused_workspace_size", "pararnn_solve_unfused", "solve_unfused",
    "pararnn_dense_workspace_size", "pararnn_dense_gru_solve", "dense_gru_solve",
    "pararnn_dense_matmul",
    "pararnn_shard_workspace_size", "pararnn_shard_eval", "pararnn_shard_combine",
    "pararnn_shard_apply",
    "pararnn_strerror", "gru_solve", "lstm_solve", "adjoint", "seq_baseline",
    "gru_step", "lstm_step",
    "Workspace", "read_stats",
]

PARARNN_F32, PARARNN_BF16 = 0, 1
PARARNN_GRU, PARARNN_LSTM = 0, 1
PARARNN_FLAG_INJECT_WITHHOLD = 1
PARARNN_FLAG_FORCE_CHUNKED = 2
PARARNN_FLAG_FORCE_ROW = 4
PARARNN_FLAG_DENSE_SIMT = 8
PARARNN_FLAG_EXACT_STEPS = 16
STATUS_NAMES = {0: "converged", 1: "not_converged", 2: "nonfinite", 3: "timeout"}

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None


class PararnnError(RuntimeError):
    def __init__(self, code, what):
        super().__init__(f"{what}: pararnn error {code} "
                         f"({pararnn_strerror(code) if _LIB else '?'})")
        self.code = code


class PararnnOpts(ctypes.Structure):
    _fields_ = [("tol", ctypes.c_float), ("max_iters", ctypes.c_int),
                ("flags", ctypes.c_uint), ("inject_chunk", ctypes.c_int),
                ("timeout_us", ctypes.c_uint), ("max_cluster", ctypes.c_int),
                ("chan_iters", ctypes.c_void_p)]


def library_path() -> str:
    return os.path.join(_HERE, "libpararnn.so")


def load_library():
    """Load the CUDA library (raises if it is missing: no fallback)."""
    global _LIB
    if _LIB is not None:
        return _LIB
    path = library_path()
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing; build it with "
            "`python -m nonlinear_rnn_paragru_b200.build` (nvcc, sm_100a)")
    lib = ctypes.CDLL(path)
    vp, fp, ip = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
    i, sz = ctypes.c_int, ctypes.c_size_t
    op = ctypes.POINTER(PararnnOpts)
    sigs = {
        "pararnn_workspace_size": (sz, [i, i, i, i, i, i]),
        "pararnn_workspace_init": (i, [vp, sz, vp]),
        "pararnn_gru_solve": (i, [vp, i, fp, fp, fp, fp, i, i, i, op, vp, ip,
                                  vp, sz, vp]),
        "pararnn_lstm_solve": (i, [vp, i, fp, fp, fp, fp, fp, fp, i, i, i, op,
                                   vp, ip, vp, sz, vp]),
        "pararnn_adjoint": (i, [i, vp, i, fp, fp, fp, fp, fp, fp, fp, fp, fp,
                                fp, fp, fp, i, i, i, ip, vp, sz, vp]),
        "pararnn_seq_baseline": (i, [i, vp, i, fp, fp, fp, fp, fp, fp, i, i,
                                     i, vp]),
        "pararnn_adjoint_ex": (i, [i, vp, i, fp, fp, fp, fp, fp, fp, fp, fp, fp,
                                   fp, fp, fp, i, i, i, ip, vp, sz, op, vp]),
        "pararnn_adjoint_noalloc": (i, [i, vp, i, fp, fp, fp, fp, fp, fp, fp,
                                        fp, fp, fp, fp, fp, i, i, i, ip, vp]),
        "pararnn_unfused_workspace_size": (sz, [i, i, i, i]),
        "pararnn_solve_unfused": (i, [i, vp, i, fp, fp, fp, fp, fp, fp, i, i, i,
                                      op, vp, vp, sz, vp]),
        "pararnn_dense_workspace_size": (sz, [i, i, i]),
        "pararnn_dense_matmul": (i, [fp, fp, fp, i, i, i, i, i, ip, vp]),
        "pararnn_dense_gru_solve": (i, [vp, i, fp, fp, fp, fp, i, i, i, op, vp, vp,
                                        sz, vp]),
        "pararnn_shard_workspace_size": (sz, [i, i, i, i]),
        "pararnn_shard_eval": (i, [i, vp, i, fp, fp, fp, fp, fp, fp, i, i, i, fp, fp, fp,
                                   vp, sz, vp]),
        "pararnn_shard_combine": (i, [i, fp, fp, i, i, i, i, fp, fp, vp]),
        "pararnn_shard_apply": (i, [i, fp, fp, fp, i, i, i, vp, sz, vp]),
        "pararnn_gru_step": (i, [vp, i, fp, fp, fp, fp, i, i, vp]),
        "pararnn_lstm_step": (i, [vp, i, fp, fp, fp, fp, fp, fp, i, i, vp]),
        "pararnn_strerror": (ctypes.c_char_p, [i]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _LIB = lib
    return lib


# ------------------------------------------------------------ marshalling --
def _ptr(t, dtype=torch.float32):
    """Device pointer of a contiguous CUDA tensor of `dtype` (None -> NULL)."""
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("pararnn expects contiguous CUDA tensors")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"pararnn expects {dtype}, got {t.dtype}")
    return t.data_ptr()


def _uptr(u):
    return _ptr(u, None)


def _iptr(t):
    return _ptr(t, torch.int32)


def _wptr(t):
    return _ptr(t, None)


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(u):
    if u.dtype == torch.bfloat16:
        return PARARNN_BF16
    if u.dtype == torch.float32:
        return PARARNN_F32
    return -1  # let the library reject it


def _check(rc, what):
    if rc != 0:
        raise PararnnError(rc, what)


def _opts(tol=1e-6, max_iters=0, flags=0, inject_chunk=-1, timeout_us=0,
          max_cluster=0, chan_iters=None):
    return PararnnOpts(float(tol), int(max_iters), int(flags), int(inject_chunk),
                       int(timeout_us), int(max_cluster), _iptr(chan_iters))


# ------------------------------------------------------------ C entry points --
def pararnn_workspace_size(cell, B, T, D, max_iters=0, adjoint=0) -> int:
    return int(load_library().pararnn_workspace_size(cell, B, T, D, max_iters,
                                                     adjoint))


def pararnn_workspace_init(workspace, stream=None):
    _check(load_library().pararnn_workspace_init(
        _wptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)), "pararnn_workspace_init")


def pararnn_gru_solve(u, a, bias, h0, h, opts, stats, iter_hist, workspace,
                      stream=None):
    _check(load_library().pararnn_gru_solve(
        _uptr(u), _dtype_code(u), _ptr(a), _ptr(bias), _ptr(h0), _ptr(h),
        u.shape[0], u.shape[1], u.shape[3], ctypes.byref(opts), _iptr(stats),
        _iptr(iter_hist), _wptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)),
        "pararnn_gru_solve")


def pararnn_lstm_solve(u, a, bias, c0, h0, c, h, opts, stats, iter_hist,
                       workspace, stream=None):
    _check(load_library().pararnn_lstm_solve(
        _uptr(u), _dtype_code(u), _ptr(a), _ptr(bias), _ptr(c0), _ptr(h0),
        _ptr(c), _ptr(h), u.shape[0], u.shape[1], u.shape[3],
        ctypes.byref(opts), _iptr(stats), _iptr(iter_hist), _wptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)),
        "pararnn_lstm_solve")


def pararnn_adjoint(cell, u, a, bias, c0, h0, c, h, dLdh, du, da, dbias, dc0,
                    dh0, status, workspace, stream=None):
    _check(load_library().pararnn_adjoint(
        cell, _uptr(u), _dtype_code(u), _ptr(a), _ptr(bias), _ptr(c0),
        _ptr(h0), _ptr(c), _ptr(h), _ptr(dLdh), _ptr(du), _ptr(da),
        _ptr(dbias), _ptr(dc0), _ptr(dh0), u.shape[0], u.shape[1], u.shape[3],
        _iptr(status), _wptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)),
        "pararnn_adjoint")


def pararnn_adjoint_ex(cell, u, a, bias, c0, h0, c, h, dLdh, du, da, dbias, dc0,
                       dh0, status, workspace, opts, stream=None):
    _check(load_library().pararnn_adjoint_ex(
        cell, _uptr(u), _dtype_code(u), _ptr(a), _ptr(bias), _ptr(c0),
        _ptr(h0), _ptr(c), _ptr(h), _ptr(dLdh), _ptr(du), _ptr(da),
        _ptr(dbias), _ptr(dc0), _ptr(dh0), u.shape[0], u.shape[1], u.shape[3],
        _iptr(status), _wptr(workspace),
        workspace.numel() * workspace.element_size(),
        ctypes.byref(opts) if opts is not None else None, _stream(stream)),
        "pararnn_adjoint_ex")


def pararnn_adjoint_noalloc(cell, u, a, bias, c0, h0, c, h, dLdh, du, da, dbias,
                            dc0, dh0, status, stream=None):
    """pararnn_adjoint with the library's built-in scratch instead of a
    workspace: for callers that cannot provide device scratch memory."""
    _check(load_library().pararnn_adjoint_noalloc(
        cell, _uptr(u), _dtype_code(u), _ptr(a), _ptr(bias), _ptr(c0),
        _ptr(h0), _ptr(c), _ptr(h), _ptr(dLdh), _ptr(du), _ptr(da),
        _ptr(dbias), _ptr(dc0), _ptr(dh0), u.shape[0], u.shape[1], u.shape[3],
        _iptr(status), _stream(stream)), "pararnn_adjoint_noalloc")


def pararnn_seq_baseline(cell, u, a, bias, c0, h0, c, h, stream=None):
    _check(load_library().pararnn_seq_baseline(
        cell, _uptr(u), _dtype_code(u), _ptr(a), _ptr(bias), _ptr(c0),
        _ptr(h0), _ptr(c), _ptr(h), u.shape[0], u.shape[1], u.shape[3],
        _stream(stream)), "pararnn_seq_baseline")


def pararnn_unfused_workspace_size(cell, B, T, D) -> int:
    return int(load_library().pararnn_unfused_workspace_size(cell, B, T, D))


def pararnn_solve_unfused(cell, u, a, bias, c0, h0, c, h, opts, stats, workspace,
                          stream=None):
    _check(load_library().pararnn_solve_unfused(
        cell, _uptr(u), _dtype_code(u), _ptr(a), _ptr(bias), _ptr(c0), _ptr(h0),
        _ptr(c), _ptr(h), u.shape[0], u.shape[1], u.shape[3], ctypes.byref(opts),
        _iptr(stats), _wptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)),
        "pararnn_solve_unfused")


def pararnn_dense_matmul(A, Bm, C, store_mode, err, stream=None):
    """C[z] = A[z] @ Bm[z].T on the tensor cores (tf32 products, fp32 sums):
    A [Z, M, K], Bm [Z, N, K], C [Z, M, N] (or [Z, N, M] transposed per
    store_mode), err int32 [1]."""
    Z, M, K = A.shape
    N = Bm.shape[1]
    _check(load_library().pararnn_dense_matmul(
        _ptr(A), _ptr(Bm), _ptr(C), M, N, K, Z, int(store_mode), _iptr(err), _stream(stream)),
        "pararnn_dense_matmul")


def pararnn_dense_workspace_size(B, T, D) -> int:
    return int(load_library().pararnn_dense_workspace_size(B, T, D))


def pararnn_dense_gru_solve(u, W, bias, h0, h, opts, stats, workspace, stream=None):
    _check(load_library().pararnn_dense_gru_solve(
        _uptr(u), _dtype_code(u), _ptr(W), _ptr(bias), _ptr(h0), _ptr(h), u.shape[0],
        u.shape[1], u.shape[3], ctypes.byref(opts), _iptr(stats), _wptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)),
        "pararnn_dense_gru_solve")


def pararnn_shard_workspace_size(cell, B, Ts, D) -> int:
    return int(load_library().pararnn_shard_workspace_size(cell, B, Ts, D))


def pararnn_shard_eval(cell, u, a, bias, c_bound, h_bound, c, h, agg, last, rmax, workspace,
                       stream=None):
    _check(load_library().pararnn_shard_eval(
        cell, _uptr(u), _dtype_code(u), _ptr(a), _ptr(bias), _ptr(c_bound), _ptr(h_bound),
        _ptr(c), _ptr(h), u.shape[0], u.shape[1], u.shape[3], _ptr(agg), _ptr(last),
        _ptr(rmax), _wptr(workspace), workspace.numel() * workspace.element_size(),
        _stream(stream)), "pararnn_shard_eval")


def pararnn_shard_combine(cell, aggs, lasts, r, din, bound, stream=None):
    W, _, B, D = aggs.shape
    _check(load_library().pararnn_shard_combine(
        cell, _ptr(aggs), _ptr(lasts), W, r, B, D, _ptr(din), _ptr(bound), _stream(stream)),
        "pararnn_shard_combine")


def pararnn_shard_apply(cell, din, c, h, workspace, stream=None):
    B, Ts, D = h.shape
    _check(load_library().pararnn_shard_apply(
        cell, _ptr(din), _ptr(c), _ptr(h), B, Ts, D, _wptr(workspace),
        workspace.numel() * workspace.element_size(), _stream(stream)), "pararnn_shard_apply")


def pararnn_gru_step(u_t, a, bias, h_prev, h_next, stream=None):
    _check(load_library().pararnn_gru_step(
        _uptr(u_t), _dtype_code(u_t), _ptr(a), _ptr(bias), _ptr(h_prev),
        _ptr(h_next), u_t.shape[0], u_t.shape[2], _stream(stream)),
        "pararnn_gru_step")


def pararnn_lstm_step(u_t, a, bias, c_prev, h_prev, c_next, h_next, stream=None):
    _check(load_library().pararnn_lstm_step(
        _uptr(u_t), _dtype_code(u_t), _ptr(a), _ptr(bias), _ptr(c_prev),
        _ptr(h_prev), _ptr(c_next), _ptr(h_next), u_t.shape[0], u_t.shape[2],
        _stream(stream)), "pararnn_lstm_step")


def pararnn_strerror(code) -> str:
    return load_library().pararnn_strerror(int(code)).decode()


# --------------------------------------------------------------- wrappers --
class Workspace:
    """A zero-initialised device workspace that grows on demand."""

    def __init__(self, device="cuda"):
        self.device = device
        self.buf = None

    def get(self, nbytes, stream=None):
        nbytes = max(int(nbytes), 256)
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(nbytes, dtype=torch.uint8, device=self.device)
            pararnn_workspace_init(self.buf, stream)
        return self.buf


def read_stats(stats) -> dict:
    s = stats.cpu()
    return {"iters": int(s[0]), "max_residual": float(s[1:2].view(torch.float32)[0]),
            "status": STATUS_NAMES.get(int(s[2]), int(s[2])), "evals": int(s[3])}


def _new_stats(device):
    return torch.zeros(4, dtype=torch.int32, device=device)


def gru_solve(u, a, bias=None, h0=None, *, tol=1e-6, max_iters=64, hist=False,
              workspace=None, h=None, stats=None, stream=None, opts=None,
              max_cluster=0, flags=0, chan_iters=None):
    """ParaGRU solve -> (h, stats, iter_hist or None).  `chan_iters`: an
    int32 [B, D] CUDA tensor that receives each channel's iteration index."""
    B, T, G, D = u.shape
    dev = u.device
    h = torch.empty((B, T, D), dtype=torch.float32, device=dev) if h is None else h
    stats = _new_stats(dev) if stats is None else stats
    ih = torch.empty(max_iters + 2, dtype=torch.int32, device=dev) if hist else None
    ws = workspace if workspace is not None else Workspace(dev)
    buf = ws.get(pararnn_workspace_size(PARARNN_GRU, B, T, D, max_iters, 0), stream)
    o = opts if opts is not None else _opts(tol, max_iters, flags=flags,
                                            max_cluster=max_cluster,
                                            chan_iters=chan_iters)
    pararnn_gru_solve(u, a, bias, h0, h, o, stats, ih, buf, stream)
    return h, stats, ih


def lstm_solve(u, a, bias=None, c0=None, h0=None, *, tol=1e-6, max_iters=64,
               hist=False, workspace=None, c=None, h=None, stats=None,
               stream=None, opts=None, max_cluster=0, flags=0, chan_iters=None):
    """ParaLSTM solve -> (c, h, stats, iter_hist or None); `chan_iters` as
    for gru_solve."""
    B, T, G, D = u.shape
    dev = u.device
    c = torch.empty((B, T, D), dtype=torch.float32, device=dev) if c is None else c
    h = torch.empty((B, T, D), dtype=torch.float32, device=dev) if h is None else h
    stats = _new_stats(dev) if stats is None else stats
    ih = torch.empty(max_iters + 2, dtype=torch.int32, device=dev) if hist else None
    ws = workspace if workspace is not None else Workspace(dev)
    buf = ws.get(pararnn_workspace_size(PARARNN_LSTM, B, T, D, max_iters, 0), stream)
    o = opts if opts is not None else _opts(tol, max_iters, flags=flags,
                                            max_cluster=max_cluster,
                                            chan_iters=chan_iters)
    pararnn_lstm_solve(u, a, bias, c0, h0, c, h, o, stats, ih, buf, stream)
    return c, h, stats, ih


def adjoint(cell, u, a, bias, h0, h, dLdh, c0=None, c=None, *, workspace=None,
            want_dbias=True, want_dh0=True, stream=None, out=None, opts=None):
    B, T, G, D = u.shape
    dev = u.device
    o = out or {}
    du = o.get("du") if o.get("du") is not None else torch.empty((B, T, G, D), dtype=torch.float32, device=dev)
    da = o.get("da") if o.get("da") is not None else torch.empty((G, D), dtype=torch.float32, device=dev)
    db = (o.get("dbias") if o.get("dbias") is not None else torch.empty((G, D), dtype=torch.float32, device=dev)) if want_dbias else None
    dh0 = (o.get("dh0") if o.get("dh0") is not None else torch.empty((B, D), dtype=torch.float32, device=dev)) if want_dh0 else None
    dc0 = None
    if cell == PARARNN_LSTM and want_dh0:
        dc0 = o.get("dc0") if o.get("dc0") is not None else torch.empty((B, D), dtype=torch.float32, device=dev)
    status = o.get("status") if o.get("status") is not None else torch.zeros(1, dtype=torch.int32, device=dev)
    ws = workspace if workspace is not None else Workspace(dev)
    buf = ws.get(pararnn_workspace_size(cell, B, T, D, 0, 1), stream)
    if opts is None:
        pararnn_adjoint(cell, u, a, bias, c0, h0, c, h, dLdh, du, da, db, dc0, dh0,
                        status, buf, stream)
    else:
        pararnn_adjoint_ex(cell, u, a, bias, c0, h0, c, h, dLdh, du, da, db, dc0, dh0,
                           status, buf, opts, stream)
    return {"du": du, "da": da, "dbias": db, "dh0": dh0, "dc0": dc0,
            "status": status}


def solve_unfused(cell, u, a, bias=None, c0=None, h0=None, *, tol=1e-6, max_iters=64,
                  workspace=None, stream=None):
    """The unfused tier: returns (c, h, stats) with c None for ParaGRU.
    Synchronises the stream (the host checks the residual each iteration)."""
    B, T, G, D = u.shape
    dev = u.device
    h = torch.empty((B, T, D), dtype=torch.float32, device=dev)
    c = torch.empty((B, T, D), dtype=torch.float32, device=dev) if cell == PARARNN_LSTM else None
    stats = _new_stats(dev)
    ws = workspace if workspace is not None else Workspace(dev)
    buf = ws.get(pararnn_unfused_workspace_size(cell, B, T, D), stream)
    pararnn_solve_unfused(cell, u, a, bias, c0, h0, c, h, _opts(tol, max_iters), stats,
                          buf, stream)
    return c, h, stats


def dense_gru_solve(u, W, bias=None, h0=None, *, tol=1e-6, max_iters=64, workspace=None,
                    stream=None, flags=0):
    """Newton solve of the GRU with full recurrent matrices W [3, D, D]:
    returns (h, stats).  Synchronises the stream."""
    B, T, G, D = u.shape
    h = torch.empty((B, T, D), dtype=torch.float32, device=u.device)
    stats = _new_stats(u.device)
    ws = workspace if workspace is not None else Workspace(u.device)
    nbytes = pararnn_dense_workspace_size(B, T, D)
    if nbytes == 0:
        raise PararnnError(-1, "pararnn_dense_workspace_size (unsupported shape)")
    buf = ws.get(nbytes, stream)
    pararnn_dense_gru_solve(u, W, bias, h0, h, _opts(tol, max_iters, flags=flags), stats, buf,
                            stream)
    return h, stats


def gru_step(u_t, a, bias=None, h_prev=None, *, out=None, stream=None):
    """One ParaGRU decode step: u_t [B, 3, D] -> the next state [B, D].
    `out` may be `h_prev` (in-place update)."""
    B, G, D = u_t.shape
    h = torch.empty((B, D), dtype=torch.float32, device=u_t.device) if out is None else out
    pararnn_gru_step(u_t, a, bias, h_prev, h, stream)
    return h


def lstm_step(u_t, a, bias=None, c_prev=None, h_prev=None, *, out=None, stream=None):
    """One ParaLSTM decode step: u_t [B, 4, D] -> (c, h) [B, D] each.
    `out` = (c, h) may be (c_prev, h_prev) (in-place update)."""
    B, G, D = u_t.shape
    if out is None:
        out = (torch.empty((B, D), dtype=torch.float32, device=u_t.device),
               torch.empty((B, D), dtype=torch.float32, device=u_t.device))
    pararnn_lstm_step(u_t, a, bias, c_prev, h_prev, out[0], out[1], stream)
    return out


def seq_baseline(cell, u, a, bias=None, c0=None, h0=None, stream=None):
    B, T, G, D = u.shape
    h = torch.empty((B, T, D), dtype=torch.float32, device=u.device)
    c = torch.empty((B, T, D), dtype=torch.float32, device=u.device) if cell == PARARNN_LSTM else None
    pararnn_seq_baseline(cell, u, a, bias, c0, h0, c, h, stream)
    return c, h
