"""float64 CPU oracle for the Hyena gated long convolution.

TEST INFRASTRUCTURE ONLY: the product path never imports this package.  Only
``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` / reference
leg of ``bench.py`` use it.  It shares no code with the CUDA library.

The arithmetic lives in ``hyena_oracle.c`` (plain C, double precision); this
module compiles it with gcc on first use and marshals numpy arrays through
ctypes.  Sources, per function:

* ``shortconv`` -- [P4] "HyenaDNA operator walk-through" (adg.csdn.net),
  section 二.1: depthwise Conv1d, kernel 3, padding 2, first L outputs kept.
* ``causal_conv_direct`` / ``causal_conv_fft`` -- [P4] section 二.2:
  ``fftconv(x, k, bias)``, the FFT evaluation of a long causal convolution
  plus the per-channel skip.
* ``conv2d_direct`` / ``conv2d_fft`` -- [P5] "Native Multi-Dimensional
  Subquadratic Operators via Input Dependent Long Convolutions", 方法论
  (原生 ND 卷积, 边界处理): N-D FFT convolution, non-circular by zero-padding
  each axis to twice its length.
* ``split_rows`` -- [P4] section 二.1, ``*x, v = uc.split(d_model, dim=1)``:
  chunk j of row (b, c) of the stacked stream is channel j*C + c (taps and
  bias alike); filters at index c, or b*C + c for per-sample filters.
* ``hyena_rows`` -- [P4] section 二.1, ``HyenaOperator.forward`` on one row's
  chunks: ``for o, x_i in enumerate(reversed(x[1:]))`` gate then long conv,
  output gate ``y = v * x[0]``.
* ``hyena_stacked`` -- the two above on the stacked tensors the CUDA path
  receives.
* ``in_proj`` / ``out_proj`` -- [P4] section 二.1: ``in_proj =
  nn.Linear(d_model, (order+1) d_model)`` followed by ``rearrange(u, 'b l d
  -> b d l')``, and ``out_proj = nn.Linear(d_model, d_model)`` applied to
  ``rearrange(y, 'b d l -> b l d')`` (``nn.Linear(x) = x W^T + bias``).
* ``conv2d_circ_*`` -- [P5] 边界处理: the circular (periodic) 2-D form.
* ``conv3d_*`` / ``hyena_rows3`` -- [P5] 原生 ND 卷积: the 3-D form.
* ``fft`` -- a hand-written iterative radix-2 FFT (the textbook algorithm).
* ``filter_gen`` (submodule) -- [P4] section 二.2: the implicit filter
  (positional embedding -> MLP with Sin -> exponential modulation), plain
  numpy in float64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "hyena_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "liboracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


def build(force: bool = False, src: str = _SRC, out: str = _LIB) -> str:
    """Compile the oracle C source into a shared library (gcc, OpenMP)."""
    os.makedirs(os.path.dirname(out), exist_ok=True)
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        tmp = out + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c99",
                               "-o", tmp, src, "-lm"])
        os.replace(tmp, out)
    return out


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_dp)


class Oracle:
    """ctypes view of one build of hyena_oracle.c."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        lib.oracle_shortconv_row.argtypes = [_dp, _dp, _dp, ctypes.c_double, _i64]
        lib.oracle_causal_conv_direct.argtypes = [_dp, ctypes.c_double, _dp, _dp, _i64]
        lib.oracle_causal_conv_fft.argtypes = [_dp, ctypes.c_double, _dp, _dp, _i64]
        lib.oracle_fft.argtypes = [_dp, _dp, _i64, ctypes.c_int]
        lib.oracle_conv2d_direct.argtypes = [_dp, ctypes.c_double, _dp, _dp, _i64, _i64]
        lib.oracle_conv2d_fft.argtypes = [_dp, ctypes.c_double, _dp, _dp, _i64, _i64]
        lib.oracle_conv2d_circ_direct.argtypes = [_dp, ctypes.c_double, _dp, _dp, _i64, _i64]
        lib.oracle_conv3d_direct.argtypes = [_dp, ctypes.c_double, _dp, _dp, _i64, _i64, _i64]
        lib.oracle_conv3d_fft.argtypes = [_dp, ctypes.c_double, _dp, _dp, _i64, _i64, _i64]
        lib.oracle_hyena_rows3.argtypes = [_dp, _dp, _dp, _i64, _i64, _i64, _i64, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, _dp]
        lib.oracle_hyena_rows3.restype = ctypes.c_int
        lib.oracle_conv2d_circ_fft.argtypes = [_dp, ctypes.c_double, _dp, _dp, _i64, _i64]
        lib.oracle_hyena_rows.argtypes = [_dp, _dp, _dp, _dp, _dp, _i64, _i64, _i64,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, _dp]
        lib.oracle_hyena_rows.restype = ctypes.c_int
        lib.oracle_split_rows.argtypes = [ctypes.c_void_p, ctypes.c_int, ctypes.c_void_p, ctypes.c_int, _dp, _dp,
                                          _dp, _i64, _i64, ctypes.c_int, _i64, ctypes.c_int,
                                          ctypes.POINTER(_i64), _i64, _dp, _dp, _dp, _dp, _dp]
        lib.oracle_split_rows.restype = ctypes.c_int
        lib.oracle_in_proj.argtypes = [_dp, _dp, _dp, _i64, _i64, _i64, _i64, _dp]
        lib.oracle_out_proj.argtypes = [_dp, _dp, _dp, _i64, _i64, _i64, _i64, _dp]
        lib.oracle_max_threads.restype = ctypes.c_int
        self.lib = lib
        self.path = path

    def max_threads(self) -> int:
        return int(self.lib.oracle_max_threads())

    def shortconv(self, u, w, bias: float = 0.0) -> np.ndarray:
        """One channel: out[t] = w[0] u[t-2] + w[1] u[t-1] + w[2] u[t] + bias."""
        u = _f64(u); w = _f64(w)
        out = np.empty_like(u)
        self.lib.oracle_shortconv_row(_ptr(u), _ptr(out), _ptr(w), float(bias), u.shape[-1])
        return out

    def causal_conv_direct(self, k, D: float, x) -> np.ndarray:
        """out[t] = sum_{tau<=t} k[tau] x[t-tau] + D x[t] by its direct sum."""
        k = _f64(k); x = _f64(x)
        out = np.empty_like(x)
        self.lib.oracle_causal_conv_direct(_ptr(k), float(D), _ptr(x), _ptr(out), x.shape[-1])
        return out

    def causal_conv_fft(self, k, D: float, x) -> np.ndarray:
        """The same causal convolution through a zero-padded radix-2 FFT."""
        k = _f64(k); x = _f64(x)
        out = np.empty_like(x)
        self.lib.oracle_causal_conv_fft(_ptr(k), float(D), _ptr(x), _ptr(out), x.shape[-1])
        return out

    def fft(self, z, inverse: bool = False) -> np.ndarray:
        """Hand-written radix-2 FFT (unnormalised inverse when inverse=True)."""
        z = np.asarray(z, dtype=np.complex128)
        re = np.ascontiguousarray(z.real.copy()); im = np.ascontiguousarray(z.imag.copy())
        self.lib.oracle_fft(_ptr(re), _ptr(im), re.shape[-1], +1 if inverse else -1)
        return re + 1j * im

    def conv2d_direct(self, K, D: float, x) -> np.ndarray:
        K = _f64(K); x = _f64(x)
        out = np.empty_like(x)
        self.lib.oracle_conv2d_direct(_ptr(K), float(D), _ptr(x), _ptr(out), x.shape[0], x.shape[1])
        return out

    def conv2d_fft(self, K, D: float, x) -> np.ndarray:
        K = _f64(K); x = _f64(x)
        out = np.empty_like(x)
        self.lib.oracle_conv2d_fft(_ptr(K), float(D), _ptr(x), _ptr(out), x.shape[0], x.shape[1])
        return out

    def conv2d_circ_direct(self, K, D: float, x) -> np.ndarray:
        """Circular 2-D convolution by its direct sum ([P5] 边界处理)."""
        K = _f64(K); x = _f64(x)
        out = np.empty_like(x)
        self.lib.oracle_conv2d_circ_direct(_ptr(K), float(D), _ptr(x), _ptr(out), x.shape[0], x.shape[1])
        return out

    def conv2d_circ_fft(self, K, D: float, x) -> np.ndarray:
        """The same through an unpadded H x W radix-2 FFT."""
        K = _f64(K); x = _f64(x)
        out = np.empty_like(x)
        self.lib.oracle_conv2d_circ_fft(_ptr(K), float(D), _ptr(x), _ptr(out), x.shape[0], x.shape[1])
        return out

    def conv3d_direct(self, K, D: float, x) -> np.ndarray:
        """3-D non-circular convolution by its direct sum ([P5] 原生 ND 卷积)."""
        K = _f64(K); x = _f64(x)
        out = np.empty_like(x)
        self.lib.oracle_conv3d_direct(_ptr(K), float(D), _ptr(x), _ptr(out), *x.shape)
        return out

    def conv3d_fft(self, K, D: float, x) -> np.ndarray:
        """The same through a zero-padded (2x per axis) radix-2 3-D FFT."""
        K = _f64(K); x = _f64(x)
        out = np.empty_like(x)
        self.lib.oracle_conv3d_fft(_ptr(K), float(D), _ptr(x), _ptr(out), *x.shape)
        return out

    def hyena_rows3(self, u_rows, k_rows, D_rows, *, method: int = 2, nthreads: int = 0) -> np.ndarray:
        """The operator on self-contained 3-D rows: u_rows [R, order+1, N1, N2, N3],
        k_rows [R, order-1, N1, N2, N3], D_rows [R, order-1]; y [R, N1, N2, N3]."""
        u_rows = _f64(u_rows); k_rows = _f64(k_rows); D_rows = _f64(D_rows)
        R, ch = u_rows.shape[0], u_rows.shape[1]
        order = ch - 1
        N1, N2, N3 = u_rows.shape[2:]
        if k_rows.shape != (R, order - 1, N1, N2, N3) or D_rows.shape != (R, order - 1):
            raise ValueError("k_rows / D_rows shape does not match u_rows")
        y = np.empty((R, N1, N2, N3), dtype=np.float64)
        rc = self.lib.oracle_hyena_rows3(_ptr(u_rows), _ptr(k_rows), _ptr(D_rows), R, N1, N2, N3, order, method,
                                         nthreads, _ptr(y))
        if rc != 0:
            raise ValueError("oracle_hyena_rows3 rejected its arguments")
        return y

    def hyena_rows(self, u_rows, k_rows, D_rows, sc_w_rows=None, sc_b_rows=None, *,
                   ndim: int = 1, method: int = 0, nthreads: int = 0,
                   circular: bool = False) -> np.ndarray:
        """The operator on self-contained rows.

        u_rows   : [R, order+1, L] (1-D) or [R, order+1, H, W] (2-D) -- chunks
                   x0..x(order-1), v of one (b, c), before the short conv
        k_rows   : [R, order-1, L] or [R, order-1, H, W]
        D_rows   : [R, order-1]
        sc_w_rows: [R, order+1, 3] or None;  sc_b_rows: [R, order+1] or None
        method   : 1 direct sums, 2 FFT, 0 direct when small
        circular : 2-D only: the circular (periodic) form instead of the
                   zero-padded one
        Returns y: [R, L] or [R, H, W] in float64.
        """
        if circular and ndim != 2:
            raise ValueError("the circular form is 2-D")
        u_rows = _f64(u_rows); k_rows = _f64(k_rows); D_rows = _f64(D_rows)
        R, ch = u_rows.shape[0], u_rows.shape[1]
        order = ch - 1
        if ndim == 1:
            H, W = 1, u_rows.shape[2]
        else:
            H, W = u_rows.shape[2], u_rows.shape[3]
        if k_rows.shape[:2] != (R, order - 1) or D_rows.shape != (R, order - 1):
            raise ValueError("k_rows / D_rows shape does not match u_rows")
        scw = None if sc_w_rows is None else _f64(sc_w_rows)
        scb = None if sc_b_rows is None else _f64(sc_b_rows)
        if scw is not None and scw.shape != (R, order + 1, 3):
            raise ValueError("sc_w_rows must be [R, order+1, 3]")
        y = np.empty((R, H * W), dtype=np.float64)
        rc = self.lib.oracle_hyena_rows(_ptr(u_rows), _ptr(k_rows), _ptr(D_rows), _ptr(scw),
                                        _ptr(scb), R, H, W, 3 if circular else ndim, order, method,
                                        nthreads, _ptr(y))
        if rc != 0:
            raise ValueError("oracle_hyena_rows rejected its arguments")
        return y.reshape((R, W) if ndim == 1 else (R, H, W))

    def split_rows(self, u, k, D, sc_w=None, sc_b=None, *, B: int, C: int, order: int, shape,
                   rows=None, per_sample: bool = False):
        """The split of the stacked projected stream ([P4] 二.1,
        ``*x, v = uc.split(d_model, dim=1)``), done by ``oracle_split_rows``.

        u    : [B, (order+1)*C, *shape] -- float64, float32, or uint16 holding
               bfloat16 bit patterns (exact values are used)
        k    : [order-1, FC, *shape] (same element kinds); FC = C, or B*C with
               per_sample (filter of row (b, c) at index b*C + c)
        D    : [order-1, FC] or None;  sc_w: [(order+1)*C, 3] or None;
        sc_b : [(order+1)*C] or None
        rows : row ids b*C + c (default: all B*C rows in order)
        Returns the self-contained rows of ``hyena_rows``: u_rows
        [R, order+1, *shape], k_rows [R, order-1, *shape], D_rows
        [R, order-1], sc_w_rows [R, order+1, 3] or None, sc_b_rows or None.
        """
        shape = tuple(int(x) for x in shape)
        n = int(np.prod(shape))
        rows = np.ascontiguousarray(np.arange(B * C) if rows is None else rows, dtype=np.int64).reshape(-1)
        R = rows.size
        FC = B * C if per_sample else C
        u = np.ascontiguousarray(u)
        k = np.ascontiguousarray(k)
        if u.shape != (B, (order + 1) * C) + shape:
            raise ValueError(f"u must be [B, (order+1)*C, *shape] = {(B, (order + 1) * C) + shape}, got {u.shape}")
        if k.shape != (order - 1, FC) + shape:
            raise ValueError(f"k must be [order-1, FC, *shape] = {(order - 1, FC) + shape}, got {k.shape}")
        Dd = None if D is None else _f64(D)
        if Dd is not None and Dd.shape != (order - 1, FC):
            raise ValueError("D must be [order-1, FC]")
        scw = None if sc_w is None else _f64(sc_w)
        scb = None if (sc_w is None or sc_b is None) else _f64(sc_b)
        if scw is not None and scw.shape != ((order + 1) * C, 3):
            raise ValueError("sc_w must be [(order+1)*C, 3]")
        u_rows = np.empty((R, order + 1) + shape, dtype=np.float64)
        k_rows = np.empty((R, order - 1) + shape, dtype=np.float64)
        D_rows = np.empty((R, order - 1), dtype=np.float64)
        scw_rows = np.empty((R, order + 1, 3), dtype=np.float64) if scw is not None else None
        scb_rows = np.empty((R, order + 1), dtype=np.float64) if scw is not None else None
        rc = self.lib.oracle_split_rows(u.ctypes.data, _kind(u), k.ctypes.data, _kind(k), _ptr(Dd), _ptr(scw),
                                        _ptr(scb), B, C, order, n, 1 if per_sample else 0,
                                        rows.ctypes.data_as(ctypes.POINTER(_i64)), R, _ptr(u_rows),
                                        _ptr(k_rows), _ptr(D_rows), _ptr(scw_rows), _ptr(scb_rows))
        if rc != 0:
            raise ValueError("oracle_split_rows rejected its arguments")
        return u_rows, k_rows, D_rows, scw_rows, scb_rows

    def hyena_stacked(self, u, k, D, sc_w=None, sc_b=None, *, B: int, C: int, order: int, shape,
                      rows=None, per_sample: bool = False, circular: bool = False, method: int = 0,
                      nthreads: int = 0) -> np.ndarray:
        """The operator on the stacked tensors the CUDA path receives
        (u [B, (order+1)*C, *shape] -> y rows [R, *shape], R = len(rows),
        default all B*C rows in order b*C + c): ``split_rows`` followed by
        ``hyena_rows`` (1-D, 2-D) or ``hyena_rows3`` (3-D)."""
        shape = tuple(int(x) for x in shape)
        u_rows, k_rows, D_rows, w, b = self.split_rows(u, k, D, sc_w, sc_b, B=B, C=C, order=order, shape=shape,
                                                       rows=rows, per_sample=per_sample)
        if len(shape) == 3:
            if w is not None:
                raise ValueError("the 3-D form has no short conv")
            return self.hyena_rows3(u_rows, k_rows, D_rows, method=2 if method == 0 else method,
                                    nthreads=nthreads)
        return self.hyena_rows(u_rows, k_rows, D_rows, w, b, ndim=len(shape), method=method, nthreads=nthreads,
                               circular=circular)

    def in_proj(self, x, W, bias=None) -> np.ndarray:
        """x [B, L, D], W [J, D] (nn.Linear weight), bias [J] or None ->
        u [B, J, L] = rearrange(x W^T + bias, 'b l d -> b d l').  Arrays may
        be float64, float32 or uint16 bfloat16 bit patterns."""
        x = _values(x); W = _values(W)
        B, L, D = x.shape
        J = W.shape[0]
        if W.shape != (J, D):
            raise ValueError("W must be [J, D]")
        b = None if bias is None else _f64(bias)
        u = np.empty((B, J, L), dtype=np.float64)
        self.lib.oracle_in_proj(_ptr(x), _ptr(W), _ptr(b), B, L, D, J, _ptr(u))
        return u

    def out_proj(self, y, W, bias=None) -> np.ndarray:
        """y [B, D, L], W [J, D], bias [J] or None -> out [B, L, J] =
        rearrange(y, 'b d l -> b l d') W^T + bias."""
        y = _values(y); W = _values(W)
        B, D, L = y.shape
        J = W.shape[0]
        if W.shape != (J, D):
            raise ValueError("W must be [J, D]")
        b = None if bias is None else _f64(bias)
        out = np.empty((B, L, J), dtype=np.float64)
        self.lib.oracle_out_proj(_ptr(y), _ptr(W), _ptr(b), B, L, D, J, _ptr(out))
        return out


def _values(a) -> np.ndarray:
    """Exact float64 values of an array of float64, float32 or uint16
    bfloat16 bit patterns (the upper 16 bits of an IEEE binary32)."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return np.ascontiguousarray((a.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64))
    return _f64(a)


def _kind(a: np.ndarray) -> int:
    """Element kind of a stacked tensor for oracle_split_rows."""
    if a.dtype == np.float64:
        return 0
    if a.dtype == np.float32:
        return 1
    if a.dtype == np.uint16:
        return 2          # bfloat16 bit patterns
    raise ValueError(f"unsupported element type {a.dtype} (float64, float32 or uint16 bf16 bits)")


def default() -> Oracle:
    """The oracle built from hyena_oracle.c as committed."""
    global _lib
    with _lock:
        if _lib is None:
            _lib = Oracle(build())
    return _lib


def max_threads() -> int:
    return default().max_threads()


def shortconv(u, w, bias: float = 0.0):
    return default().shortconv(u, w, bias)


def causal_conv_direct(k, D, x):
    return default().causal_conv_direct(k, D, x)


def causal_conv_fft(k, D, x):
    return default().causal_conv_fft(k, D, x)


def fft(z, inverse: bool = False):
    return default().fft(z, inverse)


def conv2d_direct(K, D, x):
    return default().conv2d_direct(K, D, x)


def conv2d_fft(K, D, x):
    return default().conv2d_fft(K, D, x)


def conv2d_circ_direct(K, D, x):
    return default().conv2d_circ_direct(K, D, x)


def conv2d_circ_fft(K, D, x):
    return default().conv2d_circ_fft(K, D, x)


def conv3d_direct(K, D, x):
    return default().conv3d_direct(K, D, x)


def conv3d_fft(K, D, x):
    return default().conv3d_fft(K, D, x)


def hyena_rows3(u_rows, k_rows, D_rows, **kw):
    return default().hyena_rows3(u_rows, k_rows, D_rows, **kw)


def hyena_rows(u_rows, k_rows, D_rows, sc_w_rows=None, sc_b_rows=None, **kw):
    return default().hyena_rows(u_rows, k_rows, D_rows, sc_w_rows, sc_b_rows, **kw)


def split_rows(u, k, D, sc_w=None, sc_b=None, **kw):
    return default().split_rows(u, k, D, sc_w, sc_b, **kw)


def hyena_stacked(u, k, D, sc_w=None, sc_b=None, **kw):
    return default().hyena_stacked(u, k, D, sc_w, sc_b, **kw)


def in_proj(x, W, bias=None):
    return default().in_proj(x, W, bias)


def out_proj(y, W, bias=None):
    return default().out_proj(y, W, bias)
