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
* ``hyena_rows`` -- [P4] section 二.1, ``HyenaOperator.forward``: split into
  gates and value, ``for o, x_i in enumerate(reversed(x[1:]))`` gate then
  long conv, output gate ``y = v * x[0]``.
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
