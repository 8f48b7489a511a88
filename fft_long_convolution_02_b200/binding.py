"""Thin ctypes binding of libhyena_b200.so (declared in include/hyena.h).

Argument marshalling only: every step of the operator runs in the CUDA
library.  Tensors are torch CUDA tensors (torch supplies device memory and
streams); the functions take the same names as the C entry points.  There
is no fallback: if the shared library is missing, loading raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhyena_b200.so")

HYENA_F32, HYENA_BF16 = 0, 1
STATUS = {0: "HYENA_OK", 1: "HYENA_ERR_INVALID_ARG", 2: "HYENA_ERR_UNSUPPORTED_SHAPE",
          3: "HYENA_ERR_MISALIGNED", 4: "HYENA_ERR_SPECTRUM_MISMATCH",
          5: "HYENA_ERR_WORKSPACE_TOO_SMALL", 6: "HYENA_ERR_CUDA", 7: "HYENA_ERR_INTERNAL",
          8: "HYENA_ERR_TIMEOUT"}

# every symbol include/hyena.h declares
EXPORTS = ["hyena_version", "hyena_status_string", "hyena_last_error_detail", "hyena_spectrum_bytes",
           "hyena_filter_spectrum", "hyena_shortconv", "hyena_gated_fftconv_workspace_bytes",
           "hyena_gated_fftconv_workspace_min_bytes", "hyena_gated_fftconv", "hyena_gated_fftconv_noalloc",
           "hyena_gated_fftconv_per_sample", "hyena_gated_fftconv_host", "hyena_spectrum_check",
           "hyena_debug_conv_tc", "hyena_debug_conv_cluster", "hyena_debug_conv_2d_tc", "hyena_debug_conv_2dc_tc", "hyena_gated_fftconv_ex", "hyena_kernel_status", "hyena_in_proj",
           "hyena_out_proj", "hyena_implicit_filter_workspace_bytes", "hyena_filter_spectrum_implicit"]

_lock = threading.Lock()
_lib = None


class HyenaError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{STATUS.get(status, status)}: {detail}")
        self.status = status
        self.detail = detail


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise RuntimeError(f"{path} is missing: build it with "
                               "`python -m fft_long_convolution_02_b200.build`")
        lib = ctypes.CDLL(path)
        i64, vp, sz, fp = ctypes.c_int64, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p
        i64p = ctypes.POINTER(ctypes.c_int64)
        lib.hyena_version.restype = ctypes.c_int
        lib.hyena_status_string.restype = ctypes.c_char_p
        lib.hyena_status_string.argtypes = [ctypes.c_int]
        lib.hyena_last_error_detail.restype = ctypes.c_char_p
        lib.hyena_spectrum_bytes.restype = sz
        lib.hyena_spectrum_bytes.argtypes = [i64, ctypes.c_int, i64p, ctypes.c_int]
        lib.hyena_filter_spectrum.restype = ctypes.c_int
        lib.hyena_filter_spectrum.argtypes = [vp, ctypes.c_int, fp, i64, ctypes.c_int, i64p, ctypes.c_int,
                                              vp, sz, vp]
        lib.hyena_shortconv.restype = ctypes.c_int
        lib.hyena_shortconv.argtypes = [vp, vp, fp, fp, i64, i64, i64, ctypes.c_int, vp]
        lib.hyena_gated_fftconv_workspace_bytes.restype = sz
        lib.hyena_gated_fftconv_workspace_bytes.argtypes = [i64, i64, ctypes.c_int, i64p, ctypes.c_int]
        lib.hyena_gated_fftconv_workspace_min_bytes.restype = sz
        lib.hyena_gated_fftconv_workspace_min_bytes.argtypes = [i64, ctypes.c_int, i64p, ctypes.c_int]
        lib.hyena_gated_fftconv.restype = ctypes.c_int
        lib.hyena_gated_fftconv.argtypes = [vp, vp, vp, sz, fp, fp, i64, i64, ctypes.c_int, i64p, ctypes.c_int,
                                            ctypes.c_int, vp, sz, vp]
        lib.hyena_gated_fftconv_per_sample.restype = ctypes.c_int
        lib.hyena_gated_fftconv_per_sample.argtypes = [vp, vp, vp, sz, fp, fp, i64, i64, ctypes.c_int, i64p,
                                                       ctypes.c_int, ctypes.c_int, vp, sz, vp]
        lib.hyena_gated_fftconv_host.restype = ctypes.c_int
        lib.hyena_gated_fftconv_host.argtypes = [vp, vp, vp, vp, vp, sz, fp, fp, i64, i64, ctypes.c_int, i64p,
                                                 ctypes.c_int, ctypes.c_int, vp, sz, i64, vp]
        lib.hyena_gated_fftconv_noalloc.restype = ctypes.c_int
        lib.hyena_gated_fftconv_noalloc.argtypes = [vp, vp, vp, sz, fp, fp, i64, i64, ctypes.c_int, i64p,
                                                    ctypes.c_int, ctypes.c_int, vp]
        lib.hyena_gated_fftconv_ex.restype = ctypes.c_int
        lib.hyena_gated_fftconv_ex.argtypes = [vp, vp, vp, sz, fp, fp, i64, i64, ctypes.c_int, i64p, ctypes.c_int,
                                               ctypes.c_int, vp, sz, ctypes.c_uint, vp]
        lib.hyena_in_proj.restype = ctypes.c_int
        lib.hyena_in_proj.argtypes = [vp, vp, fp, vp, i64, i64, i64, ctypes.c_int, vp]
        lib.hyena_out_proj.restype = ctypes.c_int
        lib.hyena_out_proj.argtypes = [vp, vp, fp, vp, i64, i64, i64, vp]
        lib.hyena_implicit_filter_workspace_bytes.restype = sz
        lib.hyena_implicit_filter_workspace_bytes.argtypes = [i64, ctypes.c_int]
        lib.hyena_filter_spectrum_implicit.restype = ctypes.c_int
        lib.hyena_filter_spectrum_implicit.argtypes = [ctypes.POINTER(ImplicitFilter), fp, i64, i64, ctypes.c_int, vp,
                                                       sz, vp, sz, fp, vp]
        lib.hyena_kernel_status.restype = ctypes.c_int
        lib.hyena_kernel_status.argtypes = [vp]
        lib.hyena_spectrum_check.restype = ctypes.c_int
        lib.hyena_spectrum_check.argtypes = [vp, i64, ctypes.c_int, i64p, ctypes.c_int, vp]
        lib.hyena_debug_conv_tc.restype = ctypes.c_int
        lib.hyena_debug_conv_tc.argtypes = [vp, vp, vp, sz, fp, fp, i64, i64, ctypes.c_int, ctypes.c_uint64,
                                            ctypes.c_int, vp]
        lib.hyena_debug_conv_cluster.restype = ctypes.c_int
        lib.hyena_debug_conv_cluster.argtypes = [vp, vp, vp, sz, fp, fp, i64, i64, ctypes.c_int, vp, sz,
                                                 ctypes.c_uint64, ctypes.c_int, vp]
        lib.hyena_debug_conv_2d_tc.restype = ctypes.c_int
        lib.hyena_debug_conv_2d_tc.argtypes = [vp, vp, vp, sz, i64, i64, i64, ctypes.c_int, vp, sz,
                                               ctypes.c_uint64, ctypes.c_int, vp]
        lib.hyena_debug_conv_2dc_tc.restype = ctypes.c_int
        lib.hyena_debug_conv_2dc_tc.argtypes = [vp, vp, vp, sz, i64, i64, ctypes.c_int, vp, sz,
                                                ctypes.c_uint64, ctypes.c_int, vp]
        _lib = lib
    return _lib


HYENA_CIRCULAR = 0x100   # include/hyena.h: OR-ed into ndim for the circular 2-D form


class Circular(tuple):
    """sizes (H, W) of the circular (periodic) 2-D form: pass Circular((H, W))
    wherever a shape is taken."""


def _sizes(sizes):
    circ = isinstance(sizes, Circular)
    sizes = [int(s) for s in sizes]
    nd = len(sizes)
    if circ:
        if nd != 2:
            raise ValueError("the circular form is 2-D")
        nd |= HYENA_CIRCULAR
    return (ctypes.c_int64 * len(sizes))(*sizes), nd


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return HYENA_F32
    if t.dtype == torch.bfloat16:
        return HYENA_BF16
    raise TypeError(f"unsupported tensor dtype {t.dtype}")


def _check(rc: int):
    if rc != 0:
        detail = load().hyena_last_error_detail().decode()
        raise HyenaError(rc, detail)


def hyena_version() -> int:
    return load().hyena_version()


def hyena_spectrum_bytes(C: int, sizes, order: int) -> int:
    arr, nd = _sizes(sizes)
    return int(load().hyena_spectrum_bytes(C, nd, arr, order))


def hyena_gated_fftconv_workspace_bytes(B: int, C: int, sizes, order: int) -> int:
    arr, nd = _sizes(sizes)
    return int(load().hyena_gated_fftconv_workspace_bytes(B, C, nd, arr, order))


def hyena_gated_fftconv_workspace_min_bytes(C: int, sizes, order: int) -> int:
    arr, nd = _sizes(sizes)
    return int(load().hyena_gated_fftconv_workspace_min_bytes(C, nd, arr, order))


def hyena_filter_spectrum(k, D, C: int, sizes, order: int, spectrum, stream=None) -> None:
    """k: [order-1, C, *sizes] (f32/bf16 CUDA), D: [order-1, C] f32 or None,
    spectrum: uint8 CUDA tensor of hyena_spectrum_bytes(...) bytes."""
    arr, nd = _sizes(sizes)
    _check(load().hyena_filter_spectrum(_ptr(k), _dtype_code(k), _ptr(D), C, nd, arr, order, _ptr(spectrum),
                                        spectrum.numel() * spectrum.element_size(), _stream(stream)))


def hyena_shortconv(u, out, w, bias=None, stream=None) -> None:
    """u, out: [B, Ctot, L]; w: [Ctot, 3] f32; bias: [Ctot] f32 or None."""
    B, Ctot, L = u.shape
    _check(load().hyena_shortconv(_ptr(u), _ptr(out), _ptr(w), _ptr(bias), B, Ctot, L, _dtype_code(u),
                                  _stream(stream)))


def hyena_gated_fftconv(u, y, spectrum, sc_w, sc_bias, B: int, C: int, sizes, order: int, workspace=None,
                        stream=None) -> None:
    """u: [B, (order+1)*C, *sizes], y: [B, C, *sizes] (same dtype), spectrum from
    hyena_filter_spectrum, sc_w [(order+1)*C, 3] f32 or None, workspace uint8 or None."""
    arr, nd = _sizes(sizes)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().hyena_gated_fftconv(_ptr(u), _ptr(y), _ptr(spectrum), spectrum.numel() * spectrum.element_size(),
                                      _ptr(sc_w), _ptr(sc_bias), B, C, nd, arr, order, _dtype_code(u),
                                      _ptr(workspace), ws_bytes, _stream(stream)))


HYENA_FLAG_FP32_TRANSFORM = 0x1


def hyena_gated_fftconv_ex(u, y, spectrum, sc_w, sc_bias, B: int, C: int, sizes, order: int, workspace=None,
                           flags: int = 0, stream=None) -> None:
    """hyena_gated_fftconv with flags (HYENA_FLAG_FP32_TRANSFORM: the fp32
    transform at L = 8192 with bf16 storage)."""
    arr, nd = _sizes(sizes)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().hyena_gated_fftconv_ex(_ptr(u), _ptr(y), _ptr(spectrum), spectrum.numel() * spectrum.element_size(),
                                         _ptr(sc_w), _ptr(sc_bias), B, C, nd, arr, order, _dtype_code(u),
                                         _ptr(workspace), ws_bytes, int(flags), _stream(stream)))


def hyena_in_proj(x, W, bias, u, order: int, stream=None) -> None:
    """x [B, L, D] bf16, W [(order+1)*D, D] bf16, bias [(order+1)*D] f32 or
    None -> u [B, (order+1)*D, L] bf16 (in_proj then 'b l d -> b d l')."""
    B, L, D = x.shape
    _check(load().hyena_in_proj(_ptr(x), _ptr(W), _ptr(bias), _ptr(u), B, L, D, int(order), _stream(stream)))


def hyena_out_proj(y, W, bias, out, stream=None) -> None:
    """y [B, D, L] bf16, W [D, D] bf16, bias [D] f32 or None -> out [B, L, D]
    bf16 ('b d l -> b l d' then out_proj)."""
    B, D, L = y.shape
    _check(load().hyena_out_proj(_ptr(y), _ptr(W), _ptr(bias), _ptr(out), B, L, D, _stream(stream)))


class ImplicitFilter(ctypes.Structure):
    """hyena_implicit_filter_t (device pointers)."""
    _fields_ = [("emb_dim", ctypes.c_int), ("width", ctypes.c_int), ("num_inner", ctypes.c_int),
                ("W_in", ctypes.c_void_p), ("b_in", ctypes.c_void_p), ("W_inner", ctypes.c_void_p),
                ("b_inner", ctypes.c_void_p), ("W_out", ctypes.c_void_p), ("w", ctypes.c_void_p),
                ("alpha", ctypes.c_void_p)]


def hyena_implicit_filter_workspace_bytes(L: int, width: int) -> int:
    return int(load().hyena_implicit_filter_workspace_bytes(L, width))


def hyena_filter_spectrum_implicit(params: dict, D, C: int, L: int, order: int, spectrum, workspace, k_out=None,
                                   stream=None) -> None:
    """params: emb_dim, width, num_inner (ints) and CUDA float32 tensors W_in,
    b_in, W_inner, b_inner (or None), W_out, w, alpha (hyena_implicit_filter_t)."""
    f = ImplicitFilter(int(params["emb_dim"]), int(params["width"]), int(params["num_inner"]),
                       _ptr(params["W_in"]), _ptr(params["b_in"]), _ptr(params.get("W_inner")),
                       _ptr(params.get("b_inner")), _ptr(params["W_out"]), _ptr(params["w"]), _ptr(params["alpha"]))
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(load().hyena_filter_spectrum_implicit(ctypes.byref(f), _ptr(D), C, L, int(order), _ptr(spectrum),
                                                 spectrum.numel() * spectrum.element_size(), _ptr(workspace),
                                                 ws_bytes, _ptr(k_out), _stream(stream)))


def hyena_kernel_status(stream=None) -> None:
    """Raises HyenaError (HYENA_ERR_TIMEOUT or HYENA_ERR_SPECTRUM_MISMATCH)
    when a convolution kernel on the current device recorded one since the
    last call; synchronises the stream and clears the record."""
    _check(load().hyena_kernel_status(_stream(stream)))


def hyena_gated_fftconv_per_sample(u, y, spectrum, sc_w, sc_bias, B: int, C: int, sizes, order: int,
                                   workspace=None, stream=None) -> None:
    """hyena_gated_fftconv with one filter per (b, c) row: spectrum from
    hyena_filter_spectrum over B*C channels (k [order-1, B, C, *sizes])."""
    arr, nd = _sizes(sizes)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().hyena_gated_fftconv_per_sample(_ptr(u), _ptr(y), _ptr(spectrum),
                                                 spectrum.numel() * spectrum.element_size(), _ptr(sc_w),
                                                 _ptr(sc_bias), B, C, nd, arr, order, _dtype_code(u),
                                                 _ptr(workspace), ws_bytes, _stream(stream)))


def hyena_gated_fftconv_host(u_host, y_host, u_dev, y_dev, spectrum, sc_w, sc_bias, B: int, C: int, sizes,
                             order: int, workspace=None, chunk_rows: int = 0, stream=None) -> None:
    """u_host / y_host: CPU tensors (pinned for overlap); u_dev / y_dev: CUDA
    tensors of the same shapes; the copies are pipelined against the kernels."""
    if u_host.is_cuda or y_host.is_cuda:
        raise ValueError("u_host and y_host must be host (CPU) tensors")
    if not (u_host.is_contiguous() and y_host.is_contiguous()):
        raise ValueError("u_host and y_host must be contiguous")
    arr, nd = _sizes(sizes)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().hyena_gated_fftconv_host(u_host.data_ptr(), y_host.data_ptr(), _ptr(u_dev), _ptr(y_dev),
                                           _ptr(spectrum), spectrum.numel() * spectrum.element_size(), _ptr(sc_w),
                                           _ptr(sc_bias), B, C, nd, arr, order, _dtype_code(u_dev),
                                           _ptr(workspace), ws_bytes, int(chunk_rows), _stream(stream)))


def hyena_gated_fftconv_noalloc(u, y, spectrum, sc_w, sc_bias, B: int, C: int, sizes, order: int,
                                stream=None) -> None:
    """hyena_gated_fftconv without a workspace argument: the library's fixed
    scratch array is used instead (for callers that cannot allocate)."""
    arr, nd = _sizes(sizes)
    _check(load().hyena_gated_fftconv_noalloc(_ptr(u), _ptr(y), _ptr(spectrum),
                                              spectrum.numel() * spectrum.element_size(), _ptr(sc_w),
                                              _ptr(sc_bias), B, C, nd, arr, order, _dtype_code(u),
                                              _stream(stream)))


def hyena_spectrum_check(spectrum, C: int, sizes, order: int, stream=None) -> None:
    arr, nd = _sizes(sizes)
    _check(load().hyena_spectrum_check(_ptr(spectrum), C, nd, arr, order, _stream(stream)))


def hyena_debug_conv_tc(u, y, spectrum, sc_w, sc_bias, B: int, C: int, order: int, wait_budget_ns: int,
                        issue_mma: bool = True, stream=None) -> None:
    """Test hook of the L = 8192 bf16 tensor-core kernel: its bounded waits give
    up after wait_budget_ns; issue_mma=False issues no tensor-core work, so the
    first wait runs out (read back with hyena_kernel_status)."""
    _check(load().hyena_debug_conv_tc(_ptr(u), _ptr(y), _ptr(spectrum), spectrum.numel() * spectrum.element_size(),
                                      _ptr(sc_w), _ptr(sc_bias), B, C, order, int(wait_budget_ns),
                                      1 if issue_mma else 0, _stream(stream)))


def hyena_debug_conv_2d_tc(u, y, spectrum, B: int, C: int, W: int, order: int, workspace, wait_budget_ns: int,
                           issue_mma: bool = True, stream=None) -> None:
    """The same test hook for the 2-D tensor-core column pass (H = 256, bf16)."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().hyena_debug_conv_2d_tc(_ptr(u), _ptr(y), _ptr(spectrum), spectrum.numel() * spectrum.element_size(),
                                         B, C, W, order, _ptr(workspace), ws_bytes, int(wait_budget_ns),
                                         1 if issue_mma else 0, _stream(stream)))


def hyena_debug_conv_2dc_tc(u, y, spectrum, B: int, C: int, order: int, workspace, wait_budget_ns: int,
                            issue_mma: bool = True, stream=None) -> None:
    """The same test hook for the circular form's paired tensor-core passes
    (256 x 256, bf16, even B)."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().hyena_debug_conv_2dc_tc(_ptr(u), _ptr(y), _ptr(spectrum), spectrum.numel() * spectrum.element_size(),
                                          B, C, order, _ptr(workspace), ws_bytes, int(wait_budget_ns),
                                          1 if issue_mma else 0, _stream(stream)))


def hyena_debug_conv_cluster(u, y, spectrum, sc_w, sc_bias, B: int, C: int, order: int, workspace,
                             wait_budget_ns: int, issue_mma: bool = True, stream=None) -> None:
    """The same test hook for the L = 65536 bf16 cluster kernel."""
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(load().hyena_debug_conv_cluster(_ptr(u), _ptr(y), _ptr(spectrum),
                                           spectrum.numel() * spectrum.element_size(), _ptr(sc_w), _ptr(sc_bias), B,
                                           C, order, _ptr(workspace), ws_bytes, int(wait_budget_ns),
                                           1 if issue_mma else 0, _stream(stream)))
