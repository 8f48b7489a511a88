"""Helpers shared by the GPU parity tests: run the CUDA path through the C
ABI on seeded inputs and compare with the float64 oracle."""
from __future__ import annotations

import numpy as np

from fft_long_convolution_02_b200 import binding as hb
from fft_long_convolution_02_b200 import inputs as I

# Tolerances on the max over rows of ||y_gpu - y_ref||_2 / ||y_ref||_2.
TOL = {"f32": 1e-4, "bf16": 2e-2}


def api_shape(p: I.Problem):
    """The shape argument of the C ABI calls (the circular 2-D form flagged)."""
    return hb.Circular(p.shape) if p.circular else p.shape


def to_torch(p: I.Problem, stored: np.ndarray, device="cuda"):
    import torch
    if p.dtype == "bf16":
        t = torch.from_numpy(np.ascontiguousarray(stored).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(stored, dtype=np.float32))
    return t.to(device)


def from_torch(t) -> np.ndarray:
    import torch
    return t.detach().to(torch.float64).cpu().numpy()


class Run:
    """Device buffers and the C-ABI calls for one problem."""

    def __init__(self, p: I.Problem, data: dict, use_shortconv: bool = True, workspace_bytes=None):
        import torch
        self.p = p
        self.u = to_torch(p, data["u"])
        self.k = to_torch(p, data["k"])
        self.D = torch.from_numpy(data["D"]).cuda()
        self.sc_w = torch.from_numpy(data["sc_w"]).cuda() if (use_shortconv and data["sc_w"] is not None) else None
        self.sc_b = (torch.from_numpy(data["sc_b"]).cuda()
                     if (self.sc_w is not None and data.get("sc_b") is not None) else None)
        self.spectrum = torch.empty(hb.hyena_spectrum_bytes(p.C, api_shape(p), p.order), dtype=torch.uint8,
                                    device="cuda")
        self.y = torch.empty((p.B, p.C) + p.shape, dtype=self.u.dtype, device="cuda")
        if workspace_bytes is None:
            workspace_bytes = hb.hyena_gated_fftconv_workspace_bytes(p.B, p.C, api_shape(p), p.order)
        self.workspace = (torch.empty(workspace_bytes, dtype=torch.uint8, device="cuda")
                          if workspace_bytes else None)

    def build_spectrum(self):
        hb.hyena_filter_spectrum(self.k, self.D, self.p.C, api_shape(self.p), self.p.order, self.spectrum)

    def conv(self, u=None, y=None):
        p = self.p
        hb.hyena_gated_fftconv(self.u if u is None else u, self.y if y is None else y, self.spectrum,
                               self.sc_w, self.sc_b, p.B, p.C, api_shape(p), p.order, self.workspace)

    def run(self) -> np.ndarray:
        import torch
        self.build_spectrum()
        self.conv()
        torch.cuda.synchronize()
        return from_torch(self.y)


def row_rel_err(y_gpu_rows: np.ndarray, y_ref_rows: np.ndarray) -> np.ndarray:
    R = y_ref_rows.shape[0]
    a = y_gpu_rows.reshape(R, -1)
    b = y_ref_rows.reshape(R, -1)
    return np.linalg.norm(a - b, axis=1) / np.maximum(np.linalg.norm(b, axis=1), 1e-300)


def oracle_for_rows(orc, p: I.Problem, rows, data, use_shortconv=True, method=0):
    """The oracle's y for row ids b*C + c of the stacked tensors in ``data``
    (from inputs.make_all): the oracle does the split itself."""
    w = data["sc_w"] if use_shortconv else None
    b = data.get("sc_b") if use_shortconv else None
    return orc.hyena_stacked(data["u"], data["k"], data["D"], w, b, B=p.B, C=p.C, order=p.order, shape=p.shape,
                             rows=rows, per_sample=p.per_sample, circular=p.circular, method=method)


def gpu_rows(y: np.ndarray, p: I.Problem, rows) -> np.ndarray:
    rows = np.asarray(rows)
    return y.reshape(p.B * p.C, -1)[rows].reshape((len(rows),) + p.shape)
