"""GPU parity of the 3-D non-circular form (ndim = 3, N1 x H x W volumes)
against the float64 oracle through the C ABI: axis lengths 16-128, fp32 and
bf16, orders, small workspaces, per-sample filters, the full vol3d workload
(sampled volumes) and the delta invariant."""
import numpy as np
import pytest

from fft_long_convolution_02_b200 import binding as hb
from fft_long_convolution_02_b200 import inputs as I
from gpu_helpers import TOL, Run, from_torch, gpu_rows, oracle_for_rows, row_rel_err, to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fft_long_convolution_02_b200 import build
    build.build()


def _check(orc, p, rows=None, workspace_bytes=None):
    data = I.make_all(p)
    y = Run(p, data, False, workspace_bytes).run()
    if rows is None:
        rows = np.arange(p.B * p.C)
    ref = oracle_for_rows(orc, p, rows, data, use_shortconv=False, method=2)
    err = row_rel_err(gpu_rows(y, p, rows), ref)
    assert err.max() <= TOL[p.dtype], f"{p.name} {p.shape}: max row rel err {err.max():.3e}"
    assert np.isfinite(y).all()
    return err.max()


@pytest.mark.parametrize("N1,H,W", [(16, 16, 16), (16, 32, 64), (32, 16, 16), (16, 16, 128), (128, 16, 16),
                                    (16, 128, 16)])
def test_3d_shapes_f32(orc, N1, H, W):
    p = I.WORKLOADS["vol3d"].with_(B=2, C=2, N1=N1, H=H, W=W, dtype="f32", sigma=(2.0, 12.0),
                                   seed=1600 + N1 + 2 * H + 3 * W)
    assert _check(orc, p) < 1e-5


@pytest.mark.parametrize("order", [2, 3])
def test_3d_orders_bf16(orc, order):
    p = I.WORKLOADS["vol3d"].with_(B=3, C=2, N1=16, H=32, W=32, order=order, seed=1700 + order)
    _check(orc, p)


def test_3d_small_workspaces(orc):
    p = I.WORKLOADS["vol3d"].with_(B=2, C=3, N1=16, H=16, W=32, dtype="f32", seed=1800)
    one = hb.hyena_gated_fftconv_workspace_min_bytes(p.C, p.shape, p.order)
    _check(orc, p, workspace_bytes=one)
    _check(orc, p, workspace_bytes=3 * one + 8)
    _check(orc, p.with_(dtype="bf16", seed=1801), workspace_bytes=one)


def test_3d_per_sample_filters(orc):
    import torch
    p = I.WORKLOADS["vol3d"].with_(B=2, C=2, N1=16, H=16, W=16, per_sample=True, seed=1850)
    data = I.make_all(p)
    u = to_torch(p, data["u"]); k = to_torch(p, data["k"])
    D = torch.from_numpy(data["D"]).cuda()
    spec = torch.empty(hb.hyena_spectrum_bytes(p.B * p.C, p.shape, p.order), dtype=torch.uint8, device="cuda")
    hb.hyena_filter_spectrum(k, D, p.B * p.C, p.shape, p.order, spec)
    y = torch.empty((p.B, p.C) + p.shape, dtype=u.dtype, device="cuda")
    ws = torch.empty(hb.hyena_gated_fftconv_workspace_bytes(p.B, p.C, p.shape, p.order), dtype=torch.uint8,
                     device="cuda")
    hb.hyena_gated_fftconv_per_sample(u, y, spec, None, None, p.B, p.C, p.shape, p.order, ws)
    torch.cuda.synchronize()
    rows = np.arange(p.B * p.C)
    ref = oracle_for_rows(orc, p, rows, data, use_shortconv=False, method=2)
    err = row_rel_err(from_torch(y).reshape(p.B * p.C, -1), ref.reshape(p.B * p.C, -1))
    assert err.max() <= TOL["bf16"]


def test_3d_workload_full_size_all_volumes(orc):
    """B=2 C=32 64x64x64 order 2 bf16 at full size; all 64 volumes vs the oracle."""
    p = I.WORKLOADS["vol3d"]
    _check(orc, p, rows=np.arange(p.B * p.C))


def test_3d_delta_gives_kernel_plus_D():
    """x0 = x1 = 1, v = delta at the origin: y = K + D delta (anchored crop)."""
    p = I.WORKLOADS["vol3d"].with_(B=1, C=2, N1=16, H=16, W=32, dtype="f32", seed=1900)
    data = I.make_all(p)
    u = np.ones_like(data["u"])
    u[:, 2 * p.C:] = 0.0
    u[:, 2 * p.C:, 0, 0, 0] = 1.0
    data["u"] = u
    y = Run(p, data, False).run()
    want = data["k"][0].astype(np.float64).copy()
    want[:, 0, 0, 0] += data["D"][0]
    assert np.abs(y[0] - want).max() <= 1e-5 * np.abs(want).max()
