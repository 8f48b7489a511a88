"""GPU parity of the circular (periodic) 2-D form, ndim = 2 | HYENA_CIRCULAR,
against the float64 oracle through the C ABI: every row and column length,
orders, bf16, small workspaces, per-sample filters, the full grid2d_circ
workload (sampled images), the delta invariant and the no-wrap equality with
the zero-padded form."""
import numpy as np
import pytest

from fft_long_convolution_02_b200 import binding as hb
from fft_long_convolution_02_b200 import inputs as I
from gpu_helpers import TOL, Run, api_shape, from_torch, gpu_rows, oracle_for_rows, row_rel_err, to_torch

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


@pytest.mark.parametrize("H,W", [(16, 16), (16, 64), (64, 16), (32, 32), (128, 64), (512, 32), (32, 512),
                                 (256, 256)])
def test_circular_shapes_f32(orc, H, W):
    p = I.WORKLOADS["grid2d_circ"].with_(B=2, C=3, H=H, W=W, dtype="f32", seed=1100 + H + W)
    assert _check(orc, p) < 1e-5


@pytest.mark.parametrize("order", [2, 3, 4])
def test_circular_orders_bf16(orc, order):
    p = I.WORKLOADS["grid2d_circ"].with_(B=3, C=2, H=64, W=128, order=order, seed=1200 + order)
    _check(orc, p)


def test_circular_small_workspaces(orc):
    p = I.WORKLOADS["grid2d_circ"].with_(B=3, C=3, H=32, W=64, dtype="f32", seed=1300)
    one = hb.hyena_gated_fftconv_workspace_min_bytes(p.C, api_shape(p), p.order)
    _check(orc, p, workspace_bytes=one)
    _check(orc, p, workspace_bytes=4 * one + 8)
    pb = p.with_(dtype="bf16", seed=1301)
    _check(orc, pb, workspace_bytes=one)


def test_circular_per_sample_filters(orc):
    import torch
    p = I.WORKLOADS["grid2d_circ"].with_(B=2, C=3, H=32, W=32, per_sample=True, seed=1350)
    data = I.make_all(p)
    u = to_torch(p, data["u"]); k = to_torch(p, data["k"])
    D = torch.from_numpy(data["D"]).cuda()
    shape = api_shape(p)
    spec = torch.empty(hb.hyena_spectrum_bytes(p.B * p.C, shape, p.order), dtype=torch.uint8, device="cuda")
    hb.hyena_filter_spectrum(k, D, p.B * p.C, shape, p.order, spec)
    y = torch.empty((p.B, p.C) + p.shape, dtype=u.dtype, device="cuda")
    ws = torch.empty(hb.hyena_gated_fftconv_workspace_bytes(p.B, p.C, shape, p.order), dtype=torch.uint8,
                     device="cuda")
    hb.hyena_gated_fftconv_per_sample(u, y, spec, None, None, p.B, p.C, shape, p.order, ws)
    torch.cuda.synchronize()
    rows = np.arange(p.B * p.C)
    ref = oracle_for_rows(orc, p, rows, data, use_shortconv=False, method=2)
    err = row_rel_err(from_torch(y).reshape(p.B * p.C, -1), ref.reshape(p.B * p.C, -1))
    assert err.max() <= TOL["bf16"]


def test_circular_workload_full_size_all_images(orc):
    """B=2 C=256 256x256 order 2 bf16, circular, at full size; all 512 images vs the oracle."""
    p = I.WORKLOADS["grid2d_circ"]
    _check(orc, p, rows=np.arange(p.B * p.C))


def test_circular_delta_gives_kernel_plus_D():
    """x0 = x1 = 1, v = delta at (0,0): y = K + D delta on the whole grid."""
    p = I.WORKLOADS["grid2d_circ"].with_(B=1, C=2, H=32, W=64, dtype="f32", seed=1400)
    data = I.make_all(p)
    u = np.ones_like(data["u"])
    u[:, 2 * p.C:] = 0.0
    u[:, 2 * p.C:, 0, 0] = 1.0
    data["u"] = u
    y = Run(p, data, False).run()
    want = data["k"][0].astype(np.float64).copy()
    want[:, 0, 0] += data["D"][0]
    assert np.abs(y[0] - want).max() <= 1e-5 * np.abs(want).max()


def test_circular_without_wrap_equals_padded():
    """Filter and inputs supported in the top-left quarter never wrap: the
    circular and the zero-padded path give the same images."""
    p = I.WORKLOADS["grid2d_circ"].with_(B=2, C=2, H=32, W=64, dtype="f32", seed=1500)
    data = I.make_all(p)
    q = (slice(None), slice(None), slice(p.H // 2, None))
    r = (slice(None), slice(None), slice(None), slice(p.W // 2, None))
    for key in ("u", "k"):
        data[key][q] = 0.0
        data[key][r] = 0.0
    y_circ = Run(p, data, False).run()
    y_pad = Run(p.with_(circular=False), data, False).run()
    err = row_rel_err(y_circ.reshape(p.B * p.C, -1), y_pad.reshape(p.B * p.C, -1))
    assert err.max() < 1e-5
