"""GPU parity: the four-step multi-pass path (1-D, 32768 <= L <= 2^20) and the
2-D path, against the float64 oracle through the C ABI."""
import numpy as np
import pytest

from fft_long_convolution_02_b200 import binding as hb
from fft_long_convolution_02_b200 import inputs as I
from gpu_helpers import TOL, Run, gpu_rows, oracle_for_rows, row_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fft_long_convolution_02_b200 import build
    build.build()


def _check(orc, p, rows=None, use_shortconv=True, workspace_bytes=None, tol=None):
    data = I.make_all(p)
    y = Run(p, data, use_shortconv, workspace_bytes).run()
    if rows is None:
        rows = np.arange(p.B * p.C)
    ref = oracle_for_rows(orc, p, rows, data, use_shortconv, method=2)
    err = row_rel_err(gpu_rows(y, p, rows), ref)
    assert err.max() <= (tol or TOL[p.dtype]), f"{p.name} {p.shape}: max row rel err {err.max():.3e}"
    assert np.isfinite(y).all()
    return err.max()


@pytest.mark.parametrize("L", [1 << 15, 1 << 16, 1 << 17, 1 << 18, 1 << 19, 1 << 20])
def test_multipass_lengths_f32(orc, L):
    p = I.WORKLOADS["tiny"].with_(B=1, C=2, L=L, seed=500 + L.bit_length())
    err = _check(orc, p)
    assert err < 1e-5


@pytest.mark.parametrize("L", [1 << 15, 1 << 16, 1 << 17, 1 << 18, 1 << 19, 1 << 20])
def test_multipass_lengths_bf16(orc, L):
    """bf16 storage keeps the workspace in bf16: every (M1, M2) split of the
    four-step path within the bf16 tolerance."""
    p = I.WORKLOADS["dna_1m"].with_(B=2, C=1, L=L, seed=520 + L.bit_length())
    err = _check(orc, p)
    print(f"L={L} bf16 max row rel err {err:.3e}")


@pytest.mark.parametrize("order", [2, 3, 4])
def test_multipass_orders_bf16(orc, order):
    p = I.WORKLOADS["order3"].with_(B=3, C=3, L=1 << 15, order=order, sc_bias=True, seed=600 + order)
    _check(orc, p)


def test_multipass_small_workspace_groups(orc):
    """A workspace of one and of three rows: the row-group loop must give the same result."""
    p = I.WORKLOADS["order3"].with_(B=2, C=5, L=1 << 15, seed=700)
    row = hb.hyena_gated_fftconv_workspace_min_bytes(p.C, p.shape, p.order)
    _check(orc, p, workspace_bytes=row)
    _check(orc, p, workspace_bytes=3 * row + 100)


def test_multipass_no_shortconv(orc):
    p = I.WORKLOADS["dna_1m"].with_(L=1 << 16, C=4, seed=701)
    _check(orc, p, use_shortconv=False)


def test_order3_workload_full_size_sampled_rows(orc):
    """B=2 C=2048 L=65536 order 3 bf16 at full size; 66 seeded rows (the
    first, the last and 64 drawn) vs the oracle."""
    p = I.WORKLOADS["order3"]
    rows = np.random.default_rng(8).choice(np.arange(1, p.B * p.C - 1), 64, replace=False)
    rows = np.concatenate([[0, p.B * p.C - 1], rows])
    _check(orc, p, rows=rows)


def test_dna_1m_workload_full_size_sampled_rows(orc):
    """B=1 C=256 L=2^20 order 2 bf16 (ACGT embedding) at full size; 66 seeded
    rows (the first, the last and 64 drawn) vs the oracle."""
    p = I.WORKLOADS["dna_1m"]
    rows = np.random.default_rng(12).choice(np.arange(1, p.B * p.C - 1), 64, replace=False)
    rows = np.concatenate([[0, p.B * p.C - 1], rows])
    _check(orc, p, rows=rows)


# ------------------------------------------------------------------- 2-D
@pytest.mark.parametrize("H,W", [(16, 16), (16, 64), (64, 16), (32, 32), (128, 64), (512, 32), (32, 512)])
def test_grid2d_shapes_f32(orc, H, W):
    p = I.WORKLOADS["grid2d"].with_(B=2, C=3, H=H, W=W, dtype="f32", sigma=(2.0, 16.0), seed=800 + H + W)
    err = _check(orc, p)
    assert err < 1e-5


@pytest.mark.parametrize("order", [2, 3])
def test_grid2d_orders_bf16(orc, order):
    p = I.WORKLOADS["grid2d"].with_(B=3, C=2, H=64, W=128, order=order, sigma=(4.0, 32.0), seed=900 + order)
    _check(orc, p)


def test_grid2d_small_workspace(orc):
    p = I.WORKLOADS["grid2d"].with_(B=2, C=3, H=32, W=32, dtype="f32", seed=950)
    one = hb.hyena_gated_fftconv_workspace_min_bytes(p.C, p.shape, p.order)
    _check(orc, p, workspace_bytes=one)


def test_grid2d_workload_full_size_all_images(orc):
    """B=2 C=256 256x256 order 2 bf16 at full size; all 512 images vs the oracle."""
    p = I.WORKLOADS["grid2d"]
    _check(orc, p, rows=np.arange(p.B * p.C))


def test_grid2d_delta_gives_kernel_plus_D():
    """x0 = x1 = 1, v = delta at (0,0): y = K + D delta (anchored crop)."""
    import torch
    p = I.WORKLOADS["grid2d"].with_(B=1, C=2, H=32, W=64, dtype="f32", seed=960)
    data = I.make_all(p)
    u = np.ones_like(data["u"])
    u[:, 2 * p.C:] = 0.0
    u[:, 2 * p.C:, 0, 0] = 1.0
    data["u"] = u
    r = Run(p, data)
    y = r.run()
    K = data["k"][0]
    want = K.astype(np.float64).copy()
    want[:, 0, 0] += data["D"][0]
    assert np.abs(y[0] - want).max() <= 1e-5 * np.abs(want).max()
    del torch
