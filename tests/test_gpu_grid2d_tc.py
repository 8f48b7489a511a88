"""GPU parity: the tensor-core column pass of the 2-D form (grid2d_tc.cu: bf16
storage, H = 256, columns 0 .. W-1 as 512-point transforms on tcgen05, the
last bin column on the register engine), against the float64 oracle through
the C ABI, and against the fp32 register-engine column pass the same shapes
take with HYENA_FLAG_FP32_TRANSFORM."""
import numpy as np
import pytest

from fft_long_convolution_02_b200 import binding as hb
from fft_long_convolution_02_b200 import inputs as I
from gpu_helpers import TOL, Run, api_shape, from_torch, oracle_for_rows, row_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fft_long_convolution_02_b200 import build
    build.build()


def _conv(p, r, flags=0, y=None):
    import torch
    hb.hyena_gated_fftconv_ex(r.u, r.y if y is None else y, r.spectrum, r.sc_w, r.sc_b, p.B, p.C, api_shape(p),
                              p.order, r.workspace, flags=flags)
    torch.cuda.synchronize()
    hb.hyena_kernel_status()
    return from_torch(r.y if y is None else y)


def _rows_err(orc, p, data, y):
    rows = np.arange(p.B * p.C)
    ref = oracle_for_rows(orc, p, rows, data, method=2).reshape(len(rows), -1)
    return row_rel_err(y.reshape(len(rows), -1), ref)


@pytest.mark.parametrize("W,order,B,C", [(256, 2, 2, 3), (32, 2, 3, 2), (64, 3, 2, 2), (512, 2, 1, 2)])
def test_tc_columns_against_oracle(orc, W, order, B, C):
    """Widths of 1, 2, 8 and 16 column groups, orders 2 and 3, odd batch."""
    p = I.WORKLOADS["grid2d"].with_(B=B, C=C, H=256, W=W, order=order, sigma=(4.0, 64.0), seed=3000 + W + order)
    data = I.make_all(p)
    r = Run(p, data)
    r.build_spectrum()
    y = _conv(p, r)
    assert np.isfinite(y).all()
    err = _rows_err(orc, p, data, y)
    print(f"W={W} order={order}: max image rel err {err.max():.3e}")
    assert err.max() <= TOL["bf16"], err.max()


def test_tc_columns_against_fp32_columns(orc):
    """The fp32 register column pass (flag) and the tensor-core one agree within
    the bf16 tolerance, the fp32 one is the closer to the oracle, and they are
    not the same kernel's output."""
    p = I.WORKLOADS["grid2d"].with_(B=2, C=4, H=256, W=128, seed=3100)
    data = I.make_all(p)
    r = Run(p, data)
    r.build_spectrum()
    y_tc = _conv(p, r).copy()
    y_32 = _conv(p, r, flags=hb.HYENA_FLAG_FP32_TRANSFORM)
    e_tc = _rows_err(orc, p, data, y_tc).max()
    e_32 = _rows_err(orc, p, data, y_32).max()
    print(f"tensor-core columns {e_tc:.3e}, fp32 columns {e_32:.3e}")
    assert e_tc <= TOL["bf16"] and e_32 <= TOL["bf16"]
    assert e_32 < e_tc
    assert not np.array_equal(y_tc, y_32)


def test_tc_columns_deterministic():
    import torch
    p = I.WORKLOADS["grid2d"].with_(B=2, C=2, H=256, W=64, seed=3200)
    r = Run(p, I.make_all(p))
    r.build_spectrum()
    _conv(p, r)
    a = r.y.clone()
    _conv(p, r)
    assert torch.equal(a, r.y)


def test_tc_columns_per_sample(orc):
    """Per-sample filters: the plane rows follow the spectrum rows (b, c)."""
    import torch
    p = I.WORKLOADS["grid2d"].with_(B=2, C=2, H=256, W=64, per_sample=True, seed=3300)
    data = I.make_all(p)
    r = Run(p, data)
    spec = torch.empty(hb.hyena_spectrum_bytes(p.B * p.C, api_shape(p), p.order), dtype=torch.uint8, device="cuda")
    hb.hyena_filter_spectrum(r.k, r.D, p.B * p.C, api_shape(p), p.order, spec)
    hb.hyena_gated_fftconv_per_sample(r.u, r.y, spec, None, None, p.B, p.C, api_shape(p), p.order, r.workspace)
    torch.cuda.synchronize()
    hb.hyena_kernel_status()
    err = _rows_err(orc, p, data, from_torch(r.y))
    assert err.max() <= TOL["bf16"], err.max()


def test_tc_columns_report_a_spectrum_header_mismatch():
    """A spectrum that was never filled: the tensor-core column kernel writes
    nothing and the status word reports HYENA_ERR_SPECTRUM_MISMATCH."""
    import torch
    p = I.WORKLOADS["grid2d"].with_(B=2, C=2, H=256, W=64, seed=3400)
    r = Run(p, I.make_all(p))
    hb.hyena_kernel_status()
    fresh = torch.zeros_like(r.spectrum)
    hb.hyena_gated_fftconv(r.u, r.y, fresh, None, None, p.B, p.C, api_shape(p), p.order, r.workspace)
    with pytest.raises(hb.HyenaError) as e:
        hb.hyena_kernel_status()
    assert e.value.status == 4
    r.build_spectrum()
    _conv(p, r)
    assert np.isfinite(from_torch(r.y)).all()


@pytest.mark.parametrize("B,C,order", [(2, 3, 2), (4, 2, 2), (3, 2, 2), (2, 2, 3), (2, 1, 4)])
def test_paired_images_against_oracle(orc, B, C, order):
    """256 x 256 images: with an even batch the two images of a channel travel
    as one complex image through tensor-core row, column and row passes, once
    per order step (orders 2 and 3); an odd batch takes the unpaired passes,
    order 4 the fp32 passes."""
    p = I.WORKLOADS["grid2d"].with_(B=B, C=C, H=256, W=256, order=order, seed=3500 + 10 * B + order)
    data = I.make_all(p)
    r = Run(p, data)
    r.build_spectrum()
    y = _conv(p, r)
    assert np.isfinite(y).all()
    err = _rows_err(orc, p, data, y)
    print(f"B={B} order={order}: max image rel err {err.max():.3e}")
    assert err.max() <= TOL["bf16"], err.max()


def test_paired_images_small_workspace(orc):
    """Workspaces of one and of three images: pairs are never split (one image
    of scratch falls back to the unpaired passes), results within the bound."""
    p = I.WORKLOADS["grid2d"].with_(B=2, C=3, H=256, W=256, seed=3600)
    data = I.make_all(p)
    row = hb.hyena_gated_fftconv_workspace_min_bytes(p.C, api_shape(p), p.order)
    for nrows in (1, 3):
        r = Run(p, data, workspace_bytes=nrows * row)
        r.build_spectrum()
        err = _rows_err(orc, p, data, _conv(p, r))
        assert err.max() <= TOL["bf16"], (nrows, err.max())


def test_paired_images_timeout_is_reported():
    import torch
    p = I.WORKLOADS["grid2d"].with_(B=2, C=2, H=256, W=256, seed=3700)
    r = Run(p, I.make_all(p))
    r.build_spectrum()
    hb.hyena_kernel_status()
    y = torch.zeros_like(r.y)
    hb.hyena_debug_conv_2d_tc(r.u, y, r.spectrum, p.B, p.C, p.W, p.order, r.workspace, wait_budget_ns=1_000_000,
                              issue_mma=False)
    torch.cuda.synchronize()
    with pytest.raises(hb.HyenaError) as ei:
        hb.hyena_kernel_status()
    assert ei.value.status == 8
    assert torch.isnan(y.float()).all()
    _conv(p, r)
    assert np.isfinite(from_torch(r.y)).all()


def _circ(**kw):
    return I.WORKLOADS["grid2d_circ"].with_(H=256, W=256, **kw)


@pytest.mark.parametrize("B,C,order", [(2, 3, 2), (4, 2, 2), (2, 2, 3), (3, 2, 2), (2, 1, 4)])
def test_circular_pairs_against_oracle(orc, B, C, order):
    """Circular 256 x 256 images: an even batch pairs the two images of a channel
    through tensor-core row, column and row passes (256-point transforms, two
    16-point stages each), once per order step; an odd batch takes the
    unpaired passes, order 4 the fp32 passes."""
    p = _circ(B=B, C=C, order=order, seed=3800 + 10 * B + order)
    data = I.make_all(p)
    r = Run(p, data, False)
    r.build_spectrum()
    y = _conv(p, r)
    assert np.isfinite(y).all()
    err = _rows_err(orc, p, data, y)
    print(f"circular B={B} order={order}: max image rel err {err.max():.3e}")
    assert err.max() <= TOL["bf16"], err.max()


def test_circular_pairs_against_fp32_passes(orc):
    """The fp32 passes (flag) and the paired tensor-core passes agree within the
    bf16 tolerance, the fp32 ones are the closer to the oracle, and the outputs
    differ (two different kernel sets ran)."""
    p = _circ(B=2, C=3, seed=3900)
    data = I.make_all(p)
    r = Run(p, data, False)
    r.build_spectrum()
    y_tc = _conv(p, r).copy()
    y_32 = _conv(p, r, flags=hb.HYENA_FLAG_FP32_TRANSFORM)
    e_tc = _rows_err(orc, p, data, y_tc).max()
    e_32 = _rows_err(orc, p, data, y_32).max()
    print(f"circular: tensor-core pairs {e_tc:.3e}, fp32 passes {e_32:.3e}")
    assert e_tc <= TOL["bf16"] and e_32 <= TOL["bf16"]
    assert e_32 < e_tc
    assert not np.array_equal(y_tc, y_32)


def test_circular_pairs_deterministic_and_small_workspace(orc):
    """Bitwise repeatable; workspaces of one image (unpaired passes) and of
    three images (one pair per group) stay within the bound."""
    import torch
    p = _circ(B=2, C=3, seed=4000)
    data = I.make_all(p)
    r = Run(p, data, False)
    r.build_spectrum()
    _conv(p, r)
    a = r.y.clone()
    _conv(p, r)
    assert torch.equal(a, r.y)
    row = hb.hyena_gated_fftconv_workspace_min_bytes(p.C, api_shape(p), p.order)
    for nrows in (1, 3):
        rs = Run(p, data, False, workspace_bytes=nrows * row)
        rs.build_spectrum()
        err = _rows_err(orc, p, data, _conv(p, rs))
        assert err.max() <= TOL["bf16"], (nrows, err.max())


def test_circular_pairs_report_a_spectrum_header_mismatch():
    import torch
    p = _circ(B=2, C=2, seed=4100)
    r = Run(p, I.make_all(p), False)
    hb.hyena_kernel_status()
    fresh = torch.zeros_like(r.spectrum)
    hb.hyena_gated_fftconv(r.u, r.y, fresh, None, None, p.B, p.C, api_shape(p), p.order, r.workspace)
    with pytest.raises(hb.HyenaError) as e:
        hb.hyena_kernel_status()
    assert e.value.status == 4
    r.build_spectrum()
    _conv(p, r)
    assert np.isfinite(from_torch(r.y)).all()


def test_circular_pairs_timeout_is_reported():
    """The circular paired passes' bounded waits: no tensor-core work issued,
    1 ms budget: HYENA_ERR_TIMEOUT, NaN outputs, the next call correct."""
    import torch
    p = _circ(B=2, C=2, seed=4200)
    r = Run(p, I.make_all(p), False)
    r.build_spectrum()
    hb.hyena_kernel_status()
    y = torch.zeros_like(r.y)
    hb.hyena_debug_conv_2dc_tc(r.u, y, r.spectrum, p.B, p.C, p.order, r.workspace, wait_budget_ns=1_000_000,
                               issue_mma=False)
    torch.cuda.synchronize()
    with pytest.raises(hb.HyenaError) as ei:
        hb.hyena_kernel_status()
    assert ei.value.status == 8
    assert torch.isnan(y.float()).all()
    _conv(p, r)
    assert np.isfinite(from_torch(r.y)).all()
