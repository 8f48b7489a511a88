"""GPU parity: the cluster path for L = 65536 with bf16 storage (cluster.cu:
the zero-padded 131072-point transform of a row pair split over a cluster of
8 CTAs, tensor-core stages per CTA), against the float64 oracle through the C
ABI, and against the multi-pass fp32 transform the same shapes take with
HYENA_FLAG_FP32_TRANSFORM."""
import numpy as np
import pytest

from fft_long_convolution_02_b200 import binding as hb
from fft_long_convolution_02_b200 import inputs as I
from gpu_helpers import TOL, Run, from_torch, gpu_rows, oracle_for_rows, row_rel_err

pytestmark = pytest.mark.gpu

L = 1 << 16


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fft_long_convolution_02_b200 import build
    build.build()


def _run(p, data, use_shortconv=True, workspace_bytes=None, flags=0):
    import torch
    r = Run(p, data, use_shortconv, workspace_bytes)
    r.build_spectrum()
    hb.hyena_gated_fftconv_ex(r.u, r.y, r.spectrum, r.sc_w, r.sc_b, p.B, p.C, p.shape, p.order, r.workspace,
                              flags=flags)
    torch.cuda.synchronize()
    hb.hyena_kernel_status()
    return r


@pytest.mark.parametrize("order,B,C", [(3, 2, 6), (2, 2, 5), (3, 3, 3), (2, 1, 4)])
def test_cluster_all_rows(orc, order, B, C):
    """Every row vs the oracle; odd B leaves a pair with one row."""
    p = I.WORKLOADS["order3"].with_(B=B, C=C, L=L, order=order, sc_bias=True, seed=9000 + 10 * order + B)
    data = I.make_all(p)
    r = _run(p, data)
    y = from_torch(r.y)
    assert np.isfinite(y).all()
    rows = np.arange(p.B * p.C)
    ref = oracle_for_rows(orc, p, rows, data, method=2)
    err = row_rel_err(gpu_rows(y, p, rows), ref)
    print(f"order {order} B {B}: max row rel err {err.max():.3e}")
    assert err.max() <= TOL["bf16"], err.max()


def test_cluster_matches_fp32_transform(orc):
    """The fp32 multi-pass transform (flag) and the cluster path agree within
    the bf16 tolerance, and the fp32 one is the closer to the oracle."""
    p = I.WORKLOADS["order3"].with_(B=2, C=4, L=L, seed=9100)
    data = I.make_all(p)
    y_cl = from_torch(_run(p, data).y)
    y_32 = from_torch(_run(p, data, flags=hb.HYENA_FLAG_FP32_TRANSFORM).y)
    rows = np.arange(p.B * p.C)
    ref = oracle_for_rows(orc, p, rows, data, method=2)
    e_cl = row_rel_err(gpu_rows(y_cl, p, rows), ref).max()
    e_32 = row_rel_err(gpu_rows(y_32, p, rows), ref).max()
    assert e_cl <= TOL["bf16"] and e_32 <= TOL["bf16"], (e_cl, e_32)
    assert e_32 < e_cl
    assert row_rel_err(gpu_rows(y_cl, p, rows), gpu_rows(y_32, p, rows)).max() <= TOL["bf16"]


def test_cluster_one_cluster_workspace_is_bitwise_equal():
    """With the minimum workspace only one cluster runs (all pairs in turn);
    each pair's arithmetic does not depend on which cluster takes it."""
    import torch
    p = I.WORKLOADS["order3"].with_(B=4, C=3, L=L, seed=9200)
    data = I.make_all(p)
    y_all = _run(p, data).y.clone()
    y_one = _run(p, data, workspace_bytes=hb.hyena_gated_fftconv_workspace_min_bytes(p.C, p.shape, p.order)).y
    assert torch.equal(y_all, y_one)


def test_cluster_no_shortconv(orc):
    p = I.WORKLOADS["order3"].with_(B=2, C=3, L=L, order=2, seed=9300)
    data = I.make_all(p)
    r = _run(p, data, use_shortconv=False)
    rows = np.arange(p.B * p.C)
    ref = oracle_for_rows(orc, p, rows, data, use_shortconv=False, method=2)
    assert row_rel_err(gpu_rows(from_torch(r.y), p, rows), ref).max() <= TOL["bf16"]


def test_cluster_reports_a_spectrum_header_mismatch():
    """A spectrum that was never filled: no output written, the status word
    reports HYENA_ERR_SPECTRUM_MISMATCH, and the next call is clean."""
    import torch
    p = I.WORKLOADS["order3"].with_(B=2, C=2, L=L, seed=9400)
    r = Run(p, I.make_all(p))
    hb.hyena_kernel_status()
    fresh = torch.zeros_like(r.spectrum)
    y = torch.full_like(r.y, 3.0)
    hb.hyena_gated_fftconv(r.u, y, fresh, r.sc_w, None, p.B, p.C, p.shape, p.order, r.workspace)
    with pytest.raises(hb.HyenaError) as e:
        hb.hyena_kernel_status()
    assert e.value.status == 4
    assert bool((y == 3.0).all())
    r.build_spectrum()
    hb.hyena_gated_fftconv(r.u, y, r.spectrum, r.sc_w, None, p.B, p.C, p.shape, p.order, r.workspace)
    hb.hyena_kernel_status()
    assert torch.isfinite(y.float()).all()


def test_order4_at_65536_takes_the_multipass_path(orc):
    """Above order 3 the bf16-operand error would accumulate past the
    tolerance, so L = 65536 with order 4 runs the fp32 multi-pass kernels:
    within the bf16 storage tolerance and closer to the oracle than the
    cluster path's order-3 error."""
    p = I.WORKLOADS["order3"].with_(B=2, C=2, L=L, order=4, seed=9500)
    data = I.make_all(p)
    r = _run(p, data)
    rows = np.arange(p.B * p.C)
    ref = oracle_for_rows(orc, p, rows, data, method=2)
    err = row_rel_err(gpu_rows(from_torch(r.y), p, rows), ref).max()
    assert err <= 5e-3, err
