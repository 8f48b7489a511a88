"""GPU: the bounded waits of the L = 8192 tensor-core kernel.  The test hook
issues no tensor-core work, so the kernel's first wait runs out on a barrier
that nothing completes (1 ms budget, one CTA); the timeout must be reported
through the device's kernel status word (hyena_kernel_status), the outputs
of the pair must be NaN, the spectrum must be left as it was, and the context
must stay usable.  Nothing faults, traps or hangs."""
import numpy as np
import pytest

from fft_long_convolution_02_b200 import binding as hb
from fft_long_convolution_02_b200 import inputs as I
from gpu_helpers import TOL, Run, from_torch, gpu_rows, oracle_for_rows, row_rel_err

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fft_long_convolution_02_b200 import build
    build.build()


def test_tensor_core_wait_timeout_is_reported(orc):
    import torch
    p = I.WORKLOADS["d768_l8k"].with_(B=2, C=1, seed=5101)     # one row pair: a 1-CTA launch
    data = I.make_all(p)
    r = Run(p, data)
    r.build_spectrum()
    hb.hyena_spectrum_check(r.spectrum, p.C, p.shape, p.order)
    hb.hyena_kernel_status()                                      # start from a clear record
    spec_before = r.spectrum.clone()
    y = torch.zeros_like(r.y)
    hb.hyena_debug_conv_tc(r.u, y, r.spectrum, r.sc_w, None, p.B, p.C, p.order, wait_budget_ns=1_000_000,
                           issue_mma=False)
    torch.cuda.synchronize()
    with pytest.raises(hb.HyenaError) as ei:
        hb.hyena_kernel_status()
    assert ei.value.status == 8                                   # HYENA_ERR_TIMEOUT
    hb.hyena_kernel_status()                                      # reading cleared it
    assert torch.isnan(y.float()).all()
    assert torch.equal(r.spectrum, spec_before)                   # the spectrum is only read
    # the context is still usable: run normally
    hb.hyena_spectrum_check(r.spectrum, p.C, p.shape, p.order)
    r.conv()
    torch.cuda.synchronize()
    got = from_torch(r.y)
    rows = np.arange(p.B * p.C)
    err = row_rel_err(gpu_rows(got, p, rows), oracle_for_rows(orc, p, rows, data))
    assert err.max() <= TOL["bf16"], err.max()
    # the hook with the tensor-core work issued and the default budget gives the same result
    y2 = torch.zeros_like(r.y)
    hb.hyena_debug_conv_tc(r.u, y2, r.spectrum, r.sc_w, None, p.B, p.C, p.order, wait_budget_ns=2_000_000_000,
                           issue_mma=True)
    torch.cuda.synchronize()
    assert torch.equal(y2, r.y)
    hb.hyena_kernel_status()


def test_cluster_wait_timeout_is_reported(orc):
    """The cluster kernel (L = 65536, bf16): one pair, one cluster of 8 CTAs.
    With no tensor-core work issued every CTA's first wait runs out; each
    still takes every cluster barrier, so the launch completes, the timeout
    is recorded, the outputs are NaN, and the next normal call is correct."""
    import torch
    p = I.WORKLOADS["order3"].with_(B=2, C=1, L=1 << 16, seed=5102)
    data = I.make_all(p)
    r = Run(p, data)
    r.build_spectrum()
    hb.hyena_kernel_status()
    spec_before = r.spectrum.clone()
    y = torch.zeros_like(r.y)
    hb.hyena_debug_conv_cluster(r.u, y, r.spectrum, r.sc_w, None, p.B, p.C, p.order, r.workspace,
                                wait_budget_ns=1_000_000, issue_mma=False)
    torch.cuda.synchronize()
    with pytest.raises(hb.HyenaError) as ei:
        hb.hyena_kernel_status()
    assert ei.value.status == 8                                   # HYENA_ERR_TIMEOUT
    assert torch.isnan(y.float()).all()
    assert torch.equal(r.spectrum, spec_before)
    r.conv()
    torch.cuda.synchronize()
    hb.hyena_kernel_status()
    rows = np.arange(p.B * p.C)
    err = row_rel_err(gpu_rows(from_torch(r.y), p, rows), oracle_for_rows(orc, p, rows, data, method=2))
    assert err.max() <= TOL["bf16"], err.max()


def test_2d_tc_column_wait_timeout_is_reported(orc):
    """The 2-D tensor-core column pass (H = 256, bf16): with no tensor-core work
    issued each CTA's first wait runs out; the launch completes, the timeout
    is recorded, the NaN columns reach every output through the inverse row
    pass, and the next normal call is correct."""
    import torch
    p = I.WORKLOADS["grid2d"].with_(B=2, C=2, H=256, W=64, seed=5103)
    data = I.make_all(p)
    r = Run(p, data)
    r.build_spectrum()
    hb.hyena_kernel_status()
    spec_before = r.spectrum.clone()
    y = torch.zeros_like(r.y)
    hb.hyena_debug_conv_2d_tc(r.u, y, r.spectrum, p.B, p.C, p.W, p.order, r.workspace, wait_budget_ns=1_000_000,
                              issue_mma=False)
    torch.cuda.synchronize()
    with pytest.raises(hb.HyenaError) as ei:
        hb.hyena_kernel_status()
    assert ei.value.status == 8                                   # HYENA_ERR_TIMEOUT
    assert torch.isnan(y.float()).all()
    assert torch.equal(r.spectrum, spec_before)
    r.conv()
    torch.cuda.synchronize()
    hb.hyena_kernel_status()
    rows = np.arange(p.B * p.C)
    ref = oracle_for_rows(orc, p, rows, data, use_shortconv=False, method=2).reshape(len(rows), -1)
    err = row_rel_err(from_torch(r.y).reshape(len(rows), -1), ref)
    assert err.max() <= TOL["bf16"], err.max()
