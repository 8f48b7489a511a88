"""GPU parity: the on-chip path (1-D, L <= 16384) against the float64 oracle,
called through the C ABI.  Metric: max over (b, c) rows of
||y_gpu - y_oracle||_2 / ||y_oracle||_2 <= 1e-4 (fp32 storage) or 2e-2 (bf16)."""
import numpy as np
import pytest

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


def _check_all_rows(orc, p, use_shortconv=True, method=0):
    data = I.make_all(p)
    y = Run(p, data, use_shortconv).run()
    rows = np.arange(p.B * p.C)
    ref = oracle_for_rows(orc, p, rows, data, use_shortconv, method)
    err = row_rel_err(gpu_rows(y, p, rows), ref)
    assert err.max() <= TOL[p.dtype], f"{p}: max row rel err {err.max():.3e}"
    return err.max()


@pytest.mark.parametrize("use_shortconv", [True, False])
def test_tiny_workload_all_rows(orc, use_shortconv):
    """B=1 C=64 L=1024 order 2 fp32, every row against the direct-sum oracle."""
    err = _check_all_rows(orc, I.WORKLOADS["tiny"], use_shortconv, method=1)
    assert err < 1e-5


@pytest.mark.parametrize("L", [16, 32, 64, 128, 256, 512, 2048, 4096, 8192, 16384])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_lengths(orc, L, dtype):
    p = I.WORKLOADS["tiny"].with_(B=3, C=5, L=L, dtype=dtype, seed=101 + L)
    _check_all_rows(orc, p)


@pytest.mark.parametrize("order", [2, 3, 4, 8])
def test_orders(orc, order):
    p = I.WORKLOADS["tiny"].with_(B=2, C=7, L=2048, order=order, seed=300 + order, sc_bias=True)
    _check_all_rows(orc, p)


@pytest.mark.parametrize("order,dtype", [(3, "bf16"), (4, "bf16"), (4, "f32"), (8, "bf16")])
def test_orders_at_8192(orc, order, dtype):
    """L = 8192 across several order steps: bf16 order <= 3 on the tensor-core
    kernel, higher orders and fp32 on the fp32 register kernel."""
    p = I.WORKLOADS["d768_l8k"].with_(B=2, C=5, order=order, dtype=dtype, sc_bias=True, seed=310 + order)
    _check_all_rows(orc, p)


def test_tensor_core_single_row_order3_no_shortconv(orc):
    """The bf16 L = 8192 tensor-core kernel with one batch row (every pair has an
    empty imaginary half), two order steps, and no short conv."""
    p = I.WORKLOADS["d768_l8k"].with_(B=1, C=3, order=3, seed=4401)
    _check_all_rows(orc, p, use_shortconv=False)


def test_bf16_order8_single_row_no_shortconv(orc):
    """bf16 L = 8192 at order 8 (seven steps, fp32 register kernel), one row."""
    p = I.WORKLOADS["d768_l8k"].with_(B=1, C=3, order=8, seed=4401)
    _check_all_rows(orc, p, use_shortconv=False)


def test_tensor_core_causality():
    """bf16 L = 8192 (tensor-core kernel): replacing every sample of u after t0 by
    fresh values of the same distribution leaves y[0:t0] unchanged within the bf16
    tolerance; a transform without the zero padding would wrap the change into
    y[0:t0] at full size."""
    import torch
    from gpu_helpers import from_torch
    p = I.WORKLOADS["d768_l8k"].with_(B=2, C=6, seed=4402)
    data = I.make_all(p)
    r = Run(p, data)
    y0 = r.run()
    t0 = 3000
    u2 = r.u.clone()
    g = torch.Generator(device="cuda").manual_seed(7)
    u2[..., t0:] = torch.randn(u2[..., t0:].shape, device="cuda", generator=g).to(u2.dtype)
    y1 = torch.empty_like(r.y)
    r.conv(u=u2, y=y1)
    torch.cuda.synchronize()
    y1 = from_torch(y1)
    a = y0[..., :t0].reshape(p.B * p.C, -1)
    b = y1[..., :t0].reshape(p.B * p.C, -1)
    err = np.linalg.norm(a - b, axis=1) / np.linalg.norm(a, axis=1)
    assert err.max() <= TOL["bf16"], err.max()
    # and the tail did change
    assert not np.allclose(y0[..., t0:], y1[..., t0:])


def test_shortconv_bias_and_odd_batch(orc):
    p = I.WORKLOADS["d768_l8k"].with_(B=3, C=9, sc_bias=True, seed=77)
    _check_all_rows(orc, p)


def test_d768_l8k_full_size_all_rows(orc):
    """The 1-D workload at width 768, L = 8192, bf16, full size as benchmarked;
    every one of the B*C = 3072 rows checked against the oracle."""
    p = I.WORKLOADS["d768_l8k"]
    data = I.make_all(p)
    y = Run(p, data).run()
    rows = np.arange(p.B * p.C)
    ref = oracle_for_rows(orc, p, rows, data, method=2)
    err = row_rel_err(gpu_rows(y, p, rows), ref)
    assert err.max() <= TOL["bf16"], err.max()
    # every output is finite
    assert np.isfinite(y).all()


def test_unfused_composition_matches_fused():
    """hyena_shortconv then hyena_gated_fftconv(sc_w=NULL) equals the fused path."""
    import torch
    from fft_long_convolution_02_b200 import binding as hb
    for dtype in ("f32", "bf16"):
        p = I.WORKLOADS["tiny"].with_(B=2, C=16, L=4096, dtype=dtype, sc_bias=True, seed=9)
        data = I.make_all(p)
        r = Run(p, data)
        y_fused = r.run()
        uc = torch.empty_like(r.u)
        hb.hyena_shortconv(r.u, uc, r.sc_w, r.sc_b)
        r2 = Run(p, data, use_shortconv=False)
        r2.spectrum = r.spectrum
        r2.conv(u=uc)
        torch.cuda.synchronize()
        y2 = r2.y.double().cpu().numpy()
        rel = np.linalg.norm(y2 - y_fused) / np.linalg.norm(y_fused)
        assert rel <= (1e-6 if dtype == "f32" else 1e-2), rel


def test_shortconv_matches_oracle(orc):
    import torch
    from fft_long_convolution_02_b200 import binding as hb
    for dtype in ("f32", "bf16"):
        p = I.WORKLOADS["tiny"].with_(B=2, C=4, L=256, dtype=dtype, sc_bias=True, seed=12)
        data = I.make_all(p)
        r = Run(p, data)
        out = torch.empty_like(r.u)
        hb.hyena_shortconv(r.u, out, r.sc_w, r.sc_b)
        torch.cuda.synchronize()
        got = out.double().cpu().numpy()
        u = I.stored_values(p, data["u"])
        for b in range(p.B):
            for ch in range(p.Ctot):
                w = data["sc_w"][ch].astype(np.float64)
                bias = float(data["sc_b"][ch])
                ref = orc.shortconv(u[b, ch], w, bias)
                # fp32 accumulation error scales with the sum of |terms|;
                # bf16 storage adds half an ulp (2^-9 relative) of the result
                terms = orc.shortconv(np.abs(u[b, ch]), np.abs(w), abs(bias))
                tol = 1e-6 * terms + (2.0 ** -8 * np.abs(ref) if dtype == "bf16" else 0.0)
                assert np.all(np.abs(got[b, ch] - ref) <= tol), (b, ch)


def test_causality_on_gpu():
    """Perturbing u at t > s leaves y[0..s] unchanged to rounding level."""
    import torch
    p = I.WORKLOADS["tiny"].with_(B=1, C=4, L=1024, seed=21)
    data = I.make_all(p)
    r = Run(p, data)
    y1 = r.run()
    s = 600
    u2 = r.u.clone()
    u2[..., s + 1:] += torch.randn_like(u2[..., s + 1:])
    y2 = torch.empty_like(r.y)
    r.conv(u=u2, y=y2)
    torch.cuda.synchronize()
    y2 = y2.double().cpu().numpy()
    scale = np.abs(y1).max()
    assert np.abs(y2[..., : s + 1] - y1[..., : s + 1]).max() <= 1e-5 * scale
    assert np.abs(y2[..., s + 1:] - y1[..., s + 1:]).max() > 1e-2 * scale


def test_deterministic():
    import torch
    p = I.WORKLOADS["d768_l8k"].with_(C=32, seed=3)
    data = I.make_all(p)
    r = Run(p, data)
    r.run()
    a = r.y.clone()
    r.conv()
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), r.y.view(torch.int16))


def test_spectrum_check_and_mismatch():
    import torch
    from fft_long_convolution_02_b200 import binding as hb
    p = I.WORKLOADS["tiny"].with_(C=8, L=256)
    r = Run(p, I.make_all(p))
    r.build_spectrum()
    hb.hyena_spectrum_check(r.spectrum, p.C, p.shape, p.order)
    with pytest.raises(hb.HyenaError) as e:
        hb.hyena_spectrum_check(r.spectrum, p.C + 1, p.shape, p.order)
    assert e.value.status == 4
    fresh = torch.zeros_like(r.spectrum)
    with pytest.raises(hb.HyenaError):
        hb.hyena_spectrum_check(fresh, p.C, p.shape, p.order)


@pytest.mark.parametrize("L,dtype", [(256, "f32"), (8192, "bf16"), (8192, "f32")])
def test_kernel_reports_a_spectrum_header_mismatch(L, dtype):
    """A convolution given a spectrum that was never filled (right size, no
    header) writes no output and records HYENA_ERR_SPECTRUM_MISMATCH in the
    device's status word; the next call with a filled spectrum is clean."""
    import torch
    from fft_long_convolution_02_b200 import binding as hb
    p = I.WORKLOADS["d768_l8k"].with_(B=2, C=4, L=L, dtype=dtype, seed=5200 + L)
    r = Run(p, I.make_all(p))
    hb.hyena_kernel_status()
    fresh = torch.zeros_like(r.spectrum)
    y = torch.full_like(r.y, 3.0)
    hb.hyena_gated_fftconv(r.u, y, fresh, r.sc_w, None, p.B, p.C, p.shape, p.order)
    with pytest.raises(hb.HyenaError) as e:
        hb.hyena_kernel_status()
    assert e.value.status == 4                                    # HYENA_ERR_SPECTRUM_MISMATCH
    assert bool((y == 3.0).all())
    r.build_spectrum()
    hb.hyena_gated_fftconv(r.u, y, r.spectrum, r.sc_w, None, p.B, p.C, p.shape, p.order)
    hb.hyena_kernel_status()
    assert torch.isfinite(y.float()).all()


def test_fp32_transform_flag_at_8192(orc):
    """HYENA_FLAG_FP32_TRANSFORM: bf16 storage at L = 8192 with the fp32
    transform (no bf16 tensor-core operands); against the oracle it is far
    more accurate than the bf16-operand transform."""
    import torch
    from fft_long_convolution_02_b200 import binding as hb
    p = I.WORKLOADS["d768_l8k"].with_(B=3, C=6, seed=5300)
    data = I.make_all(p)
    r = Run(p, data)
    r.build_spectrum()
    hb.hyena_gated_fftconv_ex(r.u, r.y, r.spectrum, r.sc_w, None, p.B, p.C, p.shape, p.order,
                              flags=hb.HYENA_FLAG_FP32_TRANSFORM)
    torch.cuda.synchronize()
    rows = np.arange(p.B * p.C)
    ref = oracle_for_rows(orc, p, rows, data, method=2)
    err32 = row_rel_err(gpu_rows(from_torch(r.y), p, rows), ref).max()
    r.conv()
    torch.cuda.synchronize()
    err_tc = row_rel_err(gpu_rows(from_torch(r.y), p, rows), ref).max()
    # fp32 transform: only the bf16 rounding of the stored output remains (~2^-9 / sqrt(3))
    assert err32 <= 3e-3, err32
    assert err_tc <= TOL["bf16"], err_tc
    with pytest.raises(hb.HyenaError) as e:
        hb.hyena_gated_fftconv_ex(r.u, r.y, r.spectrum, r.sc_w, None, p.B, p.C, p.shape, p.order, flags=0x80)
    assert e.value.status == 1
