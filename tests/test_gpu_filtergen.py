"""GPU parity: the implicit long filter generated on the device and fed into
the spectrum build (hyena_filter_spectrum_implicit), against the float64
oracle of HyenaFilter (oracle/filter_gen.py) and the float64 operator oracle.

* The generated filters (the k_out copy) match the oracle's filter(L): fp32
  MLP and modulation against float64, per row max |diff| <= 2e-5 max |k|.
* The spectrum equals, bit for bit, the one hyena_filter_spectrum builds
  from that copy (the same FFT on the same samples).
* The operator run with it matches the oracle operator run with the oracle's
  filters, at L = 1024 (fp32 storage, 1e-4) and L = 8192 (bf16 storage on the
  tensor-core kernel, 2e-2).
"""
import numpy as np
import pytest

from fft_long_convolution_02_b200 import binding as hb
from fft_long_convolution_02_b200 import inputs as I
from gpu_helpers import TOL, from_torch, row_rel_err, to_torch
from oracle import filter_gen as F

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fft_long_convolution_02_b200 import build
    build.build()


def _oracle_filters(p, prm):
    k = F.hyena_filter(p.L, prm["emb_dim"], prm["W_in"], prm["b_in"],
                       [(prm["W_inner"][i], prm["b_inner"][i]) for i in range(prm["num_inner"])],
                       prm["W_out"], prm["w"], prm["alpha"])
    return F.operator_filters(k, p.order)             # [order-1, C, L]


def _device_params(prm):
    import torch
    return {k: (torch.from_numpy(v).cuda() if isinstance(v, np.ndarray) else v) for k, v in prm.items()}


@pytest.mark.parametrize("L,dtype,order,width", [(1024, "f32", 2, 64), (8192, "bf16", 2, 64), (256, "f32", 3, 32),
                                                 (16384, "f32", 2, 16), (16, "f32", 2, 64)])
def test_implicit_filter_spectrum(orc, L, dtype, order, width):
    import torch
    p = I.WORKLOADS["d768_l8k"].with_(B=2, C=12, L=L, dtype=dtype, order=order, seed=7000 + L + order)
    prm = I.implicit_filter_params(p, width=width)
    dprm = _device_params(prm)
    data = I.make_all(p)
    D = torch.from_numpy(data["D"]).cuda()
    nbytes = hb.hyena_spectrum_bytes(p.C, p.shape, p.order)
    # zero-filled: the alignment gap between the tables and the rows is never written
    spec = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    ws = torch.empty(hb.hyena_implicit_filter_workspace_bytes(L, width), dtype=torch.uint8, device="cuda")
    k_out = torch.empty((p.order - 1, p.C, L), dtype=torch.float32, device="cuda")
    hb.hyena_filter_spectrum_implicit(dprm, D, p.C, L, p.order, spec, ws, k_out)
    torch.cuda.synchronize()
    # the generated filters against the oracle's
    k_ref = _oracle_filters(p, prm)
    k_got = k_out.double().cpu().numpy()
    scale = np.abs(k_ref).max(axis=-1, keepdims=True)
    assert (np.abs(k_got - k_ref) / scale).max() <= 2e-5
    # the same spectrum as the stored-filter build from the copy
    spec2 = torch.zeros_like(spec)
    hb.hyena_filter_spectrum(k_out, D, p.C, p.shape, p.order, spec2)
    torch.cuda.synchronize()
    assert torch.equal(spec, spec2)
    # the operator with it, against the oracle operator with the oracle's filters
    u = to_torch(p, data["u"])
    sc_w = torch.from_numpy(data["sc_w"]).cuda()
    y = torch.empty((p.B, p.C, L), dtype=u.dtype, device="cuda")
    hb.hyena_gated_fftconv(u, y, spec, sc_w, None, p.B, p.C, p.shape, p.order)
    torch.cuda.synchronize()
    hb.hyena_kernel_status()
    ref = orc.hyena_stacked(data["u"], k_ref, data["D"], data["sc_w"], B=p.B, C=p.C, order=p.order,
                            shape=p.shape, method=2)
    err = row_rel_err(from_torch(y).reshape(p.B * p.C, -1), ref)
    assert err.max() <= TOL[dtype], err.max()


def test_implicit_filter_without_copy_and_errors():
    """k_out = NULL builds the same spectrum; bad arguments are refused
    before any launch."""
    import torch
    p = I.WORKLOADS["tiny"].with_(C=4, L=512, seed=7100)
    prm = _device_params(I.implicit_filter_params(p, width=32, num_inner=0))
    D = torch.zeros((p.order - 1, p.C), device="cuda")
    nbytes = hb.hyena_spectrum_bytes(p.C, p.shape, p.order)
    ws = torch.empty(hb.hyena_implicit_filter_workspace_bytes(p.L, 32), dtype=torch.uint8, device="cuda")
    a, b = (torch.zeros(nbytes, dtype=torch.uint8, device="cuda") for _ in range(2))
    k_out = torch.empty((p.order - 1, p.C, p.L), device="cuda")
    hb.hyena_filter_spectrum_implicit(prm, D, p.C, p.L, p.order, a, ws, k_out)
    hb.hyena_filter_spectrum_implicit(prm, D, p.C, p.L, p.order, b, ws, None)
    torch.cuda.synchronize()
    assert torch.equal(a, b)
    with pytest.raises(hb.HyenaError) as e:
        hb.hyena_filter_spectrum_implicit(prm, D, p.C, p.L, p.order, a, ws[:-16])
    assert e.value.status == 5                       # workspace too small
    big = I.WORKLOADS["tiny"].with_(C=1, L=32768)
    with pytest.raises(hb.HyenaError) as e:
        hb.hyena_filter_spectrum_implicit(prm, D, 1, 32768, 2,
                                          torch.empty(hb.hyena_spectrum_bytes(1, big.shape, 2), dtype=torch.uint8,
                                                      device="cuda"),
                                          torch.empty(32768 * 32 * 4, dtype=torch.uint8, device="cuda"))
    assert e.value.status == 2                       # not an on-chip length
    bad = dict(prm, emb_dim=4)
    with pytest.raises(hb.HyenaError) as e:
        hb.hyena_filter_spectrum_implicit(bad, D, p.C, p.L, p.order, a, ws)
    assert e.value.status == 1
