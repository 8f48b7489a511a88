"""GPU parity of hyena_gated_fftconv_per_sample (one long filter per (b, c)
row, the input-dependent kernels of HyenaND) on every path, against the
float64 oracle, plus the invariant that per-sample filters which repeat the
shared filters for every b give the shared-filter result."""
import numpy as np
import pytest

from fft_long_convolution_02_b200 import binding as hb
from fft_long_convolution_02_b200 import inputs as I
from gpu_helpers import TOL, from_torch, oracle_for_rows, row_rel_err, to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fft_long_convolution_02_b200 import build
    build.build()


def _run(p, data, per_sample, k=None, D=None, use_shortconv=True):
    """One spectrum build and one convolution; k/D override data's filters."""
    import torch
    u = to_torch(p, data["u"])
    kk = to_torch(p, data["k"] if k is None else k)
    DD = torch.from_numpy(np.ascontiguousarray(data["D"] if D is None else D)).cuda()
    FC = kk.shape[1]
    sc_w = torch.from_numpy(data["sc_w"]).cuda() if (use_shortconv and data["sc_w"] is not None) else None
    spec = torch.empty(hb.hyena_spectrum_bytes(FC, p.shape, p.order), dtype=torch.uint8, device="cuda")
    y = torch.empty((p.B, p.C) + p.shape, dtype=u.dtype, device="cuda")
    wsb = hb.hyena_gated_fftconv_workspace_bytes(p.B, p.C, p.shape, p.order)
    ws = torch.empty(wsb, dtype=torch.uint8, device="cuda") if wsb else None
    hb.hyena_filter_spectrum(kk, DD, FC, p.shape, p.order, spec)
    conv = hb.hyena_gated_fftconv_per_sample if per_sample else hb.hyena_gated_fftconv
    conv(u, y, spec, sc_w, None, p.B, p.C, p.shape, p.order, ws)
    torch.cuda.synchronize()
    return from_torch(y)


CASES = [
    # (base workload, overrides): one per path
    ("tiny", dict(B=3, C=4, L=1024)),                                   # on-chip, fp32
    ("tiny", dict(B=2, C=3, L=4096, dtype="bf16")),                     # on-chip, bf16
    ("d768_l8k", dict(B=4, C=3)),                                       # L = 8192 bf16 (fp32 register kernel)
    ("d768_l8k", dict(B=2, C=2, dtype="f32", order=3)),                 # L = 8192 fp32, two order steps
    ("order3", dict(B=3, C=2, L=1 << 15)),                              # four-step, bf16, order 3
    ("dna_1m", dict(B=2, C=2, L=1 << 16, u_kind="normal", dtype="f32")),  # four-step, fp32
    ("grid2d", dict(B=2, C=3, H=32, W=64)),                             # 2-D, bf16
]


@pytest.mark.parametrize("name,kw", CASES)
def test_per_sample_matches_oracle(orc, name, kw):
    p = I.WORKLOADS[name].with_(per_sample=True, seed=900 + len(kw) + kw.get("L", 0) % 97, **kw)
    data = I.make_all(p)
    assert data["k"].shape[1] == p.B * p.C
    y = _run(p, data, per_sample=True)
    rows = np.arange(p.B * p.C)
    ref = oracle_for_rows(orc, p, rows, data, method=2)
    err = row_rel_err(y.reshape(p.B * p.C, -1), ref)
    assert err.max() <= TOL[p.dtype], f"{name} {kw}: max row rel err {err.max():.3e}"


@pytest.mark.parametrize("name,kw", CASES)
def test_repeated_filters_equal_shared(name, kw):
    """k_ps[s, b*C + c] = k[s, c] (and D likewise) gives the shared-filter
    output: bit for bit where both calls run the same kernel, within the
    tolerance at L = 8192 bf16 (shared filters run the tensor-core kernel)."""
    p = I.WORKLOADS[name].with_(seed=950, **kw)
    data = I.make_all(p)
    k_ps = np.concatenate([data["k"]] * p.B, axis=1)
    D_ps = np.concatenate([data["D"]] * p.B, axis=1)
    y_shared = _run(p, data, per_sample=False)
    y_ps = _run(p, data, per_sample=True, k=k_ps, D=D_ps)
    if p.ndim == 1 and p.L == 8192 and p.dtype == "bf16":
        err = row_rel_err(y_ps.reshape(p.B * p.C, -1), y_shared.reshape(p.B * p.C, -1))
        assert err.max() <= TOL["bf16"]
    else:
        assert np.array_equal(y_ps, y_shared)


def test_per_sample_rejects_a_shared_spectrum():
    """A spectrum built for C filters is the wrong size for B*C rows."""
    import torch
    p = I.WORKLOADS["tiny"].with_(B=2, C=4)
    data = I.make_all(p)
    u = to_torch(p, data["u"])
    k = to_torch(p, data["k"])
    spec = torch.empty(hb.hyena_spectrum_bytes(p.C, p.shape, p.order), dtype=torch.uint8, device="cuda")
    hb.hyena_filter_spectrum(k, torch.from_numpy(data["D"]).cuda(), p.C, p.shape, p.order, spec)
    y = torch.empty((p.B, p.C) + p.shape, dtype=u.dtype, device="cuda")
    with pytest.raises(RuntimeError, match="SPECTRUM_MISMATCH"):
        hb.hyena_gated_fftconv_per_sample(u, y, spec, None, None, p.B, p.C, p.shape, p.order)
