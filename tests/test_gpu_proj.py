"""GPU parity: the in/out projections on the tensor cores (hyena_in_proj,
hyena_out_proj) against the float64 oracle, through the C ABI.

Tolerance: the result is rounded to bf16 once after an fp32 accumulation over
D <= 768 products of exact bf16 values.  Round to nearest with 8 significant
bits is off by at most half an ulp, 2^-8 of the value at the bottom of a
binade, so every element and hence every row's relative L2 error is at most
2^-8 (about 1.1e-3 on average for long rows); the fp32 accumulation adds
about D 2^-24.  The tests assert 2^-8 + 1e-5.  The layer test chains in_proj, the operator and out_proj
(three bf16 roundings of the intermediates plus the operator's own error)
against the oracle's chain at the operator's bf16 tolerance."""
import numpy as np
import pytest

from fft_long_convolution_02_b200 import binding as hb
from fft_long_convolution_02_b200 import inputs as I
from gpu_helpers import TOL, from_torch, row_rel_err, to_torch

pytestmark = pytest.mark.gpu
PROJ_TOL = 2.0 ** -8 + 1e-5


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fft_long_convolution_02_b200 import build
    build.build()


def _layer_tensors(p, lay):
    import torch
    t = {k: to_torch(p, v) for k, v in lay.items() if k in ("x", "W_in", "W_out")}
    t["b_in"] = torch.from_numpy(lay["b_in"]).cuda()
    t["b_out"] = torch.from_numpy(lay["b_out"]).cuda()
    return t


def _rows_err(got, ref):
    return row_rel_err(got.reshape(-1, got.shape[-1]), ref.reshape(-1, ref.shape[-1])).max()


@pytest.mark.parametrize("B,L,D,order", [(1, 256, 64, 2), (2, 136, 72, 3), (3, 520, 128, 2), (1, 64, 8, 2),
                                         (2, 1024, 200, 4)])
def test_projections_small_shapes(orc, B, L, D, order):
    """Every output element, shapes with ragged tiles (L, D not multiples of
    the 128 x 256 tile or the 64-wide K block), with and without bias."""
    import torch
    p = I.WORKLOADS["d768_l8k"].with_(B=B, C=D, L=L, order=order, seed=6000 + L + D)
    lay = I.make_layer(p)
    t = _layer_tensors(p, lay)
    J = (order + 1) * D
    for bias in (True, False):
        u = torch.full((B, J, L), float("nan"), dtype=torch.bfloat16, device="cuda")
        hb.hyena_in_proj(t["x"], t["W_in"], t["b_in"] if bias else None, u, order)
        y = torch.full((B, L, D), float("nan"), dtype=torch.bfloat16, device="cuda")
        v = u[:, :D].contiguous()                 # any [B, D, L] tensor serves as out_proj input
        hb.hyena_out_proj(v, t["W_out"], t["b_out"] if bias else None, y)
        torch.cuda.synchronize()
        hb.hyena_kernel_status()
        ref_u = orc.in_proj(lay["x"], lay["W_in"], lay["b_in"] if bias else None)
        assert _rows_err(from_torch(u), ref_u) <= PROJ_TOL
        ref_y = orc.out_proj(from_torch(v), lay["W_out"], lay["b_out"] if bias else None)
        assert _rows_err(from_torch(y), ref_y) <= PROJ_TOL


def test_projections_full_size_sampled(orc):
    """B=4, L=8192, D=768, order 2 (the benchmarked width and length): in_proj
    on 64 sampled output channels over every (b, l), out_proj on 64 sampled
    positions over every (b, j)."""
    import torch
    p = I.WORKLOADS["d768_l8k"]
    lay = I.make_layer(p)
    t = _layer_tensors(p, lay)
    B, L, D, J = p.B, p.L, p.C, p.Ctot
    u = torch.empty((B, J, L), dtype=torch.bfloat16, device="cuda")
    hb.hyena_in_proj(t["x"], t["W_in"], t["b_in"], u, p.order)
    v = u[:, J - D:].contiguous()
    out = torch.empty((B, L, D), dtype=torch.bfloat16, device="cuda")
    hb.hyena_out_proj(v, t["W_out"], t["b_out"], out)
    torch.cuda.synchronize()
    hb.hyena_kernel_status()
    rng = np.random.default_rng(61)
    js = np.sort(rng.choice(J, 64, replace=False))
    ref_u = orc.in_proj(lay["x"], lay["W_in"][js], lay["b_in"][js])
    assert _rows_err(from_torch(u[:, js]), ref_u) <= PROJ_TOL
    ls = np.sort(rng.choice(L, 64, replace=False))
    ref_o = orc.out_proj(from_torch(v[:, :, ls]), lay["W_out"], lay["b_out"])
    assert _rows_err(from_torch(out[:, ls]), ref_o) <= PROJ_TOL


def test_layer_chain_matches_oracle(orc):
    """x -> in_proj -> hyena_gated_fftconv -> out_proj against the oracle's
    chain in float64 (the CUDA side rounds u and y to bf16 on the way)."""
    import torch
    p = I.WORKLOADS["d768_l8k"].with_(B=2, C=64, L=1024, seed=6100)
    lay = I.make_layer(p)
    data = I.make_all(p)
    t = _layer_tensors(p, lay)
    k = to_torch(p, data["k"])
    Dk = torch.from_numpy(data["D"]).cuda()
    sc_w = torch.from_numpy(data["sc_w"]).cuda()
    spec = torch.empty(hb.hyena_spectrum_bytes(p.C, p.shape, p.order), dtype=torch.uint8, device="cuda")
    hb.hyena_filter_spectrum(k, Dk, p.C, p.shape, p.order, spec)
    u = torch.empty((p.B, p.Ctot, p.L), dtype=torch.bfloat16, device="cuda")
    y = torch.empty((p.B, p.C, p.L), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((p.B, p.L, p.C), dtype=torch.bfloat16, device="cuda")
    hb.hyena_in_proj(t["x"], t["W_in"], t["b_in"], u, p.order)
    hb.hyena_gated_fftconv(u, y, spec, sc_w, None, p.B, p.C, p.shape, p.order)
    hb.hyena_out_proj(y, t["W_out"], t["b_out"], out)
    torch.cuda.synchronize()
    hb.hyena_kernel_status()
    u_ref = orc.in_proj(lay["x"], lay["W_in"], lay["b_in"])
    y_ref = orc.hyena_stacked(u_ref, data["k"], data["D"], data["sc_w"], B=p.B, C=p.C, order=p.order, shape=p.shape,
                              method=2).reshape(p.B, p.C, p.L)
    o_ref = orc.out_proj(y_ref, lay["W_out"], lay["b_out"])
    assert _rows_err(from_torch(out), o_ref) <= TOL["bf16"]
