"""hyena_gated_fftconv_noalloc: the entry point for callers that cannot
allocate device memory (a plugin whose host framework owns all device memory,
or a serving loop that must never call cudaMalloc).  It uses the library's
fixed scratch array instead of a caller workspace.

Each case calls it twice in a row through the C ABI and compares both
outputs with hyena_gated_fftconv given an ordinary workspace, within the
parity tolerance the other tests use.  The file is named so that pytest
collects it last; it also passes when run alone in a fresh process.
"""
import numpy as np
import pytest

from fft_long_convolution_02_b200 import inputs as I
from gpu_helpers import TOL, Run

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fft_long_convolution_02_b200 import build
    build.build()


CASES = [
    # four-step path, bf16, order 3, more rows than fit the scratch at once
    I.WORKLOADS["order3"].with_(B=2, C=40, L=1 << 16, sc_bias=True, seed=1201),
    # 2-D path, fp32
    I.WORKLOADS["grid2d"].with_(B=2, C=5, H=64, W=128, dtype="f32", sigma=(4.0, 32.0), seed=1202),
    # on-chip path (no scratch needed), bf16
    I.WORKLOADS["d768_l8k"].with_(C=16, seed=1203),
]


def _rel(a, b):
    a = a.reshape(a.shape[0] * a.shape[1], -1)
    b = b.reshape(b.shape[0] * b.shape[1], -1)
    return (np.linalg.norm(a - b, axis=1) / np.maximum(np.linalg.norm(b, axis=1), 1e-30)).max()


@pytest.mark.parametrize("p", CASES, ids=lambda p: f"{p.name}-{p.shape}-{p.dtype}")
def test_noalloc_matches_workspace_entry_point(p):
    import torch
    from fft_long_convolution_02_b200 import binding as hb
    data = I.make_all(p)
    r = Run(p, data)
    ref = r.run()                      # hyena_gated_fftconv with a workspace
    for _ in range(2):                 # two calls in a row share the fixed scratch
        y = torch.full_like(r.y, float("nan"))
        hb.hyena_gated_fftconv_noalloc(r.u, y, r.spectrum, r.sc_w, r.sc_b, p.B, p.C, p.shape, p.order)
        torch.cuda.synchronize()
        got = y.double().cpu().numpy()
        assert np.isfinite(got).all()
        assert _rel(got, ref) <= TOL[p.dtype]


def test_noalloc_rejects_bad_arguments_before_launch():
    import torch
    from fft_long_convolution_02_b200 import binding as hb
    p = CASES[0]
    r = Run(p, I.make_all(p))
    r.build_spectrum()
    with pytest.raises(hb.HyenaError) as e:
        hb.hyena_gated_fftconv_noalloc(r.u, r.y, r.spectrum, r.sc_w, r.sc_b, p.B, p.C + 1, p.shape, p.order)
    assert e.value.status == 4          # spectrum size does not match the shape
    torch.cuda.synchronize()
