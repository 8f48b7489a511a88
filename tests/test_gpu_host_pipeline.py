"""GPU checks of hyena_gated_fftconv_host (host buffers, copies pipelined
against the kernels): the result in host memory equals the device-path
result, bit for bit when each chunk runs the same kernel on the same rows,
and matches the oracle otherwise; every path, odd batches, one-row chunks."""
import numpy as np
import pytest

from fft_long_convolution_02_b200 import binding as hb
from fft_long_convolution_02_b200 import inputs as I
from gpu_helpers import TOL, Run, api_shape, oracle_for_rows, row_rel_err, to_torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fft_long_convolution_02_b200 import build
    build.build()


CASES = [
    ("tiny", dict(B=3, C=4, L=1024), 2),                      # on-chip fp32, odd batch
    ("d768_l8k", dict(B=4, C=8), 2),                          # tensor-core kernel, pairs kept whole
    ("d768_l8k", dict(B=4, C=8), 0),                          # default chunk (2 rows): pairs kept whole
    ("d768_l8k", dict(B=3, C=8), 0),                          # default chunk rounded up to 2 rows
    ("order3", dict(B=3, C=2, L=1 << 15), 1),                 # four-step: chunks share the workspace
    ("order3", dict(B=4, C=2, L=1 << 16), 2),                 # cluster kernel, pairs kept whole
    ("grid2d", dict(B=2, C=3, H=32, W=64), 1),                # 2-D
]


@pytest.mark.parametrize("name,kw,chunk", CASES)
def test_host_pipeline_equals_device_path(name, kw, chunk):
    import torch
    p = I.WORKLOADS[name].with_(seed=2000 + chunk, **kw)
    data = I.make_all(p)
    use_sc = p.shortconv
    r = Run(p, data, use_sc)
    want = r.run()
    u_host = to_torch(p, data["u"], device="cpu").pin_memory()
    y_host = torch.empty(r.y.shape, dtype=r.y.dtype).pin_memory()
    u_dev = torch.empty_like(r.u)
    y_dev = torch.empty_like(r.y)
    hb.hyena_gated_fftconv_host(u_host, y_host, u_dev, y_dev, r.spectrum, r.sc_w, r.sc_b, p.B, p.C, api_shape(p),
                                p.order, r.workspace, chunk_rows=chunk)
    torch.cuda.synchronize()
    got = y_host.to(torch.float64).numpy()
    assert np.array_equal(got, want)


def test_host_pipeline_one_row_chunks_match_oracle(orc):
    """B = 4 at L = 8192 bf16 in one-row chunks (the tensor-core kernel pairs
    each row with zeros): within the bf16 tolerance of the oracle."""
    import torch
    p = I.WORKLOADS["d768_l8k"].with_(B=4, C=6, seed=2100)
    data = I.make_all(p)
    r = Run(p, data, True)
    r.build_spectrum()
    u_host = to_torch(p, data["u"], device="cpu").pin_memory()
    y_host = torch.empty(r.y.shape, dtype=r.y.dtype).pin_memory()
    hb.hyena_gated_fftconv_host(u_host, y_host, torch.empty_like(r.u), torch.empty_like(r.y), r.spectrum, r.sc_w,
                                None, p.B, p.C, p.shape, p.order, None, chunk_rows=1)
    torch.cuda.synchronize()
    rows = np.arange(p.B * p.C)
    ref = oracle_for_rows(orc, p, rows, data, method=2)
    err = row_rel_err(y_host.to(torch.float64).numpy().reshape(p.B * p.C, -1), ref)
    assert err.max() <= TOL["bf16"]
