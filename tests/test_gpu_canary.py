"""GPU: out-of-bounds writes.  Every buffer the library writes (y, the
workspace, the spectrum) sits between guard regions filled with a NaN bit
pattern; after the calls the guards must be bit-identical and the results
must still match the oracle.  One case per kernel family."""
import numpy as np
import pytest

from fft_long_convolution_02_b200 import binding as hb
from fft_long_convolution_02_b200 import inputs as I
from gpu_helpers import TOL, api_shape, gpu_rows, oracle_for_rows, row_rel_err, to_torch

pytestmark = pytest.mark.gpu

GUARD = 4096            # bytes on each side (keeps 16-byte alignment)
PATTERN = 0x7FC1        # a quiet-NaN half-word, repeated


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fft_long_convolution_02_b200 import build
    build.build()


def _guarded(nbytes):
    """(full uint8 buffer, middle uint8 view of nbytes) with guard regions."""
    import torch
    full = torch.empty(GUARD + nbytes + GUARD, dtype=torch.uint8, device="cuda")
    full.view(torch.int16).fill_(PATTERN - 0x10000 if PATTERN >= 0x8000 else PATTERN)
    return full, full[GUARD:GUARD + nbytes]


def _guards_intact(full, nbytes):
    import torch
    ref = torch.full((GUARD // 2,), PATTERN, dtype=torch.int16, device="cuda")
    head = full[:GUARD].view(torch.int16)
    tail = full[GUARD + nbytes:].view(torch.int16)
    return bool(torch.equal(head, ref)) and bool(torch.equal(tail, ref))


CASES = [
    I.WORKLOADS["tiny"].with_(B=3, C=5, L=1024, seed=6001),                               # CTA engine, fp32
    I.WORKLOADS["d768_l8k"].with_(B=3, C=5, seed=6002),                                   # tensor cores, bf16
    I.WORKLOADS["d768_l8k"].with_(B=2, C=3, dtype="f32", seed=6003),                      # fp32 register kernel
    I.WORKLOADS["order3"].with_(B=2, C=3, L=1 << 15, seed=6004),                          # four-step, order 3
    I.WORKLOADS["order3"].with_(B=3, C=2, L=1 << 16, seed=6006),                          # 8-CTA clusters, order 3
    I.WORKLOADS["grid2d"].with_(B=2, C=3, H=64, W=32, sigma=(4.0, 16.0), seed=6005),      # 2-D
    I.WORKLOADS["grid2d"].with_(B=3, C=2, H=256, W=64, seed=6009),                         # 2-D tensor-core columns
    I.WORKLOADS["grid2d"].with_(B=2, C=2, H=256, W=256, seed=6010),                        # 2-D paired images
    I.WORKLOADS["grid2d_circ"].with_(B=2, C=2, H=256, W=256, seed=6011),                   # circular, paired
]


@pytest.mark.parametrize("p", CASES, ids=lambda p: f"{p.name}-{p.shape}-{p.dtype}-o{p.order}")
def test_writes_stay_inside_their_buffers(orc, p):
    import torch
    data = I.make_all(p)
    u = to_torch(p, data["u"])
    k = to_torch(p, data["k"])
    D = torch.from_numpy(data["D"]).cuda()
    sc_w = torch.from_numpy(data["sc_w"]).cuda() if data["sc_w"] is not None else None
    sb = hb.hyena_spectrum_bytes(p.C, api_shape(p), p.order)
    spec_full, spec = _guarded(sb)
    es = u.element_size()
    yb = p.B * p.C * int(np.prod(p.shape)) * es
    y_full, y8 = _guarded(yb)
    y = y8.view(u.dtype).view((p.B, p.C) + p.shape)
    wb = hb.hyena_gated_fftconv_workspace_bytes(p.B, p.C, api_shape(p), p.order)
    ws_full, ws = _guarded(wb) if wb else (None, None)
    hb.hyena_filter_spectrum(k, D, p.C, api_shape(p), p.order, spec)
    hb.hyena_gated_fftconv(u, y, spec, sc_w, None, p.B, p.C, api_shape(p), p.order, ws)
    hb.hyena_gated_fftconv(u, y, spec, sc_w, None, p.B, p.C, api_shape(p), p.order, ws)   # twice: reuse
    torch.cuda.synchronize()
    assert _guards_intact(spec_full, sb), "spectrum guard overwritten"
    assert _guards_intact(y_full, yb), "output guard overwritten"
    if wb:
        assert _guards_intact(ws_full, wb), "workspace guard overwritten"
    got = y.detach().to(torch.float64).cpu().numpy()
    rows = np.arange(p.B * p.C)
    err = row_rel_err(gpu_rows(got, p, rows), oracle_for_rows(orc, p, rows, data, sc_w is not None))
    assert err.max() <= TOL[p.dtype], err.max()
