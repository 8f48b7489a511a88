"""hyena_gated_fftconv_noalloc: the entry point for callers that cannot
allocate device memory (a plugin whose host framework owns all device memory,
or a serving loop that must never call cudaMalloc).  It uses the library's
fixed 32 MiB scratch array instead of a caller workspace.

Each case calls it twice in a row through the C ABI.  Both outputs must be
bit for bit those of hyena_gated_fftconv given an ordinary workspace: the
same kernels compute every row the same way whatever the group of rows that
shares the scratch.  One case is also compared with the float64 oracle.
The file is named so that pytest collects it last; it also passes when run
alone in a fresh process.
"""
import numpy as np
import pytest

from fft_long_convolution_02_b200 import binding as hb
from fft_long_convolution_02_b200 import inputs as I
from gpu_helpers import TOL, Run, api_shape, oracle_for_rows, row_rel_err

pytestmark = pytest.mark.gpu

SCRATCH = 32 << 20      # HYENA_NOALLOC_SCRATCH_BYTES


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    import torch
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from fft_long_convolution_02_b200 import build
    build.build()


def _groups(p):
    """Groups of rows the fixed scratch is cut into for problem p."""
    row = hb.hyena_gated_fftconv_workspace_min_bytes(p.C, api_shape(p), p.order)
    per_group = SCRATCH // row
    if p.ndim in (1, 2) and p.dtype == "bf16":
        per_group *= 2          # the four-step and 2-D workspaces hold bf16 pairs with bf16 storage
    return -(-p.B * p.C // per_group)


CASES = [
    # four-step path, bf16, L = 2^20: 8 rows per group, 20 rows -> 3 groups
    I.WORKLOADS["dna_1m"].with_(B=1, C=20, u_kind="normal", seed=1201),
    # four-step path, fp32, order 3, L = 2^16: 64 rows per group, 80 rows -> 2 groups
    I.WORKLOADS["order3"].with_(B=2, C=40, L=1 << 16, dtype="f32", sc_bias=True, seed=1202),
    # 3-D path, bf16: one 64x128x128 volume per group, 8 volumes -> 8 groups
    I.WORKLOADS["vol3d"].with_(B=2, C=4, N1=64, H=128, W=128, seed=1203),
    # 2-D path, fp32: one group
    I.WORKLOADS["grid2d"].with_(B=2, C=5, H=64, W=128, dtype="f32", sigma=(4.0, 32.0), seed=1204),
    # 2-D path with the tensor-core column pass, bf16: 256 x 512 images (513 bin
    # columns of 256 bf16 pairs, 0.5 MB of scratch each) -> 62 per group, 70 -> 2 groups
    I.WORKLOADS["grid2d"].with_(B=2, C=35, H=256, W=512, seed=1207),
    # 2-D paired images (256 x 256, order 2): 126 images per group, 140 -> 2 groups of whole pairs
    I.WORKLOADS["grid2d"].with_(B=2, C=70, H=256, W=256, seed=1208),
    # on-chip path (no scratch needed), bf16
    I.WORKLOADS["d768_l8k"].with_(C=16, seed=1205),
    # cluster path, bf16, order 3, L = 2^16: the scratch holds one 512 KB slice per cluster
    I.WORKLOADS["order3"].with_(B=3, C=7, L=1 << 16, seed=1206),
    # circular 2-D paired images (256 x 256, order 2): 254 images per group, 280 -> 2 groups of whole pairs
    I.WORKLOADS["grid2d_circ"].with_(B=2, C=140, seed=1209),
]
EXPECTED_GROUPS = [3, 2, 8, 1, 2, 2, None, None, 2]


def test_cases_span_several_groups():
    for p, want in zip(CASES, EXPECTED_GROUPS):
        if want is not None:
            assert _groups(p) == want, (p.name, _groups(p))


@pytest.mark.parametrize("p", CASES, ids=lambda p: f"{p.name}-{p.shape}-{p.dtype}")
def test_noalloc_matches_workspace_entry_point(p):
    import torch
    data = I.make_all(p)
    r = Run(p, data)
    ref = r.run()                      # hyena_gated_fftconv with a workspace
    for _ in range(2):                 # two calls in a row share the fixed scratch
        y = torch.full_like(r.y, float("nan"))
        hb.hyena_gated_fftconv_noalloc(r.u, y, r.spectrum, r.sc_w, r.sc_b, p.B, p.C, api_shape(p), p.order)
        torch.cuda.synchronize()
        got = y.double().cpu().numpy()
        assert np.isfinite(got).all()
        assert np.array_equal(got, ref), f"max |diff| {np.abs(got - ref).max():.3e}"


def test_noalloc_against_the_oracle(orc):
    """Three scratch groups at L = 2^20 (bf16): every row against the oracle."""
    import torch
    p = CASES[0]
    data = I.make_all(p)
    r = Run(p, data)
    r.build_spectrum()
    hb.hyena_gated_fftconv_noalloc(r.u, r.y, r.spectrum, r.sc_w, r.sc_b, p.B, p.C, p.shape, p.order)
    torch.cuda.synchronize()
    got = r.y.double().cpu().numpy().reshape(p.B * p.C, -1)
    ref = oracle_for_rows(orc, p, np.arange(p.B * p.C), data, method=2).reshape(p.B * p.C, -1)
    assert row_rel_err(got, ref).max() <= TOL[p.dtype]


def test_noalloc_rejects_bad_arguments_before_launch():
    import torch
    p = CASES[3]
    r = Run(p, I.make_all(p))
    r.build_spectrum()
    with pytest.raises(hb.HyenaError) as e:
        hb.hyena_gated_fftconv_noalloc(r.u, r.y, r.spectrum, r.sc_w, r.sc_b, p.B, p.C + 1, p.shape, p.order)
    assert e.value.status == 4          # spectrum size does not match the shape
    torch.cuda.synchronize()


def test_noalloc_rejects_a_row_larger_than_the_scratch():
    """A 128^3 volume needs ~50.7 MB of scratch (> 32 MiB): rejected with
    HYENA_ERR_WORKSPACE_TOO_SMALL before anything runs; y is left untouched."""
    import torch
    p = I.WORKLOADS["vol3d"].with_(B=1, C=1, N1=128, H=128, W=128, seed=1206)
    assert hb.hyena_gated_fftconv_workspace_min_bytes(p.C, p.shape, p.order) > SCRATCH
    data = I.make_all(p)
    r = Run(p, data, workspace_bytes=0)
    r.build_spectrum()
    y = torch.full_like(r.y, 7.0)
    with pytest.raises(hb.HyenaError) as e:
        hb.hyena_gated_fftconv_noalloc(r.u, y, r.spectrum, None, None, p.B, p.C, p.shape, p.order)
    assert e.value.status == 5
    torch.cuda.synchronize()
    assert bool((y == 7.0).all())
