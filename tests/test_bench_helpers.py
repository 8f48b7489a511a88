"""CPU checks of bench.py's bookkeeping: the kernels a call launches (the
`gpu_launches` claim), the spectrum bytes each path reads and the
algorithmic bytes of the roofline, per workload, written out from the
dispatch rules of the library (which path serves which shape)."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from fft_long_convolution_02_b200 import inputs as I  # noqa: E402

W = I.WORKLOADS


@pytest.mark.parametrize("name,want", [
    ("tiny", 1),            # on-chip kernel, all order steps inside
    ("d768_l8k", 1),        # the L = 8192 tensor-core kernel
    ("order3", 1),          # the 8-CTA cluster kernel, both steps inside
    ("dna_1m", 3),          # columns forward, rows, inverse columns
    ("grid2d", 3),          # paired images: rows, columns, rows inverse
    ("grid2d_circ", 3),     # circular pairs: the same three passes
    ("vol3d", 5),           # rows, columns, depth, columns inverse, rows inverse
])
def test_launches_per_call(name, want):
    assert bench.launches_per_step(W[name]) == want


def test_launches_follow_the_dispatch():
    # an odd batch has no image pairs: rows forward, then per step columns and rows inverse
    assert bench.launches_per_step(W["grid2d_circ"].with_(B=3)) == 3
    assert bench.launches_per_step(W["grid2d_circ"].with_(B=3, order=3)) == 5
    # order 3 pairs: three passes per step
    assert bench.launches_per_step(W["grid2d_circ"].with_(order=3)) == 6
    assert bench.launches_per_step(W["grid2d"].with_(order=3)) == 6
    # order 4 on the fp32 passes
    assert bench.launches_per_step(W["grid2d"].with_(order=4)) == 7
    # 2-D H = 256 with W = 64: the tensor-core column pass between fp32 row passes
    assert bench.launches_per_step(W["grid2d"].with_(W=64)) == 4


def test_spectrum_bytes_per_row():
    # L = 8192: one plane of 2L bf16 pairs (or the fp32 position layout), 8L bytes
    assert bench.spectrum_row_bytes(W["d768_l8k"]) == 8 * 8192
    # paired 2-D: the whole bf16 plane, 2H x 2W padded, H x W circular
    assert bench.spectrum_row_bytes(W["grid2d"]) == 512 * 512 * 4
    assert bench.spectrum_row_bytes(W["grid2d_circ"]) == 256 * 256 * 4
    # unpaired circular: (W/2 + 1) H complex64
    assert bench.spectrum_row_bytes(W["grid2d_circ"].with_(B=3)) == 129 * 256 * 8


def test_algorithmic_bytes_of_the_headline():
    p = W["d768_l8k"]
    alg = bench.algorithmic_bytes(p, bench.spectrum_row_bytes(p))
    # u: 4 x 2304 x 8192 bf16, y: 4 x 768 x 8192 bf16, spectrum: 768 rows of 64 KB
    assert alg == 4 * 2304 * 8192 * 2 + 4 * 768 * 8192 * 2 + 768 * 8 * 8192
    assert round(alg / 1e6, 1) == 251.7
