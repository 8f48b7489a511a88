"""CPU checks of the seeded input recipes that the oracle and the CUDA path
share: per-sample (input-dependent) filters are indexed b*C + c, and the
shared-filter recipes are unchanged by that option."""
import numpy as np

from fft_long_convolution_02_b200 import inputs as I


def test_per_sample_filter_layout_and_oracle_rows():
    p = I.WORKLOADS["tiny"].with_(B=3, C=4, L=64, order=3, per_sample=True, seed=11)
    data = I.make_all(p)
    assert data["k"].shape == (p.order - 1, p.B * p.C, p.L)
    assert data["D"].shape == (p.order - 1, p.B * p.C)
    rows = np.arange(p.B * p.C)
    _, k_rows, D_rows, _, _ = I.oracle_rows(p, rows, data)
    for r in rows:
        b, c = divmod(int(r), p.C)
        for s in range(p.order - 1):
            assert np.array_equal(k_rows[r, s], data["k"][s, b * p.C + c].astype(np.float64))
            assert D_rows[r, s] == np.float64(data["D"][s, b * p.C + c])
    # rows generated without the full tensors agree with the cut ones
    _, k2, D2, _, _ = I.oracle_rows(p, rows[[0, 5, 11]])
    assert np.array_equal(k2, k_rows[[0, 5, 11]]) and np.array_equal(D2, D_rows[[0, 5, 11]])
    # different samples get different filters
    assert not np.array_equal(data["k"][0, 0], data["k"][0, p.C])


def test_shared_filters_unchanged_by_the_option():
    p = I.WORKLOADS["tiny"].with_(B=2, C=3, L=64, seed=12)
    data = I.make_all(p)
    assert p.FC == p.C and data["k"].shape == (1, p.C, p.L)
    _, k_rows, D_rows, _, _ = I.oracle_rows(p, np.arange(p.B * p.C), data)
    for r in range(p.B * p.C):
        assert np.array_equal(k_rows[r, 0], data["k"][0, r % p.C].astype(np.float64))
        assert D_rows[r, 0] == np.float64(data["D"][0, r % p.C])
