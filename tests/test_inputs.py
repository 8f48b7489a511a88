"""CPU checks of the seeded input recipes that the oracle and the CUDA path
share: per-sample (input-dependent) filters come as [order-1, B*C, ...] and
the oracle's split takes row (b, c)'s filter at b*C + c; the shared-filter
recipes are unchanged by that option."""
import numpy as np

import oracle
from fft_long_convolution_02_b200 import inputs as I


def _split(p, data, rows):
    return oracle.split_rows(data["u"], data["k"], data["D"], data["sc_w"], data["sc_b"], B=p.B, C=p.C,
                             order=p.order, shape=p.shape, rows=rows, per_sample=p.per_sample)


def test_per_sample_filter_layout():
    p = I.WORKLOADS["tiny"].with_(B=3, C=4, L=64, order=3, per_sample=True, seed=11)
    data = I.make_all(p)
    assert data["k"].shape == (p.order - 1, p.B * p.C, p.L)
    assert data["D"].shape == (p.order - 1, p.B * p.C)
    rows = np.arange(p.B * p.C)
    _, k_rows, D_rows, _, _ = _split(p, data, rows)
    for r in rows:
        b, c = divmod(int(r), p.C)
        for s in range(p.order - 1):
            assert np.array_equal(k_rows[r, s], data["k"][s, b * p.C + c].astype(np.float64))
            assert D_rows[r, s] == np.float64(data["D"][s, b * p.C + c])
    # every filter is its own draw: k_row(s, b*C + c) regenerates it alone
    assert np.array_equal(I.store(p, I.k_row(p, 1, 2 * p.C + 3)), data["k"][1, 2 * p.C + 3])
    # different samples get different filters
    assert not np.array_equal(data["k"][0, 0], data["k"][0, p.C])


def test_shared_filters_unchanged_by_the_option():
    p = I.WORKLOADS["tiny"].with_(B=2, C=3, L=64, seed=12)
    data = I.make_all(p)
    assert p.FC == p.C and data["k"].shape == (1, p.C, p.L)
    _, k_rows, D_rows, _, _ = _split(p, data, np.arange(p.B * p.C))
    for r in range(p.B * p.C):
        assert np.array_equal(k_rows[r, 0], data["k"][0, r % p.C].astype(np.float64))
        assert D_rows[r, 0] == np.float64(data["D"][0, r % p.C])
