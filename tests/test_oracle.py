"""CPU tests: the float64 oracle against its pins, and the input generators."""
import numpy as np
import pytest

import oracle_pins
from fft_long_convolution_02_b200 import inputs as I


@pytest.mark.parametrize("pin", oracle_pins.ALL_PINS, ids=lambda f: f.__name__)
def test_pin(orc, pin):
    pin(orc)


def test_tiny_workload_direct_equals_fft(orc):
    """The whole small workload: the direct-sum oracle and the FFT oracle agree."""
    p = I.WORKLOADS["tiny"]
    data = I.make_all(p)
    kw = dict(B=p.B, C=p.C, order=p.order, shape=p.shape)
    y1 = orc.hyena_stacked(data["u"], data["k"], data["D"], data["sc_w"], data["sc_b"], method=1, **kw)
    y2 = orc.hyena_stacked(data["u"], data["k"], data["D"], data["sc_w"], data["sc_b"], method=2, **kw)
    rel = np.linalg.norm(y1 - y2, axis=-1) / np.linalg.norm(y1, axis=-1)
    assert rel.max() < 1e-12


@pytest.mark.slow
def test_d768_l8k_sampled_rows_direct_equals_fft(orc):
    """Full L = 8192 on sampled rows: direct sums and the radix-2 FFT agree."""
    p = I.WORKLOADS["d768_l8k"]
    data = I.make_all(p)
    kw = dict(B=p.B, C=p.C, order=p.order, shape=p.shape, rows=np.array([0, 767, 2 * 768 + 5]))
    y1 = orc.hyena_stacked(data["u"], data["k"], data["D"], data["sc_w"], method=1, **kw)
    y2 = orc.hyena_stacked(data["u"], data["k"], data["D"], data["sc_w"], method=2, **kw)
    rel = np.linalg.norm(y1 - y2, axis=-1) / np.linalg.norm(y1, axis=-1)
    assert rel.max() < 1e-11


def test_bf16_rounding_matches_torch():
    """Round-to-nearest-even float32 -> bf16 against torch's conversion."""
    import torch
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(100000).astype(np.float32) * 10.0 ** rng.integers(-6, 6, 100000),
                        np.array([0.0, -0.0, 1.0, 1.00390625, 1.01171875, 65504.0], np.float32)])
    mine = I.to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, ref)
    back = I.bf16_bits_to_f32(mine)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_generators_are_row_addressable():
    """A channel row generated on its own equals the same row of the full tensor."""
    for p in (I.WORKLOADS["tiny"].with_(B=2, C=8, L=64), I.WORKLOADS["dna_1m"].with_(L=256)):
        data = I.make_all(p)
        for b, ch in ((0, 3), (p.B - 1, p.Ctot - 1)):
            assert np.array_equal(I.store(p, I.u_row(p, b, ch)), data["u"][b, ch])
        assert np.array_equal(I.store(p, I.k_row(p, 0, p.C - 1)), data["k"][0, p.C - 1])


def test_generator_recipes():
    p = I.WORKLOADS["d768_l8k"]
    k = I.k_row(p, 0, 5)
    assert k.shape == (8192,)
    # exponential decay: late samples are much smaller than early ones
    assert np.abs(k[-512:]).mean() < np.abs(k[:512]).mean()
    g = I.WORKLOADS["grid2d"].with_(C=2, H=32, W=32)
    K = I.k_row(g, 0, 1).reshape(32, 32)
    assert np.abs(K[:4, :4]).mean() > np.abs(K[-4:, -4:]).mean() * 0.5
    dna = I.WORKLOADS["dna_1m"].with_(L=1024)
    r0 = I.u_row(dna, 0, 0)
    assert len(np.unique(r0)) <= 4          # one value per base
    tok = I._tokens(dna)
    emb = I._embedding(dna)
    assert np.array_equal(I.u_row(dna, 0, 300), emb[tok, 300])
