"""Pins of the implicit-filter oracle (oracle/filter_gen.py): hand-derived
values, closed forms and the channel rearrangement; each would fail for a
plausible mistake (wrong band frequency, time term, activation frequency,
missing layer, wrong decay sign or channel order)."""
import numpy as np

from oracle import filter_gen as F


def test_positional_embedding_hand_values():
    z, t = F.positional_embedding(4, 5)          # 2 bands
    assert z.shape == (4, 5)
    np.testing.assert_allclose(t, [0.0, 1 / 3, 2 / 3, 1.0])
    # l = 1 of L = 4: band 1 at a quarter turn, band 2 at a half turn
    np.testing.assert_allclose(z[1], [1 / 3, 0.0, -1.0, 1.0, 0.0], atol=1e-15)
    np.testing.assert_allclose(z[0], [0.0, 1.0, 1.0, 0.0, 0.0])


def test_constant_mlp_gives_exponential_decay():
    """Zero weights, biases b: every hidden unit is sin(w b) (then sin(w sin(w b)))
    and the output a fixed mix; the filter is that constant times exp(-alpha t)."""
    L, E, Wd, dm = 9, 3, 4, 3
    rng = np.random.default_rng(0)
    b_in = rng.standard_normal(Wd); b1 = rng.standard_normal(Wd)
    w = np.full(Wd, 1.5)
    W_out = rng.standard_normal((dm, Wd))
    alpha = np.array([0.0, 0.5, 3.0])
    k = F.hyena_filter(L, E, np.zeros((Wd, E)), b_in, [(np.zeros((Wd, Wd)), b1)], W_out, w, alpha)
    h1 = np.sin(1.5 * b1)                         # second layer input is constant, weights zero
    const = W_out @ h1
    t = np.arange(L) / (L - 1)
    np.testing.assert_allclose(k, const[None, :] * np.exp(-alpha[None, :] * t[:, None]), rtol=1e-14)
    assert np.allclose(k[:, 0], k[0, 0])          # alpha = 0: no decay


def test_single_layer_hand_example():
    """emb_dim 3, width 1, d_model 1, L 2: z = [[0, 1, 0], [1, -1, 0]];
    h = sin(w (z . W + b)) * W_out; k = h exp(-alpha t)."""
    W_in = np.array([[0.5, 0.25, 2.0]]); b_in = np.array([0.1]); w = np.array([2.0])
    W_out = np.array([[3.0]]); alpha = np.array([0.7])
    k = F.hyena_filter(2, 3, W_in, b_in, [], W_out, w, alpha)
    want0 = 3.0 * np.sin(2.0 * (0.25 + 0.1))
    want1 = 3.0 * np.sin(2.0 * (0.5 - 0.25 + 0.1)) * np.exp(-0.7)
    np.testing.assert_allclose(k[:, 0], [want0, want1], rtol=1e-14)


def test_operator_filter_rearrangement():
    L, order, C = 5, 3, 4
    k = np.arange(L * (order - 1) * C, dtype=np.float64).reshape(L, (order - 1) * C)
    ko = F.operator_filters(k, order)
    assert ko.shape == (order - 1, C, L)
    for o in range(order - 1):
        for d in range(C):
            np.testing.assert_array_equal(ko[o, d], k[:, o * C + d])
