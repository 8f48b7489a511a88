"""float64 oracle of the implicit long filter (TEST INFRASTRUCTURE ONLY: the
product path never imports it).

[P4] "HyenaDNA operator walk-through" (adg.csdn.net), section 二.2 核心卷积核
HyenaFilter介绍: the long filters are not stored but generated,
``filter(L) = modulation(t, implicit_filter(pos_emb(L)))``:

* ``pos_emb``: per time step a linear time term plus sin/cos features;
  ``(emb_dim - 1) // 2`` is the number of bands (emb_dim odd, >= 3).
* ``implicit_filter``: Linear(emb_dim, width) -> Sin, then ``num_inner``
  times Linear(width, width) -> Sin, then Linear(width, d_model) without bias.
  Sin is a sine activation whose frequency ``w`` sets how fast the generated
  filter oscillates.
* ``modulation`` (ExponentialModulation): the generated filter times an
  exponential decay in time with per-channel learnable rates.
* The operator takes the d_model = (order - 1) C output channels rearranged
  ``'l (o d) -> o d l'``: step o's filters are channels o C .. o C + C - 1.

Readings where the page prints no formula (plainest forms consistent with
the text):
* time term ``t[l] = l / (L - 1)`` (0 .. 1; 0 for L = 1); band b = 1..nb has
  angle ``2 pi b l / L``; feature order ``[t, cos_1..cos_nb, sin_1..sin_nb]``;
* Sin(x) = sin(w * x) elementwise with a per-feature frequency vector w
  (the activation is built as Sin(dim=width, w=w));
* modulation: ``h[l, c] * exp(-alpha[c] * t[l])``, alpha >= 0 per channel.
Weights are plain arrays (synthetic in tests); Linear(x) = x @ W.T + b.
"""
from __future__ import annotations

import numpy as np


def positional_embedding(L: int, emb_dim: int):
    """z [L, emb_dim] and the time term t [L]."""
    if emb_dim < 3 or emb_dim % 2 == 0:
        raise ValueError("emb_dim must be odd and >= 3 (time, cosine and sine bands)")
    nb = (emb_dim - 1) // 2
    ell = np.arange(L, dtype=np.float64)
    t = ell / (L - 1) if L > 1 else np.zeros(1)
    ang = 2.0 * np.pi * np.arange(1, nb + 1, dtype=np.float64)[None, :] * ell[:, None] / L
    z = np.concatenate([t[:, None], np.cos(ang), np.sin(ang)], axis=1)
    return z, t


def sin_act(x, w):
    """Sine activation with per-feature frequencies w (broadcast over rows)."""
    return np.sin(np.asarray(w, dtype=np.float64)[None, :] * x)


def implicit_filter(z, W_in, b_in, inner, W_out, w):
    """MLP of the implicit filter: z [L, emb_dim] -> h [L, d_model].
    inner: list of (W, b) for the Linear(width, width) layers."""
    h = sin_act(z @ np.asarray(W_in, np.float64).T + np.asarray(b_in, np.float64)[None, :], w)
    for W, b in inner:
        h = sin_act(h @ np.asarray(W, np.float64).T + np.asarray(b, np.float64)[None, :], w)
    return h @ np.asarray(W_out, np.float64).T


def exponential_modulation(t, h, alpha):
    """h [L, d_model] times exp(-alpha[c] t[l])."""
    return h * np.exp(-np.asarray(alpha, np.float64)[None, :] * np.asarray(t, np.float64)[:, None])


def hyena_filter(L: int, emb_dim: int, W_in, b_in, inner, W_out, w, alpha):
    """k [L, d_model] = modulation(t, implicit_filter(pos_emb(L)))."""
    z, t = positional_embedding(L, emb_dim)
    return exponential_modulation(t, implicit_filter(z, W_in, b_in, inner, W_out, w), alpha)


def operator_filters(k, order: int):
    """k [L, (order-1) C] -> [order-1, C, L] ('l (o d) -> o d l')."""
    L, dm = k.shape
    if dm % (order - 1):
        raise ValueError("d_model must be (order - 1) * C")
    C = dm // (order - 1)
    return np.ascontiguousarray(k.T.reshape(order - 1, C, L))
